// Host-side argument rules shared by the C-ABI entry points (api.cu and the allocation-free
// alltoallv in a2a_static.cu), so that calls documented as taking the same arguments check
// them the same way.
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/cc.h"

namespace cc {

inline bool valid_ranks(int nranks) { return nranks >= 1 && nranks <= CC_MAX_RANKS; }

inline bool all_nonnull(const void* const* p, int n) {
  if (!p) return false;
  for (int i = 0; i < n; ++i)
    if (!p[i]) return false;
  return true;
}

// Shapes the alltoallv kernels take: topk in [1, 8], at most 1024 experts in total, and a
// row index (token * topk + k) that fits an int32.
inline bool a2a_shape_ok(int nranks, int tokens, int topk, int experts_per_rank) {
  return valid_ranks(nranks) && tokens >= 0 && topk >= 1 && topk <= 8 && experts_per_rank >= 1 &&
         (long long)nranks * experts_per_rank <= 1024 && (long long)tokens * topk < (1ll << 31);
}

// Every argument of cc_alltoallv except the workspace: the shape, non-null send / recv /
// expert-id arrays, a row size that is a positive multiple of 16 bytes, a direction of 0
// or 1, and 16-byte aligned send and receive buffers.
inline bool a2a_args_ok(const void* const* send, void* const* recv, int nranks, size_t row_bytes,
                        const int32_t* const* expert_ids, int tokens, int topk, int experts_per_rank,
                        int direction) {
  if (!a2a_shape_ok(nranks, tokens, topk, experts_per_rank)) return false;
  if (!all_nonnull(send, nranks) || !all_nonnull((const void* const*)recv, nranks) ||
      !all_nonnull((const void* const*)expert_ids, nranks))
    return false;
  if (row_bytes == 0 || row_bytes % 16 != 0 || (direction != 0 && direction != 1)) return false;
  for (int r = 0; r < nranks; ++r)
    if ((reinterpret_cast<uintptr_t>(send[r]) | reinterpret_cast<uintptr_t>(recv[r])) & 15) return false;
  return true;
}

}  // namespace cc
