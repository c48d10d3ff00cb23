// Host-side launch interfaces between the C-ABI layer (api.cu) and the kernel files.
// Arguments are validated by the caller; these only build parameter blocks and launch.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/cc.h"

namespace cc {

// Reduction family: allreduce, reduce-scatter, reduce-to-root.
enum ReduceMode { kAllReduce = 0, kReduceScatter = 1, kReduceRoot = 2 };
enum FoldKind { kFoldRing = 0, kFoldTree = 1, kFoldBinomial = 2, kFoldHier = 3, kFoldMultiRing = 4 };

// `root` is the root rank for kFoldBinomial, the ranks per node for kFoldHier and the number
// of rings for kFoldMultiRing; only the
// elements [lo, hi) of the count are folded and written (the whole buffer by default).
cudaError_t launch_reduce(const void* const* send, void* const* dst, int ndst, int nranks,
                          size_t count, cc_dtype in_t, cc_op op, FoldKind fold, ReduceMode mode,
                          int root, float scale, cudaStream_t stream, size_t lo = 0,
                          size_t hi = ~(size_t)0);

// Fused DDP bucket allreduce over a tensor group (tables fit one launch).
struct BucketTensorDesc {
  uint64_t numel;
  uint64_t bucket_off;    // element offset of the tensor inside its bucket
  uint64_t bucket_count;  // elements in the tensor's bucket
};
int bucket_group_limit(int nranks);        // tensors one launch can take
int bucket_small_group_limit(int nranks);  // tensors a launch with a small (< 4 KB) parameter block takes
cudaError_t launch_bucket_allreduce(const void* const* grads, void* const* out, int nranks,
                                    int ntensors_total, const int32_t* ids, int nids,
                                    const BucketTensorDesc* desc, FoldKind fold, float scale,
                                    cudaStream_t stream);

// Copies with fan-out: entry k copies numel[k] elements from src[k] either to every
// dst_base[r] + dst_off[k] (fanout = true, r != skip) or to dst[k] + dst_off[k]. `plain`
// keeps to ordinary loads and stores (no bulk copies), for destinations in peer memory.
struct CopyEntry {
  const void* src;
  void* dst;          // fanout == false
  uint64_t numel;
  uint64_t dst_off;   // elements
};
cudaError_t launch_copy(const CopyEntry* entries, int nentries, void* const* dst_base, int ndst,
                        bool fanout, int skip, size_t elem_bytes, cudaStream_t stream, bool plain = false);

// Device status word of the bounded waits (CC_OK or CC_ERR_TIMEOUT), read with a
// stream synchronisation; `reset` clears it afterwards.
cudaError_t read_async_status(int* out, bool reset, cudaStream_t stream);
cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, cudaStream_t stream);
int* async_status_word();  // device address of that status word (current device), or null

// Stepped (schedule-faithful) allreduce: one cooperative launch, a grid barrier between the
// schedule's dependent steps; `barrier` is 4 bytes of caller device memory.
cudaError_t launch_stepped_allreduce(const void* const* send, void* const* recv, int nranks, size_t count,
                                     cc_dtype in_t, cc_op op, FoldKind fold, float scale, unsigned* barrier,
                                     cudaStream_t s);

// MoE
cudaError_t launch_route_topk(const float* const* logits, int32_t* const* ids, int nranks, int tokens,
                              int experts_total, int topk, cudaStream_t stream);
size_t a2a_workspace_bytes(int nranks, int tokens, int topk, int experts_per_rank);
// Which parts of an alltoallv to run: the routing tables (the plan), the row copy, or both.
enum A2AParts { kA2ATables = 1, kA2ACopy = 2, kA2ABoth = 3 };
cudaError_t launch_alltoallv(const void* const* send, void* const* recv, int nranks, size_t row_bytes,
                             const int32_t* const* ids, int tokens, int topk, int experts_per_rank,
                             size_t capacity_rows, int direction, void* workspace, cudaStream_t stream,
                             A2AParts parts = kA2ABoth);
cudaError_t copy_recv_counts(const void* workspace, int nranks, int32_t* out, cudaStream_t stream);

// Device properties, cached per device.
int sm_count();

}  // namespace cc
