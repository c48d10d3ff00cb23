// MoE expert parallelism: top-k routing and the alltoallv dispatch / combine
// (lecture 09 §6.4; AllToAll semantics §3.8 and experiment 4 §7.4).
//
// Dispatch layout: rank d's receive buffer is the concatenation over source ranks
// s = 0..N-1 of s's rows for d, each block ordered by (local expert, token, slot).
// The position of row i = t * topk + k of source s routed to global expert e is
//   base[s][e] + tile_off[s][tile(i)][e] + rank_in_tile(i)
// where base[s][e] = rows of earlier sources for the same destination + rows of s for
// earlier local experts of that destination, tile_off is the exclusive prefix over
// tiles of 256 rows, and rank_in_tile counts earlier rows of the tile with the same
// expert (warp match + per-warp counts). All of it is integer and deterministic.
//
// Kernels: K1 tile counts and per-row ranks, K2 tile prefix per (s, e), K3 bases and
// receive counts, K4 the row copy (one warp per token: the token row is read once and
// written topk times; combine reads topk rows and writes topk rows).
#include <algorithm>

#include "cc_device.cuh"
#include "cc_launch.h"

namespace cc {

constexpr int kTileRows = 256;  // rows per K1 tile: 8 warps
constexpr int kMaxTopk = 8;

struct A2AWorkspace {
  // byte offsets inside the caller's workspace; the receive counts sit first, at a
  // fixed place, so that they can be read back without knowing the other sizes
  size_t recv_count, tile_cnt, row_rank, totals, base, total;
};

static A2AWorkspace a2a_layout(int nranks, int tokens, int topk, int experts_per_rank) {
  const size_t E = (size_t)nranks * experts_per_rank;
  const size_t rows = (size_t)tokens * topk;
  const size_t ntiles = (rows + kTileRows - 1) / kTileRows;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  A2AWorkspace w;
  w.recv_count = 0;
  w.tile_cnt = up(sizeof(int) * kMaxRanks);
  w.row_rank = up(w.tile_cnt + sizeof(int) * nranks * ntiles * E);
  w.totals = up(w.row_rank + sizeof(int) * nranks * rows);
  w.base = up(w.totals + sizeof(int) * nranks * E);
  w.total = up(w.base + sizeof(int) * nranks * E);
  return w;
}

size_t a2a_workspace_bytes(int nranks, int tokens, int topk, int experts_per_rank) {
  return a2a_layout(nranks, tokens, topk, experts_per_rank).total;
}

struct IdPtrs {
  const int32_t* ids[kMaxRanks];
};

// ---- top-k routing ---------------------------------------------------------------------------------

struct RouteParams {
  const float* logits[kMaxRanks];
  int32_t* ids[kMaxRanks];
  int tokens, experts, topk;
};

// Eight lanes per token. Lane g of a token's group scans the 4-expert chunks g, g+8, ... in
// expert order with a running, descending top-k list in registers (a later expert enters
// only with a strictly larger value, so equal values keep the lower id first); the eight
// lists are then merged pairwise with shuffles (three butterfly steps), ordering by larger
// value, then lower id. All lanes end with the token's top-k; lane 0 writes it.
constexpr int kRouteLanes = 8;

__device__ __forceinline__ bool route_better(float a, int ia, float b, int ib) {
  return ib < 0 || (ia >= 0 && (a > b || (a == b && ia < ib)));
}

template <int K>
__global__ void __launch_bounds__(256) route_topk_kernel(const __grid_constant__ RouteParams P) {
  const int s = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int g = lane % kRouteLanes;
  const int t = (blockIdx.x * blockDim.x + threadIdx.x) / kRouteLanes;
  const bool live = t < P.tokens;  // dead groups still take part in the shuffles
  float val[K];
  int idx[K];
#pragma unroll
  for (int j = 0; j < K; ++j) { val[j] = -INFINITY; idx[j] = -1; }
  auto insert = [&](float v, int e) {
    if (idx[K - 1] >= 0 && !(v > val[K - 1])) return;
    int pos = K - 1;
#pragma unroll
    for (int j = K - 1; j >= 1; --j)
      if (pos == j && (idx[j - 1] < 0 || v > val[j - 1])) {
        val[j] = val[j - 1];
        idx[j] = idx[j - 1];
        pos = j - 1;
      }
#pragma unroll
    for (int j = 0; j < K; ++j)
      if (j == pos) { val[j] = v; idx[j] = e; }
  };
  if (live) {
    const float* row = P.logits[s] + (size_t)t * P.experts;
    const bool vec = (P.experts % 4 == 0) && ((reinterpret_cast<uintptr_t>(P.logits[s]) & 15) == 0);
    if (vec) {
      for (int e = 4 * g; e < P.experts; e += 4 * kRouteLanes) {
        const float4 v = __ldcs(reinterpret_cast<const float4*>(row + e));
        insert(v.x, e);
        insert(v.y, e + 1);
        insert(v.z, e + 2);
        insert(v.w, e + 3);
      }
    } else {
      for (int e = g; e < P.experts; e += kRouteLanes) insert(__ldcs(row + e), e);
    }
  }
#pragma unroll
  for (int off = kRouteLanes / 2; off >= 1; off >>= 1) {
    float ov[K];
    int oi[K];
#pragma unroll
    for (int j = 0; j < K; ++j) {
      ov[j] = __shfl_xor_sync(0xffffffffu, val[j], off);
      oi[j] = __shfl_xor_sync(0xffffffffu, idx[j], off);
    }
    // merge the two descending lists, keep the first K
    float mv[K];
    int mi[K];
    int a = 0, b = 0;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      float va = -INFINITY, vb = -INFINITY;
      int ia = -1, ib = -1;
#pragma unroll
      for (int x = 0; x < K; ++x) {
        if (x == a) { va = val[x]; ia = idx[x]; }
        if (x == b) { vb = ov[x]; ib = oi[x]; }
      }
      if (route_better(va, ia, vb, ib)) { mv[j] = va; mi[j] = ia; ++a; }
      else { mv[j] = vb; mi[j] = ib; ++b; }
    }
#pragma unroll
    for (int j = 0; j < K; ++j) { val[j] = mv[j]; idx[j] = mi[j]; }
  }
  if (live && g == 0) {
    int32_t* out = P.ids[s] + (size_t)t * K;
#pragma unroll
    for (int j = 0; j < K; ++j) out[j] = idx[j];
  }
}

cudaError_t launch_route_topk(const float* const* logits, int32_t* const* ids, int nranks, int tokens,
                              int experts_total, int topk, cudaStream_t stream) {
  RouteParams P{};
  for (int r = 0; r < nranks; ++r) {
    P.logits[r] = logits[r];
    P.ids[r] = ids[r];
  }
  P.tokens = tokens;
  P.experts = experts_total;
  P.topk = topk;
  const long long threads = (long long)tokens * kRouteLanes;
  dim3 grid((unsigned)((threads + 255) / 256), nranks);
  switch (topk) {
    case 1: route_topk_kernel<1><<<grid, 256, 0, stream>>>(P); break;
    case 2: route_topk_kernel<2><<<grid, 256, 0, stream>>>(P); break;
    case 3: route_topk_kernel<3><<<grid, 256, 0, stream>>>(P); break;
    case 4: route_topk_kernel<4><<<grid, 256, 0, stream>>>(P); break;
    case 5: route_topk_kernel<5><<<grid, 256, 0, stream>>>(P); break;
    case 6: route_topk_kernel<6><<<grid, 256, 0, stream>>>(P); break;
    case 7: route_topk_kernel<7><<<grid, 256, 0, stream>>>(P); break;
    default: route_topk_kernel<8><<<grid, 256, 0, stream>>>(P); break;
  }
  return cudaGetLastError();
}

// ---- K1: per-tile expert counts and per-row rank within the tile -------------------------------------

__global__ void __launch_bounds__(kTileRows) a2a_count_kernel(const __grid_constant__ IdPtrs I, int rows, int E,
                                                              int* __restrict__ tile_cnt, int* __restrict__ row_rank) {
  extern __shared__ int warp_cnt[];  // [8][E]
  const int s = blockIdx.y, tile = blockIdx.x, ntiles = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 8 * E; i += blockDim.x) warp_cnt[i] = 0;
  __syncthreads();
  const int row = tile * kTileRows + threadIdx.x;
  int e = row < rows ? I.ids[s][row] : -1;
  const bool valid = e >= 0 && e < E;  // rows with an out-of-range expert id are not sent
  if (!valid) e = -1 - lane;           // invalid lanes match nobody
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const unsigned lt = (1u << lane) - 1;
  const int rank_w = __popc(peers & lt);
  if (valid && rank_w == 0) warp_cnt[warp * E + e] = __popc(peers);
  __syncthreads();
  // exclusive prefix over the 8 warps, per expert; tile total to global memory
  for (int x = threadIdx.x; x < E; x += blockDim.x) {
    int run = 0;
    for (int w = 0; w < 8; ++w) {
      const int c = warp_cnt[w * E + x];
      warp_cnt[w * E + x] = run;
      run += c;
    }
    tile_cnt[((size_t)s * ntiles + tile) * E + x] = run;
  }
  __syncthreads();
  if (valid) row_rank[(size_t)s * rows + row] = warp_cnt[warp * E + e] + rank_w;
}

// ---- K2: exclusive prefix over tiles, per (source, expert); one warp each -----------------------------

__global__ void a2a_tile_scan_kernel(int ntiles, int E, int* __restrict__ tile_cnt, int* __restrict__ totals) {
  const int s = blockIdx.y, e = blockIdx.x, lane = threadIdx.x;
  int carry = 0;
  for (int t0 = 0; t0 < ntiles; t0 += 32) {
    const int t = t0 + lane;
    int* p = tile_cnt + ((size_t)s * ntiles + t) * E + e;
    const int v = t < ntiles ? *p : 0;
    int inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += o;
    }
    if (t < ntiles) *p = carry + inc - v;
    carry += __shfl_sync(0xffffffffu, inc, 31);
  }
  if (lane == 0) totals[(size_t)s * E + e] = carry;
}

// ---- K3: bases per (source, expert) and receive counts per destination (one CTA) -------------------------

__global__ void __launch_bounds__(1024) a2a_base_kernel(int nranks, int epr, const int* __restrict__ tot,
                                                        int* __restrict__ base, int* __restrict__ recv_count) {
  __shared__ int cnt[kMaxRanks * kMaxRanks];  // rows s -> d
  const int E = nranks * epr;
  for (int i = threadIdx.x; i < nranks * nranks; i += blockDim.x) {
    const int s = i / nranks, d = i % nranks;
    int c = 0;
    for (int l = 0; l < epr; ++l) c += tot[s * E + d * epr + l];
    cnt[i] = c;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nranks * E; i += blockDim.x) {
    const int s = i / E, e = i % E, d = e / epr;
    int off = 0;
    for (int sp = 0; sp < s; ++sp) off += cnt[sp * nranks + d];
    for (int l = d * epr; l < e; ++l) off += tot[s * E + l];
    base[i] = off;
  }
  for (int d = threadIdx.x; d < nranks; d += blockDim.x) {
    int c = 0;
    for (int s = 0; s < nranks; ++s) c += cnt[s * nranks + d];
    recv_count[d] = c;
  }
}

// ---- K4: row copies ----------------------------------------------------------------------------------

struct A2ACopyParams {
  const char* send[kMaxRanks];
  char* recv[kMaxRanks];
  const int32_t* ids[kMaxRanks];
  const int* tile_off;   // [N][ntiles][E]
  const int* row_rank;   // [N][rows]
  const int* base;       // [N][E]
  uint64_t row_bytes;
  uint64_t capacity;
  int tokens, topk, epr, E, ntiles, direction;
};

__global__ void __launch_bounds__(256) a2a_copy_kernel(const __grid_constant__ A2ACopyParams P) {
  const int lane = threadIdx.x & 31;
  const int s = blockIdx.y;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= P.tokens) return;
  const int rows = P.tokens * P.topk;
  char* ptr[kMaxTopk];
  bool ok[kMaxTopk];
  for (int k = 0; k < P.topk; ++k) {
    const int i = t * P.topk + k;
    const int e = P.ids[s][i];
    if (e < 0 || e >= P.E) { ok[k] = false; ptr[k] = nullptr; continue; }
    const int d = e / P.epr;
    const uint64_t pos = (uint64_t)P.base[s * P.E + e] +
                         P.tile_off[((size_t)s * P.ntiles + i / kTileRows) * P.E + e] +
                         P.row_rank[(size_t)s * rows + i];
    ok[k] = pos < P.capacity;
    ptr[k] = (P.direction == 0 ? P.recv[d] : const_cast<char*>(P.send[d])) + pos * P.row_bytes;
  }
  // 16 loads per lane in flight before the stores that consume them (a whole 8 KiB row per
  // warp; measured faster than 8 or 32)
  constexpr int B = 16;
  const uint64_t nvec = P.row_bytes / 16;
  if (P.direction == 0) {
    const uint4* src = reinterpret_cast<const uint4*>(P.send[s] + (uint64_t)t * P.row_bytes);
    for (uint64_t v0 = lane; v0 < nvec; v0 += 32 * B) {
      uint4 x[B];
#pragma unroll
      for (int b = 0; b < B; ++b)
        if (v0 + 32 * b < nvec) x[b] = __ldcs(src + v0 + 32 * b);
      for (int k = 0; k < P.topk; ++k) {
        if (!ok[k]) continue;
        uint4* d = reinterpret_cast<uint4*>(ptr[k]);
#pragma unroll
        for (int b = 0; b < B; ++b)
          if (v0 + 32 * b < nvec) __stcs(d + v0 + 32 * b, x[b]);
      }
    }
  } else {
    char* dst = P.recv[s] + (uint64_t)t * P.topk * P.row_bytes;
    for (int k = 0; k < P.topk; ++k) {
      if (!ok[k]) continue;
      const uint4* src = reinterpret_cast<const uint4*>(ptr[k]);
      uint4* d = reinterpret_cast<uint4*>(dst + k * P.row_bytes);
      for (uint64_t v0 = lane; v0 < nvec; v0 += 32 * B) {
        uint4 x[B];
#pragma unroll
        for (int b = 0; b < B; ++b)
          if (v0 + 32 * b < nvec) x[b] = __ldcs(src + v0 + 32 * b);
#pragma unroll
        for (int b = 0; b < B; ++b)
          if (v0 + 32 * b < nvec) __stcs(d + v0 + 32 * b, x[b]);
      }
    }
  }
}

cudaError_t launch_alltoallv(const void* const* send, void* const* recv, int nranks, size_t row_bytes,
                             const int32_t* const* ids, int tokens, int topk, int experts_per_rank,
                             size_t capacity_rows, int direction, void* workspace, cudaStream_t stream) {
  const int E = nranks * experts_per_rank;
  const int rows = tokens * topk;
  const int ntiles = (rows + kTileRows - 1) / kTileRows;
  const A2AWorkspace w = a2a_layout(nranks, tokens, topk, experts_per_rank);
  char* ws = static_cast<char*>(workspace);
  int* tile_cnt = reinterpret_cast<int*>(ws + w.tile_cnt);
  int* row_rank = reinterpret_cast<int*>(ws + w.row_rank);
  int* totals = reinterpret_cast<int*>(ws + w.totals);
  int* base = reinterpret_cast<int*>(ws + w.base);
  int* recv_count = reinterpret_cast<int*>(ws + w.recv_count);
  IdPtrs I{};
  for (int r = 0; r < nranks; ++r) I.ids[r] = ids[r];
  if (rows > 0) {
    a2a_count_kernel<<<dim3(ntiles, nranks), kTileRows, sizeof(int) * 8 * E, stream>>>(I, rows, E, tile_cnt, row_rank);
    a2a_tile_scan_kernel<<<dim3(E, nranks), 32, 0, stream>>>(ntiles, E, tile_cnt, totals);
  } else {
    // no rows: the bases read zero totals (the only write to this scratch before K3)
    const cudaError_t e = cudaMemsetAsync(totals, 0, sizeof(int) * nranks * E, stream);
    if (e != cudaSuccess) return e;
  }
  a2a_base_kernel<<<1, 1024, 0, stream>>>(nranks, experts_per_rank, totals, base, recv_count);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess || rows == 0) return err;
  A2ACopyParams P{};
  for (int r = 0; r < nranks; ++r) {
    P.send[r] = static_cast<const char*>(send[r]);
    P.recv[r] = static_cast<char*>(recv[r]);
    P.ids[r] = ids[r];
  }
  P.tile_off = tile_cnt;
  P.row_rank = row_rank;
  P.base = base;
  P.row_bytes = row_bytes;
  P.capacity = capacity_rows;
  P.tokens = tokens;
  P.topk = topk;
  P.epr = experts_per_rank;
  P.E = E;
  P.ntiles = ntiles;
  P.direction = direction;
  a2a_copy_kernel<<<dim3((tokens + 7) / 8, nranks), 256, 0, stream>>>(P);
  return cudaGetLastError();
}

cudaError_t copy_recv_counts(const void* workspace, int nranks, int32_t* out, cudaStream_t stream) {
  return cudaMemcpyAsync(out, static_cast<const char*>(workspace), sizeof(int32_t) * nranks, cudaMemcpyDefault,
                         stream);
}

}  // namespace cc
