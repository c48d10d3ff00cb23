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
// Kernels: the routing tables in one launch (tile counts and per-row ranks in every CTA;
// the last CTA of each source to finish builds that source's tile prefix per expert, and the
// last of those the bases and receive counts), then the row copy (one warp per token: the
// token row is read once and written topk times; combine reads topk rows and writes topk
// rows). "Last to finish" is an atomic ticket on counters the call clears first.
// cc_alltoallv_plan launches the first alone, cc_alltoallv_run the second alone.
#include <algorithm>

#include "cc_device.cuh"
#include "cc_launch.h"

namespace cc {

constexpr int kTileRows = 256;  // rows per K1 tile: 8 warps
constexpr int kMaxTopk = 8;

struct A2AWorkspace {
  // byte offsets inside the caller's workspace; the receive counts sit first, at a
  // fixed place, so that they can be read back without knowing the other sizes; then the
  // finish tickets (one per source and one for all)
  size_t recv_count, done, tile_cnt, row_rank, totals, base, total;
};

static A2AWorkspace a2a_layout(int nranks, int tokens, int topk, int experts_per_rank) {
  const size_t E = (size_t)nranks * experts_per_rank;
  const size_t rows = (size_t)tokens * topk;
  const size_t ntiles = (rows + kTileRows - 1) / kTileRows;
  auto up = [](size_t x) { return (x + 255) / 256 * 256; };
  A2AWorkspace w;
  w.recv_count = 0;
  w.done = up(sizeof(int) * kMaxRanks);
  w.tile_cnt = w.done + up(sizeof(unsigned) * (kMaxRanks + 1));
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

// Four lanes per token. Lane g of a token's group scans the 4-expert chunks g, g+4, ... in
// expert order with a running, descending top-k list in registers (a later expert enters
// only with a strictly larger value, so equal values keep the lower id first); the four
// lists are then merged pairwise with shuffles (two butterfly steps), ordering by larger
// value, then lower id. All lanes end with the token's top-k; lane 0 writes it. (Measured on
// 8 x 8192 tokens x 64 experts: 8 lanes 11.3-12.1 us, 4 lanes 9.7 us, 2 lanes 10.2 us.)
constexpr int kRouteLanes = 4;
constexpr int kRoutePre = 4;  // chunks per lane loaded before the first insert

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
      // kRoutePre chunks per lane loaded before the first insert (one DRAM round trip for up to
      // 4 * 8 * kRoutePre experts), then inserted in the same expert order as one at a time
      for (int e0 = 4 * g; e0 < P.experts; e0 += 4 * kRouteLanes * kRoutePre) {
        float4 v[kRoutePre];
#pragma unroll
        for (int q = 0; q < kRoutePre; ++q) {
          const int e = e0 + 4 * kRouteLanes * q;
          if (e < P.experts) v[q] = __ldcs(reinterpret_cast<const float4*>(row + e));
        }
#pragma unroll
        for (int q = 0; q < kRoutePre; ++q) {
          const int e = e0 + 4 * kRouteLanes * q;
          if (e >= P.experts) break;
          insert(v[q].x, e);
          insert(v[q].y, e + 1);
          insert(v[q].z, e + 2);
          insert(v[q].w, e + 3);
        }
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

// ---- routing tables -----------------------------------------------------------------------------------
// Every CTA counts one tile of 256 rows of one source: per expert the rows of the tile, and
// each row's rank among the tile's rows of its expert (warp match + per-warp prefix).

constexpr int kScanSplit = 4;  // threads per expert in the per-source tile prefix

// Bases and receive counts from the per-(source, expert) totals, by one CTA. `sm` holds
// sm_ints ints: the rows s -> d (nranks^2 <= 4096 ints) first, then, when they fit, the totals
// staged with one coalesced pass (nranks * E ints: up to 64 x 1024); otherwise the totals are
// read from global memory.
__device__ __forceinline__ void bases_and_counts(int nranks, int epr, const int* tot_g, int* base, int* recv_count,
                                                 int* sm, int sm_ints) {
  const int E = nranks * epr;
  int* cnt = sm;  // rows s -> d
  int* tot_s = sm + nranks * nranks;
  const bool staged = nranks * nranks + nranks * E <= sm_ints;
  const int* tot = staged ? tot_s : tot_g;
  if (staged)
    for (int i = threadIdx.x; i < nranks * E; i += blockDim.x) tot_s[i] = __ldcg(tot_g + i);
  __syncthreads();
  for (int i = threadIdx.x; i < nranks * nranks; i += blockDim.x) {
    const int s = i / nranks, d = i % nranks;
    int c = 0;
    for (int l = 0; l < epr; ++l) c += staged ? tot[s * E + d * epr + l] : __ldcg(tot + s * E + d * epr + l);
    cnt[i] = c;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nranks * E; i += blockDim.x) {
    const int s = i / E, e = i % E, d = e / epr;
    int off = 0;
    for (int sp = 0; sp < s; ++sp) off += cnt[sp * nranks + d];
    for (int l = d * epr; l < e; ++l) off += staged ? tot[s * E + l] : __ldcg(tot + s * E + l);
    base[i] = off;
  }
  for (int d = threadIdx.x; d < nranks; d += blockDim.x) {
    int c = 0;
    for (int s = 0; s < nranks; ++s) c += cnt[s * nranks + d];
    recv_count[d] = c;
  }
}

// Dynamic shared memory of the table kernel, in ints (with its static words, within the 48 KiB
// a launch gets without opting in): a tile's [8][E] warp counts, the source's [tiles][E] counts
// when they fit kScanSmemInts, and the bases' rows s -> d with the totals when they fit.
constexpr int kTablesSmemInts = 12000;
constexpr int kScanSmemInts = 10240;  // a source's [tiles][experts] counts scanned in shared memory up to this

__global__ void __launch_bounds__(kTileRows) a2a_tables_kernel(const __grid_constant__ IdPtrs I, int rows, int nranks,
                                                               int epr, int* __restrict__ tile_cnt,
                                                               int* __restrict__ row_rank, int* __restrict__ totals,
                                                               int* __restrict__ base, int* __restrict__ recv_count,
                                                               unsigned* __restrict__ done, int sm_ints) {
  extern __shared__ int warp_cnt[];  // [8][E]; reused by the last CTAs (scan, then bases)
  __shared__ int s_last;
  // the copy kernel (a programmatic dependent) may launch now: it waits for this grid to
  // complete before it reads any table
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int E = nranks * epr;
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

  // the last tile of source s to finish turns the tile counts into exclusive prefixes over
  // tiles, per expert, and the source's totals. Thread 0 publishes the CTA's writes (the
  // barrier orders the other threads' writes before its fence) and takes the ticket; the last
  // CTA's thread 0 fences again before the barrier that lets its threads read the others' counts.
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(&done[1 + s], 1u) == (unsigned)ntiles - 1;
    __threadfence();
  }
  __syncthreads();
  if (!s_last) return;
  const size_t blk = (size_t)ntiles * E;
  int* src_cnt = tile_cnt + (size_t)s * blk;
  if (blk <= (size_t)kScanSmemInts) {
    // the source's counts staged in shared memory with one coalesced pass; kScanSplit threads
    // per expert each sum a run of tiles, an exclusive prefix over the runs (shuffles), then
    // each thread turns its run into exclusive prefixes in place. The totals are published
    // (and the next ticket taken) before the prefixes go back to global memory: only the copy
    // kernel reads those, after this grid has completed.
    for (size_t i = threadIdx.x; i < blk; i += blockDim.x) warp_cnt[i] = __ldcg(src_cnt + i);
    __syncthreads();
    const int q = threadIdx.x % kScanSplit;
    const int per = (ntiles + kScanSplit - 1) / kScanSplit;
    const int t0 = q * per, t1 = min(ntiles, t0 + per);
    for (int e0 = 0; e0 < E; e0 += kTileRows / kScanSplit) {
      const int x = e0 + threadIdx.x / kScanSplit;
      const bool live = x < E;
      int part = 0;
      for (int t = t0; live && t < t1; ++t) part += warp_cnt[t * E + x];
      int inc = part;
#pragma unroll
      for (int off = 1; off < kScanSplit; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, inc, off, kScanSplit);
        if (q >= off) inc += o;
      }
      int run = inc - part;
      for (int t = t0; live && t < t1; ++t) {
        const int v = warp_cnt[t * E + x];
        warp_cnt[t * E + x] = run;
        run += v;
      }
      if (live && q == kScanSplit - 1) totals[(size_t)s * E + x] = run;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      s_last = atomicAdd(&done[0], 1u) == (unsigned)nranks - 1;
      __threadfence();
    }
    __syncthreads();
    for (size_t i = threadIdx.x; i < blk; i += blockDim.x) src_cnt[i] = warp_cnt[i];
    if (!s_last) return;
    __syncthreads();  // every thread is done with warp_cnt before the bases reuse it
    bases_and_counts(nranks, epr, totals, base, recv_count, warp_cnt, sm_ints);
    return;
  } else {
    const int q = threadIdx.x % kScanSplit;
    const int per = (ntiles + kScanSplit - 1) / kScanSplit;
    const int t0 = q * per, t1 = min(ntiles, t0 + per);
    for (int e0 = 0; e0 < E; e0 += kTileRows / kScanSplit) {
      const int x = e0 + threadIdx.x / kScanSplit;
      const bool live = x < E;
      int* col = src_cnt + (live ? x : 0);
      int part = 0;
      for (int t = t0; live && t < t1; ++t) part += __ldcg(col + (size_t)t * E);
      // exclusive prefix of the kScanSplit partial sums (the lanes of one expert are adjacent)
      int inc = part;
#pragma unroll
      for (int off = 1; off < kScanSplit; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, inc, off, kScanSplit);
        if (q >= off) inc += o;
      }
      int run = inc - part;
      for (int t = t0; live && t < t1; ++t) {
        const int v = __ldcg(col + (size_t)t * E);
        col[(size_t)t * E] = run;
        run += v;
      }
      if (live && q == kScanSplit - 1) totals[(size_t)s * E + x] = run;
    }
  }
  // the last source to finish builds the bases and the receive counts
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(&done[0], 1u) == (unsigned)nranks - 1;
    __threadfence();
  }
  __syncthreads();
  if (!s_last) return;
  bases_and_counts(nranks, epr, totals, base, recv_count, warp_cnt, sm_ints);
}

// ---- no rows: bases and receive counts from zero totals (one CTA) ------------------------------------

constexpr int kBaseSmemInts = 8192;

__global__ void __launch_bounds__(1024) a2a_base_kernel(int nranks, int epr, const int* __restrict__ tot,
                                                        int* __restrict__ base, int* __restrict__ recv_count) {
  __shared__ int sm[kBaseSmemInts];
  bases_and_counts(nranks, epr, tot, base, recv_count, sm, kBaseSmemInts);
}

// ---- row copies ---------------------------------------------------------------------------------------

struct A2ACopyParams {
  const char* send[kMaxRanks];
  char* recv[kMaxRanks];
  const int32_t* ids[kMaxRanks];
  const int* tile_off;   // [N][ntiles][E] exclusive prefixes over tiles
  const int* row_rank;   // [N][rows] rank in the row's tile
  const int* base;       // [N][E]
  uint64_t row_bytes;
  uint64_t capacity;
  int tokens, topk, epr, E, ntiles, direction;
};

constexpr int kCopyVecs = 16;  // 16-byte loads per lane in flight before the stores that consume
                               // them (a whole 8 KiB row per warp; measured faster than 8 or 32)

// The first kCopyVecs vectors per lane of a dispatch row (the token row of source s).
__device__ __forceinline__ void load_token_head(const A2ACopyParams& P, int s, int t, int lane, uint4 (&x)[kCopyVecs]) {
  const uint64_t nvec = P.row_bytes / 16;
  const uint4* row = reinterpret_cast<const uint4*>(P.send[s] + (uint64_t)t * P.row_bytes);
#pragma unroll
  for (int b = 0; b < kCopyVecs; ++b)
    if (lane + 32 * b < nvec) x[b] = __ldcs(row + lane + 32 * b);
}

// One token of source s, by one warp: dispatch writes its row to each selected expert's
// position; combine reads the rows back from those positions into slots [t][k]. `base` is
// [N][E]; the table entries are read once each, through L2. With `head` the dispatch row's
// first vectors are already in x.
__device__ __forceinline__ void copy_token(const A2ACopyParams& P, const int* base, int s, int t, int lane,
                                           uint4 (&x)[kCopyVecs], bool head) {
  constexpr int B = kCopyVecs;
  const uint64_t nvec = P.row_bytes / 16;
  const int rows = P.tokens * P.topk;
  char* ptr[kMaxTopk];
  bool ok[kMaxTopk];
  for (int k = 0; k < P.topk; ++k) {
    const int i = t * P.topk + k;
    const int e = P.ids[s][i];
    if (e < 0 || e >= P.E) { ok[k] = false; ptr[k] = nullptr; continue; }
    const int d = e / P.epr;
    const uint64_t pos = (uint64_t)base[s * P.E + e] +
                         __ldcg(P.tile_off + ((size_t)s * P.ntiles + i / kTileRows) * P.E + e) +
                         __ldcg(P.row_rank + (size_t)s * rows + i);
    ok[k] = pos < P.capacity;
    ptr[k] = (P.direction == 0 ? P.recv[d] : const_cast<char*>(P.send[d])) + pos * P.row_bytes;
  }
  if (P.direction == 0) {
    const uint4* row = reinterpret_cast<const uint4*>(P.send[s] + (uint64_t)t * P.row_bytes);
    for (uint64_t v0 = lane; v0 < nvec; v0 += 32 * B) {
      if (v0 != (uint64_t)lane || !head) {
#pragma unroll
        for (int b = 0; b < B; ++b)
          if (v0 + 32 * b < nvec) x[b] = __ldcs(row + v0 + 32 * b);
      }
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

// The copy alone, one warp per token. After a table kernel it is launched as that kernel's
// programmatic dependent: its CTAs may start while the tables are still being built, and wait
// (griddepcontrol.wait) for the table kernel to complete before they read a position. A
// dispatch row does not depend on the tables, so its first vectors are loaded before that wait.
// Launched on its own (a run over an earlier plan) it follows plain stream order, where the
// wait returns at once.
__global__ void __launch_bounds__(256) a2a_copy_kernel(const __grid_constant__ A2ACopyParams P) {
  const int lane = threadIdx.x & 31;
  const int s = blockIdx.y;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= P.tokens) return;
  uint4 x[kCopyVecs];
  if (P.direction == 0) load_token_head(P, s, t, lane, x);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  copy_token(P, P.base, s, t, lane, x, P.direction == 0);
}

static A2ACopyParams copy_params(const void* const* send, void* const* recv, int nranks, size_t row_bytes,
                                 const int32_t* const* ids, int tokens, int topk, int experts_per_rank,
                                 size_t capacity_rows, int direction, const int* tile_off, const int* row_rank,
                                 const int* base) {
  A2ACopyParams P{};
  for (int r = 0; r < nranks; ++r) {
    P.send[r] = static_cast<const char*>(send[r]);
    P.recv[r] = static_cast<char*>(recv[r]);
    P.ids[r] = ids[r];
  }
  P.tile_off = tile_off;
  P.row_rank = row_rank;
  P.base = base;
  P.row_bytes = row_bytes;
  P.capacity = capacity_rows;
  P.tokens = tokens;
  P.topk = topk;
  P.epr = experts_per_rank;
  P.E = nranks * experts_per_rank;
  P.ntiles = (tokens * topk + kTileRows - 1) / kTileRows;
  P.direction = direction;
  return P;
}

cudaError_t launch_alltoallv(const void* const* send, void* const* recv, int nranks, size_t row_bytes,
                             const int32_t* const* ids, int tokens, int topk, int experts_per_rank,
                             size_t capacity_rows, int direction, void* workspace, cudaStream_t stream,
                             A2AParts parts) {
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
  unsigned* done = reinterpret_cast<unsigned*>(ws + w.done);
  IdPtrs I{};
  for (int r = 0; r < nranks; ++r) I.ids[r] = ids[r];
  if (parts & kA2ATables) {
    if (rows > 0) {
      // the finish tickets start at zero (stream-ordered), then one launch builds every table
      const cudaError_t e = cudaMemsetAsync(done, 0, sizeof(unsigned) * (kMaxRanks + 1), stream);
      if (e != cudaSuccess) return e;
      const int scan = (int)std::min<size_t>((size_t)ntiles * E, kScanSmemInts);
      const int bases = std::min(nranks * nranks + nranks * E, kTablesSmemInts);
      const int sm_ints = std::max(std::max(8 * E, nranks * nranks), std::max(scan, bases));
      a2a_tables_kernel<<<dim3(ntiles, nranks), kTileRows, sizeof(int) * sm_ints, stream>>>(
          I, rows, nranks, experts_per_rank, tile_cnt, row_rank, totals, base, recv_count, done, sm_ints);
    } else {
      // no rows: the bases read zero totals (the only write to this scratch before them)
      const cudaError_t e = cudaMemsetAsync(totals, 0, sizeof(int) * nranks * E, stream);
      if (e != cudaSuccess) return e;
      a2a_base_kernel<<<1, 1024, 0, stream>>>(nranks, experts_per_rank, totals, base, recv_count);
    }
    const cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  // the copy; with parts == kA2ACopy it reads the tables an earlier plan left in the workspace
  if (!(parts & kA2ACopy) || rows == 0) return cudaSuccess;
  const A2ACopyParams P = copy_params(send, recv, nranks, row_bytes, ids, tokens, topk, experts_per_rank,
                                      capacity_rows, direction, tile_cnt, row_rank, base);
  // a programmatic dependent of the table kernel launched just before it (see a2a_copy_kernel).
  // A copy on its own follows plain stream order: the kernel before it may be the one that
  // writes the rows this copy reads ahead of its griddepcontrol.wait.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((tokens + 7) / 8, nranks);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (parts & kA2ATables) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, a2a_copy_kernel, P);
}

cudaError_t copy_recv_counts(const void* workspace, int nranks, int32_t* out, cudaStream_t stream) {
  return cudaMemcpyAsync(out, static_cast<const char*>(workspace), sizeof(int32_t) * nranks, cudaMemcpyDefault,
                         stream);
}

}  // namespace cc
