// Stepped allreduce: the schedule executed step by step, in place on the N output buffers.
//
// The fused kernels (k_reduce.cu) compute every rank's final value in one pass. This kernel
// instead performs the schedule's dependent steps, one grid-wide phase per step, with a
// barrier between phases (lecture 09 §4.3 ring: N-1 reduce-scatter steps then N-1 allgather
// steps; §5.2 and the multi-node page §4.3.2 double binary tree: reduce up one tree level per
// step, then broadcast down one level per step). Every rank's buffer holds what that rank
// would hold after each step, so the result equals the fused kernels' bit for bit, and the
// time shows the latency of 2(N-1) dependent steps against 2·depth next to the bandwidth.
//
//   phase 0   recv[r] = send[r] (bf16 widened), unless in place
//   ring RS   step s: rank r: chunk c = (r-s-1) mod N:  recv[r][c] = recv[r][c] (+) recv[r-1][c]
//             (the last step multiplies the completed chunk by `scale`)
//   ring AG   step s: rank r: chunk c = (r-s) mod N:    recv[r][c] = recv[r-1][c]
//   tree up   level h: every node of level h: recv[v] = (recv[left] (+) recv[v]) (+) recv[right]
//             (the root multiplies by `scale`)
//   tree down depth d: every node at depth d: recv[v] = recv[parent]
// Tree A works on elements [0, ceil(count/2)), tree B on the rest, in the same phases.
//
// Work split. A phase is a list of jobs (one per rank for the ring; the nodes of one level
// for the tree), each a contiguous element range of one rank. Large phases cut each job's
// 16-byte units into tiles of kStepThreads x kUnits units that never cross a job; CTAs take
// tiles in turn, and a thread issues the loads of its kUnits units before any fold or store;
// element-wise heads and tails (ranges that do not start or end on a 16-byte boundary) are
// done by the first tile of the job. Small phases (when one slot per unit fits the resident
// grid) give every thread up to kUnits slots of the flattened (job, unit) space per round,
// the last slot of a job taking its head and tail, with the loads of every slot issued before
// the first fold, so a phase costs one or two dependent load-store round trips.
//
// Grid. The launch is cooperative (all CTAs resident). A small phase takes as many CTAs as
// its slots need (kTileUnits slots per CTA), and one CTA when that is one or two, whose
// barrier is __syncthreads(); a large one about kTilesPerCta tiles per CTA, at most the
// resident CTAs. Between phases of a multi-CTA grid the barrier is a monotonic counter in the
// caller's workspace; waits are bounded by time: a barrier that does not complete within 2 s
// records CC_ERR_TIMEOUT in the device status word and every CTA leaves.
#include <algorithm>
#include <vector>

#include "cc_device.cuh"
#include "cc_launch.h"

namespace cc {

constexpr int kStepThreads = 256;
constexpr int kUnits = 4;                                   // 16-byte units per thread and tile
constexpr uint64_t kTileUnits = (uint64_t)kStepThreads * kUnits;
constexpr int kTilesPerCta = 4;                             // tiles of one phase per CTA (grid sizing)
constexpr uint64_t kBarrierLimitNs = 2000000000ull;
constexpr int kMaxTreeJobs = 4 * kMaxRanks;                 // up and down jobs of both trees
constexpr int kMaxTreePhases = 32;

struct StepParams {
  const void* src[kMaxRanks];
  void* buf[kMaxRanks];
  int8_t parent[2][kMaxRanks], left[2][kMaxRanks], right[2][kMaxRanks];
  uint8_t tree_job[kMaxTreeJobs];          // rank | tree << 7, grouped by phase
  uint16_t phase_start[kMaxTreePhases + 1];
  uint64_t count;
  uint64_t chunk_q, chunk_r;               // count / N, count % N
  uint64_t tiles_per_job;                  // large phases: tiles covering the longest job
  uint64_t slots_per_job;                  // small phases: unit slots per job (+1 for head and tail)
  int small;                               // the small-phase kernel runs (slots rather than tiles)
  unsigned* barrier;
  int* status;  // the library's device status word
  int nranks;
  int fold;      // kFoldRing or kFoldTree
  int copy_in;   // phase 0 needed
  int vec;       // every buffer 16-byte aligned (units need 16-byte aligned bases)
  int src_vec;   // every source 16-byte aligned too (16-byte copy-in)
  int phases;
  int up_phases;
  float scale;
  int do_scale;
};

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Barrier number `phase` (0, 1, ...) between phases: __syncthreads() on a one-CTA grid,
// else a grid barrier on the counter. Returns false when it timed out (the caller leaves).
__device__ __forceinline__ bool phase_barrier(unsigned* counter, int* status, unsigned phase) {
  __shared__ int s_abort;
  if (gridDim.x == 1) {
    __syncthreads();  // global writes of the block are visible to the block after it
    return true;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    s_abort = 0;
    __threadfence();
    atomicAdd(counter, 1u);
    const unsigned target = (phase + 1) * gridDim.x;
    const uint64_t t0 = now_ns();
    int polls = 0;
    for (;;) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
      if (v >= target) break;
      if (now_ns() - t0 > kBarrierLimitNs) {
        atomicExch(status, (int)CC_ERR_TIMEOUT);
        s_abort = 1;
        break;
      }
      if (++polls > 256) __nanosleep(128);  // poll back-to-back first: a phase ends within microseconds
    }
    __threadfence();
  }
  __syncthreads();
  return s_abort == 0;
}

// One job: buf[dst][e] = ((buf[l][e] (+) buf[dst][e]) (+) buf[r][e]) (l, r may be -1), or a
// copy buf[dst][e] = buf[l][e]; elements [a, b).
struct Job {
  int dst, l, r;
  bool copy, scale;
  uint64_t a, b;
};

__device__ __forceinline__ void chunk_bounds_dev(const StepParams& P, int c, uint64_t& a, uint64_t& b) {
  const uint64_t cu = (uint64_t)c;
  a = cu * P.chunk_q + (cu < P.chunk_r ? cu : P.chunk_r);
  b = a + P.chunk_q + (cu < P.chunk_r ? 1 : 0);
}

__device__ __forceinline__ int phase_jobs(const StepParams& P, int ph) {
  if (P.fold == kFoldRing) return P.nranks;
  return P.phase_start[ph + 1] - P.phase_start[ph];
}

__device__ __forceinline__ Job phase_job(const StepParams& P, int ph, int k) {
  const int n = P.nranks;
  Job j;
  if (P.fold == kFoldRing) {
    const int r = k;
    const int left = r == 0 ? n - 1 : r - 1;
    if (ph < n - 1) {  // reduce-scatter step s: rank r folds the chunk its left neighbour sends
      const int s = ph;
      const int c = ((r - s - 1) % n + n) % n;
      j = Job{r, -1, left, false, P.do_scale != 0 && s == n - 2, 0, 0};
      chunk_bounds_dev(P, c, j.a, j.b);
    } else {  // allgather step s: rank r takes the completed chunk from its left neighbour
      const int s = ph - (n - 1);
      const int c = ((r - s) % n + n) % n;
      j = Job{r, left, -1, true, false, 0, 0};
      chunk_bounds_dev(P, c, j.a, j.b);
    }
    return j;
  }
  const uint8_t code = P.tree_job[P.phase_start[ph] + k];
  const int t = code >> 7, r = code & 127;
  const uint64_t mid = (P.count + 1) / 2;
  const uint64_t a = t ? mid : 0, b = t ? P.count : mid;
  if (ph < P.up_phases) return Job{r, P.left[t][r], P.right[t][r], false, P.do_scale != 0 && P.parent[t][r] < 0, a, b};
  return Job{r, P.parent[t][r], -1, true, false, a, b};
}

template <typename V> __device__ __forceinline__ V ldcg_elem(const V* p) { return __ldcg(p); }

// One element of a job (heads, tails, and every element of unaligned buffers).
template <int OT, int OP>
__device__ __forceinline__ void job_elem(const StepParams& P, const Job& j, uint64_t e) {
  using V = typename Tr<OT>::Acc;
  V* d = static_cast<V*>(P.buf[j.dst]) + e;
  V x;
  if (j.copy) {
    x = ldcg_elem(static_cast<const V*>(P.buf[j.l]) + e);
  } else {
    x = ldcg_elem(d);
    if (j.l >= 0) x = op<OT, OP>(ldcg_elem(static_cast<const V*>(P.buf[j.l]) + e), x);
    if (j.r >= 0) x = op<OT, OP>(x, ldcg_elem(static_cast<const V*>(P.buf[j.r]) + e));
    if constexpr (OT != CC_I32)
      if (j.scale) x = __fmul_rn(x, P.scale);
  }
  *d = x;
}

// Up to `nunits` (<= kUnits) 16-byte units of a job, `stride` elements apart, starting at
// element e0 (units at or past `vb` are skipped): every load is issued before the first fold.
template <int OT, int OP>
__device__ __forceinline__ void job_units(const StepParams& P, const Job& j, uint64_t e0, uint64_t stride,
                                          uint64_t vb, int nunits) {
  using V = typename Tr<OT>::Acc;
  V* d = static_cast<V*>(P.buf[j.dst]);
  const V* l = j.l >= 0 ? static_cast<const V*>(P.buf[j.l]) : nullptr;
  const V* r = j.r >= 0 ? static_cast<const V*>(P.buf[j.r]) : nullptr;
  uint4 xd[kUnits], xl[kUnits], xr[kUnits];
#pragma unroll
  for (int i = 0; i < kUnits; ++i) {
    const uint64_t e = e0 + i * stride;
    if (i < nunits && e < vb) {
      if (!j.copy) xd[i] = __ldcg(reinterpret_cast<const uint4*>(d + e));
      if (l) xl[i] = __ldcg(reinterpret_cast<const uint4*>(l + e));
      if (r) xr[i] = __ldcg(reinterpret_cast<const uint4*>(r + e));
    }
  }
#pragma unroll
  for (int i = 0; i < kUnits; ++i) {
    const uint64_t e = e0 + i * stride;
    if (i >= nunits || e >= vb) continue;
    uint4 out;
    if (j.copy) {
      out = xl[i];
    } else {
      Unit<OT> x = to_unit<OT>(xd[i]);
      if (l) {
        Unit<OT> y = to_unit<OT>(xl[i]);
        op_unit<OT, OP>(y, x);
        x = y;
      }
      if (r) op_unit<OT, OP>(x, to_unit<OT>(xr[i]));
      if (j.scale) scale_unit<OT>(x, P.scale);
      const uint32_t* w = reinterpret_cast<const uint32_t*>(x.v);
      out = make_uint4(w[0], w[1], w[2], w[3]);
    }
    *reinterpret_cast<uint4*>(d + e) = out;
  }
}

template <int IN, int OP, bool SMALL>
__global__ void __launch_bounds__(kStepThreads, SMALL ? 1 : 3) stepped_kernel(const __grid_constant__ StepParams P) {
  using In = typename Tr<IN>::In;
  constexpr int OT = IN == CC_I32 ? CC_I32 : CC_F32;  // the buffers hold 4-byte fp32 / int32
  using V = typename Tr<OT>::Acc;
  constexpr uint64_t UE = 4;
  const uint64_t T = (uint64_t)gridDim.x * kStepThreads;
  const uint64_t tid = (uint64_t)blockIdx.x * kStepThreads + threadIdx.x;
  const int n = P.nranks;
  unsigned barrier_no = 0;
  if (P.copy_in) {
    const bool scale_in = n == 1 && P.do_scale;
    for (int r = 0; r < n; ++r) {
      const In* s = static_cast<const In*>(P.src[r]);
      V* d = static_cast<V*>(P.buf[r]);
      uint64_t done = 0;
      if (P.src_vec && P.vec) {
        // 16-byte source loads: 4 elements of 4 bytes, or 8 bf16 elements (two output units)
        constexpr uint64_t SE = IN == CC_BF16 ? 8 : 4;
        const uint64_t nv = P.count / SE;
        for (uint64_t v = tid; v < nv; v += T) {
          const uint4 w = __ldcs(reinterpret_cast<const uint4*>(s) + v);
          Unit<IN> u = to_unit<IN>(w);
          if (scale_in) scale_unit<IN>(u, P.scale);
          const uint32_t* b = reinterpret_cast<const uint32_t*>(u.v);
#pragma unroll
          for (int q = 0; q < (int)SE / 4; ++q)  // plain stores: the next phase reads them back
            reinterpret_cast<uint4*>(d + v * SE)[q] = make_uint4(b[4 * q], b[4 * q + 1], b[4 * q + 2], b[4 * q + 3]);
        }
        done = nv * SE;
      }
      for (uint64_t e = done + tid; e < P.count; e += T) {
        V v;
        if constexpr (IN == CC_BF16) v = __uint_as_float(((uint32_t)reinterpret_cast<const unsigned short*>(s)[e]) << 16);
        else v = s[e];
        if constexpr (IN != CC_I32)
          if (scale_in) v = __fmul_rn(v, P.scale);
        d[e] = v;
      }
    }
    if (P.phases > 0 && !phase_barrier(P.barrier, P.status, barrier_no++)) return;
  }
  const uint64_t tpj = P.tiles_per_job, spj = P.slots_per_job;
  for (int ph = 0; ph < P.phases; ++ph) {
    const uint32_t njobs = (uint32_t)phase_jobs(P, ph);
    if constexpr (SMALL) {
      // slots f0 + i*T (i < kUnits) per round: unit u of job k, or (the job's last slot) its
      // head and tail; every unit slot's loads are issued before the first fold
      const uint64_t nslots = (uint64_t)njobs * spj;
      for (uint64_t f0 = tid; f0 < nslots; f0 += T * kUnits) {
        V* dp[kUnits];
        const V* lp[kUnits];
        const V* rp[kUnits];
        int fl[kUnits];  // bit 0: a unit to fold, bit 1: copy, bit 2: scale
        uint4 xd[kUnits], xl[kUnits], xr[kUnits];
#pragma unroll
        for (int i = 0; i < kUnits; ++i) {
          fl[i] = 0;
          dp[i] = nullptr;
          lp[i] = rp[i] = nullptr;
          const uint64_t f = f0 + (uint64_t)i * T;
          if (f >= nslots) continue;
          const uint32_t k = (uint32_t)f / (uint32_t)spj;
          const uint64_t u = f - (uint64_t)k * spj;
          const Job j = phase_job(P, ph, (int)k);
          if (!P.vec) {
            if (j.a + u < j.b) job_elem<OT, OP>(P, j, j.a + u);
            continue;
          }
          uint64_t va = (j.a + UE - 1) / UE * UE;
          if (va > j.b) va = j.b;
          uint64_t vb = j.b / UE * UE;
          if (vb < va) vb = va;
          if (u < (vb - va) / UE) {
            const uint64_t e = va + u * UE;
            dp[i] = static_cast<V*>(P.buf[j.dst]) + e;
            if (j.l >= 0) lp[i] = static_cast<const V*>(P.buf[j.l]) + e;
            if (j.r >= 0) rp[i] = static_cast<const V*>(P.buf[j.r]) + e;
            fl[i] = 1 | (j.copy ? 2 : 0) | (j.scale ? 4 : 0);
          } else if (u == spj - 1) {
            for (uint64_t e = j.a; e < va; ++e) job_elem<OT, OP>(P, j, e);
            for (uint64_t e = vb; e < j.b; ++e) job_elem<OT, OP>(P, j, e);
          }
        }
#pragma unroll
        for (int i = 0; i < kUnits; ++i) {
          if (!(fl[i] & 1)) continue;
          if (!(fl[i] & 2)) xd[i] = __ldcg(reinterpret_cast<const uint4*>(dp[i]));
          if (lp[i]) xl[i] = __ldcg(reinterpret_cast<const uint4*>(lp[i]));
          if (rp[i]) xr[i] = __ldcg(reinterpret_cast<const uint4*>(rp[i]));
        }
#pragma unroll
        for (int i = 0; i < kUnits; ++i) {
          if (!(fl[i] & 1)) continue;
          uint4 out;
          if (fl[i] & 2) {
            out = xl[i];
          } else {
            Unit<OT> x = to_unit<OT>(xd[i]);
            if (lp[i]) {
              Unit<OT> y = to_unit<OT>(xl[i]);
              op_unit<OT, OP>(y, x);
              x = y;
            }
            if (rp[i]) op_unit<OT, OP>(x, to_unit<OT>(xr[i]));
            if (fl[i] & 4) scale_unit<OT>(x, P.scale);
            const uint32_t* w = reinterpret_cast<const uint32_t*>(x.v);
            out = make_uint4(w[0], w[1], w[2], w[3]);
          }
          *reinterpret_cast<uint4*>(dp[i]) = out;
        }
      }
    } else {
      for (uint64_t tile = blockIdx.x; tile < njobs * tpj; tile += gridDim.x) {
        const uint32_t k = (uint32_t)tile / (uint32_t)tpj;
        const uint64_t part = tile - (uint64_t)k * tpj;
        const Job j = phase_job(P, ph, (int)k);
        if (P.vec) {
          uint64_t va = (j.a + UE - 1) / UE * UE;
          if (va > j.b) va = j.b;
          uint64_t vb = j.b / UE * UE;
          if (vb < va) vb = va;
          const uint64_t e0 = va + (part * kTileUnits + threadIdx.x) * UE;
          job_units<OT, OP>(P, j, e0, (uint64_t)kStepThreads * UE, vb, kUnits);
          if (part == 0) {
            const uint64_t nh = va - j.a, nt = j.b - vb;
            if (threadIdx.x < nh) job_elem<OT, OP>(P, j, j.a + threadIdx.x);
            else if (threadIdx.x < nh + nt) job_elem<OT, OP>(P, j, vb + (threadIdx.x - nh));
          }
        } else {
          const uint64_t base = j.a + part * kTileUnits;
          for (int i = 0; i < kUnits; ++i) {
            const uint64_t e = base + (uint64_t)i * kStepThreads + threadIdx.x;
            if (e < j.b) job_elem<OT, OP>(P, j, e);
          }
        }
      }
    }
    if (ph + 1 < P.phases && !phase_barrier(P.barrier, P.status, barrier_no++)) return;
  }
}

// ---- host ------------------------------------------------------------------------------------------

// Double-binary-tree tables in rank terms (the shape rule of k_reduce.cu's tree program) and
// the phase-grouped job lists: up phase h holds the nodes of subtree height h (h = 1, 2, ...),
// down phase d the nodes at depth d (d = 1, 2, ...), both trees in the same phases.
static bool tree_tables(int n, StepParams& P) {
  std::vector<int> lev[2], dep[2];
  int up = 0, down = 0;
  for (int t = 0; t < 2; ++t) {
    for (int r = 0; r < kMaxRanks; ++r) P.parent[t][r] = P.left[t][r] = P.right[t][r] = -1;
    auto rank_of = [&](int q) { return t ? n - q : q - 1; };  // label q = position + 1
    for (int q = 1; q <= n; ++q) {
      const int h = __builtin_ctz((unsigned)q);
      if (h == 0) continue;
      const int lq = q - (1 << (h - 1));
      P.left[t][rank_of(q)] = (int8_t)rank_of(lq);
      P.parent[t][rank_of(lq)] = (int8_t)rank_of(q);
      for (int j = h; j >= 1; --j) {
        const int rq = q + (1 << (j - 1));
        if (rq <= n) {
          P.right[t][rank_of(q)] = (int8_t)rank_of(rq);
          P.parent[t][rank_of(rq)] = (int8_t)rank_of(q);
          break;
        }
      }
    }
    // level = height of the node's subtree (leaves 0); depth = distance from the root
    lev[t].assign(n, 0);
    dep[t].assign(n, 0);
    for (int pass = 0; pass < n; ++pass)
      for (int r = 0; r < n; ++r) {
        int l = 0;
        if (P.left[t][r] >= 0) l = std::max(l, lev[t][P.left[t][r]] + 1);
        if (P.right[t][r] >= 0) l = std::max(l, lev[t][P.right[t][r]] + 1);
        lev[t][r] = l;
        dep[t][r] = P.parent[t][r] >= 0 ? dep[t][P.parent[t][r]] + 1 : 0;
      }
    for (int r = 0; r < n; ++r) {
      up = std::max(up, lev[t][r]);
      down = std::max(down, dep[t][r]);
    }
  }
  if (up + down > kMaxTreePhases) return false;
  int pos = 0, ph = 0;
  for (int h = 1; h <= up; ++h, ++ph) {
    P.phase_start[ph] = (uint16_t)pos;
    for (int t = 0; t < 2; ++t)
      for (int r = 0; r < n; ++r)
        if (lev[t][r] == h) P.tree_job[pos++] = (uint8_t)(r | (t << 7));
  }
  for (int d = 1; d <= down; ++d, ++ph) {
    P.phase_start[ph] = (uint16_t)pos;
    for (int t = 0; t < 2; ++t)
      for (int r = 0; r < n; ++r)
        if (dep[t][r] == d) P.tree_job[pos++] = (uint8_t)(r | (t << 7));
  }
  P.phase_start[ph] = (uint16_t)pos;
  P.up_phases = up;
  P.phases = up + down;
  return pos <= kMaxTreeJobs;
}

template <typename K> static int resident_ctas(K kernel, int& cache) {
  if (!cache && (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&cache, kernel, kStepThreads, 0) != cudaSuccess ||
                 cache <= 0)) {
    cache = 0;
    return 0;
  }
  return sm_count() * cache;
}

// Launch the small-phase kernel (slots) when its grid fits the resident CTAs, else the
// large-phase kernel (tiles); never more CTAs than the occupancy the runtime reports for that
// exact kernel (static shared memory included), since every CTA of a cooperative launch must
// be resident at once. A small grid of one or two CTAs' worth of slots runs on one CTA.
template <int IN, int OP>
static cudaError_t launch_stepped(StepParams& P, uint64_t slot_ctas, uint64_t tile_ctas, cudaStream_t s) {
  auto ks = stepped_kernel<IN, OP, true>;
  auto kl = stepped_kernel<IN, OP, false>;
  static int bps_s = 0, bps_l = 0;
  const int res_s = resident_ctas(ks, bps_s), res_l = resident_ctas(kl, bps_l);
  if (!res_s || !res_l) return cudaErrorInvalidConfiguration;
  const bool small = P.small > 0 || (P.small < 0 && slot_ctas <= (uint64_t)res_s);
  P.small = small ? 1 : 0;
  uint64_t want = small ? (slot_ctas <= 2 ? 1 : slot_ctas) : tile_ctas;
  want = std::max<uint64_t>(1, std::min<uint64_t>(want, (uint64_t)(small ? res_s : res_l)));
  void* args[] = {&P};
  return cudaLaunchCooperativeKernel(small ? reinterpret_cast<void*>(ks) : reinterpret_cast<void*>(kl),
                                     dim3((unsigned)want), dim3(kStepThreads), args, 0, s);
}

cudaError_t launch_stepped_allreduce(const void* const* send, void* const* recv, int nranks, size_t count,
                                     cc_dtype in_t, cc_op op, FoldKind fold, float scale, unsigned* barrier,
                                     cudaStream_t s) {
  StepParams P{};
  P.count = count;
  P.nranks = nranks;
  P.fold = fold;
  P.scale = scale;
  P.do_scale = in_t != CC_I32 && scale != 1.0f;
  P.barrier = barrier;
  P.chunk_q = count / nranks;
  P.chunk_r = count % nranks;
  P.status = async_status_word();
  if (!P.status) return cudaErrorInvalidSymbol;
  bool in_place = true, vec = true, src_vec = true;
  for (int r = 0; r < nranks; ++r) {
    P.src[r] = send[r];
    P.buf[r] = recv[r];
    in_place = in_place && send[r] == recv[r];
    vec = vec && (reinterpret_cast<uintptr_t>(recv[r]) & 15) == 0;
    src_vec = src_vec && (reinterpret_cast<uintptr_t>(send[r]) & 15) == 0;
  }
  P.copy_in = !in_place || nranks == 1;
  P.vec = vec;
  P.src_vec = src_vec;
  // the longest job of any phase: a ring chunk, or a tree half
  uint64_t longest;
  if (fold == kFoldRing) {
    P.phases = nranks > 1 ? 2 * (nranks - 1) : 0;
    longest = P.chunk_q + (P.chunk_r ? 1 : 0);
  } else {
    if (!tree_tables(nranks, P)) return cudaErrorInvalidValue;  // not reached for N <= 64
    longest = (count + 1) / 2;
  }
  // a job's units start at its first 16-byte boundary: a job of `longest` elements spans at
  // most longest / 4 whole units; tiles (large phases) cover them, slots (small phases) cover
  // them plus one slot for the element-wise head and tail
  const uint64_t units = vec ? longest / 4 : longest;
  P.tiles_per_job = std::max<uint64_t>(1, (units + kTileUnits - 1) / kTileUnits);
  P.slots_per_job = units + 1;
  int max_jobs = fold == kFoldRing ? nranks : 0;
  for (int ph = 0; fold != kFoldRing && ph < P.phases; ++ph)
    max_jobs = std::max(max_jobs, (int)(P.phase_start[ph + 1] - P.phase_start[ph]));
  max_jobs = std::max(1, max_jobs);
  // small: the slots of the busiest phase fit the resident grid (decided at launch); the grid
  // is sized to those slots, or else to the busiest phase's tiles
  const uint64_t slot_ctas = ((uint64_t)max_jobs * P.slots_per_job + kTileUnits - 1) / kTileUnits;
  const uint64_t tile_ctas = ((uint64_t)max_jobs * P.tiles_per_job + kTilesPerCta - 1) / kTilesPerCta;
  P.small = -1;
  uint64_t want = slot_ctas;
  if (P.phases == 0) {
    P.small = 1;  // copy-in only
    want = std::max<uint64_t>(1, (count * nranks / 4 + kTileUnits - 1) / kTileUnits);
  }
  cudaError_t e = cudaMemsetAsync(barrier, 0, sizeof(unsigned), s);
  if (e != cudaSuccess) return e;
#define CC_STEP_OPS(INT)                                                   \
  switch (op) {                                                            \
    case CC_SUM: return launch_stepped<INT, CC_SUM>(P, want, tile_ctas, s);   \
    case CC_MAX: return launch_stepped<INT, CC_MAX>(P, want, tile_ctas, s);   \
    case CC_MIN: return launch_stepped<INT, CC_MIN>(P, want, tile_ctas, s);   \
    case CC_PROD: return launch_stepped<INT, CC_PROD>(P, want, tile_ctas, s); \
  }
  switch (in_t) {
    case CC_F32: CC_STEP_OPS(CC_F32) break;
    case CC_BF16: CC_STEP_OPS(CC_BF16) break;
    case CC_I32: CC_STEP_OPS(CC_I32) break;
  }
#undef CC_STEP_OPS
  return cudaErrorInvalidValue;
}

}  // namespace cc
