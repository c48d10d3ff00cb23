// Stepped allreduce: the schedule executed step by step, in place on the N output buffers.
//
// The fused kernels (k_reduce.cu) compute every rank's final value in one pass. This kernel
// instead performs the schedule's dependent steps, one grid-wide phase per step, with a
// grid barrier between phases (lecture 09 §4.3 ring: N-1 reduce-scatter steps then N-1
// allgather steps; §5.2 and the multi-node page §4.3.2 double binary tree: reduce up one
// tree level per step, then broadcast down one level per step). Every rank's buffer holds
// what that rank would hold after each step, so the result equals the fused kernels' bit
// for bit, and the time shows the latency of 2(N-1) dependent steps against 2·depth.
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
// The launch is cooperative (all CTAs resident). The grid barrier is a monotonic counter
// in the caller's workspace; waits are bounded by time: a barrier that does not complete
// within 2 s records CC_ERR_TIMEOUT in the device status word and every CTA leaves.
#include <algorithm>
#include <vector>

#include "cc_device.cuh"
#include "cc_launch.h"

namespace cc {

constexpr int kStepThreads = 256;
constexpr uint64_t kBarrierLimitNs = 2000000000ull;

struct StepParams {
  const void* src[kMaxRanks];
  void* buf[kMaxRanks];
  int8_t parent[2][kMaxRanks], left[2][kMaxRanks], right[2][kMaxRanks];
  int8_t level[2][kMaxRanks], depth[2][kMaxRanks];
  uint64_t count;
  unsigned* barrier;
  int* status;  // the library's device status word
  int nranks;
  int fold;      // kFoldRing or kFoldTree
  int copy_in;   // phase 0 needed
  int vec;       // all buffers 16-byte aligned and every job range starts 16-byte aligned
  int up_phases, down_phases;
  float scale;
  int do_scale;
};

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Grid barrier number `phase` (0, 1, ...): returns false when it timed out (the caller leaves).
__device__ __forceinline__ bool grid_barrier(unsigned* counter, int* status, unsigned phase, bool& abort) {
  __shared__ int s_abort;
  __syncthreads();
  if (threadIdx.x == 0) {
    s_abort = 0;
    __threadfence();
    atomicAdd(counter, 1u);
    const unsigned target = (phase + 1) * gridDim.x;
    const uint64_t t0 = now_ns();
    for (;;) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(counter) : "memory");
      if (v >= target) break;
      if (now_ns() - t0 > kBarrierLimitNs) {
        atomicExch(status, (int)CC_ERR_TIMEOUT);
        s_abort = 1;
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
  }
  __syncthreads();
  abort = s_abort != 0;
  return !abort;
}

// Loads that bypass L1 (L1 is not coherent across SMs, and a phase reads what other SMs
// wrote in earlier phases).
template <int T> __device__ __forceinline__ Unit<T> load_cg(const typename Tr<T>::Out* p) {
  return to_unit<T>(__ldcg(reinterpret_cast<const uint4*>(p)));
}
template <typename V> __device__ __forceinline__ V load_cg_elem(const V* p) { return __ldcg(p); }

// One job: buf[dst][e] = ((buf[l][e] (+) buf[dst][e]) (+) buf[r][e]) (l, r may be -1), or a
// copy buf[dst][e] = buf[l][e]; elements [a, b).
struct Job {
  int dst, l, r;
  bool copy, scale;
  uint64_t a, b;
};

template <int IN, int OP>
__device__ __forceinline__ void run_job_unit(const StepParams& P, const Job& j, uint64_t e) {
  using Out = typename Tr<IN>::Out;
  constexpr int OUT_T = IN == CC_I32 ? CC_I32 : CC_F32;
  Out* d = static_cast<Out*>(P.buf[j.dst]) + e;
  Unit<OUT_T> x;
  if (j.copy) {
    x = load_cg<OUT_T>(static_cast<const Out*>(P.buf[j.l]) + e);
  } else {
    x = load_cg<OUT_T>(d);
    if (j.l >= 0) {
      Unit<OUT_T> y = load_cg<OUT_T>(static_cast<const Out*>(P.buf[j.l]) + e);
      op_unit<OUT_T, OP>(y, x);
      x = y;
    }
    if (j.r >= 0) op_unit<OUT_T, OP>(x, load_cg<OUT_T>(static_cast<const Out*>(P.buf[j.r]) + e));
    if (j.scale) scale_unit<OUT_T>(x, P.scale);
  }
  store_unit<OUT_T>(d, x);
}

template <int IN, int OP>
__device__ __forceinline__ void run_job_elem(const StepParams& P, const Job& j, uint64_t e) {
  using Out = typename Tr<IN>::Out;
  Out* d = static_cast<Out*>(P.buf[j.dst]) + e;
  Out x;
  if (j.copy) {
    x = load_cg_elem(static_cast<const Out*>(P.buf[j.l]) + e);
  } else {
    x = load_cg_elem(d);
    if (j.l >= 0) x = op<IN == CC_I32 ? CC_I32 : CC_F32, OP>(load_cg_elem(static_cast<const Out*>(P.buf[j.l]) + e), x);
    if (j.r >= 0) x = op<IN == CC_I32 ? CC_I32 : CC_F32, OP>(x, load_cg_elem(static_cast<const Out*>(P.buf[j.r]) + e));
    if constexpr (IN != CC_I32)
      if (j.scale) x = __fmul_rn(x, P.scale);
  }
  *d = x;
}

__device__ __forceinline__ void chunk_bounds_dev(uint64_t count, int n, int c, uint64_t& a, uint64_t& b) {
  const uint64_t q = count / n, r = count % n, cu = (uint64_t)c;
  a = cu * q + (cu < r ? cu : r);
  b = a + q + (cu < r ? 1 : 0);
}

// The jobs of one phase, job k of njobs (k indexes ranks for the ring, (tree, rank) for the tree).
__device__ __forceinline__ bool phase_job(const StepParams& P, int phase, int k, Job& j) {
  const int n = P.nranks;
  if (P.fold == kFoldRing) {
    const int r = k;
    const int left = (r - 1 + n) % n;
    if (phase < n - 1) {  // reduce-scatter step s
      const int s = phase;
      const int c = ((r - s - 1) % n + n) % n;
      j = Job{r, -1, left, false, P.do_scale != 0 && s == n - 2, 0, 0};
      chunk_bounds_dev(P.count, n, c, j.a, j.b);
    } else {  // allgather step s
      const int s = phase - (n - 1);
      const int c = ((r - s) % n + n) % n;
      j = Job{r, left, -1, true, false, 0, 0};
      chunk_bounds_dev(P.count, n, c, j.a, j.b);
    }
    return true;
  }
  const int t = k / n, r = k % n;
  const uint64_t mid = (P.count + 1) / 2;
  const uint64_t a = t ? mid : 0, b = t ? P.count : mid;
  if (phase < P.up_phases) {
    if (P.level[t][r] != phase + 1) return false;
    j = Job{r, P.left[t][r], P.right[t][r], false, P.do_scale != 0 && P.parent[t][r] < 0, a, b};
    return true;
  }
  const int d = phase - P.up_phases + 1;
  if (P.depth[t][r] != d) return false;
  j = Job{r, P.parent[t][r], -1, true, false, a, b};
  return true;
}

template <int IN, int OP>
__global__ void __launch_bounds__(kStepThreads) stepped_kernel(const __grid_constant__ StepParams P) {
  using In = typename Tr<IN>::In;
  using Out = typename Tr<IN>::Out;
  constexpr uint64_t UE = 4;  // buffers hold 4-byte fp32 / int32
  const uint64_t T = (uint64_t)gridDim.x * blockDim.x;
  const uint64_t tid = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int n = P.nranks;
  unsigned barrier_no = 0;
  bool abort = false;
  if (P.copy_in) {
    const uint64_t total = (uint64_t)n * P.count;
    for (uint64_t i = tid; i < total; i += T) {
      const int r = (int)(i / P.count);
      const uint64_t e = i % P.count;
      const In* s = static_cast<const In*>(P.src[r]);
      Out v;
      if constexpr (IN == CC_BF16) v = __uint_as_float(((uint32_t)reinterpret_cast<const unsigned short*>(s)[e]) << 16);
      else v = s[e];
      if constexpr (IN != CC_I32)
        if (n == 1 && P.do_scale) v = __fmul_rn(v, P.scale);
      static_cast<Out*>(P.buf[r])[e] = v;
    }
    if (!grid_barrier(P.barrier, P.status, barrier_no++, abort)) return;
  }
  const int phases = P.fold == kFoldRing ? 2 * (n - 1) : P.up_phases + P.down_phases;
  const int njobs = P.fold == kFoldRing ? n : 2 * n;
  // every job covers at most `span` elements: a chunk (ring) or a half (tree)
  const uint64_t span = P.fold == kFoldRing ? P.count / n + 1 : (P.count + 1) / 2;
  for (int ph = 0; ph < phases; ++ph) {
    if (P.vec) {
      const uint64_t units = (span + UE - 1) / UE;
      for (uint64_t v = tid; v < (uint64_t)njobs * units; v += T) {
        Job j;
        if (!phase_job(P, ph, (int)(v / units), j)) continue;
        const uint64_t e = j.a + (v % units) * UE;
        if (e + UE <= j.b) run_job_unit<IN, OP>(P, j, e);
        else for (uint64_t x = e; x < j.b; ++x) run_job_elem<IN, OP>(P, j, x);
      }
    } else {
      for (uint64_t v = tid; v < (uint64_t)njobs * span; v += T) {
        Job j;
        if (!phase_job(P, ph, (int)(v / span), j)) continue;
        const uint64_t e = j.a + v % span;
        if (e < j.b) run_job_elem<IN, OP>(P, j, e);
      }
    }
    if (ph + 1 < phases && !grid_barrier(P.barrier, P.status, barrier_no++, abort)) return;
  }
}

// ---- host ------------------------------------------------------------------------------------------

// Double-binary-tree tables in rank terms (the shape rule of k_reduce.cu's tree program).
static void tree_tables(int n, StepParams& P) {
  for (int t = 0; t < 2; ++t) {
    for (int r = 0; r < kMaxRanks; ++r) {
      P.parent[t][r] = P.left[t][r] = P.right[t][r] = -1;
      P.level[t][r] = P.depth[t][r] = 0;
    }
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
    std::vector<int> lev(n, 0), dep(n, 0);
    for (int pass = 0; pass < n; ++pass)
      for (int r = 0; r < n; ++r) {
        int l = 0;
        if (P.left[t][r] >= 0) l = std::max(l, lev[P.left[t][r]] + 1);
        if (P.right[t][r] >= 0) l = std::max(l, lev[P.right[t][r]] + 1);
        lev[r] = l;
        dep[r] = P.parent[t][r] >= 0 ? dep[P.parent[t][r]] + 1 : 0;
      }
    for (int r = 0; r < n; ++r) {
      P.level[t][r] = (int8_t)lev[r];
      P.depth[t][r] = (int8_t)dep[r];
      P.up_phases = std::max(P.up_phases, lev[r]);
      P.down_phases = std::max(P.down_phases, dep[r]);
    }
  }
}

template <int IN, int OP>
static cudaError_t launch_stepped_t(StepParams& P, cudaStream_t s) {
  auto k = stepped_kernel<IN, OP>;
  static int bps = 0;
  if (!bps && (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, k, kStepThreads, 0) != cudaSuccess || bps <= 0))
    return cudaErrorInvalidConfiguration;
  const unsigned grid = (unsigned)(sm_count() * std::min(bps, 4));
  void* args[] = {&P};
  return cudaLaunchCooperativeKernel(reinterpret_cast<void*>(k), dim3(grid), dim3(kStepThreads), args, 0, s);
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
  P.status = async_status_word();
  if (!P.status) return cudaErrorInvalidSymbol;
  bool in_place = true, vec = true;
  for (int r = 0; r < nranks; ++r) {
    P.src[r] = send[r];
    P.buf[r] = recv[r];
    in_place = in_place && send[r] == recv[r];
    vec = vec && (reinterpret_cast<uintptr_t>(recv[r]) & 15) == 0;
  }
  P.copy_in = !in_place || nranks == 1;
  if (fold == kFoldRing) {
    // every chunk must start on a 16-byte boundary for the 16-byte path
    const size_t q = count / nranks, rem = count % nranks;
    vec = vec && q % 4 == 0 && rem == 0;
  } else {
    tree_tables(nranks, P);
    vec = vec && ((count + 1) / 2) % 4 == 0;
  }
  P.vec = vec;
  cudaError_t e = cudaMemsetAsync(barrier, 0, sizeof(unsigned), s);
  if (e != cudaSuccess) return e;
#define CC_STEP_OPS(INT)                                                   \
  switch (op) {                                                            \
    case CC_SUM: return launch_stepped_t<INT, CC_SUM>(P, s);               \
    case CC_MAX: return launch_stepped_t<INT, CC_MAX>(P, s);               \
    case CC_MIN: return launch_stepped_t<INT, CC_MIN>(P, s);               \
    case CC_PROD: return launch_stepped_t<INT, CC_PROD>(P, s);             \
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
