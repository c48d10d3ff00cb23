// Reduction kernels: fused ring / double-binary-tree allreduce, ring reduce-scatter,
// binomial reduce-to-root, and the fused DDP bucket allreduce.
//
// All simulated ranks live in this GPU's memory, so one pass computes what every rank
// would hold at the end of the schedule: each thread owns a 16-byte column of the N rank
// buffers, loads it from every rank (streaming 128-bit loads), folds the N values in the
// schedule's order in registers, multiplies by the scale, and stores the result to every
// output (allreduce), to the owning shard (reduce-scatter) or to the root (reduce).
// HBM traffic is the minimum the operation allows (N·T in + N·T out for allreduce).
//
// Fold orders (collective pages: lecture 09 §4.3 and experiment 1 §7.1 for the ring, §5.2
// and the multi-node page §4.3.2 for the double binary tree, §3.4 for reduce):
//   ring      chunk c folds ((x_c (+) x_{c+1}) (+) ...) (+) x_{c-1}
//   tree      half A / half B fold over tree A / tree B, ((S_left (+) x) (+) S_right)
//   binomial  node v folds x_v, then each child's partial in send order
//   multi-ring  part k of K (chunk rule), chunk c inside it: the ring fold starting at rank c,
//             walking up the ranks for even k and down for odd k (lecture 09 §5.3)
//
// The folds and the plain reduction kernel are in k_reduce_kernels.cuh (shared with
// k_reduce_binom.cu); this file holds the bucket allreduce kernel and the host side.
#include <algorithm>
#include <mutex>
#include <vector>

#include "k_reduce_kernels.cuh"

namespace cc {

// ---- fused DDP bucket allreduce --------------------------------------------------------------------
// One launch covers a group of gradient tensors. Work is cut into tiles of kBucketTile
// elements that never cross a tensor, one CTA per tile; a CTA finds its tile's tensor by
// binary search in the tile prefix table, stages that tensor's 2N pointers in shared
// memory, and splits the tile at the fold-group boundaries of the tensor's bucket (ring
// chunks or tree halves, in bucket coordinates).
// Every element is folded exactly as in flatten -> allreduce -> unflatten, with no flat
// buffer: N·G bytes in, N·G bytes out.

#ifndef CC_BUCKET_TILE
#define CC_BUCKET_TILE 1024        // elements per tile (one 16-byte unit per thread)
#endif
#ifndef CC_BUCKET_MIN_BLOCKS
#define CC_BUCKET_MIN_BLOCKS 4     // resident 256-thread CTAs per SM the ring variant is compiled for
#endif
#ifndef CC_BUCKET_TREE_MIN_BLOCKS
#define CC_BUCKET_TREE_MIN_BLOCKS 4  // the same for the tree variant (fold machine; DDP step 6022 vs 5313 GB/s at 2)
#endif
#ifndef CC_BUCKET_OVERSUB
#define CC_BUCKET_OVERSUB 1024     // grid = tiles, capped at this many times the resident CTAs
#endif
constexpr int kBucketMaxTensors = 192;
constexpr int kBucketMaxPtrs = 1536;
constexpr uint64_t kBucketTile = CC_BUCKET_TILE;

// Tables travel as kernel parameters: a large block (up to 192 tensors, 30 KB) for whole
// tensor lists, and a small one (under 4 KB) for the short lists of the host-buffer
// pipeline, whose many queued launches would otherwise hold the driver's parameter space.
template <int MAXT, int MAXP> struct BucketParamsT {
  static constexpr int kMaxT = MAXT, kMaxP = MAXP;
  int nranks;
  int ntensors;
  int fold;
  int vec;
  float scale;
  int do_scale;
  FoldProgram prog;
  uint32_t tile_prefix[MAXT + 1];
  BucketTensorDesc t[MAXT];
  const float* in[MAXP];
  float* out[MAXP];
};
using BucketParams = BucketParamsT<kBucketMaxTensors, kBucketMaxPtrs>;
using BucketParamsSmall = BucketParamsT<8, 64>;
static_assert(sizeof(BucketParams) <= 32000, "kernel parameter block too large");
static_assert(sizeof(BucketParamsSmall) <= 4096, "small parameter block must stay under 4 KB");

// KIND: kLinear (ring), kTree8 / kTree16 (the compiled double binary tree of 8 / 16 ranks),
// kMachine (the tree of any other rank count, on the fold machine).
template <int KIND, typename PT>
__global__ void __launch_bounds__(kThreads, KIND == kMachine ? CC_BUCKET_TREE_MIN_BLOCKS : CC_BUCKET_MIN_BLOCKS)
    bucket_allreduce_kernel(const __grid_constant__ PT P) {
  constexpr int IN = CC_F32, OP = CC_SUM;
  constexpr bool RING = KIND == kLinear;
  // the tile's per-rank pointers, staged once per tile: the fold reads them for every
  // 16-byte unit, and the parameter table is too large to stay in the constant cache
  __shared__ const float* s_in[kMaxRanks];
  __shared__ float* s_out[kMaxRanks];
  __shared__ int s_tensor;
  __shared__ uint4 s_stk[KIND == kMachine ? kStackSlots * kThreads : 1];  // the machine's pending partials
  const int n = P.nranks, nt = P.ntensors;
  const uint32_t ntiles = P.tile_prefix[nt];
  for (uint32_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    if (threadIdx.x == 0) {
      int lo = 0, hi = nt - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (P.tile_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
      }
      s_tensor = lo;
    }
    __syncthreads();
    const int i = s_tensor;
    if (threadIdx.x < n) {
      s_in[threadIdx.x] = P.in[threadIdx.x * nt + i];
      s_out[threadIdx.x] = P.out[threadIdx.x * nt + i];
    }
    __syncthreads();
    const BucketTensorDesc d = P.t[i];
    const uint64_t ea = (uint64_t)(tile - P.tile_prefix[i]) * kBucketTile;
    const uint64_t eb = min(ea + kBucketTile, d.numel);
    auto src = [&](int r) { return s_in[r]; };
    auto emit_unit = [&](uint64_t e, Unit<IN> u) {
      if (P.do_scale) scale_unit<IN>(u, P.scale);
      for (int r = 0; r < n; ++r) store_unit<IN>(s_out[r] + e, u);
    };
    auto emit_elem = [&](uint64_t e, float v) {
      if (P.do_scale) v = __fmul_rn(v, P.scale);
      for (int r = 0; r < n; ++r) store_elem<IN>(s_out[r] + e, v);
    };
    uint64_t s = ea;
    while (s < eb) {
      const uint64_t o = d.bucket_off + s;
      uint64_t gend;
      int g;
      if (RING) {
        uint64_t gstart;
        g = chunk_of(d.bucket_count, n, o, gstart, gend);
      } else {
        const uint64_t mid = (d.bucket_count + 1) / 2;
        g = o >= mid;
        gend = g ? d.bucket_count : mid;
      }
      const uint64_t se = min(eb, gend - d.bucket_off);
      const bool mirror = !RING && g == 1;
      auto rank_of = [&](int p) {
        const int rk = P.prog.rmap[p];
        return mirror ? n - 1 - rk : rk;
      };
      reduce_range<IN, OP, KIND>(n, g, rank_of, P.prog, s, se, threadIdx.x, blockDim.x, P.vec != 0, src, emit_unit,
                                 emit_elem, s_stk + threadIdx.x, g, true);
      s = se;
    }
    __syncthreads();  // every thread is done with s_in / s_out before the next tile restages them
  }
}

// ---- host side --------------------------------------------------------------------------------------

static int ctz_int(int q) { return __builtin_ctz((unsigned)q); }

// Double binary tree, tree A, in fold-machine codes (tree B uses the same codes mirrored).
static void tree_program(int n, FoldProgram& fp) {
  int left[kMaxRanks + 2] = {0}, right[kMaxRanks + 2] = {0}, parent[kMaxRanks + 2] = {0};
  bool is_right[kMaxRanks + 2] = {false};
  for (int q = 1; q <= n; ++q) {
    const int h = ctz_int(q);
    if (h == 0) continue;
    const int lq = q - (1 << (h - 1));
    left[q] = lq;
    parent[lq] = q;
    for (int j = h; j >= 1; --j) {
      const int rq = q + (1 << (j - 1));
      if (rq <= n) {
        right[q] = rq;
        parent[rq] = q;
        is_right[rq] = true;
        break;
      }
    }
  }
  for (int p = 0; p < n; ++p) {
    const int q = p + 1;
    uint8_t code = left[q] ? kFoldCur : 0;
    if (right[q]) {
      code |= kPush;
    } else {
      int npop = 0, u = q;
      while (parent[u] && is_right[u]) { ++npop; u = parent[u]; }
      code |= (uint8_t)(npop << 2);
    }
    fp.code[p] = code;
    fp.rmap[p] = (uint8_t)p;
  }
  // A right child that is a leaf is the very next position: instead of pushing
  // (S_left (+) x) and popping it back after the leaf, fold the leaf into cur directly
  // (((S_left (+) x) (+) leaf), the same operations in the same order).
  for (int p = 0; p + 1 < n; ++p) {
    const int q = p + 1;
    if (right[q] == q + 1 && (fp.code[p] & kPush) && npop_of(fp.code[p + 1]) > 0) {
      fp.code[p] &= (uint8_t)~kPush;
      const int np = npop_of(fp.code[p + 1]) - 1;
      fp.code[p + 1] = (uint8_t)((fp.code[p + 1] & ~(7 << 2)) | kFoldCur | (np << 2));
    }
  }
}

// Whether a program computes a plain left fold of its positions in order,
// ((x_0 (+) x_1) (+) x_2) ..., and walks the ranks upwards from rmap[0] (tree A folds ranks
// 0, 1, ..., n-1; tree B is its mirror; a binomial program from its root): it then runs as
// the linear fold. The program is run symbolically: a value is "the left fold of positions
// 0..k" (k >= 0; a single x_0 is k = 0), "position p alone", or anything else; one (+) of
// the left fold of 0..k and position k+1 (in either operand order: each operator is
// commutative) is the left fold of 0..k+1. Binomial programs for 2 and 3 ranks use a push
// and a pop and still reduce to the left fold.
static bool program_is_rotation(int n, const FoldProgram& fp) {
  for (int p = 0; p < n; ++p)
    if (fp.rmap[p] != (fp.rmap[0] + p) % n) return false;
  // value encoding: v >= 0 left fold of 0..v; v = -2 - p position p alone; kOther otherwise
  constexpr int kOther = -1;
  auto leaf = [](int p) { return p == 0 ? 0 : -2 - p; };
  auto comb = [&](int a, int b) {
    if (a >= 0 && b <= -2 && -2 - b == a + 1) return a + 1;
    if (b >= 0 && a <= -2 && -2 - a == b + 1) return b + 1;
    return kOther;
  };
  int cur = kOther;
  std::vector<int> st;
  for (int p = 0; p < n; ++p) {
    const uint8_t c = fp.code[p];
    int node = leaf(p);
    if (c & kFoldCur) node = comb(cur, node);
    if (c & kPush) st.push_back(node); else cur = node;
    for (int k = npop_of(c); k > 0; --k) {
      if (st.empty()) return false;
      cur = comb(st.back(), cur);
      st.pop_back();
    }
    if (c & kFoldTop) {
      if (st.empty()) return false;
      st.back() = comb(st.back(), cur);
    }
  }
  return st.empty() && cur == n - 1;
}

// Binomial tree rooted at `root` (relative rank v = (r - root) mod n; parent v - 2^floor(log2 v);
// children v + 2^k for 2^k > v), visited in pre-order.
static void binomial_program(int n, int root, FoldProgram& fp) {
  auto children = [n](int v) {
    std::vector<int> ch;
    int k = 0;
    if (v) while ((1 << k) <= v) ++k;
    for (; v + (1 << k) < n; ++k) ch.push_back(v + (1 << k));
    return ch;
  };
  auto parent_of = [](int v) { int k = 0; while ((2 << k) <= v) ++k; return v - (1 << k); };
  std::vector<int> order;
  std::vector<int> stack = {0};
  while (!stack.empty()) {
    const int v = stack.back();
    stack.pop_back();
    order.push_back(v);
    auto ch = children(v);
    for (auto it = ch.rbegin(); it != ch.rend(); ++it) stack.push_back(*it);
  }
  for (int p = 0; p < n; ++p) {
    const int v = order[p];
    uint8_t code = 0;
    if (!children(v).empty()) {
      code = kPush;
    } else {
      int npop = 0, u = v;
      while (u != 0) {
        const int par = parent_of(u);
        const auto sib = children(par);
        if (sib.back() == u) { ++npop; u = par; continue; }
        code |= kFoldTop;
        break;
      }
      code |= (uint8_t)(npop << 2);
    }
    fp.code[p] = code;
    fp.rmap[p] = (uint8_t)((v + root) % n);
  }
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int sm_count() {
  static int cached[64];
  static std::once_flag once[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  std::call_once(once[dev], [dev] {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cached[dev] = v;
  });
  return cached[dev];
}

// Sums over sources at one offset into outputs at another: element stores on the sources' units.
template <int IN>
static cudaError_t dispatch_scalar_out(ReduceParams& P, int kind, cudaStream_t s) {
  switch (kind) {
    case kLinear: return run_reduce<IN, CC_SUM, kLinear, true>(P, s);
    case kLinSmall: return run_reduce<IN, CC_SUM, kLinSmall, true>(P, s);
    case kHier: return run_reduce<IN, CC_SUM, kHier, true>(P, s);
    case kShallow: return run_reduce<IN, CC_SUM, kShallow, true>(P, s);
    case kMid: return run_reduce<IN, CC_SUM, kMid, true>(P, s);
    case kMachine: return run_reduce<IN, CC_SUM, kMachine, true>(P, s);
  }
  return cudaErrorInvalidValue;
}

// Linear folds over buffers without 16-byte units: the element-path kernel.
template <int IN>
static cudaError_t dispatch_elements(ReduceParams& P, cc_op op, cudaStream_t s) {
  switch (op) {
    case CC_SUM: return run_reduce<IN, CC_SUM, kLinear, false, true>(P, s);
    case CC_MAX: return run_reduce<IN, CC_MAX, kLinear, false, true>(P, s);
    case CC_MIN: return run_reduce<IN, CC_MIN, kLinear, false, true>(P, s);
    case CC_PROD: return run_reduce<IN, CC_PROD, kLinear, false, true>(P, s);
  }
  return cudaErrorInvalidValue;
}

template <int IN>
static cudaError_t dispatch_op(ReduceParams& P, cc_op op, int kind, cudaStream_t s) {
#define CC_KINDS(OPV)                                                                         \
  if (kind == kLinear) return run_reduce<IN, OPV, kLinear>(P, s);                         \
  if (kind == kLinSmall) return run_reduce<IN, OPV, kLinSmall>(P, s);                     \
  if (kind == kHier) return run_reduce<IN, OPV, kHier>(P, s);                             \
  if (kind == kShallow) return run_reduce<IN, OPV, kShallow>(P, s);                       \
  if (kind == kMid) return run_reduce<IN, OPV, kMid>(P, s);                               \
  return run_reduce<IN, OPV, kMachine>(P, s);
  switch (kind) {  // compiled binomial programs: SUM only (launch_reduce picks them for SUM)
    case kBinom4: return run_reduce<IN, CC_SUM, kBinom4>(P, s);
    case kBinom8: return run_reduce<IN, CC_SUM, kBinom8>(P, s);
    case kBinom16: return run_reduce<IN, CC_SUM, kBinom16>(P, s);
    case kBinom32: return run_reduce<IN, CC_SUM, kBinom32>(P, s);
    case kBinom64: return run_reduce<IN, CC_SUM, kBinom64>(P, s);
  }
  switch (op) {
    case CC_SUM: CC_KINDS(CC_SUM)
    case CC_MAX: CC_KINDS(CC_MAX)
    case CC_MIN: CC_KINDS(CC_MIN)
    case CC_PROD: CC_KINDS(CC_PROD)
  }
#undef CC_KINDS
  return cudaErrorInvalidValue;
}

// Deepest stack of pending partials a fold program reaches.
static int program_depth(int n, const FoldProgram& fp) {
  int d = 0, m = 0;
  for (int p = 0; p < n; ++p) {
    if (fp.code[p] & kPush) m = std::max(m, ++d);
    d -= npop_of(fp.code[p]);
  }
  return m;
}

cudaError_t launch_reduce(const void* const* send, void* const* dst, int ndst, int nranks, size_t count,
                          cc_dtype in_t, cc_op op, FoldKind fold, ReduceMode mode, int root, float scale,
                          cudaStream_t stream, size_t lo, size_t hi) {
  ReduceParams P{};
  P.count = count;
  P.hi = std::min<uint64_t>(hi, count);
  P.lo = std::min<uint64_t>(lo, P.hi);
  if (P.lo == P.hi) return cudaSuccess;
  P.nranks = nranks;
  P.mode = mode;
  P.fold = fold;
  P.scale = scale;
  P.do_scale = (in_t != CC_I32) && scale != 1.0f;
  // 16-byte units when every source sits at the same offset from a 16-byte boundary, a whole
  // number of elements (bf16 sources: aligned). The units then start `shift` elements past each
  // boundary. Allreduce / root outputs at that same offset (for equal element sizes; fp32
  // outputs of bf16 sources: aligned) take 16-byte stores; reduce-scatter shards are checked one
  // by one in the kernel. fp32 / int32 sums into outputs at another offset keep the units and
  // store element by element; other folds over such buffers take the element path.
  const size_t es_in = in_t == CC_BF16 ? 2 : 4;
  const uintptr_t m0 = reinterpret_cast<uintptr_t>(send[0]) & 15;
  bool src_vec = m0 % es_in == 0 && (m0 == 0 || es_in == 4);
  bool dst_vec = true;
  for (int r = 0; r < nranks; ++r) {
    P.src[r] = send[r];
    src_vec = src_vec && (reinterpret_cast<uintptr_t>(send[r]) & 15) == m0;
  }
  for (int r = 0; r < ndst; ++r) {
    P.dst[r] = dst[r];
    if (mode != kReduceScatter) dst_vec = dst_vec && (reinterpret_cast<uintptr_t>(dst[r]) & 15) == m0;
  }
  const bool scalar_out = src_vec && !dst_vec && op == CC_SUM && es_in == 4;
  const bool vec = src_vec && (dst_vec || scalar_out);
  P.vec = vec;
  P.shift = vec ? m0 / es_in : 0;
  P.lshift = vec ? (reinterpret_cast<uintptr_t>(send[0]) & 127) / es_in : 0;
  P.per_node = 1;
  if (fold == kFoldTree) tree_program(nranks, P.prog);
  else if (fold == kFoldBinomial) binomial_program(nranks, root, P.prog);
  else if (fold == kFoldHier || fold == kFoldMultiRing) P.per_node = root;
  // the ring, a tree whose fold is a plain left fold (N <= 5) and a binomial program that is
  // one (N <= 3, ranks in order from the root) run the linear fold; the hierarchical fold has
  // its own nested loop; other programs run the fold machine with the smallest stack that
  // holds their pending partials (more resident CTAs for smaller stacks)
  int kind = kMachine;
  if (fold == kFoldRing || fold == kFoldMultiRing || fold == kFoldHier) {
    kind = fold == kFoldHier ? kHier : kLinear;
  } else if (program_is_rotation(nranks, P.prog)) {
    kind = kLinear;
  } else {
    const int depth = program_depth(nranks, P.prog);
    if (depth > kStackSlots) return cudaErrorInvalidValue;  // not reached for N <= 64
    kind = depth <= 2 ? kShallow : depth <= 4 ? kMid : kMachine;
  }
  // two ranks give a thread only two loads per unit: fold four units at a time (measured at
  // N = 2 × 256 MiB: ring 5667 -> 6663 GB/s, reduce-scatter 5399 -> 6832; at N = 3..4 the
  // one-unit fold with 4 resident CTAs is faster)
  if (kind == kLinear && nranks == 2) kind = kLinSmall;
  // linear folds with no 16-byte units take the element-path kernel (several elements per
  // thread in flight)
  if (!vec && (kind == kLinear || kind == kLinSmall)) {
    switch (in_t) {
      case CC_F32: return dispatch_elements<CC_F32>(P, op, stream);
      case CC_BF16: return dispatch_elements<CC_BF16>(P, op, stream);
      case CC_I32: return dispatch_elements<CC_I32>(P, op, stream);
    }
    return cudaErrorInvalidValue;
  }
  // element stores: the runtime folds and the trees compiled for 8 and 16 ranks (binomial
  // programs run on the fold machine)
  if (scalar_out) {
    if (fold == kFoldTree && kind != kLinear && (nranks == 8 || nranks == 16))
      return run_reduce_tree_ct(P, in_t, nranks == 8 ? kTree8 : kTree16, stream, true);
    switch (in_t) {
      case CC_F32: return dispatch_scalar_out<CC_F32>(P, kind, stream);
      case CC_I32: return dispatch_scalar_out<CC_I32>(P, kind, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  // tree sums at 8 and 16 ranks run the tree compiled to straight-line code (as the bucket
  // kernel does); binomial sums at 4, 8, 16, 32, 64 ranks, and at every other rank count from
  // 5 to 15, their program compiled likewise (k_reduce_binom.cu holds the ones not here)
  if (fold == kFoldTree && op == CC_SUM && kind != kLinear && (nranks == 8 || nranks == 16))
    return run_reduce_tree_ct(P, in_t, nranks == 8 ? kTree8 : kTree16, stream);
  if (fold == kFoldBinomial && op == CC_SUM && kind != kLinear && nranks >= 4) {
    if ((nranks & (nranks - 1)) == 0) kind = kBinom4 + __builtin_ctz((unsigned)nranks) - 2;
    else if (nranks >= kBinomNLo && nranks <= kBinomNHi) return run_reduce_binom_np2(P, in_t, kBinomN0 + nranks, stream);
  }
  switch (in_t) {
    case CC_F32: return dispatch_op<CC_F32>(P, op, kind, stream);
    case CC_BF16: return dispatch_op<CC_BF16>(P, op, kind, stream);
    case CC_I32: return dispatch_op<CC_I32>(P, op, kind, stream);
  }
  return cudaErrorInvalidValue;
}

int bucket_group_limit(int nranks) {
  return std::max(1, std::min(kBucketMaxTensors, kBucketMaxPtrs / nranks));
}

int bucket_small_group_limit(int nranks) {
  return std::max(1, std::min(BucketParamsSmall::kMaxT, BucketParamsSmall::kMaxP / nranks));
}

template <typename PT>
static cudaError_t launch_bucket_with(PT& P, const void* const* grads, void* const* out, int nranks,
                                      int ntensors_total, const int32_t* ids, int nids, const BucketTensorDesc* desc,
                                      FoldKind fold, float scale, cudaStream_t stream) {
  P.nranks = nranks;
  P.ntensors = nids;
  P.fold = fold;
  P.scale = scale;
  P.do_scale = scale != 1.0f;
  bool vec = true;
  uint32_t tiles = 0;
  for (int k = 0; k < nids; ++k) {
    const int i = ids[k];
    P.t[k] = desc[i];
    P.tile_prefix[k] = tiles;
    tiles += (uint32_t)((desc[i].numel + kBucketTile - 1) / kBucketTile);
    for (int r = 0; r < nranks; ++r) {
      const void* g = grads[(size_t)r * ntensors_total + i];
      void* o = out[(size_t)r * ntensors_total + i];
      P.in[r * nids + k] = static_cast<const float*>(g);
      P.out[r * nids + k] = static_cast<float*>(o);
      vec = vec && aligned16(g) && aligned16(o);
    }
  }
  P.tile_prefix[nids] = tiles;
  P.vec = vec;
  if (fold == kFoldTree) tree_program(nranks, P.prog);
  if (tiles == 0) return cudaSuccess;
  const bool ring = fold == kFoldRing;
  // the ring; the tree compiled for 8 or 16 ranks; the fold machine for any other tree
  const int kind = ring ? kLinear : nranks == 8 ? kTree8 : nranks == 16 ? kTree16 : kMachine;
  auto k = kind == kLinear ? bucket_allreduce_kernel<kLinear, PT>
           : kind == kTree8 ? bucket_allreduce_kernel<kTree8, PT>
           : kind == kTree16 ? bucket_allreduce_kernel<kTree16, PT>
                             : bucket_allreduce_kernel<kMachine, PT>;
  static const int bps[4] = {blocks_per_sm(bucket_allreduce_kernel<kLinear, PT>),
                             blocks_per_sm(bucket_allreduce_kernel<kTree8, PT>),
                             blocks_per_sm(bucket_allreduce_kernel<kTree16, PT>),
                             blocks_per_sm(bucket_allreduce_kernel<kMachine, PT>)};
  const int b = bps[kind == kLinear ? 0 : kind == kTree8 ? 1 : kind == kTree16 ? 2 : 3];
  const uint32_t grid = std::min<uint32_t>(tiles, (uint32_t)(CC_BUCKET_OVERSUB * sm_count() * b));
  k<<<grid, kThreads, 0, stream>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_bucket_allreduce(const void* const* grads, void* const* out, int nranks, int ntensors_total,
                                    const int32_t* ids, int nids, const BucketTensorDesc* desc, FoldKind fold,
                                    float scale, cudaStream_t stream) {
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (nids <= BucketParamsSmall::kMaxT && nids * nranks <= BucketParamsSmall::kMaxP) {
    BucketParamsSmall P{};
    return launch_bucket_with(P, grads, out, nranks, ntensors_total, ids, nids, desc, fold, scale, stream);
  }
  static BucketParams P;  // large: kept off the stack
  return launch_bucket_with(P, grads, out, nranks, ntensors_total, ids, nids, desc, fold, scale, stream);
}

}  // namespace cc
