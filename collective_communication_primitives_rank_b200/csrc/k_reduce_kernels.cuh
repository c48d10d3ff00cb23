// Reduction kernels shared by k_reduce.cu and k_reduce_binom.cu: the folds over the N ranks,
// the chunk rule, the plain reduction kernel and its launcher. k_reduce.cu holds the host side
// (fold programs, kind selection, the bucket allreduce); k_reduce_binom.cu the binomial
// programs compiled for rank counts that are not powers of two, in a translation unit of its
// own so that the two compile in parallel.
#pragma once

#include <algorithm>
#include <mutex>
#include <vector>

#include "cc_device.cuh"
#include "cc_launch.h"

namespace cc {

constexpr int kThreads = 256;
// Grids are sized to one CTA per tile (capped at this many times the resident CTAs): with
// the hardware handing tiles to CTAs as earlier ones finish, DRAM stayed busier than with
// persistent CTAs looping over tiles (measured: 2x -> 93%, 8x -> 99.5%, one tile per CTA
// -> 101% of the copy rate on the DDP step).
#ifndef CC_REDUCE_OVERSUB
#define CC_REDUCE_OVERSUB 1024
#endif
#ifndef CC_RING_MIN_BLOCKS
#define CC_RING_MIN_BLOCKS 4  // resident 256-thread CTAs per SM the linear-fold kernel is compiled for
#endif
// The fold machines keep their pending partials in shared memory, so they fit the same
// register budget; measured against 3 (2- and 4-slot) and 2 (6-slot) resident CTAs:
// reduce N=8 6392 vs 5570 GB/s, N=64 5788 vs 4542, trees within 1.3%.
#ifndef CC_SHALLOW_MIN_BLOCKS
#define CC_SHALLOW_MIN_BLOCKS 4  // the same for the 2- and 4-slot fold machines
#endif
#ifndef CC_LINSMALL_MIN_BLOCKS
#define CC_LINSMALL_MIN_BLOCKS 3  // the same for the linear fold of 2 ranks, four units at once (80 registers, no spills)
#endif
#ifndef CC_MACHINE_MIN_BLOCKS
#define CC_MACHINE_MIN_BLOCKS 4  // the same for the 6-slot fold machine
#endif

// ---- folds over the N ranks ---------------------------------------------------------------------

// Left fold starting at rank c: loads go out in windows of 8 so that 8 independent
// 128-bit loads per thread are in flight before the in-order folds consume them.
// V is the accumulator (a unit or an element), X what one load returns (raw 16 bytes for a
// unit, the element itself otherwise).
// `up` false walks the ranks downwards (the left fold of a mirrored tree).
template <int IN, int OP, typename V, typename X, int W = 8, typename Load, typename Widen>
__device__ __forceinline__ V ring_fold(int n, int c, Load ld, Widen widen, bool up = true) {
  V acc = widen(ld(c));
  int r = c;
  for (int j0 = 1; j0 < n; j0 += W) {
    X x[W];
#pragma unroll
    for (int k = 0; k < W; ++k)
      if (j0 + k < n) {
        r = up ? (r + 1 == n ? 0 : r + 1) : (r == 0 ? n - 1 : r - 1);
        x[k] = ld(r);
      }
#pragma unroll
    for (int k = 0; k < W; ++k)
      if (j0 + k < n) comb<IN, OP>(acc, x[k]);
  }
  return acc;
}

// Fold machine (tree / binomial): position p holds rank rank_of(p); `st` is an empty stack
// of pending partials (registers or shared memory).
template <int IN, int OP, typename V, typename X, int W, typename St, typename RankOf, typename Load,
          typename Widen>
__device__ __forceinline__ V machine_fold(int n, const FoldProgram& prog, RankOf rank_of, Load ld, Widen widen,
                                          St& st) {
  V cur;
  st.depth = 0;
  for (int p0 = 0; p0 < n; p0 += W) {
    X x[W];
#pragma unroll
    for (int k = 0; k < W; ++k)
      if (p0 + k < n) x[k] = ld(rank_of(p0 + k));
#pragma unroll
    for (int k = 0; k < W; ++k)
      if (p0 + k < n) fold_step<IN, OP>(prog.code[p0 + k], widen(x[k]), cur, st);
  }
  return cur;
}

// Hierarchical fold: node by node, starting at node j, each node's G ranks left-folded
// starting at local rank c (windows of 8 loads), the node sums left-folded in node order.
template <int IN, int OP, typename V, typename X, typename Load, typename Widen>
__device__ __forceinline__ V hier_fold(int n, int G, int c, int j, Load ld, Widen widen) {
  const int M = n / G;
  V outer;
  int m = j;
  for (int k = 0; k < M; ++k) {
    const int base = m * G;
    V inner = widen(ld(base + c));
    int l = c;
    for (int i0 = 1; i0 < G; i0 += 8) {
      X x[8];
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (i0 + q < G) {
          l = (l + 1 == G) ? 0 : l + 1;
          x[q] = ld(base + l);
        }
#pragma unroll
      for (int q = 0; q < 8; ++q)
        if (i0 + q < G) comb<IN, OP>(inner, x[q]);
    }
    if (k == 0) outer = inner;
    else comb<IN, OP>(outer, inner);
    m = (m + 1 == M) ? 0 : m + 1;
  }
  return outer;
}


// Elements [a, b) of one fold group, spread over threads t = 0..T-1: 16-byte units where
// every address is aligned, element-wise head and tail around them. Each thread folds one
// unit at a time (consecutive threads take consecutive units, so warps stay coalesced) with
// windows of 8 positions: up to 8 loads in flight per thread.
// Linear fold of NU units at once (T·UE elements apart, so warps stay coalesced) for small
// rank counts (n <= NR): all n·NU loads are issued before the first fold, so a thread keeps
// about 8 loads in flight where one unit alone would give it only n. Same order as
// ring_fold: rank `start` first, then walking up (or down).
template <int IN, int OP, int NR, int NU, typename Src, typename EmitU>
__device__ __forceinline__ void linear_fold_units(int n, int start, bool up, uint64_t e0, uint64_t step,
                                                  uint64_t vb, Src src, EmitU emit_unit) {
  uint4 x[NU][NR];
  int r = start;
#pragma unroll
  for (int k = 0; k < NR; ++k) {
    if (k < n) {
#pragma unroll
      for (int i = 0; i < NU; ++i)
        if (e0 + i * step < vb) x[i][k] = load_raw(src(r) + e0 + i * step);
      r = up ? (r + 1 == n ? 0 : r + 1) : (r == 0 ? n - 1 : r - 1);
    }
  }
#pragma unroll
  for (int i = 0; i < NU; ++i) {
    if (e0 + i * step < vb) {
      Unit<IN> m = to_unit<IN>(x[i][0]);
#pragma unroll
      for (int k = 1; k < NR; ++k)
        if (k < n) comb<IN, OP>(m, x[i][k]);
      emit_unit(e0 + i * step, m);
    }
  }
}

// Binomial reduce programs compiled for a fixed rank count: the pre-order walk of the
// binomial tree (relative rank v; children v + 2^k for every 2^k > v, in send order) with the
// fold-machine code of every position, computed at compile time, so that a fully unrolled
// fold resolves every code and keeps the pending partials in registers. The same walk and
// codes as binomial_program() below builds at run time for any rank count.
template <int NB> struct BinomialPlan {
  uint8_t order[NB];
  uint8_t code[NB];
  int depth;
  constexpr BinomialPlan() : order(), code(), depth(0) {
    int stack[NB] = {};
    int sp = 0, pos = 0;
    stack[sp++] = 0;
    while (sp > 0) {
      const int v = stack[--sp];
      order[pos++] = (uint8_t)v;
      int k = 0;
      if (v) while ((1 << k) <= v) ++k;
      int ch[8] = {}, nch = 0;
      for (; v + (1 << k) < NB; ++k) ch[nch++] = v + (1 << k);
      for (int c = nch - 1; c >= 0; --c) stack[sp++] = ch[c];
    }
    int d = 0;
    for (int p = 0; p < NB; ++p) {
      const int v = order[p];
      int k = 0;
      if (v) while ((1 << k) <= v) ++k;
      const bool leaf = !(v + (1 << k) < NB);
      uint8_t c = 0;
      if (!leaf) {
        c = kPush;
        if (++d > depth) depth = d;
      } else {
        int npop = 0, u = v;
        while (u != 0) {
          int hb = 0;
          while ((2 << hb) <= u) ++hb;
          const int par = u - (1 << hb);
          int kk = 0;
          if (par) while ((1 << kk) <= par) ++kk;
          int last = -1;
          for (; par + (1 << kk) < NB; ++kk) last = par + (1 << kk);
          if (last == u) { ++npop; u = par; continue; }
          c |= kFoldTop;
          break;
        }
        c |= (uint8_t)(npop << 2);
        d -= npop;
      }
      code[p] = c;
    }
  }
};

// NU units (or elements) at once, each folded over the NB ranks in the compiled binomial
// order from `root`: the loads of a window of 8 positions of every unit go out before the
// folds that consume them.
template <int IN, int OP, int NB, int NU, typename V, typename X, typename Load, typename Widen>
__device__ __forceinline__ void binomial_fold_ct(int root, Load ld, Widen widen, V (&cur)[NU]) {
  constexpr BinomialPlan<NB> plan{};
  constexpr int S = plan.depth > 0 ? plan.depth : 1;
  FoldStack<V, S> st[NU];
#pragma unroll
  for (int i = 0; i < NU; ++i) st[i].depth = 0;
#pragma unroll
  for (int p0 = 0; p0 < NB; p0 += 8) {
    X x[NU][8];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (p0 + k < NB) {
        int r = plan.order[p0 + k] + root;
        if (r >= NB) r -= NB;
#pragma unroll
        for (int i = 0; i < NU; ++i) x[i][k] = ld(i, r);
      }
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (p0 + k < NB)
#pragma unroll
        for (int i = 0; i < NU; ++i) fold_step<IN, OP>(plan.code[p0 + k], widen(x[i][k]), cur[i], st[i]);
  }
}

// Double-binary-tree programs compiled for a fixed rank count: tree A in the in-order
// labelling (position p = rank p, node q = p + 1: a node of height h > 0 has the left child
// q - 2^(h-1) and as right child the first of q + 2^(j-1), j = h..1, that exists), with the
// fold-machine code of every position and the same leaf merge as tree_program() below; tree B
// is the mirror (position p = rank N-1-p). Computed at compile time, so that a fully unrolled
// fold resolves every code and keeps the pending partials in registers.
template <int NT> struct TreePlan {
  uint8_t code[NT];
  int depth;
  constexpr TreePlan() : code(), depth(0) {
    int left[NT + 2] = {}, right[NT + 2] = {}, parent[NT + 2] = {};
    bool is_right[NT + 2] = {};
    for (int q = 1; q <= NT; ++q) {
      int h = 0;
      while (!((q >> h) & 1)) ++h;
      if (h == 0) continue;
      const int lq = q - (1 << (h - 1));
      left[q] = lq;
      parent[lq] = q;
      for (int j = h; j >= 1; --j) {
        const int rq = q + (1 << (j - 1));
        if (rq <= NT) {
          right[q] = rq;
          parent[rq] = q;
          is_right[rq] = true;
          break;
        }
      }
    }
    for (int p = 0; p < NT; ++p) {
      const int q = p + 1;
      uint8_t c = left[q] ? kFoldCur : 0;
      if (right[q]) {
        c |= kPush;
      } else {
        int npop = 0, u = q;
        while (parent[u] && is_right[u]) { ++npop; u = parent[u]; }
        c |= (uint8_t)(npop << 2);
      }
      code[p] = c;
    }
    for (int p = 0; p + 1 < NT; ++p) {
      const int q = p + 1;
      if (right[q] == q + 1 && (code[p] & kPush) && npop_of(code[p + 1]) > 0) {
        code[p] &= (uint8_t)~kPush;
        const int np = npop_of(code[p + 1]) - 1;
        code[p + 1] = (uint8_t)((code[p + 1] & ~(7 << 2)) | kFoldCur | (np << 2));
      }
    }
    int d = 0;
    for (int p = 0; p < NT; ++p) {
      if (code[p] & kPush)
        if (++d > depth) depth = d;
      d -= npop_of(code[p]);
    }
  }
};

// One unit (or element) folded over the NT ranks in the compiled tree order, every load
// issued before the first fold; `mirror` selects tree B.
template <int IN, int OP, int NT, typename V, typename X, typename Load, typename Widen>
__device__ __forceinline__ V tree_fold_ct(bool mirror, Load ld, Widen widen) {
  constexpr TreePlan<NT> plan{};
  constexpr int S = plan.depth > 0 ? plan.depth : 1;
  FoldStack<V, S> st;
  st.depth = 0;
  X x[NT];
#pragma unroll
  for (int p = 0; p < NT; ++p) x[p] = ld(mirror ? NT - 1 - p : p);
  V cur;
#pragma unroll
  for (int p = 0; p < NT; ++p) fold_step<IN, OP>(plan.code[p], widen(x[p]), cur, st);
  return cur;
}

// KIND: kLinear (ring order or a linear tree), kMachine (tree / binomial programs),
// kHier (two-level), kShallow / kMid (the fold machine with 2 / 4 stack slots, for programs
// that never hold more pending partials), kLinSmall (the linear fold of 2 ranks, four units
// per iteration); hG / hc / hj describe the hierarchical group.
constexpr int kLinear = 0, kMachine = 1, kHier = 2, kShallow = 3, kMid = 4, kLinSmall = 5;
// binomial programs compiled for 4, 8, 16, 32, 64 ranks (SUM only): kBinom4 + log2(N / 4)
constexpr int kBinom4 = 10, kBinom8 = 11, kBinom16 = 12, kBinom32 = 13, kBinom64 = 14;
// and for the other rank counts from 5 to 15: kBinomN0 + N (k_reduce_binom.cu)
constexpr int kBinomN0 = 40, kBinomNLo = 5, kBinomNHi = 15;
__host__ __device__ constexpr bool is_binom_ct(int kind) {
  return (kind >= kBinom4 && kind <= kBinom64) || (kind >= kBinomN0 + kBinomNLo && kind <= kBinomN0 + kBinomNHi);
}
__host__ __device__ constexpr int binom_ct_ranks(int kind) {
  return kind >= kBinomN0 ? kind - kBinomN0 : 4 << (kind - kBinom4);
}
// units folded at once: about 16 loads in flight per thread for the small rank counts
__host__ __device__ constexpr int binom_ct_units(int kind) {
  return binom_ct_ranks(kind) <= 4 ? 4 : binom_ct_ranks(kind) <= 8 ? 2 : 1;
}
// double-binary-tree programs compiled for 8 and 16 ranks (the bucket allreduce)
constexpr int kTree8 = 20, kTree16 = 21;
__host__ __device__ constexpr bool is_tree_ct(int kind) { return kind == kTree8 || kind == kTree16; }
__host__ __device__ constexpr int tree_ct_ranks(int kind) { return kind == kTree8 ? 8 : 16; }

template <int IN, int OP, int KIND, bool EL = false, typename RankOf, typename Src, typename EmitU, typename EmitE>
__device__ __forceinline__ void reduce_range(int n, int g, RankOf rank_of, const FoldProgram& prog,
                                             uint64_t a, uint64_t b, uint64_t t, uint64_t T, bool vec,
                                             Src src, EmitU emit_unit, EmitE emit_elem, uint4* stk,
                                             int start = 0, bool up = true, int hG = 1, int hc = 0, int hj = 0,
                                             uint64_t shift = 0) {
  constexpr bool RING = KIND == kLinear || KIND == kLinSmall;
  constexpr int SLOTS = KIND == kShallow ? 2 : KIND == kMid ? 4 : kStackSlots;
  using A = typename Tr<IN>::Acc;
  constexpr int UE = Tr<IN>::UE;
  auto same = [](const A& x) { return x; };
  // a linear fold starts at rank `start` and walks up (or down) the ranks
  auto fold_elem = [&](uint64_t e) -> A {
    auto ld = [&](int r) { return load_elem<IN>(src(r) + e); };
    if constexpr (RING) return ring_fold<IN, OP, A, A>(n, start, ld, same, up);
    else if constexpr (KIND == kHier) return hier_fold<IN, OP, A, A>(n, hG, hc, hj, ld, same);
    else if constexpr (is_binom_ct(KIND)) {
      A cur[1];
      binomial_fold_ct<IN, OP, binom_ct_ranks(KIND), 1, A, A>(start, [&](int, int r) { return ld(r); }, same, cur);
      return cur[0];
    }
    else if constexpr (is_tree_ct(KIND)) return tree_fold_ct<IN, OP, tree_ct_ranks(KIND), A, A>(start != 0, ld, same);
    else {
      FoldStack<A, SLOTS> st;
      return machine_fold<IN, OP, A, A, 8>(n, prog, rank_of, ld, same, st);
    }
  };
  if constexpr (EL) {
    // element-path kernel (no 16-byte units: sources at unequal offsets, bf16 off a boundary,
    // or other folds over unequally placed buffers): a linear fold keeps NE elements per thread
    // (T apart) in flight, each window of W ranks loaded for all of them before it is folded
    // in, in the same order per element as ring_fold
    static_assert(RING, "the element-path kernel takes the linear folds");
    constexpr int NE = 4, W = 4;
    for (uint64_t e0 = a + t; e0 < b; e0 += NE * T) {
      A acc[NE];
      int r = start;
#pragma unroll
      for (int q = 0; q < NE; ++q)
        if (e0 + q * T < b) acc[q] = load_elem<IN>(src(r) + e0 + q * T);
      for (int j0 = 1; j0 < n; j0 += W) {
        A x[W][NE];
#pragma unroll
        for (int k = 0; k < W; ++k) {
          const int rk = up ? (r + 1 + k) % n : ((r - 1 - k) % n + n) % n;
          if (j0 + k < n) {
#pragma unroll
            for (int q = 0; q < NE; ++q)
              if (e0 + q * T < b) x[k][q] = load_elem<IN>(src(rk) + e0 + q * T);
          }
        }
#pragma unroll
        for (int k = 0; k < W; ++k)
          if (j0 + k < n) {
#pragma unroll
            for (int q = 0; q < NE; ++q)
              if (e0 + q * T < b) acc[q] = op<IN, OP, A>(acc[q], x[k][q]);
          }
        r = up ? (r + W) % n : ((r - W) % n + n) % n;
      }
#pragma unroll
      for (int q = 0; q < NE; ++q)
        if (e0 + q * T < b) emit_elem(e0 + q * T, acc[q]);
    }
  } else if (vec) {
    // 16-byte units start where (e + shift) is a multiple of UE: every buffer sits `shift`
    // elements past a 16-byte boundary (0 when aligned)
    uint64_t va = a + (UE - (a + shift) % UE) % UE;
    if (va > b) va = b;
    const uint64_t vbs = (b + shift) / UE * UE;  // the last unit boundary, in shifted coordinates
    uint64_t vb = vbs >= shift ? vbs - shift : 0;
    if (vb < va) vb = va;
    const uint64_t step = T * UE;
    auto widen = [](const uint4& x) { return to_unit<IN>(x); };
    bool done = false;
    if constexpr (KIND == kLinSmall) {  // two ranks: four units per iteration
      for (uint64_t e0 = va + t * UE; e0 < vb; e0 += 4 * step)
        linear_fold_units<IN, OP, 2, 4>(n, start, up, e0, step, vb, src, emit_unit);
      done = true;
    }
    if constexpr (is_binom_ct(KIND)) {  // compiled binomial program, NU units per iteration
      constexpr int NU = binom_ct_units(KIND);
      for (uint64_t e0 = va + t * UE; e0 < vb; e0 += NU * step) {
        // a unit past vb re-reads the last whole unit and is not emitted
        auto ld = [&](int i, int r) {
          const uint64_t e = e0 + i * step < vb ? e0 + i * step : vb - UE;
          return load_raw(src(r) + e);
        };
        Unit<IN> m[NU];
        binomial_fold_ct<IN, OP, binom_ct_ranks(KIND), NU, Unit<IN>, uint4>(start, ld, widen, m);
#pragma unroll
        for (int i = 0; i < NU; ++i)
          if (e0 + i * step < vb) emit_unit(e0 + i * step, m[i]);
      }
      done = true;
    }
    for (uint64_t e0 = va + t * UE; !done && e0 < vb; e0 += step) {
      auto ld = [&](int r) { return load_raw(src(r) + e0); };
      Unit<IN> m;
      if constexpr (RING) m = ring_fold<IN, OP, Unit<IN>, uint4>(n, start, ld, widen, up);
      else if constexpr (KIND == kHier) m = hier_fold<IN, OP, Unit<IN>, uint4>(n, hG, hc, hj, ld, widen);
      else if constexpr (is_tree_ct(KIND)) m = tree_fold_ct<IN, OP, tree_ct_ranks(KIND), Unit<IN>, uint4>(start != 0, ld, widen);
      else {
        SmemStack<IN> st{stk, (int)T};
        m = machine_fold<IN, OP, Unit<IN>, uint4, 8>(n, prog, rank_of, ld, widen, st);
      }
      emit_unit(e0, m);
    }
    const uint64_t nh = va - a, nt = b - vb;
    if (t < nh) emit_elem(a + t, fold_elem(a + t));
    else if (t < nh + nt) emit_elem(vb + (t - nh), fold_elem(vb + (t - nh)));
  } else {
    for (uint64_t e = a + t; e < b; e += T) emit_elem(e, fold_elem(e));
  }
}

// ---- chunk rule ---------------------------------------------------------------------------------
// q = count / n, r = count % n; chunk c has q + (c < r) elements, starting at c*q + min(c, r).

__host__ __device__ __forceinline__ void chunk_range(uint64_t count, int n, int c, uint64_t& a, uint64_t& b) {
  const uint64_t q = count / n, r = count % n, cc_ = (uint64_t)c;
  a = cc_ * q + (cc_ < r ? cc_ : r);
  b = a + q + (cc_ < r ? 1 : 0);
}

// Chunk of element o and that chunk's [start, end).
__device__ __forceinline__ int chunk_of(uint64_t count, int n, uint64_t o, uint64_t& start, uint64_t& end) {
  const uint64_t q = count / n, r = count % n;
  const uint64_t big = r * (q + 1);
  if (o < big) {
    const uint64_t c = o / (q + 1);
    start = c * (q + 1);
    end = start + q + 1;
    return (int)c;
  }
  const uint64_t c = r + (o - big) / q;
  start = big + (c - r) * q;
  end = start + q;
  return (int)c;
}

// The fold group of element o in a buffer of `count` elements: the ring chunk, the tree
// half, the (part, chunk) pair of the multi-ring, or the single binomial group; returns the
// group and its [start, end).
__device__ __forceinline__ int group_of(int fold, uint64_t count, int n, uint64_t o, uint64_t& start,
                                        uint64_t& end, int per_node = 1) {
  if (fold == kFoldRing) return chunk_of(count, n, o, start, end);
  if (fold == kFoldHier) {
    // local chunk c of the node's G-way split, then sub-chunk j of that chunk's M-way split
    const int G = per_node, M = n / per_node;
    uint64_t ca, cb, ja, jb;
    const int c = chunk_of(count, G, o, ca, cb);
    const int j = chunk_of(cb - ca, M, o - ca, ja, jb);
    start = ca + ja;
    end = ca + jb;
    return c * M + j;
  }
  if (fold == kFoldMultiRing) {
    // part k of the K rings' split, then chunk c of that part's N-way split; group k * n + c
    const int K = per_node;
    uint64_t pa, pb, ca, cb;
    const int k = chunk_of(count, K, o, pa, pb);
    const int c = chunk_of(pb - pa, n, o - pa, ca, cb);
    start = pa + ca;
    end = pa + cb;
    return k * n + c;
  }
  if (fold == kFoldTree) {
    const uint64_t mid = (count + 1) / 2;
    const int g = o >= mid;
    start = g ? mid : 0;
    end = g ? count : mid;
    return g;
  }
  start = 0;
  end = count;
  return 0;
}

// ---- plain reduction kernel ------------------------------------------------------------------------

struct ReduceParams {
  const void* src[kMaxRanks];
  void* dst[kMaxRanks];
  FoldProgram prog;
  uint64_t count;
  uint64_t lo, hi;       // the elements this launch folds: [lo, hi) of the count
  uint64_t tile;         // elements per tile (a multiple of 8, or one fold group of fewer than 8)
  uint64_t skew;         // tile k >= 1 starts at lo + k * tile - skew (the first tile is that much shorter)
  uint64_t lshift;       // elements the first source sits past a 128-byte line (16-byte units only)
  uint64_t shift;        // elements every source (and allreduce / root output) sits past a 16-byte boundary
  int nranks;
  int per_node;  // ranks per node (hierarchical fold)
  int mode;
  int fold;
  int vec;  // every source sits `shift` elements past a 16-byte boundary (and so does every
            // allreduce / root output, unless the kernel stores element by element)
  float scale;
  int do_scale;
};

// Each CTA folds contiguous tiles (normally exactly one: the grid is sized to the tile
// count); a tile is split where it crosses a fold group (ring chunk or tree half) and each
// piece is folded by the whole CTA.
// SS: the units follow the sources and the allreduce / root outputs, which sit at another
// offset from a 16-byte boundary, take four element stores per unit (fp32 / int32), as
// reduce-scatter shards that the units meet off a boundary always do.
template <int IN, int OP, int KIND, bool SS = false, bool EL = false>
__global__ void __launch_bounds__(kThreads, KIND == kLinear ? CC_RING_MIN_BLOCKS
                                           : KIND == kLinSmall ? CC_LINSMALL_MIN_BLOCKS
                                           : is_binom_ct(KIND) ? (binom_ct_units(KIND) > 1 ? 2 : KIND == kBinom64 ? 3 : 4)
                                           : KIND == kHier ? 3
                                           : KIND == kShallow || KIND == kMid ? CC_SHALLOW_MIN_BLOCKS
                                                                              : CC_MACHINE_MIN_BLOCKS)
    reduce_kernel(const __grid_constant__ ReduceParams P) {
  // the fold machines' pending partials, one column of 16-byte words per thread
  constexpr int kSlots = KIND == kShallow ? 2 : KIND == kMid ? 4 : KIND == kMachine ? kStackSlots : 0;
  __shared__ uint4 s_stk[kSlots > 0 ? kSlots * (int)(sizeof(Unit<IN>) / 16) * kThreads : 1];
  using In = typename Tr<IN>::In;
  using Out = typename Tr<IN>::Out;
  using A = typename Tr<IN>::Acc;
  const int n = P.nranks;
  const int mode = P.mode;
  const uint64_t ntiles = (P.hi - P.lo + P.skew + P.tile - 1) / P.tile;
  auto src = [&](int r) { return static_cast<const In*>(P.src[r]); };
  for (uint64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    const uint64_t ea = tile == 0 ? P.lo : P.lo + tile * P.tile - P.skew;
    const uint64_t eb = min(P.lo + (tile + 1) * P.tile - P.skew, P.hi);
    uint64_t s = ea;
    while (s < eb) {
      uint64_t ga, gb;
      const int g = group_of(P.fold, P.count, n, s, ga, gb, P.per_node);
      const uint64_t se = min(eb, gb);
      const bool mirror = (P.fold == kFoldTree && g == 1);
      const int G = P.per_node, M = n / P.per_node, hc = g / M, hj = g % M;
      auto rank_of = [&](int p) {
        const int rk = P.prog.rmap[p];
        return mirror ? n - 1 - rk : rk;
      };
      // a shard takes whole-unit stores when its element under the group's first unit is aligned
      constexpr uint64_t UEk = Tr<IN>::UE;
      const uint64_t first_unit = ga + (UEk - (ga + P.shift) % UEk) % UEk;
      const bool shard_vec = mode == kReduceScatter &&
                             ((reinterpret_cast<uintptr_t>(static_cast<Out*>(P.dst[g]) + (first_unit - ga)) & 15) == 0);
      auto emit_unit = [&](uint64_t e, Unit<IN> u) {
        if (P.do_scale) scale_unit<IN>(u, P.scale);
        if (mode == kAllReduce) {
          for (int r = 0; r < n; ++r) {
            if constexpr (SS) store_unit_scalar<IN>(static_cast<Out*>(P.dst[r]) + e, u);
            else store_unit<IN>(static_cast<Out*>(P.dst[r]) + e, u);
          }
        } else if (mode == kReduceScatter) {
          Out* d = static_cast<Out*>(P.dst[g]) + (e - ga);
          if (shard_vec) store_unit<IN>(d, u); else store_unit_scalar<IN>(d, u);
        } else if constexpr (SS) {
          store_unit_scalar<IN>(static_cast<Out*>(P.dst[0]) + e, u);
        } else {
          store_unit<IN>(static_cast<Out*>(P.dst[0]) + e, u);
        }
      };
      auto emit_elem = [&](uint64_t e, A v) {
        if constexpr (IN != CC_I32) if (P.do_scale) v = __fmul_rn(v, P.scale);
        if (mode == kAllReduce) {
          for (int r = 0; r < n; ++r) store_elem<IN>(static_cast<Out*>(P.dst[r]) + e, v);
        } else if (mode == kReduceScatter) {
          store_elem<IN>(static_cast<Out*>(P.dst[g]) + (e - ga), v);
        } else {
          store_elem<IN>(static_cast<Out*>(P.dst[0]) + e, v);
        }
      };
      // linear folds: a ring chunk starts at rank g and walks up; a multi-ring chunk (group
      // k * n + c) starts at rank c and walks up for even k, down for odd k; a linear tree
      // (g = 0 or 1 for tree A / B) starts at rank 0 and walks up, or at rank n-1 and walks
      // down; a linear binomial program starts at the root and walks up
      const int lstart = P.fold == kFoldRing ? g
                         : P.fold == kFoldMultiRing ? g % n
                         : P.fold == kFoldTree ? (g == 0 ? 0 : n - 1) : P.prog.rmap[0];
      const bool lup = P.fold == kFoldMultiRing ? ((g / n) % 2 == 0) : (P.fold != kFoldTree || g == 0);
      reduce_range<IN, OP, KIND, EL>(n, g, rank_of, P.prog, s, se, threadIdx.x, blockDim.x, P.vec != 0, src,
                                    emit_unit, emit_elem, s_stk + threadIdx.x, lstart, lup, G, hc, hj, P.shift);
      s = se;
    }
  }
}

template <typename K>
static int blocks_per_sm(K kernel) {
  int b = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, kThreads, 0) != cudaSuccess || b <= 0) b = 2;
  return b;
}

template <int IN, int OP, int KIND, bool SS = false, bool EL = false>
static cudaError_t run_reduce(ReduceParams& P, cudaStream_t s) {
  auto k = reduce_kernel<IN, OP, KIND, SS, EL>;
  static const int bps = blocks_per_sm(k);
  constexpr uint64_t UE = Tr<IN>::UE;
  const uint64_t resident = (uint64_t)sm_count() * bps;
  // a tile never spans much more than one fold group, so that the groups of a small
  // buffer (N ring chunks of a few elements each) are folded by different CTAs in parallel
  const uint64_t ngroups = P.fold == kFoldRing ? (uint64_t)P.nranks
                           : P.fold == kFoldTree ? 2
                           : P.fold == kFoldHier ? (uint64_t)P.nranks
                           : P.fold == kFoldMultiRing ? (uint64_t)P.nranks * P.per_node : 1;
  // (groups of fewer than 8 elements keep their own size: a tile that spans several of them
  // folds them one after another, each a dependent round trip)
  const uint64_t gsz = (P.count + ngroups - 1) / ngroups;
  const uint64_t per_group = gsz < 8 ? gsz : (gsz + 7) / 8 * 8;
  // units per thread and tile (measured): the linear folds (ring, linear tree, hierarchical)
  // run best with about 24 memory operations per thread and CTA (a unit costs N loads plus
  // N stores for allreduce, one store otherwise), the small-stack tree machines with 16 / N
  // units, the binomial and deep-stack machines with 8: many short-lived CTAs keep more
  // loads in flight than long per-CTA streams. Small buffers take fewer, so that every
  // resident CTA gets a tile.
  const int ops = P.mode == kAllReduce ? 2 * P.nranks : P.nranks + 1;
  const uint64_t target = (KIND == kMachine || P.fold == kFoldBinomial) ? 8
                          : KIND == kLinSmall ? 8  // two iterations of four units
                          : (KIND == kLinear || KIND == kHier) ? (uint64_t)std::max(1, std::min(8, 24 / ops))
                          : (uint64_t)std::max(1, std::min(8, 16 / P.nranks));
  const uint64_t units = (P.hi - P.lo + UE - 1) / UE;
  const uint64_t upt = std::max<uint64_t>(1, std::min<uint64_t>(target, units / (resident * kThreads)));
  P.tile = std::max<uint64_t>(1, std::min<uint64_t>(upt * kThreads * UE, per_group));
  // tiles after the first start on a 128-byte line of the first source (and of the others
  // that share its offset modulo 128 bytes), so that each warp's 512 bytes per buffer fill four
  // whole lines when the buffers sit off a line; aligned buffers keep skew 0
  constexpr uint64_t L = 128 / sizeof(typename Tr<IN>::In);
  P.skew = (P.vec && P.tile % L == 0) ? (P.lo + P.lshift) % L : 0;
  const uint64_t ntiles = (P.hi - P.lo + P.skew + P.tile - 1) / P.tile;
  const uint64_t grid = std::max<uint64_t>(1, std::min<uint64_t>(ntiles, CC_REDUCE_OVERSUB * resident));
  k<<<(unsigned)grid, kThreads, 0, s>>>(P);
  return cudaGetLastError();
}

// The binomial SUM programs compiled for 5..7 and 9..15 ranks (k_reduce_binom.cu); `kind` is
// kBinomN0 + N.
cudaError_t run_reduce_binom_np2(ReduceParams& P, cc_dtype in_t, int kind, cudaStream_t s);
// The double-binary-tree SUM programs compiled for 8 and 16 ranks (k_reduce_binom.cu); `kind`
// is kTree8 or kTree16; `scalar_out`: outputs stored element by element (fp32 / int32).
cudaError_t run_reduce_tree_ct(ReduceParams& P, cc_dtype in_t, int kind, cudaStream_t s, bool scalar_out = false);

}  // namespace cc
