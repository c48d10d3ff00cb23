// Device-side building blocks of the collective kernels: element traits, the four
// reduction operators, 128-bit streaming loads/stores, and the fold machine that
// evaluates one element's reduction in a schedule's order.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/cc.h"

namespace cc {

constexpr int kMaxRanks = CC_MAX_RANKS;
constexpr int kStackSlots = 6;   // pending partials of a fold program (binomial N = 64 needs 6, trees <= 4)

// ---- reduction operators (one binary32 / int32 operation, never contracted) ----------------

// Order on binary32 values with -0 below +0 (inputs are never NaN).
__device__ __forceinline__ bool less_f(float a, float b) {
  return a < b || (a == b && __float_as_int(a) < 0 && __float_as_int(b) >= 0);
}

template <int OP> __device__ __forceinline__ float op_f(float a, float b) {
  if constexpr (OP == CC_SUM) return __fadd_rn(a, b);
  else if constexpr (OP == CC_PROD) return __fmul_rn(a, b);
  else if constexpr (OP == CC_MAX) return less_f(a, b) ? b : a;
  else return less_f(b, a) ? b : a;
}

template <int OP> __device__ __forceinline__ int op_i(int a, int b) {
  if constexpr (OP == CC_SUM) return (int)((unsigned)a + (unsigned)b);
  else if constexpr (OP == CC_PROD) return (int)((unsigned)a * (unsigned)b);
  else if constexpr (OP == CC_MAX) return a < b ? b : a;
  else return b < a ? b : a;
}

// ---- element traits ---------------------------------------------------------------------------
// UE = elements per 16-byte input vector (the unit one thread moves per rank).

template <int IN> struct Tr;
template <> struct Tr<CC_F32> { using In = float; using Acc = float; using Out = float; static constexpr int UE = 4; };
template <> struct Tr<CC_BF16> { using In = uint16_t; using Acc = float; using Out = float; static constexpr int UE = 8; };
template <> struct Tr<CC_I32> { using In = int32_t; using Acc = int32_t; using Out = int32_t; static constexpr int UE = 4; };

template <int IN, int OP, typename A> __device__ __forceinline__ A op(A a, A b) {
  if constexpr (IN == CC_I32) return op_i<OP>(a, b);
  else return op_f<OP>(a, b);
}

template <int IN> struct Unit { typename Tr<IN>::Acc v[Tr<IN>::UE]; };

// 16-byte streaming load (evict-first: every input byte is read once), kept as raw bits
// until it is folded, so that a window of loads in flight costs 4 registers per load for
// every dtype.
__device__ __forceinline__ uint4 load_raw(const void* p) { return __ldcs(reinterpret_cast<const uint4*>(p)); }

// The raw 16 bytes as one unit of accumulator values (bf16 widens exactly: bits << 16).
template <int IN> __device__ __forceinline__ Unit<IN> to_unit(const uint4& w) {
  Unit<IN> u;
  if constexpr (IN == CC_F32) {
    u.v[0] = __uint_as_float(w.x); u.v[1] = __uint_as_float(w.y);
    u.v[2] = __uint_as_float(w.z); u.v[3] = __uint_as_float(w.w);
  } else if constexpr (IN == CC_I32) {
    u.v[0] = (int)w.x; u.v[1] = (int)w.y; u.v[2] = (int)w.z; u.v[3] = (int)w.w;
  } else {
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      u.v[2 * i] = __uint_as_float(ws[i] << 16);             // element 2i (low half)
      u.v[2 * i + 1] = __uint_as_float(ws[i] & 0xFFFF0000u); // element 2i+1
    }
  }
  return u;
}

template <int IN> __device__ __forceinline__ Unit<IN> load_unit(const typename Tr<IN>::In* p) {
  return to_unit<IN>(load_raw(p));
}

template <int IN> __device__ __forceinline__ typename Tr<IN>::Acc load_elem(const typename Tr<IN>::In* p) {
  if constexpr (IN == CC_BF16) return __uint_as_float(((uint32_t)__ldcs(reinterpret_cast<const unsigned short*>(p))) << 16);
  else return __ldcs(p);
}

// Streaming store of one unit of outputs (UE elements of Out; 16 or 32 bytes).
template <int IN> __device__ __forceinline__ void store_unit(typename Tr<IN>::Out* p, const Unit<IN>& u) {
  if constexpr (IN == CC_I32) {
    __stcs(reinterpret_cast<int4*>(p), make_int4(u.v[0], u.v[1], u.v[2], u.v[3]));
  } else {
#pragma unroll
    for (int i = 0; i < Tr<IN>::UE; i += 4)
      __stcs(reinterpret_cast<float4*>(p + i), make_float4(u.v[i], u.v[i + 1], u.v[i + 2], u.v[i + 3]));
  }
}

template <int IN> __device__ __forceinline__ void store_unit_scalar(typename Tr<IN>::Out* p, const Unit<IN>& u) {
#pragma unroll
  for (int i = 0; i < Tr<IN>::UE; ++i) __stcs(p + i, u.v[i]);
}

template <int IN> __device__ __forceinline__ void store_elem(typename Tr<IN>::Out* p, typename Tr<IN>::Acc v) {
  __stcs(p, v);
}

template <int IN, int OP> __device__ __forceinline__ void op_unit(Unit<IN>& a, const Unit<IN>& b) {
#pragma unroll
  for (int i = 0; i < Tr<IN>::UE; ++i) a.v[i] = op<IN, OP>(a.v[i], b.v[i]);
}

template <int IN> __device__ __forceinline__ void scale_unit(Unit<IN>& a, float s) {
  if constexpr (IN != CC_I32) {
#pragma unroll
    for (int i = 0; i < Tr<IN>::UE; ++i) a.v[i] = __fmul_rn(a.v[i], s);
  }
}

// ---- the fold machine ---------------------------------------------------------------------------
// A schedule's fold order over the N ranks, as one code byte per position p = 0..N-1 (the
// position's value is rank rmap[p]'s element):
//   bit 0 FOLD_CUR : node = cur (+) x     (else node = x)
//   bit 1 PUSH     : push node as a pending partial (else cur = node)
//   bits 2-4 NPOP  : then NPOP times: cur = pop() (+) cur
//   bit 5 FOLD_TOP : then top = top (+) cur
// The double binary tree (in-order, ((S_left (+) x) (+) S_right)) uses FOLD_CUR / PUSH /
// NPOP; the binomial reduce (x_v first, then each child's partial) uses PUSH / NPOP /
// FOLD_TOP. The host builds the codes; a stack of at most 6 pending partials is kept in
// shared memory for 16-byte units (SmemStack) and in registers for single elements
// (FoldStack: each access is a warp-uniform switch).

constexpr uint8_t kFoldCur = 1, kPush = 2, kFoldTop = 32;
__host__ __device__ constexpr int npop_of(uint8_t code) { return (code >> 2) & 7; }

struct FoldProgram {
  uint8_t code[kMaxRanks];
  uint8_t rmap[kMaxRanks];
};

// Combine for a unit (UE lanes), a raw 16-byte load, or one element.
template <int IN, int OP> __device__ __forceinline__ void comb(Unit<IN>& a, const Unit<IN>& b) { op_unit<IN, OP>(a, b); }
template <int IN, int OP> __device__ __forceinline__ void comb(Unit<IN>& a, const uint4& b) {
  op_unit<IN, OP>(a, to_unit<IN>(b));
}
template <int IN, int OP> __device__ __forceinline__ void comb(typename Tr<IN>::Acc& a, const typename Tr<IN>::Acc& b) {
  a = op<IN, OP>(a, b);
}


template <typename V, int S = kStackSlots> struct FoldStack {
  static_assert(S >= 1 && S <= 8, "1..8 stack slots");
  V s[S];
  int depth = 0;
  __device__ __forceinline__ void push(const V& u) {
    switch (depth) {
#define CC_PUSH_CASE(k) case k: if constexpr (k < S) s[k] = u; break;
      CC_PUSH_CASE(0) CC_PUSH_CASE(1) CC_PUSH_CASE(2) CC_PUSH_CASE(3)
      CC_PUSH_CASE(4) CC_PUSH_CASE(5) CC_PUSH_CASE(6) CC_PUSH_CASE(7)
#undef CC_PUSH_CASE
    }
    ++depth;
  }
  __device__ __forceinline__ V top() const {
    switch (depth - 1) {
#define CC_TOP_CASE(k) case k: if constexpr (k < S) return s[k]; break;
      CC_TOP_CASE(0) CC_TOP_CASE(1) CC_TOP_CASE(2) CC_TOP_CASE(3)
      CC_TOP_CASE(4) CC_TOP_CASE(5) CC_TOP_CASE(6)
#undef CC_TOP_CASE
    }
    return s[S - 1];
  }
  __device__ __forceinline__ void set_top(const V& u) {
    switch (depth - 1) {
#define CC_SET_CASE(k) case k: if constexpr (k < S) s[k] = u; break;
      CC_SET_CASE(0) CC_SET_CASE(1) CC_SET_CASE(2) CC_SET_CASE(3)
      CC_SET_CASE(4) CC_SET_CASE(5) CC_SET_CASE(6) CC_SET_CASE(7)
#undef CC_SET_CASE
    }
  }
};

// The same stack in shared memory, for units: each thread owns a column of kThreads-strided
// 16-byte words (slot k, word w at base[(k * UW + w) * stride]; UW = 1 word per unit for
// fp32 / int32, 2 for widened bf16), so a push or a pop is one shared-memory access at a
// computed address instead of a switch over register slots.
template <int IN> struct SmemStack {
  static constexpr int UW = (int)(sizeof(Unit<IN>) / 16);
  uint4* base;
  int stride;
  int depth = 0;
  __device__ __forceinline__ void put(int k, const Unit<IN>& u) {
#pragma unroll
    for (int w = 0; w < UW; ++w) {
      const uint32_t* b = reinterpret_cast<const uint32_t*>(u.v) + 4 * w;
      base[(k * UW + w) * stride] = make_uint4(b[0], b[1], b[2], b[3]);
    }
  }
  __device__ __forceinline__ Unit<IN> get(int k) const {
    Unit<IN> u;
#pragma unroll
    for (int w = 0; w < UW; ++w) {
      const uint4 q = base[(k * UW + w) * stride];
      uint32_t* b = reinterpret_cast<uint32_t*>(u.v) + 4 * w;
      b[0] = q.x; b[1] = q.y; b[2] = q.z; b[3] = q.w;
    }
    return u;
  }
  __device__ __forceinline__ void push(const Unit<IN>& u) { put(depth++, u); }
  __device__ __forceinline__ Unit<IN> top() const { return get(depth - 1); }
  __device__ __forceinline__ void set_top(const Unit<IN>& u) { put(depth - 1, u); }
};

// One position of the machine; `x` is the position's loaded value (a unit or an element).
template <int IN, int OP, typename V, typename St>
__device__ __forceinline__ void fold_step(uint8_t code, const V& x, V& cur, St& st) {
  V node = x;
  if (code & kFoldCur) { node = cur; comb<IN, OP>(node, x); }
  if (code & kPush) st.push(node); else cur = node;
  for (int k = npop_of(code); k > 0; --k) {
    V t = st.top();
    --st.depth;
    comb<IN, OP>(t, cur);
    cur = t;
  }
  if (code & kFoldTop) { V t = st.top(); comb<IN, OP>(t, cur); st.set_top(t); }
}

}  // namespace cc
