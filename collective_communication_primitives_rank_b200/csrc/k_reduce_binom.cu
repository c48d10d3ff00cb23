// Binomial reduce-to-root programs (lecture 09 §3.4) compiled to straight-line code for the
// rank counts from 5 to 15 that are not powers of two (SUM only; the powers of two are in
// k_reduce.cu), and the double-binary-tree allreduce programs (lecture 09 §5.2) of 8 and 16
// ranks (SUM; TreePlan, the same program as tree_program in k_reduce.cu; also with element
// stores into outputs at another offset than the sources). Each is the same pre-order walk and fold-machine codes as the run-time program
// of any rank count (binomial_program in k_reduce.cu), built at compile time by BinomialPlan,
// so the result is bit for bit the fold machine's. A translation unit of its own: the build
// compiles it beside k_reduce.cu.
#include "k_reduce_kernels.cuh"

namespace cc {

template <int IN>
static cudaError_t run_binom_np2(ReduceParams& P, int kind, cudaStream_t s) {
  switch (kind - kBinomN0) {
    case 5: return run_reduce<IN, CC_SUM, kBinomN0 + 5>(P, s);
    case 6: return run_reduce<IN, CC_SUM, kBinomN0 + 6>(P, s);
    case 7: return run_reduce<IN, CC_SUM, kBinomN0 + 7>(P, s);
    case 9: return run_reduce<IN, CC_SUM, kBinomN0 + 9>(P, s);
    case 10: return run_reduce<IN, CC_SUM, kBinomN0 + 10>(P, s);
    case 11: return run_reduce<IN, CC_SUM, kBinomN0 + 11>(P, s);
    case 12: return run_reduce<IN, CC_SUM, kBinomN0 + 12>(P, s);
    case 13: return run_reduce<IN, CC_SUM, kBinomN0 + 13>(P, s);
    case 14: return run_reduce<IN, CC_SUM, kBinomN0 + 14>(P, s);
    case 15: return run_reduce<IN, CC_SUM, kBinomN0 + 15>(P, s);
  }
  return cudaErrorInvalidValue;
}

cudaError_t run_reduce_binom_np2(ReduceParams& P, cc_dtype in_t, int kind, cudaStream_t s) {
  switch (in_t) {
    case CC_F32: return run_binom_np2<CC_F32>(P, kind, s);
    case CC_BF16: return run_binom_np2<CC_BF16>(P, kind, s);
    case CC_I32: return run_binom_np2<CC_I32>(P, kind, s);
  }
  return cudaErrorInvalidValue;
}

template <int IN, bool SS>
static cudaError_t run_tree_ct(ReduceParams& P, int kind, cudaStream_t s) {
  return kind == kTree8 ? run_reduce<IN, CC_SUM, kTree8, SS>(P, s) : run_reduce<IN, CC_SUM, kTree16, SS>(P, s);
}

cudaError_t run_reduce_tree_ct(ReduceParams& P, cc_dtype in_t, int kind, cudaStream_t s, bool scalar_out) {
  if (kind != kTree8 && kind != kTree16) return cudaErrorInvalidValue;
  if (scalar_out) {  // 4-byte elements only
    switch (in_t) {
      case CC_F32: return run_tree_ct<CC_F32, true>(P, kind, s);
      case CC_I32: return run_tree_ct<CC_I32, true>(P, kind, s);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (in_t) {
    case CC_F32: return run_tree_ct<CC_F32, false>(P, kind, s);
    case CC_BF16: return run_tree_ct<CC_BF16, false>(P, kind, s);
    case CC_I32: return run_tree_ct<CC_I32, false>(P, kind, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace cc
