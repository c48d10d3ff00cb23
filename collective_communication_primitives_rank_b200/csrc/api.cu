// C-ABI entry points of libcc: argument validation, then a launch of the matching kernel.
// Nothing here allocates device memory; every call is stream-ordered and returns after
// enqueuing (only argument and launch errors are reported synchronously).
#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "cc_args.h"
#include "cc_launch.h"

using namespace cc;

namespace {

cc_status cuda_status(cudaError_t e) { return e == cudaSuccess ? CC_OK : CC_ERR_CUDA; }

size_t dtype_bytes(cc_dtype t) { return t == CC_BF16 ? 2 : 4; }

bool valid_dtype(int t) { return t == CC_F32 || t == CC_BF16 || t == CC_I32; }

// The reduction dtype pairs: (F32, F32), (BF16, F32), (I32, I32).
cc_status check_reduce(int in_t, int out_t, int op, float scale) {
  if (!valid_dtype(in_t) || !valid_dtype(out_t)) return CC_ERR_INVALID_ARG;
  const bool pair_ok = (in_t == CC_F32 && out_t == CC_F32) || (in_t == CC_BF16 && out_t == CC_F32) ||
                       (in_t == CC_I32 && out_t == CC_I32);
  if (!pair_ok) return CC_ERR_INVALID_ARG;
  if (op < CC_SUM || op > CC_PROD) return CC_ERR_INVALID_ARG;
  if (in_t == CC_I32 && scale != 1.0f) return CC_ERR_INVALID_ARG;  // CC_SCALE_MEAN included
  return CC_OK;
}

// CC_SCALE_MEAN (any NaN) asks for the average over the N ranks: one binary32 multiply of
// the folded sum by fl(1/N), the DDP average of lecture 09 §3.5 / §6.1.
float resolve_scale(float scale, int nranks) { return scale == scale ? scale : 1.0f / (float)nranks; }

void chunk_bounds(size_t count, int n, int c, size_t& a, size_t& len) {
  const size_t q = count / n, r = count % n;
  a = (size_t)c * q + ((size_t)c < r ? (size_t)c : r);
  len = q + ((size_t)c < r ? 1 : 0);
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Bucket layout of a tensor list: ids in bucket order, bucket boundaries, per-tensor
// descriptors (offset and element count of the tensor's bucket).
struct BucketLayout {
  std::vector<int32_t> order, start;
  std::vector<BucketTensorDesc> desc;
  int32_t nb = 0;
};

BucketLayout bucket_layout(const size_t* numels, int ntensors, size_t cap_bytes) {
  BucketLayout L;
  L.order.resize(ntensors);
  L.start.resize(ntensors + 1);
  L.desc.resize(ntensors);
  cc_bucket_assign(numels, ntensors, 4, cap_bytes, L.order.data(), L.start.data(), &L.nb);
  for (int b = 0; b < L.nb; ++b) {
    uint64_t count = 0;
    for (int k = L.start[b]; k < L.start[b + 1]; ++k) count += numels[L.order[k]];
    uint64_t off = 0;
    for (int k = L.start[b]; k < L.start[b + 1]; ++k) {
      L.desc[L.order[k]] = BucketTensorDesc{numels[L.order[k]], off, count};
      off += numels[L.order[k]];
    }
  }
  return L;
}

// Launch groups (at most bucket_group_limit tensors each, empty tensors skipped) for the
// tensors order[first .. last).
cudaError_t launch_bucket_range(const void* const* grads, void* const* out, int nranks, int ntensors,
                                const BucketLayout& L, int first, int last, FoldKind fold, float scale,
                                cudaStream_t s) {
  const int limit = bucket_group_limit(nranks);
  std::vector<int32_t> ids;
  ids.reserve(limit);
  for (int k = first; k <= last; ++k) {
    if (k < last && L.desc[L.order[k]].numel > 0) ids.push_back(L.order[k]);
    if ((int)ids.size() == limit || (k == last && !ids.empty())) {
      cudaError_t err =
          launch_bucket_allreduce(grads, out, nranks, ntensors, ids.data(), (int)ids.size(), L.desc.data(), fold, scale, s);
      if (err != cudaSuccess) return err;
      ids.clear();
    }
  }
  return cudaSuccess;
}

// Streams and events of the host-buffer pipeline, created once per device and kept.
struct HostPipeline {
  std::mutex mu;
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  std::vector<cudaEvent_t> ev;  // grows on demand
  cudaEvent_t event(size_t i) {
    while (ev.size() <= i) {
      cudaEvent_t e = nullptr;
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
      ev.push_back(e);
    }
    return ev[i];
  }
};
HostPipeline g_pipe[64];

// Host-buffer pipeline. The gradients are cut, in registration order (for packed buffers:
// ascending addresses), into slices of at most kSliceElems elements per rank; consecutive slices
// form stages of about kStageElems per rank. A stage's host-to-device copies run on one stream,
// its fused allreduce on the caller's stream, its device-to-host copies on a third stream, so
// the two PCIe directions and the kernels overlap stage by stage. A slice keeps its offset
// inside its bucket, so every element is folded exactly as in the unsliced call, whatever order
// the stages take. Measured on the DDP step with merged copies, one box, interleaved runs: the
// duplex floor of plain copies 72.7 ms; stages cut in bucket order (reverse registration) 83.3
// ms at 8M elements per rank; in registration order 79.5 ms at 8M, 76.8 ms at 4M (a torch
// pipeline of the same copies: 76.8 ms at 4M, 77.7 at 8M). The kernels cost nothing measurable
// (81.2 ms without them against 81.5 with them, bucket order).
#ifndef CC_HOST_STAGE_ELEMS
#define CC_HOST_STAGE_ELEMS (4ull << 20)
#endif
constexpr uint64_t kSliceElems = 1ull << 20;
constexpr uint64_t kStageElems = CC_HOST_STAGE_ELEMS;

cudaError_t bucket_allreduce_pipelined(const void* const* hg, void* const* ho, void* const* dg, void* const* dout,
                                       int nranks, int ntensors, const size_t* numels, size_t cap_bytes, FoldKind fold,
                                       float scale, bool packed, cudaStream_t s) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  HostPipeline& P = g_pipe[dev];
  std::lock_guard<std::mutex> lock(P.mu);
  if (!P.ready) {
    if ((e = cudaStreamCreateWithFlags(&P.in, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithFlags(&P.out, cudaStreamNonBlocking)) != cudaSuccess) return e;
    P.ready = true;
  }
  const BucketLayout L = bucket_layout(numels, ntensors, cap_bytes);
  size_t ne = 0;
  auto next_event = [&]() { return P.event(ne++); };
  cudaEvent_t start = next_event();
  if (!start) return cudaErrorMemoryAllocation;
  if ((e = cudaEventRecord(start, s)) != cudaSuccess) return e;
  if ((e = cudaStreamWaitEvent(P.in, start, 0)) != cudaSuccess) return e;
  if ((e = cudaStreamWaitEvent(P.out, start, 0)) != cudaSuccess) return e;

  // cut the work into stages of slices, in registration order
  struct Slice { int i; uint64_t a, len; };
  std::vector<std::vector<Slice>> stages(1);
  uint64_t stage_elems = 0;
  for (int i = 0; i < ntensors; ++i) {
    for (uint64_t a = 0; a < numels[i]; a += kSliceElems) {
      const uint64_t len = std::min<uint64_t>(kSliceElems, numels[i] - a);
      stages.back().push_back(Slice{i, a, len});
      stage_elems += len;
      if (stage_elems >= kStageElems) {
        stages.emplace_back();
        stage_elems = 0;
      }
    }
  }
  if (stages.back().empty()) stages.pop_back();
  const size_t ns = stages.size();
  std::vector<cudaEvent_t> in_done(ns), red_done(ns);
  for (size_t k = 0; k < ns; ++k) {
    in_done[k] = next_event();
    red_done[k] = next_event();
    if (!in_done[k] || !red_done[k]) return cudaErrorMemoryAllocation;
  }
  auto at = [](const void* p, uint64_t elems) { return static_cast<const char*>(p) + elems * 4; };
  auto atw = [](void* p, uint64_t elems) { return static_cast<char*>(p) + elems * 4; };
  // enqueue order: copies in of stage k+1, then the kernels and the copies out of stage k, so
  // that each stream is fed just ahead of where the GPU is (a stream fed thousands of
  // commands ahead blocks the enqueuing thread until its queue drains)
  std::vector<const void*> vg;
  std::vector<void*> vo;
  std::vector<BucketTensorDesc> vd;
  std::vector<int32_t> ids;
  const int limit = bucket_small_group_limit(nranks);
  // A stage's copies of one direction are unordered among themselves, so slices that are
  // contiguous on both sides merge into one copy (fewer, larger DMA transfers): always
  // within one tensor, across tensors only when the caller promises one allocation per
  // rank and table (`packed`), since a copy may not run from one allocation into another.
  struct Copy { char* dst; const char* src; uint64_t bytes; size_t tensor; };
  std::vector<Copy> cps;
  auto merged_copies = [&](cudaStream_t st, cudaMemcpyKind kind) -> cudaError_t {
    std::sort(cps.begin(), cps.end(), [](const Copy& x, const Copy& y) { return x.src < y.src; });
    size_t w = 0;
    for (size_t k = 0; k < cps.size(); ++k) {
      const Copy& p = w > 0 ? cps[w - 1] : cps[k];
      if (w > 0 && (packed || p.tensor == cps[k].tensor) && p.src + p.bytes == cps[k].src &&
          p.dst + p.bytes == cps[k].dst)
        cps[w - 1].bytes += cps[k].bytes;
      else
        cps[w++] = cps[k];
    }
    cps.resize(w);
    for (const Copy& c : cps) {
      cudaError_t err = cudaMemcpyAsync(c.dst, c.src, c.bytes, kind, st);
      if (err != cudaSuccess) return err;
    }
    return cudaSuccess;
  };
  auto copies_in = [&](size_t k) -> cudaError_t {
    cps.clear();
    for (const Slice& c : stages[k])
      for (int r = 0; r < nranks; ++r) {
        const size_t j = (size_t)r * ntensors + c.i;
        cps.push_back(Copy{atw(dg[j], c.a), at(hg[j], c.a), c.len * 4, j});
      }
    cudaError_t err = merged_copies(P.in, cudaMemcpyHostToDevice);
    if (err != cudaSuccess) return err;
    return cudaEventRecord(in_done[k], P.in);
  };
  auto reduce_and_copy_out = [&](size_t k) -> cudaError_t {
    cudaError_t err;
    if ((err = cudaStreamWaitEvent(s, in_done[k], 0)) != cudaSuccess) return err;
    const std::vector<Slice>& st = stages[k];
    for (size_t g0 = 0; g0 < st.size(); g0 += limit) {
      const int nv = (int)std::min<size_t>(limit, st.size() - g0);
      vg.assign((size_t)nranks * nv, nullptr);
      vo.assign((size_t)nranks * nv, nullptr);
      vd.resize(nv);
      ids.resize(nv);
      for (int v = 0; v < nv; ++v) {
        const Slice& c = st[g0 + v];
        const BucketTensorDesc& d = L.desc[c.i];
        vd[v] = BucketTensorDesc{c.len, d.bucket_off + c.a, d.bucket_count};
        ids[v] = v;
        for (int r = 0; r < nranks; ++r) {
          const size_t j = (size_t)r * ntensors + c.i;
          vg[(size_t)r * nv + v] = at(dg[j], c.a);
          vo[(size_t)r * nv + v] = atw(dout[j], c.a);
        }
      }
      if ((err = launch_bucket_allreduce(vg.data(), vo.data(), nranks, nv, ids.data(), nv, vd.data(), fold, scale, s)) !=
          cudaSuccess)
        return err;
    }
    if ((err = cudaEventRecord(red_done[k], s)) != cudaSuccess) return err;
    if ((err = cudaStreamWaitEvent(P.out, red_done[k], 0)) != cudaSuccess) return err;
    cps.clear();
    for (const Slice& c : st)
      for (int r = 0; r < nranks; ++r) {
        const size_t j = (size_t)r * ntensors + c.i;
        cps.push_back(Copy{atw(ho[j], c.a), at(dout[j], c.a), c.len * 4, j});
      }
    return merged_copies(P.out, cudaMemcpyDeviceToHost);
  };
  if ((e = copies_in(0)) != cudaSuccess) return e;
  for (size_t k = 0; k < ns; ++k) {
    if (k + 1 < ns && (e = copies_in(k + 1)) != cudaSuccess) return e;
    if ((e = reduce_and_copy_out(k)) != cudaSuccess) return e;
  }
  cudaEvent_t end = next_event();
  if (!end) return cudaErrorMemoryAllocation;
  if ((e = cudaEventRecord(end, P.out)) != cudaSuccess) return e;
  return cudaStreamWaitEvent(s, end, 0);
}

}  // namespace

extern "C" {

const char* cc_status_string(cc_status s) {
  switch (s) {
    case CC_OK: return "CC_OK";
    case CC_ERR_INVALID_ARG: return "CC_ERR_INVALID_ARG";
    case CC_ERR_UNSUPPORTED: return "CC_ERR_UNSUPPORTED";
    case CC_ERR_CUDA: return "CC_ERR_CUDA";
    case CC_ERR_TIMEOUT: return "CC_ERR_TIMEOUT";
  }
  return "CC_ERR_UNKNOWN";
}

int cc_version(void) { return 100; }

cc_status cc_async_status(int reset, void* stream) {
  int v = 0;
  if (read_async_status(&v, reset != 0, as_stream(stream)) != cudaSuccess) return CC_ERR_CUDA;
  return v == CC_OK ? CC_OK : CC_ERR_TIMEOUT;
}

cc_status cc_selftest_bounded_wait(unsigned timeout_us, void* stream) {
  if (timeout_us == 0 || timeout_us > 10000000u) return CC_ERR_INVALID_ARG;
  return cuda_status(launch_bounded_wait_selftest((uint64_t)timeout_us * 1000ull, as_stream(stream)));
}

cc_status cc_chunk(size_t count, int nranks, int c, size_t* start, size_t* len) {
  if (!valid_ranks(nranks) || c < 0 || c >= nranks || !start || !len) return CC_ERR_INVALID_ARG;
  chunk_bounds(count, nranks, c, *start, *len);
  return CC_OK;
}

cc_status cc_allreduce(const void* const* send, void* const* recv, int nranks, size_t count, cc_dtype in_t,
                       cc_dtype out_t, cc_op op, cc_algo algo, float scale, void* stream) {
  if (!valid_ranks(nranks) || !send || !recv) return CC_ERR_INVALID_ARG;
  if (cc_status st = check_reduce(in_t, out_t, op, scale)) return st;
  if (algo != CC_ALGO_RING && algo != CC_ALGO_TREE) return CC_ERR_INVALID_ARG;
  if (count == 0) return CC_OK;
  if (!all_nonnull(send, nranks) || !all_nonnull((const void* const*)recv, nranks)) return CC_ERR_INVALID_ARG;
  for (int r = 0; r < nranks; ++r)
    if (recv[r] == send[r] && dtype_bytes(in_t) != dtype_bytes(out_t)) return CC_ERR_INVALID_ARG;
  return cuda_status(launch_reduce(send, recv, nranks, nranks, count, in_t, op,
                                   algo == CC_ALGO_RING ? kFoldRing : kFoldTree, kAllReduce, 0,
                                   resolve_scale(scale, nranks), as_stream(stream)));
}

cc_status cc_allreduce_stepped(const void* const* send, void* const* recv, int nranks, size_t count, cc_dtype in_t,
                               cc_dtype out_t, cc_op op, cc_algo algo, float scale, void* workspace,
                               size_t workspace_bytes, void* stream) {
  if (!valid_ranks(nranks) || !send || !recv) return CC_ERR_INVALID_ARG;
  if (cc_status st = check_reduce(in_t, out_t, op, scale)) return st;
  if (algo != CC_ALGO_RING && algo != CC_ALGO_TREE) return CC_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < 256 || (reinterpret_cast<uintptr_t>(workspace) & 255)) return CC_ERR_INVALID_ARG;
  if (count == 0) return CC_OK;
  if (!all_nonnull(send, nranks) || !all_nonnull((const void* const*)recv, nranks)) return CC_ERR_INVALID_ARG;
  for (int r = 0; r < nranks; ++r)
    if (recv[r] == send[r] && dtype_bytes(in_t) != dtype_bytes(out_t)) return CC_ERR_INVALID_ARG;
  return cuda_status(launch_stepped_allreduce(send, recv, nranks, count, in_t, op,
                                              algo == CC_ALGO_RING ? kFoldRing : kFoldTree,
                                              resolve_scale(scale, nranks), static_cast<unsigned*>(workspace),
                                              as_stream(stream)));
}

cc_status cc_allreduce_hierarchical(const void* const* send, void* const* recv, int nranks, int ranks_per_node,
                                    size_t count, cc_dtype in_t, cc_dtype out_t, cc_op op, float scale, void* stream) {
  if (!valid_ranks(nranks) || !send || !recv || ranks_per_node < 1 || nranks % ranks_per_node)
    return CC_ERR_INVALID_ARG;
  if (cc_status st = check_reduce(in_t, out_t, op, scale)) return st;
  if (count == 0) return CC_OK;
  if (!all_nonnull(send, nranks) || !all_nonnull((const void* const*)recv, nranks)) return CC_ERR_INVALID_ARG;
  for (int r = 0; r < nranks; ++r)
    if (recv[r] == send[r] && dtype_bytes(in_t) != dtype_bytes(out_t)) return CC_ERR_INVALID_ARG;
  return cuda_status(launch_reduce(send, recv, nranks, nranks, count, in_t, op, kFoldHier, kAllReduce, ranks_per_node,
                                   resolve_scale(scale, nranks), as_stream(stream)));
}

cc_status cc_allreduce_multiring(const void* const* send, void* const* recv, int nranks, int nrings, size_t count,
                                 cc_dtype in_t, cc_dtype out_t, cc_op op, float scale, void* stream) {
  if (!valid_ranks(nranks) || !send || !recv || nrings < 1 || nrings > CC_MAX_RINGS) return CC_ERR_INVALID_ARG;
  if (cc_status st = check_reduce(in_t, out_t, op, scale)) return st;
  if (count == 0) return CC_OK;
  if (!all_nonnull(send, nranks) || !all_nonnull((const void* const*)recv, nranks)) return CC_ERR_INVALID_ARG;
  for (int r = 0; r < nranks; ++r)
    if (recv[r] == send[r] && dtype_bytes(in_t) != dtype_bytes(out_t)) return CC_ERR_INVALID_ARG;
  return cuda_status(launch_reduce(send, recv, nranks, nranks, count, in_t, op, kFoldMultiRing, kAllReduce, nrings,
                                   resolve_scale(scale, nranks), as_stream(stream)));
}

cc_status cc_reduce_scatter(const void* const* send, void* const* recv, int nranks, size_t count, cc_dtype in_t,
                            cc_dtype out_t, cc_op op, cc_algo algo, float scale, void* stream) {
  if (!valid_ranks(nranks) || !send || !recv) return CC_ERR_INVALID_ARG;
  if (cc_status st = check_reduce(in_t, out_t, op, scale)) return st;
  if (algo == CC_ALGO_TREE) return CC_ERR_UNSUPPORTED;
  if (algo != CC_ALGO_RING) return CC_ERR_INVALID_ARG;
  if (count == 0) return CC_OK;
  if (!all_nonnull(send, nranks)) return CC_ERR_INVALID_ARG;
  for (int c = 0; c < nranks; ++c) {
    size_t a, len;
    chunk_bounds(count, nranks, c, a, len);
    if (len && !recv[c]) return CC_ERR_INVALID_ARG;  // an empty shard may be null
  }
  return cuda_status(launch_reduce(send, recv, nranks, nranks, count, in_t, op, kFoldRing, kReduceScatter, 0,
                                   resolve_scale(scale, nranks), as_stream(stream)));
}

cc_status cc_reduce(const void* const* send, void* recv_root, int nranks, int root, size_t count, cc_dtype in_t,
                    cc_dtype out_t, cc_op op, float scale, void* stream) {
  if (!valid_ranks(nranks) || !send || root < 0 || root >= nranks) return CC_ERR_INVALID_ARG;
  if (cc_status st = check_reduce(in_t, out_t, op, scale)) return st;
  if (count == 0) return CC_OK;
  if (!all_nonnull(send, nranks) || !recv_root) return CC_ERR_INVALID_ARG;
  void* dst[1] = {recv_root};
  return cuda_status(launch_reduce(send, dst, 1, nranks, count, in_t, op, kFoldBinomial, kReduceRoot, root,
                                   resolve_scale(scale, nranks), as_stream(stream)));
}

cc_status cc_allgather(const void* const* send, void* const* recv, int nranks, size_t count, cc_dtype dtype,
                       void* stream) {
  if (!valid_ranks(nranks) || !send || !recv || !valid_dtype(dtype)) return CC_ERR_INVALID_ARG;
  if (count == 0) return CC_OK;
  if (!all_nonnull((const void* const*)recv, nranks)) return CC_ERR_INVALID_ARG;
  std::vector<CopyEntry> e(nranks);
  for (int c = 0; c < nranks; ++c) {
    size_t a, len;
    chunk_bounds(count, nranks, c, a, len);
    if (len && !send[c]) return CC_ERR_INVALID_ARG;  // an empty shard may be null
    e[c] = CopyEntry{send[c], nullptr, len, a};
  }
  return cuda_status(launch_copy(e.data(), nranks, recv, nranks, true, -1, dtype_bytes(dtype), as_stream(stream)));
}

cc_status cc_broadcast(const void* src, void* const* recv, int nranks, int root, size_t count, cc_dtype dtype,
                       void* stream) {
  if (!valid_ranks(nranks) || !recv || !valid_dtype(dtype) || root < 0 || root >= nranks)
    return CC_ERR_INVALID_ARG;
  if (count == 0) return CC_OK;
  if (!src || !all_nonnull((const void* const*)recv, nranks)) return CC_ERR_INVALID_ARG;
  CopyEntry e{src, nullptr, count, 0};
  const int skip = recv[root] == src ? root : -1;
  return cuda_status(launch_copy(&e, 1, recv, nranks, true, skip, dtype_bytes(dtype), as_stream(stream)));
}

cc_status cc_scatter(const void* src, void* const* recv, int nranks, int root, size_t count, cc_dtype dtype,
                     void* stream) {
  if (!valid_ranks(nranks) || !recv || !valid_dtype(dtype) || root < 0 || root >= nranks)
    return CC_ERR_INVALID_ARG;
  if (count == 0) return CC_OK;
  if (!src) return CC_ERR_INVALID_ARG;
  const size_t es = dtype_bytes(dtype);
  std::vector<CopyEntry> e(nranks);
  for (int c = 0; c < nranks; ++c) {
    size_t a, len;
    chunk_bounds(count, nranks, c, a, len);
    if (len && !recv[c]) return CC_ERR_INVALID_ARG;
    e[c] = CopyEntry{static_cast<const char*>(src) + a * es, recv[c], len, 0};
  }
  return cuda_status(launch_copy(e.data(), nranks, nullptr, 0, false, -1, es, as_stream(stream)));
}

cc_status cc_gather(const void* const* send, void* recv_root, int nranks, int root, size_t count, cc_dtype dtype,
                    void* stream) {
  if (!valid_ranks(nranks) || !send || !valid_dtype(dtype) || root < 0 || root >= nranks)
    return CC_ERR_INVALID_ARG;
  if (count == 0) return CC_OK;
  if (!recv_root) return CC_ERR_INVALID_ARG;
  std::vector<CopyEntry> e(nranks);
  for (int c = 0; c < nranks; ++c) {
    size_t a, len;
    chunk_bounds(count, nranks, c, a, len);
    if (len && !send[c]) return CC_ERR_INVALID_ARG;
    e[c] = CopyEntry{send[c], recv_root, len, a};
  }
  return cuda_status(launch_copy(e.data(), nranks, nullptr, 0, false, -1, dtype_bytes(dtype), as_stream(stream)));
}

// ---- MoE ------------------------------------------------------------------------------------------

cc_status cc_route_topk(const float* const* logits, int32_t* const* expert_ids, int nranks, int tokens,
                        int experts_total, int topk, void* stream) {
  if (!valid_ranks(nranks) || !all_nonnull((const void* const*)logits, nranks) ||
      !all_nonnull((const void* const*)expert_ids, nranks) || tokens < 0 || topk < 1 || topk > 8 ||
      experts_total < topk || experts_total > 1024)
    return CC_ERR_INVALID_ARG;
  if (tokens == 0) return CC_OK;
  return cuda_status(launch_route_topk(logits, expert_ids, nranks, tokens, experts_total, topk, as_stream(stream)));
}

size_t cc_alltoallv_workspace_size(int nranks, int tokens, int topk, int experts_per_rank) {
  if (!a2a_shape_ok(nranks, tokens, topk, experts_per_rank)) return 0;
  return a2a_workspace_bytes(nranks, tokens, topk, experts_per_rank);
}

cc_status cc_alltoallv(const void* const* send, void* const* recv, int nranks, size_t row_bytes,
                       const int32_t* const* expert_ids, int tokens, int topk, int experts_per_rank,
                       size_t recv_capacity_rows, int direction, void* workspace, size_t workspace_bytes,
                       void* stream) {
  if (!a2a_args_ok(send, recv, nranks, row_bytes, expert_ids, tokens, topk, experts_per_rank, direction))
    return CC_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) ||
      workspace_bytes < a2a_workspace_bytes(nranks, tokens, topk, experts_per_rank))
    return CC_ERR_INVALID_ARG;
  return cuda_status(launch_alltoallv(send, recv, nranks, row_bytes, expert_ids, tokens, topk, experts_per_rank,
                                      recv_capacity_rows, direction, workspace, as_stream(stream)));
}

cc_status cc_alltoallv_plan(const int32_t* const* expert_ids, int nranks, int tokens, int topk, int experts_per_rank,
                            void* workspace, size_t workspace_bytes, void* stream) {
  if (!a2a_shape_ok(nranks, tokens, topk, experts_per_rank) ||
      !all_nonnull((const void* const*)expert_ids, nranks))
    return CC_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) ||
      workspace_bytes < a2a_workspace_bytes(nranks, tokens, topk, experts_per_rank))
    return CC_ERR_INVALID_ARG;
  return cuda_status(launch_alltoallv(nullptr, nullptr, nranks, 0, expert_ids, tokens, topk, experts_per_rank, 0, 0,
                                      workspace, as_stream(stream), kA2ATables));
}

cc_status cc_alltoallv_run(const void* const* send, void* const* recv, int nranks, size_t row_bytes,
                           const int32_t* const* expert_ids, int tokens, int topk, int experts_per_rank,
                           size_t recv_capacity_rows, int direction, void* workspace, size_t workspace_bytes,
                           void* stream) {
  if (!a2a_args_ok(send, recv, nranks, row_bytes, expert_ids, tokens, topk, experts_per_rank, direction))
    return CC_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) ||
      workspace_bytes < a2a_workspace_bytes(nranks, tokens, topk, experts_per_rank))
    return CC_ERR_INVALID_ARG;
  return cuda_status(launch_alltoallv(send, recv, nranks, row_bytes, expert_ids, tokens, topk, experts_per_rank,
                                      recv_capacity_rows, direction, workspace, as_stream(stream), kA2ACopy));
}

cc_status cc_alltoallv_recv_counts(const void* workspace, int nranks, int32_t* recv_rows, void* stream) {
  if (!workspace || !recv_rows || !valid_ranks(nranks)) return CC_ERR_INVALID_ARG;
  return cuda_status(copy_recv_counts(workspace, nranks, recv_rows, as_stream(stream)));
}

// ---- DDP buckets ------------------------------------------------------------------------------------

cc_status cc_bucket_assign(const size_t* numels, int ntensors, size_t elem_bytes, size_t cap_bytes, int32_t* order,
                           int32_t* bucket_start, int32_t* nbuckets) {
  if (ntensors < 0 || (ntensors > 0 && (!numels || !order)) || !bucket_start || !nbuckets || elem_bytes == 0 ||
      cap_bytes == 0)
    return CC_ERR_INVALID_ARG;
  int nb = 0, pos = 0;
  size_t cur = 0;
  bool open = false;
  for (int i = ntensors - 1; i >= 0; --i) {
    const size_t b = numels[i] * elem_bytes;
    if (open && cur + b > cap_bytes) {
      open = false;
      cur = 0;
    }
    if (!open) {
      bucket_start[nb++] = pos;
      open = true;
    }
    order[pos++] = i;
    cur += b;
  }
  bucket_start[nb] = pos;
  *nbuckets = nb;
  return CC_OK;
}

cc_status cc_bucket_flatten(const void* const* tensors, const size_t* numels, int ntensors, void* bucket,
                            cc_dtype dtype, void* stream) {
  if (ntensors < 0 || !valid_dtype(dtype) || (ntensors > 0 && (!numels || !tensors))) return CC_ERR_INVALID_ARG;
  std::vector<CopyEntry> e(ntensors);
  size_t off = 0;
  for (int i = 0; i < ntensors; ++i) {
    if (numels[i] && (!tensors[i] || !bucket)) return CC_ERR_INVALID_ARG;
    e[i] = CopyEntry{tensors[i], bucket, numels[i], off};
    off += numels[i];
  }
  return cuda_status(launch_copy(e.data(), ntensors, nullptr, 0, false, -1, dtype_bytes(dtype), as_stream(stream)));
}

cc_status cc_bucket_unflatten(const void* bucket, void* const* tensors, const size_t* numels, int ntensors,
                              cc_dtype dtype, void* stream) {
  if (ntensors < 0 || !valid_dtype(dtype) || (ntensors > 0 && (!numels || !tensors))) return CC_ERR_INVALID_ARG;
  const size_t es = dtype_bytes(dtype);
  std::vector<CopyEntry> e(ntensors);
  size_t off = 0;
  for (int i = 0; i < ntensors; ++i) {
    if (numels[i] && (!tensors[i] || !bucket)) return CC_ERR_INVALID_ARG;
    e[i] = CopyEntry{static_cast<const char*>(bucket) + off * es, tensors[i], numels[i], 0};
    off += numels[i];
  }
  return cuda_status(launch_copy(e.data(), ntensors, nullptr, 0, false, -1, es, as_stream(stream)));
}

cc_status cc_bucket_allreduce(const void* const* grads, void* const* out, int nranks, int ntensors,
                              const size_t* numels, size_t cap_bytes, cc_algo algo, float scale, void* stream) {
  if (!valid_ranks(nranks) || ntensors < 0 || cap_bytes == 0) return CC_ERR_INVALID_ARG;
  if (algo != CC_ALGO_RING && algo != CC_ALGO_TREE) return CC_ERR_INVALID_ARG;
  if (ntensors == 0) return CC_OK;
  if (!numels || !grads || !out) return CC_ERR_INVALID_ARG;
  scale = resolve_scale(scale, nranks);
  for (int r = 0; r < nranks; ++r)
    for (int i = 0; i < ntensors; ++i)
      if (numels[i] && (!grads[(size_t)r * ntensors + i] || !out[(size_t)r * ntensors + i]))
        return CC_ERR_INVALID_ARG;  // empty tensors may be null
  const BucketLayout L = bucket_layout(numels, ntensors, cap_bytes);
  if (launch_bucket_range(grads, out, nranks, ntensors, L, 0, ntensors, algo == CC_ALGO_RING ? kFoldRing : kFoldTree,
                          scale, as_stream(stream)) != cudaSuccess)
    return CC_ERR_CUDA;
  return CC_OK;
}

cc_status cc_bucket_allreduce_buckets(const void* const* grads, void* const* out, int nranks, int ntensors,
                                      const size_t* numels, size_t cap_bytes, int first_bucket, int nbuckets,
                                      cc_algo algo, float scale, void* stream) {
  if (!valid_ranks(nranks) || ntensors < 0 || cap_bytes == 0 || first_bucket < 0 || nbuckets < 0)
    return CC_ERR_INVALID_ARG;
  scale = resolve_scale(scale, nranks);
  if (algo != CC_ALGO_RING && algo != CC_ALGO_TREE) return CC_ERR_INVALID_ARG;
  if (ntensors == 0 || nbuckets == 0) return CC_OK;
  if (!numels || !grads || !out) return CC_ERR_INVALID_ARG;
  const BucketLayout L = bucket_layout(numels, ntensors, cap_bytes);
  if (first_bucket + nbuckets > L.nb) return CC_ERR_INVALID_ARG;
  for (int k = L.start[first_bucket]; k < L.start[first_bucket + nbuckets]; ++k)
    for (int r = 0; r < nranks; ++r) {
      const int i = L.order[k];
      if (numels[i] && (!grads[(size_t)r * ntensors + i] || !out[(size_t)r * ntensors + i])) return CC_ERR_INVALID_ARG;
    }
  if (launch_bucket_range(grads, out, nranks, ntensors, L, L.start[first_bucket], L.start[first_bucket + nbuckets],
                          algo == CC_ALGO_RING ? kFoldRing : kFoldTree, scale, as_stream(stream)) != cudaSuccess)
    return CC_ERR_CUDA;
  return CC_OK;
}

cc_status cc_bucket_allreduce_host(const void* const* host_grads, void* const* host_out, void* const* dev_grads,
                                   void* const* dev_out, int nranks, int ntensors, const size_t* numels,
                                   size_t cap_bytes, cc_algo algo, float scale, int packed, void* stream) {
  if (!valid_ranks(nranks) || ntensors < 0 || cap_bytes == 0) return CC_ERR_INVALID_ARG;
  scale = resolve_scale(scale, nranks);
  if (algo != CC_ALGO_RING && algo != CC_ALGO_TREE) return CC_ERR_INVALID_ARG;
  if (ntensors == 0) return CC_OK;
  if (!host_grads || !host_out || !dev_grads || !dev_out || !numels) return CC_ERR_INVALID_ARG;
  const size_t total = (size_t)nranks * ntensors;
  for (size_t j = 0; j < total; ++j)
    if (numels[j % ntensors] && (!host_grads[j] || !host_out[j] || !dev_grads[j] || !dev_out[j]))
      return CC_ERR_INVALID_ARG;
  return cuda_status(bucket_allreduce_pipelined(host_grads, host_out, dev_grads, dev_out, nranks, ntensors, numels,
                                                cap_bytes, algo == CC_ALGO_RING ? kFoldRing : kFoldTree, scale,
                                                packed != 0, as_stream(stream)));
}

// ---- one rank's slice (ranks in separate processes) -------------------------------------

cc_status cc_allreduce_slice(const void* const* send, void* const* recv, int nranks, int rank, size_t count,
                             cc_dtype in_t, cc_dtype out_t, cc_op op, cc_algo algo, float scale, void* stream) {
  if (!valid_ranks(nranks) || !send || !recv || rank < 0 || rank >= nranks) return CC_ERR_INVALID_ARG;
  if (cc_status st = check_reduce(in_t, out_t, op, scale)) return st;
  if (algo != CC_ALGO_RING && algo != CC_ALGO_TREE) return CC_ERR_INVALID_ARG;
  if (count == 0) return CC_OK;
  if (!all_nonnull(send, nranks) || !all_nonnull((const void* const*)recv, nranks)) return CC_ERR_INVALID_ARG;
  for (int r = 0; r < nranks; ++r)
    if (recv[r] == send[r] && dtype_bytes(in_t) != dtype_bytes(out_t)) return CC_ERR_INVALID_ARG;
  size_t a, len;
  chunk_bounds(count, nranks, rank, a, len);
  if (len == 0) return CC_OK;
  return cuda_status(launch_reduce(send, recv, nranks, nranks, count, in_t, op,
                                   algo == CC_ALGO_RING ? kFoldRing : kFoldTree, kAllReduce, 0,
                                   resolve_scale(scale, nranks), as_stream(stream), a, a + len));
}

cc_status cc_reduce_scatter_slice(const void* const* send, void* recv_shard, int nranks, int rank, size_t count,
                                  cc_dtype in_t, cc_dtype out_t, cc_op op, float scale, void* stream) {
  if (!valid_ranks(nranks) || !send || rank < 0 || rank >= nranks) return CC_ERR_INVALID_ARG;
  if (cc_status st = check_reduce(in_t, out_t, op, scale)) return st;
  if (count == 0) return CC_OK;
  if (!all_nonnull(send, nranks)) return CC_ERR_INVALID_ARG;
  size_t a, len;
  chunk_bounds(count, nranks, rank, a, len);
  if (len == 0) return CC_OK;
  if (!recv_shard) return CC_ERR_INVALID_ARG;
  // the reduce-scatter kernel writes chunk c to dst[c]; only chunk `rank` is folded here
  std::vector<void*> dst(nranks, nullptr);
  dst[rank] = recv_shard;
  return cuda_status(launch_reduce(send, dst.data(), nranks, nranks, count, in_t, op, kFoldRing, kReduceScatter, 0,
                                   resolve_scale(scale, nranks), as_stream(stream), a, a + len));
}

cc_status cc_allgather_slice(const void* send_shard, void* const* recv, int nranks, int rank, size_t count,
                             cc_dtype dtype, void* stream) {
  if (!valid_ranks(nranks) || !recv || !valid_dtype(dtype) || rank < 0 || rank >= nranks) return CC_ERR_INVALID_ARG;
  if (count == 0) return CC_OK;
  if (!all_nonnull((const void* const*)recv, nranks)) return CC_ERR_INVALID_ARG;
  size_t a, len;
  chunk_bounds(count, nranks, rank, a, len);
  if (len == 0) return CC_OK;
  if (!send_shard) return CC_ERR_INVALID_ARG;
  CopyEntry e{send_shard, nullptr, len, a};
  return cuda_status(launch_copy(&e, 1, recv, nranks, true, -1, dtype_bytes(dtype), as_stream(stream), true));
}

}  // extern "C"
