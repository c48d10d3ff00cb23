// C-ABI entry points of libcc: argument validation, then a launch of the matching kernel.
// Nothing here allocates device memory; every call is stream-ordered and returns after
// enqueuing (only argument and launch errors are reported synchronously).
#include <cstring>
#include <vector>

#include "cc_launch.h"

using namespace cc;

namespace {

cc_status cuda_status(cudaError_t e) { return e == cudaSuccess ? CC_OK : CC_ERR_CUDA; }

size_t dtype_bytes(cc_dtype t) { return t == CC_BF16 ? 2 : 4; }

bool valid_dtype(int t) { return t == CC_F32 || t == CC_BF16 || t == CC_I32; }

bool valid_ranks(int nranks) { return nranks >= 1 && nranks <= CC_MAX_RANKS; }

bool all_nonnull(const void* const* p, int n) {
  if (!p) return false;
  for (int i = 0; i < n; ++i)
    if (!p[i]) return false;
  return true;
}

// The reduction dtype pairs: (F32, F32), (BF16, F32), (I32, I32).
cc_status check_reduce(int in_t, int out_t, int op, float scale) {
  if (!valid_dtype(in_t) || !valid_dtype(out_t)) return CC_ERR_INVALID_ARG;
  const bool pair_ok = (in_t == CC_F32 && out_t == CC_F32) || (in_t == CC_BF16 && out_t == CC_F32) ||
                       (in_t == CC_I32 && out_t == CC_I32);
  if (!pair_ok) return CC_ERR_INVALID_ARG;
  if (op < CC_SUM || op > CC_PROD) return CC_ERR_INVALID_ARG;
  if (in_t == CC_I32 && scale != 1.0f) return CC_ERR_INVALID_ARG;
  if (!(scale == scale)) return CC_ERR_INVALID_ARG;  // NaN scale
  return CC_OK;
}

void chunk_bounds(size_t count, int n, int c, size_t& a, size_t& len) {
  const size_t q = count / n, r = count % n;
  a = (size_t)c * q + ((size_t)c < r ? (size_t)c : r);
  len = q + ((size_t)c < r ? 1 : 0);
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

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
                                   algo == CC_ALGO_RING ? kFoldRing : kFoldTree, kAllReduce, 0, scale,
                                   as_stream(stream)));
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
                                   scale, as_stream(stream)));
}

cc_status cc_reduce(const void* const* send, void* recv_root, int nranks, int root, size_t count, cc_dtype in_t,
                    cc_dtype out_t, cc_op op, float scale, void* stream) {
  if (!valid_ranks(nranks) || !send || root < 0 || root >= nranks) return CC_ERR_INVALID_ARG;
  if (cc_status st = check_reduce(in_t, out_t, op, scale)) return st;
  if (count == 0) return CC_OK;
  if (!all_nonnull(send, nranks) || !recv_root) return CC_ERR_INVALID_ARG;
  void* dst[1] = {recv_root};
  return cuda_status(launch_reduce(send, dst, 1, nranks, count, in_t, op, kFoldBinomial, kReduceRoot, root, scale,
                                   as_stream(stream)));
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

static bool a2a_shape_ok(int nranks, int tokens, int topk, int experts_per_rank) {
  return valid_ranks(nranks) && tokens >= 0 && topk >= 1 && topk <= 8 && experts_per_rank >= 1 &&
         (long long)nranks * experts_per_rank <= 1024 && (long long)tokens * topk < (1ll << 31);
}

size_t cc_alltoallv_workspace_size(int nranks, int tokens, int topk, int experts_per_rank) {
  if (!a2a_shape_ok(nranks, tokens, topk, experts_per_rank)) return 0;
  return a2a_workspace_bytes(nranks, tokens, topk, experts_per_rank);
}

cc_status cc_alltoallv(const void* const* send, void* const* recv, int nranks, size_t row_bytes,
                       const int32_t* const* expert_ids, int tokens, int topk, int experts_per_rank,
                       size_t recv_capacity_rows, int direction, void* workspace, size_t workspace_bytes,
                       void* stream) {
  if (!a2a_shape_ok(nranks, tokens, topk, experts_per_rank)) return CC_ERR_INVALID_ARG;
  if (!all_nonnull(send, nranks) || !all_nonnull((const void* const*)recv, nranks) ||
      !all_nonnull((const void* const*)expert_ids, nranks))
    return CC_ERR_INVALID_ARG;
  if (row_bytes == 0 || row_bytes % 16 != 0 || (direction != 0 && direction != 1)) return CC_ERR_INVALID_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255) ||
      workspace_bytes < a2a_workspace_bytes(nranks, tokens, topk, experts_per_rank))
    return CC_ERR_INVALID_ARG;
  for (int r = 0; r < nranks; ++r)
    if ((reinterpret_cast<uintptr_t>(send[r]) | reinterpret_cast<uintptr_t>(recv[r])) & 15) return CC_ERR_INVALID_ARG;
  return cuda_status(launch_alltoallv(send, recv, nranks, row_bytes, expert_ids, tokens, topk, experts_per_rank,
                                      recv_capacity_rows, direction, workspace, as_stream(stream)));
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
  if (!valid_ranks(nranks) || ntensors < 0 || cap_bytes == 0 || !(scale == scale)) return CC_ERR_INVALID_ARG;
  if (algo != CC_ALGO_RING && algo != CC_ALGO_TREE) return CC_ERR_INVALID_ARG;
  if (ntensors == 0) return CC_OK;
  if (!numels || !grads || !out) return CC_ERR_INVALID_ARG;
  for (int r = 0; r < nranks; ++r)
    for (int i = 0; i < ntensors; ++i)
      if (numels[i] && (!grads[(size_t)r * ntensors + i] || !out[(size_t)r * ntensors + i]))
        return CC_ERR_INVALID_ARG;  // empty tensors may be null
  std::vector<int32_t> order(ntensors), start(ntensors + 1);
  int32_t nb = 0;
  cc_bucket_assign(numels, ntensors, 4, cap_bytes, order.data(), start.data(), &nb);
  std::vector<BucketTensorDesc> desc(ntensors);
  for (int b = 0; b < nb; ++b) {
    uint64_t count = 0;
    for (int k = start[b]; k < start[b + 1]; ++k) count += numels[order[k]];
    uint64_t off = 0;
    for (int k = start[b]; k < start[b + 1]; ++k) {
      desc[order[k]] = BucketTensorDesc{numels[order[k]], off, count};
      off += numels[order[k]];
    }
  }
  // launch groups in bucket order, skipping empty tensors
  const int limit = bucket_group_limit(nranks);
  std::vector<int32_t> ids;
  ids.reserve(limit);
  const FoldKind fold = algo == CC_ALGO_RING ? kFoldRing : kFoldTree;
  for (int k = 0; k <= ntensors; ++k) {
    if (k < ntensors && numels[order[k]] > 0) ids.push_back(order[k]);
    if ((int)ids.size() == limit || (k == ntensors && !ids.empty())) {
      cudaError_t err = launch_bucket_allreduce(grads, out, nranks, ntensors, ids.data(), (int)ids.size(),
                                                desc.data(), fold, scale, as_stream(stream));
      if (err != cudaSuccess) return CC_ERR_CUDA;
      ids.clear();
    }
  }
  return CC_OK;
}

cc_status cc_bucket_allreduce_host(const void* const* host_grads, void* const* host_out, void* const* dev_grads,
                                   void* const* dev_out, int nranks, int ntensors, const size_t* numels,
                                   size_t cap_bytes, cc_algo algo, float scale, void* stream) {
  if (!valid_ranks(nranks) || ntensors < 0 || cap_bytes == 0) return CC_ERR_INVALID_ARG;
  if (ntensors == 0) return CC_OK;
  if (!host_grads || !host_out || !dev_grads || !dev_out || !numels) return CC_ERR_INVALID_ARG;
  const size_t total = (size_t)nranks * ntensors;
  for (size_t j = 0; j < total; ++j)
    if (numels[j % ntensors] && (!host_grads[j] || !host_out[j] || !dev_grads[j] || !dev_out[j]))
      return CC_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  for (size_t j = 0; j < total; ++j) {
    const size_t nb = numels[j % ntensors] * 4;
    if (nb && cudaMemcpyAsync(dev_grads[j], host_grads[j], nb, cudaMemcpyHostToDevice, s) != cudaSuccess)
      return CC_ERR_CUDA;
  }
  cc_status st = cc_bucket_allreduce((const void* const*)dev_grads, dev_out, nranks, ntensors, numels, cap_bytes,
                                     algo, scale, stream);
  if (st != CC_OK) return st;
  for (size_t j = 0; j < total; ++j) {
    const size_t nb = numels[j % ntensors] * 4;
    if (nb && cudaMemcpyAsync(host_out[j], dev_out[j], nb, cudaMemcpyDeviceToHost, s) != cudaSuccess)
      return CC_ERR_CUDA;
  }
  return CC_OK;
}

}  // extern "C"
