// cc_alltoallv_noalloc: the MoE alltoallv for callers that cannot allocate device memory.
//
// cc_alltoallv takes its routing scratch (tile counts, row ranks, bases, receive counts)
// from a caller-provided workspace. Some callers have no way to provide one: a plugin or
// custom-operator host that hands over only input and output buffers, or a runtime that
// has reserved all device memory for its own pool and forbids side allocations (and
// cudaMalloc, which also synchronizes the device, is off limits on a latency-bound path).
// This variant keeps the scratch in a fixed array in the library's own device memory
// instead: kStaticScratchBytes per GPU, held by every GPU that loads the library until
// the process exits.
#include <mutex>

#include "cc_args.h"
#include "cc_launch.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(1) << 20;  // 1 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_a2a_scratch[kStaticScratchBytes];

// In host code g_a2a_scratch names a host-side stand-in, not device memory: the device
// address is looked up with the device current, and only a successful lookup is kept, so a
// call that failed (for instance one made while a stream was being captured) leaves the
// next call free to try again.
struct DeviceScratch {
  std::mutex mu;
  void* ptr = nullptr;
};
DeviceScratch g_scratch[kMaxDevices];

cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  DeviceScratch& s = g_scratch[dev];
  std::lock_guard<std::mutex> lock(s.mu);
  if (!s.ptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_a2a_scratch);
    if (e != cudaSuccess) {
      cudaGetLastError();  // do not leave the failed lookup pending for the caller
      return e;
    }
    s.ptr = p;
  }
  *out = s.ptr;
  return cudaSuccess;
}

}  // namespace

extern "C" cc_status cc_alltoallv_noalloc(const void* const* send, void* const* recv, int nranks, size_t row_bytes,
                                          const int32_t* const* expert_ids, int tokens, int topk,
                                          int experts_per_rank, size_t recv_capacity_rows, int direction,
                                          int32_t* recv_rows, void* stream) {
  if (!cc::a2a_args_ok(send, recv, nranks, row_bytes, expert_ids, tokens, topk, experts_per_rank, direction))
    return CC_ERR_INVALID_ARG;
  // the routing scratch must fit the fixed array
  if (cc::a2a_workspace_bytes(nranks, tokens, topk, experts_per_rank) > kStaticScratchBytes) return CC_ERR_INVALID_ARG;
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return CC_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cc::launch_alltoallv(send, recv, nranks, row_bytes, expert_ids, tokens, topk, experts_per_rank,
                           recv_capacity_rows, direction, scratch, s) != cudaSuccess)
    return CC_ERR_CUDA;
  if (recv_rows && cc::copy_recv_counts(scratch, nranks, recv_rows, s) != cudaSuccess) return CC_ERR_CUDA;
  return CC_OK;
}
