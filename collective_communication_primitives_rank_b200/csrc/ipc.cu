// CUDA IPC for the slice calls: export a device allocation from one process, map it in
// another (peer access enabled lazily), reference-counted per allocation.
#include <cuda_runtime.h>

#include <cstring>
#include <map>
#include <mutex>
#include <string>

#include "../../include/cc.h"

namespace {

// cuMemGetAddressRange (driver API) through the runtime's entry-point lookup, so that the
// library needs no link against the driver library: (base, size) of the allocation that
// holds a device pointer.
typedef int (*GetRangeFn)(unsigned long long* base, size_t* size, unsigned long long ptr);

GetRangeFn get_range_fn() {
  static GetRangeFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (GetRangeFn) nullptr;
    return reinterpret_cast<GetRangeFn>(p);
  }();
  return fn;
}

struct Mapping {
  void* base = nullptr;
  int refs = 0;
};

std::mutex g_mu;
std::map<std::string, Mapping> g_by_handle;  // handle bytes -> mapping
std::map<void*, std::string> g_by_ptr;       // pointer returned by cc_ipc_open -> handle bytes
std::map<void*, int> g_ptr_refs;             // opens outstanding per returned pointer

}  // namespace

extern "C" {

size_t cc_ipc_handle_bytes(void) { return sizeof(cudaIpcMemHandle_t); }

cc_status cc_ipc_export(const void* dev_ptr, void* handle, size_t* offset) {
  if (!dev_ptr || !handle || !offset) return CC_ERR_INVALID_ARG;
  GetRangeFn range = get_range_fn();
  if (!range) return CC_ERR_CUDA;
  unsigned long long base = 0;
  size_t size = 0;
  if (range(&base, &size, (unsigned long long)(uintptr_t)dev_ptr) != 0) return CC_ERR_INVALID_ARG;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void*>((uintptr_t)base)) != cudaSuccess) return CC_ERR_CUDA;
  std::memcpy(handle, &h, sizeof(h));
  *offset = (size_t)((uintptr_t)dev_ptr - (uintptr_t)base);
  return CC_OK;
}

cc_status cc_ipc_open(const void* handle, size_t offset, void** dev_ptr) {
  if (!handle || !dev_ptr) return CC_ERR_INVALID_ARG;
  const std::string key(static_cast<const char*>(handle), sizeof(cudaIpcMemHandle_t));
  std::lock_guard<std::mutex> lock(g_mu);
  Mapping& m = g_by_handle[key];
  if (m.refs == 0) {
    cudaIpcMemHandle_t h;
    std::memcpy(&h, handle, sizeof(h));
    void* base = nullptr;
    if (cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess) {
      g_by_handle.erase(key);
      cudaGetLastError();  // a failed open is not a sticky error; clear it for later calls
      return CC_ERR_CUDA;
    }
    m.base = base;
  }
  ++m.refs;
  void* p = static_cast<char*>(m.base) + offset;
  g_by_ptr[p] = key;
  ++g_ptr_refs[p];
  *dev_ptr = p;
  return CC_OK;
}

cc_status cc_ipc_close(void* dev_ptr) {
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = g_by_ptr.find(dev_ptr);
  if (it == g_by_ptr.end()) return CC_ERR_INVALID_ARG;
  const std::string key = it->second;
  if (--g_ptr_refs[dev_ptr] == 0) {
    g_ptr_refs.erase(dev_ptr);
    g_by_ptr.erase(it);
  }
  Mapping& m = g_by_handle[key];
  if (--m.refs == 0) {
    const cudaError_t e = cudaIpcCloseMemHandle(m.base);
    g_by_handle.erase(key);
    if (e != cudaSuccess) return CC_ERR_CUDA;
  }
  return CC_OK;
}

}  // extern "C"
