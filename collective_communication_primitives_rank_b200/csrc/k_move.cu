// Data-movement kernel: allgather, broadcast, scatter, gather, bucket flatten/unflatten.
//
// All of them are "copy entry k (src, bytes) to one destination, or to the same offset
// of every rank's buffer" (fan-out). The kernel reads each source byte once and writes it
// to each destination: allgather reads T and writes N·T, the minimum. Entries are cut
// into 64 KiB tiles; a CTA takes tiles round-robin (binary search in the tile prefix
// table) and moves them with 128-bit streaming loads/stores when every address of the
// entry is 16-byte aligned, element by element otherwise.
#include <algorithm>

#include "cc_device.cuh"
#include "cc_launch.h"

namespace cc {

constexpr int kCopyThreads = 256;
constexpr int kCopyMaxEntries = 128;
constexpr uint64_t kCopyTile = 64 * 1024;  // bytes

struct CopyParams {
  int nentries;
  int fanout;
  int ndst;
  int skip;
  uint32_t esize;
  uint32_t tile_prefix[kCopyMaxEntries + 1];
  uint64_t vec_mask[kCopyMaxEntries / 64];
  const char* src[kCopyMaxEntries];
  char* dst[kCopyMaxEntries];
  uint64_t nbytes[kCopyMaxEntries];
  uint64_t dst_off[kCopyMaxEntries];
  char* dst_base[kMaxRanks];
};

__device__ __forceinline__ void copy_elem(char* d, const char* s, uint32_t esize) {
  if (esize == 4) __stcs(reinterpret_cast<unsigned*>(d), __ldcs(reinterpret_cast<const unsigned*>(s)));
  else __stcs(reinterpret_cast<unsigned short*>(d), __ldcs(reinterpret_cast<const unsigned short*>(s)));
}

__global__ void __launch_bounds__(kCopyThreads) copy_kernel(const __grid_constant__ CopyParams P) {
  const uint32_t ntiles = P.tile_prefix[P.nentries];
  for (uint32_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
    int lo = 0, hi = P.nentries - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (P.tile_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int k = lo;
    const char* src = P.src[k];
    const uint64_t a = (uint64_t)(tile - P.tile_prefix[k]) * kCopyTile;
    const uint64_t b = min(a + kCopyTile, P.nbytes[k]);
    const bool vec = (P.vec_mask[k >> 6] >> (k & 63)) & 1;
    const uint64_t vb = vec ? a + (b - a) / 16 * 16 : a;
    for (uint64_t o = a + threadIdx.x * 16ull; o < vb; o += kCopyThreads * 16ull) {
      const uint4 v = __ldcs(reinterpret_cast<const uint4*>(src + o));
      if (P.fanout) {
        for (int r = 0; r < P.ndst; ++r)
          if (r != P.skip) __stcs(reinterpret_cast<uint4*>(P.dst_base[r] + P.dst_off[k] + o), v);
      } else {
        __stcs(reinterpret_cast<uint4*>(P.dst[k] + o), v);
      }
    }
    for (uint64_t o = vb + threadIdx.x * (uint64_t)P.esize; o < b; o += (uint64_t)kCopyThreads * P.esize) {
      if (P.fanout) {
        for (int r = 0; r < P.ndst; ++r)
          if (r != P.skip) copy_elem(P.dst_base[r] + P.dst_off[k] + o, src + o, P.esize);
      } else {
        copy_elem(P.dst[k] + o, src + o, P.esize);
      }
    }
  }
}

static bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

cudaError_t launch_copy(const CopyEntry* entries, int nentries, void* const* dst_base, int ndst, bool fanout,
                        int skip, size_t elem_bytes, cudaStream_t stream) {
  static int bps = 0;
  if (!bps && (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, copy_kernel, kCopyThreads, 0) != cudaSuccess || bps <= 0))
    bps = 4;
  bool bases_aligned = true;
  for (int r = 0; r < ndst && fanout; ++r)
    if (r != skip) bases_aligned = bases_aligned && al16(dst_base[r]);
  for (int first = 0; first < nentries; first += kCopyMaxEntries) {
    CopyParams P{};
    P.fanout = fanout;
    P.ndst = ndst;
    P.skip = skip;
    P.esize = (uint32_t)elem_bytes;
    for (int r = 0; r < ndst && fanout; ++r) P.dst_base[r] = static_cast<char*>(dst_base[r]);
    uint32_t tiles = 0;
    int m = 0;
    const int last = std::min(nentries, first + kCopyMaxEntries);
    for (int k = first; k < last; ++k) {
      const CopyEntry& e = entries[k];
      const uint64_t nb = e.numel * elem_bytes;
      if (nb == 0) continue;
      P.src[m] = static_cast<const char*>(e.src);
      P.dst[m] = fanout ? nullptr : static_cast<char*>(e.dst) + e.dst_off * elem_bytes;
      P.nbytes[m] = nb;
      P.dst_off[m] = e.dst_off * elem_bytes;
      const bool v = al16(P.src[m]) && (fanout ? bases_aligned && (P.dst_off[m] % 16 == 0) : al16(P.dst[m]));
      if (v) P.vec_mask[m >> 6] |= 1ull << (m & 63);
      P.tile_prefix[m] = tiles;
      tiles += (uint32_t)((nb + kCopyTile - 1) / kCopyTile);
      ++m;
    }
    P.nentries = m;
    P.tile_prefix[m] = tiles;
    if (tiles == 0) continue;
    const uint32_t grid = std::min<uint32_t>(tiles, (uint32_t)(sm_count() * bps));
    copy_kernel<<<grid, kCopyThreads, 0, stream>>>(P);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace cc
