// Data-movement kernels: allgather, broadcast, scatter, gather, bucket flatten/unflatten.
//
// All of them are "copy entry k (src, bytes) to one destination, or to the same offset
// of every rank's buffer" (fan-out). Each source byte is read once and written to each
// destination: allgather reads T and writes N·T, the minimum. Entries are cut into tiles;
// a CTA finds its tile's entry by binary search in the tile prefix table.
//
// copy_bulk_tile_kernel (every entry 16-byte aligned): the tensor memory accelerator moves
// the data. One CTA per tile; its one working thread issues a cp.async.bulk load of the
// tile into shared memory (completion on an mbarrier), then one cp.async.bulk store of the
// same shared-memory tile per destination, so a tile costs the SM a handful of instructions
// however many replicas it has, and several CTAs per SM keep loads in flight. (Measured
// against a persistent 4-stage pipeline per SM: 98–100% vs 88% of the copy rate.) Tiles are
// 2 KiB (32 CTAs per SM) for a launch that reads less than 1 GiB and 32 KiB above: measured on
// allgather N = 8..64 × 16–512 MiB, broadcast and scatter, 2 KiB tiles took the write-heavy
// fan-out from 5.3–6.5 to 6.2–6.8 TB/s, while the 1.2 GB shards of an N = 8 allgather ran 2%
// slower with them than with 32 KiB tiles; 1 KiB tiles halved a one-destination copy.
// The wait is bounded: one that gives up records CC_ERR_TIMEOUT in the device status word.
//
// copy_kernel (any alignment, and every copy that touches peer memory): 128-bit streaming
// loads/stores, four in flight per thread, where source and destinations share their offset
// from a 16-byte boundary; where only the destinations share theirs, 128-bit stores with each
// 16 bytes loaded element by element; element copies, eight in flight per thread, for the rest.
// The 128-bit part starts on a 128-byte line of the buffer it is aligned to. Measured on an
// allgather N = 8 × 256 MiB, fp32: shards one element off, outputs aligned 1.25 TB/s one
// element at a time, 4.79 with eight in flight, 5.16 with the 128-bit stores; shards aligned,
// outputs one element off 2.25 element-wise, 3.62 with 128-bit stores from a 16-byte boundary,
// 4.53 from a line.
#include <algorithm>
#include <mutex>

#include "cc_device.cuh"
#include "cc_launch.h"

namespace cc {

constexpr int kCopyThreads = 256;
constexpr int kCopyMaxEntries = 128;
constexpr uint64_t kCopyTile = 64 * 1024;  // bytes

struct CopyParams {
  uint32_t bulk_tile;  // bytes per CTA of copy_bulk_tile_kernel
  int nentries;
  int fanout;
  int ndst;
  int skip;
  uint32_t esize;
  uint32_t tile_prefix[kCopyMaxEntries + 1];
  uint64_t vec_mask[kCopyMaxEntries / 64];   // every address of the entry 16-byte aligned
  uint64_t coal_mask[kCopyMaxEntries / 64];  // source and destinations equal modulo 16 bytes
  uint64_t dco_mask[kCopyMaxEntries / 64];   // the destinations equal modulo 16 bytes (not the source)
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

// Element-wise part of a tile, kCopyElems elements per thread in flight before their stores;
// the 128-bit part keeps kCopyVecs loads per thread in flight.
constexpr int kCopyElems = 8;
constexpr int kCopyVecs = 4;

template <typename E>
__device__ __forceinline__ void copy_elems(const CopyParams& P, int k, const char* src, uint64_t lo, uint64_t hi) {
  constexpr uint64_t ES = sizeof(E);
  for (uint64_t o0 = lo + threadIdx.x * ES; o0 < hi; o0 += (uint64_t)kCopyThreads * ES * kCopyElems) {
    E v[kCopyElems];
#pragma unroll
    for (int q = 0; q < kCopyElems; ++q) {
      const uint64_t o = o0 + (uint64_t)q * kCopyThreads * ES;
      if (o < hi) v[q] = __ldcs(reinterpret_cast<const E*>(src + o));
    }
#pragma unroll
    for (int q = 0; q < kCopyElems; ++q) {
      const uint64_t o = o0 + (uint64_t)q * kCopyThreads * ES;
      if (o >= hi) continue;
      if (P.fanout) {
        for (int r = 0; r < P.ndst; ++r)
          if (r != P.skip) __stcs(reinterpret_cast<E*>(P.dst_base[r] + P.dst_off[k] + o), v[q]);
      } else {
        __stcs(reinterpret_cast<E*>(P.dst[k] + o), v[q]);
      }
    }
  }
}

// 16 bytes from a source that is only element-aligned: element loads, packed.
template <typename E>
__device__ __forceinline__ uint4 load16_elems(const char* p) {
  if constexpr (sizeof(E) == 4) {
    const unsigned* q = reinterpret_cast<const unsigned*>(p);
    return make_uint4(__ldcs(q), __ldcs(q + 1), __ldcs(q + 2), __ldcs(q + 3));
  } else {
    const unsigned short* q = reinterpret_cast<const unsigned short*>(p);
    unsigned w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w[i] = (unsigned)__ldcs(q + 2 * i) | ((unsigned)__ldcs(q + 2 * i + 1) << 16);
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// One tile of an entry: 128-bit loads and stores over the part where the source and every
// destination sit on 16-byte boundaries (the whole tile when all are aligned; after a head of
// under 16 bytes when they are equally misaligned); where only the destinations share their
// offset, 128-bit stores on their boundaries with each 16 bytes loaded element by element;
// element copies for the rest.
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
    const bool coal = (P.coal_mask[k >> 6] >> (k & 63)) & 1;
    const bool dco = !vec && !coal && ((P.dco_mask[k >> 6] >> (k & 63)) & 1);
    uint64_t va = a, vb = a;
    if (vec || coal || dco) {
      // the 16-byte boundaries of the source, or of the destinations (the first one written);
      // the 128-bit part starts on a 128-byte line of that buffer, so that each warp's 512
      // bytes fill four whole lines
      const uintptr_t at = dco ? (P.fanout ? reinterpret_cast<uintptr_t>(P.dst_base[P.skip == 0 && P.ndst > 1 ? 1 : 0]) + P.dst_off[k]
                                           : reinterpret_cast<uintptr_t>(P.dst[k]))
                               : reinterpret_cast<uintptr_t>(src);
      const uint64_t head = (128 - ((at + a) & 127)) & 127;
      va = min(b, a + head);
      vb = va + (b - va) / 16 * 16;
    }
    for (uint64_t o0 = va + threadIdx.x * 16ull; o0 < vb; o0 += kCopyThreads * 16ull * kCopyVecs) {
      uint4 v[kCopyVecs];
#pragma unroll
      for (int q = 0; q < kCopyVecs; ++q) {
        const uint64_t o = o0 + (uint64_t)q * kCopyThreads * 16;
        if (o < vb) {
          if (!dco) v[q] = __ldcs(reinterpret_cast<const uint4*>(src + o));
          else if (P.esize == 4) v[q] = load16_elems<unsigned>(src + o);
          else v[q] = load16_elems<unsigned short>(src + o);
        }
      }
#pragma unroll
      for (int q = 0; q < kCopyVecs; ++q) {
        const uint64_t o = o0 + (uint64_t)q * kCopyThreads * 16;
        if (o >= vb) continue;
        if (P.fanout) {
          for (int r = 0; r < P.ndst; ++r)
            if (r != P.skip) __stcs(reinterpret_cast<uint4*>(P.dst_base[r] + P.dst_off[k] + o), v[q]);
        } else {
          __stcs(reinterpret_cast<uint4*>(P.dst[k] + o), v[q]);
        }
      }
    }
    if (P.esize == 4) {
      copy_elems<unsigned>(P, k, src, a, va);
      copy_elems<unsigned>(P, k, src, vb, b);
    } else {
      copy_elems<unsigned short>(P, k, src, a, va);
      copy_elems<unsigned short>(P, k, src, vb, b);
    }
  }
}

// ---- bulk (TMA) path ----------------------------------------------------------------------------

__device__ int g_async_status;  // CC_OK, or CC_ERR_TIMEOUT after a bounded wait gave up

constexpr uint32_t kBulkTileSmall = 2 * 1024;   // bytes; multiples of 16
constexpr uint32_t kBulkTileLarge = 32 * 1024;
constexpr uint64_t kBulkLargeLaunch = 1ull << 30;  // source bytes from which a launch takes large tiles
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // a wait gives up after 2 s (no load takes that long)
constexpr long kWaitPolls = 1l << 30;             // and after this many polls, whatever the clock says

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t* m) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(m)));
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* m, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(m)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* m, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
      : "=r"(ok) : "r"(smem_addr(m)), "r"(parity) : "memory");
  return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}
// Bounded wait for the phase `parity` of an mbarrier; on giving up it records
// CC_ERR_TIMEOUT in the device status word and returns false.
__device__ __forceinline__ bool mbar_wait(uint64_t* m, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
  const uint64_t t0 = global_ns();
  for (long i = 0; i < kWaitPolls; ++i) {
    if (mbar_test(m, parity)) return true;
    if (global_ns() - t0 > limit_ns) break;
  }
  atomicExch(&g_async_status, (int)CC_ERR_TIMEOUT);
  return false;
}

// Self-test of the bounded-wait path: one thread waits on an mbarrier that nothing will
// ever arrive at, gives up after limit_ns and records CC_ERR_TIMEOUT. No fault, no trap:
// the context stays usable.
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&bar)));
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  mbar_wait(&bar, 0, limit_ns);
}
__device__ __forceinline__ void bulk_load(void* smem, const void* gmem, uint32_t bytes, uint64_t* m) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_addr(smem)), "l"(gmem), "r"(bytes), "r"(smem_addr(m)) : "memory");
}
__device__ __forceinline__ void bulk_store(void* gmem, const void* smem, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
               ::"l"(gmem), "r"(smem_addr(smem)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// One tile per CTA, no pipeline inside the CTA: load the tile, store it to every
// destination, wait until the stores have read shared memory, exit. Several CTAs per SM
// keep loads in flight; the hardware hands out tiles as CTAs finish.
__global__ void __launch_bounds__(32) copy_bulk_tile_kernel(const __grid_constant__ CopyParams P) {
  extern __shared__ __align__(128) unsigned char smem[];
  const uint32_t tile_bytes = P.bulk_tile;
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + tile_bytes);
  if (threadIdx.x != 0) return;
  const uint32_t tile = blockIdx.x;
  if (tile >= P.tile_prefix[P.nentries]) return;
  int lo = 0, hi = P.nentries - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (P.tile_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  const int k = lo;
  const uint64_t a = (uint64_t)(tile - P.tile_prefix[k]) * tile_bytes;
  const uint64_t nb = P.nbytes[k];
  // An entry whose source sits h0 bytes before a 16-byte boundary (its destinations the same):
  // tile t moves [a + h0, a + h0 + tile) in bulk, clipped to the entry; the entry's first h0
  // bytes (tile 0) and a last partial 16 bytes go element by element. h0 = 0 when aligned.
  const uint64_t h0 = (16 - (reinterpret_cast<uintptr_t>(P.src[k]) & 15)) & 15;
  const uint64_t blo = min(nb, a + h0), bhi = min(nb, a + tile_bytes + h0);
  const uint32_t bulk = (uint32_t)((bhi - blo) & ~15ull);
  if (bulk) {
    mbar_init(bar);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_arrive_tx(bar, bulk);
    bulk_load(smem, P.src[k] + blo, bulk, bar);
    if (!mbar_wait(bar, 0)) {
      // one more bounded chance for the load to land before leaving. If it still has not,
      // the CTA leaves with the bulk load in flight: that load may still write this CTA's
      // shared memory after the SM has handed it to another CTA (of this or any kernel),
      // so the outputs of this call and of whatever runs next on that SM are undefined; the
      // status word reads CC_ERR_TIMEOUT (only a memory system that stalls a 2 KiB read for
      // seconds gets here)
      mbar_wait(bar, 0);
      return;
    }
  }
  for (int r = 0; r < (P.fanout ? P.ndst : 1); ++r) {
    if (P.fanout && r == P.skip) continue;
    char* d = P.fanout ? P.dst_base[r] + P.dst_off[k] : P.dst[k];
    if (bulk) bulk_store(d + blo, smem, bulk);
    if (a == 0)
      for (uint64_t o = 0; o < min(h0, nb); o += P.esize) copy_elem(d + o, P.src[k] + o, P.esize);
    for (uint64_t o = blo + bulk; o < bhi; o += P.esize) copy_elem(d + o, P.src[k] + o, P.esize);
  }
  bulk_commit();
  bulk_wait_all();
}

static bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int* async_status_word() {
  // looked up with the device current; only a successful lookup is kept, so a failed one
  // (for instance during a stream capture) is retried by the next call
  static int* ptr[64];
  static std::mutex mu[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu[dev]);
  if (!ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_async_status) == cudaSuccess) ptr[dev] = static_cast<int*>(p);
    else cudaGetLastError();
  }
  return ptr[dev];
}

cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, cudaStream_t stream) {
  bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns);
  return cudaGetLastError();
}

cudaError_t read_async_status(int* out, bool reset, cudaStream_t stream) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_async_status, sizeof(int), 0, cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess && reset) {
    const int zero = 0;
    e = cudaMemcpyToSymbolAsync(g_async_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  }
  return e;
}

cudaError_t launch_copy(const CopyEntry* entries, int nentries, void* const* dst_base, int ndst, bool fanout,
                        int skip, size_t elem_bytes, cudaStream_t stream, bool plain) {
  static int bps = 0;
  if (!bps && (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&bps, copy_kernel, kCopyThreads, 0) != cudaSuccess || bps <= 0))
    bps = 4;
  static const size_t bulk_smem = (size_t)kBulkTileLarge + 16;
  static const cudaError_t bulk_attr =
      cudaFuncSetAttribute(copy_bulk_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bulk_smem);
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
      // equally misaligned source and destinations: 128-bit copies after a short head
      bool c = true;
      const uintptr_t sa = reinterpret_cast<uintptr_t>(P.src[m]) & 15;
      if (fanout) {
        for (int r = 0; r < ndst; ++r)
          if (r != skip) c = c && ((reinterpret_cast<uintptr_t>(P.dst_base[r]) + P.dst_off[m]) & 15) == sa;
      } else {
        c = (reinterpret_cast<uintptr_t>(P.dst[m]) & 15) == sa;
      }
      if (c) P.coal_mask[m >> 6] |= 1ull << (m & 63);
      // destinations at one offset among themselves (a whole number of elements, as the source)
      bool dc = (reinterpret_cast<uintptr_t>(P.src[m]) % elem_bytes) == 0;
      uintptr_t da = 16;
      if (fanout) {
        for (int r = 0; r < ndst; ++r) {
          if (r == skip) continue;
          const uintptr_t x = (reinterpret_cast<uintptr_t>(P.dst_base[r]) + P.dst_off[m]) & 15;
          if (da == 16) da = x;
          dc = dc && x == da && x % elem_bytes == 0;
        }
      } else {
        da = reinterpret_cast<uintptr_t>(P.dst[m]) & 15;
        dc = dc && da % elem_bytes == 0;
      }
      if (dc) P.dco_mask[m >> 6] |= 1ull << (m & 63);
      P.tile_prefix[m] = tiles;
      tiles += (uint32_t)((nb + kCopyTile - 1) / kCopyTile);
      ++m;
    }
    P.nentries = m;
    P.tile_prefix[m] = tiles;
    if (tiles == 0) continue;
    // the bulk kernel when every entry's source and destinations are equally aligned
    bool all_coal = true;
    for (int k = 0; k < m; ++k) all_coal = all_coal && ((P.coal_mask[k >> 6] >> (k & 63)) & 1);
    if (all_coal && !plain && bulk_attr == cudaSuccess) {
      // retile for the bulk kernel, one CTA per tile
      uint64_t total = 0;
      for (int k = 0; k < m; ++k) total += P.nbytes[k];
      P.bulk_tile = total >= kBulkLargeLaunch ? kBulkTileLarge : kBulkTileSmall;
      uint32_t bt = 0;
      for (int k = 0; k < m; ++k) {
        P.tile_prefix[k] = bt;
        bt += (uint32_t)((P.nbytes[k] + P.bulk_tile - 1) / P.bulk_tile);
      }
      P.tile_prefix[m] = bt;
      copy_bulk_tile_kernel<<<bt, 32, (size_t)P.bulk_tile + 16, stream>>>(P);
    } else {
      const uint32_t grid = std::min<uint32_t>(tiles, (uint32_t)(sm_count() * bps));
      copy_kernel<<<grid, kCopyThreads, 0, stream>>>(P);
    }
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

}  // namespace cc
