// mk_probe.cu -- read-only HBM streaming probe.
//
// The decode step only reads its weights and KV cache, so its bandwidth
// ceiling is a pure read stream, not the read+write copy that the measured
// peak of the pool is.  This kernel measures that ceiling on the device it
// runs on: every byte of a large buffer is read exactly once per pass with
// 16-byte loads that bypass L1, eight loads in flight per thread, over a grid
// of whole waves of resident blocks; nothing is written except one word per
// block (so the loads cannot be dropped).  Two forms: plain vector loads, and
// bulk asynchronous copies into shared memory (cp.async.bulk, the same
// engine the megakernel's weight ring uses).
#include <cstdint>
#include <cstdio>

#include "mk_internal.h"

namespace mk {
namespace {

constexpr int kProbeThreads = 512;
constexpr int kProbeUnroll = 8;

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Each thread reads kProbeUnroll 16-byte words per round, a block's words
// contiguous; rounds stride over the whole grid.
__global__ void __launch_bounds__(kProbeThreads) probe_ld_kernel(const uint4 *buf, size_t n16, uint32_t *sink) {
  const size_t per_round = static_cast<size_t>(gridDim.x) * kProbeThreads * kProbeUnroll;
  uint32_t acc = 0;
  for (size_t base = static_cast<size_t>(blockIdx.x) * kProbeThreads * kProbeUnroll + threadIdx.x; base < n16;
       base += per_round) {
    uint4 v[kProbeUnroll];
#pragma unroll
    for (int k = 0; k < kProbeUnroll; ++k) {
      const size_t i = base + static_cast<size_t>(k) * kProbeThreads;
      v[k] = i < n16 ? ld_stream(buf + i) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int k = 0; k < kProbeUnroll; ++k) acc ^= v[k].x ^ v[k].y ^ v[k].z ^ v[k].w;
  }
  acc = __reduce_xor_sync(0xffffffffu, acc);
  if ((threadIdx.x & 31) == 0) atomicXor(&sink[blockIdx.x], acc);
}

// Bulk form: one thread per block issues 32 KB bulk copies into a ring of
// four shared-memory buffers (mbarrier completion); the block then reads one
// word of each buffer back so that nothing can be elided.  Waits are bounded
// by %globaltimer; a wait that runs out sets the flag word sink[8 * gridDim.x]
// and the block stops.
constexpr int kBulkBytes = 32768;
constexpr int kBulkSlots = 4;

__device__ __forceinline__ uint32_t sa(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ uint64_t gtime() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__global__ void __launch_bounds__(128) probe_bulk_kernel(const uint8_t *buf, size_t bytes, uint32_t *sink) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t bar[kBulkSlots];
  __shared__ int s_ok;
  const size_t chunks = bytes / kBulkBytes;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kBulkSlots; ++s)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sa(&bar[s])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  uint32_t acc = 0;
  size_t issued = 0, done = 0;
  const size_t mine = chunks > blockIdx.x ? (chunks - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  bool failed = false;
  while (done < mine && !failed) {
    if (threadIdx.x == 0) {
      while (issued < mine && issued < done + kBulkSlots) {
        const int s = static_cast<int>(issued % kBulkSlots);
        const size_t c = blockIdx.x + issued * gridDim.x;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(sa(&bar[s])), "r"(kBulkBytes)
                     : "memory");
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                sa(smem + s * kBulkBytes)),
            "l"(buf + c * kBulkBytes), "r"(kBulkBytes), "r"(sa(&bar[s]))
            : "memory");
        ++issued;
      }
    }
    // thread 0 waits (bounded) for the slot; the block follows its decision
    const int s = static_cast<int>(done % kBulkSlots);
    if (threadIdx.x == 0) {
      const uint32_t par = static_cast<uint32_t>((done / kBulkSlots) & 1);
      const uint64_t t0 = gtime();
      int ok = 0;
      for (;;) {
        uint32_t r;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
            : "=r"(r)
            : "r"(sa(&bar[s])), "r"(par)
            : "memory");
        if (r) {
          ok = 1;
          break;
        }
        if (gtime() - t0 > 1000000000ull) break;
      }
      s_ok = ok;
      if (!ok) atomicExch(&sink[8 * gridDim.x], 1u);
    }
    __syncthreads();
    if (!s_ok) {
      failed = true;
      break;
    }
    acc ^= reinterpret_cast<const uint32_t *>(smem + s * kBulkBytes)[threadIdx.x * 64];
    ++done;
    __syncthreads();  // every thread has read slot s before it is refilled
  }
  // a block that stopped on a timeout still waits (bounded) for its copies in flight
  if (threadIdx.x == 0) {
    for (size_t k = done; k < issued; ++k) {
      const int s = static_cast<int>(k % kBulkSlots);
      const uint32_t par = static_cast<uint32_t>((k / kBulkSlots) & 1);
      const uint64_t t0 = gtime();
      for (;;) {
        uint32_t ok;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
            : "=r"(ok)
            : "r"(sa(&bar[s])), "r"(par)
            : "memory");
        if (ok || gtime() - t0 > 50000000ull) break;
      }
    }
  }
  acc = __reduce_xor_sync(0xffffffffu, acc);
  if ((threadIdx.x & 31) == 0) atomicXor(&sink[blockIdx.x], acc);
}

}  // namespace

size_t probe_sink_words(int n_sm) { return static_cast<size_t>(n_sm) * 8 + 1; }

cudaError_t launch_read_probe(const void *buf, size_t bytes, int form, int n_sm, uint32_t *sink, cudaStream_t s) {
  if (form == 0) {
    int per = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, probe_ld_kernel, kProbeThreads, 0);
    if (e != cudaSuccess) return e;
    if (per < 1) per = 1;
    if (per > 8) per = 8;
    probe_ld_kernel<<<n_sm * per, kProbeThreads, 0, s>>>(static_cast<const uint4 *>(buf), bytes / 16, sink);
    return cudaGetLastError();
  }
  static bool attr_set = false;
  const int smem = kBulkSlots * kBulkBytes;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(probe_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  // one block of 128 KB per SM: the whole grid is one wave
  probe_bulk_kernel<<<n_sm, 128, smem, s>>>(static_cast<const uint8_t *>(buf), bytes, sink);
  return cudaGetLastError();
}

}  // namespace mk
