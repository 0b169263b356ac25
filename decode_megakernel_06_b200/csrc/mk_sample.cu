// mk_sample.cu -- temperature / top-p (nucleus) sampling of one token per
// logits row, the sampler that can stand in place of the decode step's argmax
// (tpu-megakernels README, serving demos: greedy or temperature / top-p
// generation; the nucleus itself is Holtzman et al. 2020, section 3.1).
//
// What is computed, per row of V fp32 logits l, with one uniform u in [0, 1):
//   p_i = exp((l_i - max l) / T) in fp64; q_i = round_half_even(p_i * 2^46),
//   an exact fixed-point mass (every later sum is an integer sum, so no
//   decision depends on a summation order); need = max(1, min(Q, ceil(top_p *
//   Q))), Q = sum q, the product in fp64; the nucleus is the smallest prefix of the tokens sorted by
//   logit, descending, ties by lower id, whose mass reaches need; the token is
//   the first nucleus id, in id order, whose cumulative mass exceeds
//   y = min(S - 1, floor(u * S)), S the nucleus mass.  T <= 0 is greedy: the
//   argmax, lowest id on ties.
//
// Design.  One cluster of kSampleCluster CTAs per row, each CTA holding a
// contiguous slice of the row in shared memory (logits and masses) for the
// whole kernel, so the row is read from memory once.  The nucleus threshold is
// a radix select on an order-preserving 32-bit key of the logit, one byte per
// pass from the top: every CTA builds a histogram of fixed-point mass per
// digit value over its slice, the histograms are summed through distributed
// shared memory, and every CTA takes the same decision from the same integer
// totals.  After four passes the threshold key tau, the mass above it and the
// number r of tokens tied at tau that enter the nucleus are known.  The draw is
// an inverse CDF in id order: per-warp segment totals are summed across the
// cluster, and only the warp whose segment holds the point y scans its
// segment, 32 tokens at a time.  Seven cluster barriers when sampling, three
// when greedy; no spin-waits.
#include <cooperative_groups.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "mk_internal.h"

namespace cg = cooperative_groups;

namespace mk {
namespace {

constexpr int kSThreads = kSampleThreads;
constexpr int kSWarps = kSThreads / 32;
constexpr int kHistCopies = 8;  // warp w adds into copy w % 8
constexpr double kMassScale = 70368744177664.0;  // 2^46
constexpr int kSampleMaxDevices = 64;

// Order-preserving key: larger logit <-> larger key; -0 and +0 share one key.
__device__ __forceinline__ uint32_t logit_key(float x) {
  uint32_t b = __float_as_uint(x);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_logit(uint32_t k) {
  uint32_t b = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
  return __uint_as_float(b);
}

__device__ __forceinline__ uint64_t mass_of(float l, float m, double inv_t) {
  double z = ((double)l - (double)m) * inv_t;
  return __double2ull_rn(exp(z) * kMassScale);
}

__device__ __forceinline__ uint64_t warp_sum_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ uint64_t warp_incl_scan_u64(uint64_t v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint64_t t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// Adds mass q to bucket b of hist for every lane with `valid`; lanes that hit
// the same bucket are summed first and their lowest lane adds once, so a warp
// issues one atomic per distinct bucket instead of one per lane.  All 32 lanes
// must call it together; stage is this warp's 32-word scratch.
__device__ __forceinline__ void hist_add(uint64_t *hist, uint32_t b, uint64_t qv, bool valid,
                                         uint64_t *stage, int lane) {
  if (!__any_sync(0xffffffffu, valid)) return;
  const unsigned peers = __match_any_sync(0xffffffffu, valid ? b : 0xffffffffu);
  stage[lane] = qv;
  __syncwarp();
  if (valid && lane == __ffs(peers) - 1) {
    uint64_t sum = 0;
    for (unsigned mm = peers; mm; mm &= mm - 1) sum += stage[__ffs(mm) - 1];
    atomicAdd(reinterpret_cast<unsigned long long *>(&hist[b]), (unsigned long long)sum);
  }
  __syncwarp();
}

struct SampleShared {
  uint64_t chist[2][256];   // this CTA's merged histogram, read by the cluster
  uint64_t tot[256];        // cluster totals of the current pass
  uint64_t seg[2];          // this CTA's (mass above tau, tokens at tau), read by the cluster
  uint64_t stage[kSWarps][32];  // per-warp scratch of hist_add
  uint64_t wmass[kSWarps];   // per-warp segment totals
  uint32_t wtie[kSWarps];
  uint32_t wkey[kSWarps];
  int32_t wid[kSWarps];
  uint32_t cta_key;         // this CTA's largest key, read by the cluster
  int32_t cta_id;           // this CTA's lowest argmax id, read by the cluster
  uint32_t gmax_key;
  uint32_t prefix;          // key bits fixed so far
  uint64_t above;           // mass of keys above the current bucket range
  uint64_t need;
};

// Phase clock (stamps != nullptr): thread 0 of the first CTA of row 0 records
// %globaltimer at each phase boundary, stamps[0 .. kSamplePhases).
__device__ __forceinline__ void phase_stamp(unsigned long long *stamps, int i, bool me) {
  if (stamps && me) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    stamps[i] = t;
  }
}

__global__ void __launch_bounds__(kSThreads, 1)
top_p_kernel(const float *__restrict__ logits, int vocab, int slice, double inv_t, float top_p,
             int greedy, int vec4, const double *__restrict__ uniforms, int32_t *__restrict__ out,
             unsigned long long *stamps) {
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) unsigned char dyn[];
  __shared__ SampleShared sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned rank = cluster.block_rank();
  const int row = blockIdx.x / kSampleCluster;
  const int lo = (int)rank * slice;
  const int n = max(0, min(slice, vocab - lo));
  uint64_t *q = reinterpret_cast<uint64_t *>(dyn);
  float *l = reinterpret_cast<float *>(dyn + sizeof(uint64_t) * (size_t)slice);
  uint64_t *whist = reinterpret_cast<uint64_t *>(dyn + 12 * (size_t)((slice + 1) & ~1));
  const float *src = logits + (size_t)row * vocab + lo;
  const bool stamper = row == 0 && rank == 0 && tid == 0;
  phase_stamp(stamps, 0, stamper);

  for (int i = tid; i < kHistCopies * 256; i += kSThreads) whist[i] = 0;
  // ---- load the slice; this CTA's largest key --------------------------------
  uint32_t kmax = 0;
  if (vec4) {  // rows and slices start on 16-byte boundaries and n % 4 == 0
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
    float4 *l4 = reinterpret_cast<float4 *>(l);
#pragma unroll 4
    for (int i = tid; i < n / 4; i += kSThreads) {
      float4 x = s4[i];
      l4[i] = x;
      kmax = max(max(kmax, max(logit_key(x.x), logit_key(x.y))), max(logit_key(x.z), logit_key(x.w)));
    }
  } else {
#pragma unroll 8
    for (int i = tid; i < n; i += kSThreads) {
      float x = src[i];
      l[i] = x;
      kmax = max(kmax, logit_key(x));
    }
  }
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) sh.wkey[warp] = kmax;
  __syncthreads();
  if (tid == 0) {
    uint32_t k = 0;
    for (int w = 0; w < kSWarps; ++w) k = max(k, sh.wkey[w]);
    sh.cta_key = k;
  }
  phase_stamp(stamps, 1, stamper);
  cluster.sync();  // 1: every CTA's largest key is visible
  phase_stamp(stamps, 2, stamper);
  if (tid == 0) {
    uint32_t k = 0;
    for (unsigned r = 0; r < kSampleCluster; ++r) k = max(k, cluster.map_shared_rank(&sh.cta_key, r)[0]);
    sh.gmax_key = k;
  }
  __syncthreads();
  const uint32_t gkey = sh.gmax_key;

  if (greedy) {
    // ---- argmax, lowest id on ties ---------------------------------------------
    int best = 0x7fffffff;
    for (int i = tid; i < n; i += kSThreads)
      if (logit_key(l[i]) == gkey) { best = lo + i; break; }  // i rises: the first hit is this thread's lowest
    best = __reduce_min_sync(0xffffffffu, best);
    if (lane == 0) sh.wid[warp] = best;
    __syncthreads();
    if (tid == 0) {
      int b = 0x7fffffff;
      for (int w = 0; w < kSWarps; ++w) b = min(b, sh.wid[w]);
      sh.cta_id = b;
    }
    cluster.sync();  // 2
    if (rank == 0 && tid == 0) {
      int b = 0x7fffffff;
      for (unsigned r = 0; r < kSampleCluster; ++r) b = min(b, cluster.map_shared_rank(&sh.cta_id, r)[0]);
      out[row] = b;
    }
    cluster.sync();  // 3: no CTA leaves while its shared memory is being read
    return;
  }

  // ---- masses and the histogram of the top key byte ------------------------------
  const float m = key_logit(gkey);
  uint64_t *myhist = whist + (warp % kHistCopies) * 256;
  uint64_t *stage = sh.stage[warp];
  for (int i0 = tid - lane; i0 < n; i0 += kSThreads) {  // warp-uniform trip count
    const int i = i0 + lane;
    uint64_t qi = 0;
    uint32_t k = 0;
    if (i < n) {
      float x = l[i];
      qi = mass_of(x, m, inv_t);
      q[i] = qi;
      k = logit_key(x);
    }
    hist_add(myhist, k >> 24, qi, qi != 0, stage, lane);
  }
  if (tid == 0) {
    sh.prefix = 0;
    sh.above = 0;
  }
  phase_stamp(stamps, 3, stamper);

  // ---- radix select of the threshold key, one byte per pass -----------------------
  for (int d = 0; d < 4; ++d) {
    const int buf = d & 1;
    __syncthreads();
    if (tid < 256) {
      uint64_t s = 0;
#pragma unroll
      for (int c = 0; c < kHistCopies; ++c) {
        s += whist[c * 256 + tid];
        whist[c * 256 + tid] = 0;
      }
      sh.chist[buf][tid] = s;
    }
    cluster.sync();  // 2..5: every CTA's histogram of this pass is visible
    if (tid < 256) {
      uint64_t s = 0;
#pragma unroll
      for (unsigned r = 0; r < kSampleCluster; ++r) s += cluster.map_shared_rank(&sh.chist[buf][0], r)[tid];
      sh.tot[tid] = s;
    }
    __syncthreads();
    if (warp == 0) {
      // lane j holds buckets 255 - 8j .. 248 - 8j, scanned from the top
      uint64_t v[8], s = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        v[k] = sh.tot[255 - 8 * lane - k];
        s += v[k];
      }
      if (d == 0) {
        uint64_t total = warp_sum_u64(s);
        if (lane == 0) {
          double x = ceil((double)top_p * __ull2double_rn(total));
          uint64_t need;
          if (!(x >= 1.0)) need = 1;  // also top_p NaN or negative
          else if (x >= 18446744073709551616.0) need = total;  // 2^64
          else need = min((uint64_t)x, total);
          sh.need = need > 0 ? need : 1;
        }
        __syncwarp();
      }
      const uint64_t need = sh.need, above = sh.above;
      uint64_t incl = warp_incl_scan_u64(s, lane) + above;
      unsigned hit = __ballot_sync(0xffffffffu, incl >= need);
      int jl = hit ? __ffs(hit) - 1 : 31;  // no lane reaches need only on non-finite input
      if (lane == jl) {
        uint64_t c = incl - s;
        int chosen = 248 - 8 * lane;  // fallback: the lowest bucket of this lane
        uint64_t new_above = c;
        for (int k = 0; k < 8; ++k) {
          if (c + v[k] >= need) {
            chosen = 255 - 8 * lane - k;
            new_above = c;
            break;
          }
          c += v[k];
          new_above = c;
        }
        sh.prefix = (sh.prefix << 8) | (uint32_t)chosen;
        sh.above = new_above;
      }
    }
    __syncthreads();
    if (d < 3) {
      const uint32_t pre = sh.prefix;
      const int shift = 24 - 8 * d;  // bits above the next digit
      for (int i0 = tid - lane; i0 < n; i0 += kSThreads) {  // warp-uniform trip count
        const int i = i0 + lane;
        uint32_t k = 0;
        uint64_t qi = 0;
        if (i < n) {
          k = logit_key(l[i]);
          qi = q[i];
        }
        hist_add(myhist, (k >> (shift - 8)) & 255u, qi, i < n && qi != 0 && (k >> shift) == pre, stage, lane);
      }
    }
    phase_stamp(stamps, 4 + d, stamper);
  }

  // ---- the nucleus: keys above tau, and the first r tokens at tau by id -----------
  const uint32_t tau = sh.prefix;
  const uint64_t above = sh.above, need = sh.need;
  uint64_t q_tau = mass_of(key_logit(tau), m, inv_t);
  if (q_tau == 0) q_tau = 1;  // only on non-finite input
  const uint64_t r = need > above ? (need - above + q_tau - 1) / q_tau : 1;
  const uint64_t S = above + r * q_tau;
  double uu = uniforms[row];
  if (!(uu >= 0.0)) uu = 0.0;
  uint64_t y = (uint64_t)floor(fmin(uu, 1.0) * __ull2double_rn(S));
  if (y >= S) y = S - 1;

  // ---- inverse CDF in id order: per-warp segment totals --------------------------
  const int seg = ((slice + kSWarps - 1) / kSWarps + 31) & ~31;
  const int s0 = warp * seg, s1 = min(n, s0 + seg);
  uint64_t gm = 0;
  uint32_t ge = 0;
  for (int i = s0 + lane; i < s1; i += 32) {
    uint32_t k = logit_key(l[i]);
    if (k > tau) gm += q[i];
    ge += (k == tau);
  }
  gm = warp_sum_u64(gm);
  ge = __reduce_add_sync(0xffffffffu, ge);
  if (lane == 0) {
    sh.wmass[warp] = gm;
    sh.wtie[warp] = ge;
  }
  __syncthreads();
  if (tid == 0) {
    uint64_t a = 0, e = 0;
    for (int w = 0; w < kSWarps; ++w) {
      a += sh.wmass[w];
      e += sh.wtie[w];
    }
    sh.seg[0] = a;
    sh.seg[1] = e;
  }
  phase_stamp(stamps, 8, stamper);
  cluster.sync();  // 6: every CTA's segment totals are visible
  phase_stamp(stamps, 9, stamper);
  // mass above tau and tokens at tau before this warp's segment, over the row
  uint64_t gb = 0, eb = 0;
  for (unsigned rr = 0; rr < rank; ++rr) {
    const uint64_t *o = cluster.map_shared_rank(&sh.seg[0], rr);
    gb += o[0];
    eb += o[1];
  }
  for (int w = 0; w < warp; ++w) {
    gb += sh.wmass[w];
    eb += sh.wtie[w];
  }
  const uint64_t before = gb + q_tau * min(eb, r);
  const uint64_t after = gb + gm + q_tau * min(eb + ge, r);
  if (before <= y && y < after) {
    uint64_t run = before;
    uint64_t ties = eb;
    for (int base = s0; base < s1; base += 32) {
      const int i = base + lane;
      uint64_t inc = 0;
      bool tie = false;
      if (i < s1) {
        uint32_t k = logit_key(l[i]);
        if (k > tau) inc = q[i];
        tie = (k == tau);
      }
      const unsigned tb = __ballot_sync(0xffffffffu, tie);
      if (tie && ties + __popc(tb & ((1u << lane) - 1u)) < r) inc = q_tau;
      const uint64_t cum = run + warp_incl_scan_u64(inc, lane);
      const unsigned hit = __ballot_sync(0xffffffffu, i < s1 && cum > y);
      if (hit) {
        if (lane == __ffs(hit) - 1) out[row] = lo + i;
        break;
      }
      run = __shfl_sync(0xffffffffu, cum, 31);
      ties += __popc(tb);
    }
  }
  phase_stamp(stamps, 10, stamper);
  cluster.sync();  // 7: no CTA leaves while its shared memory is being read
  phase_stamp(stamps, 11, stamper);
}

}  // namespace

size_t sample_smem_bytes(int slice) {
  return 12 * (size_t)((slice + 1) & ~1) + sizeof(uint64_t) * kHistCopies * 256;
}

cudaError_t launch_top_p(const float *logits, int rows, int vocab, float temperature, float top_p,
                         const double *uniforms, int32_t *out, cudaStream_t stream, unsigned long long *stamps) {
  const int slice = (vocab + kSampleCluster - 1) / kSampleCluster;
  const size_t smem = sample_smem_bytes(slice);
  // the largest dynamic size set so far, per device: the attribute is set only
  // when a launch needs more than that (never on the steady-state path)
  static std::atomic<size_t> configured[kSampleMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kSampleMaxDevices) return cudaErrorInvalidDevice;
  if (smem > configured[dev].load(std::memory_order_acquire)) {
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    if (smem > configured[dev].load(std::memory_order_relaxed)) {
      e = cudaFuncSetAttribute(top_p_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      configured[dev].store(smem, std::memory_order_release);
    }
  }
  const int greedy = !(temperature > 0.0f);
  const double inv_t = greedy ? 0.0 : 1.0 / (double)temperature;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)rows * kSampleCluster);
  cfg.blockDim = dim3(kSThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kSampleCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const int vec4 = (vocab % 4 == 0) && (slice % 4 == 0) && ((reinterpret_cast<uintptr_t>(logits) & 15) == 0);
  return cudaLaunchKernelEx(&cfg, top_p_kernel, logits, vocab, slice, inv_t, top_p, greedy, vec4, uniforms, out,
                            stamps);
}

}  // namespace mk
