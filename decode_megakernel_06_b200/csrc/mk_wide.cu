// mk_wide.cu -- the decode step for wide blocks (8 < M <= 64 rows, e.g. a
// speculative verify block of 7 rows for 8 sequences), as a short sequence of
// launches.  With this many rows the dense projections are real contractions,
// so every matrix product runs on the 5th-generation tensor cores (tcgen05.mma
// from TMA-fed shared memory into a tensor-memory accumulator, bf16 in, fp32
// accumulate).  Activations enter the tensor cores as a bf16 pair
// (x = hi + lo, hi = bf16(x), lo = bf16(x - hi)), so each product keeps close
// to fp32 accuracy; weights are bf16 already.  The remaining steps (norms,
// rotary + cache append, attention merge, top-k, expert lists, SwiGLU,
// combine, argmax) are plain CUDA-core kernels.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <utility>

#include "mk_internal.h"

namespace mk {
namespace {

__device__ __forceinline__ uint32_t sptr(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

// Programmatic dependent launch.  pdl_wait() returns once the previous
// kernel in the stream has completed and its writes are visible; every CTA of
// every kernel here calls it before it reads what an earlier kernel wrote or
// writes what an earlier kernel reads (and before it exits, so that each
// kernel completes after its predecessor).  pdl_launch() lets the next
// kernel's CTAs be scheduled (they then wait in their own pdl_wait()).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Y[r][n] (+)= sum_k W[n][k] * (xhi[r][k] + xlo[r][k]) on the 5th-generation
// tensor cores.  A unit of work is 128 weight rows (the MMA's M) of one
// problem against all of its activation rows (the MMA's N: 16 to 64), over
// one share of K.  The kernel is persistent: CTA b takes units b, b + grid,
// ... and streams them through one pipeline, so the set-up and the first
// loads are paid once per CTA, not once per unit:
//  - warp 0 (one thread) streams each unit's K in stages of 128 columns by
//    TMA: per 64 columns a 128 x 64 weight box and the activation rows in
//    16-row boxes, hi and lo, all 128B-swizzled, completing on the stage's
//    full mbarrier;
//  - warp 1 (one thread) issues tcgen05.mma kind::f16 (bf16 x bf16 -> fp32),
//    K = 16 each, hi then lo into one of two accumulators in tensor memory,
//    releases each stage with tcgen05.commit on its empty mbarrier, and marks
//    the unit's accumulator full;
//  - warps 2-5 read the accumulator (each its 32 lanes = weight rows) with
//    tcgen05.ld, write the unit out and hand the accumulator back, while the
//    next unit's products go into the other one.
// Units: (problem, K share, 128-row tile), tile fastest.  Problem p's weights
// are rows [p * N, (p + 1) * N) of the weight map, its activation rows
// [row_off[p], row_off[p] + row_cnt[p]) (or [0, R) when row_off is NULL); it
// writes the same rows of Y.  A launch may hold two products over the same
// activations (gate and up): problems pe .. 2 pe - 1 take the second weight
// map and write from column ycol2 of Y on.  With ksplit > 1 a unit writes its
// K share into part[ks][row][n] for wide_gemm_finish.
// ---------------------------------------------------------------------------
constexpr int kTcM = 128;                              // weight rows per CTA (MMA M)
constexpr int kTcK = 64;                               // K columns per box: one 128-byte swizzled row
constexpr int kTcBoxes = 2;                            // K boxes per stage (a stage spans 128 columns)
constexpr int kTcStages = 3;                           // measured against 1 box x 6 stages: 4.7 / 4.0 TB/s
constexpr int kTcRowBox = 16;                          // activation rows per TMA box
constexpr int kTcBoxBytes = kTcRowBox * kTcK * 2;      // 2 KB
constexpr int kTcWBox = kTcM * kTcK * 2;               // 16 KB weight box
constexpr int kTcXBox = kWideMaxRows * kTcK * 2;       // 8 KB: up to 64 activation rows of one box
constexpr int kTcA = kTcBoxes * kTcWBox;               // weights per stage
constexpr int kTcB = kTcBoxes * kTcXBox;               // one activation half (hi or lo) per stage
constexpr int kTcStage = kTcA + 2 * kTcB;
constexpr int kTcThreads = 192;                        // producer warp, MMA warp, 4 epilogue warps
constexpr int kTcAccCols = 64;                         // fp32 accumulator columns: one per activation row
constexpr int kTcTmemCols = 2 * kTcAccCols;            // two accumulators
static_assert(kWideMaxRows <= kTcAccCols, "one accumulator column per activation row");

struct GemmArgs {
  CUtensorMap mw, mw2;     // weights: [pe * N rows][K], box 64 x 128 (mw2: the second product, if any)
  CUtensorMap mxh, mxl;    // activations hi / lo: [rows][K], box 64 x 16
  int N, K;
  int pe;                  // problems per weight map; problem p >= pe is p - pe of mw2
  int ycol2;               // column of Y (and part) where the second product's outputs start
  int nb, ksplit, units;   // 128-row tiles per problem, K shares, nb * ksplit * problems
  int halves;              // 2 when mw2 holds a second product, else 1
  // grouped products: the problems that have rows, in increasing order, and
  // how many (written by an earlier kernel); units then run over these only,
  // so that every CTA gets an even share of the real work
  const int *active, *n_active;
  const int *row_off, *row_cnt;
  int R;
  float *Y;
  int ldy;
  int accumulate;  // 1: Y += result (ksplit == 1 only)
  float *part;     // [ksplit][rows][ldy] when ksplit > 1
  int rows_total;  // rows of Y (for part's stride)
  int *error;      // [0] code, [1] op: a bounded wait that ran out
};

__device__ __forceinline__ uint64_t tc_now() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool tc_try_wait(uint64_t *bar, uint32_t par) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(r)
      : "r"(sptr(bar)), "r"(par)
      : "memory");
  return r != 0;
}
// Bounded wait (1 s); on timeout the error word is set and false returned.
__device__ __forceinline__ bool tc_wait(uint64_t *bar, uint32_t par, int *error) {
  const uint64_t t0 = tc_now();
  while (!tc_try_wait(bar, par)) {
    if (tc_now() - t0 > 1000000000ull) {
      if (atomicCAS(&error[0], 0, -5) == 0) atomicExch(&error[1], -2);
      return false;
    }
  }
  return true;
}
__device__ __forceinline__ void tc_tma(void *dst, const CUtensorMap *m, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          sptr(dst)),
      "l"(m), "r"(x), "r"(y), "r"(sptr(bar))
      : "memory");
}
// Shared-memory operand descriptor: K-major rows of 128 bytes, 128-byte
// swizzle, 8-row groups 1024 bytes apart (descriptor version 1).
__device__ __forceinline__ uint64_t tc_desc(const void *p) {
  return static_cast<uint64_t>((sptr(p) >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(0), "r"(0), "r"(0), "r"(0));
}
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(sptr(bar))
               : "memory");
}

// One unit's coordinates; R <= 0 marks a problem without rows (skipped by
// every role alike).
struct TcUnit {
  const CUtensorMap *mw;
  int wrow, r0, R, n0, kc0, nk, G, ycol, ks;
};
__device__ __forceinline__ TcUnit tc_unit(const GemmArgs &a, int u, int nkc, int pe) {
  TcUnit t;
  const int tile = u % a.nb, ks = (u / a.nb) % a.ksplit, pz = u / (a.nb * a.ksplit);
  const int half = pz >= pe, pi = pz - (half ? pe : 0), prob = a.active ? a.active[pi] : pi;
  t.mw = half ? &a.mw2 : &a.mw;
  t.r0 = a.row_off ? a.row_off[prob] : 0;
  t.R = a.row_off ? a.row_cnt[prob] : a.R;
  t.n0 = tile * kTcM;
  t.wrow = prob * a.N + t.n0;
  t.kc0 = (nkc * ks) / a.ksplit;
  t.nk = (nkc * (ks + 1)) / a.ksplit - t.kc0;
  t.G = (t.R + kTcRowBox - 1) / kTcRowBox;
  t.ycol = half ? a.ycol2 : 0;
  t.ks = ks;
  return t;
}

// Bounded wait that also gives up once another role has (abort != 0).
__device__ __forceinline__ bool tc_wait_or_abort(uint64_t *bar, uint32_t par, int *error, volatile int *abort) {
  const uint64_t t0 = tc_now();
  while (!tc_try_wait(bar, par)) {
    if (*abort) return false;
    if (tc_now() - t0 > 1000000000ull) {
      if (atomicCAS(&error[0], 0, -5) == 0) atomicExch(&error[1], -2);
      *abort = 1;
      return false;
    }
  }
  return true;
}

__global__ void __launch_bounds__(kTcThreads, 1) wide_gemm(const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // stages start on 1024-byte boundaries (the 128-byte swizzle repeats every 8 rows)
  uint8_t *smem = smem_raw + ((1024u - (sptr(smem_raw) & 1023u)) & 1023u);
  __shared__ __align__(8) uint64_t full[kTcStages], empty[kTcStages], accf[2], acce[2];
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int nkc = (a.K + kTcBoxes * kTcK - 1) / (kTcBoxes * kTcK);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sptr(&tmem_base)),
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < kTcStages; ++s) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sptr(&full[s])) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sptr(&empty[s])) : "memory");
    }
    for (int b = 0; b < 2; ++b) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sptr(&accf[b])) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(sptr(&acce[b])), "r"(32 * 4) : "memory");
    }
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = tmem_base;
  volatile int *abort = &abort_flag;
  if (warp == 0) {
    if (lane == 0) {  // TMA producer: every unit's stages through one ring
      // A dense product's rows are known without the previous kernel, and no
      // kernel writes weights: the first unit's first stages of weights go
      // out before the wait (a grouped product's rows come from an earlier
      // kernel, so it waits first).
      int pre = 0;
      if (!a.row_off) {
        const TcUnit t = tc_unit(a, blockIdx.x, nkc, a.pe);
        if (t.R > 0) pre = min(t.nk, kTcStages);
        for (int i = 0; i < pre; ++i) {
          uint8_t *st = smem + i * kTcStage;
          asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(sptr(&full[i])),
                       "r"(kTcBoxes * (kTcWBox + 2 * t.G * kTcBoxBytes))
                       : "memory");
          for (int b = 0; b < kTcBoxes; ++b)
            tc_tma(st + b * kTcWBox, t.mw, ((t.kc0 + i) * kTcBoxes + b) * kTcK, t.wrow, &full[i]);
        }
      }
      pdl_wait();
      pdl_launch();
      const int pe = a.active ? *a.n_active : a.pe, units = a.active ? a.nb * a.ksplit * a.halves * pe : a.units;
      int it = 0;
      for (int u = blockIdx.x; u < units && !*abort; u += gridDim.x) {
        const TcUnit t = tc_unit(a, u, nkc, pe);
        if (t.R <= 0) continue;
        for (int i = 0; i < t.nk; ++i, ++it) {
          const int s = it % kTcStages;
          if (it >= kTcStages && !tc_wait_or_abort(&empty[s], ((it / kTcStages) & 1) ^ 1, a.error, abort)) break;
          uint8_t *st = smem + s * kTcStage;
          const bool weights_out = it < pre;  // sent before the wait, with the stage's byte count
          if (!weights_out)
            asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(sptr(&full[s])),
                         "r"(kTcBoxes * (kTcWBox + 2 * t.G * kTcBoxBytes))
                         : "memory");
          for (int b = 0; b < kTcBoxes; ++b) {  // columns past K read as zeros
            const int x = ((t.kc0 + i) * kTcBoxes + b) * kTcK;
            if (!weights_out) tc_tma(st + b * kTcWBox, t.mw, x, t.wrow, &full[s]);
            for (int g = 0; g < t.G; ++g) {
              tc_tma(st + kTcA + b * kTcXBox + g * kTcBoxBytes, &a.mxh, x, t.r0 + kTcRowBox * g, &full[s]);
              tc_tma(st + kTcA + kTcB + b * kTcXBox + g * kTcBoxBytes, &a.mxl, x, t.r0 + kTcRowBox * g, &full[s]);
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    pdl_wait();
    if (lane == 0) {  // MMA issuer
      const int pe = a.active ? *a.n_active : a.pe, units = a.active ? a.nb * a.ksplit * a.halves * pe : a.units;
      int it = 0, lu = 0;
      for (int u = blockIdx.x; u < units && !*abort; u += gridDim.x, ++lu) {
        const TcUnit t = tc_unit(a, u, nkc, pe);
        if (t.R <= 0) {
          --lu;
          continue;
        }
        const int buf = lu & 1;
        if (lu >= 2 && !tc_wait_or_abort(&acce[buf], ((lu >> 1) & 1) ^ 1, a.error, abort)) break;
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        const uint32_t acc = tmem + static_cast<uint32_t>(buf * kTcAccCols);
        // kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B,
        // both K-major, N = 16 G, M = 128
        const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) |
                               (static_cast<uint32_t>((kTcRowBox * t.G) >> 3) << 17) |
                               (static_cast<uint32_t>(kTcM >> 4) << 24);
        bool ok = true;
        for (int i = 0; i < t.nk; ++i, ++it) {
          const int s = it % kTcStages;
          if (!tc_wait_or_abort(&full[s], (it / kTcStages) & 1, a.error, abort)) {
            ok = false;
            break;
          }
          asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
          const uint8_t *st = smem + s * kTcStage;
#pragma unroll
          for (int b = 0; b < kTcBoxes; ++b) {
            const uint64_t da = tc_desc(st + b * kTcWBox), dh = tc_desc(st + kTcA + b * kTcXBox),
                           dl = tc_desc(st + kTcA + kTcB + b * kTcXBox);
#pragma unroll
            for (int kk = 0; kk < kTcK / 16; ++kk) {  // 16 columns = 32 bytes = 2 descriptor units
              tc_mma(acc, da + 2 * kk, dh + 2 * kk, idesc, (i > 0 || b > 0 || kk > 0) ? 1u : 0u);
              tc_mma(acc, da + 2 * kk, dl + 2 * kk, idesc, 1u);
            }
          }
          tc_commit(&empty[s]);  // the stage is free once these products have read it
        }
        if (!ok) break;
        tc_commit(&accf[buf]);  // the unit's accumulator is complete
      }
    }
  } else {  // epilogue: warp w reads accumulator lanes 32 (w mod 4) ..
    pdl_wait();
    const int q = warp & 3;
    const int pe = a.active ? *a.n_active : a.pe, units = a.active ? a.nb * a.ksplit * a.halves * pe : a.units;
    int lu = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      const TcUnit t = tc_unit(a, u, nkc, pe);
      if (t.R <= 0) continue;
      const int buf = lu & 1;
      const bool ok = __all_sync(0xffffffffu, tc_wait_or_abort(&accf[buf], (lu >> 1) & 1, a.error, abort));
      if (!ok) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const int n = t.n0 + 32 * q + lane;
      const int NM = kTcRowBox * t.G;
      for (int c0 = 0; c0 < NM; c0 += 16) {
        uint32_t v[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
            : "r"(tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(buf * kTcAccCols + c0)));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int r = c0 + j;
          if (r >= t.R || n >= a.N) continue;
          const float val = __uint_as_float(v[j]);
          if (a.ksplit > 1) {
            a.part[(static_cast<long long>(t.ks) * a.rows_total + t.r0 + r) * a.ldy + t.ycol + n] = val;
          } else {
            float *y = a.Y + static_cast<long long>(t.r0 + r) * a.ldy + t.ycol + n;
            *y = a.accumulate ? *y + val : val;
          }
        }
      }
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(sptr(&acce[buf])) : "memory");
      ++lu;
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols) : "memory");
  }
}

// Y[r][n] (+)= sum over ks of part[ks][r][n], in order.
__global__ void wide_gemm_finish(const float *part, int ksplit, int rows, int N, int ld, float *Y, int accumulate) {
  pdl_wait();
  pdl_launch();
  const long long total = static_cast<long long>(rows) * N;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(i / N), n = static_cast<int>(i % N);
    float s = 0.f;
    for (int k = 0; k < ksplit; ++k) s += part[(static_cast<long long>(k) * rows + r) * ld + n];
    float *y = Y + static_cast<long long>(r) * ld + n;
    *y = accumulate ? *y + s : s;
  }
}

// ---------------------------------------------------------------------------
// Row-wise steps (one block per row unless stated)
// ---------------------------------------------------------------------------
__device__ __forceinline__ float block_sum(float v, float *red) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
  for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) s += red[i];
  return s;
}

__device__ __forceinline__ void split_store(float x, __nv_bfloat16 *hi, __nv_bfloat16 *lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  *hi = h;
  *lo = __float2bfloat16_rn(x - __bfloat162float(h));
}

// A product whose K shares are still in the split-K buffer: the consumer adds
// part[0][r][col] + part[1][r][col] + ... in that order (as wide_gemm_finish
// would have) instead of reading the finished value.  ks <= 1: nothing
// deferred, the product is in its output already.
struct Split {
  const float *part;
  int ks, rows, ld;
};
__device__ __forceinline__ float split_sum(const Split &p, int r, int col) {
  float s = 0.f;
  const float *q = p.part + static_cast<long long>(r) * p.ld + col;
  const long long step = static_cast<long long>(p.rows) * p.ld;
#pragma unroll 4
  for (int k = 0; k < p.ks; ++k) s += __ldcg(q + k * step);  // the loads go out together, the sum stays in order
  return s;
}

// h[m] = embed[token[m]]; the debug copy of the layer-0 input.
__global__ void wide_embed(const int32_t *tokens, const __nv_bfloat16 *embed, int d, float *h, float *dbg) {
  pdl_wait();
  pdl_launch();
  const int m = blockIdx.x;
  const int tok = tokens[m];
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const float v = __bfloat162float(embed[static_cast<long long>(tok) * d + c]);
    h[static_cast<long long>(m) * d + c] = v;
    if (dbg) dbg[static_cast<long long>(m) * d + c] = v;
  }
}

// x = h / sqrt(mean(h^2) + eps) * g, as a bf16 pair.  With a deferred
// product `add` (the attention output projection), h += that product first.
__global__ void wide_norm_split(float *h, const __nv_bfloat16 *g, int d, float eps, __nv_bfloat16 *xhi,
                                __nv_bfloat16 *xlo, int ldx, Split add) {
  pdl_wait();
  pdl_launch();
  __shared__ float red[32];
  const int m = blockIdx.x;
  float *row = h + static_cast<long long>(m) * d;
  float s = 0.f;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float x = row[c];
    if (add.ks > 1) {
      x = x + split_sum(add, m, c);
      row[c] = x;  // read back below by this same thread
    }
    s = fmaf(x, x, s);
  }
  s = block_sum(s, red);
  const float inv = 1.0f / sqrtf(s / static_cast<float>(d) + eps);
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const float x = row[c] * inv * __bfloat162float(g[c]);
    split_store(x, xhi + static_cast<long long>(m) * ldx + c, xlo + static_cast<long long>(m) * ldx + c);
  }
}

// Rotary embedding of k at each new row's position, k and v rounded to bf16
// and written into the cache.  grid = (M, Hkv).  With the QKV product's K
// shares deferred, block (m, g) first finishes row m's q heads of group g
// and its k and v heads in qkv.
__global__ void wide_kv_append(float *qkv, int W3, const int32_t *positions, int T, int Hq, int Hkv, int hd,
                               const float2 *rope, __nv_bfloat16 *kc, __nv_bfloat16 *vc, int Bmax, int cap,
                               int layer, Split sp) {
  pdl_wait();
  pdl_launch();
  const int m = blockIdx.x, g = blockIdx.y, b = m / T, t = m % T;
  if (sp.ks > 1) {
    const int G = Hq / Hkv;
    float *row = qkv + static_cast<long long>(m) * W3;
    for (int i = threadIdx.x; i < (G + 2) * hd; i += blockDim.x) {
      const int col = i < G * hd ? g * G * hd + i : i < (G + 1) * hd ? (Hq + g) * hd + i - G * hd
                                                                     : (Hq + Hkv + g) * hd + i - (G + 1) * hd;
      row[col] = split_sum(sp, m, col);
    }
    __syncthreads();
  }
  const int p = positions[b] + t, half = hd / 2;
  const float *k = qkv + static_cast<long long>(m) * W3 + (Hq + g) * hd;
  const float *v = qkv + static_cast<long long>(m) * W3 + (Hq + Hkv + g) * hd;
  const long long base = ((static_cast<long long>(layer) * Bmax + b) * Hkv + g) * cap + p;
  for (int i = threadIdx.x; i < hd; i += blockDim.x) {
    const int j = i < half ? i : i - half;
    const float2 cs = rope[static_cast<long long>(p) * half + j];
    const float kr = i < half ? k[i] * cs.x - k[i + half] * cs.y : k[i] * cs.x + k[i - half] * cs.y;
    kc[base * hd + i] = __float2bfloat16_rn(kr);
    vc[base * hd + i] = __float2bfloat16_rn(v[i]);
  }
}

// Attention of a wide block on the tensor cores, split over the KV positions.
// One CTA per (chunk of kAcN cache positions, sequence x KV head, tile of up
// to kAcQ query vectors) scores the group's query vectors (T rows x Hq/Hkv
// heads, each seeing positions up to its own) against the chunk, with the
// chunk's positions as the MMA's M and the query vectors as its N:
//  - one thread brings the chunk's K rows by TMA (128B-swizzled, K-major: the
//    A operand of S^T = K Q^T); every thread loads its share of the V rows,
//    and once S^T is complete writes them transposed over the K rows (V^T,
//    K-major: the A operand of O^T = V^T P^T), so that a CTA needs 49 KB of
//    shared memory and four fit on an SM;
//  - the rotated, scaled query vectors go into shared memory as a bf16 pair
//    (q = hi + lo), one row each (the B operand, N = kAcQ);
//  - S^T (positions x queries, fp32) accumulates K Q_hi^T + K Q_lo^T in tensor
//    memory; thread j reads position j's row, masks the queries that do not
//    see position j, and the CTA reduces the max and then the sum of
//    p = exp(s - max) over the positions of each query (a transposing shuffle
//    reduction in each warp, then across the warps); p is written as a bf16
//    pair, one row per query (the B operand of O^T);
//  - O^T (hd x queries, fp32) accumulates V^T P_hi^T + V^T P_lo^T; thread d
//    writes dim d of every query's unnormalised partial output, thread q the
//    query's max and sum.
// wide_attn_merge combines a query's chunks with the log-sum-exp rule.
// ---------------------------------------------------------------------------
constexpr int kAcN = 128;             // cache positions per chunk (M of S^T, K of O^T)
constexpr int kAcQ = 32;              // query vectors per CTA (N of both products): 32, or 16 for
                                      // groups of at most 16 (one row per sequence, say)
constexpr int kAcThreads = 128;
constexpr int kAcTmemCols = 64;       // S^T: columns [0, 32), O^T: [32, 64)
constexpr int kAcAtom = 128 * 128;    // a swizzled block of 128 rows x 128 bytes

struct AttnArgs {
  CUtensorMap mk;  // K cache as [L * Bmax * Hkv * cap][hd], box 64 x 128
  const float *qkv;
  int W3;
  const int32_t *positions;
  int T, Hq, Hkv;
  const float2 *rope;
  const __nv_bfloat16 *vc;
  int Bmax, cap, layer, nch_max;
  float *opart, *mlpart;  // [slot][hd], [slot][2]; slot = (bg * nch_max + chunk) * T * G + query
  int *error;
};

// dynamic shared memory: K then V^T (2 blocks), Q then P (4 blocks of qn rows
// x 128 bytes), + room to align them to 1024 bytes
constexpr int attn_smem_bytes(int qn) { return 2 * kAcAtom + 4 * qn * 128 + 1024; }

__device__ __forceinline__ uint32_t pack_bf16(float lo_elem, float hi_elem) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo_elem, hi_elem);  // .x at the lower address
  return *reinterpret_cast<const uint32_t *>(&v);
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// byte offset of the 16-byte piece `piece` (0..7) of row r in a swizzled block
__device__ __forceinline__ int sw_off(int r, int piece) { return r * 128 + ((piece ^ (r & 7)) << 4); }

// Reduces each of the NV values over the warp's lanes: afterwards lane l
// holds the reduction of value l mod NV (NV - 1 shuffles, then one per
// remaining lane bit; v is overwritten).  Each step trades half of the
// values with the lane `o` away and combines.
template <bool MAX, int NV>
__device__ __forceinline__ float warp_transpose_reduce(float (&v)[NV], int lane) {
#pragma unroll
  for (int o = NV / 2; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = upper ? v[i] : v[i + o];
      const float keep = upper ? v[i + o] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, o);
      v[i] = MAX ? fmaxf(keep, got) : keep + got;
    }
  }
  float r = v[0];
#pragma unroll
  for (int o = NV; o < 32; o <<= 1) {  // lanes l and l ^ o hold the same value's partials
    const float got = __shfl_xor_sync(0xffffffffu, r, o);
    r = MAX ? fmaxf(r, got) : r + got;
  }
  return r;
}

template <int HD, int QN>
__global__ void __launch_bounds__(kAcThreads) wide_attn_tc(const __grid_constant__ AttnArgs a) {
  pdl_wait();
  pdl_launch();
  constexpr int NA = HD / 64, HALF = HD / 2;
  constexpr int QA = QN * 128;  // a swizzled block of QN rows x 128 bytes
  static_assert(QN == 16 || QN == 32, "N of the products: 16 or 32 query vectors");
  constexpr int NU = 64 * (HD / 8) / kAcThreads;  // (position pair, 8 dims) units of V per thread
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = smem_raw + ((1024u - (sptr(smem_raw) & 1023u)) & 1023u);
  uint8_t *sK = smem;                         // NA blocks: 128 positions x 64 dims; then
  uint8_t *sVT = smem;                        //   V^T, 2 blocks: 128 dim rows (HD used) x 64 positions
  uint8_t *sQ = smem + 2 * kAcAtom;           // Q hi: NA blocks, Q lo: NA blocks; then P hi: 2, P lo: 2
  __shared__ __align__(8) uint64_t kbar, sbar, obar;
  __shared__ uint32_t tmem_base;
  __shared__ __align__(16) float red[4][QN], sM[QN];
  const int c = blockIdx.x, bg = blockIdx.y, b = bg / a.Hkv, g = bg % a.Hkv, G = a.Hq / a.Hkv;
  const int Q = a.T * G, q0 = blockIdx.z * QN, nq = min(QN, Q - q0);
  const int pos0 = a.positions[b], last = pos0 + a.T - 1;
  const int j0 = c * kAcN;
  if (j0 > last || nq <= 0) return;  // the whole CTA, before anything is allocated
  const int nj = min(kAcN, last + 1 - j0);
  const long long krow0 = ((static_cast<long long>(a.layer) * a.Bmax + b) * a.Hkv + g) * a.cap;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sptr(&tmem_base)),
                 "r"(kAcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (threadIdx.x == 32) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sptr(&kbar)) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sptr(&sbar)) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sptr(&obar)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = tmem_base;
  if (threadIdx.x == 0) {  // K rows of the chunk (rows past the cache tensor read as zeros)
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(sptr(&kbar)), "r"(NA * kAcAtom)
                 : "memory");
#pragma unroll
    for (int i = 0; i < NA; ++i) tc_tma(sK + i * kAcAtom, &a.mk, 64 * i, static_cast<int>(krow0 + j0), &kbar);
  }
  // this thread's V units: positions 2 pp and 2 pp + 1, dims [8 dc, 8 dc + 8)
  uint4 va[NU], vb[NU];
  {
    const __nv_bfloat16 *vbase = a.vc + (krow0 + j0) * HD;
#pragma unroll
    for (int i = 0; i < NU; ++i) {
      const int u = threadIdx.x + kAcThreads * i, pp = u & 63, dc = u >> 6;
      va[i] = 2 * pp < nj ? *reinterpret_cast<const uint4 *>(vbase + (2 * pp) * HD + 8 * dc) : make_uint4(0, 0, 0, 0);
      vb[i] = 2 * pp + 1 < nj ? *reinterpret_cast<const uint4 *>(vbase + (2 * pp + 1) * HD + 8 * dc)
                              : make_uint4(0, 0, 0, 0);
    }
  }
  // the query vectors: rotate-half pairs at the query's position, scaled, as a bf16 pair
  {
    const float scale = 1.0f / sqrtf(static_cast<float>(HD));
    for (int it = threadIdx.x; it < nq * (HALF / 8); it += kAcThreads) {
      const int ql = it / (HALF / 8), cc = it % (HALF / 8), qi = q0 + ql;
      const int t = qi / G, h = g * G + qi % G, m = b * a.T + t, lim = pos0 + t;
      const float *q = a.qkv + static_cast<long long>(m) * a.W3 + h * HD + 8 * cc;
      const float4 *cs4 = reinterpret_cast<const float4 *>(a.rope + static_cast<long long>(lim) * HALF + 8 * cc);
      float x1[8], x2[8], cs[16];
      *reinterpret_cast<float4 *>(&x1[0]) = *reinterpret_cast<const float4 *>(q);
      *reinterpret_cast<float4 *>(&x1[4]) = *reinterpret_cast<const float4 *>(q + 4);
      *reinterpret_cast<float4 *>(&x2[0]) = *reinterpret_cast<const float4 *>(q + HALF);
      *reinterpret_cast<float4 *>(&x2[4]) = *reinterpret_cast<const float4 *>(q + HALF + 4);
#pragma unroll
      for (int i = 0; i < 4; ++i) *reinterpret_cast<float4 *>(&cs[4 * i]) = cs4[i];
      uint32_t y1h[4], y1l[4], y2h[4], y2l[4];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        float y1[2], y2[2], r1[2], r2[2];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const float co = cs[2 * (e + k)], si = cs[2 * (e + k) + 1];
          y1[k] = (x1[e + k] * co - x2[e + k] * si) * scale;
          y2[k] = (x2[e + k] * co + x1[e + k] * si) * scale;
          r1[k] = y1[k] - __bfloat162float(__float2bfloat16_rn(y1[k]));
          r2[k] = y2[k] - __bfloat162float(__float2bfloat16_rn(y2[k]));
        }
        y1h[e / 2] = pack_bf16(y1[0], y1[1]);
        y1l[e / 2] = pack_bf16(r1[0], r1[1]);
        y2h[e / 2] = pack_bf16(y2[0], y2[1]);
        y2l[e / 2] = pack_bf16(r2[0], r2[1]);
      }
      const int d1 = 8 * cc, d2 = HALF + 8 * cc;
      const int o1 = (d1 >> 6) * QA + sw_off(ql, (d1 & 63) >> 3),
                o2 = (d2 >> 6) * QA + sw_off(ql, (d2 & 63) >> 3);
      *reinterpret_cast<uint4 *>(sQ + o1) = make_uint4(y1h[0], y1h[1], y1h[2], y1h[3]);
      *reinterpret_cast<uint4 *>(sQ + NA * QA + o1) = make_uint4(y1l[0], y1l[1], y1l[2], y1l[3]);
      *reinterpret_cast<uint4 *>(sQ + o2) = make_uint4(y2h[0], y2h[1], y2h[2], y2h[3]);
      *reinterpret_cast<uint4 *>(sQ + NA * QA + o2) = make_uint4(y2l[0], y2l[1], y2l[2], y2l[3]);
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  // kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B, both
  // K-major, N = QN, M = 128 (both products)
  constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((QN >> 3) << 17) | ((128 >> 4) << 24);
  if (threadIdx.x == 0) {
    if (tc_wait(&kbar, 0, a.error)) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
      for (int i = 0; i < NA; ++i) {
        const uint64_t dk = tc_desc(sK + i * kAcAtom), dqh = tc_desc(sQ + i * QA),
                       dql = tc_desc(sQ + (NA + i) * QA);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 16 dims = 32 bytes = 2 descriptor units
          tc_mma(tmem, dk + 2 * kk, dqh + 2 * kk, kIdesc, (i > 0 || kk > 0) ? 1u : 0u);
          tc_mma(tmem, dk + 2 * kk, dql + 2 * kk, kIdesc, 1u);
        }
      }
    }
    tc_commit(&sbar);
  }
  __syncwarp();
  bool ok = tc_wait(&sbar, 0, a.error);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  // V^T over the K rows (read by S^T, now complete): row d, positions 2 pp
  // and 2 pp + 1 in one 32-bit word
#pragma unroll
  for (int i = 0; i < NU; ++i) {
    const int u = threadIdx.x + kAcThreads * i, pp = u & 63, dc = u >> 6;
    const uint32_t wa[4] = {va[i].x, va[i].y, va[i].z, va[i].w}, wb[4] = {vb[i].x, vb[i].y, vb[i].z, vb[i].w};
    uint8_t *blk = sVT + (pp >> 5) * kAcAtom + (pp & 3) * 4;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int d = 8 * dc + e;
      const uint32_t word = __byte_perm(wa[e >> 1], wb[e >> 1], (e & 1) ? 0x7632 : 0x5410);
      *reinterpret_cast<uint32_t *>(blk + sw_off(d, (pp & 31) >> 2)) = word;
    }
  }
  // position j = this thread's accumulator lane: its scores for the QN query vectors
  const int j = threadIdx.x;
  const uint32_t tlane = tmem + (static_cast<uint32_t>(32 * warp) << 16);
  float sc[QN];
  {
    uint32_t v0[16], v1[16];
    tmem_ld16(tlane, v0);
    if constexpr (QN == 32) tmem_ld16(tlane + 16, v1);
    // query ql sees position j0 + j iff it exists and j0 + j <= pos0 + (q0 + ql) / G
    const int dj = j0 + j - pos0;
#pragma unroll
    for (int ql = 0; ql < QN; ++ql) {
      const bool see = ql < nq && j < nj && (dj <= 0 || q0 + ql >= G * dj);
      sc[ql] = see ? __uint_as_float(ql < 16 ? v0[ql] : v1[ql - 16]) : -INFINITY;
    }
  }
  {
    float t[QN];
#pragma unroll
    for (int ql = 0; ql < QN; ++ql) t[ql] = sc[ql];
    const float r = warp_transpose_reduce<true, QN>(t, lane);
    if (lane < QN) red[warp][lane] = r;
  }
  __syncthreads();
  if (threadIdx.x < QN)
    sM[threadIdx.x] = fmaxf(fmaxf(red[0][threadIdx.x], red[1][threadIdx.x]), fmaxf(red[2][threadIdx.x], red[3][threadIdx.x]));
  __syncthreads();
  float pv[QN];
#pragma unroll
  for (int q4 = 0; q4 < QN / 4; ++q4) {
    const float4 m4 = *reinterpret_cast<const float4 *>(&sM[4 * q4]);
    const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int ql = 4 * q4 + k;
      pv[ql] = sc[ql] == -INFINITY ? 0.f : expf(sc[ql] - mm[k]);
    }
  }
  // p^T as a bf16 pair: row ql, K index j (the Q rows are no longer read)
  {
    uint8_t *base = sQ + (j >> 6) * QA + (j & 7) * 2;
#pragma unroll
    for (int ql = 0; ql < QN; ++ql) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(pv[ql]);
      const __nv_bfloat16 lo = __float2bfloat16_rn(pv[ql] - __bfloat162float(hi));
      const int off = sw_off(ql, (j & 63) >> 3);
      *reinterpret_cast<__nv_bfloat16 *>(base + off) = hi;
      *reinterpret_cast<__nv_bfloat16 *>(base + 2 * QA + off) = lo;
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();  // also: every warp has read red (the maxima) before it is reused below
  if (threadIdx.x == 0) {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (ok) {
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint64_t dv = tc_desc(sVT + i * kAcAtom), dph = tc_desc(sQ + i * QA),
                       dpl = tc_desc(sQ + (2 + i) * QA);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {  // 16 positions per product
          tc_mma(tmem + QN, dv + 2 * kk, dph + 2 * kk, kIdesc, (i > 0 || kk > 0) ? 1u : 0u);
          tc_mma(tmem + QN, dv + 2 * kk, dpl + 2 * kk, kIdesc, 1u);
        }
      }
    }
    tc_commit(&obar);
  }
  // meanwhile: the sum of p over the positions of each query
  {
    const float r = warp_transpose_reduce<false, QN>(pv, lane);
    if (lane < QN) red[warp][lane] = r;
  }
  __syncthreads();
  __syncwarp();
  ok = tc_wait(&obar, 0, a.error) && ok;
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const long long slot0 = (static_cast<long long>(bg) * a.nch_max + c) * Q + q0;
  {
    // dim d = this thread's accumulator lane of O^T
    uint32_t v0[16], v1[16];
    tmem_ld16(tlane + QN, v0);
    if constexpr (QN == 32) tmem_ld16(tlane + QN + 16, v1);
    const int d = threadIdx.x;
    if (d < HD) {
#pragma unroll
      for (int ql = 0; ql < QN; ++ql)
        if (ql < nq) a.opart[(slot0 + ql) * HD + d] = ok ? __uint_as_float(ql < 16 ? v0[ql] : v1[ql - 16]) : 0.f;
    }
  }
  if (threadIdx.x < nq) {
    const int ql = threadIdx.x;
    a.mlpart[2 * (slot0 + ql)] = sM[ql];
    a.mlpart[2 * (slot0 + ql) + 1] = ((red[0][ql] + red[1][ql]) + red[2][ql]) + red[3][ql];
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kAcTmemCols) : "memory");
  }
}

// Query (m, h)'s chunk partials combined with the log-sum-exp rule, written
// straight into the bf16 pair that feeds the output projection (row m,
// columns [h hd, h hd + hd)).  One block of groups x hd threads per (row,
// head), groups = blockDim / hd (up to kMgGroups, more for longer caches).  Warp 0 folds the chunks' (max, sum) pairs into the overall
// max and the weighted sum in one pass: each lane keeps a running pair over
// its chunks, then the lanes' pairs are folded by shuffles.  Then thread group
// r adds chunks r, r + groups, ... for dim i, and group 0 adds the groups'
// sums in order and writes the result.
constexpr int kMgGroups = 4;
__global__ void wide_attn_merge(const int32_t *positions, int T, int Hq, int Hkv, int hd, int nch_max,
                                const float *opart, const float *mlpart, __nv_bfloat16 *xhi, __nv_bfloat16 *xlo,
                                int ldx) {
  pdl_wait();
  pdl_launch();
  __shared__ float s_md[2];
  __shared__ float s_num[kMgGroups - 1][128];
  const int m = blockIdx.x, h = blockIdx.y, b = m / T, t = m % T, G = Hq / Hkv, g = h / G;
  const int Q = T * G, qi = t * G + h % G, bg = b * Hkv + g;
  const int nch = (positions[b] + t) / kAcN + 1;  // chunks holding positions this query sees
  const long long slot0 = static_cast<long long>(bg) * nch_max * Q + qi;  // chunk c: slot0 + c Q
  if (threadIdx.x < 32) {
    float M = -INFINITY, den = 0.f;
    for (int c = threadIdx.x; c < nch; c += 32) {
      const float *ml = mlpart + 2 * (slot0 + static_cast<long long>(c) * Q);
      const float mc = ml[0];
      if (mc == -INFINITY) continue;  // a chunk this query sees nothing of
      const float nm = fmaxf(M, mc);
      den = den * expf(M - nm) + ml[1] * expf(mc - nm);
      M = nm;
    }
    for (int o = 16; o; o >>= 1) {
      const float oM = __shfl_xor_sync(0xffffffffu, M, o), od = __shfl_xor_sync(0xffffffffu, den, o);
      const float nm = fmaxf(M, oM);
      den = nm == -INFINITY ? 0.f : den * expf(M - nm) + od * expf(oM - nm);
      M = nm;
    }
    if (threadIdx.x == 0) {
      s_md[0] = M;
      s_md[1] = den;
    }
  }
  __syncthreads();
  const float M = s_md[0], den = s_md[1];
  const int groups = blockDim.x / hd, grp = threadIdx.x / hd, i = threadIdx.x % hd;
  float num = 0.f;
#pragma unroll 4
  for (int c = grp; c < nch; c += groups) {
    const long long slot = slot0 + static_cast<long long>(c) * Q;
    num = fmaf(expf(mlpart[2 * slot] - M), opart[slot * hd + i], num);
  }
  if (grp > 0) s_num[grp - 1][i] = num;
  __syncthreads();
  if (grp == 0) {
    for (int r = 0; r < groups - 1; ++r) num += s_num[r][i];
    const long long at = static_cast<long long>(m) * ldx + h * hd + i;
    split_store(num / den, xhi + at, xlo + at);
  }
}

// Per row: softmax over the E router logits, top-k (ties to the lower id),
// weights renormalised by their sum.  One warp per row.
__global__ void wide_topk(const float *logits, int E, int K, int32_t *sel_e, float *sel_w, int32_t *dbg_ids,
                          float *dbg_w, Split sp) {
  pdl_wait();
  pdl_launch();
  const int m = blockIdx.x, lane = threadIdx.x;
  float z[kMaxExperts / 32];  // lane's logits: expert lane + 32 i (from the split-K buffer when deferred)
#pragma unroll
  for (int i = 0; i < kMaxExperts / 32; ++i) {
    const int e = lane + 32 * i;
    z[i] = e < E ? (sp.ks > 1 ? split_sum(sp, m, e) : logits[static_cast<long long>(m) * E + e]) : 0.f;
  }
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < kMaxExperts / 32; ++i)
    if (lane + 32 * i < E) mx = fmaxf(mx, z[i]);
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
#pragma unroll
  for (int i = 0; i < kMaxExperts / 32; ++i)
    if (lane + 32 * i < E) sum += expf(z[i] - mx);
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  uint32_t taken[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // bit e of expert e (E <= 256)
  float sel = 0.f, my_w = 0.f;
  int my_e = 0;
  for (int j = 0; j < K; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < kMaxExperts / 32; ++i) {
      const int e = lane + 32 * i;
      if (e >= E || ((taken[e >> 5] >> (e & 31)) & 1u)) continue;
      const float pe = expf(z[i] - mx) / sum;
      if (pe > bv || (pe == bv && e < bi)) {
        bv = pe;
        bi = e;
      }
    }
    for (int o = 16; o; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    taken[bi >> 5] |= 1u << (bi & 31);
    if (lane == j) {
      my_e = bi;
      my_w = bv;
    }
    sel += bv;
  }
  if (lane < K) {
    sel_e[m * K + lane] = my_e;
    sel_w[m * K + lane] = my_w / sel;
    if (dbg_ids) dbg_ids[m * K + lane] = my_e;
    if (dbg_w) dbg_w[m * K + lane] = my_w / sel;
  }
}

// The routed (row, choice) pairs in expert-major order, and each pair's row
// gathered there, in one launch.  Block i owns pair i = (m, j) (in (m, j)
// order): its place is the number of pairs of a lower expert plus the earlier
// pairs of its own expert (so the pairs of one expert keep (m, j) order), and
// it copies row m of the bf16 pair to that place.  Block 0 also writes each
// expert's count and first place, the list of experts with rows, and adds
// the number of experts in use to the statistics.
__global__ void wide_route_gather(const int32_t *sel_e, int M, int K, int E, const __nv_bfloat16 *xhi,
                                  const __nv_bfloat16 *xlo, int ldx, int d, int *count, int *off, int *pair_row,
                                  int *pair_slot, unsigned long long *stats, __nv_bfloat16 *ghi, __nv_bfloat16 *glo,
                                  int *active, int *n_active) {
  pdl_wait();
  pdl_launch();
  __shared__ float red[32];
  __shared__ int s_q;
  const int i = blockIdx.x, MK = M * K, e = sel_e[i];
  float before = 0.f;  // exact: at most a few thousand
  for (int j = threadIdx.x; j < MK; j += blockDim.x) {
    const int ej = sel_e[j];
    before += (ej < e || (ej == e && j < i)) ? 1.f : 0.f;
  }
  before = block_sum(before, red);
  if (threadIdx.x == 0) {
    const int q = static_cast<int>(before);
    s_q = q;
    pair_slot[i] = q;
    pair_row[q] = i / K;
  }
  if (i == 0) {
    __shared__ int s_cnt[kMaxExperts];
    unsigned long long used = 0;
    for (int x = threadIdx.x; x < E; x += blockDim.x) {
      int c = 0, o = 0;
      for (int j = 0; j < MK; ++j) {
        const int ej = sel_e[j];
        c += ej == x;
        o += ej < x;
      }
      count[x] = c;
      off[x] = o;
      s_cnt[x] = c;
      used += c > 0;
    }
    if (used) atomicAdd(stats, used);
    __syncthreads();
    if (threadIdx.x == 0) {  // the experts with rows, in increasing order
      int na = 0;
      for (int x = 0; x < E; ++x)
        if (s_cnt[x] > 0) active[na++] = x;
      *n_active = na;
    }
  }
  __syncthreads();
  const long long src = static_cast<long long>(i / K) * ldx, dst = static_cast<long long>(s_q) * ldx;
  if ((d & 7) == 0) {  // 16-byte pieces (ldx is a multiple of 8)
    for (int c = threadIdx.x; c < d / 8; c += blockDim.x) {
      reinterpret_cast<uint4 *>(ghi + dst)[c] = reinterpret_cast<const uint4 *>(xhi + src)[c];
      reinterpret_cast<uint4 *>(glo + dst)[c] = reinterpret_cast<const uint4 *>(xlo + src)[c];
    }
  } else {
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
      ghi[dst + c] = xhi[src + c];
      glo[dst + c] = xlo[src + c];
    }
  }
}

// act = silu(gate) * up for rows [rows][2F] (gate then up), as a bf16 pair;
// gate and up come from the split-K buffer when deferred.  grid = (rows,
// ceil(F / blockDim)).
__global__ void wide_swiglu(const float *gu, int F, __nv_bfloat16 *ahi, __nv_bfloat16 *alo, int lda, Split sp) {
  pdl_wait();
  pdl_launch();
  const int q = blockIdx.x;
  for (int c = blockIdx.y * blockDim.x + threadIdx.x; c < F; c += gridDim.y * blockDim.x) {
    const float gt = sp.ks > 1 ? split_sum(sp, q, c) : gu[static_cast<long long>(q) * 2 * F + c];
    const float up = sp.ks > 1 ? split_sum(sp, q, F + c) : gu[static_cast<long long>(q) * 2 * F + F + c];
    split_store(gt / (1.0f + expf(-gt)) * up, ahi + static_cast<long long>(q) * lda + c,
                alo + static_cast<long long>(q) * lda + c);
  }
}

// h[m] += sum_j w[m][j] y[pair(m, j)] (selection order) + shared[m]
// grid = (rows, ceil(d / blockDim)): one column per thread.  The shared
// expert's output comes from the split-K buffer when deferred.
__global__ void wide_combine(float *h, int d, int K, const float *sel_w, const int *pair_slot, const float *y,
                             const float *ys, float *dbg, Split sp) {
  pdl_wait();
  pdl_launch();
  const int m = blockIdx.x;
  for (int c = blockIdx.y * blockDim.x + threadIdx.x; c < d; c += gridDim.y * blockDim.x) {
    float moe = 0.f;
    for (int j = 0; j < K; ++j)
      moe = fmaf(sel_w[m * K + j], y[static_cast<long long>(pair_slot[m * K + j]) * d + c], moe);
    const float sh = ys ? (sp.ks > 1 ? split_sum(sp, m, c) : ys[static_cast<long long>(m) * d + c]) : 0.f;
    const float v = h[static_cast<long long>(m) * d + c] + (ys ? moe + sh : moe);
    h[static_cast<long long>(m) * d + c] = v;
    if (dbg) dbg[static_cast<long long>(m) * d + c] = v;
  }
}

// argmax over the vocabulary per row (ties to the lowest index)
// One block per row; with V a multiple of 4 each thread reads 16-byte pieces.
__global__ void __launch_bounds__(1024) wide_argmax(const float *logits, int V, int32_t *out) {
  pdl_wait();
  pdl_launch();
  __shared__ float bvs[32];
  __shared__ int bis[32];
  const int m = blockIdx.x;
  const float *row = logits + static_cast<long long>(m) * V;
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  auto take = [&](float x, int v) {
    if (x > bv || (x == bv && v < bi)) {
      bv = x;
      bi = v;
    }
  };
  if ((V & 3) == 0) {
    const float4 *r4 = reinterpret_cast<const float4 *>(row);
#pragma unroll 4
    for (int v4 = threadIdx.x; v4 < V / 4; v4 += blockDim.x) {
      const float4 x = r4[v4];
      take(x.x, 4 * v4);
      take(x.y, 4 * v4 + 1);
      take(x.z, 4 * v4 + 2);
      take(x.w, 4 * v4 + 3);
    }
  } else {
    for (int v = threadIdx.x; v < V; v += blockDim.x) take(row[v], v);
  }
  for (int o = 16; o; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    if (ov > bv || (ov == bv && oi < bi)) {
      bv = ov;
      bi = oi;
    }
  }
  if ((threadIdx.x & 31) == 0) {
    bvs[threadIdx.x >> 5] = bv;
    bis[threadIdx.x >> 5] = bi;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float best = bvs[0];
    int besti = bis[0];
    for (int i = 1; i < static_cast<int>(blockDim.x >> 5); ++i)
      if (bvs[i] > best || (bvs[i] == best && bis[i] < besti)) {
        best = bvs[i];
        besti = bis[i];
      }
    out[m] = besti == 0x7fffffff ? 0 : besti;
  }
}

// Checks of token ids and positions.  A bad value sets the device error
// (MK_ERR_DEVICE_CHECK); the launches that follow read clamped copies, so no
// access leaves its buffer, and the status marks the step's results invalid.
__global__ void wide_check(const int32_t *tokens, const int32_t *positions, int B, int T, int V, int cap,
                           int32_t *tokens_safe, int32_t *positions_safe, int *error) {
  pdl_wait();
  pdl_launch();
  bool bad = false;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int p = positions[b];
    if (p < 0 || p + T > cap) bad = true;
    positions_safe[b] = min(max(p, 0), cap - T);
  }
  for (int m = threadIdx.x; m < B * T; m += blockDim.x) {
    const int t = tokens[m];
    if (t < 0 || t >= V) bad = true;
    tokens_safe[m] = min(max(t, 0), V - 1);
  }
  if (bad && atomicCAS(&error[0], 0, -6) == 0) atomicExch(&error[1], 0);
}

// Acceptance after verify block s of the wide path (one thread per
// sequence): the longest run of drafts that each equal the argmax of the row
// before them, plus one token.  The accepted tokens (-1 after them) and their
// count go out, and the next block replaces this one in place: the last
// accepted token at the advanced position, then the drafts proposed for the
// positions after it (drafts[b][j] is for cache position pos0[b] + j).
__global__ void wide_accept(int B, int T, int s, const int32_t *argmax, int32_t *tok, int32_t *pos,
                            const int32_t *pos0, const int32_t *drafts, int draft_len, int32_t *out_tokens,
                            int32_t *out_accepted) {
  pdl_wait();
  pdl_launch();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  const int32_t *am = argmax + static_cast<long long>(b) * T;
  int32_t *tb = tok + static_cast<long long>(b) * T;
  int a = 1;
  while (a < T && tb[a] == am[a - 1]) ++a;
  for (int i = 0; i < T; ++i) out_tokens[(static_cast<long long>(s) * B + b) * T + i] = i < a ? am[i] : -1;
  out_accepted[static_cast<long long>(s) * B + b] = a;
  const int p = pos[b] + a;
  pos[b] = p;
  tb[0] = am[a - 1];
  for (int t = 1; t < T; ++t) {
    const int j = p + t - pos0[b];  // below draft_len for every block that runs
    tb[t] = j >= 0 && j < draft_len ? drafts[static_cast<long long>(b) * draft_len + j] : 0;
  }
}

int gemm_smem_bytes() { return kTcStages * kTcStage + 1024; }  // + room to align the stages to 1024 bytes

}  // namespace

// ---------------------------------------------------------------------------
// Host driver
// ---------------------------------------------------------------------------
// Every launch of the step may start while its predecessor in the stream
// finishes (programmatic dependent launch, kept as such by graph capture);
// each kernel waits for the predecessor with pdl_wait() before it touches
// memory that kernels before it use.
template <typename... KArgs, typename... Args>
static cudaError_t launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                          Args &&...args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

#define WIDE_TRY(x)                   \
  do {                                \
    cudaError_t e__ = (x);            \
    if (e__ != cudaSuccess) return e__; \
  } while (0)

// One product (or one grouped launch of per-expert products) on the tensor
// cores: weight rows [p * N, (p + 1) * N) x K for problem p, activation rows
// of the xrows-row buffers xhi / xlo (row stride ldx).  A single dense problem
// whose 128-row tiles do not fill the GPU splits K, through `part`; with
// `defer` the shares stay there for the consumer to add (no finish launch),
// which must run before the next product that splits K.
static cudaError_t gemm(int &n, const WideStep &s, const __nv_bfloat16 *W, const __nv_bfloat16 *W2, int pe, int N,
                        int K, const __nv_bfloat16 *xhi, const __nv_bfloat16 *xlo, int ldx, int xrows,
                        const int *row_off, const int *row_cnt, int R, float *Y, int ldy, int ycol2, int accumulate,
                        float *part, cudaStream_t st, Split *defer = nullptr, const int *active = nullptr,
                        const int *n_active = nullptr) {
  GemmArgs a{};
  const int problems = W2 ? 2 * pe : pe;
  if (encode_2d_sw128(&a.mw, W, static_cast<uint64_t>(pe) * N, K, K, kTcM) != MK_OK ||
      encode_2d_sw128(&a.mw2, W2 ? W2 : W, static_cast<uint64_t>(pe) * N, K, K, kTcM) != MK_OK ||
      encode_2d_sw128(&a.mxh, xhi, xrows, K, ldx, kTcRowBox) != MK_OK ||
      encode_2d_sw128(&a.mxl, xlo, xrows, K, ldx, kTcRowBox) != MK_OK)
    return cudaErrorInvalidValue;
  a.N = N;
  a.K = K;
  a.pe = pe;
  a.ycol2 = ycol2;
  a.row_off = row_off;
  a.row_cnt = row_cnt;
  a.R = R;
  a.Y = Y;
  a.ldy = ldy;
  a.accumulate = accumulate;
  a.rows_total = R;
  a.error = s.error;
  const int nb = (N + kTcM - 1) / kTcM;
  int ksplit = 1;
  if (!row_off) {  // one dense problem: about one CTA per SM, at least two K stages each
    // a consumer that adds the shares itself reads each of them per output:
    // at most 4 then (2.05 / 5.09 / 7.51 ms against 2.08 / 5.13 / 7.56 with up
    // to 16, for the small model's 56 rows and the large model's 4 and 8)
    const int nkc = (K + kTcBoxes * kTcK - 1) / (kTcBoxes * kTcK);
    ksplit = std::max(1, std::min(std::min(s.n_sm / (nb * problems), nkc / 2), defer ? 4 : 16));
    if (static_cast<long long>(ksplit) * R * ldy > s.part_floats) ksplit = 1;
  }
  a.part = ksplit > 1 ? part : nullptr;
  a.nb = nb;
  a.ksplit = ksplit;
  a.units = nb * ksplit * problems;
  a.halves = W2 ? 2 : 1;
  a.active = active;
  a.n_active = active ? n_active : nullptr;
  WIDE_TRY(launch(wide_gemm, dim3(std::min(a.units, s.n_sm)), dim3(kTcThreads), gemm_smem_bytes(), st, a));
  ++n;
  if (defer) *defer = Split{part, ksplit > 1 ? ksplit : 0, R, ldy};
  if (ksplit > 1 && !defer) {
    WIDE_TRY(launch(wide_gemm_finish, dim3(2 * s.n_sm), dim3(256), 0, st, part, ksplit, R, W2 ? ycol2 + N : N, ldy, Y, accumulate));
    ++n;
  }
  return cudaSuccess;
}

cudaError_t wide_accept_step(int B, int T, int s, const int32_t *argmax, int32_t *tok, int32_t *pos,
                             const int32_t *pos0, const int32_t *drafts, int draft_len, int32_t *out_tokens,
                             int32_t *out_accepted, cudaStream_t st) {
  return launch(wide_accept, dim3((B + 127) / 128), dim3(128), 0, st, B, T, s, argmax, tok, pos, pos0, drafts, draft_len,
                out_tokens, out_accepted);
}

cudaError_t wide_prepare() {
  WIDE_TRY(cudaFuncSetAttribute(wide_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem_bytes()));
  WIDE_TRY(cudaFuncSetAttribute(wide_attn_tc<64, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize, attn_smem_bytes(16)));
  WIDE_TRY(cudaFuncSetAttribute(wide_attn_tc<64, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize, attn_smem_bytes(32)));
  WIDE_TRY(cudaFuncSetAttribute(wide_attn_tc<128, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize, attn_smem_bytes(16)));
  return cudaFuncSetAttribute(wide_attn_tc<128, 32>, cudaFuncAttributeMaxDynamicSharedMemorySize, attn_smem_bytes(32));
}

cudaError_t wide_step(const WideStep &s, cudaStream_t st, int *launches) {
  int n = 0;
  const int M = s.B * s.T, d = s.d, L = s.L, K = s.topk, E = s.E, F = s.F, Fs = s.Fs;
  const int W3 = (s.Hq + 2 * s.Hkv) * s.hd, HD = s.Hq * s.hd;
  const int ldx = s.ldx;  // >= max(d, HD), multiple of 8
  WIDE_TRY(launch(wide_check, dim3(1), dim3(256), 0, st, s.tokens, s.positions, s.B, s.T, s.V, s.cap, s.tokens_safe, s.positions_safe,
                                s.error));
  ++n;
  WIDE_TRY(launch(wide_embed, dim3(M), dim3(256), 0, st, s.tokens_safe, s.embed, d, s.h, s.dbg_hidden));
  ++n;
  for (int l = 0; l < L; ++l) {
    const mk_layer_weights &lw = s.layers[l];
    // Products that split K leave their shares in s.part for the next kernel
    // to add (Split), so each is consumed before the next such product.
    // attention block
    WIDE_TRY(launch(wide_norm_split, dim3(M), dim3(1024), 0, st, s.h, static_cast<const __nv_bfloat16 *>(lw.attn_norm), d, s.eps, s.xhi,
                                       s.xlo, ldx, Split{}));
    ++n;
    Split sq{};
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.wqkv), nullptr, 1, W3, d, s.xhi, s.xlo, ldx, M, nullptr,
                  nullptr, M, s.qkv, W3, 0, 0, s.part, st, &sq));
    WIDE_TRY(launch(wide_kv_append, dim3(M, s.Hkv), dim3(256), 0, st, s.qkv, W3, s.positions_safe, s.T, s.Hq, s.Hkv, s.hd, s.rope, s.kc,
                                                   s.vc, s.Bmax, s.cap, l, sq));
    ++n;
    {  // attention: chunk partials on the tensor cores, then the merge into the bf16 pair
      const int G = s.Hq / s.Hkv, nch = (s.cap + kAcN - 1) / kAcN;
      AttnArgs aa{};
      // the kernel's TMA row coordinate is 32-bit
      if (static_cast<uint64_t>(s.L) * s.Bmax * s.Hkv * s.cap > 0x7fffffffull ||
          encode_2d_sw128(&aa.mk, s.kc, static_cast<uint64_t>(s.L) * s.Bmax * s.Hkv * s.cap, s.hd, s.hd, kAcN) != MK_OK)
        return cudaErrorInvalidValue;
      aa.qkv = s.qkv;
      aa.W3 = W3;
      aa.positions = s.positions_safe;
      aa.T = s.T;
      aa.Hq = s.Hq;
      aa.Hkv = s.Hkv;
      aa.rope = s.rope;
      aa.vc = s.vc;
      aa.Bmax = s.Bmax;
      aa.cap = s.cap;
      aa.layer = l;
      aa.nch_max = nch;
      aa.opart = s.attn_o;
      aa.mlpart = s.attn_ml;
      aa.error = s.error;
      const int qn = s.T * G <= 16 ? 16 : kAcQ;  // N of the products: the group's query vectors
      const dim3 grid(nch, s.B * s.Hkv, (s.T * G + qn - 1) / qn);
      if (s.hd == 64 && qn == 16)
        WIDE_TRY(launch(wide_attn_tc<64, 16>, dim3(grid), dim3(kAcThreads), attn_smem_bytes(16), st, aa));
      else if (s.hd == 64)
        WIDE_TRY(launch(wide_attn_tc<64, 32>, dim3(grid), dim3(kAcThreads), attn_smem_bytes(32), st, aa));
      else if (qn == 16)
        WIDE_TRY(launch(wide_attn_tc<128, 16>, dim3(grid), dim3(kAcThreads), attn_smem_bytes(16), st, aa));
      else
        WIDE_TRY(launch(wide_attn_tc<128, 32>, dim3(grid), dim3(kAcThreads), attn_smem_bytes(32), st, aa));
      ++n;
      // chunk groups per block: enough threads for long caches, few blocks' worth for short ones
      const int mg = nch >= 32 ? kMgGroups : nch >= 16 ? 2 : 1;
      WIDE_TRY(launch(wide_attn_merge, dim3(M, s.Hq), dim3(mg * s.hd), 0, st, s.positions_safe, s.T, s.Hq, s.Hkv, s.hd, nch, s.attn_o,
                                                      s.attn_ml, s.xhi, s.xlo, ldx));
      ++n;
    }
    Split so{};
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.wo), nullptr, 1, d, HD, s.xhi, s.xlo, ldx, M, nullptr,
                  nullptr, M, s.h, d, 0, 1, s.part, st, &so));
    // MoE block: h += the output projection, norm; router, top-k
    WIDE_TRY(launch(wide_norm_split, dim3(M), dim3(1024), 0, st, s.h, static_cast<const __nv_bfloat16 *>(lw.ffn_norm), d, s.eps, s.xhi, s.xlo,
                                       ldx, so));
    ++n;
    Split sr{};
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.router), nullptr, 1, E, d, s.xhi, s.xlo, ldx, M, nullptr,
                  nullptr, M, s.rlog, E, 0, 0, s.part, st, &sr));
    int32_t *dbg_ids = s.dbg_ids ? s.dbg_ids + static_cast<long long>(l) * s.max_rows * K : nullptr;
    float *dbg_w = s.dbg_w ? s.dbg_w + static_cast<long long>(l) * s.max_rows * K : nullptr;
    WIDE_TRY(launch(wide_topk, dim3(M), dim3(32), 0, st, s.rlog, E, K, s.sel_e, s.sel_w, dbg_ids, dbg_w, sr));
    ++n;
    // shared expert on every row (gate and up in one launch); its down
    // product's shares are added by the combine (the routed products below
    // do not split K, so they leave s.part alone)
    Split sd{};
    if (Fs > 0) {
      Split sg{};
      WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.ws_gate), static_cast<const __nv_bfloat16 *>(lw.ws_up),
                    1, Fs, d, s.xhi, s.xlo, ldx, M, nullptr, nullptr, M, s.gs, 2 * Fs, Fs, 0, s.part, st, &sg));
      WIDE_TRY(launch(wide_swiglu, dim3(M, (Fs + 255) / 256), dim3(256), 0, st, s.gs, Fs, s.shi, s.slo, s.lda, sg));
      ++n;
      WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.ws_down), nullptr, 1, d, Fs, s.shi, s.slo, s.lda, M,
                    nullptr, nullptr, M, s.ys, d, 0, 0, s.part, st, &sd));
    }
    // routed experts: expert lists + gather, gate and up over each expert's rows, SwiGLU, down
    WIDE_TRY(launch(wide_route_gather, dim3(M * K), dim3(256), 0, st, s.sel_e, M, K, E, s.xhi, s.xlo, ldx, d, s.count, s.off, s.pair_row,
                                             s.pair_slot, s.stats, s.ghi, s.glo, s.active, s.n_active));
    ++n;
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.w_gate), static_cast<const __nv_bfloat16 *>(lw.w_up), E, F,
                  d, s.ghi, s.glo, ldx, M * K, s.off, s.count, M * K, s.gu, 2 * F, F, 0, s.part, st, nullptr,
                  s.active, s.n_active));
    WIDE_TRY(launch(wide_swiglu, dim3(M * K, (F + 255) / 256), dim3(256), 0, st, s.gu, F, s.ahi, s.alo, s.lda, Split{}));
    ++n;
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.w_down), nullptr, E, d, F, s.ahi, s.alo, s.lda, M * K,
                  s.off, s.count, M * K, s.yd, d, 0, 0, s.part, st, nullptr, s.active, s.n_active));
    float *dbg = s.dbg_hidden ? s.dbg_hidden + static_cast<long long>(l + 1) * s.max_rows * d : nullptr;
    WIDE_TRY(launch(wide_combine, dim3(M, (d + 255) / 256), dim3(256), 0, st, s.h, d, K, s.sel_w, s.pair_slot, s.yd, Fs > 0 ? s.ys : nullptr,
                                                           dbg, sd));
    ++n;
  }
  // final norm, lm_head, argmax
  WIDE_TRY(launch(wide_norm_split, dim3(M), dim3(1024), 0, st, s.h, s.final_norm, d, s.eps, s.xhi, s.xlo, ldx, Split{}));
  ++n;
  WIDE_TRY(gemm(n, s, s.lm_head, nullptr, 1, s.V, d, s.xhi, s.xlo, ldx, M, nullptr, nullptr, M, s.logits, s.V, 0, 0, s.part,
                st));
  WIDE_TRY(launch(wide_argmax, dim3(M), dim3(1024), 0, st, s.logits, s.V, s.argmax));
  if (launches) *launches = n + 1;
  return cudaSuccess;
}

}  // namespace mk
