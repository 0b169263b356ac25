// mk_wide.cu -- the decode step for wide blocks (8 < M <= 64 rows, e.g. a
// speculative verify block of 7 rows for 8 sequences), as a short sequence of
// launches.  With this many rows the dense projections are real contractions,
// so every matrix product runs on the 5th-generation tensor cores (tcgen05.mma
// from TMA-fed shared memory into a tensor-memory accumulator, bf16 in, fp32
// accumulate).  Activations enter the tensor cores as a bf16 pair
// (x = hi + lo, hi = bf16(x), lo = bf16(x - hi)), so each product keeps close
// to fp32 accuracy; weights are bf16 already.  The remaining steps (norms,
// rotary + cache append, attention, top-k, expert lists, SwiGLU, combine,
// argmax) are plain CUDA-core kernels.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "mk_internal.h"

namespace mk {
namespace {

__device__ __forceinline__ uint32_t sptr(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

// ---------------------------------------------------------------------------
// Y[r][n] (+)= sum_k W[n][k] * (xhi[r][k] + xlo[r][k]) on the 5th-generation
// tensor cores.  A CTA owns 128 weight rows (the MMA's M) of one problem and
// all of its activation rows (the MMA's N: 16 to 64), over its share of K:
//  - warp 0 (one thread) streams K in stages of 128 columns by TMA: per 64
//    columns a 128 x 64 weight box and the activation rows in 16-row boxes,
//    hi and lo, all 128B-swizzled, completing on the stage's full mbarrier;
//  - warp 1 (one thread) issues tcgen05.mma kind::f16 (bf16 x bf16 -> fp32),
//    K = 16 each, hi then lo into one accumulator in tensor memory, and
//    releases the stage with tcgen05.commit on its empty mbarrier;
//  - then every warp reads its 32 accumulator lanes (weight rows) with
//    tcgen05.ld and writes them out.
// grid = (ceil(N / 128), ksplit, problems).  Problem p's weights are rows
// [p * N, (p + 1) * N) of the weight map, its activation rows [row_off[p],
// row_off[p] + row_cnt[p]) (or [0, R) when row_off is NULL); it writes the
// same rows of Y.  With ksplit > 1 the CTA writes its K share into
// part[ks][row][n] for wide_gemm_finish.
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
constexpr int kTcThreads = 128;
constexpr int kTcTmemCols = 64;                        // fp32 accumulator columns: one per activation row
static_assert(kWideMaxRows <= kTcTmemCols, "one accumulator column per activation row");

struct GemmArgs {
  CUtensorMap mw;          // weights: [problems * N rows][K], box 64 x 128
  CUtensorMap mxh, mxl;    // activations hi / lo: [rows][K], box 64 x 16
  int N, K;
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

__global__ void __launch_bounds__(kTcThreads, 1) wide_gemm(const __grid_constant__ GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  // stages start on 1024-byte boundaries (the 128-byte swizzle repeats every 8 rows)
  uint8_t *smem = smem_raw + ((1024u - (sptr(smem_raw) & 1023u)) & 1023u);
  __shared__ __align__(8) uint64_t full[kTcStages], empty[kTcStages], done;
  __shared__ uint32_t tmem_base;
  const int prob = blockIdx.z;
  const int r0 = a.row_off ? a.row_off[prob] : 0;
  const int R = a.row_off ? a.row_cnt[prob] : a.R;
  if (R <= 0) return;  // the whole CTA, before anything is allocated
  const int n0 = blockIdx.x * kTcM;
  const int ksplit = gridDim.y, ks = blockIdx.y;
  const int nkc = (a.K + kTcBoxes * kTcK - 1) / (kTcBoxes * kTcK);
  const int kc0 = (nkc * ks) / ksplit, kc1 = (nkc * (ks + 1)) / ksplit, nk = kc1 - kc0;
  const int G = (R + kTcRowBox - 1) / kTcRowBox, NM = kTcRowBox * G;
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
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(sptr(&done)) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = tmem_base;
  // kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B, both
  // K-major, N = NM, M = 128
  const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(NM >> 3) << 17) |
                         (static_cast<uint32_t>(kTcM >> 4) << 24);
  if (warp == 0 && lane == 0) {  // TMA producer
    for (int i = 0; i < nk; ++i) {
      const int s = i % kTcStages;
      if (i >= kTcStages && !tc_wait(&empty[s], ((i / kTcStages) & 1) ^ 1, a.error)) break;
      uint8_t *st = smem + s * kTcStage;
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(sptr(&full[s])),
                   "r"(kTcBoxes * (kTcWBox + 2 * G * kTcBoxBytes))
                   : "memory");
      for (int b = 0; b < kTcBoxes; ++b) {  // columns past K read as zeros
        const int x = ((kc0 + i) * kTcBoxes + b) * kTcK;
        tc_tma(st + b * kTcWBox, &a.mw, x, prob * a.N + n0, &full[s]);
        for (int g = 0; g < G; ++g) {
          tc_tma(st + kTcA + b * kTcXBox + g * kTcBoxBytes, &a.mxh, x, r0 + kTcRowBox * g, &full[s]);
          tc_tma(st + kTcA + kTcB + b * kTcXBox + g * kTcBoxBytes, &a.mxl, x, r0 + kTcRowBox * g, &full[s]);
        }
      }
    }
  }
  if (warp == 1 && lane == 0) {  // MMA issuer
    for (int i = 0; i < nk; ++i) {
      const int s = i % kTcStages;
      if (!tc_wait(&full[s], (i / kTcStages) & 1, a.error)) break;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint8_t *st = smem + s * kTcStage;
#pragma unroll
      for (int b = 0; b < kTcBoxes; ++b) {
        const uint64_t da = tc_desc(st + b * kTcWBox), dh = tc_desc(st + kTcA + b * kTcXBox),
                       dl = tc_desc(st + kTcA + kTcB + b * kTcXBox);
#pragma unroll
        for (int kk = 0; kk < kTcK / 16; ++kk) {  // 16 columns = 32 bytes = 2 descriptor units
          tc_mma(tmem, da + 2 * kk, dh + 2 * kk, idesc, (i > 0 || b > 0 || kk > 0) ? 1u : 0u);
          tc_mma(tmem, da + 2 * kk, dl + 2 * kk, idesc, 1u);
        }
      }
      tc_commit(&empty[s]);  // the stage is free once these products have read it
    }
    tc_commit(&done);
  }
  __syncwarp();
  const bool ok = tc_wait(&done, 0, a.error) && nk > 0;
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  // warp w holds accumulator lanes 32w .. 32w + 31 = weight rows n0 + 32w + lane
  const int n = n0 + 32 * warp + lane;
  for (int c0 = 0; c0 < NM; c0 += 16) {
    uint32_t v[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
          "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(tmem + (static_cast<uint32_t>(32 * warp) << 16) + static_cast<uint32_t>(c0)));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const int r = c0 + j;
      if (r >= R || n >= a.N) continue;
      const float val = ok ? __uint_as_float(v[j]) : 0.f;
      if (ksplit > 1) {
        a.part[(static_cast<long long>(ks) * a.rows_total + r0 + r) * a.ldy + n] = val;
      } else {
        float *y = a.Y + static_cast<long long>(r0 + r) * a.ldy + n;
        *y = a.accumulate ? *y + val : val;
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTcTmemCols) : "memory");
}

// Y[r][n] (+)= sum over ks of part[ks][r][n], in order.
__global__ void wide_gemm_finish(const float *part, int ksplit, int rows, int N, int ld, float *Y, int accumulate) {
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

// h[m] = embed[token[m]]; the debug copy of the layer-0 input.
__global__ void wide_embed(const int32_t *tokens, const __nv_bfloat16 *embed, int d, float *h, float *dbg) {
  const int m = blockIdx.x;
  const int tok = tokens[m];
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const float v = __bfloat162float(embed[static_cast<long long>(tok) * d + c]);
    h[static_cast<long long>(m) * d + c] = v;
    if (dbg) dbg[static_cast<long long>(m) * d + c] = v;
  }
}

// x = h / sqrt(mean(h^2) + eps) * g, as a bf16 pair.
__global__ void wide_norm_split(const float *h, const __nv_bfloat16 *g, int d, float eps, __nv_bfloat16 *xhi,
                                __nv_bfloat16 *xlo, int ldx) {
  __shared__ float red[32];
  const int m = blockIdx.x;
  const float *row = h + static_cast<long long>(m) * d;
  float s = 0.f;
  for (int c = threadIdx.x; c < d; c += blockDim.x) s = fmaf(row[c], row[c], s);
  s = block_sum(s, red);
  const float inv = 1.0f / sqrtf(s / static_cast<float>(d) + eps);
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    const float x = row[c] * inv * __bfloat162float(g[c]);
    split_store(x, xhi + static_cast<long long>(m) * ldx + c, xlo + static_cast<long long>(m) * ldx + c);
  }
}

// plain split of rows [M][K] (stride lds) into the bf16 pair
__global__ void wide_split(const float *src, int K, int lds, __nv_bfloat16 *xhi, __nv_bfloat16 *xlo, int ldx) {
  const int m = blockIdx.x;
  for (int c = threadIdx.x; c < K; c += blockDim.x)
    split_store(src[static_cast<long long>(m) * lds + c], xhi + static_cast<long long>(m) * ldx + c,
                xlo + static_cast<long long>(m) * ldx + c);
}

// Rotary embedding of k at each new row's position, k and v rounded to bf16
// and written into the cache.  grid = (M, Hkv).
__global__ void wide_kv_append(const float *qkv, int W3, const int32_t *positions, int T, int Hq, int Hkv, int hd,
                               const float2 *rope, __nv_bfloat16 *kc, __nv_bfloat16 *vc, int Bmax, int cap,
                               int layer) {
  const int m = blockIdx.x, g = blockIdx.y, b = m / T, t = m % T;
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

// Attention of a wide block, split over the KV positions: one block per
// (sequence, KV head, chunk of kWaChunk positions) stages the chunk's K and V
// rows in shared memory once and scores every query vector of the group
// against them (T rows x Hq/Hkv heads, each seeing positions up to its own),
// writing per query an unnormalised partial output with its running max and
// sum; wide_attn_merge combines a query's chunks with the log-sum-exp rule.
// Lane j of a warp scores positions j and j + 32 of the chunk (rows padded
// by 8 bf16 so that the lanes' row reads fall in different banks); for P.V
// lane l owns dims [DPL l, DPL l + DPL).
constexpr int kWaChunk = 64;
constexpr int kWaWarps = 8;
constexpr int kWaPad = 8;
template <int DPL>
__global__ void __launch_bounds__(kWaWarps * 32) wide_attn_chunk(
    const float *qkv, int W3, const int32_t *positions, int T, int Hq, int Hkv, const float2 *rope,
    const __nv_bfloat16 *kc, const __nv_bfloat16 *vc, int Bmax, int cap, int layer, int nch_max, float *opart,
    float *mlpart) {
  constexpr int HD = 32 * DPL, HALF = HD / 2, LD = HD + kWaPad;
  __shared__ __align__(16) __nv_bfloat16 sk[kWaChunk * LD], sv[kWaChunk * LD];
  __shared__ __align__(16) float sq[kWaWarps][HD];
  const int c = blockIdx.x, bg = blockIdx.y, b = bg / Hkv, g = bg % Hkv, G = Hq / Hkv;
  const int pos0 = positions[b], last = pos0 + T - 1;  // the block's last query sees up to `last`
  const int j0 = c * kWaChunk;
  if (j0 > last) return;
  const int nj = min(kWaChunk, last + 1 - j0);
  const long long base = ((static_cast<long long>(layer) * Bmax + b) * Hkv + g) * cap;
  // stage the chunk's rows: 16-byte pieces, HD / 8 per row
  for (int i = threadIdx.x; i < nj * (HD / 8); i += blockDim.x) {
    const int j = i / (HD / 8), piece = i % (HD / 8);
    const uint4 kv4 = *reinterpret_cast<const uint4 *>(kc + (base + j0 + j) * HD + piece * 8);
    const uint4 vv4 = *reinterpret_cast<const uint4 *>(vc + (base + j0 + j) * HD + piece * 8);
    *reinterpret_cast<uint4 *>(sk + j * LD + piece * 8) = kv4;
    *reinterpret_cast<uint4 *>(sv + j * LD + piece * 8) = vv4;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float scale = 1.0f / sqrtf(static_cast<float>(HD));
  const int Q = T * G;
  for (int qi = warp; qi < Q; qi += kWaWarps) {
    const int t = qi / G, h = g * G + qi % G, m = b * T + t, lim = pos0 + t;
    // the query vector, rotated (rotate-half pairs) and scaled, in this warp's buffer
    const float *q = qkv + static_cast<long long>(m) * W3 + h * HD;
    for (int i = lane; i < HALF; i += 32) {
      const float2 cs = rope[static_cast<long long>(lim) * HALF + i];
      const float x1 = q[i], x2 = q[i + HALF];
      sq[warp][i] = (x1 * cs.x - x2 * cs.y) * scale;
      sq[warp][i + HALF] = (x2 * cs.x + x1 * cs.y) * scale;
    }
    __syncwarp();
    float s[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int j = lane + 32 * u;
      float acc = 0.f;
      if (j < nj && j0 + j <= lim) {
        const __nv_bfloat16 *kr = sk + j * LD;
#pragma unroll 8
        for (int d = 0; d < HD; d += 8) {
          const uint4 kk = *reinterpret_cast<const uint4 *>(kr + d);
          const float4 qa = *reinterpret_cast<const float4 *>(&sq[warp][d]);
          const float4 qb = *reinterpret_cast<const float4 *>(&sq[warp][d + 4]);
          acc = fmaf(qa.x, __uint_as_float(kk.x << 16), acc);
          acc = fmaf(qa.y, __uint_as_float(kk.x & 0xffff0000u), acc);
          acc = fmaf(qa.z, __uint_as_float(kk.y << 16), acc);
          acc = fmaf(qa.w, __uint_as_float(kk.y & 0xffff0000u), acc);
          acc = fmaf(qb.x, __uint_as_float(kk.z << 16), acc);
          acc = fmaf(qb.y, __uint_as_float(kk.z & 0xffff0000u), acc);
          acc = fmaf(qb.z, __uint_as_float(kk.w << 16), acc);
          acc = fmaf(qb.w, __uint_as_float(kk.w & 0xffff0000u), acc);
        }
        s[u] = acc;
      } else {
        s[u] = -INFINITY;
      }
    }
    float mx = fmaxf(s[0], s[1]);
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float p[2], l = 0.f;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      p[u] = (s[u] == -INFINITY) ? 0.f : expf(s[u] - mx);
      l += p[u];
    }
    for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    float acc[DPL];
#pragma unroll
    for (int dd = 0; dd < DPL; ++dd) acc[dd] = 0.f;
    if (mx != -INFINITY) {
      for (int j = 0; j < nj; ++j) {
        const float pj = __shfl_sync(0xffffffffu, p[j >> 5], j & 31);
        const __nv_bfloat16 *vr = sv + j * LD + lane * DPL;
#pragma unroll
        for (int dd = 0; dd < DPL; ++dd) acc[dd] = fmaf(pj, __bfloat162float(vr[dd]), acc[dd]);
      }
    }
    const long long slot = (static_cast<long long>(bg) * nch_max + c) * (static_cast<long long>(T) * G) + qi;
    float *dst = opart + slot * HD + lane * DPL;
#pragma unroll
    for (int dd = 0; dd < DPL; ++dd) dst[dd] = acc[dd];
    if (lane == 0) {
      mlpart[2 * slot] = mx;
      mlpart[2 * slot + 1] = l;
    }
    __syncwarp();  // the buffer of q is rewritten by the warp's next query
  }
}

// o[m][h] = the log-sum-exp combination of query (m, h)'s chunk partials.
// One block of HD threads per (row, head); thread i owns dim i.
__global__ void wide_attn_merge(const int32_t *positions, int T, int Hq, int Hkv, int hd, int nch_max,
                                const float *opart, const float *mlpart, float *o) {
  const int m = blockIdx.x, h = blockIdx.y, b = m / T, t = m % T, G = Hq / Hkv, g = h / G;
  const int qi = t * G + h % G, bg = b * Hkv + g;
  const int nch = (positions[b] + t) / kWaChunk + 1;  // chunks holding positions this query sees
  float M = -INFINITY;
  for (int c = 0; c < nch; ++c) {
    const long long slot = (static_cast<long long>(bg) * nch_max + c) * (static_cast<long long>(T) * G) + qi;
    M = fmaxf(M, mlpart[2 * slot]);
  }
  for (int i = threadIdx.x; i < hd; i += blockDim.x) {
    float num = 0.f, den = 0.f;
    for (int c = 0; c < nch; ++c) {
      const long long slot = (static_cast<long long>(bg) * nch_max + c) * (static_cast<long long>(T) * G) + qi;
      const float mc = mlpart[2 * slot];
      if (mc == -INFINITY) continue;
      const float w = expf(mc - M);
      num = fmaf(w, opart[slot * hd + i], num);
      den = fmaf(w, mlpart[2 * slot + 1], den);
    }
    o[static_cast<long long>(m) * Hq * hd + h * hd + i] = num / den;
  }
}

// Per row: softmax over the E router logits, top-k (ties to the lower id),
// weights renormalised by their sum.  One warp per row.
__global__ void wide_topk(const float *logits, int E, int K, int32_t *sel_e, float *sel_w, int32_t *dbg_ids,
                          float *dbg_w) {
  const int m = blockIdx.x, lane = threadIdx.x;
  const float *z = logits + static_cast<long long>(m) * E;
  float mx = -INFINITY;
  for (int e = lane; e < E; e += 32) mx = fmaxf(mx, z[e]);
  for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
  for (int e = lane; e < E; e += 32) sum += expf(z[e] - mx);
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  uint32_t taken[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // bit e of expert e (E <= 256)
  float sel = 0.f, my_w = 0.f;
  int my_e = 0;
  for (int j = 0; j < K; ++j) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int e = lane; e < E; e += 32) {
      if ((taken[e >> 5] >> (e & 31)) & 1u) continue;
      const float pe = expf(z[e] - mx) / sum;
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

// Pairs (row m, selection j) grouped by expert, in (expert, m, j) order:
// count[e], off[e], pair_row[q], pair_slot[m * K + j] = position q of the
// pair.  One block; also adds the number of distinct experts to stats.
__global__ void wide_expert_lists(const int32_t *sel_e, int M, int K, int E, int *count, int *off, int *pair_row,
                                  int *pair_slot, unsigned long long *stats) {
  __shared__ int cnt[kMaxExperts], start[kMaxExperts];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < M * K; i += blockDim.x) atomicAdd(&cnt[sel_e[i]], 1);
  __syncthreads();
  if (threadIdx.x == 0) {
    int s = 0, nu = 0;
    for (int e = 0; e < E; ++e) {
      start[e] = s;
      off[e] = s;
      count[e] = cnt[e];
      s += cnt[e];
      nu += cnt[e] ? 1 : 0;
    }
    atomicAdd(stats, static_cast<unsigned long long>(nu));
    // stable placement in (m, j) order
    for (int i = 0; i < M * K; ++i) {
      const int e = sel_e[i];
      const int q = start[e]++;
      pair_row[q] = i / K;
      pair_slot[i] = q;
    }
  }
}

// rows of the bf16 pair gathered into pair order
__global__ void wide_gather(const __nv_bfloat16 *xhi, const __nv_bfloat16 *xlo, int ldx, const int *pair_row, int K,
                            __nv_bfloat16 *ghi, __nv_bfloat16 *glo) {
  const int q = blockIdx.x, m = pair_row[q];
  for (int c = threadIdx.x; c < K; c += blockDim.x) {
    ghi[static_cast<long long>(q) * ldx + c] = xhi[static_cast<long long>(m) * ldx + c];
    glo[static_cast<long long>(q) * ldx + c] = xlo[static_cast<long long>(m) * ldx + c];
  }
}

// act = silu(gate) * up for rows [rows][2F] (gate then up), as a bf16 pair
__global__ void wide_swiglu(const float *gu, int F, __nv_bfloat16 *ahi, __nv_bfloat16 *alo, int lda) {
  const int q = blockIdx.x;
  for (int c = threadIdx.x; c < F; c += blockDim.x) {
    const float gt = gu[static_cast<long long>(q) * 2 * F + c], up = gu[static_cast<long long>(q) * 2 * F + F + c];
    split_store(gt / (1.0f + expf(-gt)) * up, ahi + static_cast<long long>(q) * lda + c,
                alo + static_cast<long long>(q) * lda + c);
  }
}

// h[m] += sum_j w[m][j] y[pair(m, j)] (selection order) + shared[m]
__global__ void wide_combine(float *h, int d, int K, const float *sel_w, const int *pair_slot, const float *y,
                             const float *ys, float *dbg) {
  const int m = blockIdx.x;
  for (int c = threadIdx.x; c < d; c += blockDim.x) {
    float moe = 0.f;
    for (int j = 0; j < K; ++j)
      moe = fmaf(sel_w[m * K + j], y[static_cast<long long>(pair_slot[m * K + j]) * d + c], moe);
    const float v = h[static_cast<long long>(m) * d + c] + (ys ? moe + ys[static_cast<long long>(m) * d + c] : moe);
    h[static_cast<long long>(m) * d + c] = v;
    if (dbg) dbg[static_cast<long long>(m) * d + c] = v;
  }
}

// argmax over the vocabulary per row (ties to the lowest index)
__global__ void wide_argmax(const float *logits, int V, int32_t *out) {
  __shared__ float bvs[32];
  __shared__ int bis[32];
  const int m = blockIdx.x;
  float bv = -INFINITY;
  int bi = 0x7fffffff;
  for (int v = threadIdx.x; v < V; v += blockDim.x) {
    const float x = logits[static_cast<long long>(m) * V + v];
    if (x > bv || (x == bv && v < bi)) {
      bv = x;
      bi = v;
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

int gemm_smem_bytes() { return kTcStages * kTcStage + 1024; }  // + room to align the stages to 1024 bytes

}  // namespace

// ---------------------------------------------------------------------------
// Host driver
// ---------------------------------------------------------------------------
#define WIDE_TRY(x)                   \
  do {                                \
    cudaError_t e__ = (x);            \
    if (e__ != cudaSuccess) return e__; \
  } while (0)

// One product (or one grouped launch of per-expert products) on the tensor
// cores: weight rows [p * N, (p + 1) * N) x K for problem p, activation rows
// of the xrows-row buffers xhi / xlo (row stride ldx).  A single dense problem
// whose 128-row tiles do not fill the GPU splits K.
static cudaError_t gemm(int &n, const WideStep &s, const __nv_bfloat16 *W, int problems, int N, int K,
                        const __nv_bfloat16 *xhi, const __nv_bfloat16 *xlo, int ldx, int xrows, const int *row_off,
                        const int *row_cnt, int R, float *Y, int ldy, int accumulate, cudaStream_t st) {
  GemmArgs a{};
  if (encode_2d_sw128(&a.mw, W, static_cast<uint64_t>(problems) * N, K, K, kTcM) != MK_OK ||
      encode_2d_sw128(&a.mxh, xhi, xrows, K, ldx, kTcRowBox) != MK_OK ||
      encode_2d_sw128(&a.mxl, xlo, xrows, K, ldx, kTcRowBox) != MK_OK)
    return cudaErrorInvalidValue;
  a.N = N;
  a.K = K;
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
    const int nkc = (K + kTcBoxes * kTcK - 1) / (kTcBoxes * kTcK);
    ksplit = std::max(1, std::min(std::min(s.n_sm / nb, nkc / 2), 16));
    if (static_cast<long long>(ksplit) * R * ldy > s.part_floats) ksplit = 1;
  }
  a.part = ksplit > 1 ? s.part : nullptr;
  wide_gemm<<<dim3(nb, ksplit, problems), kTcThreads, gemm_smem_bytes(), st>>>(a);
  WIDE_TRY(cudaGetLastError());
  ++n;
  if (ksplit > 1) {
    wide_gemm_finish<<<2 * s.n_sm, 256, 0, st>>>(s.part, ksplit, R, N, ldy, Y, accumulate);
    WIDE_TRY(cudaGetLastError());
    ++n;
  }
  return cudaSuccess;
}

cudaError_t wide_prepare() {
  return cudaFuncSetAttribute(wide_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, gemm_smem_bytes());
}

cudaError_t wide_step(const WideStep &s, cudaStream_t st, int *launches) {
  int n = 0;
  const int M = s.B * s.T, d = s.d, L = s.L, K = s.topk, E = s.E, F = s.F, Fs = s.Fs;
  const int W3 = (s.Hq + 2 * s.Hkv) * s.hd, HD = s.Hq * s.hd;
  const int ldx = s.ldx;  // >= max(d, HD), multiple of 8
  wide_check<<<1, 256, 0, st>>>(s.tokens, s.positions, s.B, s.T, s.V, s.cap, s.tokens_safe, s.positions_safe,
                                s.error);
  WIDE_TRY(cudaGetLastError());
  ++n;
  wide_embed<<<M, 256, 0, st>>>(s.tokens_safe, s.embed, d, s.h, s.dbg_hidden);
  WIDE_TRY(cudaGetLastError());
  ++n;
  for (int l = 0; l < L; ++l) {
    const mk_layer_weights &lw = s.layers[l];
    // attention block
    wide_norm_split<<<M, 256, 0, st>>>(s.h, static_cast<const __nv_bfloat16 *>(lw.attn_norm), d, s.eps, s.xhi,
                                       s.xlo, ldx);
    WIDE_TRY(cudaGetLastError());
    ++n;
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.wqkv), 1, W3, d, s.xhi, s.xlo, ldx, M, nullptr, nullptr, M,
                  s.qkv, W3, 0, st));
    wide_kv_append<<<dim3(M, s.Hkv), 128, 0, st>>>(s.qkv, W3, s.positions_safe, s.T, s.Hq, s.Hkv, s.hd, s.rope, s.kc,
                                                   s.vc, s.Bmax, s.cap, l);
    WIDE_TRY(cudaGetLastError());
    ++n;
    {
      const int nch = (s.cap + kWaChunk - 1) / kWaChunk;
      const dim3 grid(nch, s.B * s.Hkv);
      if (s.hd == 64)
        wide_attn_chunk<2><<<grid, kWaWarps * 32, 0, st>>>(s.qkv, W3, s.positions_safe, s.T, s.Hq, s.Hkv, s.rope, s.kc,
                                                            s.vc, s.Bmax, s.cap, l, nch, s.attn_o, s.attn_ml);
      else
        wide_attn_chunk<4><<<grid, kWaWarps * 32, 0, st>>>(s.qkv, W3, s.positions_safe, s.T, s.Hq, s.Hkv, s.rope, s.kc,
                                                            s.vc, s.Bmax, s.cap, l, nch, s.attn_o, s.attn_ml);
      WIDE_TRY(cudaGetLastError());
      ++n;
      wide_attn_merge<<<dim3(M, s.Hq), s.hd, 0, st>>>(s.positions_safe, s.T, s.Hq, s.Hkv, s.hd, nch, s.attn_o,
                                                      s.attn_ml, s.o);
      WIDE_TRY(cudaGetLastError());
      ++n;
    }
    wide_split<<<M, 256, 0, st>>>(s.o, HD, HD, s.xhi, s.xlo, ldx);
    WIDE_TRY(cudaGetLastError());
    ++n;
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.wo), 1, d, HD, s.xhi, s.xlo, ldx, M, nullptr, nullptr, M,
                  s.h, d, 1, st));
    // MoE block: router on the normed row, top-k, expert lists
    wide_norm_split<<<M, 256, 0, st>>>(s.h, static_cast<const __nv_bfloat16 *>(lw.ffn_norm), d, s.eps, s.xhi, s.xlo,
                                       ldx);
    WIDE_TRY(cudaGetLastError());
    ++n;
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.router), 1, E, d, s.xhi, s.xlo, ldx, M, nullptr, nullptr, M,
                  s.rlog, E, 0, st));
    int32_t *dbg_ids = s.dbg_ids ? s.dbg_ids + static_cast<long long>(l) * s.max_rows * K : nullptr;
    float *dbg_w = s.dbg_w ? s.dbg_w + static_cast<long long>(l) * s.max_rows * K : nullptr;
    wide_topk<<<M, 32, 0, st>>>(s.rlog, E, K, s.sel_e, s.sel_w, dbg_ids, dbg_w);
    WIDE_TRY(cudaGetLastError());
    ++n;
    wide_expert_lists<<<1, 256, 0, st>>>(s.sel_e, M, K, E, s.count, s.off, s.pair_row, s.pair_slot, s.stats);
    WIDE_TRY(cudaGetLastError());
    ++n;
    // routed experts: gate and up over each expert's rows, SwiGLU, down
    wide_gather<<<M * K, 256, 0, st>>>(s.xhi, s.xlo, ldx, s.pair_row, d, s.ghi, s.glo);
    WIDE_TRY(cudaGetLastError());
    ++n;
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.w_gate), E, F, d, s.ghi, s.glo, ldx, M * K, s.off, s.count,
                  M * K, s.gu, 2 * F, 0, st));
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.w_up), E, F, d, s.ghi, s.glo, ldx, M * K, s.off, s.count,
                  M * K, s.gu + F, 2 * F, 0, st));
    wide_swiglu<<<M * K, 256, 0, st>>>(s.gu, F, s.ahi, s.alo, s.lda);
    WIDE_TRY(cudaGetLastError());
    ++n;
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.w_down), E, d, F, s.ahi, s.alo, s.lda, M * K, s.off,
                  s.count, M * K, s.yd, d, 0, st));
    // shared expert on every row
    if (Fs > 0) {
      WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.ws_gate), 1, Fs, d, s.xhi, s.xlo, ldx, M, nullptr,
                    nullptr, M, s.gs, 2 * Fs, 0, st));
      WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.ws_up), 1, Fs, d, s.xhi, s.xlo, ldx, M, nullptr, nullptr,
                    M, s.gs + Fs, 2 * Fs, 0, st));
      wide_swiglu<<<M, 256, 0, st>>>(s.gs, Fs, s.shi, s.slo, s.lda);
      WIDE_TRY(cudaGetLastError());
      ++n;
      WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.ws_down), 1, d, Fs, s.shi, s.slo, s.lda, M, nullptr,
                    nullptr, M, s.ys, d, 0, st));
    }
    float *dbg = s.dbg_hidden ? s.dbg_hidden + static_cast<long long>(l + 1) * s.max_rows * d : nullptr;
    wide_combine<<<M, 256, 0, st>>>(s.h, d, K, s.sel_w, s.pair_slot, s.yd, Fs > 0 ? s.ys : nullptr, dbg);
    WIDE_TRY(cudaGetLastError());
    ++n;
  }
  // final norm, lm_head, argmax
  wide_norm_split<<<M, 256, 0, st>>>(s.h, s.final_norm, d, s.eps, s.xhi, s.xlo, ldx);
  WIDE_TRY(cudaGetLastError());
  ++n;
  WIDE_TRY(gemm(n, s, s.lm_head, 1, s.V, d, s.xhi, s.xlo, ldx, M, nullptr, nullptr, M, s.logits, s.V, 0, st));
  wide_argmax<<<M, 256, 0, st>>>(s.logits, s.V, s.argmax);
  WIDE_TRY(cudaGetLastError());
  if (launches) *launches = n + 1;
  return cudaSuccess;
}

}  // namespace mk
