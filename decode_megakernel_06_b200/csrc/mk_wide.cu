// mk_wide.cu -- the decode step for wide blocks (8 < M <= 64 rows, e.g. a
// speculative verify block of 7 rows for 8 sequences), as a short sequence of
// launches.  With this many rows the dense projections are real contractions,
// so every matrix product runs on the tensor cores (mma.sync m16n8k16, bf16 in,
// fp32 accumulate).  Activations enter the tensor cores as a bf16 pair
// (x = hi + lo, hi = bf16(x), lo = bf16(x - hi)), so each product keeps close
// to fp32 accuracy; weights are bf16 already.  The remaining steps (norms,
// rotary + cache append, attention, top-k, expert lists, SwiGLU, combine,
// argmax) are plain CUDA-core kernels.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "mk_internal.h"

namespace mk {
namespace {

constexpr int kGemmN = 64;    // weight rows per block (MMA M, 4 warps x 16)
constexpr int kGemmR = 64;    // activation rows per block (MMA N, 8 x 8)
constexpr int kGemmK = 64;    // K columns per stage
constexpr int kLd = kGemmK + 8;  // padded smem row (bf16): ldmatrix without bank conflicts
constexpr int kGemmThreads = 128;

__device__ __forceinline__ uint32_t sptr(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

// 16-byte async copy; src_bytes < 16 fills the rest with zeros.
__device__ __forceinline__ void cp16(void *dst, const void *src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sptr(dst)), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all_but_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(sptr(p)));
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// Y[r][n] (+)= sum_k W[n][k] * (xhi[r][k] + xlo[r][k]) for the rows of one
// problem.  grid = (ceil(N / 64), ksplit, problems).  Problem p uses weights
// W + p * wstride, activation rows [row_off[p], row_off[p] + row_cnt[p]) (or
// [0, R) when row_off is NULL) and writes the same rows of Y.  With ksplit > 1
// the block writes its K share into part[ks][row][n] for wide_gemm_finish.
// ---------------------------------------------------------------------------
struct GemmArgs {
  const __nv_bfloat16 *W;
  long long wstride;
  int N, K;
  const __nv_bfloat16 *xhi, *xlo;
  int ldx;
  const int *row_off, *row_cnt;
  int R;
  float *Y;
  int ldy;
  int accumulate;  // 1: Y += result (ksplit == 1 only)
  float *part;     // [ksplit][rows][ldy] when ksplit > 1
  int rows_total;  // rows of Y (for part's stride)
};

__global__ void __launch_bounds__(kGemmThreads) wide_gemm(GemmArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int prob = blockIdx.z;
  const int r0 = a.row_off ? a.row_off[prob] : 0;
  const int R = a.row_off ? a.row_cnt[prob] : a.R;
  if (R <= 0) return;
  const int n0 = blockIdx.x * kGemmN;
  const int ksplit = gridDim.y, ks = blockIdx.y;
  const int nkc = (a.K + kGemmK - 1) / kGemmK;
  const int kc0 = (nkc * ks) / ksplit, kc1 = (nkc * (ks + 1)) / ksplit;
  const __nv_bfloat16 *W = a.W + static_cast<long long>(prob) * a.wstride;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __nv_bfloat16 *sW = reinterpret_cast<__nv_bfloat16 *>(smem);           // [2][64][kLd]
  __nv_bfloat16 *sH = sW + 2 * kGemmN * kLd;                               // [2][64][kLd]
  __nv_bfloat16 *sL = sH + 2 * kGemmR * kLd;                               // [2][64][kLd]

  auto load_stage = [&](int st, int kc) {
    const int k0 = kc * kGemmK;
    // weights: 64 rows x 8 chunks of 8 bf16
    for (int i = tid; i < kGemmN * 8; i += kGemmThreads) {
      const int row = i >> 3, ch = i & 7, k = k0 + ch * 8, n = n0 + row;
      const bool ok = n < a.N && k < a.K;
      const __nv_bfloat16 *src = ok ? W + static_cast<long long>(n) * a.K + k : W;
      cp16(sW + (st * kGemmN + row) * kLd + ch * 8, src, ok ? 16 : 0);
    }
    for (int i = tid; i < kGemmR * 8; i += kGemmThreads) {
      const int row = i >> 3, ch = i & 7, k = k0 + ch * 8;
      const bool ok = row < R && k < a.K;
      const long long off = ok ? static_cast<long long>(r0 + row) * a.ldx + k : 0;
      cp16(sH + (st * kGemmR + row) * kLd + ch * 8, a.xhi + off, ok ? 16 : 0);
      cp16(sL + (st * kGemmR + row) * kLd + ch * 8, a.xlo + off, ok ? 16 : 0);
    }
    cp_commit();
  };

  float acc[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[j][q] = 0.f;
  const int nrt = (R + 7) / 8;  // 8-row activation tiles that hold rows

  if (kc0 < kc1) load_stage(0, kc0);
  for (int kc = kc0; kc < kc1; ++kc) {
    const int st = (kc - kc0) & 1;
    if (kc + 1 < kc1) {
      load_stage(st ^ 1, kc + 1);
      cp_wait_all_but_one();
    } else {
      cp_wait_all();
    }
    __syncthreads();
    const __nv_bfloat16 *w_s = sW + st * kGemmN * kLd;
    const __nv_bfloat16 *h_s = sH + st * kGemmR * kLd;
    const __nv_bfloat16 *l_s = sL + st * kGemmR * kLd;
#pragma unroll
    for (int kk = 0; kk < kGemmK; kk += 16) {
      uint32_t af[4];
      {
        const int mi = lane >> 3, ri = lane & 7;
        ldsm_x4(af, w_s + (warp * 16 + (mi & 1) * 8 + ri) * kLd + kk + (mi >> 1) * 8);
      }
#pragma unroll
      for (int jp = 0; jp < 4; ++jp) {  // two 8-row activation tiles per ldmatrix
        if (2 * jp >= nrt) break;
        const int mi = lane >> 3, ri = lane & 7;
        const int row = jp * 16 + (mi >> 1) * 8 + ri, col = kk + (mi & 1) * 8;
        uint32_t bh[4], bl[4];
        ldsm_x4(bh, h_s + row * kLd + col);
        ldsm_x4(bl, l_s + row * kLd + col);
        mma_bf16(acc[2 * jp], af, bh[0], bh[1]);
        mma_bf16(acc[2 * jp], af, bl[0], bl[1]);
        mma_bf16(acc[2 * jp + 1], af, bh[2], bh[3]);
        mma_bf16(acc[2 * jp + 1], af, bl[2], bl[3]);
      }
    }
    __syncthreads();
  }
  // D fragment: acc[j] = (weight row g, act rows 2t, 2t+1), (weight row g + 8, same)
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int n = n0 + warp * 16 + g + (q >> 1) * 8;
      const int r = j * 8 + 2 * t + (q & 1);
      if (n >= a.N || r >= R) continue;
      if (ksplit > 1) {
        a.part[(static_cast<long long>(ks) * a.rows_total + r0 + r) * a.ldy + n] = acc[j][q];
      } else {
        float *y = a.Y + static_cast<long long>(r0 + r) * a.ldy + n;
        *y = a.accumulate ? *y + acc[j][q] : acc[j][q];
      }
    }
  }
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

// Softmax attention of one (row, query head) over cache positions 0..p,
// including the rows this step appended.  grid = (M, Hq), 128 threads: each
// warp keeps an online softmax over every 4th position, lanes across the
// head dimension; the warps merge at the end.
constexpr int kAttnWarps = 4;
__global__ void __launch_bounds__(kAttnWarps * 32) wide_attention(
    const float *qkv, int W3, const int32_t *positions, int T, int Hq, int Hkv, int hd, const float2 *rope,
    const __nv_bfloat16 *kc, const __nv_bfloat16 *vc, int Bmax, int cap, int layer, float *o) {
  __shared__ float sq[128];
  __shared__ float sm[kAttnWarps], sl[kAttnWarps];
  __shared__ float so[kAttnWarps][128];
  const int m = blockIdx.x, h = blockIdx.y, b = m / T, t = m % T;
  const int p = positions[b] + t, half = hd / 2, G = Hq / Hkv, g = h / G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float scale = 1.0f / sqrtf(static_cast<float>(hd));
  const float *q = qkv + static_cast<long long>(m) * W3 + h * hd;
  for (int i = threadIdx.x; i < hd; i += blockDim.x) {
    const int j = i < half ? i : i - half;
    const float2 cs = rope[static_cast<long long>(p) * half + j];
    const float qr = i < half ? q[i] * cs.x - q[i + half] * cs.y : q[i] * cs.x + q[i - half] * cs.y;
    sq[i] = qr * scale;
  }
  __syncthreads();
  const int dpl = hd / 32;  // 2 or 4 dims per lane
  float qv[4], acc[4];
  for (int i = 0; i < 4; ++i) {
    qv[i] = i < dpl ? sq[lane * dpl + i] : 0.f;
    acc[i] = 0.f;
  }
  const long long base = ((static_cast<long long>(layer) * Bmax + b) * Hkv + g) * cap;
  float mrun = -INFINITY, lrun = 0.f;
  for (int j = warp; j <= p; j += kAttnWarps) {
    const __nv_bfloat16 *kr = kc + (base + j) * hd + lane * dpl;
    float s = 0.f;
    for (int i = 0; i < dpl; ++i) s = fmaf(qv[i], __bfloat162float(kr[i]), s);
    for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    const float mn = fmaxf(mrun, s);
    const float a = (mrun == -INFINITY) ? 0.f : expf(mrun - mn);
    const float e = expf(s - mn);
    lrun = lrun * a + e;
    const __nv_bfloat16 *vr = vc + (base + j) * hd + lane * dpl;
    for (int i = 0; i < dpl; ++i) acc[i] = acc[i] * a + e * __bfloat162float(vr[i]);
    mrun = mn;
  }
  if (lane == 0) {
    sm[warp] = mrun;
    sl[warp] = lrun;
  }
  for (int i = 0; i < dpl; ++i) so[warp][lane * dpl + i] = acc[i];
  __syncthreads();
  float M = -INFINITY;
  for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, sm[w]);
  float L = 0.f;
  for (int w = 0; w < kAttnWarps; ++w) L += (sm[w] == -INFINITY) ? 0.f : expf(sm[w] - M) * sl[w];
  for (int i = threadIdx.x; i < hd; i += blockDim.x) {
    float s = 0.f;
    for (int w = 0; w < kAttnWarps; ++w) s += (sm[w] == -INFINITY) ? 0.f : expf(sm[w] - M) * so[w][i];
    o[static_cast<long long>(m) * Hq * hd + h * hd + i] = s / L;
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

int gemm_smem_bytes() { return 2 * (kGemmN + 2 * kGemmR) * kLd * static_cast<int>(sizeof(__nv_bfloat16)); }

}  // namespace

// ---------------------------------------------------------------------------
// Host driver
// ---------------------------------------------------------------------------
#define WIDE_TRY(x)                   \
  do {                                \
    cudaError_t e__ = (x);            \
    if (e__ != cudaSuccess) return e__; \
  } while (0)

static cudaError_t gemm(int &n, const WideStep &s, const __nv_bfloat16 *W, long long wstride, int N, int K,
                        const __nv_bfloat16 *xhi, const __nv_bfloat16 *xlo, int ldx, const int *row_off,
                        const int *row_cnt, int problems, int R, float *Y, int ldy, int accumulate,
                        cudaStream_t st) {
  GemmArgs a{};
  a.W = W;
  a.wstride = wstride;
  a.N = N;
  a.K = K;
  a.xhi = xhi;
  a.xlo = xlo;
  a.ldx = ldx;
  a.row_off = row_off;
  a.row_cnt = row_cnt;
  a.R = R;
  a.Y = Y;
  a.ldy = ldy;
  a.accumulate = accumulate;
  a.rows_total = R;
  const int nb = (N + kGemmN - 1) / kGemmN;
  int ksplit = 1;
  if (!row_off) {  // one dense problem: split K until the grid covers the GPU twice
    const int nkc = (K + kGemmK - 1) / kGemmK;
    while (nb * ksplit < 2 * s.n_sm && ksplit * 2 <= nkc && ksplit < 16) ksplit *= 2;
    if (static_cast<long long>(ksplit) * R * ldy > s.part_floats) ksplit = 1;
  }
  a.part = ksplit > 1 ? s.part : nullptr;
  wide_gemm<<<dim3(nb, ksplit, problems), kGemmThreads, gemm_smem_bytes(), st>>>(a);
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
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.wqkv), 0, W3, d, s.xhi, s.xlo, ldx, nullptr, nullptr, 1, M,
                  s.qkv, W3, 0, st));
    wide_kv_append<<<dim3(M, s.Hkv), 128, 0, st>>>(s.qkv, W3, s.positions_safe, s.T, s.Hq, s.Hkv, s.hd, s.rope, s.kc,
                                                   s.vc, s.Bmax, s.cap, l);
    WIDE_TRY(cudaGetLastError());
    ++n;
    wide_attention<<<dim3(M, s.Hq), kAttnWarps * 32, 0, st>>>(s.qkv, W3, s.positions_safe, s.T, s.Hq, s.Hkv, s.hd,
                                                              s.rope, s.kc, s.vc, s.Bmax, s.cap, l, s.o);
    WIDE_TRY(cudaGetLastError());
    ++n;
    wide_split<<<M, 256, 0, st>>>(s.o, HD, HD, s.xhi, s.xlo, ldx);
    WIDE_TRY(cudaGetLastError());
    ++n;
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.wo), 0, d, HD, s.xhi, s.xlo, ldx, nullptr, nullptr, 1, M,
                  s.h, d, 1, st));
    // MoE block: router on the normed row, top-k, expert lists
    wide_norm_split<<<M, 256, 0, st>>>(s.h, static_cast<const __nv_bfloat16 *>(lw.ffn_norm), d, s.eps, s.xhi, s.xlo,
                                       ldx);
    WIDE_TRY(cudaGetLastError());
    ++n;
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.router), 0, E, d, s.xhi, s.xlo, ldx, nullptr, nullptr, 1, M,
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
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.w_gate), static_cast<long long>(F) * d, F, d, s.ghi, s.glo,
                  ldx, s.off, s.count, E, M * K, s.gu, 2 * F, 0, st));
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.w_up), static_cast<long long>(F) * d, F, d, s.ghi, s.glo,
                  ldx, s.off, s.count, E, M * K, s.gu + F, 2 * F, 0, st));
    wide_swiglu<<<M * K, 256, 0, st>>>(s.gu, F, s.ahi, s.alo, s.lda);
    WIDE_TRY(cudaGetLastError());
    ++n;
    WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.w_down), static_cast<long long>(d) * F, d, F, s.ahi, s.alo,
                  s.lda, s.off, s.count, E, M * K, s.yd, d, 0, st));
    // shared expert on every row
    if (Fs > 0) {
      WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.ws_gate), 0, Fs, d, s.xhi, s.xlo, ldx, nullptr, nullptr,
                    1, M, s.gs, 2 * Fs, 0, st));
      WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.ws_up), 0, Fs, d, s.xhi, s.xlo, ldx, nullptr, nullptr, 1,
                    M, s.gs + Fs, 2 * Fs, 0, st));
      wide_swiglu<<<M, 256, 0, st>>>(s.gs, Fs, s.shi, s.slo, s.lda);
      WIDE_TRY(cudaGetLastError());
      ++n;
      WIDE_TRY(gemm(n, s, static_cast<const __nv_bfloat16 *>(lw.ws_down), 0, d, Fs, s.shi, s.slo, s.lda, nullptr, nullptr,
                    1, M, s.ys, d, 0, st));
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
  WIDE_TRY(gemm(n, s, s.lm_head, 0, s.V, d, s.xhi, s.xlo, ldx, nullptr, nullptr, 1, M, s.logits, s.V, 0, st));
  wide_argmax<<<M, 256, 0, st>>>(s.logits, s.V, s.argmax);
  WIDE_TRY(cudaGetLastError());
  if (launches) *launches = n + 1;
  return cudaSuccess;
}

}  // namespace mk
