/*
 * oracle.c -- plain, slow, fp32 CPU reference of one decode step of the
 * layered MoE decoder that the megakernel library fuses.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path: it is the plain definition,
 * written out op by op so that a reader can check it by eye.
 *
 * What it computes (the decode step the megakernel pages describe as one
 * fused program: attention, MoE, normalisation and the residual stream --
 * tpu-megakernels README, FAQ entry on why a custom megakernel is built; the
 * German report, section "Der Trick: 92 Schichten zu einem Programm
 * verschmelzen"; the decoder itself is the synthetic MoE workload
 * specification: RMSNorm, QKV + rotary embedding, bf16 KV-cache append, GQA
 * softmax attention, o-projection, softmax router with renormalised top-k,
 * SwiGLU routed experts plus an optional shared expert, final norm, lm_head
 * and greedy argmax):
 *
 *   per row m (sequence b, block offset t, position p = positions[b] + t):
 *     h = float(embed[token])
 *     per layer:
 *       x = rms(h) * g_attn,  rms(v) = v / sqrt(mean(v^2) + eps)
 *       q, k, v = Wq x, Wk x, Wv x         (Wqkv stacks Wq; Wk; Wv)
 *       rotary embedding at p on every q head and k head (rotate-half pairs
 *       i, i + hd/2, inverse frequency theta^(-2i/hd), angle in fp64, cos and
 *       sin rounded to fp32)
 *       cache[b][g][p] = bf16(k_g), bf16(v_g)    (round to nearest even)
 *       o_h = sum_j softmax_j(q_h . K[g][j] / sqrt(hd)) V[g][j], j = 0..p,
 *             g = h / (Hq / Hkv)
 *       h += Wo concat(o)
 *       y = rms(h) * g_ffn
 *       pi = softmax(Wr y); S = top-k of pi (ties to the lower index);
 *       w_e = pi_e / sum_S pi
 *       h += sum_{e in S} w_e Wd_e (silu(Wg_e y) * (Wu_e y)) + shared(y)
 *     logits = Wlm (rms(h) * g_final);  argmax with ties to the lowest index
 *
 * Everything is fp32 except the weights and the KV cache (bf16 bytes) and the
 * rotary angle (fp64).  Matrices are row-major [out][in]; the KV cache of one
 * layer is [max_seqs][Hkv][kv_capacity][hd].
 *
 * Parity pins (tests, not this file): hand-worked closed-form cases, router
 * invariants, brute-force full-sequence recomputation against the incremental
 * cache, verify block == sequential steps, batch == single rows.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct or_dims {
  int d_model, n_q_heads, n_kv_heads, head_dim;
  int n_experts, top_k, expert_ffn, shared_ffn, vocab;
  int max_seqs, kv_capacity;
  float rms_eps;
  double rope_theta;
} or_dims;

/* ---- bf16 <-> fp32 --------------------------------------------------------- */

static float bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* Round to nearest, ties to even (NaN stays NaN). */
static uint16_t f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

void or_bf16_round(long n, const float *x, uint16_t *out) {
  for (long i = 0; i < n; ++i) out[i] = f32_to_bf16(x[i]);
}

void or_bf16_to_f32(long n, const uint16_t *x, float *out) {
  for (long i = 0; i < n; ++i) out[i] = bf16_to_f32(x[i]);
}

int or_set_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
  return omp_get_max_threads();
#else
  (void)n;
  return 1;
#endif
}

/* ---- single ops -------------------------------------------------------------- */

/* out = h / sqrt(mean(h^2) + eps) * g */
void or_rmsnorm(int d, const float *h, const uint16_t *g, float eps, float *out) {
  float ss = 0.0f;
  for (int i = 0; i < d; ++i) ss += h[i] * h[i];
  float denom = sqrtf(ss / (float)d + eps);
  for (int i = 0; i < d; ++i) out[i] = h[i] / denom * bf16_to_f32(g[i]);
}

/* y = W x, W bf16 [rows][cols] row-major; one sequential fp32 sum per row. */
void or_matvec(int rows, int cols, const uint16_t *W, const float *x, float *y) {
#pragma omp parallel for schedule(static) if ((long)rows * cols > 65536)
  for (int r = 0; r < rows; ++r) {
    const uint16_t *row = W + (size_t)r * cols;
    float acc = 0.0f;
    for (int c = 0; c < cols; ++c) acc += bf16_to_f32(row[c]) * x[c];
    y[r] = acc;
  }
}

/* Rotary embedding of one head vector in place (rotate-half convention). */
void or_rope(int hd, int pos, double theta, float *v) {
  int half = hd / 2;
  for (int i = 0; i < half; ++i) {
    double inv_freq = pow(theta, -2.0 * (double)i / (double)hd);
    double angle = (double)pos * inv_freq;
    float c = (float)cos(angle);
    float s = (float)sin(angle);
    float x1 = v[i], x2 = v[i + half];
    v[i] = x1 * c - x2 * s;
    v[i + half] = x2 * c + x1 * s;
  }
}

/* Softmax attention of one query over n cached positions.
 * K, V: bf16 [n][hd] (consecutive cache rows of one KV head). */
void or_attend(int hd, int n, const float *q, const uint16_t *K, const uint16_t *V,
               float *out) {
  float *s = (float *)malloc(sizeof(float) * (size_t)(n > 0 ? n : 1));
  float scale_div = sqrtf((float)hd);
  float mx = -INFINITY;
  for (int j = 0; j < n; ++j) {
    const uint16_t *kj = K + (size_t)j * hd;
    float dot = 0.0f;
    for (int i = 0; i < hd; ++i) dot += q[i] * bf16_to_f32(kj[i]);
    s[j] = dot / scale_div;
    if (s[j] > mx) mx = s[j];
  }
  float sum = 0.0f;
  for (int j = 0; j < n; ++j) {
    s[j] = expf(s[j] - mx);
    sum += s[j];
  }
  for (int i = 0; i < hd; ++i) out[i] = 0.0f;
  for (int j = 0; j < n; ++j) {
    const uint16_t *vj = V + (size_t)j * hd;
    float a = s[j] / sum;
    for (int i = 0; i < hd; ++i) out[i] += a * bf16_to_f32(vj[i]);
  }
  free(s);
}

/* Router: pi = softmax(z) over E; S = the k largest pi (scan in ascending index
 * order, strictly-greater wins, so ties go to the lower index); weights are
 * pi renormalised over S.  ids/w are written in selection order. */
void or_topk_softmax(int E, int k, const float *z, int *ids, float *w) {
  float mx = -INFINITY;
  for (int e = 0; e < E; ++e)
    if (z[e] > mx) mx = z[e];
  float *pi = (float *)malloc(sizeof(float) * (size_t)E);
  char *taken = (char *)calloc((size_t)E, 1);
  float sum = 0.0f;
  for (int e = 0; e < E; ++e) {
    pi[e] = expf(z[e] - mx);
    sum += pi[e];
  }
  for (int e = 0; e < E; ++e) pi[e] /= sum;
  float sel = 0.0f;
  for (int j = 0; j < k; ++j) {
    int best = -1;
    for (int e = 0; e < E; ++e)
      if (!taken[e] && (best < 0 || pi[e] > pi[best])) best = e;
    taken[best] = 1;
    ids[j] = best;
    w[j] = pi[best];
    sel += pi[best];
  }
  for (int j = 0; j < k; ++j) w[j] /= sel;
  free(pi);
  free(taken);
}

static float silu(float u) { return u / (1.0f + expf(-u)); }

/* One SwiGLU expert: out = Wd (silu(Wg y) * (Wu y)).
 * Wg, Wu: bf16 [F][d]; Wd: bf16 [d][F]. */
void or_swiglu(int F, int d, const uint16_t *Wg, const uint16_t *Wu, const uint16_t *Wd,
               const float *y, float *out) {
  float *g = (float *)malloc(sizeof(float) * (size_t)F);
  float *u = (float *)malloc(sizeof(float) * (size_t)F);
  or_matvec(F, d, Wg, y, g);
  or_matvec(F, d, Wu, y, u);
  for (int f = 0; f < F; ++f) g[f] = silu(g[f]) * u[f];
  or_matvec(d, F, Wd, g, out);
  free(g);
  free(u);
}

/* Index of the largest value; the lowest index wins ties. */
int or_argmax(int n, const float *v) {
  int best = 0;
  for (int i = 1; i < n; ++i)
    if (v[i] > v[best]) best = i;
  return best;
}

/* ---- blocks of the step ------------------------------------------------------- */

/* h[m] = float(embed[tokens[m]]) */
void or_embed(int d, const uint16_t *embed, int M, const int *tokens, float *h) {
  for (int m = 0; m < M; ++m)
    for (int i = 0; i < d; ++i)
      h[(size_t)m * d + i] = bf16_to_f32(embed[(size_t)tokens[m] * d + i]);
}

/* Attention half of one layer for M = B*T rows (row m = b*T + t), in place on
 * h [M][d].  kc / vc: this layer's bf16 cache [max_seqs][Hkv][capacity][hd].
 * The T new keys/values of sequence b go to positions positions[b] .. +T-1
 * before any row attends, and row t attends positions 0 .. positions[b] + t. */
void or_attn_block(const or_dims *D, const uint16_t *attn_norm, const uint16_t *wqkv,
                   const uint16_t *wo, uint16_t *kc, uint16_t *vc, int B, int T,
                   const int *positions, float *h) {
  const int d = D->d_model, Hq = D->n_q_heads, Hkv = D->n_kv_heads, hd = D->head_dim;
  const int M = B * T, qkv_rows = (Hq + 2 * Hkv) * hd, group = Hq / Hkv;
  const int cap = D->kv_capacity;
  float *x = (float *)malloc(sizeof(float) * (size_t)d);
  float *qkv = (float *)malloc(sizeof(float) * (size_t)M * qkv_rows);
  float *o = (float *)malloc(sizeof(float) * (size_t)M * Hq * hd);
  float *y = (float *)malloc(sizeof(float) * (size_t)d);

  for (int m = 0; m < M; ++m) {
    int b = m / T, t = m % T, p = positions[b] + t;
    float *r = qkv + (size_t)m * qkv_rows;
    or_rmsnorm(d, h + (size_t)m * d, attn_norm, D->rms_eps, x);
    or_matvec(qkv_rows, d, wqkv, x, r);
    for (int hh = 0; hh < Hq; ++hh) or_rope(hd, p, D->rope_theta, r + (size_t)hh * hd);
    for (int g = 0; g < Hkv; ++g) {
      float *kg = r + (size_t)(Hq + g) * hd;
      float *vg = r + (size_t)(Hq + Hkv + g) * hd;
      or_rope(hd, p, D->rope_theta, kg);
      size_t slot = (((size_t)b * Hkv + g) * cap + p) * hd;
      for (int i = 0; i < hd; ++i) {
        kc[slot + i] = f32_to_bf16(kg[i]);
        vc[slot + i] = f32_to_bf16(vg[i]);
      }
    }
  }
#pragma omp parallel for schedule(dynamic) collapse(2)
  for (int m = 0; m < M; ++m)
    for (int hh = 0; hh < Hq; ++hh) {
      int b = m / T, t = m % T, p = positions[b] + t, g = hh / group;
      size_t base = ((size_t)b * Hkv + g) * cap * hd;
      or_attend(hd, p + 1, qkv + (size_t)m * qkv_rows + (size_t)hh * hd, kc + base, vc + base,
                o + ((size_t)m * Hq + hh) * hd);
    }
  for (int m = 0; m < M; ++m) {
    or_matvec(d, Hq * hd, wo, o + (size_t)m * Hq * hd, y);
    for (int i = 0; i < d; ++i) h[(size_t)m * d + i] += y[i];
  }
  free(x);
  free(qkv);
  free(o);
  free(y);
}

/* Router half of the MoE block: y[m] = rms(h[m]) * g_ffn, router logits,
 * top-k ids (selection order) and renormalised weights. */
void or_ffn_route(const or_dims *D, const uint16_t *ffn_norm, const uint16_t *router, int M,
                  const float *h, float *y, float *logits, int *ids, float *w) {
  const int d = D->d_model, E = D->n_experts, k = D->top_k;
  for (int m = 0; m < M; ++m) {
    or_rmsnorm(d, h + (size_t)m * d, ffn_norm, D->rms_eps, y + (size_t)m * d);
    or_matvec(E, d, router, y + (size_t)m * d, logits + (size_t)m * E);
    or_topk_softmax(E, k, logits + (size_t)m * E, ids + (size_t)m * k, w + (size_t)m * k);
  }
}

/* Expert half: h[m] += sum_j w[m][j] * expert_j(y[m]) + shared(y[m]).
 * wg/wu/wd hold M*k pointers, entry m*k + j to the matrices of the expert
 * selected in slot j of row m.  ws_* are NULL when there is no shared expert. */
void or_ffn_apply(const or_dims *D, int M, const float *y, const float *w,
                  const uint16_t *const *wg, const uint16_t *const *wu,
                  const uint16_t *const *wd, const uint16_t *ws_gate,
                  const uint16_t *ws_up, const uint16_t *ws_down, float *h) {
  const int d = D->d_model, k = D->top_k, F = D->expert_ffn, Fs = D->shared_ffn;
  float *moe = (float *)malloc(sizeof(float) * (size_t)d);
  float *one = (float *)malloc(sizeof(float) * (size_t)d);
  float *shared = (float *)malloc(sizeof(float) * (size_t)d);
  for (int m = 0; m < M; ++m) {
    const float *ym = y + (size_t)m * d;
    for (int i = 0; i < d; ++i) moe[i] = 0.0f;
    for (int j = 0; j < k; ++j) {
      or_swiglu(F, d, wg[m * k + j], wu[m * k + j], wd[m * k + j], ym, one);
      float wj = w[(size_t)m * k + j];
      for (int i = 0; i < d; ++i) moe[i] += wj * one[i];
    }
    if (Fs > 0 && ws_gate) {
      or_swiglu(Fs, d, ws_gate, ws_up, ws_down, ym, shared);
    } else {
      for (int i = 0; i < d; ++i) shared[i] = 0.0f;
    }
    for (int i = 0; i < d; ++i) h[(size_t)m * d + i] += moe[i] + shared[i];
  }
  free(moe);
  free(one);
  free(shared);
}

/* logits[m] = Wlm (rms(h[m]) * g_final); argmax[m] = lowest index of the max. */
void or_final(const or_dims *D, const uint16_t *final_norm, const uint16_t *lm_head, int M,
              const float *h, float *logits, int *argmax) {
  const int d = D->d_model, V = D->vocab;
  float *x = (float *)malloc(sizeof(float) * (size_t)d);
  for (int m = 0; m < M; ++m) {
    or_rmsnorm(d, h + (size_t)m * d, final_norm, D->rms_eps, x);
    or_matvec(V, d, lm_head, x, logits + (size_t)m * V);
    argmax[m] = or_argmax(V, logits + (size_t)m * V);
  }
  free(x);
}
