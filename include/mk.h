/*
 * mk.h -- C ABI of the fused MoE decode-step library (libmk.so).
 *
 * The library runs one decode step of a layered MoE transformer on one B200
 * as a single persistent kernel: one CTA per SM walks a fixed op schedule,
 * synchronises through global-memory counters instead of kernel boundaries,
 * and streams every weight tile through a TMA ring in shared memory that is
 * filled ahead of the op that consumes it, across op and layer boundaries.
 * This is the method of the TPU megakernel pages: the whole decode step as
 * one program, with each weight load decoupled from its consumer so that the
 * next layer's weights are in flight while the current layer computes
 * (video "700 tok/s on a 2.8 Trillion Model: The 92-Layer TPU Megakernel",
 * key technical takeaways; Chinese report "TPU 巨核", section 差距从哪里来;
 * German report, section "Der Trick").  A one-launch-per-op variant of the
 * same path (optionally replayed from a CUDA graph) is built in for
 * comparison: the pages attribute the gap to the idle time between the many
 * kernels of a stock engine (same sections).
 *
 * The step computed, per row m of sequence b at position p (the decoder the
 * pages fuse: attention, MoE, normalisation and residual -- tpu-megakernels
 * README, FAQ entry on why a custom megakernel is built):
 *   h = embed[token]; per layer: x = rms(h) g_attn; q,k,v = Wqkv x; rotary
 *   embedding (rotate-half, theta) on q and k at p; bf16 k,v appended to the
 *   cache at p; GQA softmax attention over positions 0..p (causal inside a
 *   verify block); h += Wo o; y = rms(h) g_ffn; softmax router, top-k
 *   renormalised; h += sum_k w_e Wd_e(silu(Wg_e y) * Wu_e y) + shared(y);
 *   finally logits = Wlm (rms(h) g_final) and argmax (lowest index on ties).
 * Arithmetic is fp32 on bf16 weights and a bf16 KV cache.
 *
 * Conventions.  All tensors are row-major.  Weight matrices are [out][in]
 * bf16 (y = W x).  Expert tensors put the expert index first.  Pointers marked
 * "device" are CUDA device pointers in the current device's context; the
 * caller owns every buffer it passes and keeps weights alive until
 * mk_destroy.  Functions return MK_OK (0) or a negative MK_ERR_* code and
 * never abort; mk_last_error() returns a thread-local message for the last
 * failure.  Work is asynchronous on the given stream unless stated otherwise.
 */
#ifndef MK_H
#define MK_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MK_API __attribute__((visibility("default")))

/* ---- status codes ---------------------------------------------------------- */
#define MK_OK 0
#define MK_ERR_ARG (-1)          /* invalid argument or descriptor              */
#define MK_ERR_CAPACITY (-2)     /* B, T, B*T or positions exceed the handle    */
#define MK_ERR_CUDA (-3)         /* a CUDA runtime/driver call failed           */
#define MK_ERR_LAUNCH (-4)       /* cooperative launch refused / not co-resident */
#define MK_ERR_TIMEOUT (-5)      /* a bounded device-side wait ran out           */
#define MK_ERR_DEVICE_CHECK (-6) /* the kernel rejected an input (token id,      */
                                 /* position) before touching memory with it    */
#define MK_ERR_UNSUPPORTED (-7)  /* shape outside what this build supports       */

/* ---- execution variants ---------------------------------------------------- */
#define MK_MEGAKERNEL 0         /* one persistent cooperative launch per step    */
#define MK_MULTIKERNEL 1        /* one launch per op, no cross-op prefetch       */
#define MK_MULTIKERNEL_GRAPH 2  /* the per-op launches replayed from a CUDA graph */
#define MK_TENSORCORE 3         /* blocks of 2 or more rows on the tensor-core     */
                                /* launch sequence that blocks above 8 rows always */
                                /* take (MoE models; 1-row steps, dense models and */
                                /* the allocation-free entry stay on the megakernel) */

/* ---- debug fault injection ---------------------------------------------------- */
#define MK_FAULT_NONE 0
#define MK_FAULT_UNREACHABLE_WAIT 1 /* next step: one dependency waits for a count
                                       that is never reached (bounded wait test) */

/* Model description.  Supported: head_dim in {64, 128};
 * n_q_heads % n_kv_heads == 0; d_model, n_q_heads*head_dim multiples of 8;
 * expert_ffn and shared_ffn multiples of 16 (shared_ffn may be 0 = no shared
 * expert); n_experts <= 256; top_k <= min(16, n_experts);
 * 1 <= max_rows <= 64; 1 <= max_seqs <= max_rows.
 * A dense decoder (one SwiGLU FFN per layer, no router) is n_experts = 0 and
 * top_k = 0 with the FFN given as the shared expert (shared_ffn > 0, weights
 * ws_gate/ws_up/ws_down; router and w_gate/w_up/w_down may be NULL and
 * expert_ffn is ignored beyond its check); it serves max_rows <= 8. */
typedef struct mk_model_desc {
  int32_t n_layers, d_model, n_q_heads, n_kv_heads, head_dim;
  int32_t n_experts, top_k, expert_ffn, shared_ffn, vocab;
  float rope_theta; /* rotary base, e.g. 1e4                         */
  float rms_eps;    /* RMSNorm epsilon inside the square root, 1e-6  */
  int32_t max_rows;     /* cap on rows per step M = B*T              */
  int32_t max_seqs;     /* cap on sequences B (KV cache batch extent) */
  int32_t kv_capacity;  /* cache slots per sequence                   */
  int32_t variant;      /* MK_MEGAKERNEL | MK_MULTIKERNEL | MK_MULTIKERNEL_GRAPH */
} mk_model_desc;

/* One layer's weights: device pointers to bf16, caller-owned.
 *   attn_norm, ffn_norm : [d]
 *   wqkv  : [(Hq + 2 Hkv) hd][d]   rows: Wq (Hq heads), then Wk, then Wv
 *   wo    : [d][Hq hd]
 *   router: [E][d]
 *   w_gate, w_up: [E][F][d];  w_down: [E][d][F]
 *   ws_gate, ws_up: [Fs][d];  ws_down: [d][Fs]   (NULL when Fs == 0)
 * Each matrix must start on a 16-byte boundary. */
typedef struct mk_layer_weights {
  const void *attn_norm, *wqkv, *wo, *ffn_norm, *router;
  const void *w_gate, *w_up, *w_down;
  const void *ws_gate, *ws_up, *ws_down;
} mk_layer_weights;

/* embed, lm_head: [V][d]; final_norm: [d]; layers: HOST array of n_layers
 * entries (copied during mk_create). */
typedef struct mk_weights {
  const void *embed, *final_norm, *lm_head;
  const mk_layer_weights *layers;
} mk_weights;

/* KV cache, device bf16, each [n_layers][max_seqs][Hkv][kv_capacity][hd].
 * Keys are stored after the rotary embedding.  Caller-owned; written in place
 * at positions[b] .. positions[b] + T - 1 of every layer. */
typedef struct mk_kv_cache {
  void *k, *v;
} mk_kv_cache;

typedef struct mk_handle mk_handle;

/* Counters kept by a handle (read with mk_get_stats). */
typedef struct mk_stats {
  uint64_t steps;              /* decode steps launched                    */
  uint64_t expert_union_total; /* sum over steps and layers of the number of
                                  distinct routed experts (device-counted)  */
  uint64_t kernel_launches;    /* kernels launched by the library           */
  uint64_t graph_launches;     /* CUDA graphs launched by the library (their
                                  kernels are counted in kernel_launches)   */
} mk_stats;

/* Schedule summary for a shape (host-only planning; see mk_plan_describe). */
typedef struct mk_plan_info {
  int32_t n_ops;           /* ops in one step's schedule                     */
  int32_t n_cta;           /* CTAs of the persistent grid (= SM count)       */
  int32_t warps_per_cta;   /* compute warps per CTA (as many more issue TMA) */
  int32_t rows_per_tile;   /* weight rows per ring tile (4: tiles are 4 x 1024) */
  int32_t mmax;            /* row capacity of the kernel instance (1,2,4,8)  */
  int32_t attn_chunk;      /* KV positions per attention work item          */
  int32_t attn_qsplit;     /* query-vector groups per (sequence, KV head)    */
  int32_t smem_bytes;      /* dynamic shared memory per CTA                  */
  int64_t scratch_bytes;   /* device scratch owned by a handle of this shape */
} mk_plan_info;

/* Ops of one step's schedule: EMBED, then per layer QKV ATTN OPROJ SHARED_GU
 * ROUTED_GU DOWN COMBINE, then LMHEAD. */
#define MK_OP_EMBED 0
#define MK_OP_QKV 1        /* RMSNorm + QKV projection                          */
#define MK_OP_ATTN 2       /* rotary, KV append, split-K attention, LSE merge   */
#define MK_OP_OPROJ 3      /* o-projection + residual; each unit also adds its
                              rows' share of the router logits (fixed point)   */
#define MK_OP_SHARED_GU 4  /* shared expert gate/up rows                        */
#define MK_OP_ROUTED_GU 5  /* routed experts' gate/up rows (union of the batch);
                              each CTA first computes the softmax top-k itself */
#define MK_OP_DOWN 6       /* down projections, added into the residual's
                              fixed-point sum with the routing weights          */
#define MK_OP_COMBINE 7    /* above one row per step: residual + that sum; at one
                              row the next op's staging forms it (no work here) */
#define MK_OP_LMHEAD 8     /* final RMSNorm + lm_head; last warp: argmax        */

/* Create a handle: validates the descriptor, plans the schedule, encodes the
 * weight tensor maps, allocates scratch on the current device.  No kernel
 * runs.  `out` receives the handle (NULL on failure).
 * Passage: one of the two calls of the decode-step specification this library
 * implements, mk_create(model_desc, weight_ptrs); the plan it builds is the
 * pages' whole-model program with decoupled weight loads (video "700 tok/s on
 * a 2.8 Trillion Model", key technical takeaways). */
MK_API int mk_create(const mk_model_desc *desc, const mk_weights *weights, mk_handle **out);

/* One decode step of M = B*T rows (row m = b*T + t).
 * Passage: the specification's mk_decode_step(tokens, positions, kv_cache,
 * out_logits, out_argmax, stream), with the handle, B and T added; the step
 * is the pages' fused decoder (tpu-megakernels README, FAQ on what the
 * megakernel fuses: attention, MoE, normalisation, residual).
 *   tokens     : device int32 [B*T], ids in [0, vocab)
 *   positions  : device int32 [B], cache index of sequence b's first new token;
 *                0 <= positions[b] and positions[b] + T <= kv_capacity
 *   B, T       : 1 <= B <= max_seqs, T >= 1, B*T <= max_rows.  T > 1 scores a
 *                verify block: row t attends positions 0 .. positions[b] + t.
 *   kv         : the cache (see mk_kv_cache); appended in place
 *   out_logits : device fp32 [B*T][vocab], or NULL (kept in handle scratch)
 *   out_argmax : device int32 [B*T] (may alias tokens: read before written)
 *   stream     : cudaStream_t (NULL = legacy default stream)
 * Blocks of up to 8 rows run the variant the handle is set to (with
 * MK_TENSORCORE: the tensor-core launch sequence for 2 rows or more on a MoE
 * model); blocks above 8 rows always run the tensor-core launch sequence.
 * Asynchronous.  Invalid token ids or positions are detected on the device:
 * the step stops and mk_get_device_status reports MK_ERR_DEVICE_CHECK. */
MK_API int mk_decode_step(mk_handle *h, const int32_t *tokens, const int32_t *positions,
                          int32_t B, int32_t T, mk_kv_cache kv, float *out_logits,
                          int32_t *out_argmax, void *stream);

/* n_steps greedy decode steps of B sequences (one new token each, T = 1) in
 * ONE persistent launch, with no host round trip between steps: step s
 * embeds `tokens` (s = 0) or step s-1's argmax, appends K/V at
 * positions[b] + s, and writes its argmax to out_tokens[s*B + b].  The
 * megakernel pages' single program extended over steps; the schedule of each
 * step is that of mk_decode_step (same arithmetic, same results).
 *   tokens     : device int32 [B], ids in [0, vocab)
 *   positions  : device int32 [B]; 0 <= positions[b], positions[b] + n_steps <= kv_capacity
 *   B          : 1 <= B <= min(max_seqs, max_rows, 8)
 *   n_steps    : >= 1
 *   kv         : the cache, appended in place
 *   out_logits : device fp32 [B][vocab]: the LAST step's logits, or NULL
 *   out_tokens : device int32 [n_steps][B] (row 0 may alias tokens)
 *   stream     : cudaStream_t (NULL = legacy default stream)
 * Always runs as the megakernel, whatever variant the handle is set to.
 * Asynchronous; device-side errors (bad ids or positions, timeouts) stop the
 * launch and are read with mk_get_device_status.  Errors: MK_ERR_ARG,
 * MK_ERR_CAPACITY and MK_ERR_UNSUPPORTED (B > 8) from the host checks. */
MK_API int mk_decode_steps(mk_handle *h, const int32_t *tokens, const int32_t *positions,
                           int32_t B, int32_t n_steps, mk_kv_cache kv, float *out_logits,
                           int32_t *out_tokens, void *stream);

/* n_steps speculative-verify steps of B sequences in ONE persistent launch,
 * with greedy acceptance and rollback on the device.  Step s scores, for each
 * sequence, a block of T rows at positions p_s .. p_s + T - 1 (p_0 =
 * positions[b]): row 0 is the last accepted token, rows 1..T-1 the drafts
 * proposed for the next positions.  Its argmax accepts the longest prefix of
 * drafts that each equal the argmax of the row before them, plus one token
 * (a = 1..T tokens: the argmax of rows 0..a-1).  The next block starts at
 * p_{s+1} = p_s + a with the last accepted token; K/V rows written past the
 * accepted ones are overwritten by the next block before anything reads them.
 *   tokens      : device int32 [B*T], the first block (row b*T + t)
 *   positions   : device int32 [B]; positions[b] + n_steps*T <= kv_capacity
 *   B, T        : T >= 2, B*T <= max_rows
 *   drafts      : device int32 [B][draft_len]: drafts[b][j] is the token proposed
 *                 for cache position positions[b] + j; draft_len >= n_steps*T
 *   out_logits  : device fp32 [B*T][vocab] of the LAST step, or NULL
 *   out_tokens  : device int32 [n_steps][B*T]: accepted tokens, -1 after the count
 *   out_accepted: device int32 [n_steps][B]: tokens accepted per step (1..T)
 * Blocks of up to 8 rows run as ONE persistent megakernel launch.  Blocks
 * above 8 rows (and, with MK_TENSORCORE, blocks on a MoE model) run the
 * tensor-core launch sequence: n_steps x (the step, then the acceptance on
 * the device, which writes the next block in place) as one CUDA graph launch.
 * Asynchronous; device-side errors are read with mk_get_device_status.
 * Errors: MK_ERR_ARG and MK_ERR_CAPACITY from the host checks. */
MK_API int mk_verify_steps(mk_handle *h, const int32_t *tokens, const int32_t *positions,
                           int32_t B, int32_t T, int32_t n_steps, const int32_t *drafts,
                           int32_t draft_len, mk_kv_cache kv, float *out_logits,
                           int32_t *out_tokens, int32_t *out_accepted, void *stream);

/* Temperature / top-p (nucleus) sampling of one token per logits row, the
 * sampler that stands in place of the argmax (tpu-megakernels README, serving
 * demos: greedy or temperature / top-p generation; the nucleus is Holtzman et
 * al. 2020, section 3.1).  Per row of V logits l and its uniform u:
 *   p_i = exp((l_i - max l) / T) in fp64, held as the fixed-point mass
 *   q_i = round_half_even(p_i * 2^46) (all sums exact integers);
 *   need = max(1, min(Q, ceil(top_p * Q))), Q = sum q, computed in fp64;
 *   nucleus = the smallest prefix of the tokens sorted by logit, descending,
 *   ties by lower id, whose mass reaches need;
 *   token = the first nucleus id, in id order, whose cumulative mass exceeds
 *   y = min(S - 1, floor(u * S)), S the nucleus mass.
 * temperature <= 0 is greedy (the argmax, lowest id on ties; uniforms unread).
 * top_p <= 0 keeps the most probable token, top_p >= 1 every token.
 *   logits     : device fp32 [rows][vocab], finite (non-finite rows give an
 *                unspecified token or none, never an out-of-bounds access)
 *   rows       : >= 1;  vocab: 1 .. 131072
 *   uniforms   : device fp64 [rows], each in [0, 1) (values outside are clamped);
 *                the random numbers are the caller's, so a draw is reproducible
 *   out_tokens : device int32 [rows]
 *   stream     : cudaStream_t (NULL = legacy default stream)
 * One launch: a cluster of 8 CTAs per row.  Asynchronous.  Errors: MK_ERR_ARG
 * (NULL pointer, rows or vocab < 1, NaN temperature or top_p, uniforms NULL
 * with temperature > 0), MK_ERR_UNSUPPORTED (vocab > 131072), MK_ERR_CUDA. */
MK_API int mk_sample_top_p(const float *logits, int32_t rows, int32_t vocab, float temperature,
                           float top_p, const double *uniforms, int32_t *out_tokens, void *stream);

/* mk_sample_top_p, and the device clock (%globaltimer, ns) at each phase
 * boundary of row 0's first CTA written to stamps[0 .. MK_SAMPLE_PHASES):
 *   0 start, 1 slice loaded and its largest key found, 2 after the cluster
 *   barrier that shares the largest key, 3 masses and first histogram done,
 *   4..7 end of radix pass 0..3 (histogram of the next key byte included),
 *   8 the nucleus and this CTA's segment totals done, 9 after the barrier that
 *   shares them, 10 the draw done, 11 after the closing barrier.
 * stamps: device uint64 [MK_SAMPLE_PHASES], caller-owned; a greedy call
 * (temperature <= 0) writes entries 0..2 only.  A measurement aid: the
 * sample drawn is the same as mk_sample_top_p's.  Errors as mk_sample_top_p,
 * and MK_ERR_ARG for a NULL stamps. */
#define MK_SAMPLE_PHASES 12
MK_API int mk_sample_top_p_phases(const float *logits, int32_t rows, int32_t vocab, float temperature,
                                  float top_p, const double *uniforms, int32_t *out_tokens,
                                  unsigned long long *stamps, void *stream);

/* mk_decode_step followed by mk_sample_top_p on its logits: one decode step of
 * B*T rows whose next tokens are sampled instead of taken greedily.  Arguments
 * as mk_decode_step (out_logits may be NULL: the handle's scratch holds them)
 * and mk_sample_top_p (uniforms [B*T]); out_tokens [B*T] receives the sampled
 * ids (the step's argmax passes through it first).  Errors: those of both. */
MK_API int mk_decode_step_sample(mk_handle *h, const int32_t *tokens, const int32_t *positions,
                                 int32_t B, int32_t T, mk_kv_cache kv, float *out_logits,
                                 float temperature, float top_p, const double *uniforms,
                                 int32_t *out_tokens, void *stream);

/* n_steps sampled decode steps of B sequences (one row each) as ONE CUDA graph
 * launch: step s runs the megakernel at positions[b] + s on the tokens
 * sampled by step s-1 (step 0: tokens), then mk_sample_top_p on its logits
 * with uniforms[s][B] into out_tokens[s][B].  Passage: the pages' serving
 * loop offers greedy or temperature / top-p generation (tpu-megakernels
 * README, serving paragraph); this is the sampled form of mk_decode_steps.
 *   tokens     : device int32 [B], the first step's tokens
 *   positions  : device int32 [B]; positions[b] + n_steps <= kv_capacity
 *   B          : 1 <= B <= min(max_seqs, 8)
 *   out_logits : device fp32 [B][vocab]: the LAST step's logits, or NULL
 *   uniforms   : device fp64 [n_steps][B] in [0, 1) (may be NULL when
 *                temperature <= 0: greedy)
 *   out_tokens : device int32 [n_steps][B]
 * The graph is recorded once per (B, n_steps, buffers, temperature, top_p)
 * and replayed; where a cooperative launch cannot be captured, the same
 * 2 * n_steps launches are enqueued one by one.  Asynchronous; device-side
 * errors are read with mk_get_device_status.  Errors: MK_ERR_ARG,
 * MK_ERR_CAPACITY, MK_ERR_UNSUPPORTED (B > 8, vocab above the sampler's
 * limit) from the host checks. */
MK_API int mk_decode_steps_sample(mk_handle *h, const int32_t *tokens, const int32_t *positions,
                                  int32_t B, int32_t n_steps, mk_kv_cache kv, float *out_logits,
                                  float temperature, float top_p, const double *uniforms,
                                  int32_t *out_tokens, void *stream);

/* The same step driven from HOST buffers: copies tokens [B*T] and positions
 * [B] to the device, runs the step, copies argmax [B*T] back to
 * out_argmax_host, and waits for the stream.  Logits stay on the device
 * (out_logits may be NULL).  Returns the device status of the step. */
MK_API int mk_decode_step_host(mk_handle *h, const int32_t *tokens_host,
                               const int32_t *positions_host, int32_t B, int32_t T,
                               mk_kv_cache kv, float *out_logits, int32_t *out_argmax_host,
                               void *stream);

/* Size of the fixed device array that mk_decode_step_static works in. */
#define MK_STATIC_SCRATCH_BYTES (32u << 20)

/* The decode step of mk_decode_step, run as the megakernel (one persistent
 * launch, whatever variant the handle is set to), without allocating.
 * The megakernel pages have no counterpart for this call; it exists for
 * callers that must not allocate device memory when they step, for example a
 * serving process that hands every free byte of the device to its own
 * KV-cache pool once its models are loaded, where a later cudaMalloc fails.
 *
 * Arguments, their layout and ownership are those of mk_decode_step.  The
 * step's working memory (hidden rows, projections, attention partials,
 * routing, expert activations, the synchronisation counters, and the logits
 * when out_logits is NULL) comes from one array of MK_STATIC_SCRATCH_BYTES in
 * the library's device module instead of from the handle; the tensor maps,
 * norm pointers, rotary table, device status word and statistics stay in the
 * handle.  No call allocates or frees memory.
 *
 * Every call resolves the array's device address (cudaGetSymbolAddress, a
 * host-side query that allocates nothing) with the handle's device current;
 * the first call on a device may load the library's device module there, so
 * make that first call before any stream capture.  Each call clears the
 * counters and fixed-point sums that must start at zero (an asynchronous
 * memset on `stream`), then launches the step.
 *
 * Every handle and stream on a device shares the one array: calls whose work
 * overlaps on the GPU race and corrupt each other's results.  Order them on
 * one stream, or finish one before the next starts.
 *
 * Errors: the host-side checks of mk_decode_step; MK_ERR_CAPACITY when the
 * step (for this B, T and model) needs more than MK_STATIC_SCRATCH_BYTES, with
 * the size it needs in mk_last_error(); MK_ERR_ARG when another device is
 * current.  Device-side errors are read with mk_get_device_status. */
MK_API int mk_decode_step_static(mk_handle *h, const int32_t *tokens, const int32_t *positions,
                                 int32_t B, int32_t T, mk_kv_cache kv, float *out_logits,
                                 int32_t *out_argmax, void *stream);

/* Passage: none in the pages (they define no error interface); this call
 * completes the boundary with the device-side status of bounded waits.
 * Synchronises `stream`, then returns MK_OK or the first device-side error of
 * the steps since the last call (MK_ERR_TIMEOUT, MK_ERR_DEVICE_CHECK).  An
 * error clears the handle's synchronisation state so the next step starts
 * clean; the failed step's outputs and cache writes are undefined. */
MK_API int mk_get_device_status(mk_handle *h, void *stream);

/* Device-side detail of the last error returned by mk_get_device_status:
 * the op index that failed (or -1). */
MK_API int mk_last_device_error_op(mk_handle *h);

/* Thread-local message for the last failing call (never NULL).  Passage: none
 * in the pages; part of the boundary's error reporting. */
MK_API const char *mk_last_error(void);

/* Frees everything the handle owns.  Safe on NULL.  Call after the last step
 * has finished.  Passage: none in the pages; the handle's end of life. */
MK_API void mk_destroy(mk_handle *h);

/* Switch the execution variant (MK_MEGAKERNEL, MK_MULTIKERNEL,
 * MK_MULTIKERNEL_GRAPH, MK_TENSORCORE).  The first three run the same math in
 * the same order; MK_TENSORCORE computes the same step with tensor-core
 * products (activations as a bf16 pair, about 2^-16 relative), so its results
 * agree with the others within the parity tolerance, not bit for bit. */
MK_API int mk_set_variant(mk_handle *h, int32_t variant);

/* Bound for every device-side wait, in nanoseconds (default 1e9). */
MK_API int mk_set_timeout(mk_handle *h, uint64_t timeout_ns);

/* Passage: none in the pages; the per-layer states these buffers receive are
 * what the parity tests compare with the oracle's.
 * Test/debug outputs, written by every following step (NULL disables):
 *   hidden     : device fp32 [n_layers + 1][max_rows][d]: the residual stream
 *                after the embedding and after each layer
 *   expert_ids : device int32 [n_layers][max_rows][top_k], selection order
 *   expert_w   : device fp32  [n_layers][max_rows][top_k], renormalised */
MK_API int mk_set_debug(mk_handle *h, float *hidden, int32_t *expert_ids, float *expert_w);

/* Arm a fault for the next step (MK_FAULT_*).  Passage: none in the pages;
 * it makes one bounded wait run out so that the error path can be tested
 * without faulting the GPU. */
MK_API int mk_debug_inject(mk_handle *h, int32_t fault);

/* Per-op timeline of every following step (NULL disables): device uint64
 * [n_ops][n_cta * warps_per_cta][MK_TRACE_WORDS] per warp slot:
 *   [0] %globaltimer (ns) when the warp began the op's units (inputs ready),
 *   [1] when its first weight/KV tile of the op was ready (0: none),
 *   [2] when it finished consuming its last tile of the op (0: none),
 *   [3] when it arrived at the op's completion counter,
 *   [4] ns it spent blocked on tiles that had not landed yet,
 *   [5] tiles it consumed in the op,
 *   [6], [7] ROUTED_GU: when this warp first found its CTA's routing
 *            ready, and 1 if it computed it; other ops: when the warp's wait
 *            for the op's inputs ended, and when its CTA had staged them
 *            (the staged activation row of a batch-1 step; else = [6]);
 *   [8], [9] the warp's TMA-issuing warp: when it issued its first and its
 *            last tile of the op (0: none),
 *   [10] ns that issuing warp spent, while on this op, waiting for an input
 *        its tile addresses or their release depend on (the routing, an
 *        expert's gate/up units),
 *   [11] ns it spent, while on this op, waiting for a free ring slot.
 * n_ops and the grid come from mk_plan_describe. */
#define MK_TRACE_WORDS 12
MK_API int mk_set_trace(mk_handle *h, uint64_t *trace);

/* Read-only HBM bandwidth probe: the ceiling that the decode step, which only
 * reads its weights and cache, is measured against beside the copy peak.
 * Reads the first bytes of `buf` (rounded down to 16 B for form 0, to 32 KiB
 * for form 1) once per pass and writes nothing but a few words of its own:
 *   form 0: 16-byte vector loads that bypass L1, 8 in flight per thread, a
 *           grid of whole waves of resident blocks;
 *   form 1: bulk asynchronous copies (cp.async.bulk, 32 KiB each, 4 in flight
 *           per SM) into shared memory, the engine of the step's weight ring.
 * One untimed pass, then `reps` passes timed with CUDA events on `stream`;
 * *out_gbs = bytes read / time in GB/s (1e9).  buf: device, 16-byte aligned,
 * at least 64 MiB (use a buffer well above the 126 MB L2); caller-owned and
 * unchanged.  Allocates and frees a small result buffer; synchronises the
 * stream.  Errors: MK_ERR_ARG, MK_ERR_CUDA, MK_ERR_TIMEOUT (a bounded wait of
 * form 1 ran out). */
MK_API int mk_hbm_read_probe(const void *buf, uint64_t bytes, int32_t form, int32_t reps, double *out_gbs,
                             void *stream);

/* Copies the handle's counters; reset != 0 zeroes them afterwards.  Waits for
 * the device (reads a device counter). */
MK_API int mk_get_stats(mk_handle *h, mk_stats *out, int32_t reset);

/* Host-only: validate a descriptor without touching the GPU. */
MK_API int mk_validate_desc(const mk_model_desc *desc);

/* Host-only: plan the step for a shape on a GPU with n_sm SMs and report the
 * schedule.  If op_types/op_layers/op_dep0/op_dep1 are non-NULL they receive
 * up to `cap` entries: each op's MK_OP_* type, layer (-1 = none) and the
 * indices of the ops whose completion it waits for (-1 = none). */
MK_API int mk_plan_describe(const mk_model_desc *desc, int32_t n_sm, int32_t B, int32_t T,
                            mk_plan_info *info, int32_t *op_types, int32_t *op_layers,
                            int32_t *op_dep0, int32_t *op_dep1, int32_t cap);

#ifdef __cplusplus
}
#endif

#endif /* MK_H */
