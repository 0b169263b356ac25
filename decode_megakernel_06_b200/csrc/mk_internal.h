// mk_internal.h -- structures shared by the host planner (mk_api.cu) and the
// persistent decode-step kernel (mk_kernel.cu).  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mk.h"

namespace mk {

// ---- geometry ------------------------------------------------------------------
constexpr int kConsumers = 4;                       // compute warps per CTA
constexpr int kProducers = 4;                       // TMA-issuing warps per CTA
constexpr int kFeeds = kConsumers / kProducers;     // consumers fed by one producer
constexpr int kWarpsPerCta = kConsumers + kProducers;
constexpr int kThreads = kWarpsPerCta * 32;
constexpr int kConsumerThreads = kConsumers * 32;
constexpr int kMaxSlots = 6;                        // ring slots per consumer, at most
// Ring slots per consumer for a kernel of up to `mmax` rows: what shared
// memory leaves beside the staged activation rows (mmax rows of up to 4096
// floats): six at one row, four at two and four rows, two at eight.
__host__ __device__ constexpr int ring_slots(int mmax) { return mmax == 1 ? 6 : mmax <= 4 ? 4 : 2; }
constexpr int kSlotBytes = 8192;                    // one tile: four 2 KB weight boxes
constexpr int kPanel = 256;                         // columns per weight box
constexpr int kRows = 4;                            // rows per weight box, tile and unit
constexpr int kPanels = 4;                          // weight boxes per tile
constexpr int kTileCols = kPanels * kPanel;         // a tile is 4 rows x 1024 columns
constexpr int kBoxBytes = kPanel * kRows * 2;       // 2048
constexpr int kKvBoxBytes = 4096;                   // K or V box: ppt positions x hd
constexpr int kMaxRows = 8;                         // M = B*T cap of this build
constexpr int kMaxExperts = 256;
constexpr int kMaxTopK = 16;
constexpr int kQvp = 4;                             // query vectors per attention item
constexpr int kMaxChunks = 32;                      // CTA KV chunks per (seq, kv head, q group)
constexpr int kCounterStride = 32;                  // uint32s between counters (128 B)
constexpr int kMaxStageSegs = 4;                    // experts a CTA's staged down range may span
// Row stride of an activation row of k columns: whole 256-column panels (the
// rows are stored panel-permuted, see xs_pos4 in mk_kernel.cu).
__host__ __device__ constexpr int panel_ld(int k) { return (k + kPanel - 1) / kPanel * kPanel; }

// Ops of one step: EMBED, then per layer QKV ATTN OPROJ SHARED_GU ROUTED_GU
// DOWN COMBINE, then LMHEAD.  OPROJ also forms the layer's router logits; the
// routing itself is computed by every CTA before its routed gate/up units.
enum OpType : int {
  OP_EMBED = 0, OP_QKV = 1, OP_ATTN = 2, OP_OPROJ = 3, OP_SHARED_GU = 4,
  OP_ROUTED_GU = 5, OP_DOWN = 6, OP_COMBINE = 7, OP_LMHEAD = 8
};
constexpr int kTraceWords = 12;  // per (op, warp) trace record, as MK_TRACE_WORDS
constexpr int kOpsPerLayer = 7;
// Fixed-point scale of the integer accumulators (router logits, expert
// outputs): a value v is held as round(v * 2^32) in an int64, so that sums
// are exact integer additions whose result does not depend on their order.
constexpr int kFixShift = 32;

__host__ __device__ inline int n_ops_for(int L) { return kOpsPerLayer * L + 2; }
__host__ __device__ inline int op_type_of(int op, int L) {
  if (op == 0) return OP_EMBED;
  if (op == kOpsPerLayer * L + 1) return OP_LMHEAD;
  return 1 + (op - 1) % kOpsPerLayer;
}
__host__ __device__ inline int op_layer_of(int op, int L) {
  if (op == 0 || op == kOpsPerLayer * L + 1) return -1;
  return (op - 1) / kOpsPerLayer;
}
__host__ __device__ inline int op_index(int layer, int type) {
  return 1 + kOpsPerLayer * layer + (type - 1);
}
// Ops whose completion `op` waits for (-1 = none).
__host__ __device__ inline void op_deps(int op, int L, int *d0, int *d1) {
  int t = op_type_of(op, L), l = op_layer_of(op, L);
  *d0 = -1;
  *d1 = -1;
  const int last = OP_COMBINE;
  switch (t) {
    case OP_EMBED: break;
    case OP_QKV: *d0 = (l == 0) ? 0 : op_index(l - 1, last); break;
    case OP_ATTN: *d0 = op_index(l, OP_QKV); break;
    case OP_OPROJ: *d0 = op_index(l, OP_ATTN); break;
    case OP_SHARED_GU:
    case OP_ROUTED_GU: *d0 = op_index(l, OP_OPROJ); break;
    case OP_DOWN: *d0 = op_index(l, OP_SHARED_GU); *d1 = op_index(l, OP_ROUTED_GU); break;
    case OP_COMBINE: *d0 = op_index(l, OP_DOWN); break;
    case OP_LMHEAD: *d0 = op_index(L - 1, last); break;
  }
}
__host__ __device__ inline bool op_has_tiles(int type) {
  return type != OP_EMBED && type != OP_COMBINE;
}

// Tensor maps per layer, in this order; the lm_head map follows the last layer.
enum MapSlot : int {
  MAP_WQKV = 0, MAP_WO, MAP_ROUTER, MAP_WGATE, MAP_WUP, MAP_WDOWN,
  MAP_WSGATE, MAP_WSUP, MAP_WSDOWN, MAPS_PER_LAYER
};

struct ArgmaxPart {
  float value;
  int index;
};

struct alignas(64) Params {
  CUtensorMap kmap;   // K cache as 2-D [L*Bmax*Hkv*cap][hd], box [hd][ppt]
  CUtensorMap vmap;
  // dims
  int L, d, Hq, Hkv, hd, E, topk, F, Fs, V, Bmax, cap;
  float eps;
  int B, T, M, max_rows;
  int n_steps;         // steps in this launch; step s writes its argmax to argmax[s * M ..].
                       // Greedy (T = 1, vpos null): step s embeds tokens (s = 0) or
                       // argmax[s-1] and appends at positions[b] + s.
  // Speculative verify over the steps (vpos set): step s scores the block whose
  // start positions are vpos[s][b] and whose tokens are tokens (s = 0) or
  // vtok[s]; its final-argmax warp accepts the longest prefix of drafts its
  // argmax confirms plus one token, and writes the next block from it.
  int *vpos;                             // [n_steps + 1][B]; row 0 set by the host
  int *vtok;                             // [n_steps + 1][M]
  const int *drafts;                     // [B][draft_len]: token proposed for position positions[b] + j
  int draft_len;
  int *out_tokens;                       // [n_steps][M]: accepted tokens, -1 past the count
  int *out_accepted;                     // [n_steps][B]
  // grid / schedule
  int n_cta, n_warps, op_begin, op_end, n_ops;
  int n_hb;            // residual row blocks (ceil(d / kRows))
  int xs_floats;       // shared-memory activation row (batch 1), 0 = none
  int qkv_split;       // QKV units cover 1 or 2 halves of K; the halves are summed by their reader
  int down_groups;     // 4-row groups per down-projection unit (1 or 2)
  int n_db;            // down-projection row blocks (n_hb / down_groups)
  int down_cols;       // 8-row down units of 1-2 activation rows: boxes ordered column
                       // by column, both groups per column (others group by group)
  int down_staged;     // each CTA takes a contiguous range of down units and stages
                       // their experts' activation rows in shared memory
  int e_ld;            // row stride of the router logits (E rounded up to 4)
  int ldx, ldo, ldf, ldfs;  // activation row strides (panel_ld of d, Hq*hd, F, Fs)
  int attn_chunk;      // KV positions per warp; a CTA item covers 8 * attn_chunk
  int attn_qsplit, attn_ppt, attn_nch_max;
  // weights
  const CUtensorMap *tmaps;              // [L][MAPS_PER_LAYER] + lm_head
  const __nv_bfloat16 *const *norms;     // [L][2]: attn_norm, ffn_norm
  const __nv_bfloat16 *embed, *final_norm;
  __nv_bfloat16 *kc, *vc;                // caches (append target)
  // step io
  const int *tokens, *positions;
  float *logits;
  int *argmax;
  // scratch
  float *h;                              // residual entering the layer [8][d]
  float *hm;                             // residual after the o-projection [8][d]
  float *qkv;
  float *o;                              // attention output, panel-permuted rows [8][ldo]
  long long *ssq;                        // [2][8] fixed-point sums of h^2: the residual entering
                                         // the layer, then the residual after the o-projection
  float *xg;                             // h * (the next norm's gain), written with h,
                                         // panel-permuted rows [8][ldx]
  long long *hacc;                       // [8][d] fixed-point sum of the expert outputs
  long long *racc;                       // [L][8][e_ld] fixed-point router logits (before 1/rms)
  float *attn_o, *attn_ml;   // per-CTA-chunk partials (unnormalised o; max, sum)
  uint32_t *attn_cnt;
  float *act_shared, *act_routed;        // silu(gate) * up per row, panel-permuted rows:
                                         // [8][ldfs] and [union][8][ldf]
  ArgmaxPart *am_part;
  const float2 *rope;                    // [cap][hd/2] (cos, sin) of p * theta^(-2i/hd)
  uint32_t *counters, *epoch;
  int *error;                            // [0] code, [1] op
  unsigned long long *stats;             // [0] expert union total
  // debug
  float *dbg_hidden;
  int *dbg_ids;
  float *dbg_w;
  unsigned long long *trace;
  unsigned long long timeout_ns;
  int inject_op;                         // op whose dependency is made unreachable, -1 none
};

// Launch entry points implemented in mk_kernel.cu.  The *_traced forms are the
// same kernels built with the timeline trace compiled in (Params::trace set).
int launch_step(const Params &p, int mmax, bool cooperative, cudaStream_t stream);
int launch_step_traced(const Params &p, int mmax, bool cooperative, cudaStream_t stream);
int max_cta_per_sm_traced(int mmax, size_t smem);
inline int launch_step_any(const Params &p, int mmax, bool cooperative, cudaStream_t stream) {
  return p.trace ? launch_step_traced(p, mmax, cooperative, stream) : launch_step(p, mmax, cooperative, stream);
}
// ---- wide blocks (8 < M <= 64 rows): a sequence of launches ----------------------
constexpr int kWideMaxRows = 64;

struct WideStep {
  // model
  int L, d, Hq, Hkv, hd, E, topk, F, Fs, V, Bmax, cap;
  float eps;
  const mk_layer_weights *layers;  // host array [L]
  const __nv_bfloat16 *embed, *final_norm, *lm_head;
  const float2 *rope;
  // step
  int B, T, max_rows, n_sm;
  const int32_t *tokens, *positions;
  int32_t *tokens_safe, *positions_safe;
  __nv_bfloat16 *kc, *vc;
  float *logits;
  int32_t *argmax;
  int *error;
  unsigned long long *stats;
  float *dbg_hidden;
  int32_t *dbg_ids;
  float *dbg_w;
  // scratch
  int ldx, lda;
  float *h, *qkv, *rlog, *sel_w, *gu, *yd, *gs, *ys, *part;
  float *attn_o, *attn_ml;  // attention partials: [rows * Hq * ceil(cap / 128)] x hd and x 2
  long long part_floats;
  int32_t *sel_e;
  int *count, *off, *pair_row, *pair_slot;
  int *active, *n_active;  // experts with rows, in increasing order, and how many
  __nv_bfloat16 *xhi, *xlo, *ghi, *glo, *ahi, *alo, *shi, *slo;
};

cudaError_t wide_prepare();
// A 128B-swizzled bf16 tensor map, box 64 columns x box_rows rows (mk_api.cu).
int encode_2d_sw128(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows);
cudaError_t wide_step(const WideStep &s, cudaStream_t stream, int *launches);
// After verify block s: acceptance per sequence, and the next block written
// over tok / pos in place (one launch).
cudaError_t wide_accept_step(int B, int T, int s, const int32_t *argmax, int32_t *tok, int32_t *pos,
                             const int32_t *pos0, const int32_t *drafts, int draft_len, int32_t *out_tokens,
                             int32_t *out_accepted, cudaStream_t st);

size_t step_smem_bytes(int n_ops, int xs_floats, int mmax, int e_ld);
bool kernel_stages_x(int mmax);
int max_cta_per_sm(int mmax, size_t smem);

// Temperature / top-p sampler: one cluster of kSampleCluster CTAs per row,
// each holding a slice of ceil(V / kSampleCluster) logits in shared memory.
constexpr int kSampleCluster = 8;
constexpr int kSampleThreads = 512;
constexpr int kSampleMaxVocab = 131072;  // 64-bit mass sums and shared memory both cover this
size_t sample_smem_bytes(int slice);
constexpr int kSamplePhases = 12;  // phase stamps of a traced sampler launch
cudaError_t launch_top_p(const float *logits, int rows, int vocab, float temperature, float top_p,
                         const double *uniforms, int32_t *out, cudaStream_t stream,
                         unsigned long long *stamps = nullptr);

// Read-only HBM probe (mk_probe.cu).  form 0: 16-byte vector loads; form 1:
// bulk asynchronous copies into shared memory.  sink: probe_sink_words(n_sm)
// zeroed words; its last word is set if a bounded wait of form 1 ran out.
size_t probe_sink_words(int n_sm);
cudaError_t launch_read_probe(const void *buf, size_t bytes, int form, int n_sm, uint32_t *sink, cudaStream_t s);

}  // namespace mk
