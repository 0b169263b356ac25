// mk_api.cu -- host side of libmk.so: descriptor validation, the planner,
// tensor-map encoding, scratch ownership and the launches of the three
// execution variants.  See include/mk.h for the contract of every entry point.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/mk.h"
#include "mk_internal.h"

using namespace mk;

namespace {

thread_local std::string g_err = "ok";

int fail(int code, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

#define CUDA_TRY(expr)                                                                   \
  do {                                                                                   \
    cudaError_t e__ = (expr);                                                            \
    if (e__ != cudaSuccess)                                                              \
      return fail(MK_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(e__));         \
  } while (0)

int ceil_div(int a, int b) { return (a + b - 1) / b; }

// ---- driver entry point for tensor-map encoding --------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D bf16 map over [rows][cols] with row stride ld elements, box 64 columns
// x box_rows rows, 128-byte swizzle (the tensor-core operand layout of the
// wide-block products).  Rows or columns past the matrix read as zeros.
int encode_sw128(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint64_t ld,
                 uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MK_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  if (reinterpret_cast<uintptr_t>(base) % 16 != 0 || (ld * 2) % 16 != 0)
    return fail(MK_ERR_ARG, "tensor base %p or row stride %llu is not 16-byte aligned", base, (unsigned long long)ld);
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MK_ERR_CUDA, "cuTensorMapEncodeTiled(rows=%llu, cols=%llu, 128B swizzle) failed: %d",
                (unsigned long long)rows, (unsigned long long)cols, (int)r);
  return MK_OK;
}

// 2-D bf16 map over a row-major [rows][cols] matrix, box [box_cols][box_rows].
int encode_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint32_t box_cols,
              uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(MK_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  if (reinterpret_cast<uintptr_t>(base) % 16 != 0)
    return fail(MK_ERR_ARG, "tensor base %p is not 16-byte aligned", base);
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return fail(MK_ERR_CUDA, "cuTensorMapEncodeTiled(rows=%llu, cols=%llu) failed: %d",
                (unsigned long long)rows, (unsigned long long)cols, (int)r);
  return MK_OK;
}

// ---- planning ---------------------------------------------------------------------
struct Plan {
  int M, mmax, rows_per_tile, n_hb;
  int attn_qsplit, attn_ppt, attn_chunk, attn_nch_max;
  int n_ops, n_cta, n_warps, xs_floats, qkv_split, down_groups, down_staged, down_cols;
  size_t smem;
};

Plan make_plan(const mk_model_desc &d, int n_sm, int B, int T) {
  Plan p{};
  p.M = B * T;
  p.mmax = p.M <= 1 ? 1 : p.M <= 2 ? 2 : p.M <= 4 ? 4 : 8;
  p.rows_per_tile = kRows;
  p.n_hb = ceil_div(d.d_model, kRows);
  // QKV has few row blocks per warp; halving K per unit can even out the
  // warps' shares.  Split only if it lowers the busiest warp's tiles (each
  // unit costs a fixed overhead besides its tiles).
  {
    const int nt = ceil_div(d.d_model, kTileCols), nrb = ceil_div((d.n_q_heads + 2 * d.n_kv_heads) * d.head_dim, kRows);
    const int nw = n_sm * kConsumers;
    const int full = ceil_div(nrb, nw) * nt, half = ceil_div(2 * nrb, nw) * ceil_div(nt, 2);
    p.qkv_split = (nt >= 2 && half < full) ? 2 : 1;
  }
  // Down projection: two 4-row groups per unit when the F (or Fs) columns leave
  // the 1024-column tiles partly empty, as long as the units still outnumber
  // the warps two to one; the tiles then come out full.
  {
    const int nbx = ceil_div(d.expert_ffn, kPanel), nbs = d.shared_ffn > 0 ? ceil_div(d.shared_ffn, kPanel) : 0;
    const bool partial = (nbx % kPanels) != 0 || (nbs % kPanels) != 0;
    const long long units2 = (long long)(d.d_model / (2 * kRows)) * (d.top_k + (d.shared_ffn > 0 ? 1 : 0));
    p.down_groups = (partial && units2 >= 2LL * n_sm * kConsumers) ? 2 : 1;
  }
  const int G = d.n_q_heads / d.n_kv_heads;
  p.attn_qsplit = ceil_div(G * T, kQvp);
  p.attn_ppt = 2048 / d.head_dim;
  p.n_cta = n_sm;
  p.n_warps = n_sm * kConsumers;
  // Attention items are CTA-wide: each of the compute warps takes attn_chunk KV
  // positions of an item, a multiple of the tile height, with at most
  // kMaxChunks items per (sequence, kv head, query group) so that one merge
  // level combines them.  The chunk minimises the busiest CTA's time, taking
  // every sequence at the cache's capacity: rounds of items over the CTAs x
  // (tiles per warp + kItemCost, the fixed cost of an item -- query staging
  // and the merges -- in tile times).  A chunk just under an even split can
  // leave a second round of items for a few CTAs, which costs more than a
  // somewhat larger chunk.
  {
    constexpr long long kItemCost = 3;
    const long long seqs = (long long)B * d.n_kv_heads * p.attn_qsplit;
    const int c_min = std::max(p.attn_ppt, ceil_div(d.kv_capacity, kMaxChunks * kConsumers));
    int best_c = 0;
    long long best_cost = 0;
    for (int c = ceil_div(c_min, p.attn_ppt) * p.attn_ppt; c <= std::max(c_min, d.kv_capacity) + p.attn_ppt;
         c += p.attn_ppt) {
      const long long items = seqs * ceil_div(d.kv_capacity, c * kConsumers);
      const long long cost = ((items + n_sm - 1) / n_sm) * (c / p.attn_ppt + kItemCost);
      if (best_c == 0 || cost < best_cost) {
        best_c = c;
        best_cost = cost;
      }
    }
    p.attn_chunk = best_c;
  }
  const int c = p.attn_chunk;
  p.attn_nch_max = ceil_div(d.kv_capacity, c * kConsumers);
  p.n_ops = n_ops_for(d.n_layers);
  // shared-memory row: the staged activations (batch 1) or the attention
  // warps' partials and the item's query vectors, whichever is larger
  // (whole 256-column panels: the staged layout permutes columns within one)
  p.xs_floats = std::max((kConsumers + 1) * kQvp * d.head_dim + kMaxRows * d.head_dim,  // + new bf16 K/V rows
                         kernel_stages_x(p.mmax) ? p.mmax * panel_ld(std::max(d.d_model, d.n_q_heads * d.head_dim)) : 0);
  // Staged down projection (one row per step): a CTA's contiguous range of
  // units spans at most 1 + ceil(range / row blocks) experts (largest with the
  // largest union), whose rows must fit the shared-memory rows.  Above one row
  // the shared expert's units (all rows each) cost several routed ones, and
  // contiguous ranges leave the CTAs that hold them far behind (measured at 4
  // and 8 rows: the down projection's last CTA finished 80 and 300 us after
  // the median), so there units go round-robin and read their rows via L1.
  p.down_staged = 0;
  if (p.mmax == 1) {
    const int n_db = p.n_hb / p.down_groups;
    const int segs = std::min(d.n_experts, p.mmax * d.top_k) + (d.shared_ffn > 0 ? 1 : 0);
    const int per_cta = ceil_div(segs * n_db, p.n_cta);
    const int span = std::min(1 + ceil_div(per_cta, n_db), segs);
    const int fmax = std::max(d.expert_ffn, d.shared_ffn);
    p.down_staged = (kernel_stages_x(p.mmax) && span <= kMaxStageSegs &&
                     (long long)span * p.mmax * panel_ld(fmax) <= p.xs_floats) ? 1 : 0;
  }
  // an 8-row down unit of one or two activation rows keeps both groups' sums
  // at once, so its tiles go column by column (each column's activations
  // serve both groups); units of more rows go group by group
  p.down_cols = (p.down_groups == 2) ? 1 : 0;
  p.smem = step_smem_bytes(p.n_ops, p.xs_floats, p.mmax, ceil_div(std::max(d.n_experts, 1), 4) * 4);
  return p;
}

struct Sizes {
  size_t attn_o, attn_ml, attn_cnt;
};

Sizes scratch_sizes(const mk_model_desc &d, int n_sm) {
  Sizes s{};
  // the persistent kernel serves blocks of up to kMaxRows rows
  const int mseqs = std::min(d.max_seqs, kMaxRows), mrows = std::min(d.max_rows, kMaxRows);
  for (int B = 1; B <= mseqs; ++B)
    for (int T = 1; B * T <= mrows; ++T) {
      Plan p = make_plan(d, n_sm, B, T);
      size_t ngrp = (size_t)mseqs * d.n_kv_heads * p.attn_qsplit;
      s.attn_o = std::max(s.attn_o, ngrp * p.attn_nch_max * kQvp * d.head_dim);
      s.attn_ml = std::max(s.attn_ml, ngrp * kQvp * 2 * p.attn_nch_max);
      s.attn_cnt = std::max(s.attn_cnt, ngrp * kQvp);
    }
  return s;
}

}  // namespace

int mk::encode_2d_sw128(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint64_t ld,
                        uint32_t box_rows) {
  return encode_sw128(map, base, rows, cols, ld, box_rows);
}

struct GraphEntry {
  uint64_t key[12];
  cudaGraphExec_t exec;
  int launches;  // kernels per replay
};

struct mk_handle {
  mk_model_desc desc;
  std::vector<mk_layer_weights> layers;
  const void *embed, *final_norm, *lm_head;
  int device, n_sm;
  // device allocations owned by the handle
  std::vector<void *> allocs;
  CUtensorMap *tmaps;
  const __nv_bfloat16 **norms;
  float *h, *hm, *qkv, *o, *attn_o, *attn_ml, *act_shared, *act_routed, *logits;
  long long *hacc, *racc, *ssq;
  size_t hacc_bytes, racc_bytes;
  uint32_t *attn_cnt, *counters, *epoch;
  ArgmaxPart *am_part;
  float2 *rope;
  int *error;
  unsigned long long *stats_dev;
  int32_t *io_tokens, *io_positions, *io_argmax;
  size_t counters_bytes, attn_cnt_bytes;
  // kv maps, re-encoded when the cache pointers change
  void *kv_k, *kv_v;
  CUtensorMap kmap, vmap;
  // state
  int variant;
  unsigned long long timeout_ns;
  float *dbg_hidden;
  int32_t *dbg_ids;
  float *dbg_w;
  unsigned long long *trace;
  int inject;
  int last_error_op;
  mk_stats stats;
  std::vector<GraphEntry> graphs;
  int *vbuf = nullptr;   // verify launches: block positions, block tokens, argmax per step
  size_t vbuf_ints = 0;
  cudaStream_t capture_stream;
  // wide blocks (more than kMaxRows rows): scratch of the launch sequence
  int wide_ldx, wide_lda;
  float *w_h, *w_qkv, *w_rlog, *w_selw, *w_gu, *w_yd, *w_gs, *w_ys, *w_part, *w_attn_o, *w_attn_ml;
  long long w_part_floats;
  int32_t *w_sele, *w_tok, *w_pos;
  int32_t *w_vtok, *w_vpos, *w_vpos0, *w_vam;  // the wide verify loop: block, positions, start, argmax
  int32_t *sp_pos;  // the sampled multi-step loop's positions: [kv_capacity][min(max_seqs, 8)]
  int *w_count, *w_off, *w_pair_row, *w_pair_slot, *w_active;
  __nv_bfloat16 *w_xhi, *w_xlo, *w_ghi, *w_glo, *w_ahi, *w_alo, *w_shi, *w_slo;
};

extern "C" {

MK_API const char *mk_last_error(void) { return g_err.c_str(); }

MK_API int mk_validate_desc(const mk_model_desc *d) {
  if (!d) return fail(MK_ERR_ARG, "desc is NULL");
  if (d->n_layers < 1) return fail(MK_ERR_ARG, "n_layers must be >= 1");
  if (d->d_model < 8 || d->d_model % 8) return fail(MK_ERR_ARG, "d_model must be a positive multiple of 8");
  if (d->n_q_heads < 1 || d->n_kv_heads < 1 || d->n_q_heads % d->n_kv_heads)
    return fail(MK_ERR_ARG, "n_q_heads must be a positive multiple of n_kv_heads");
  if (d->head_dim != 64 && d->head_dim != 128)
    return fail(MK_ERR_UNSUPPORTED, "head_dim %d unsupported (64 or 128)", d->head_dim);
  if (d->n_experts == 0) {
    // a dense decoder: one SwiGLU FFN per layer, given as the shared expert;
    // no router, no routed experts
    if (d->top_k != 0 || d->shared_ffn < 16)
      return fail(MK_ERR_ARG, "a dense model (n_experts = 0) needs top_k = 0 and shared_ffn > 0");
    if (d->max_rows > kMaxRows)
      return fail(MK_ERR_UNSUPPORTED, "a dense model serves at most %d rows per step", kMaxRows);
  } else {
    if (d->n_experts < 1 || d->n_experts > kMaxExperts)
      return fail(MK_ERR_UNSUPPORTED, "n_experts must be in [0, %d]", kMaxExperts);
    if (d->top_k < 1 || d->top_k > d->n_experts || d->top_k > kMaxTopK)
      return fail(MK_ERR_ARG, "top_k must be in [1, min(%d, n_experts)]", kMaxTopK);
  }
  if (d->expert_ffn < 16 || d->expert_ffn % 16) return fail(MK_ERR_ARG, "expert_ffn must be a positive multiple of 16");
  if (d->shared_ffn < 0 || d->shared_ffn % 16) return fail(MK_ERR_ARG, "shared_ffn must be 0 or a multiple of 16");
  if (d->vocab < 1) return fail(MK_ERR_ARG, "vocab must be >= 1");
  if (d->d_model > 6144 || d->n_q_heads * d->head_dim > 6144)
    return fail(MK_ERR_UNSUPPORTED, "d_model and n_q_heads*head_dim must be <= 6144");
  if (d->max_rows < 1 || d->max_rows > kWideMaxRows)
    return fail(MK_ERR_UNSUPPORTED, "max_rows must be in [1, %d]", kWideMaxRows);
  if (d->max_seqs < 1 || d->max_seqs > d->max_rows) return fail(MK_ERR_ARG, "max_seqs must be in [1, max_rows]");
  if (d->kv_capacity < 1) return fail(MK_ERR_ARG, "kv_capacity must be >= 1");
  if (!(d->rope_theta > 0.f) || !(d->rms_eps >= 0.f)) return fail(MK_ERR_ARG, "rope_theta > 0 and rms_eps >= 0 required");
  if (d->variant < MK_MEGAKERNEL || d->variant > MK_TENSORCORE) return fail(MK_ERR_ARG, "unknown variant %d", d->variant);
  const long long kv_rows = (long long)d->n_layers * d->max_seqs * d->n_kv_heads * d->kv_capacity;
  if (kv_rows >= (1ll << 31)) return fail(MK_ERR_UNSUPPORTED, "KV cache too large");
  if ((long long)d->n_experts * d->expert_ffn >= (1ll << 31) || (long long)d->n_experts * d->d_model >= (1ll << 31))
    return fail(MK_ERR_UNSUPPORTED, "expert tensors too large");
  return MK_OK;
}

MK_API int mk_plan_describe(const mk_model_desc *desc, int32_t n_sm, int32_t B, int32_t T,
                            mk_plan_info *info, int32_t *op_types, int32_t *op_layers,
                            int32_t *op_dep0, int32_t *op_dep1, int32_t cap) {
  int rc = mk_validate_desc(desc);
  if (rc) return rc;
  if (n_sm < 1) return fail(MK_ERR_ARG, "n_sm must be >= 1");
  if (B < 1 || T < 1 || B > desc->max_seqs || B * T > desc->max_rows)
    return fail(MK_ERR_CAPACITY, "B=%d T=%d outside max_seqs=%d max_rows=%d", B, T, desc->max_seqs, desc->max_rows);
  if (B * T > kMaxRows)
    return fail(MK_ERR_UNSUPPORTED, "B*T=%d: blocks above %d rows run as a sequence of launches, not a schedule",
                B * T, kMaxRows);
  Plan p = make_plan(*desc, n_sm, B, T);
  if (info) {
    info->n_ops = p.n_ops;
    info->n_cta = p.n_cta;
    info->warps_per_cta = kConsumers;
    info->rows_per_tile = p.rows_per_tile;
    info->mmax = p.mmax;
    info->attn_chunk = p.attn_chunk;
    info->attn_qsplit = p.attn_qsplit;
    info->smem_bytes = (int32_t)p.smem;
    Sizes s = scratch_sizes(*desc, n_sm);
    const mk_model_desc &d = *desc;
    size_t f = (size_t)d.max_rows * d.d_model * 2 + (size_t)d.max_rows * ceil_div(d.d_model, kRows) +
               (size_t)kMaxRows * d.d_model * 3 +  // h_mid, and the int64 expert-output sums
               2 * (size_t)d.max_rows * (d.n_q_heads + 2 * d.n_kv_heads) * d.head_dim +
               (size_t)d.max_rows * d.d_model + (size_t)d.max_rows * d.n_q_heads * d.head_dim + s.attn_o + s.attn_ml +
               (size_t)d.n_layers * kMaxRows * (ceil_div(std::max(d.n_experts, 1), 4) * 4) * 2 +  // int64 router sums
               (size_t)kMaxRows * d.shared_ffn +
               (size_t)std::min(d.n_experts, d.max_rows * d.top_k) * kMaxRows * d.expert_ffn +
               (size_t)d.max_rows * d.vocab + (size_t)d.kv_capacity * d.head_dim;
    info->scratch_bytes = (int64_t)(f * 4 + s.attn_cnt * 4 +
                                    (size_t)p.n_warps * kMaxRows * sizeof(ArgmaxPart));
  }
  for (int i = 0; i < p.n_ops && i < cap; ++i) {
    int d0, d1;
    op_deps(i, desc->n_layers, &d0, &d1);
    if (op_types) op_types[i] = op_type_of(i, desc->n_layers);
    if (op_layers) op_layers[i] = op_layer_of(i, desc->n_layers);
    if (op_dep0) op_dep0[i] = d0;
    if (op_dep1) op_dep1[i] = d1;
  }
  return MK_OK;
}

MK_API void mk_destroy(mk_handle *h) {
  if (!h) return;
  for (auto &g : h->graphs) cudaGraphExecDestroy(g.exec);
  if (h->capture_stream) cudaStreamDestroy(h->capture_stream);
  for (void *p : h->allocs) cudaFree(p);
  delete h;
}

static int halloc(mk_handle *h, void **out, size_t bytes) {
  void *p = nullptr;
  if (bytes == 0) bytes = 16;
  cudaError_t e = cudaMalloc(&p, bytes);
  if (e != cudaSuccess) return fail(MK_ERR_CUDA, "cudaMalloc(%zu) failed: %s", bytes, cudaGetErrorString(e));
  h->allocs.push_back(p);
  e = cudaMemset(p, 0, bytes);
  if (e != cudaSuccess) return fail(MK_ERR_CUDA, "cudaMemset failed: %s", cudaGetErrorString(e));
  *out = p;
  return MK_OK;
}

#define HALLOC(ptr, bytes)                                                      \
  do {                                                                          \
    int rc__ = halloc(h, reinterpret_cast<void **>(&(ptr)), (bytes));           \
    if (rc__) {                                                                 \
      std::string keep = g_err;                                                 \
      mk_destroy(h);                                                            \
      g_err = keep;                                                             \
      return rc__;                                                              \
    }                                                                           \
  } while (0)

MK_API int mk_create(const mk_model_desc *desc, const mk_weights *w, mk_handle **out) {
  if (!out) return fail(MK_ERR_ARG, "out is NULL");
  *out = nullptr;
  int rc = mk_validate_desc(desc);
  if (rc) return rc;
  if (!w || !w->embed || !w->final_norm || !w->lm_head || !w->layers)
    return fail(MK_ERR_ARG, "weights: embed, final_norm, lm_head and layers are required");
  const mk_model_desc &d = *desc;
  for (int l = 0; l < d.n_layers; ++l) {
    const mk_layer_weights &lw = w->layers[l];
    if (!lw.attn_norm || !lw.wqkv || !lw.wo || !lw.ffn_norm ||
        (d.n_experts > 0 && (!lw.router || !lw.w_gate || !lw.w_up || !lw.w_down)))
      return fail(MK_ERR_ARG, "layer %d: a required weight pointer is NULL", l);
    if (d.shared_ffn > 0 && (!lw.ws_gate || !lw.ws_up || !lw.ws_down))
      return fail(MK_ERR_ARG, "layer %d: shared expert weights are NULL but shared_ffn > 0", l);
  }
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  int n_sm = 0, coop = 0;
  CUDA_TRY(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev));
  CUDA_TRY(cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev));
  if (!coop) return fail(MK_ERR_LAUNCH, "device does not support cooperative launches");
  for (int mm : {1, 2, 4, 8}) {
    const size_t smem = make_plan(d, n_sm, 1, mm).smem;
    int per = max_cta_per_sm(mm, smem);
    if (per < 1) return fail(MK_ERR_LAUNCH, "kernel (M<=%d) cannot keep one CTA per SM with %zu B smem", mm, smem);
    per = max_cta_per_sm_traced(mm, smem);
    if (per < 1) return fail(MK_ERR_LAUNCH, "traced kernel (M<=%d) cannot keep one CTA per SM with %zu B smem", mm, smem);
  }

  mk_handle *h = new mk_handle();
  h->desc = d;
  h->layers.assign(w->layers, w->layers + d.n_layers);
  h->embed = w->embed;
  h->final_norm = w->final_norm;
  h->lm_head = w->lm_head;
  h->device = dev;
  h->n_sm = n_sm;
  h->variant = d.variant;
  h->timeout_ns = 1000000000ull;
  h->inject = MK_FAULT_NONE;
  h->last_error_op = -1;

  const int L = d.n_layers, D = d.d_model, QKVW = (d.n_q_heads + 2 * d.n_kv_heads) * d.head_dim;
  const int n_ops = n_ops_for(L), NW = n_sm * kConsumers;
  Sizes s = scratch_sizes(d, n_sm);
  const int umax = std::min(d.n_experts, std::min(d.max_rows, kMaxRows) * d.top_k);
  HALLOC(h->tmaps, sizeof(CUtensorMap) * (size_t)(L * MAPS_PER_LAYER + 1));
  HALLOC(h->norms, sizeof(void *) * 2 * L);
  HALLOC(h->h, sizeof(float) * (size_t)kMaxRows * (D + panel_ld(D)));  // h, then h * gain (xg)
  HALLOC(h->hm, sizeof(float) * (size_t)kMaxRows * D);
  h->hacc_bytes = sizeof(long long) * (size_t)kMaxRows * D;
  HALLOC(h->hacc, h->hacc_bytes);
  h->racc_bytes = sizeof(long long) * (size_t)L * kMaxRows * (ceil_div(std::max(d.n_experts, 1), 4) * 4);
  HALLOC(h->racc, h->racc_bytes);
  HALLOC(h->ssq, sizeof(long long) * 2 * kMaxRows);
  HALLOC(h->sp_pos, sizeof(int32_t) * (size_t)d.kv_capacity * std::min(d.max_seqs, kMaxRows));
  HALLOC(h->qkv, sizeof(float) * 2 * (size_t)kMaxRows * QKVW);  // [K half][row][QKVW]
  HALLOC(h->o, sizeof(float) * (size_t)kMaxRows * panel_ld(d.n_q_heads * d.head_dim));
  HALLOC(h->attn_o, sizeof(float) * s.attn_o);
  HALLOC(h->attn_ml, sizeof(float) * s.attn_ml);
  h->attn_cnt_bytes = sizeof(uint32_t) * s.attn_cnt;
  HALLOC(h->attn_cnt, h->attn_cnt_bytes);
  HALLOC(h->act_shared, sizeof(float) * (size_t)kMaxRows * panel_ld(std::max(d.shared_ffn, 1)));
  HALLOC(h->act_routed, sizeof(float) * (size_t)umax * kMaxRows * panel_ld(std::max(d.expert_ffn, 1)));
  HALLOC(h->am_part, sizeof(ArgmaxPart) * (size_t)NW * kMaxRows);
  HALLOC(h->rope, sizeof(float2) * (size_t)d.kv_capacity * (d.head_dim / 2));
  h->counters_bytes = sizeof(uint32_t) * (size_t)n_ops * kCounterStride;
  HALLOC(h->counters, h->counters_bytes);
  HALLOC(h->epoch, sizeof(uint32_t) * kCounterStride);
  HALLOC(h->error, sizeof(int) * kCounterStride);
  HALLOC(h->stats_dev, sizeof(unsigned long long) * 4);
  HALLOC(h->logits, sizeof(float) * (size_t)d.max_rows * d.vocab);
  HALLOC(h->io_tokens, sizeof(int32_t) * (size_t)d.max_rows);
  HALLOC(h->io_positions, sizeof(int32_t) * (size_t)d.max_seqs);
  HALLOC(h->io_argmax, sizeof(int32_t) * (size_t)d.max_rows);
  // speculative-verify launches: per step the block starts, the block tokens
  // and the argmax; n_steps * T <= kv_capacity and B * T <= 8 bound them
  {
    const size_t mr = std::min(d.max_rows, kMaxRows), cap = (size_t)d.kv_capacity;
    h->vbuf_ints = (cap / 2 + 1) * mr + (cap / 2 + 1) * mr + cap * mr;
    HALLOC(h->vbuf, sizeof(int32_t) * h->vbuf_ints);
  }
  // buffers of the wide-block path: blocks above 8 rows, and MK_TENSORCORE
  // blocks of 2 or more rows on a model with routed experts
  if (d.max_rows > kMaxRows || (d.max_rows >= 2 && d.n_experts > 0)) {
    const int MR = d.max_rows, MK = MR * d.top_k, HD = d.n_q_heads * d.head_dim;
    const int ldx = ceil_div(std::max(D, HD), 8) * 8, lda = ceil_div(std::max(d.expert_ffn, std::max(d.shared_ffn, 1)), 8) * 8;
    const int Fs = std::max(d.shared_ffn, 1);
    h->wide_ldx = ldx;
    h->wide_lda = lda;
    HALLOC(h->w_h, sizeof(float) * (size_t)MR * D);
    HALLOC(h->w_qkv, sizeof(float) * (size_t)MR * QKVW);
    {  // attention partials: per query vector (row x head) and 128-position chunk of the cache
      const size_t slots = (size_t)MR * d.n_q_heads * ceil_div(d.kv_capacity, 128);
      HALLOC(h->w_attn_o, sizeof(float) * slots * d.head_dim);
      HALLOC(h->w_attn_ml, sizeof(float) * slots * 2);
    }
    HALLOC(h->w_rlog, sizeof(float) * (size_t)MR * d.n_experts);
    HALLOC(h->w_selw, sizeof(float) * (size_t)MK);
    HALLOC(h->w_sele, sizeof(int32_t) * (size_t)MK);
    HALLOC(h->w_count, sizeof(int) * (size_t)d.n_experts);
    HALLOC(h->w_off, sizeof(int) * (size_t)d.n_experts);
    HALLOC(h->w_active, sizeof(int) * (size_t)(d.n_experts + 1));  // the list, then its length
    HALLOC(h->w_pair_row, sizeof(int) * (size_t)MK);
    HALLOC(h->w_pair_slot, sizeof(int) * (size_t)MK);
    HALLOC(h->w_tok, sizeof(int32_t) * (size_t)MR);
    HALLOC(h->w_pos, sizeof(int32_t) * (size_t)d.max_seqs);
    HALLOC(h->w_vtok, sizeof(int32_t) * (size_t)MR);
    HALLOC(h->w_vpos, sizeof(int32_t) * (size_t)d.max_seqs);
    HALLOC(h->w_vpos0, sizeof(int32_t) * (size_t)d.max_seqs);
    HALLOC(h->w_vam, sizeof(int32_t) * (size_t)MR);
    HALLOC(h->w_xhi, sizeof(__nv_bfloat16) * (size_t)MR * ldx);
    HALLOC(h->w_xlo, sizeof(__nv_bfloat16) * (size_t)MR * ldx);
    HALLOC(h->w_ghi, sizeof(__nv_bfloat16) * (size_t)MK * ldx);
    HALLOC(h->w_glo, sizeof(__nv_bfloat16) * (size_t)MK * ldx);
    HALLOC(h->w_gu, sizeof(float) * (size_t)MK * 2 * d.expert_ffn);
    HALLOC(h->w_ahi, sizeof(__nv_bfloat16) * (size_t)MK * lda);
    HALLOC(h->w_alo, sizeof(__nv_bfloat16) * (size_t)MK * lda);
    HALLOC(h->w_yd, sizeof(float) * (size_t)MK * D);
    HALLOC(h->w_gs, sizeof(float) * (size_t)MR * 2 * Fs);
    HALLOC(h->w_shi, sizeof(__nv_bfloat16) * (size_t)MR * lda);
    HALLOC(h->w_slo, sizeof(__nv_bfloat16) * (size_t)MR * lda);
    HALLOC(h->w_ys, sizeof(float) * (size_t)MR * D);
    // split-K partials of the dense products: at most 16 K shares of MR rows
    const int ld_max = std::max(std::max(QKVW, D), std::max(2 * Fs, std::max(d.n_experts, HD)));
    h->w_part_floats = 16LL * MR * ld_max;
    HALLOC(h->w_part, sizeof(float) * (size_t)h->w_part_floats);
    cudaError_t pe = wide_prepare();
    if (pe != cudaSuccess) {
      mk_destroy(h);
      return fail(MK_ERR_CUDA, "wide-block setup failed: %s", cudaGetErrorString(pe));
    }
  }

  // tensor maps of every weight matrix
  std::vector<CUtensorMap> maps((size_t)L * MAPS_PER_LAYER + 1);
  std::memset(maps.data(), 0, maps.size() * sizeof(CUtensorMap));
  auto enc = [&](int idx, const void *p, uint64_t rows, uint64_t cols) -> int {
    return encode_2d(&maps[idx], p, rows, cols, kPanel, kRows);
  };
  std::vector<const void *> norm_ptrs(2 * L);
  for (int l = 0; l < L && rc == MK_OK; ++l) {
    const mk_layer_weights &lw = w->layers[l];
    const int b = l * MAPS_PER_LAYER;
    const uint64_t E = d.n_experts, F = d.expert_ffn, Fs = d.shared_ffn;
    rc = enc(b + MAP_WQKV, lw.wqkv, QKVW, D);
    if (!rc) rc = enc(b + MAP_WO, lw.wo, D, (uint64_t)d.n_q_heads * d.head_dim);
    if (E > 0) {  // a dense model has no router and no routed experts
      // the router is read 8 columns x all E rows at a time, next to the
      // o-projection rows it multiplies
      if (!rc) rc = encode_2d(&maps[b + MAP_ROUTER], lw.router, E, D, 8, (uint32_t)E);
      if (!rc) rc = enc(b + MAP_WGATE, lw.w_gate, E * F, D);
      if (!rc) rc = enc(b + MAP_WUP, lw.w_up, E * F, D);
      if (!rc) rc = enc(b + MAP_WDOWN, lw.w_down, E * D, F);
    }
    if (!rc && Fs > 0) rc = enc(b + MAP_WSGATE, lw.ws_gate, Fs, D);
    if (!rc && Fs > 0) rc = enc(b + MAP_WSUP, lw.ws_up, Fs, D);
    if (!rc && Fs > 0) rc = enc(b + MAP_WSDOWN, lw.ws_down, D, Fs);
    norm_ptrs[2 * l] = lw.attn_norm;
    norm_ptrs[2 * l + 1] = lw.ffn_norm;
  }
  if (!rc) rc = enc(L * MAPS_PER_LAYER, w->lm_head, d.vocab, D);
  if (rc) {
    std::string keep = g_err;
    mk_destroy(h);
    g_err = keep;
    return rc;
  }
  // rotary table: cos/sin of p * theta^(-2i/hd), angle in double, rounded to float
  std::vector<float2> rope((size_t)d.kv_capacity * (d.head_dim / 2));
  for (int p = 0; p < d.kv_capacity; ++p)
    for (int i = 0; i < d.head_dim / 2; ++i) {
      double inv_freq = std::pow((double)d.rope_theta, -2.0 * i / (double)d.head_dim);
      double a = (double)p * inv_freq;
      rope[(size_t)p * (d.head_dim / 2) + i] = make_float2((float)std::cos(a), (float)std::sin(a));
    }
  cudaError_t e = cudaMemcpy(h->tmaps, maps.data(), maps.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(h->norms, norm_ptrs.data(), norm_ptrs.size() * sizeof(void *), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaMemcpy(h->rope, rope.data(), rope.size() * sizeof(float2), cudaMemcpyHostToDevice);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&h->capture_stream, cudaStreamNonBlocking);
  if (e != cudaSuccess) {
    mk_destroy(h);
    return fail(MK_ERR_CUDA, "mk_create upload failed: %s", cudaGetErrorString(e));
  }
  *out = h;
  g_err = "ok";
  return MK_OK;
}

static int reset_sync_state(mk_handle *h, cudaStream_t s) {
  CUDA_TRY(cudaMemsetAsync(h->counters, 0, h->counters_bytes, s));
  CUDA_TRY(cudaMemsetAsync(h->epoch, 0, sizeof(uint32_t) * kCounterStride, s));
  CUDA_TRY(cudaMemsetAsync(h->attn_cnt, 0, h->attn_cnt_bytes, s));
  CUDA_TRY(cudaMemsetAsync(h->error, 0, sizeof(int) * kCounterStride, s));
  // a failed step may leave partial fixed-point sums behind
  CUDA_TRY(cudaMemsetAsync(h->hacc, 0, h->hacc_bytes, s));
  CUDA_TRY(cudaMemsetAsync(h->racc, 0, h->racc_bytes, s));
  CUDA_TRY(cudaMemsetAsync(h->ssq, 0, sizeof(long long) * 2 * kMaxRows, s));
  CUDA_TRY(cudaStreamSynchronize(s));
  return MK_OK;
}

static int fill_params(mk_handle *h, const int32_t *tokens, const int32_t *positions, int B, int T,
                       mk_kv_cache kv, float *logits, int32_t *argmax, Params &p, Plan &pl) {
  const mk_model_desc &d = h->desc;
  if (!tokens || !positions || !argmax) return fail(MK_ERR_ARG, "tokens, positions and out_argmax are required");
  if (!kv.k || !kv.v) return fail(MK_ERR_ARG, "kv.k and kv.v are required");
  if (B < 1 || T < 1) return fail(MK_ERR_ARG, "B and T must be >= 1");
  if (B > d.max_seqs || (long long)B * T > d.max_rows)
    return fail(MK_ERR_CAPACITY, "B=%d T=%d exceeds max_seqs=%d / max_rows=%d", B, T, d.max_seqs, d.max_rows);
  if (T > d.kv_capacity) return fail(MK_ERR_CAPACITY, "T=%d exceeds kv_capacity=%d", T, d.kv_capacity);
  if (reinterpret_cast<uintptr_t>(kv.k) % 16 || reinterpret_cast<uintptr_t>(kv.v) % 16)
    return fail(MK_ERR_ARG, "KV cache pointers must be 16-byte aligned");
  pl = make_plan(d, h->n_sm, B, T);
  if (kv.k != h->kv_k || kv.v != h->kv_v) {
    const uint64_t rows = (uint64_t)d.n_layers * d.max_seqs * d.n_kv_heads * d.kv_capacity;
    int rc = encode_2d(&h->kmap, kv.k, rows, d.head_dim, d.head_dim, pl.attn_ppt);
    if (!rc) rc = encode_2d(&h->vmap, kv.v, rows, d.head_dim, d.head_dim, pl.attn_ppt);
    if (rc) {
      h->kv_k = h->kv_v = nullptr;
      return rc;
    }
    h->kv_k = kv.k;
    h->kv_v = kv.v;
  }
  std::memset(&p, 0, sizeof p);
  p.kmap = h->kmap;
  p.vmap = h->vmap;
  p.L = d.n_layers; p.d = d.d_model; p.Hq = d.n_q_heads; p.Hkv = d.n_kv_heads; p.hd = d.head_dim;
  p.E = d.n_experts; p.topk = d.top_k; p.F = d.expert_ffn; p.Fs = d.shared_ffn; p.V = d.vocab;
  p.Bmax = d.max_seqs; p.cap = d.kv_capacity; p.eps = d.rms_eps;
  p.B = B; p.T = T; p.M = B * T; p.max_rows = d.max_rows;
  p.n_steps = 1;
  p.n_cta = pl.n_cta; p.n_warps = pl.n_warps; p.op_begin = 0; p.op_end = pl.n_ops; p.n_ops = pl.n_ops;
  p.n_hb = pl.n_hb;
  p.xs_floats = pl.xs_floats;
  p.qkv_split = pl.qkv_split;
  p.down_groups = pl.down_groups;
  p.n_db = pl.n_hb / pl.down_groups;
  p.down_staged = pl.down_staged;
  p.down_cols = pl.down_cols;
  p.e_ld = ceil_div(std::max(d.n_experts, 1), 4) * 4;
  p.ldx = panel_ld(d.d_model); p.ldo = panel_ld(d.n_q_heads * d.head_dim);
  p.ldf = panel_ld(std::max(d.expert_ffn, 1)); p.ldfs = panel_ld(std::max(d.shared_ffn, 1));
  p.attn_chunk = pl.attn_chunk; p.attn_qsplit = pl.attn_qsplit;
  p.attn_ppt = pl.attn_ppt; p.attn_nch_max = pl.attn_nch_max;
  p.tmaps = h->tmaps; p.norms = h->norms;
  p.embed = static_cast<const __nv_bfloat16 *>(h->embed);
  p.final_norm = static_cast<const __nv_bfloat16 *>(h->final_norm);
  p.kc = static_cast<__nv_bfloat16 *>(kv.k); p.vc = static_cast<__nv_bfloat16 *>(kv.v);
  p.tokens = tokens; p.positions = positions; p.logits = logits ? logits : h->logits; p.argmax = argmax;
  p.h = h->h; p.hm = h->hm; p.ssq = h->ssq; p.qkv = h->qkv; p.o = h->o;
  p.hacc = h->hacc; p.racc = h->racc;
  p.xg = h->h + (size_t)kMaxRows * d.d_model;
  p.attn_o = h->attn_o; p.attn_ml = h->attn_ml;
  p.attn_cnt = h->attn_cnt;
  p.act_shared = h->act_shared; p.act_routed = h->act_routed;
  p.am_part = h->am_part; p.rope = h->rope;
  p.counters = h->counters;
  p.epoch = h->epoch; p.error = h->error;
  p.stats = h->stats_dev;
  p.dbg_hidden = h->dbg_hidden; p.dbg_ids = h->dbg_ids; p.dbg_w = h->dbg_w;
  p.trace = h->trace;
  p.timeout_ns = h->timeout_ns;
  p.inject_op = -1;
  return MK_OK;
}

static int launch_variant(mk_handle *h, Params &p, const Plan &pl, cudaStream_t stream, int variant) {
  if (variant == MK_MEGAKERNEL) {
    int e = launch_step_any(p, pl.mmax, true, stream);
    if (e) return fail(MK_ERR_LAUNCH, "cooperative launch failed: %s", cudaGetErrorString((cudaError_t)e));
    h->stats.kernel_launches += 1;
    return MK_OK;
  }
  for (int op = 0; op < pl.n_ops; ++op) {
    p.op_begin = op;
    p.op_end = op + 1;
    int e = launch_step_any(p, pl.mmax, false, stream);
    if (e) return fail(MK_ERR_LAUNCH, "launch of op %d failed: %s", op, cudaGetErrorString((cudaError_t)e));
  }
  p.op_begin = 0;
  p.op_end = pl.n_ops;
  h->stats.kernel_launches += pl.n_ops;
  return MK_OK;
}

// A block of more than kMaxRows rows: the launch sequence of mk_wide.cu.
// The wide-block step's arguments: the handle's buffers and the call's.
static void fill_wide(mk_handle *h, const int32_t *tokens, const int32_t *positions, int B, int T, mk_kv_cache kv,
                      float *logits, int32_t *argmax, WideStep &s) {
  const mk_model_desc &d = h->desc;
  s = WideStep{};
  s.L = d.n_layers; s.d = d.d_model; s.Hq = d.n_q_heads; s.Hkv = d.n_kv_heads; s.hd = d.head_dim;
  s.E = d.n_experts; s.topk = d.top_k; s.F = d.expert_ffn; s.Fs = d.shared_ffn; s.V = d.vocab;
  s.Bmax = d.max_seqs; s.cap = d.kv_capacity; s.eps = d.rms_eps;
  s.layers = h->layers.data();
  s.embed = static_cast<const __nv_bfloat16 *>(h->embed);
  s.final_norm = static_cast<const __nv_bfloat16 *>(h->final_norm);
  s.lm_head = static_cast<const __nv_bfloat16 *>(h->lm_head);
  s.rope = h->rope;
  s.B = B; s.T = T; s.max_rows = d.max_rows; s.n_sm = h->n_sm;
  s.tokens = tokens; s.positions = positions;
  s.tokens_safe = h->w_tok; s.positions_safe = h->w_pos;
  s.kc = static_cast<__nv_bfloat16 *>(kv.k); s.vc = static_cast<__nv_bfloat16 *>(kv.v);
  s.logits = logits ? logits : h->logits;
  s.argmax = argmax;
  s.error = h->error;
  s.stats = h->stats_dev;
  s.dbg_hidden = h->dbg_hidden; s.dbg_ids = h->dbg_ids; s.dbg_w = h->dbg_w;
  s.ldx = h->wide_ldx; s.lda = h->wide_lda;
  s.attn_o = h->w_attn_o; s.attn_ml = h->w_attn_ml;
  s.h = h->w_h; s.qkv = h->w_qkv; s.rlog = h->w_rlog; s.sel_w = h->w_selw; s.gu = h->w_gu;
  s.yd = h->w_yd; s.gs = h->w_gs; s.ys = h->w_ys; s.part = h->w_part; s.part_floats = h->w_part_floats;
  s.sel_e = h->w_sele; s.count = h->w_count; s.off = h->w_off; s.pair_row = h->w_pair_row;
  s.pair_slot = h->w_pair_slot;
  s.active = h->w_active; s.n_active = h->w_active + d.n_experts;
  s.xhi = h->w_xhi; s.xlo = h->w_xlo; s.ghi = h->w_ghi; s.glo = h->w_glo; s.ahi = h->w_ahi; s.alo = h->w_alo;
  s.shi = h->w_shi; s.slo = h->w_slo;
}

static int run_wide(mk_handle *h, const int32_t *tokens, const int32_t *positions, int B, int T, mk_kv_cache kv,
                    float *logits, int32_t *argmax, cudaStream_t stream) {
  const mk_model_desc &d = h->desc;
  if (!tokens || !positions || !argmax) return fail(MK_ERR_ARG, "tokens, positions and out_argmax are required");
  if (!kv.k || !kv.v) return fail(MK_ERR_ARG, "kv.k and kv.v are required");
  if (B > d.max_seqs || (long long)B * T > d.max_rows)
    return fail(MK_ERR_CAPACITY, "B=%d T=%d exceeds max_seqs=%d / max_rows=%d", B, T, d.max_seqs, d.max_rows);
  if (T > d.kv_capacity) return fail(MK_ERR_CAPACITY, "T=%d exceeds kv_capacity=%d", T, d.kv_capacity);
  WideStep s;
  fill_wide(h, tokens, positions, B, T, kv, logits, argmax, s);
  // The launch sequence is recorded once per (shape, buffers) into a CUDA graph
  // and replayed: a graph launch issues the ~300 kernels without a host call
  // each.  Graphs live in the handle's cache next to the multi-kernel ones.
  const uint64_t key[12] = {(uint64_t)B | (0x57ull << 56),  // wide-block entries
                            (uint64_t)T,
                            (uint64_t)(uintptr_t)tokens,
                            (uint64_t)(uintptr_t)positions,
                            (uint64_t)(uintptr_t)s.logits,
                            (uint64_t)(uintptr_t)argmax,
                            (uint64_t)(uintptr_t)kv.k,
                            (uint64_t)(uintptr_t)kv.v,
                            (uint64_t)(uintptr_t)h->dbg_hidden,
                            (uint64_t)(uintptr_t)h->dbg_ids ^ (uint64_t)(uintptr_t)h->dbg_w,
                            0,
                            0};
  for (auto &g : h->graphs)
    if (std::memcmp(g.key, key, sizeof key) == 0) {
      CUDA_TRY(cudaGraphLaunch(g.exec, stream));
      h->stats.graph_launches += 1;
      h->stats.kernel_launches += g.launches;
      h->stats.steps += 1;
      return MK_OK;
    }
  int launches = 0;
  CUDA_TRY(cudaStreamBeginCapture(h->capture_stream, cudaStreamCaptureModeThreadLocal));
  cudaError_t e = wide_step(s, h->capture_stream, &launches);
  cudaGraph_t graph = nullptr;
  const cudaError_t ce = cudaStreamEndCapture(h->capture_stream, &graph);
  if (e != cudaSuccess) {
    if (graph) cudaGraphDestroy(graph);
    return fail(MK_ERR_LAUNCH, "wide-block launch failed: %s", cudaGetErrorString(e));
  }
  if (ce != cudaSuccess) return fail(MK_ERR_CUDA, "graph capture failed: %s", cudaGetErrorString(ce));
  cudaGraphExec_t exec = nullptr;
  e = cudaGraphInstantiate(&exec, graph, 0);
  cudaGraphDestroy(graph);
  if (e != cudaSuccess) return fail(MK_ERR_CUDA, "graph instantiate failed: %s", cudaGetErrorString(e));
  if (h->graphs.size() >= 8) {
    cudaGraphExecDestroy(h->graphs.front().exec);
    h->graphs.erase(h->graphs.begin());
  }
  GraphEntry ge;
  std::memcpy(ge.key, key, sizeof key);
  ge.exec = exec;
  ge.launches = launches;
  h->graphs.push_back(ge);
  CUDA_TRY(cudaGraphLaunch(exec, stream));
  h->stats.graph_launches += 1;
  h->stats.kernel_launches += launches;
  h->stats.steps += 1;
  return MK_OK;
}

static int run_step(mk_handle *h, const int32_t *tokens, const int32_t *positions, int B, int T,
                    mk_kv_cache kv, float *logits, int32_t *argmax, cudaStream_t stream) {
  if (!h) return fail(MK_ERR_ARG, "handle is NULL");
  if (B >= 1 && T >= 1 &&
      ((long long)B * T > kMaxRows || (h->variant == MK_TENSORCORE && (long long)B * T >= 2 && h->desc.n_experts > 0)))
    return run_wide(h, tokens, positions, B, T, kv, logits, argmax, stream);
  Params p;
  Plan pl;
  int rc = fill_params(h, tokens, positions, B, T, kv, logits, argmax, p, pl);
  if (rc) return rc;
  if (h->inject == MK_FAULT_UNREACHABLE_WAIT) p.inject_op = op_index(0, OP_ATTN);
  int variant = h->variant;
  if (variant == MK_TENSORCORE) variant = MK_MEGAKERNEL;  // 1-row steps and dense models
  if (variant == MK_MULTIKERNEL_GRAPH && p.inject_op < 0) {
    uint64_t key[12] = {(uint64_t)B,
                        (uint64_t)T,
                        (uint64_t)(uintptr_t)tokens,
                        (uint64_t)(uintptr_t)positions,
                        (uint64_t)(uintptr_t)p.logits,
                        (uint64_t)(uintptr_t)argmax,
                        (uint64_t)(uintptr_t)kv.k,
                        (uint64_t)(uintptr_t)kv.v,
                        (uint64_t)(uintptr_t)h->dbg_hidden,
                        (uint64_t)(uintptr_t)h->dbg_ids ^ (uint64_t)(uintptr_t)h->dbg_w,
                        h->timeout_ns,
                        (uint64_t)(uintptr_t)h->trace};
    cudaGraphExec_t exec = nullptr;
    for (auto &g : h->graphs)
      if (std::memcmp(g.key, key, sizeof key) == 0) exec = g.exec;
    if (!exec) {
      CUDA_TRY(cudaStreamBeginCapture(h->capture_stream, cudaStreamCaptureModeThreadLocal));
      int lrc = launch_variant(h, p, pl, h->capture_stream, MK_MULTIKERNEL);
      cudaGraph_t graph = nullptr;
      cudaError_t ce = cudaStreamEndCapture(h->capture_stream, &graph);
      if (lrc) {
        if (graph) cudaGraphDestroy(graph);
        return lrc;
      }
      if (ce != cudaSuccess) return fail(MK_ERR_CUDA, "graph capture failed: %s", cudaGetErrorString(ce));
      ce = cudaGraphInstantiate(&exec, graph, 0);
      cudaGraphDestroy(graph);
      if (ce != cudaSuccess) return fail(MK_ERR_CUDA, "graph instantiate failed: %s", cudaGetErrorString(ce));
      if (h->graphs.size() >= 8) {
        cudaGraphExecDestroy(h->graphs.front().exec);
        h->graphs.erase(h->graphs.begin());
      }
      GraphEntry ge;
      std::memcpy(ge.key, key, sizeof key);
      ge.exec = exec;
      ge.launches = pl.n_ops;
      h->graphs.push_back(ge);
      h->stats.kernel_launches -= pl.n_ops;  // counted again below on replay
    }
    CUDA_TRY(cudaGraphLaunch(exec, stream));
    h->stats.graph_launches += 1;
    h->stats.kernel_launches += pl.n_ops;
  } else {
    if (variant == MK_MULTIKERNEL_GRAPH) variant = MK_MULTIKERNEL;
    rc = launch_variant(h, p, pl, stream, variant);
    if (rc) return rc;
  }
  h->inject = MK_FAULT_NONE;
  h->stats.steps += 1;
  return MK_OK;
}

MK_API int mk_decode_step(mk_handle *h, const int32_t *tokens, const int32_t *positions, int32_t B,
                          int32_t T, mk_kv_cache kv, float *out_logits, int32_t *out_argmax,
                          void *stream) {
  return run_step(h, tokens, positions, B, T, kv, out_logits, out_argmax, static_cast<cudaStream_t>(stream));
}

static int check_sample_args(const void *logits, int32_t rows, int32_t vocab, float temperature,
                             float top_p, const double *uniforms, const int32_t *out) {
  if (!logits || !out) return fail(MK_ERR_ARG, "logits and out_tokens must not be NULL");
  if (rows < 1 || vocab < 1) return fail(MK_ERR_ARG, "rows and vocab must be >= 1 (got %d, %d)", rows, vocab);
  if (vocab > kSampleMaxVocab)
    return fail(MK_ERR_UNSUPPORTED, "the sampler takes vocab <= %d (got %d)", kSampleMaxVocab, vocab);
  if (std::isnan(temperature) || std::isnan(top_p)) return fail(MK_ERR_ARG, "temperature and top_p must not be NaN");
  if (temperature > 0.0f && !uniforms) return fail(MK_ERR_ARG, "sampling with temperature > 0 needs uniforms");
  return MK_OK;
}

MK_API int mk_sample_top_p(const float *logits, int32_t rows, int32_t vocab, float temperature, float top_p,
                           const double *uniforms, int32_t *out_tokens, void *stream) {
  int rc = check_sample_args(logits, rows, vocab, temperature, top_p, uniforms, out_tokens);
  if (rc) return rc;
  CUDA_TRY(launch_top_p(logits, rows, vocab, temperature, top_p, uniforms, out_tokens,
                        static_cast<cudaStream_t>(stream)));
  return MK_OK;
}

MK_API int mk_sample_top_p_phases(const float *logits, int32_t rows, int32_t vocab, float temperature,
                                  float top_p, const double *uniforms, int32_t *out_tokens,
                                  unsigned long long *stamps, void *stream) {
  static_assert(MK_SAMPLE_PHASES == kSamplePhases, "phase count of the header and the kernel");
  if (!stamps) return fail(MK_ERR_ARG, "stamps is NULL");
  int rc = check_sample_args(logits, rows, vocab, temperature, top_p, uniforms, out_tokens);
  if (rc) return rc;
  CUDA_TRY(launch_top_p(logits, rows, vocab, temperature, top_p, uniforms, out_tokens,
                        static_cast<cudaStream_t>(stream), stamps));
  return MK_OK;
}

MK_API int mk_decode_step_sample(mk_handle *h, const int32_t *tokens, const int32_t *positions, int32_t B,
                                 int32_t T, mk_kv_cache kv, float *out_logits, float temperature, float top_p,
                                 const double *uniforms, int32_t *out_tokens, void *stream) {
  if (!h) return fail(MK_ERR_ARG, "handle is NULL");
  int rc = check_sample_args(h, B * T, h->desc.vocab, temperature, top_p, uniforms, out_tokens);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float *logits = out_logits ? out_logits : h->logits;
  // the step writes its argmax to out_tokens; the sampler then overwrites it
  rc = run_step(h, tokens, positions, B, T, kv, logits, out_tokens, s);
  if (rc) return rc;
  CUDA_TRY(launch_top_p(logits, B * T, h->desc.vocab, temperature, top_p, uniforms, out_tokens, s));
  h->stats.kernel_launches += 1;
  return MK_OK;
}

// positions of step s of a sampled loop: out[s][b] = positions[b] + s
__global__ void sp_positions(const int32_t *positions, int B, int n_steps, int32_t *out) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < B * n_steps; i += gridDim.x * blockDim.x)
    out[i] = positions[i % B] + i / B;
}

// The sampled loop's launches on stream s: the positions, then per step the
// megakernel (tokens: the previous step's samples) and the sampler.
static int enqueue_sampled_loop(mk_handle *h, const int32_t *tokens, const int32_t *positions, int B, int n_steps,
                                mk_kv_cache kv, float *logits, float temperature, float top_p,
                                const double *uniforms, int32_t *out_tokens, cudaStream_t s, int *launches) {
  sp_positions<<<std::max(1, std::min(ceil_div(B * n_steps, 256), 64)), 256, 0, s>>>(positions, B, n_steps, h->sp_pos);
  CUDA_TRY(cudaGetLastError());
  int n = 1;
  for (int st = 0; st < n_steps; ++st) {
    Params p;
    Plan pl;
    int rc = fill_params(h, st == 0 ? tokens : out_tokens + (size_t)(st - 1) * B, h->sp_pos + (size_t)st * B, B, 1, kv,
                         logits, out_tokens + (size_t)st * B, p, pl);
    if (rc) return rc;
    int e = launch_step_any(p, pl.mmax, true, s);
    if (e) return fail(MK_ERR_LAUNCH, "cooperative launch failed: %s", cudaGetErrorString((cudaError_t)e));
    CUDA_TRY(launch_top_p(logits, B, h->desc.vocab, temperature, top_p, uniforms ? uniforms + (size_t)st * B : nullptr,
                          out_tokens + (size_t)st * B, s));
    n += 2;
  }
  *launches = n;
  return MK_OK;
}

MK_API int mk_decode_steps_sample(mk_handle *h, const int32_t *tokens, const int32_t *positions, int32_t B,
                                  int32_t n_steps, mk_kv_cache kv, float *out_logits, float temperature,
                                  float top_p, const double *uniforms, int32_t *out_tokens, void *stream) {
  if (!h) return fail(MK_ERR_ARG, "handle is NULL");
  if (n_steps < 1) return fail(MK_ERR_ARG, "n_steps must be >= 1");
  if (B < 1 || B > kMaxRows) return fail(MK_ERR_UNSUPPORTED, "a sampled loop serves 1 to %d sequences", kMaxRows);
  if (B > h->desc.max_seqs) return fail(MK_ERR_CAPACITY, "B=%d exceeds max_seqs=%d", B, h->desc.max_seqs);
  if (n_steps > h->desc.kv_capacity) return fail(MK_ERR_CAPACITY, "n_steps=%d exceeds kv_capacity", n_steps);
  if (!tokens || !positions) return fail(MK_ERR_ARG, "tokens and positions are required");
  int rc = check_sample_args(h, B, h->desc.vocab, temperature, top_p, uniforms, out_tokens);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float *logits = out_logits ? out_logits : h->logits;
  uint32_t tb, pb;
  std::memcpy(&tb, &temperature, 4);
  std::memcpy(&pb, &top_p, 4);
  const uint64_t key[12] = {(uint64_t)B | (0x53ull << 56),  // sampled-loop entries
                            (uint64_t)n_steps,
                            (uint64_t)(uintptr_t)tokens,
                            (uint64_t)(uintptr_t)positions,
                            (uint64_t)(uintptr_t)logits,
                            (uint64_t)(uintptr_t)uniforms,
                            (uint64_t)(uintptr_t)out_tokens,
                            (uint64_t)(uintptr_t)kv.k,
                            (uint64_t)(uintptr_t)kv.v,
                            (uint64_t)tb | ((uint64_t)pb << 32),
                            (uint64_t)(uintptr_t)h->dbg_hidden ^ (uint64_t)(uintptr_t)h->dbg_ids ^
                                (uint64_t)(uintptr_t)h->dbg_w,
                            h->timeout_ns};
  for (auto &g : h->graphs)
    if (std::memcmp(g.key, key, sizeof key) == 0) {
      CUDA_TRY(cudaGraphLaunch(g.exec, s));
      h->stats.graph_launches += 1;
      h->stats.kernel_launches += g.launches;
      h->stats.steps += n_steps;
      return MK_OK;
    }
  int launches = 0;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  bool captured = false;
  if (cudaStreamBeginCapture(h->capture_stream, cudaStreamCaptureModeThreadLocal) == cudaSuccess) {
    rc = enqueue_sampled_loop(h, tokens, positions, B, n_steps, kv, logits, temperature, top_p, uniforms, out_tokens,
                              h->capture_stream, &launches);
    const cudaError_t ce = cudaStreamEndCapture(h->capture_stream, &graph);
    if (rc == MK_OK && ce == cudaSuccess && graph && cudaGraphInstantiate(&exec, graph, 0) == cudaSuccess)
      captured = true;
    if (graph) cudaGraphDestroy(graph);
    if (rc != MK_OK && rc != MK_ERR_LAUNCH && rc != MK_ERR_CUDA) return rc;  // an argument error, not the capture
  }
  if (!captured) {  // enqueue the same launches one by one
    (void)cudaGetLastError();
    rc = enqueue_sampled_loop(h, tokens, positions, B, n_steps, kv, logits, temperature, top_p, uniforms, out_tokens, s,
                              &launches);
    if (rc) return rc;
    h->stats.kernel_launches += launches;
    h->stats.steps += n_steps;
    return MK_OK;
  }
  if (h->graphs.size() >= 8) {
    cudaGraphExecDestroy(h->graphs.front().exec);
    h->graphs.erase(h->graphs.begin());
  }
  GraphEntry ge;
  std::memcpy(ge.key, key, sizeof key);
  ge.exec = exec;
  ge.launches = launches;
  h->graphs.push_back(ge);
  CUDA_TRY(cudaGraphLaunch(exec, s));
  h->stats.graph_launches += 1;
  h->stats.kernel_launches += launches;
  h->stats.steps += n_steps;
  return MK_OK;
}

// mk_verify_steps on the tensor-core launch sequence: the block and its
// positions are copied into the handle, then n_steps x (wide step, then
// acceptance on the device, which writes the next block in place) run as one
// CUDA graph, recorded once per (shape, n_steps, buffers).
static int run_wide_verify(mk_handle *h, const int32_t *tokens, const int32_t *positions, int B, int T,
                           int n_steps, const int32_t *drafts, int draft_len, mk_kv_cache kv, float *out_logits,
                           int32_t *out_tokens, int32_t *out_accepted, cudaStream_t stream) {
  const mk_model_desc &d = h->desc;
  if (!tokens || !positions) return fail(MK_ERR_ARG, "tokens and positions are required");
  if (!kv.k || !kv.v) return fail(MK_ERR_ARG, "kv.k and kv.v are required");
  if (B < 1 || B > d.max_seqs || (long long)B * T > d.max_rows)
    return fail(MK_ERR_CAPACITY, "B=%d T=%d exceeds max_seqs=%d / max_rows=%d", B, T, d.max_seqs, d.max_rows);
  CUDA_TRY(cudaMemcpyAsync(h->w_vtok, tokens, sizeof(int32_t) * B * T, cudaMemcpyDeviceToDevice, stream));
  CUDA_TRY(cudaMemcpyAsync(h->w_vpos, positions, sizeof(int32_t) * B, cudaMemcpyDeviceToDevice, stream));
  CUDA_TRY(cudaMemcpyAsync(h->w_vpos0, positions, sizeof(int32_t) * B, cudaMemcpyDeviceToDevice, stream));
  WideStep s;
  fill_wide(h, h->w_vtok, h->w_vpos, B, T, kv, out_logits, h->w_vam, s);
  const uint64_t key[12] = {(uint64_t)B | (0x56ull << 56),  // wide verify-loop entries
                            (uint64_t)T | ((uint64_t)n_steps << 32),
                            (uint64_t)(uintptr_t)drafts,
                            (uint64_t)(uintptr_t)s.logits,
                            (uint64_t)(uintptr_t)out_tokens,
                            (uint64_t)(uintptr_t)out_accepted,
                            (uint64_t)(uintptr_t)kv.k,
                            (uint64_t)(uintptr_t)kv.v,
                            (uint64_t)(uintptr_t)h->dbg_hidden,
                            (uint64_t)(uintptr_t)h->dbg_ids ^ (uint64_t)(uintptr_t)h->dbg_w,
                            (uint64_t)draft_len,
                            0};
  for (auto &g : h->graphs)
    if (std::memcmp(g.key, key, sizeof key) == 0) {
      CUDA_TRY(cudaGraphLaunch(g.exec, stream));
      h->stats.graph_launches += 1;
      h->stats.kernel_launches += g.launches;
      h->stats.steps += n_steps;
      return MK_OK;
    }
  int launches = 0;
  CUDA_TRY(cudaStreamBeginCapture(h->capture_stream, cudaStreamCaptureModeThreadLocal));
  cudaError_t e = cudaSuccess;
  for (int st = 0; st < n_steps && e == cudaSuccess; ++st) {
    int n = 0;
    e = wide_step(s, h->capture_stream, &n);
    launches += n;
    if (e == cudaSuccess)
      e = wide_accept_step(B, T, st, h->w_vam, h->w_vtok, h->w_vpos, h->w_vpos0, drafts, draft_len, out_tokens,
                           out_accepted, h->capture_stream);
    ++launches;
  }
  cudaGraph_t graph = nullptr;
  const cudaError_t ce = cudaStreamEndCapture(h->capture_stream, &graph);
  if (e != cudaSuccess) {
    if (graph) cudaGraphDestroy(graph);
    return fail(MK_ERR_LAUNCH, "wide verify launch failed: %s", cudaGetErrorString(e));
  }
  if (ce != cudaSuccess) return fail(MK_ERR_CUDA, "graph capture failed: %s", cudaGetErrorString(ce));
  cudaGraphExec_t exec = nullptr;
  e = cudaGraphInstantiate(&exec, graph, 0);
  cudaGraphDestroy(graph);
  if (e != cudaSuccess) return fail(MK_ERR_CUDA, "graph instantiate failed: %s", cudaGetErrorString(e));
  if (h->graphs.size() >= 8) {
    cudaGraphExecDestroy(h->graphs.front().exec);
    h->graphs.erase(h->graphs.begin());
  }
  GraphEntry ge;
  std::memcpy(ge.key, key, sizeof key);
  ge.exec = exec;
  ge.launches = launches;
  h->graphs.push_back(ge);
  CUDA_TRY(cudaGraphLaunch(exec, stream));
  h->stats.graph_launches += 1;
  h->stats.kernel_launches += launches;
  h->stats.steps += n_steps;
  return MK_OK;
}

MK_API int mk_verify_steps(mk_handle *h, const int32_t *tokens, const int32_t *positions, int32_t B,
                           int32_t T, int32_t n_steps, const int32_t *drafts, int32_t draft_len,
                           mk_kv_cache kv, float *out_logits, int32_t *out_tokens, int32_t *out_accepted,
                           void *stream) {
  if (!h) return fail(MK_ERR_ARG, "handle is NULL");
  if (n_steps < 1) return fail(MK_ERR_ARG, "n_steps must be >= 1");
  if (T < 2) return fail(MK_ERR_ARG, "a verify block has T >= 2 rows");
  if (!drafts || !out_tokens || !out_accepted) return fail(MK_ERR_ARG, "drafts, out_tokens and out_accepted are required");
  if ((long long)draft_len < (long long)n_steps * T)
    return fail(MK_ERR_ARG, "draft_len=%d is shorter than n_steps * T = %lld", draft_len, (long long)n_steps * T);
  if ((long long)n_steps * T > h->desc.kv_capacity) return fail(MK_ERR_CAPACITY, "n_steps * T exceeds kv_capacity");
  if (B >= 1 && ((long long)B * T > kMaxRows || (h->variant == MK_TENSORCORE && h->desc.n_experts > 0)))
    return run_wide_verify(h, tokens, positions, B, T, n_steps, drafts, draft_len, kv, out_logits, out_tokens,
                           out_accepted, static_cast<cudaStream_t>(stream));
  const size_t need = (size_t)(n_steps + 1) * B + (size_t)(n_steps + 1) * B * T + (size_t)n_steps * B * T;
  if (need > h->vbuf_ints)  // sized at mk_create for every launch the checks above admit
    return fail(MK_ERR_CAPACITY, "verify buffers: %zu ints needed, %zu held", need, h->vbuf_ints);
  int *vpos = h->vbuf, *vtok = vpos + (size_t)(n_steps + 1) * B, *am = vtok + (size_t)(n_steps + 1) * B * T;
  Params p;
  Plan pl;
  int rc = fill_params(h, tokens, positions, B, T, kv, out_logits, am, p, pl);
  if (rc) return rc;
  p.n_steps = n_steps;
  p.vpos = vpos;
  p.vtok = vtok;
  p.drafts = drafts;
  p.draft_len = draft_len;
  p.out_tokens = out_tokens;
  p.out_accepted = out_accepted;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CUDA_TRY(cudaMemcpyAsync(vpos, positions, sizeof(int32_t) * B, cudaMemcpyDeviceToDevice, s));
  int e = launch_step_any(p, pl.mmax, true, s);
  if (e) return fail(MK_ERR_LAUNCH, "cooperative launch failed: %s", cudaGetErrorString((cudaError_t)e));
  h->stats.kernel_launches += 1;
  h->stats.steps += n_steps;
  return MK_OK;
}

MK_API int mk_decode_steps(mk_handle *h, const int32_t *tokens, const int32_t *positions, int32_t B,
                           int32_t n_steps, mk_kv_cache kv, float *out_logits, int32_t *out_tokens,
                           void *stream) {
  if (!h) return fail(MK_ERR_ARG, "handle is NULL");
  if (n_steps < 1) return fail(MK_ERR_ARG, "n_steps must be >= 1");
  if (B > kMaxRows) return fail(MK_ERR_UNSUPPORTED, "a multi-step launch serves at most %d sequences", kMaxRows);
  if (n_steps > h->desc.kv_capacity) return fail(MK_ERR_CAPACITY, "n_steps=%d exceeds kv_capacity", n_steps);
  Params p;
  Plan pl;
  int rc = fill_params(h, tokens, positions, B, 1, kv, out_logits, out_tokens, p, pl);
  if (rc) return rc;
  p.n_steps = n_steps;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int e = launch_step_any(p, pl.mmax, true, s);
  if (e) return fail(MK_ERR_LAUNCH, "cooperative launch failed: %s", cudaGetErrorString((cudaError_t)e));
  h->stats.kernel_launches += 1;
  h->stats.steps += n_steps;
  return MK_OK;
}

MK_API int mk_get_device_status(mk_handle *h, void *stream) {
  if (!h) return fail(MK_ERR_ARG, "handle is NULL");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CUDA_TRY(cudaStreamSynchronize(s));
  int err[2] = {0, 0};
  CUDA_TRY(cudaMemcpy(err, h->error, sizeof err, cudaMemcpyDeviceToHost));
  if (err[0] == 0) {
    h->last_error_op = -1;
    return MK_OK;
  }
  h->last_error_op = err[1];
  int rc = reset_sync_state(h, s);
  if (rc) return rc;
  if (err[0] == MK_ERR_TIMEOUT) return fail(MK_ERR_TIMEOUT, "device wait timed out in op %d", err[1]);
  if (err[0] == MK_ERR_DEVICE_CHECK)
    return fail(MK_ERR_DEVICE_CHECK, "device rejected an input (token id or position) in op %d", err[1]);
  return fail(err[0], "device error %d in op %d", err[0], err[1]);
}

MK_API int mk_last_device_error_op(mk_handle *h) { return h ? h->last_error_op : -1; }

MK_API int mk_decode_step_host(mk_handle *h, const int32_t *tokens_host, const int32_t *positions_host,
                               int32_t B, int32_t T, mk_kv_cache kv, float *out_logits,
                               int32_t *out_argmax_host, void *stream) {
  if (!h) return fail(MK_ERR_ARG, "handle is NULL");
  if (!tokens_host || !positions_host || !out_argmax_host)
    return fail(MK_ERR_ARG, "tokens_host, positions_host and out_argmax_host are required");
  if (B < 1 || T < 1 || B > h->desc.max_seqs || (long long)B * T > h->desc.max_rows)
    return fail(MK_ERR_CAPACITY, "B=%d T=%d exceeds the handle", B, T);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CUDA_TRY(cudaMemcpyAsync(h->io_tokens, tokens_host, sizeof(int32_t) * B * T, cudaMemcpyHostToDevice, s));
  CUDA_TRY(cudaMemcpyAsync(h->io_positions, positions_host, sizeof(int32_t) * B, cudaMemcpyHostToDevice, s));
  int rc = run_step(h, h->io_tokens, h->io_positions, B, T, kv, out_logits, h->io_argmax, s);
  if (rc) return rc;
  CUDA_TRY(cudaMemcpyAsync(out_argmax_host, h->io_argmax, sizeof(int32_t) * B * T, cudaMemcpyDeviceToHost, s));
  return mk_get_device_status(h, stream);
}

MK_API int mk_set_variant(mk_handle *h, int32_t variant) {
  if (!h) return fail(MK_ERR_ARG, "handle is NULL");
  if (variant < MK_MEGAKERNEL || variant > MK_TENSORCORE) return fail(MK_ERR_ARG, "unknown variant %d", variant);
  h->variant = variant;
  return MK_OK;
}

MK_API int mk_set_timeout(mk_handle *h, uint64_t timeout_ns) {
  if (!h) return fail(MK_ERR_ARG, "handle is NULL");
  if (timeout_ns == 0) return fail(MK_ERR_ARG, "timeout must be > 0");
  h->timeout_ns = timeout_ns;
  return MK_OK;
}

MK_API int mk_set_debug(mk_handle *h, float *hidden, int32_t *expert_ids, float *expert_w) {
  if (!h) return fail(MK_ERR_ARG, "handle is NULL");
  h->dbg_hidden = hidden;
  h->dbg_ids = expert_ids;
  h->dbg_w = expert_w;
  return MK_OK;
}

MK_API int mk_set_trace(mk_handle *h, uint64_t *trace) {
  if (!h) return fail(MK_ERR_ARG, "handle is NULL");
  h->trace = reinterpret_cast<unsigned long long *>(trace);
  return MK_OK;
}

MK_API int mk_debug_inject(mk_handle *h, int32_t fault) {
  if (!h) return fail(MK_ERR_ARG, "handle is NULL");
  if (fault != MK_FAULT_NONE && fault != MK_FAULT_UNREACHABLE_WAIT) return fail(MK_ERR_ARG, "unknown fault %d", fault);
  h->inject = fault;
  return MK_OK;
}

MK_API int mk_hbm_read_probe(const void *buf, uint64_t bytes, int32_t form, int32_t reps, double *out_gbs,
                             void *stream) {
  if (!buf || !out_gbs) return fail(MK_ERR_ARG, "buf and out_gbs are required");
  if (reinterpret_cast<uintptr_t>(buf) % 16) return fail(MK_ERR_ARG, "buf must be 16-byte aligned");
  if (form != 0 && form != 1) return fail(MK_ERR_ARG, "form must be 0 (vector loads) or 1 (bulk copies)");
  if (reps < 1) return fail(MK_ERR_ARG, "reps must be >= 1");
  const uint64_t unit = form == 0 ? 16 : 32768;
  const uint64_t used = bytes / unit * unit;
  if (used < (64ull << 20)) return fail(MK_ERR_ARG, "the probe needs at least 64 MiB (got %llu bytes)",
                                        (unsigned long long)bytes);
  int dev = 0, n_sm = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  CUDA_TRY(cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t words = probe_sink_words(n_sm);
  uint32_t *sink = nullptr;
  CUDA_TRY(cudaMalloc(&sink, words * sizeof(uint32_t)));
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  cudaError_t e = cudaMemsetAsync(sink, 0, words * sizeof(uint32_t), s);
  if (e == cudaSuccess) e = launch_read_probe(buf, used, form, n_sm, sink, s);  // warm-up pass
  if (e == cudaSuccess) e = cudaEventCreate(&e0);
  if (e == cudaSuccess) e = cudaEventCreate(&e1);
  if (e == cudaSuccess) e = cudaEventRecord(e0, s);
  for (int r = 0; r < reps && e == cudaSuccess; ++r) e = launch_read_probe(buf, used, form, n_sm, sink, s);
  if (e == cudaSuccess) e = cudaEventRecord(e1, s);
  if (e == cudaSuccess) e = cudaEventSynchronize(e1);
  float ms = 0.f;
  if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, e0, e1);
  uint32_t flag = 0;
  if (e == cudaSuccess) e = cudaMemcpy(&flag, sink + words - 1, sizeof flag, cudaMemcpyDeviceToHost);
  if (e0) cudaEventDestroy(e0);
  if (e1) cudaEventDestroy(e1);
  cudaFree(sink);
  if (e != cudaSuccess) return fail(MK_ERR_CUDA, "read probe failed: %s", cudaGetErrorString(e));
  if (flag) return fail(MK_ERR_TIMEOUT, "a bounded wait of the bulk read probe ran out");
  *out_gbs = (double)used * reps / (ms * 1e-3) / 1e9;
  return MK_OK;
}

MK_API int mk_get_stats(mk_handle *h, mk_stats *out, int32_t reset) {
  if (!h || !out) return fail(MK_ERR_ARG, "handle and out are required");
  unsigned long long dev[4] = {0, 0, 0, 0};
  CUDA_TRY(cudaDeviceSynchronize());
  CUDA_TRY(cudaMemcpy(dev, h->stats_dev, sizeof dev, cudaMemcpyDeviceToHost));
  *out = h->stats;
  out->expert_union_total = dev[0];
  if (reset) {
    h->stats = mk_stats{};
    CUDA_TRY(cudaMemset(h->stats_dev, 0, sizeof dev));
  }
  return MK_OK;
}

}  // extern "C"

// ---- step without allocation ----------------------------------------------------
// Per-step working memory of mk_decode_step_static.  The array belongs to this
// module, so it exists on a device as soon as the module is loaded there and no
// call has to allocate it.  Every call on a device uses the same array.
static __device__ __align__(256) unsigned char g_static_scratch[MK_STATIC_SCRATCH_BYTES];

namespace {

// Address of the array on the current device.  Resolved on every call (a
// host-side query that allocates nothing), so that a device reset, which
// reloads the module, can never leave a stale address behind.  The first
// call on a device may load the module there.
int static_scratch_base(int dev, unsigned char **out) {
  void *p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
  if (e != cudaSuccess || !p)
    return fail(MK_ERR_CUDA, "cudaGetSymbolAddress(static scratch) on device %d failed: %s", dev,
                cudaGetErrorString(e));
  *out = static_cast<unsigned char *>(p);
  return MK_OK;
}

// Bump layout of the per-step buffers inside the array (256-byte aligned).
struct StaticCarve {
  size_t used = 0;
  template <typename T>
  void take(T *&ptr, unsigned char *base, size_t bytes) {
    ptr = reinterpret_cast<T *>(base + used);
    used += (bytes + 255) / 256 * 256;
  }
};

}  // namespace

extern "C" {

MK_API int mk_decode_step_static(mk_handle *h, const int32_t *tokens, const int32_t *positions,
                                 int32_t B, int32_t T, mk_kv_cache kv, float *out_logits,
                                 int32_t *out_argmax, void *stream) {
  if (!h) return fail(MK_ERR_ARG, "handle is NULL");
  if (B >= 1 && T >= 1 && (long long)B * T > kMaxRows)
    return fail(MK_ERR_UNSUPPORTED, "B*T=%d: blocks above %d rows take mk_decode_step", B * T, kMaxRows);
  int dev = -1;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev != h->device) return fail(MK_ERR_ARG, "device %d is current, the handle lives on device %d", dev, h->device);
  Params p;
  Plan pl;
  int rc = fill_params(h, tokens, positions, B, T, kv, out_logits, out_argmax, p, pl);
  if (rc) return rc;
  unsigned char *base = nullptr;
  rc = static_scratch_base(dev, &base);
  if (rc) return rc;

  const mk_model_desc &d = h->desc;
  const int L = d.n_layers, D = d.d_model, QKVW = (d.n_q_heads + 2 * d.n_kv_heads) * d.head_dim;
  const size_t ngrp = (size_t)B * d.n_kv_heads * pl.attn_qsplit;
  const int umax = std::min(d.n_experts, std::min(d.max_rows, kMaxRows) * d.top_k);
  StaticCarve c;
  // words that must read zero when the step starts, first, so one memset clears them
  c.take(p.counters, base, sizeof(uint32_t) * (size_t)pl.n_ops * kCounterStride);
  c.take(p.epoch, base, sizeof(uint32_t) * kCounterStride);
  c.take(p.attn_cnt, base, sizeof(uint32_t) * ngrp * kQvp);
  // fixed-point sums: the kernel clears them after use, but the array may hold
  // another handle's (or a failed step's) leftovers
  c.take(p.hacc, base, sizeof(long long) * (size_t)kMaxRows * D);
  c.take(p.racc, base, sizeof(long long) * (size_t)L * kMaxRows * p.e_ld);
  c.take(p.ssq, base, sizeof(long long) * 2 * kMaxRows);
  const size_t zero_bytes = c.used;
  // buffers every step writes before it reads them
  c.take(p.h, base, sizeof(float) * (size_t)kMaxRows * (D + panel_ld(D)));
  p.xg = p.h + (size_t)kMaxRows * D;
  c.take(p.hm, base, sizeof(float) * (size_t)kMaxRows * D);
  c.take(p.qkv, base, sizeof(float) * 2 * (size_t)kMaxRows * QKVW);
  c.take(p.o, base, sizeof(float) * (size_t)kMaxRows * panel_ld(d.n_q_heads * d.head_dim));
  c.take(p.attn_o, base, sizeof(float) * ngrp * pl.attn_nch_max * kQvp * d.head_dim);
  c.take(p.attn_ml, base, sizeof(float) * ngrp * kQvp * 2 * pl.attn_nch_max);
  c.take(p.act_shared, base, sizeof(float) * (size_t)kMaxRows * panel_ld(std::max(d.shared_ffn, 1)));
  c.take(p.act_routed, base, sizeof(float) * (size_t)umax * kMaxRows * panel_ld(std::max(d.expert_ffn, 1)));
  c.take(p.am_part, base, sizeof(ArgmaxPart) * (size_t)pl.n_warps * kMaxRows);
  if (!out_logits) c.take(p.logits, base, sizeof(float) * (size_t)B * T * d.vocab);
  if (c.used > (size_t)MK_STATIC_SCRATCH_BYTES)
    return fail(MK_ERR_CAPACITY, "this step needs %zu bytes of working memory; the static scratch holds %u",
                c.used, (unsigned)MK_STATIC_SCRATCH_BYTES);

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CUDA_TRY(cudaMemsetAsync(base, 0, zero_bytes, s));
  int e = launch_step_any(p, pl.mmax, true, s);
  if (e) return fail(MK_ERR_LAUNCH, "cooperative launch failed: %s", cudaGetErrorString((cudaError_t)e));
  h->stats.kernel_launches += 1;
  h->stats.steps += 1;
  return MK_OK;
}

}  // extern "C"
