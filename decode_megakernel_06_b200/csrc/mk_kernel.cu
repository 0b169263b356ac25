// mk_kernel.cu -- the persistent decode-step kernel for sm_100a.
//
// One CTA per SM, 8 warps per CTA.  Every warp is its own producer and
// consumer: it owns a 3-slot ring of 8 KB tiles in shared memory and keeps it
// filled with TMA loads (cp.async.bulk.tensor, completion on an mbarrier) of
// the tiles it will consume next -- across op and layer boundaries, since a
// weight load depends only on knowing which weight comes next, not on the
// activations it will meet.  This is the decoupled-load design of the TPU
// megakernel pages (video "700 tok/s on a 2.8 Trillion Model: The 92-Layer
// TPU Megakernel", key technical takeaways: layer n+1's weights stream in
// while layer n computes; Chinese report "TPU 巨核", section 差距从哪里来:
// a load is issued as early as on-chip memory allows).  Only routed-expert
// tiles wait, for the router's result.
//
// The step is a fixed list of ops (EMBED; per layer QKV, ATTN, OPROJ,
// ROUTER, SHARED_GU, ROUTED_GU, DOWN; LMHEAD).  Each op's work is cut into
// units dealt round-robin to the grid's warps.  A warp finishing its units of
// an op arrives on that op's counter (aggregated per CTA in shared memory,
// then one release-add per CTA); an op that needs an earlier op's output
// spins (bounded by %globaltimer) until that counter reaches
// epoch * n_cta.  Counters only grow, so no reset is needed between steps.
//
// GEMV math: tile = 16 weight rows x 256 columns (8 rows x 512 columns when a
// step has more than 4 rows); each lane owns 8 columns and keeps the matching
// activations of every row in registers, so one 16-byte weight load feeds
// 8*MJ FMAs.  Lane partial sums are combined with a butterfly
// (transpose-reduce) of warp shuffles.  All arithmetic is fp32.
#include <cstdio>

#include "mk_internal.h"

namespace mk {
namespace {

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t saddr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(saddr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2-D tiled TMA load, global -> this CTA's shared memory, completion counted
// on `bar`.  Never multicast.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(saddr(dst)),
      "l"(map), "r"(x), "r"(y), "r"(saddr(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_release(uint32_t *p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t *p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

__device__ __forceinline__ void fence_acq_rel() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

__device__ __forceinline__ uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint4 ld_shared_v4(const void *p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(saddr(p)));
  return v;
}

// bf16 pair in a 32-bit word -> two floats (exact).
__device__ __forceinline__ float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ void unpack8(const uint4 &w, float (&f)[8]) {
  f[0] = bf_lo(w.x); f[1] = bf_hi(w.x); f[2] = bf_lo(w.y); f[3] = bf_hi(w.y);
  f[4] = bf_lo(w.z); f[5] = bf_hi(w.z); f[6] = bf_lo(w.w); f[7] = bf_hi(w.w);
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void *p) {
  return __ldg(reinterpret_cast<const uint4 *>(p));
}

__device__ __forceinline__ float silu(float u) { return u / (1.0f + expf(-u)); }

__host__ __device__ constexpr int ilog2c(int n) { return n <= 1 ? 0 : 1 + ilog2c(n >> 1); }

__device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

// Butterfly transpose-reduce of N partial sums over the 32 lanes.  After it,
// for N >= 32 lane l holds the full sums of indices (N/32)*l + i in v[i];
// for N < 32 lane l holds index l >> (5 - log2 N) in v[0].
template <int N>
__device__ __forceinline__ void butterfly(float (&v)[N], int lane) {
  constexpr int S = (N >= 32) ? 5 : ilog2c(N);
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int o = 16 >> s;
    if (s < S) {
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < (N >> (s + 1)); ++i) {
        const int hh = N >> (s + 1);
        float send = up ? v[i] : v[i + hh];
        float recv = __shfl_xor_sync(0xffffffffu, send, o);
        v[i] = (up ? v[i + hh] : v[i]) + recv;
      }
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
}

// Store the butterfly result so that buf[i] = full sum of index i (i < N).
template <int N>
__device__ __forceinline__ void butterfly_store(const float (&v)[N], float *buf, int lane) {
  if constexpr (N >= 32) {
#pragma unroll
    for (int i = 0; i < N / 32; ++i) buf[(N / 32) * lane + i] = v[i];
  } else {
    constexpr int rep = 32 / N;
    if ((lane & (rep - 1)) == 0) buf[lane / rep] = v[0];
  }
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// Per-warp state
// ---------------------------------------------------------------------------
constexpr int kWbuf = 64;  // floats of per-warp epilogue scratch (R * MJ <= 64)

struct Warp {
  const Params *P;
  int lane, wib, slot, nw;
  uint32_t epoch;
  uint8_t *ring;
  uint64_t *bars;
  float *wbuf, *wacc, *wtmp;
  uint32_t *arrive;
  uint32_t phase;  // bit s: parity of the next completion of slot s
  int cslot, islot, inflight;
  // issue cursor
  int iop, iu, it, in_units, in_tiles;
  bool iop_init, done_issue;
  // attention items: prefix[b] = first item of sequence b
  int attn_prefix[kMaxRows + 1];
  int attn_nch[kMaxRows];
  uint64_t pol_w, pol_kv;
  bool failed;
};

__device__ __forceinline__ const Params &PP(const Warp &w) { return *w.P; }

__device__ void set_error(Warp &w, int code, int op) {
  if (w.lane == 0) {
    if (atomicCAS(&w.P->error[0], 0, code) == 0) atomicExch(&w.P->error[1], op);
  }
  w.failed = true;
}

__device__ __forceinline__ int rot_of(int op, int nw) {
  return static_cast<int>((static_cast<uint32_t>(op) * 2654435761u) % static_cast<uint32_t>(nw));
}

__device__ __forceinline__ int first_unit(const Warp &w, int op) {
  return (w.slot - rot_of(op, w.nw) + w.nw) % w.nw;
}

__device__ __forceinline__ int my_unit_count(const Warp &w, int op, int total) {
  int u0 = first_unit(w, op);
  return total > u0 ? (total - 1 - u0) / w.nw + 1 : 0;
}

__device__ __forceinline__ int tile_cols(const Params &P) { return P.rows_per_tile == 16 ? 256 : 512; }

__device__ __forceinline__ bool routing_ready(const Warp &w, int layer) {
  uint32_t v = 0;
  if (w.lane == 0) v = ld_relaxed(&w.P->route_flag[layer * kCounterStride]);
  v = __shfl_sync(0xffffffffu, v, 0);
  bool ok = static_cast<int>(v - w.epoch) >= 0;
  if (ok) fence_acq_rel();
  return ok;
}

__device__ __forceinline__ int n_union(const Warp &w, int layer) {
  return __ldcg(&w.P->routing[layer].n_union);
}

// Total units of an op over the whole grid.  ROUTED_GU / DOWN need routing.
__device__ int op_total_units(const Warp &w, int type, int layer) {
  const Params &P = PP(w);
  const int R = P.rows_per_tile;
  switch (type) {
    case OP_EMBED: return P.n_hb;
    case OP_QKV: return cdiv((P.Hq + 2 * P.Hkv) * P.hd, R);
    case OP_ATTN: return w.attn_prefix[P.B];
    case OP_OPROJ: return P.n_hb;
    case OP_ROUTER: return cdiv(P.E, R) * cdiv(P.d, tile_cols(P));
    case OP_SHARED_GU: return P.Fs > 0 ? (2 * P.Fs) / R : 0;
    case OP_ROUTED_GU: return n_union(w, layer) * ((2 * P.F) / R);
    case OP_DOWN: return P.n_hb;
    case OP_LMHEAD: return cdiv(P.V, R);
  }
  return 0;
}

struct AttnItem {
  int b, g, qs, c, pos0, npos, ntiles;
};

__device__ AttnItem attn_item(const Warp &w, int item) {
  const Params &P = PP(w);
  AttnItem a;
  int b = 0;
  while (b + 1 < P.B && item >= w.attn_prefix[b + 1]) ++b;
  int rem = item - w.attn_prefix[b];
  int nch = w.attn_nch[b];
  a.b = b;
  a.c = rem % nch;
  a.qs = (rem / nch) % P.attn_qsplit;
  a.g = rem / (nch * P.attn_qsplit);
  int len = __ldg(&P.positions[b]) + P.T;
  a.pos0 = a.c * P.attn_chunk;
  a.npos = min(P.attn_chunk, len - a.pos0);
  a.ntiles = cdiv(a.npos, P.attn_ppt);
  return a;
}

__device__ int unit_tiles(const Warp &w, int type, int layer, int unit) {
  const Params &P = PP(w);
  const int TC = tile_cols(P);
  switch (type) {
    case OP_QKV:
    case OP_SHARED_GU:
    case OP_ROUTED_GU:
    case OP_LMHEAD: return cdiv(P.d, TC);
    case OP_OPROJ: return cdiv(P.Hq * P.hd, TC);
    case OP_ROUTER: return 1;
    case OP_DOWN:
      return n_union(w, layer) * cdiv(P.F, TC) + (P.Fs > 0 ? cdiv(P.Fs, TC) : 0);
    case OP_ATTN: return attn_item(w, unit).ntiles;
    default: return 0;
  }
}

// ---------------------------------------------------------------------------
// Producer side: issue the next tiles of this warp's stream into free slots.
// ---------------------------------------------------------------------------
__device__ void issue_tile(Warp &w, int op, int type, int layer, int unit, int t) {
  const Params &P = PP(w);
  const int R = P.rows_per_tile, TC = tile_cols(P);
  const bool tall = (R == 16);
  uint8_t *dst = w.ring + w.islot * kSlotBytes;
  uint64_t *bar = &w.bars[w.islot];
  const CUtensorMap *m0 = nullptr, *m1 = nullptr;
  int x0 = 0, y0 = 0, x1 = 0, y1 = 0, K = P.d, rows = 0;
  bool two = true;
  uint64_t pol = w.pol_w;
  const CUtensorMap *lm = P.tmaps + layer * MAPS_PER_LAYER;
  if (type == OP_ATTN) {
    AttnItem a = attn_item(w, unit);
    int pos = a.pos0 + t * P.attn_ppt;
    int row = ((layer * P.Bmax + a.b) * P.Hkv + a.g) * P.cap + pos;
    m0 = &P.kmap;
    m1 = &P.vmap;
    x0 = x1 = 0;
    y0 = y1 = row;
    pol = w.pol_kv;
  } else {
    int row0 = 0, col0 = t * TC;
    switch (type) {
      case OP_QKV: m0 = lm + MAP_WQKV; row0 = unit * R; rows = (P.Hq + 2 * P.Hkv) * P.hd; break;
      case OP_OPROJ: m0 = lm + MAP_WO; row0 = unit * R; K = P.Hq * P.hd; rows = P.d; break;
      case OP_LMHEAD: m0 = P.tmaps + P.L * MAPS_PER_LAYER; row0 = unit * R; rows = P.V; break;
      case OP_ROUTER: {
        int nrb = cdiv(P.E, R);
        row0 = (unit % nrb) * R;
        col0 = (unit / nrb) * TC;
        m0 = lm + MAP_ROUTER;
        rows = P.E;
        break;
      }
      case OP_SHARED_GU:
        row0 = unit * R;
        if (row0 < P.Fs) {
          m0 = lm + MAP_WSGATE;
        } else {
          m0 = lm + MAP_WSUP;
          row0 -= P.Fs;
        }
        rows = P.Fs;
        break;
      case OP_ROUTED_GU: {
        int nrb = (2 * P.F) / R;
        int j = unit / nrb;
        int r0 = (unit % nrb) * R;
        int e = __ldcg(&P.routing[layer].expert[j]);
        if (r0 < P.F) {
          m0 = lm + MAP_WGATE;
        } else {
          m0 = lm + MAP_WUP;
          r0 -= P.F;
        }
        row0 = e * P.F + r0;
        rows = P.E * P.F;
        break;
      }
      case OP_DOWN: {
        int U = n_union(w, layer);
        int tpr = cdiv(P.F, TC);
        if (t < U * tpr) {
          int j = t / tpr;
          int e = __ldcg(&P.routing[layer].expert[j]);
          m0 = lm + MAP_WDOWN;
          row0 = e * P.d + unit * R;
          col0 = (t % tpr) * TC;
          K = P.F;
          rows = P.E * P.d;
        } else {
          m0 = lm + MAP_WSDOWN;
          row0 = unit * R;
          col0 = (t - U * tpr) * TC;
          K = P.Fs;
          rows = P.d;
        }
        break;
      }
      default: break;
    }
    m1 = m0;
    x0 = col0;
    y0 = row0;
    if (tall) {
      x1 = col0;
      y1 = row0 + kBoxRows;
      two = (y1 < rows);
    } else {
      x1 = col0 + kPanel;
      y1 = row0;
      two = (x1 < K);
    }
  }
  if (w.lane == 0) {
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, (two ? 2u : 1u) * kBoxBytes);
    tma_load_2d(dst, m0, x0, y0, bar, pol);
    if (two) tma_load_2d(dst + kBoxBytes, m1, x1, y1, bar, pol);
  }
  w.islot = (w.islot + 1 == kSlots) ? 0 : w.islot + 1;
  w.inflight++;
}

__device__ void issue_more(Warp &w) {
  const Params &P = PP(w);
  while (!w.done_issue && w.inflight < kSlots && !w.failed) {
    if (w.iop >= P.op_end) {
      w.done_issue = true;
      break;
    }
    const int type = op_type_of(w.iop, P.L), layer = op_layer_of(w.iop, P.L);
    if (!w.iop_init) {
      if ((type == OP_ROUTED_GU || type == OP_DOWN) && !routing_ready(w, layer)) return;
      w.in_units = (type == OP_EMBED) ? 0 : my_unit_count(w, w.iop, op_total_units(w, type, layer));
      w.iu = 0;
      w.it = 0;
      w.in_tiles = -1;
      w.iop_init = true;
    }
    if (w.iu >= w.in_units) {
      w.iop++;
      w.iop_init = false;
      continue;
    }
    const int unit = first_unit(w, w.iop) + w.iu * w.nw;
    if (w.in_tiles < 0) w.in_tiles = unit_tiles(w, type, layer, unit);
    if (w.it >= w.in_tiles) {
      w.iu++;
      w.it = 0;
      w.in_tiles = -1;
      continue;
    }
    issue_tile(w, w.iop, type, layer, unit, w.it);
    w.it++;
  }
}

// ---------------------------------------------------------------------------
// Consumer side
// ---------------------------------------------------------------------------
__device__ const uint8_t *consume_begin(Warp &w, int op) {
  if (w.failed) return nullptr;
  const Params &P = PP(w);
  if (w.inflight == 0) issue_more(w);
  if (w.inflight == 0) {  // the tile stream and the consumer loop disagree: never expected
    set_error(w, -8, op);
    return nullptr;
  }
  uint64_t *bar = &w.bars[w.cslot];
  const uint32_t par = (w.phase >> w.cslot) & 1u;
  uint64_t t0 = 0;
  for (int it = 0;; ++it) {
    bool ok = mbar_try_wait(bar, par);
    if (__all_sync(0xffffffffu, ok)) break;
    if ((it & 63) == 63) {
      int bad = 0;
      if (w.lane == 0) {
        uint64_t t = now_ns();
        if (t0 == 0) t0 = t;
        bad = (t - t0 > P.timeout_ns) ? 1 : 0;
      }
      if (__shfl_sync(0xffffffffu, bad, 0)) {
        set_error(w, -5, op);
        return nullptr;
      }
    }
  }
  return w.ring + w.cslot * kSlotBytes;
}

__device__ __forceinline__ void consume_end(Warp &w) {
  __syncwarp();
  w.phase ^= (1u << w.cslot);
  w.cslot = (w.cslot + 1 == kSlots) ? 0 : w.cslot + 1;
  w.inflight--;
  issue_more(w);
}

// Wait for `ctr` to reach `target` (bounded), filling the ring meanwhile.
__device__ bool wait_counter(Warp &w, const uint32_t *ctr, uint32_t target, int op) {
  const Params &P = PP(w);
  uint64_t t0 = 0;
  for (int it = 0;; ++it) {
    uint32_t v = 0;
    int err = 0;
    if (w.lane == 0) {
      v = ld_relaxed(ctr);
      err = *reinterpret_cast<volatile const int *>(P.error);
    }
    v = __shfl_sync(0xffffffffu, v, 0);
    err = __shfl_sync(0xffffffffu, err, 0);
    if (static_cast<int>(v - target) >= 0) break;
    if (err) {
      w.failed = true;
      return false;
    }
    issue_more(w);
    int bad = 0;
    if (w.lane == 0) {
      uint64_t t = now_ns();
      if (t0 == 0) t0 = t;
      bad = (t - t0 > P.timeout_ns) ? 1 : 0;
      if (!bad && it > 8) __nanosleep(64);
    }
    if (__shfl_sync(0xffffffffu, bad, 0)) {
      set_error(w, -5, op);
      return false;
    }
  }
  fence_acq_rel();
  __syncwarp();
  return true;
}

__device__ void drain(Warp &w) {
  // Wait (bounded) for every copy still in flight before the CTA may exit.
  while (w.inflight > 0) {
    uint64_t *bar = &w.bars[w.cslot];
    const uint32_t par = (w.phase >> w.cslot) & 1u;
    uint64_t t0 = now_ns();
    while (!mbar_try_wait(bar, par)) {
      if (now_ns() - t0 > 50000000ull) break;
    }
    w.phase ^= (1u << w.cslot);
    w.cslot = (w.cslot + 1 == kSlots) ? 0 : w.cslot + 1;
    w.inflight--;
  }
  __syncwarp();
}

// Arrive on an op's counter once this warp's units of it are done.  Returns
// true (on every lane) for the warp whose arrival completed the op grid-wide.
__device__ bool arrive(Warp &w, int op) {
  const Params &P = PP(w);
  __syncwarp();
  int last = 0;
  if (w.lane == 0) {
    __threadfence();
    uint32_t old = atomicAdd(&w.arrive[op], 1u);
    if (old == kWarpsPerCta - 1) {
      __threadfence();
      uint32_t g = atom_add_acq_rel(&P.counters[op * kCounterStride], 1u);
      last = (g + 1 == w.epoch * static_cast<uint32_t>(P.n_cta)) ? 1 : 0;
    }
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (last) fence_acq_rel();
  __syncwarp();
  return last != 0;
}

// ---------------------------------------------------------------------------
// Activation sources (one lane, 8 consecutive columns, MJ rows)
// ---------------------------------------------------------------------------
template <int MJ>
struct XNorm {  // x = h * inv_rms * g
  const float *h;
  int d;
  const __nv_bfloat16 *g;
  int row[MJ];
  float inv[MJ];
  int n;
  __device__ __forceinline__ void load(int col, int K, float (&x)[MJ][8]) const {
    if (col < K) {
      float gf[8];
      unpack8(ldg_nc_v4(g + col), gf);
#pragma unroll
      for (int j = 0; j < MJ; ++j) {
        if (j < n) {
          const float4 *p = reinterpret_cast<const float4 *>(h + static_cast<size_t>(row[j]) * d + col);
          float4 a = __ldcg(p), b = __ldcg(p + 1);
          x[j][0] = a.x * inv[j] * gf[0]; x[j][1] = a.y * inv[j] * gf[1];
          x[j][2] = a.z * inv[j] * gf[2]; x[j][3] = a.w * inv[j] * gf[3];
          x[j][4] = b.x * inv[j] * gf[4]; x[j][5] = b.y * inv[j] * gf[5];
          x[j][6] = b.z * inv[j] * gf[6]; x[j][7] = b.w * inv[j] * gf[7];
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) x[j][k] = 0.f;
        }
      }
    } else {
#pragma unroll
      for (int j = 0; j < MJ; ++j)
#pragma unroll
        for (int k = 0; k < 8; ++k) x[j][k] = 0.f;
    }
  }
};

template <int MJ>
struct XPlain {  // x = src[row][col]
  const float *src;
  int ld;
  int row[MJ];
  int n;
  __device__ __forceinline__ void load(int col, int K, float (&x)[MJ][8]) const {
#pragma unroll
    for (int j = 0; j < MJ; ++j) {
      if (col < K && j < n) {
        const float4 *p = reinterpret_cast<const float4 *>(src + static_cast<size_t>(row[j]) * ld + col);
        float4 a = __ldcg(p), b = __ldcg(p + 1);
        x[j][0] = a.x; x[j][1] = a.y; x[j][2] = a.z; x[j][3] = a.w;
        x[j][4] = b.x; x[j][5] = b.y; x[j][6] = b.z; x[j][7] = b.w;
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) x[j][k] = 0.f;
      }
    }
  }
};

template <int MJ>
struct XSwiGLU {  // x = silu(gu[row][col]) * gu[row][F + col]
  const float *gu;
  int ld, F;
  int row[MJ];
  int n;
  __device__ __forceinline__ void load(int col, int K, float (&x)[MJ][8]) const {
#pragma unroll
    for (int j = 0; j < MJ; ++j) {
      if (col < K && j < n) {
        const float *base = gu + static_cast<size_t>(row[j]) * ld;
        const float4 *pg = reinterpret_cast<const float4 *>(base + col);
        const float4 *pu = reinterpret_cast<const float4 *>(base + F + col);
        float4 g0 = __ldcg(pg), g1 = __ldcg(pg + 1), u0 = __ldcg(pu), u1 = __ldcg(pu + 1);
        x[j][0] = silu(g0.x) * u0.x; x[j][1] = silu(g0.y) * u0.y;
        x[j][2] = silu(g0.z) * u0.z; x[j][3] = silu(g0.w) * u0.w;
        x[j][4] = silu(g1.x) * u1.x; x[j][5] = silu(g1.y) * u1.y;
        x[j][6] = silu(g1.z) * u1.z; x[j][7] = silu(g1.w) * u1.w;
      } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) x[j][k] = 0.f;
      }
    }
  }
};

// One tile: acc[r*MJ + j] += W[r][cols] . x[j][cols] over this lane's columns.
template <int MJ, int R, int NP, class XS>
__device__ __forceinline__ void gemv_tile(const uint8_t *slot, float (&acc)[R * MJ], int colbase,
                                          int K, const XS &xs, int lane) {
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int pc = colbase + p * kPanel;
    if (pc >= K) break;
    float x[MJ][8];
    xs.load(pc + lane * 8, K, x);
    const uint8_t *pan = slot + p * kBoxBytes + lane * 16;
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float wf[8];
      unpack8(ld_shared_v4(pan + r * (kPanel * 2)), wf);
#pragma unroll
      for (int j = 0; j < MJ; ++j) {
        float a = acc[r * MJ + j];
#pragma unroll
        for (int k = 0; k < 8; ++k) a = fmaf(wf[k], x[j][k], a);
        acc[r * MJ + j] = a;
      }
    }
  }
}

// Streams `ntiles` tiles of one segment through the ring into acc.
template <int MJ, int R, int NP, class XS>
__device__ bool gemv_segment(Warp &w, int op, int ntiles, int K, const XS &xs,
                             float (&acc)[R * MJ]) {
  for (int t = 0; t < ntiles; ++t) {
    const uint8_t *slot = consume_begin(w, op);
    if (!slot) return false;
    gemv_tile<MJ, R, NP>(slot, acc, t * kPanel * NP, K, xs, w.lane);
    consume_end(w);
  }
  return true;
}

// inv_rms for rows 0..M-1 from the residual producers' partial sums of squares.
__device__ void compute_inv_rms(const Warp &w, float *inv) {
  const Params &P = PP(w);
  for (int m = 0; m < P.M; ++m) {
    float s = 0.f;
    for (int i = w.lane; i < P.n_hb; i += 32) s += __ldcg(&P.ss[m * P.n_hb + i]);
    s = warp_sum(s);
    inv[m] = 1.0f / sqrtf(s / static_cast<float>(P.d) + P.eps);
  }
}

template <int MMAX>
struct Cfg {
  static constexpr int R = (MMAX <= 4) ? 16 : 8;
  static constexpr int NP = (MMAX <= 4) ? 1 : 2;
};

// ---------------------------------------------------------------------------
// Ops
// ---------------------------------------------------------------------------
// Residual update of rows [row0, row0+R) from wacc[r*MMAX + m], plus the
// partial sum of squares of the new values for the next RMSNorm.
template <int MMAX>
__device__ void residual_epilogue(Warp &w, int unit, int row0, int dbg_layer) {
  const Params &P = PP(w);
  constexpr int R = Cfg<MMAX>::R;
  for (int e = w.lane; e < R * P.M; e += 32) {
    int m = e / R, r = e % R, row = row0 + r;
    float sq = 0.f;
    if (row < P.d) {
      float *hp = P.h + static_cast<size_t>(m) * P.d + row;
      float hn = __ldcg(hp) + w.wacc[r * MMAX + m];
      __stcg(hp, hn);
      sq = hn * hn;
      if (dbg_layer >= 0 && P.dbg_hidden)
        P.dbg_hidden[(static_cast<size_t>(dbg_layer) * P.max_rows + m) * P.d + row] = hn;
    }
    w.wtmp[m * R + r] = sq;
  }
  __syncwarp();
  if (w.lane < P.M) {
    float s = 0.f;
    for (int r = 0; r < R; ++r) s += w.wtmp[w.lane * R + r];
    __stcg(&P.ss[w.lane * P.n_hb + unit], s);
  }
  __syncwarp();
}

template <int MMAX>
__device__ void op_embed(Warp &w, int op) {
  const Params &P = PP(w);
  constexpr int R = Cfg<MMAX>::R;
  const int n = my_unit_count(w, op, P.n_hb), u0 = first_unit(w, op);
  for (int i = 0; i < n; ++i) {
    const int unit = u0 + i * w.nw, row0 = unit * R;
    for (int e = w.lane; e < R * P.M; e += 32) {
      int m = e / R, r = e % R, row = row0 + r;
      float sq = 0.f;
      if (row < P.d) {
        int tok = __ldcg(&P.tokens[m]);  // may alias the argmax output
        if (tok < 0 || tok >= P.V) tok = 0;  // rejected at kernel start
        float v = __bfloat162float(P.embed[static_cast<size_t>(tok) * P.d + row]);
        __stcg(&P.h[static_cast<size_t>(m) * P.d + row], v);
        if (P.dbg_hidden) P.dbg_hidden[static_cast<size_t>(m) * P.d + row] = v;  // layer slot 0
        sq = v * v;
      }
      w.wtmp[m * R + r] = sq;
    }
    __syncwarp();
    if (w.lane < P.M) {
      float s = 0.f;
      for (int r = 0; r < R; ++r) s += w.wtmp[w.lane * R + r];
      __stcg(&P.ss[w.lane * P.n_hb + unit], s);
    }
    __syncwarp();
  }
}

// Dense GEMV ops over all M rows: QKV, OPROJ, ROUTER, SHARED_GU, LMHEAD.
template <int MMAX>
__device__ bool op_dense(Warp &w, int op, int type, int layer, float &am_val, int &am_idx) {
  const Params &P = PP(w);
  constexpr int R = Cfg<MMAX>::R, NP = Cfg<MMAX>::NP, MJ = MMAX;
  const int total = op_total_units(w, type, layer);
  const int n = my_unit_count(w, op, total), u0 = first_unit(w, op);
  if (n == 0) return true;
  float inv[kMaxRows];
  if (type != OP_OPROJ) compute_inv_rms(w, inv);
  const __nv_bfloat16 *g = (type == OP_QKV)      ? P.norms[2 * layer]
                           : (type == OP_LMHEAD) ? P.final_norm
                                                 : P.norms[2 * layer + 1];
  XNorm<MJ> xn;
  XPlain<MJ> xp;
  xn.h = P.h; xn.d = P.d; xn.g = g; xn.n = P.M;
  xp.src = P.o; xp.ld = P.Hq * P.hd; xp.n = P.M;
#pragma unroll
  for (int j = 0; j < MJ; ++j) {
    xn.row[j] = j < P.M ? j : 0;
    xn.inv[j] = (j < P.M && type != OP_OPROJ) ? inv[j] : 0.f;
    xp.row[j] = j < P.M ? j : 0;
  }
  const int TC = R == 16 ? 256 : 512;
  for (int i = 0; i < n; ++i) {
    const int unit = u0 + i * w.nw;
    float acc[R * MJ];
#pragma unroll
    for (int q = 0; q < R * MJ; ++q) acc[q] = 0.f;
    int row0 = unit * R, N = 0;
    bool ok;
    if (type == OP_OPROJ) {
      ok = gemv_segment<MJ, R, NP>(w, op, cdiv(P.Hq * P.hd, TC), P.Hq * P.hd, xp, acc);
      N = P.d;
    } else if (type == OP_ROUTER) {
      const int nrb = cdiv(P.E, R), kc = unit / nrb;
      row0 = (unit % nrb) * R;
      // one tile of columns [kc*TC, kc*TC + TC): shift the activation source
      const uint8_t *slot = consume_begin(w, op);
      ok = slot != nullptr;
      if (ok) {
        gemv_tile<MJ, R, NP>(slot, acc, kc * TC, P.d, xn, w.lane);
        consume_end(w);
      }
      N = P.E;
    } else {
      ok = gemv_segment<MJ, R, NP>(w, op, cdiv(P.d, TC), P.d, xn, acc);
      N = (type == OP_QKV) ? (P.Hq + 2 * P.Hkv) * P.hd
          : (type == OP_SHARED_GU) ? 2 * P.Fs
                                   : P.V;
    }
    if (!ok) return false;
    butterfly<R * MJ>(acc, w.lane);
    butterfly_store<R * MJ>(acc, w.wbuf, w.lane);
    __syncwarp();
    switch (type) {
      case OP_QKV: {
        const int W3 = (P.Hq + 2 * P.Hkv) * P.hd;
        for (int e = w.lane; e < R * P.M; e += 32) {
          int m = e / R, r = e % R;
          if (row0 + r < N) __stcg(&P.qkv[static_cast<size_t>(m) * W3 + row0 + r], w.wbuf[r * MJ + m]);
        }
        break;
      }
      case OP_SHARED_GU:
        for (int e = w.lane; e < R * P.M; e += 32) {
          int m = e / R, r = e % R;
          if (row0 + r < N)
            __stcg(&P.gu_shared[static_cast<size_t>(m) * 2 * P.Fs + row0 + r], w.wbuf[r * MJ + m]);
        }
        break;
      case OP_ROUTER: {
        const int kc = unit / cdiv(P.E, R);
        for (int e = w.lane; e < R * P.M; e += 32) {
          int m = e / R, r = e % R;
          if (row0 + r < N)
            __stcg(&P.router_part[(static_cast<size_t>(kc) * kMaxRows + m) * P.E + row0 + r],
                   w.wbuf[r * MJ + m]);
        }
        break;
      }
      case OP_LMHEAD: {
        for (int e = w.lane; e < R * P.M; e += 32) {
          int m = e / R, r = e % R;
          if (row0 + r < N) P.logits[static_cast<size_t>(m) * P.V + row0 + r] = w.wbuf[r * MJ + m];
        }
        if (w.lane < P.M) {
          for (int r = 0; r < R && row0 + r < N; ++r) {
            float v = w.wbuf[r * MJ + w.lane];
            if (v > am_val) {
              am_val = v;
              am_idx = row0 + r;
            }
          }
        }
        break;
      }
      case OP_OPROJ: {
        for (int e = w.lane; e < R * MMAX; e += 32) {
          int r = e / MMAX, m = e % MMAX;
          w.wacc[r * MMAX + m] = w.wbuf[r * MJ + m];
        }
        __syncwarp();
        residual_epilogue<MMAX>(w, unit, row0, -1);
        break;
      }
      default: break;
    }
    __syncwarp();
  }
  return true;
}

// Routed gate/up rows for every expert in the union (rows of that expert only).
template <int MMAX, int MJ>
__device__ bool routed_gu_unit(Warp &w, int op, int layer, int unit, const float *inv) {
  const Params &P = PP(w);
  constexpr int R = Cfg<MMAX>::R, NP = Cfg<MMAX>::NP, TC = R == 16 ? 256 : 512;
  const int nrb = (2 * P.F) / R, j = unit / nrb, row0 = (unit % nrb) * R;
  const uint32_t mask = __ldcg(&P.routing[layer].rowmask[j]);
  XNorm<MJ> xn;
  xn.h = P.h; xn.d = P.d; xn.g = P.norms[2 * layer + 1];
  int n = 0;
#pragma unroll
  for (int q = 0; q < MJ; ++q) { xn.row[q] = 0; xn.inv[q] = 0.f; }
  for (int m = 0; m < P.M; ++m) {
    if (mask & (1u << m)) {
#pragma unroll
      for (int q = 0; q < MJ; ++q)
        if (q == n) { xn.row[q] = m; xn.inv[q] = inv[m]; }
      ++n;
    }
  }
  xn.n = n;
  float acc[R * MJ];
#pragma unroll
  for (int q = 0; q < R * MJ; ++q) acc[q] = 0.f;
  if (!gemv_segment<MJ, R, NP>(w, op, cdiv(P.d, TC), P.d, xn, acc)) return false;
  butterfly<R * MJ>(acc, w.lane);
  butterfly_store<R * MJ>(acc, w.wbuf, w.lane);
  __syncwarp();
  const size_t ld = 2 * static_cast<size_t>(P.F);
  for (int e = w.lane; e < R * n; e += 32) {
    int q = e / R, r = e % R;
    int m = 0;
#pragma unroll
    for (int qq = 0; qq < MJ; ++qq)
      if (qq == q) m = xn.row[qq];
    __stcg(&P.gu_routed[(static_cast<size_t>(j) * kMaxRows + m) * ld + row0 + r], w.wbuf[r * MJ + q]);
  }
  __syncwarp();
  return true;
}

template <int MMAX>
__device__ bool op_routed_gu(Warp &w, int op, int layer) {
  const Params &P = PP(w);
  const int total = op_total_units(w, OP_ROUTED_GU, layer);
  const int n = my_unit_count(w, op, total), u0 = first_unit(w, op);
  if (n == 0) return true;
  float inv[kMaxRows];
  compute_inv_rms(w, inv);
  const int nrb = (2 * P.F) / Cfg<MMAX>::R;
  for (int i = 0; i < n; ++i) {
    const int unit = u0 + i * w.nw;
    const uint32_t mask = __ldcg(&P.routing[layer].rowmask[unit / nrb]);
    const int cnt = __popc(mask);
    bool ok;
    if (cnt <= 1) ok = routed_gu_unit<MMAX, 1>(w, op, layer, unit, inv);
    else if (cnt <= 2) ok = routed_gu_unit<MMAX, (MMAX >= 2 ? 2 : 1)>(w, op, layer, unit, inv);
    else if (cnt <= 4) ok = routed_gu_unit<MMAX, (MMAX >= 4 ? 4 : 1)>(w, op, layer, unit, inv);
    else ok = routed_gu_unit<MMAX, (MMAX >= 8 ? 8 : 1)>(w, op, layer, unit, inv);
    if (!ok) return false;
  }
  return true;
}

// One down-projection segment (routed expert j, or the shared expert when
// j < 0) for rows [row0, row0+R): wacc[r][m] += weight(m) * (Wd[row] . act[m]).
template <int MMAX, int MJ>
__device__ bool down_segment(Warp &w, int op, int layer, int j, int row0) {
  const Params &P = PP(w);
  constexpr int R = Cfg<MMAX>::R, NP = Cfg<MMAX>::NP, TC = R == 16 ? 256 : 512;
  XSwiGLU<MJ> xs;
  float wt[MJ];
  int n = 0;
#pragma unroll
  for (int q = 0; q < MJ; ++q) { xs.row[q] = 0; wt[q] = 0.f; }
  int K;
  if (j >= 0) {
    const uint32_t mask = __ldcg(&P.routing[layer].rowmask[j]);
    xs.gu = P.gu_routed + static_cast<size_t>(j) * kMaxRows * 2 * P.F;
    xs.ld = 2 * P.F;
    xs.F = P.F;
    K = P.F;
    for (int m = 0; m < P.M; ++m) {
      if (mask & (1u << m)) {
        float wm = __ldcg(&P.routing[layer].weight[j][m]);
#pragma unroll
        for (int q = 0; q < MJ; ++q)
          if (q == n) { xs.row[q] = m; wt[q] = wm; }
        ++n;
      }
    }
  } else {
    xs.gu = P.gu_shared;
    xs.ld = 2 * P.Fs;
    xs.F = P.Fs;
    K = P.Fs;
    for (int m = 0; m < P.M; ++m) {
#pragma unroll
      for (int q = 0; q < MJ; ++q)
        if (q == m) { xs.row[q] = m; wt[q] = 1.f; }
    }
    n = P.M;
  }
  xs.n = n;
  float acc[R * MJ];
#pragma unroll
  for (int q = 0; q < R * MJ; ++q) acc[q] = 0.f;
  if (!gemv_segment<MJ, R, NP>(w, op, cdiv(K, TC), K, xs, acc)) return false;
  butterfly<R * MJ>(acc, w.lane);
  butterfly_store<R * MJ>(acc, w.wbuf, w.lane);
  __syncwarp();
  for (int e = w.lane; e < R * n; e += 32) {
    int q = e / R, r = e % R;
    int m = 0;
    float wm = 0.f;
#pragma unroll
    for (int qq = 0; qq < MJ; ++qq)
      if (qq == q) { m = xs.row[qq]; wm = wt[qq]; }
    w.wacc[r * MMAX + m] += wm * w.wbuf[r * MJ + q];
  }
  __syncwarp();
  (void)row0;
  return true;
}

template <int MMAX>
__device__ bool op_down(Warp &w, int op, int layer) {
  const Params &P = PP(w);
  constexpr int R = Cfg<MMAX>::R;
  const int n = my_unit_count(w, op, P.n_hb), u0 = first_unit(w, op);
  if (n == 0) return true;
  const int U = n_union(w, layer);
  for (int i = 0; i < n; ++i) {
    const int unit = u0 + i * w.nw, row0 = unit * R;
    for (int e = w.lane; e < R * MMAX; e += 32) w.wacc[e] = 0.f;
    __syncwarp();
    for (int j = 0; j < U; ++j) {
      const int cnt = __popc(__ldcg(&P.routing[layer].rowmask[j]));
      bool ok;
      if (cnt <= 1) ok = down_segment<MMAX, 1>(w, op, layer, j, row0);
      else if (cnt <= 2) ok = down_segment<MMAX, (MMAX >= 2 ? 2 : 1)>(w, op, layer, j, row0);
      else if (cnt <= 4) ok = down_segment<MMAX, (MMAX >= 4 ? 4 : 1)>(w, op, layer, j, row0);
      else ok = down_segment<MMAX, (MMAX >= 8 ? 8 : 1)>(w, op, layer, j, row0);
      if (!ok) return false;
    }
    if (P.Fs > 0) {
      if (!down_segment<MMAX, MMAX>(w, op, layer, -1, row0)) return false;
    }
    residual_epilogue<MMAX>(w, unit, row0, layer + 1);
  }
  return true;
}

// --- attention ---------------------------------------------------------------
template <int QVP, int DPL>
__device__ bool attn_item_run(Warp &w, int op, int layer, int item) {
  const Params &P = PP(w);
  constexpr int PG = 32 / QVP;  // positions per butterfly group
  constexpr int hd = 32 * DPL, half = hd / 2;
  const int G = P.Hq / P.Hkv;
  const AttnItem a = attn_item(w, item);
  const int pos_b = __ldg(&P.positions[a.b]);
  const int W3 = (P.Hq + 2 * P.Hkv) * hd;
  const float scale = 1.0f / sqrtf(static_cast<float>(hd));
  // query vectors of this item: qv = qs*QVP + v  ->  (t = qv / G, head = g*G + qv % G)
  float q[QVP][DPL];
  int lim[QVP];
  const int lane = w.lane, ppos = lane & 15;
#pragma unroll
  for (int v = 0; v < QVP; ++v) {
    const int qv = a.qs * QVP + v;
    lim[v] = -1;
#pragma unroll
    for (int dd = 0; dd < DPL; ++dd) q[v][dd] = 0.f;
    if (qv < G * P.T) {
      const int t = qv / G, head = a.g * G + qv % G, m = a.b * P.T + t, p = pos_b + t;
      lim[v] = p;
      const float *src = P.qkv + static_cast<size_t>(m) * W3 + head * hd + lane * DPL;
#pragma unroll
      for (int dd = 0; dd < DPL; ++dd) {
        float own = __ldcg(src + dd);
        float other = __shfl_xor_sync(0xffffffffu, own, 16);
        float2 cs = __ldg(&P.rope[static_cast<size_t>(p) * half + ppos * DPL + dd]);
        float r = (lane < 16) ? own * cs.x - other * cs.y : own * cs.x + other * cs.y;
        q[v][dd] = r * scale;
      }
    } else {
#pragma unroll
      for (int dd = 0; dd < DPL; ++dd) (void)__shfl_xor_sync(0xffffffffu, 0.f, 16);
    }
  }
  float m_run = -INFINITY, l_run = 0.f;
  float o[QVP][DPL];
#pragma unroll
  for (int v = 0; v < QVP; ++v)
#pragma unroll
    for (int dd = 0; dd < DPL; ++dd) o[v][dd] = 0.f;
  const int my_qv = lane % QVP;
  const size_t cache_row_base =
      (static_cast<size_t>(layer) * P.Bmax + a.b) * P.Hkv * P.cap + static_cast<size_t>(a.g) * P.cap;
  for (int tt = 0; tt < a.ntiles; ++tt) {
    uint8_t *slot = const_cast<uint8_t *>(consume_begin(w, op));
    if (!slot) return false;
    const int pos0 = a.pos0 + tt * P.attn_ppt;
    __nv_bfloat16 *ks = reinterpret_cast<__nv_bfloat16 *>(slot);
    __nv_bfloat16 *vs = reinterpret_cast<__nv_bfloat16 *>(slot + kBoxBytes);
    // New positions of this step inside the tile: rotate k, round k and v to
    // bf16, patch the tile and (once per chunk) append them to the cache.
    const int lo = max(pos0, pos_b), hi = min(pos0 + P.attn_ppt, pos_b + P.T);
    bool patched = false;
    for (int p = lo; p < hi; ++p) {
      const int t = p - pos_b, m = a.b * P.T + t;
      const float *kq = P.qkv + static_cast<size_t>(m) * W3 + (P.Hq + a.g) * hd + lane * DPL;
      const float *vq = P.qkv + static_cast<size_t>(m) * W3 + (P.Hq + P.Hkv + a.g) * hd + lane * DPL;
#pragma unroll
      for (int dd = 0; dd < DPL; ++dd) {
        float own = __ldcg(kq + dd);
        float other = __shfl_xor_sync(0xffffffffu, own, 16);
        float2 cs = __ldg(&P.rope[static_cast<size_t>(p) * half + ppos * DPL + dd]);
        float kr = (lane < 16) ? own * cs.x - other * cs.y : own * cs.x + other * cs.y;
        __nv_bfloat16 kb = __float2bfloat16_rn(kr);
        __nv_bfloat16 vb = __float2bfloat16_rn(__ldcg(vq + dd));
        ks[(p - pos0) * hd + lane * DPL + dd] = kb;
        vs[(p - pos0) * hd + lane * DPL + dd] = vb;
        if (a.qs == 0) {
          P.kc[(cache_row_base + p) * hd + lane * DPL + dd] = kb;
          P.vc[(cache_row_base + p) * hd + lane * DPL + dd] = vb;
        }
      }
      patched = true;
    }
    if (patched) fence_proxy_async_smem();
    __syncwarp();
    for (int jg = 0; jg < P.attn_ppt; jg += PG) {
      float part[32];
#pragma unroll
      for (int j = 0; j < PG; ++j) {
        float kf[DPL];
        const __nv_bfloat16 *kr = ks + (jg + j) * hd + lane * DPL;
#pragma unroll
        for (int dd = 0; dd < DPL; ++dd) kf[dd] = __bfloat162float(kr[dd]);
#pragma unroll
        for (int v = 0; v < QVP; ++v) {
          float s = 0.f;
#pragma unroll
          for (int dd = 0; dd < DPL; ++dd) s = fmaf(q[v][dd], kf[dd], s);
          part[j * QVP + v] = s;
        }
      }
      butterfly<32>(part, lane);
      // lane holds the score of position jg + lane / QVP for query lane % QVP
      const int pos = pos0 + jg + lane / QVP;
      int my_lim = -1;
#pragma unroll
      for (int v = 0; v < QVP; ++v)
        if (v == my_qv) my_lim = lim[v];
      const bool valid = (pos <= my_lim) && (pos < a.pos0 + a.npos);
      float s = valid ? part[0] : -INFINITY;
      float mx = s;
#pragma unroll
      for (int o2 = QVP; o2 < 32; o2 <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
      const float m_new = fmaxf(m_run, mx);
      const float pr = valid ? expf(s - m_new) : 0.f;
      const float alpha = (m_run == -INFINITY) ? 0.f : expf(m_run - m_new);
      float ps = pr;
#pragma unroll
      for (int o2 = QVP; o2 < 32; o2 <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o2);
      l_run = l_run * alpha + ps;
      m_run = m_new;
#pragma unroll
      for (int v = 0; v < QVP; ++v) {
        const float av = __shfl_sync(0xffffffffu, alpha, v);
#pragma unroll
        for (int dd = 0; dd < DPL; ++dd) o[v][dd] *= av;
      }
#pragma unroll
      for (int j = 0; j < PG; ++j) {
        float vf[DPL];
        const __nv_bfloat16 *vr = vs + (jg + j) * hd + lane * DPL;
#pragma unroll
        for (int dd = 0; dd < DPL; ++dd) vf[dd] = __bfloat162float(vr[dd]);
#pragma unroll
        for (int v = 0; v < QVP; ++v) {
          const float pj = __shfl_sync(0xffffffffu, pr, j * QVP + v);
#pragma unroll
          for (int dd = 0; dd < DPL; ++dd) o[v][dd] = fmaf(pj, vf[dd], o[v][dd]);
        }
      }
    }
    consume_end(w);
  }
  // partial of this chunk
  const int grp = (a.b * P.Hkv + a.g) * P.attn_qsplit + a.qs;
  const size_t pidx = static_cast<size_t>(grp) * P.attn_nch_max + a.c;
#pragma unroll
  for (int v = 0; v < QVP; ++v)
#pragma unroll
    for (int dd = 0; dd < DPL; ++dd)
      __stcg(&P.attn_o[(pidx * QVP + v) * hd + lane * DPL + dd], o[v][dd]);
  if (lane < QVP) {
    __stcg(&P.attn_ml[(static_cast<size_t>(grp) * QVP + lane) * 2 * P.attn_nch_max + a.c], m_run);
    __stcg(&P.attn_ml[(static_cast<size_t>(grp) * QVP + lane) * 2 * P.attn_nch_max + P.attn_nch_max + a.c],
           l_run);
  }
  return true;
}

// Merge n partials (m_i, l_i, o_i) of each query vector: level 1 keeps the
// unnormalised (max, sum, weighted o); level 2 writes o / l.
template <int QVP, int DPL>
__device__ void attn_merge(Warp &w, int grp, int first, int n, int nstride, const float *src_o,
                           const float *src_ml, float *dst_o, float *dst_ml, int dst_index,
                           int dst_stride, bool final_level, int b, int g) {
  const Params &P = PP(w);
  constexpr int hd = 32 * DPL;
  const int lane = w.lane, G = P.Hq / P.Hkv;
  for (int v = 0; v < QVP; ++v) {
    const float *mrow = src_ml + (static_cast<size_t>(grp) * QVP + v) * 2 * nstride;
    float mi = -INFINITY, li = 0.f;
    if (lane < n) {
      mi = __ldcg(mrow + first + lane);
      li = __ldcg(mrow + nstride + first + lane);
    }
    const float M = warp_max(mi);
    const float wi = (lane < n && mi != -INFINITY) ? expf(mi - M) : 0.f;
    const float L = warp_sum(wi * li);
    float acc[DPL];
#pragma unroll
    for (int dd = 0; dd < DPL; ++dd) acc[dd] = 0.f;
    for (int i = 0; i < n; ++i) {
      const float wv = __shfl_sync(0xffffffffu, wi, i);
      const float *op = src_o + ((static_cast<size_t>(grp) * nstride + first + i) * QVP + v) * hd + lane * DPL;
#pragma unroll
      for (int dd = 0; dd < DPL; ++dd) acc[dd] = fmaf(wv, __ldcg(op + dd), acc[dd]);
    }
    if (!final_level) {
      float *dop = dst_o + ((static_cast<size_t>(grp) * dst_stride + dst_index) * QVP + v) * hd + lane * DPL;
#pragma unroll
      for (int dd = 0; dd < DPL; ++dd) __stcg(dop + dd, acc[dd]);
      if (lane == 0) {
        float *dml = dst_ml + (static_cast<size_t>(grp) * QVP + v) * 2 * dst_stride;
        __stcg(dml + dst_index, M);
        __stcg(dml + dst_stride + dst_index, L);
      }
    } else {
      const int qv = (grp % P.attn_qsplit) * QVP + v;
      if (qv < G * P.T) {
        const int t = qv / G, head = g * G + qv % G, m = b * P.T + t;
        const float invl = 1.0f / L;
        float *dst = P.o + static_cast<size_t>(m) * P.Hq * hd + head * hd + lane * DPL;
#pragma unroll
        for (int dd = 0; dd < DPL; ++dd) __stcg(dst + dd, acc[dd] * invl);
      }
    }
  }
}

// Arrival on a merge counter; true for the last of `n` arrivals (resets it).
__device__ bool merge_arrive(Warp &w, uint32_t *ctr, int n) {
  __syncwarp();
  int last = 0;
  if (w.lane == 0) {
    __threadfence();
    uint32_t old = atom_add_acq_rel(ctr, 1u);
    if (old + 1 == static_cast<uint32_t>(n)) {
      last = 1;
      *ctr = 0;
    }
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (last) fence_acq_rel();
  __syncwarp();
  return last != 0;
}

template <int QVP, int DPL>
__device__ bool op_attn(Warp &w, int op, int layer) {
  const Params &P = PP(w);
  const int total = w.attn_prefix[P.B];
  const int n = my_unit_count(w, op, total), u0 = first_unit(w, op);
  for (int i = 0; i < n; ++i) {
    const int item = u0 + i * w.nw;
    if (!attn_item_run<QVP, DPL>(w, op, layer, item)) return false;
    const AttnItem a = attn_item(w, item);
    const int grp = (a.b * P.Hkv + a.g) * P.attn_qsplit + a.qs;
    const int nch = w.attn_nch[a.b];
    const int k1 = a.c / kL1Fan, n1 = min(kL1Fan, nch - k1 * kL1Fan), ngrp1 = cdiv(nch, kL1Fan);
    uint32_t *c1 = P.attn_cnt + static_cast<size_t>(grp) * (kL1Fan + 1) + k1;
    if (merge_arrive(w, c1, n1)) {
      attn_merge<QVP, DPL>(w, grp, k1 * kL1Fan, n1, P.attn_nch_max, P.attn_o, P.attn_ml, P.attn_o1,
                      P.attn_ml1, k1, kL1Fan, false, a.b, a.g);
      uint32_t *c2 = P.attn_cnt + static_cast<size_t>(grp) * (kL1Fan + 1) + kL1Fan;
      if (merge_arrive(w, c2, ngrp1)) {
        attn_merge<QVP, DPL>(w, grp, 0, ngrp1, kL1Fan, P.attn_o1, P.attn_ml1, nullptr, nullptr, 0, 0,
                        true, a.b, a.g);
      }
    }
  }
  return true;
}

// --- router top-k and the final argmax (run by the op's last arriving warp) --
__device__ void router_topk(Warp &w, int layer) {
  const Params &P = PP(w);
  const int lane = w.lane, E = P.E, K = P.topk;
  const int nkc = cdiv(P.d, tile_cols(P));
  constexpr int EPL = kMaxExperts / 32;
  uint32_t rmask[EPL];
  float wsel[EPL][kMaxRows];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    rmask[i] = 0;
#pragma unroll
    for (int m = 0; m < kMaxRows; ++m) wsel[i][m] = 0.f;
  }
  for (int m = 0; m < P.M; ++m) {
    float z[EPL];
    bool taken[EPL];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      z[i] = -INFINITY;
      taken[i] = true;
      if (e < E) {
        float s = 0.f;
        for (int kc = 0; kc < nkc; ++kc) s += __ldcg(&P.router_part[(static_cast<size_t>(kc) * kMaxRows + m) * E + e]);
        z[i] = s;
        taken[i] = false;
        mx = fmaxf(mx, s);
      }
    }
    mx = warp_max(mx);
    float pi[EPL], sum = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      pi[i] = (lane + 32 * i < E) ? expf(z[i] - mx) : 0.f;
      sum += pi[i];
    }
    sum = warp_sum(sum);
#pragma unroll
    for (int i = 0; i < EPL; ++i) pi[i] = pi[i] / sum;
    float sel = 0.f;
    int ids[kMaxTopK];
    float ws[kMaxTopK];
    for (int j = 0; j < K; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if (!taken[i] && (pi[i] > bv || (pi[i] == bv && e < bi))) {
          bv = pi[i];
          bi = e;
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) {
          bv = ov;
          bi = oi;
        }
      }
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (lane + 32 * i == bi) taken[i] = true;
      ids[j] = bi;
      ws[j] = bv;
      sel += bv;
    }
    for (int j = 0; j < K; ++j) {
      const float wn = ws[j] / sel;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        if (lane + 32 * i == ids[j]) {
          rmask[i] |= (1u << m);
#pragma unroll
          for (int mm = 0; mm < kMaxRows; ++mm)
            if (mm == m) wsel[i][mm] = wn;
        }
      }
      if (lane == 0) {
        if (P.dbg_ids) P.dbg_ids[(static_cast<size_t>(layer) * P.max_rows + m) * K + j] = ids[j];
        if (P.dbg_w) P.dbg_w[(static_cast<size_t>(layer) * P.max_rows + m) * K + j] = wn;
      }
    }
  }
  // publish the union in ascending expert order
  Routing *rt = P.routing + layer;
  int base = 0;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const bool has = rmask[i] != 0;
    const uint32_t bits = __ballot_sync(0xffffffffu, has);
    if (has) {
      const int pos = base + __popc(bits & ((1u << lane) - 1u));
      rt->expert[pos] = lane + 32 * i;
      rt->rowmask[pos] = rmask[i];
#pragma unroll
      for (int m = 0; m < kMaxRows; ++m) rt->weight[pos][m] = wsel[i][m];
    }
    base += __popc(bits);
  }
  if (lane == 0) {
    rt->n_union = base;
    atomicAdd(&P.stats[0], static_cast<unsigned long long>(base));
  }
  __syncwarp();
  if (lane == 0) {
    __threadfence();
    st_release(&P.route_flag[layer * kCounterStride], w.epoch);
  }
  __syncwarp();
}

__device__ void final_argmax(Warp &w) {
  const Params &P = PP(w);
  for (int m = 0; m < P.M; ++m) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int s = w.lane; s < P.n_warps; s += 32) {
      const ArgmaxPart *pp = P.am_part + static_cast<size_t>(s) * kMaxRows + m;
      const float v = __ldcg(&pp->value);
      const int ix = __ldcg(&pp->index);
      if (v > bv || (v == bv && ix < bi)) {
        bv = v;
        bi = ix;
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (w.lane == 0) P.argmax[m] = (bi == 0x7fffffff) ? 0 : bi;
  }
  __syncwarp();
  if (w.lane == 0) {
    __threadfence();
    st_release(P.epoch, w.epoch);
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
template <int MMAX>
__global__ void __launch_bounds__(kThreads, 1) mk_step_kernel(const __grid_constant__ Params P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  Warp w;
  w.P = &P;
  w.lane = threadIdx.x & 31;
  w.wib = threadIdx.x >> 5;
  w.nw = P.n_warps;
  w.slot = w.wib * P.n_cta + blockIdx.x;
  w.ring = smem + w.wib * kSlots * kSlotBytes;
  uint8_t *after_ring = smem + kWarpsPerCta * kSlots * kSlotBytes;
  w.bars = reinterpret_cast<uint64_t *>(after_ring) + w.wib * kSlots;
  float *fbase = reinterpret_cast<float *>(after_ring + kWarpsPerCta * kSlots * sizeof(uint64_t));
  w.wbuf = fbase + w.wib * 3 * kWbuf;
  w.wacc = w.wbuf + kWbuf;
  w.wtmp = w.wacc + kWbuf;
  w.arrive = reinterpret_cast<uint32_t *>(fbase + kWarpsPerCta * 3 * kWbuf);
  w.phase = 0;
  w.cslot = w.islot = w.inflight = 0;
  w.failed = false;
  w.pol_w = policy_evict_first();
  w.pol_kv = policy_evict_normal();
  if (w.lane == 0) {
    for (int s = 0; s < kSlots; ++s) mbar_init(&w.bars[s], 1);
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < P.n_ops; i += kThreads) w.arrive[i] = 0;
  __syncthreads();

  w.epoch = *reinterpret_cast<volatile const uint32_t *>(P.epoch) + 1u;

  // Reject bad positions / token ids before any memory is touched with them.
  // Every warp evaluates the same condition, so all exit together.
  bool bad = false;
  for (int b = 0; b < P.B; ++b) {
    int p = __ldg(&P.positions[b]);
    if (p < 0 || p + P.T > P.cap) bad = true;
  }
  for (int m = w.lane; m < P.M; m += 32) {
    int t = __ldcg(&P.tokens[m]);
    if (t < 0 || t >= P.V) bad = true;
  }
  bad = __any_sync(0xffffffffu, bad);
  if (bad) {
    set_error(w, -6, P.op_begin);
    return;
  }
  // attention work items per sequence
  w.attn_prefix[0] = 0;
  for (int b = 0; b < kMaxRows; ++b) {
    int nch = 0;
    if (b < P.B) nch = cdiv(__ldg(&P.positions[b]) + P.T, P.attn_chunk);
    if (b < kMaxRows) w.attn_nch[b] = nch;
    w.attn_prefix[b + 1] = w.attn_prefix[b] + (b < P.B ? P.Hkv * P.attn_qsplit * nch : 0);
  }

  w.iop = P.op_begin;
  w.iop_init = false;
  w.done_issue = false;
  w.in_units = w.iu = w.it = 0;
  w.in_tiles = -1;
  issue_more(w);

  float am_val = -INFINITY;
  int am_idx = 0x7fffffff;
  for (int op = P.op_begin; op < P.op_end && !w.failed; ++op) {
    const int type = op_type_of(op, P.L), layer = op_layer_of(op, P.L);
    int d0, d1;
    op_deps(op, P.L, &d0, &d1);
    const uint32_t target = w.epoch * static_cast<uint32_t>(P.n_cta);
    const uint32_t extra = (op == P.inject_op) ? 1u : 0u;
    if (d0 >= 0 && !wait_counter(w, &P.counters[d0 * kCounterStride], target + extra, op)) break;
    if (d1 >= 0 && !wait_counter(w, &P.counters[d1 * kCounterStride], target, op)) break;
    if (type == OP_ROUTED_GU || type == OP_DOWN) {
      if (!wait_counter(w, &P.route_flag[layer * kCounterStride], w.epoch, op)) break;
    }
    bool ok = true;
    switch (type) {
      case OP_EMBED: op_embed<MMAX>(w, op); break;
      case OP_ATTN:
        if (P.hd == 64)
          ok = (P.attn_qvp == 8) ? op_attn<8, 2>(w, op, layer) : op_attn<4, 2>(w, op, layer);
        else
          ok = (P.attn_qvp == 8) ? op_attn<8, 4>(w, op, layer) : op_attn<4, 4>(w, op, layer);
        break;
      case OP_ROUTED_GU: ok = op_routed_gu<MMAX>(w, op, layer); break;
      case OP_DOWN: ok = op_down<MMAX>(w, op, layer); break;
      default: ok = op_dense<MMAX>(w, op, type, layer, am_val, am_idx); break;
    }
    if (!ok || w.failed) break;
    if (type == OP_LMHEAD && w.lane < P.M) {
      P.am_part[static_cast<size_t>(w.slot) * kMaxRows + w.lane] = ArgmaxPart{am_val, am_idx};
    }
    const bool last = arrive(w, op);
    if (last && type == OP_ROUTER) router_topk(w, layer);
    if (last && type == OP_LMHEAD) final_argmax(w);
  }
  drain(w);
}

}  // namespace

size_t step_smem_bytes(int n_ops) {
  return static_cast<size_t>(kWarpsPerCta) * kSlots * kSlotBytes +
         kWarpsPerCta * kSlots * sizeof(uint64_t) + kWarpsPerCta * 3 * kWbuf * sizeof(float) +
         static_cast<size_t>(n_ops) * sizeof(uint32_t);
}

template <int MMAX>
static const void *kernel_ptr() {
  return reinterpret_cast<const void *>(&mk_step_kernel<MMAX>);
}

static const void *kernel_for(int mmax) {
  switch (mmax) {
    case 1: return kernel_ptr<1>();
    case 2: return kernel_ptr<2>();
    case 4: return kernel_ptr<4>();
    default: return kernel_ptr<8>();
  }
}

int max_cta_per_sm(int mmax, size_t smem) {
  const void *k = kernel_for(mmax);
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return -1;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kThreads, smem) != cudaSuccess) return -1;
  return n;
}

int launch_step(const Params &p, int mmax, bool cooperative, cudaStream_t stream) {
  const void *k = kernel_for(mmax);
  const size_t smem = step_smem_bytes(p.n_ops);
  void *args[] = {const_cast<Params *>(&p)};
  cudaError_t e;
  if (cooperative) {
    e = cudaLaunchCooperativeKernel(k, dim3(p.n_cta), dim3(kThreads), args, smem, stream);
  } else {
    e = cudaLaunchKernel(k, dim3(p.n_cta), dim3(kThreads), args, smem, stream);
  }
  return e == cudaSuccess ? 0 : static_cast<int>(e);
}

}  // namespace mk
