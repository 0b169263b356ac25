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
// The step is a fixed list of ops (EMBED; per layer QKV, ATTN, OPROJ, ROUTER,
// SHARED_GU, ROUTED_GU, DOWN, COMBINE; LMHEAD).  Each op's work is cut into
// units of at most 64 KB of weights, dealt round-robin to the grid's warps
// (consecutive units land on different SMs).  A warp done with an op arrives
// on the op's counter (aggregated per CTA in shared memory, then one
// release-add per CTA); an op that needs an earlier op's output spins (bounded
// by %globaltimer) until that counter reaches epoch * n_cta.  Counters only
// grow, so no reset is needed between steps.
//
// GEMV math: a tile is 4 weight rows x 1024 columns (four 4 x 256 TMA boxes);
// each lane owns 8 columns of each box and keeps the matching activations of
// every row in registers, so one 16-byte weight load feeds 8*MJ FMAs.  Lane
// partial sums are combined with a butterfly (transpose-reduce) of warp
// shuffles.  All arithmetic is fp32.
//
// Everything on the per-tile path is force-inlined so that a warp's ring and
// cursor state stays in registers.
#include <cstdio>

#include "mk_internal.h"

#define MK_INLINE __device__ __forceinline__

#ifndef MK_TRACE
#define MK_TRACE 0
#endif
#if MK_TRACE
#define MK_ENTRY(name) name##_traced
#else
#define MK_ENTRY(name) name
#endif

namespace mk {
namespace {

// This file is compiled twice: MK_TRACE=0 gives the step kernels, MK_TRACE=1
// the same kernels with the per-op / per-tile timeline compiled in (launched
// only when a trace buffer is set), so that the timed kernels carry no trace code.
constexpr bool kTrace = MK_TRACE != 0;

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
MK_INLINE uint32_t saddr(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

MK_INLINE void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr(bar)), "r"(count) : "memory");
}

MK_INLINE void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(saddr(bar)), "r"(bytes)
               : "memory");
}

MK_INLINE bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
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

// Blocking with a time limit: the thread may be suspended (issuing nothing)
// for up to about `ns` nanoseconds until the phase of `parity` completes.
MK_INLINE bool mbar_wait_hint(uint64_t *bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(saddr(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}

MK_INLINE void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(saddr(bar)) : "memory");
}

MK_INLINE void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

MK_INLINE void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// 2-D tiled TMA load, global -> this CTA's shared memory, completion counted
// on `bar`.  Never multicast.
MK_INLINE void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar,
                           uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(saddr(dst)),
      "l"(map), "r"(x), "r"(y), "r"(saddr(bar)), "l"(policy)
      : "memory");
}

// Bring the 128-byte line at p into L2 (no register result, no completion).
MK_INLINE void prefetch_l2(const void *p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

MK_INLINE uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

MK_INLINE uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

MK_INLINE uint32_t ld_relaxed(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Acquire load: later loads of this thread see what was released before the
// value it reads (and everything that release observed).
MK_INLINE uint32_t ld_acquire(const uint32_t *p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// CTA-scope acq_rel add on a shared-memory counter (generic address).
MK_INLINE uint32_t atom_add_acq_rel_cta(uint32_t *p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.cta.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

MK_INLINE void st_release(uint32_t *p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

MK_INLINE uint32_t atom_add_acq_rel(uint32_t *p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Release-add with no result: the arriving warp does not wait for the reply.
MK_INLINE void red_add_release(uint32_t *p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Fixed-point accumulation (kFixShift fraction bits in an int64): integer
// additions are exact and associative, so a sum of many contributions is the
// same whatever order the warps add them in.
MK_INLINE long long to_fix(float v) { return __float2ll_rn(v * 4294967296.0f); }
MK_INLINE float from_fix(long long a) { return static_cast<float>(static_cast<double>(a) * 0x1p-32); }
static_assert(kFixShift == 32, "to_fix / from_fix scale by 2^32");

MK_INLINE void red_add_fix(long long *p, long long v) {
  asm volatile("red.relaxed.gpu.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}


MK_INLINE uint64_t now_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

MK_INLINE uint4 ld_shared_v4(const void *p) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(saddr(p)));
  return v;
}

// bf16 pair in a 32-bit word -> two floats (exact).
MK_INLINE float bf_lo(uint32_t u) { return __uint_as_float(u << 16); }
MK_INLINE float bf_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// A bf16 pair (low half = even element) as floats.
MK_INLINE float2 bf2(uint32_t u) { return make_float2(bf_lo(u), bf_hi(u)); }
// Two fp32 FMAs / products in one instruction, each rounded as its scalar form.
MK_INLINE float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
MK_INLINE float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }



// Bring the line holding p into this SM's L1 (no register result).

MK_INLINE float silu(float u) { return u / (1.0f + expf(-u)); }

__host__ __device__ constexpr int ilog2c(int n) { return n <= 1 ? 0 : 1 + ilog2c(n >> 1); }

MK_INLINE int cdiv(int a, int b) { return (a + b - 1) / b; }

// Butterfly transpose-reduce of N partial sums over the 32 lanes.  After it,
// for N >= 32 lane l holds the full sums of indices (N/32)*l + i in v[i];
// for N < 32 lane l holds index l >> (5 - log2 N) in v[0].
template <int N>
MK_INLINE void butterfly(float (&v)[N], int lane) {
  constexpr int S = (N >= 32) ? 5 : ilog2c(N);
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int o = 16 >> s;
    if (s < S) {
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < (N >> (s + 1)); ++i) {
        const int hh = N >> (s + 1);
        const float send = up ? v[i] : v[i + hh];
        const float recv = __shfl_xor_sync(0xffffffffu, send, o);
        v[i] = (up ? v[i + hh] : v[i]) + recv;
      }
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
}

// Store the butterfly result so that buf[i] = full sum of index i (i < N).
template <int N>
MK_INLINE void butterfly_store(const float (&v)[N], float *buf, int lane) {
  if constexpr (N >= 32) {
#pragma unroll
    for (int i = 0; i < N / 32; ++i) buf[(N / 32) * lane + i] = v[i];
  } else {
    constexpr int rep = 32 / N;
    if ((lane & (rep - 1)) == 0) buf[lane / rep] = v[0];
  }
}

// Order-preserving map of a float onto uint32 (a larger float has a larger
// key), for warp-wide integer max reductions, and its inverse.
MK_INLINE uint32_t float_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
MK_INLINE float key_float(uint32_t k) { return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k); }

MK_INLINE float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

MK_INLINE float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Units are dealt round-robin: warp slot s takes units u0(s) + i * n_warps,
// with a per-op rotation so that remainders do not always land on warp 0.
MK_INLINE int op_rotation(int op, int nw) {
  return static_cast<int>((static_cast<uint32_t>(op) * 2654435761u) % static_cast<uint32_t>(nw));
}

// The first unit of `op` for warp slot `slot`: units go round-robin over the
// slots from a per-op rotation.  Routed gate/up units continue the dealing of
// the shared expert's (the op before), so the warps that took a shared unit
// take fewer routed ones.
MK_INLINE int first_unit_of(int slot, int op, int nw, int type, int shared_units) {
  int rot = op_rotation(op, nw);
  if (type == OP_ROUTED_GU) rot = (op_rotation(op - 1, nw) + shared_units) % nw;
  return (slot - rot + nw) % nw;
}

MK_INLINE int unit_count_of(int u0, int total, int nw) { return total > u0 ? (total - 1 - u0) / nw + 1 : 0; }

// ---------------------------------------------------------------------------
// Per-warp state (scalars only, so that it lives in registers)
// ---------------------------------------------------------------------------
constexpr int kWbuf = 64;  // floats of per-warp epilogue scratch (2 * 4 * MJ <= 64)

// One layer's routing, computed by every CTA for itself from the router's
// split-K partial logits: per row its selections (expert id and renormalised
// weight, in selection order), and the ascending union of the selected
// experts with the rows that chose each and in which selection slot.
struct RouteCache {
  int ready_key, fill_key;   // route_key of the layer once computed / being computed
  int n_union;
  int expert[kMaxExperts];
  uint32_t rowmask[kMaxExperts];
  int8_t kslot[kMaxExperts][kMaxRows];
  float row_w[kMaxRows][kMaxTopK];
  uint8_t row_e[kMaxRows][kMaxTopK];
};

struct Warp {
  const Params *P;
  RouteCache *rc;
  int lane, wib, cta, slot, nw;
  uint32_t epoch;
  uint8_t *ring;           // this consumer's nslots tiles
  int nslots;
  uint64_t *full, *empty;  // per slot: tile landed / tile released
  float *wbuf;
  uint32_t *arrive;
  long long *rsum;             // the CTA's router-logit sums of the current layer, [MMAX][e_ld],
                               // 2^-32 fixed point (shared memory)
  int *attn_prefix;        // this warp's: first item of each sequence, [kMaxRows + 1]
  int *attn_nch;           // this warp's: KV chunks of each sequence, [kMaxRows]
  int step;                // the step (of a multi-step launch) this warp is in
  int lstep;               // the step its attention layout was computed for
  // consumer side: bit s = parity of the next completion of full[s]
  uint32_t phase;
  int cslot;
  // producer side (a consumer's record, kept by the warp that feeds it): bit s
  // of ephase = parity to wait for on empty[s] before refilling it; filled =
  // slots filled at least once
  uint32_t ephase, filled;
  int islot;
  bool producer;
  int dseg0;  // staged down projection: the first expert segment of this CTA's range
  uint32_t xphase;  // batch 1: stagings of the activation row so far
  // producer cursor: op, this consumer's unit index in it, tile in the unit
  int iop, iu0, in_units, iu, it, in_tiles, iunit;
  int itype, ilayer;  // type and layer of op iop, once its current unit is set up
  int istride;        // unit stride of op iop for this warp
  // the current unit's tile source: maps for the first and second half of its
  // tiles (gate / up), first row of each, first column, K, tiles per half
  const CUtensorMap *um, *um2;
  int urow0, urow2, ucol0, uK, uhalf;
  bool iop_init, done_issue;
  uint64_t pol_w, pol_kv;
  bool failed;
  // per-op timeline (only with a trace buffer): first tile ready, last tile
  // consumed, ns blocked on tiles, tiles consumed
  uint64_t tr_first, tr_last, tr_wait;
  int tr_n;
};

__device__ __noinline__ void report_error(const Params &P, int lane, int code, int op) {
  if (lane == 0) {
    if (atomicCAS(&P.error[0], 0, code) == 0) atomicExch(&P.error[1], op);
  }
}

MK_INLINE void set_error(Warp &w, int code, int op) {
  report_error(*w.P, w.lane, code, op);
  w.failed = true;
}

// The layer's router logits are complete once the o-projection's counter
// reaches its target (its units add them up); every lane then re-reads it
// with acquire semantics.
MK_INLINE bool routing_ready(const Warp &w, int layer) {
  const uint32_t *ctr = &w.P->counters[op_index(layer, OP_OPROJ) * kCounterStride];
  const uint32_t target = w.epoch * static_cast<uint32_t>(w.P->n_cta);
  const uint32_t v = ld_relaxed(ctr);
  const bool ok = __all_sync(0xffffffffu, static_cast<int>(v - target) >= 0);
  if (ok) (void)ld_acquire(ctr);
  return ok;
}

// Lane l owns experts 4l..4l+3 and 128+4l..128+4l+3.
MK_INLINE int expert_of(int lane, int i) { return (i < 4) ? 4 * lane + i : 128 + 4 * lane + (i - 4); }

// The CTA's routing for `layer` (one warp; the caller has seen the
// o-projection complete).  Per row: the router logits z = u / rms(h), u the
// fixed-point sums of W_r (h * g_ffn) that the o-projection units added up;
// k rounds of argmax (ties to the lower expert id); weights = the softmax
// renormalised over the chosen experts.  Softmax is monotone, so ranking the
// logits ranks the probabilities, and the full softmax's normaliser cancels
// in the renormalisation: w_j = e^(z_j - z_max) / sum over chosen i of
// e^(z_i - z_max).  Every CTA runs this on the same sums and gets the same
// result.  The code runs once per layer per CTA (cold), so it is kept short.
__device__ __noinline__ void route_compute(const Params &P, RouteCache *rc, int lane, int key, int layer) {
  const int E = P.E, K = P.topk;
  constexpr int EPL = 8;
  uint32_t chosen[EPL];  // rows that selected each of this lane's experts
  uint64_t slots[EPL];   // byte m: the selection slot row m gave it
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    chosen[i] = 0;
    slots[i] = 0;
  }
  // the rows' sums of squares are loaded with the first row's logits (one
  // round trip at batch 1)
  const long long sqv = lane < P.M ? __ldcg(P.ssq + kMaxRows + lane) : 0ll;
  for (int m = 0; m < P.M; ++m) {
    const long long *row = P.racc + (static_cast<size_t>(layer) * kMaxRows + m) * P.e_ld;
    longlong2 ua[2], ub[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      ua[h] = 4 * lane < E ? __ldcg(reinterpret_cast<const longlong2 *>(row + 4 * lane) + h) : make_longlong2(0, 0);
      ub[h] = 128 + 4 * lane < E ? __ldcg(reinterpret_cast<const longlong2 *>(row + 128 + 4 * lane) + h)
                                 : make_longlong2(0, 0);
    }
    float z[EPL];
    const long long u[EPL] = {ua[0].x, ua[0].y, ua[1].x, ua[1].y, ub[0].x, ub[0].y, ub[1].x, ub[1].y};
    const long long sqm = __shfl_sync(0xffffffffu, sqv, m);
    const float im = 1.0f / sqrtf(static_cast<float>(static_cast<double>(sqm) * 0x1p-32) / static_cast<float>(P.d) + P.eps);
#pragma unroll
    for (int i = 0; i < EPL; ++i) z[i] = im * from_fix(u[i]);
    // the keys of this lane's experts; 0 = not a candidate (absent or taken)
    uint32_t key[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) key[i] = expert_of(lane, i) < E ? float_key(z[i]) : 0u;
    // k rounds of argmax; lane j keeps selection j.  The lane scans its
    // candidates in ascending expert id (strict >), and among lanes holding
    // the maximum the lowest id wins.
    float my_z = 0.f;
    int my_e = 0;
    for (int j = 0; j < K; ++j) {
      uint32_t bk = 0u;
      int bl = 0;
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (key[i] > bk) {
          bk = key[i];
          bl = expert_of(lane, i);
        }
      const uint32_t best = __reduce_max_sync(0xffffffffu, bk);
      const int bi = static_cast<int>(__reduce_min_sync(0xffffffffu, bk == best ? static_cast<uint32_t>(bl) : 0xffffffffu));
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (expert_of(lane, i) == bi) {
          key[i] = 0u;
          chosen[i] |= 1u << m;
          slots[i] |= static_cast<uint64_t>(j) << (8 * m);
        }
      if (lane == j) {
        my_e = bi;
        my_z = key_float(best);
      }
    }
    const float zmax = __shfl_sync(0xffffffffu, my_z, 0);
    const float e = lane < K ? expf(my_z - zmax) : 0.f;
    const float sel = warp_sum(e);
    if (lane < K) {
      rc->row_w[m][lane] = e / sel;
      rc->row_e[m][lane] = static_cast<uint8_t>(my_e);
    }
  }
  // ascending union: every id below 128 (slots i < 4) precedes every id above
  int lo = 0, hi = 0;
#pragma unroll
  for (int i = 0; i < EPL; ++i) (i < 4 ? lo : hi) += chosen[i] ? 1 : 0;
  int lo_incl = lo, hi_incl = hi;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, lo_incl, o), b = __shfl_up_sync(0xffffffffu, hi_incl, o);
    if (lane >= o) {
      lo_incl += a;
      hi_incl += b;
    }
  }
  const int lo_total = __shfl_sync(0xffffffffu, lo_incl, 31), hi_total = __shfl_sync(0xffffffffu, hi_incl, 31);
  int pos_lo = lo_incl - lo, pos_hi = lo_total + hi_incl - hi;
#pragma unroll
  for (int i = 0; i < EPL; ++i)
    if (chosen[i]) {
      const int pos = (i < 4) ? pos_lo++ : pos_hi++;
      rc->expert[pos] = expert_of(lane, i);
      rc->rowmask[pos] = chosen[i];
#pragma unroll
      for (int m = 0; m < kMaxRows; ++m) rc->kslot[pos][m] = static_cast<int8_t>((slots[i] >> (8 * m)) & 0xff);
    }
  if (lane == 0) rc->n_union = lo_total + hi_total;
  __threadfence_block();
  __syncwarp();
  if (lane == 0) *reinterpret_cast<volatile int *>(&rc->ready_key) = key;
  __syncwarp();
}

// The layer's routing statistics and debug copy, written once per (step,
// layer) by the warp that computed CTA 0's routing (nothing waits for this):
// the union size into the statistics and, if requested, each row's experts
// and weights in selection order.
__device__ __noinline__ void route_publish(const Params &P, const RouteCache *rc, int lane, int layer) {
  if (lane == 0) atomicAdd(&P.stats[0], static_cast<unsigned long long>(rc->n_union));
  const int K = P.topk;
  for (int idx = lane; idx < P.M * K; idx += 32) {
    const int m = idx / K, j = idx % K;
    if (P.dbg_ids) P.dbg_ids[(static_cast<size_t>(layer) * P.max_rows + m) * K + j] = rc->row_e[m][j];
    if (P.dbg_w) P.dbg_w[(static_cast<size_t>(layer) * P.max_rows + m) * K + j] = rc->row_w[m][j];
  }
  __syncwarp();
}

// Trace: when this warp first found its CTA's routing cache ready for the
// layer, and whether it filled it (words 6 and 7 of its ROUTED_GU record).
MK_INLINE void trace_route_cache(const Warp &w, int layer, int filler) {
  const Params &P = *w.P;
  if (kTrace && P.trace && w.lane == 0 && !w.producer) {
    unsigned long long *tr = P.trace + (static_cast<size_t>(op_index(layer, OP_ROUTED_GU)) * w.nw + w.slot) * kTraceWords;
    if (tr[6] == 0) {
      tr[6] = now_ns();
      tr[7] = static_cast<unsigned long long>(filler);
    }
  }
}

// The routing of (step, layer) is identified by step * L + layer + 1.
MK_INLINE int route_key(const Warp &w, int layer) { return w.step * w.P->L + layer + 1; }

MK_INLINE bool route_cache(Warp &w, int layer) {
  RouteCache *rc = w.rc;
  const int key = route_key(w, layer);
  if (*reinterpret_cast<volatile int *>(&rc->ready_key) == key) {
    __threadfence_block();
    trace_route_cache(w, layer, 0);
    return true;
  }
  int filler = 0;
  if (w.lane == 0) filler = atomicMax(&rc->fill_key, key) < key ? 1 : 0;
  filler = __shfl_sync(0xffffffffu, filler, 0);
  if (filler) {
    route_compute(*w.P, rc, w.lane, key, layer);
    // once per (step, layer): CTA 0 of the launch that holds the routed gate/up
    // op (a one-op-per-launch variant recomputes the routing in later launches)
    const int rgu = op_index(layer, OP_ROUTED_GU);
    if (w.cta == 0 && w.P->op_begin <= rgu && rgu < w.P->op_end) route_publish(*w.P, rc, w.lane, layer);
  } else {
    const uint64_t t0 = now_ns();
    while (*reinterpret_cast<volatile int *>(&rc->ready_key) != key) {
      __nanosleep(64);  // leave the issue slots to the warp computing it
      if (now_ns() - t0 > w.P->timeout_ns) {
        report_error(*w.P, w.lane, -5, -1);
        w.failed = true;
        return false;
      }
    }
  }
  __threadfence_block();
  __syncwarp();
  trace_route_cache(w, layer, filler);
  return true;
}

MK_INLINE int n_union(const Warp &w) { return w.rc->n_union; }

// Total units of an op over the whole grid.  ROUTED_GU / DOWN need routing.
MK_INLINE int op_total_units(const Warp &w, int type, int layer) {
  const Params &P = *w.P;
  switch (type) {
    case OP_EMBED: return P.n_hb;
    case OP_QKV: return cdiv((P.Hq + 2 * P.Hkv) * P.hd, kRows) * P.qkv_split;
    case OP_ATTN: return w.attn_prefix[P.B];
    case OP_OPROJ: return P.n_hb;
    case OP_SHARED_GU: return P.Fs / kRows;
    case OP_ROUTED_GU: return n_union(w) * (P.F / kRows);
    case OP_DOWN: return (n_union(w) + (P.Fs > 0 ? 1 : 0)) * P.n_db;
    case OP_COMBINE: return P.n_hb;
    case OP_LMHEAD: return cdiv(P.V, kRows);
  }
  return 0;
}

// This warp's units of an op: u0, u0 + stride, ... (n of them).  Attention
// items are CTA-wide; a staged down projection takes CTA-contiguous ranges;
// everything else goes round-robin over the warp slots.
// A staged down projection deals CTA c the contiguous units
// [c * total / n_cta, (c + 1) * total / n_cta), warp by warp within the CTA.
// (cta + 1) * total stays far below 2^31: at most 148 CTAs x 257 segments x
// 1536 row blocks.
MK_INLINE void down_cta_range(const Params &P, int cta, int total, int &c0, int &c1) {
  c0 = (cta * total) / P.n_cta;
  c1 = ((cta + 1) * total) / P.n_cta;
}

MK_INLINE void op_units(const Warp &w, int op, int type, int layer, int &u0, int &stride, int &n) {
  const Params &P = *w.P;
  const int total = op_total_units(w, type, layer);
  if (type == OP_ATTN) {
    u0 = w.cta;
    stride = P.n_cta;
  } else if (type == OP_DOWN && P.down_staged) {
    int c0, c1;
    down_cta_range(P, w.cta, total, c0, c1);
    u0 = c0 + w.wib;
    stride = kConsumers;
    n = c1 > u0 ? (c1 - 1 - u0) / kConsumers + 1 : 0;
    return;
  } else {
    u0 = first_unit_of(w.slot, op, w.nw, type, P.Fs / kRows);
    stride = w.nw;
  }
  n = unit_count_of(u0, total, stride);
}

// Down-projection unit -> segment (routed expert j of the union, 0 .. U-1, or
// the shared expert, U) and row block.
MK_INLINE void down_unit_seg(const Warp &w, int unit, int &seg, int &rb) {
  const Params &P = *w.P;
  seg = unit / P.n_db;
  rb = unit - seg * P.n_db;
}

// QKV unit -> rows [row0, row0 + 4) over tiles [col0, col0 + ntiles * 1024) of
// K: the first (rows / 4) units take the first half of K, the rest the second.
MK_INLINE void qkv_unit(const Params &P, int unit, int &row0, int &col0, int &ntiles, int &half) {
  const int nrb = cdiv((P.Hq + 2 * P.Hkv) * P.hd, kRows);
  const int nt = cdiv(P.d, kTileCols);
  const int h0 = P.qkv_split > 1 ? cdiv(nt, 2) : nt;
  half = unit / nrb;
  row0 = (unit - half * nrb) * kRows;
  col0 = half ? h0 * kTileCols : 0;
  ntiles = half ? nt - h0 : h0;
}

// One QKV output (row m's column i): the sum of its K halves.
MK_INLINE float qkv_load(const Params &P, size_t i) {
  float v = __ldcg(P.qkv + i);
  if (P.qkv_split > 1) v += __ldcg(P.qkv + static_cast<size_t>(kMaxRows) * (P.Hq + 2 * P.Hkv) * P.hd + i);
  return v;
}

// An attention item covers 8 * attn_chunk KV positions of one (sequence,
// kv head, query group); warp `wib` of the CTA takes attn_chunk of them.
struct AttnItem {
  int b, g, qs, c, nch;  // sequence, kv head, query group, CTA chunk, chunks of this sequence
  int pos0, npos, ntiles;  // this warp's positions: [pos0, pos0 + npos), in tiles
};

// Cache index of sequence b's first new row in step `step` of the launch:
// fixed strides for greedy steps, the accepted length so far for verify steps.
MK_INLINE int seq_pos(const Params &P, int b, int step) {
  return P.vpos ? __ldcg(&P.vpos[step * P.B + b]) : __ldg(&P.positions[b]) + step * P.T;
}

// Attention items of one step: per sequence its KV chunks and first item
// (lane 0 computes, the warp reads).
MK_INLINE void attn_layout(const Params &P, int step, int *prefix, int *nch, int lane) {
  if (lane == 0) {
    prefix[0] = 0;
    for (int b = 0; b < kMaxRows; ++b) {
      const int n = b < P.B ? cdiv(seq_pos(P, b, step) + P.T, P.attn_chunk * kConsumers) : 0;
      nch[b] = n;
      prefix[b + 1] = prefix[b] + P.Hkv * P.attn_qsplit * n;
    }
  }
  __syncwarp();
}

MK_INLINE AttnItem attn_item(const Params &P, const int *prefix, const int *nchs, int item, int wib, int step) {
  AttnItem a;
  int b = 0;
  while (b + 1 < P.B && item >= prefix[b + 1]) ++b;
  const int rem = item - prefix[b];
  const int nch = nchs[b];
  a.b = b;
  a.nch = nch;
  a.c = rem % nch;
  a.qs = (rem / nch) % P.attn_qsplit;
  a.g = rem / (nch * P.attn_qsplit);
  const int len = seq_pos(P, b, step) + P.T;
  a.pos0 = a.c * P.attn_chunk * kConsumers + wib * P.attn_chunk;
  a.npos = max(0, min(P.attn_chunk, len - a.pos0));
  a.ntiles = cdiv(a.npos, P.attn_ppt);
  return a;
}

// Tiles of one unit.  Gate/up units stream their gate rows, then their up rows.
MK_INLINE int unit_tiles(const Warp &w, int type, int layer, int unit) {
  const Params &P = *w.P;
  switch (type) {
    case OP_QKV: {
      int row0, col0, nt, half;
      qkv_unit(P, unit, row0, col0, nt, half);
      return nt;
    }
    case OP_LMHEAD: return cdiv(P.d, kTileCols);
    case OP_SHARED_GU:
    case OP_ROUTED_GU: return 2 * cdiv(P.d, kTileCols);
    // the o-projection's tiles, then (with a router) one box of the router's
    // columns of the unit's rows
    case OP_OPROJ: return cdiv(P.Hq * P.hd, kTileCols) + (P.E > 0 ? 1 : 0);
    case OP_DOWN: {
      int seg, rb;
      down_unit_seg(w, unit, seg, rb);
      const int K = seg < n_union(w) ? P.F : P.Fs;
      return cdiv(P.down_groups * cdiv(K, kPanel), kPanels);
    }
    case OP_ATTN: return attn_item(P, w.attn_prefix, w.attn_nch, unit, w.wib, w.step).ntiles;
    default: return 0;
  }
}

// ---------------------------------------------------------------------------
// Producer side: issue the tiles of this warp's next units into free slots.
// ---------------------------------------------------------------------------
// Where the tiles of a GEMV unit come from.
MK_INLINE void unit_source(Warp &w, int type, int layer, int unit) {
  const Params &P = *w.P;
  const CUtensorMap *lm = P.tmaps + layer * MAPS_PER_LAYER;
  int row0 = unit * kRows, col0 = 0, K = P.d, half = 1 << 30, row2 = 0;
  const CUtensorMap *m0 = nullptr, *m2 = nullptr;
  switch (type) {
    case OP_QKV: {
      int nt, kh;
      qkv_unit(P, unit, row0, col0, nt, kh);
      m0 = lm + MAP_WQKV;
      break;
    }
    case OP_OPROJ:
      m0 = lm + MAP_WO;
      m2 = lm + MAP_ROUTER;
      K = P.Hq * P.hd;
      half = cdiv(K, kTileCols);  // the tile after the o-projection's is the router box
      break;
    case OP_LMHEAD: m0 = P.tmaps + P.L * MAPS_PER_LAYER; break;
    case OP_SHARED_GU:
      m0 = lm + MAP_WSGATE;
      m2 = lm + MAP_WSUP;
      row2 = row0;
      half = cdiv(P.d, kTileCols);
      break;
    case OP_ROUTED_GU: {
      const int nfb = P.F / kRows;
      const int e = w.rc->expert[unit / nfb];
      row0 = row2 = e * P.F + (unit % nfb) * kRows;
      m0 = lm + MAP_WGATE;
      m2 = lm + MAP_WUP;
      half = cdiv(P.d, kTileCols);
      break;
    }
    case OP_DOWN: {
      int seg, rb;
      down_unit_seg(w, unit, seg, rb);
      if (seg < n_union(w)) {
        const int e = w.rc->expert[seg];
        m0 = lm + MAP_WDOWN;
        row0 = e * P.d + rb * kRows * P.down_groups;
        K = P.F;
      } else {
        m0 = lm + MAP_WSDOWN;
        row0 = rb * kRows * P.down_groups;
        K = P.Fs;
      }
      break;
    }
    default: break;
  }
  w.um = m0;
  w.um2 = m2;
  w.urow0 = row0;
  w.urow2 = row2;
  w.ucol0 = col0;
  w.uK = K;
  w.uhalf = half;
}

// Issue tile t of the warp's current unit into the next ring slot: its boxes
// as TMA loads completing on the slot's full barrier.
MK_INLINE void issue_tile(Warp &w, int type, int layer, int t) {
  const Params &P = *w.P;
  uint8_t *dst = w.ring + w.islot * kSlotBytes;
  uint64_t *bar = &w.full[w.islot];
  auto expect = [&](uint32_t bytes) {
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar, bytes);
  };
  if (type == OP_ATTN) {
    const AttnItem a = attn_item(P, w.attn_prefix, w.attn_nch, w.iunit, w.wib, w.step);
    const int row = ((layer * P.Bmax + a.b) * P.Hkv + a.g) * P.cap + a.pos0 + t * P.attn_ppt;
    if (w.lane == 0) {
      expect(2u * kKvBoxBytes);
      tma_load_2d(dst, &P.kmap, 0, row, bar, w.pol_kv);
      tma_load_2d(dst + kKvBoxBytes, &P.vmap, 0, row, bar, w.pol_kv);
    }
  } else if (type == OP_OPROJ && t >= w.uhalf) {
    // the router's columns [x, x + 8) of all E rows, x the unit's first row
    // rounded down to 8 (a box of 8 columns x E rows, 16 bytes per row)
    if (w.lane == 0) {
      expect(static_cast<uint32_t>(P.E) * 16u);
      tma_load_2d(dst, w.um2, w.urow0 & ~7, 0, bar, w.pol_w);
    }
  } else if (type == OP_DOWN && P.down_groups > 1) {
    // the unit's boxes run group by group (4 rows each), nbx boxes of 256
    // columns per group; tile t takes boxes 4t .. 4t+3
    const int nbx = cdiv(w.uK, kPanel), nb = P.down_groups * nbx, b0 = t * kPanels;
    const int nbox = min(kPanels, nb - b0);
    // column order for a unit of at most two rows (its consumer keeps both
    // groups' sums at once), group order above
    int seg, rb;
    down_unit_seg(w, w.iunit, seg, rb);
    const bool cols = P.down_cols && (seg < n_union(w) ? __popc(w.rc->rowmask[seg]) : P.M) <= 2;
    if (w.lane == 0) {
      expect(static_cast<uint32_t>(nbox) * kBoxBytes);
      for (int p = 0; p < nbox; ++p) {
        // box b: group b % 2, column b / 2 (column order) or group b / nbx,
        // column b % nbx (group order)
        const int b = b0 + p;
        const int g = cols ? (b & 1) : b / nbx, c = cols ? (b >> 1) : b - g * nbx;
        tma_load_2d(dst + p * kBoxBytes, w.um, c * kPanel, w.urow0 + g * kRows, bar, w.pol_w);
      }
    }
  } else {
    // up to four 4 x 256 boxes side by side; boxes starting past K are skipped
    const bool second = t >= w.uhalf;
    const int tt = second ? t - w.uhalf : t;
    const CUtensorMap *m = second ? w.um2 : w.um;
    const int y = second ? w.urow2 : w.urow0;
    const int x0 = w.ucol0 + tt * kTileCols;
    const int nbox = min(kPanels, cdiv(w.uK - x0, kPanel));
    if (w.lane == 0) {
      expect(static_cast<uint32_t>(nbox) * kBoxBytes);
      for (int p = 0; p < nbox; ++p) tma_load_2d(dst + p * kBoxBytes, m, x0 + p * kPanel, y, bar, w.pol_w);
    }
  }
  w.ephase ^= 1u << w.islot;
  w.filled |= 1u << w.islot;
  w.islot = (w.islot + 1 == w.nslots) ? 0 : w.islot + 1;
}

// Producer: issue the fed consumer's next tiles into its released slots, in
// the order it will take them (the same dealing and tile order as the
// consumer's own loop).  Weights and KV do not depend on this step's
// activations, so the stream runs ahead across ops and layers; it stops only
// at a full ring and where the routing is not known yet.  Returns true if it
// issued a tile or finished the stream.
// Why feed_more stopped without issuing: a full ring, or an input that the
// next tile's address or release depends on.
enum FeedStop : int { FEED_PROGRESS = 0, FEED_RING_FULL = 1, FEED_DEPENDENCY = 2 };

template <bool MULTI>
MK_INLINE int feed_more(Warp &w) {
  const Params &P = *w.P;
  bool progress = false;
  int stop = FEED_DEPENDENCY;
  while (!w.done_issue && !w.failed) {
    if (w.it < w.in_tiles) {  // the next tile of the current unit
      // sleep on the slot's release rather than polling it: a polling warp
      // shares its scheduler (and instruction cache) with the consumer
      if (!mbar_wait_hint(&w.empty[w.islot], (w.ephase >> w.islot) & 1u, 2000u)) {
        stop = FEED_RING_FULL;
        break;
      }
      issue_tile(w, w.itype, w.ilayer, w.it);
      if (kTrace && w.P->trace && w.lane == 0 && w.it == 0 && w.iu == 0) {
        // the op's first tile (one clock read per op: the trace must stay light)
        w.P->trace[(static_cast<size_t>(w.iop) * w.nw + w.slot) * kTraceWords + 8] = now_ns();
      }
      w.it++;
      progress = true;
      continue;
    }
    if (w.in_tiles >= 0) {  // the current unit is issued
      w.iu++;
      w.in_tiles = -1;
      continue;
    }
    if (w.iop >= P.op_end) {
      if (MULTI && w.step + 1 < P.n_steps) {  // the next step of the launch
        w.step++;
        w.epoch++;
        w.iop = P.op_begin;
        w.iop_init = false;
        continue;
      }
      w.done_issue = true;
      progress = true;
      break;
    }
    const int type = op_type_of(w.iop, P.L), layer = op_layer_of(w.iop, P.L);
    if (!op_has_tiles(type)) {
      w.iop++;
      continue;
    }
    if (!w.iop_init) {
      if (type == OP_ATTN && w.lstep != w.step) {
        // a verify step's positions come from the previous step's acceptance:
        // wait (by polling, like the routing) until that step has published
        if (P.vpos && w.step > 0) {
          const uint32_t v = ld_relaxed(P.epoch);
          if (!__all_sync(0xffffffffu, static_cast<int>(v - (w.epoch - 1u)) >= 0)) break;
          (void)ld_acquire(P.epoch);
        }
        attn_layout(P, w.step, w.attn_prefix, w.attn_nch, w.lane);
        w.lstep = w.step;
      }
      if (type == OP_ROUTED_GU || type == OP_DOWN) {
        if (!routing_ready(w, layer)) break;
        if (!route_cache(w, layer)) break;
      }
      int stride;
      op_units(w, w.iop, type, layer, w.iu0, stride, w.in_units);
      w.istride = stride;
      w.iu = 0;
      w.iop_init = true;
    }
    if (w.iu >= w.in_units) {
      if (kTrace && P.trace && w.lane == 0 && w.in_units > 0)  // the op's last tile is out
        P.trace[(static_cast<size_t>(w.iop) * w.nw + w.slot) * kTraceWords + 9] = now_ns();
      w.iop++;
      w.iop_init = false;
      continue;
    }
    w.iunit = w.iu0 + w.iu * w.istride;
    w.it = 0;
    w.in_tiles = unit_tiles(w, type, layer, w.iunit);
    if (type != OP_ATTN) unit_source(w, type, layer, w.iunit);
    w.itype = type;
    w.ilayer = layer;
  }
  return progress || w.done_issue ? FEED_PROGRESS : stop;
}

// ---------------------------------------------------------------------------
// Consumer side
// ---------------------------------------------------------------------------
__device__ __noinline__ bool wait_slot_slow(uint64_t *bar, uint32_t par, unsigned long long timeout_ns) {
  const uint64_t t0 = now_ns();
  for (;;) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, par))) return true;
    int bad = 0;
    if ((threadIdx.x & 31) == 0) bad = (now_ns() - t0 > timeout_ns) ? 1 : 0;
    if (__shfl_sync(0xffffffffu, bad, 0)) return false;
  }
}

// Consumer: wait (bounded) for the next tile of this warp's stream.
MK_INLINE const uint8_t *consume_begin(Warp &w, int op) {
  if (w.failed) return nullptr;
  uint64_t *bar = &w.full[w.cslot];
  const uint32_t par = (w.phase >> w.cslot) & 1u;
  constexpr bool tr = kTrace;
  const uint64_t t0 = tr ? now_ns() : 0;
  if (!__all_sync(0xffffffffu, mbar_try_wait(bar, par)) && !wait_slot_slow(bar, par, w.P->timeout_ns)) {
    set_error(w, -5, op);
    return nullptr;
  }
  if (tr) {
    const uint64_t t1 = now_ns();
    w.tr_wait += t1 - t0;
    if (w.tr_n == 0) w.tr_first = t1;
  }
  return w.ring + w.cslot * kSlotBytes;
}

MK_INLINE void consume_end(Warp &w) {
  if constexpr (kTrace) {
    w.tr_last = now_ns();
    w.tr_n++;
  }
  __syncwarp();  // every lane is done with the slot before it is released
  if (w.lane == 0) mbar_arrive(&w.empty[w.cslot]);
  w.phase ^= (1u << w.cslot);
  w.cslot = (w.cslot + 1 == w.nslots) ? 0 : w.cslot + 1;
}

// Wait for `ctr` to reach `target` (bounded).  Lane 0 polls with acquire
// loads, so the read that sees the target is itself the acquire (no second
// round trip); the __syncwarp after it orders the other lanes' later loads
// behind it.  The error word and the clock are looked at every 8th poll.
MK_INLINE bool wait_counter(Warp &w, const uint32_t *ctr, uint32_t target, int op) {
  const Params &P = *w.P;
  int state = 0;  // 1: reached, 2: another warp reported an error, 3: timed out
  if (w.lane == 0) {
    uint64_t t0 = 0;
    for (int it = 0;; ++it) {
      if (static_cast<int>(ld_acquire(ctr) - target) >= 0) {
        state = 1;
        break;
      }
      if ((it & 7) == 7) {
        if (*reinterpret_cast<volatile const int *>(P.error)) {
          state = 2;
          break;
        }
        const uint64_t t = now_ns();
        if (t0 == 0) {
          t0 = t;
        } else if (t - t0 > P.timeout_ns) {
          state = 3;
          break;
        }
      }
    }
  }
  state = __shfl_sync(0xffffffffu, state, 0);
  __syncwarp();
  if (state == 1) return true;
  if (state == 2) {
    w.failed = true;
    return false;
  }
  set_error(w, -5, op);
  return false;
}

// Producer, before the CTA exits: wait (bounded) until every tile it issued
// for a consumer has landed, consumed or not.  The last fill of slot s
// completes the phase of parity ephase bit s.
MK_INLINE void drain_feed(const Warp &f) {
  for (int s = 0; s < f.nslots; ++s) {
    if (!((f.filled >> s) & 1u)) continue;
    const uint64_t t0 = now_ns();
    while (!mbar_try_wait(&f.full[s], (f.ephase >> s) & 1u)) {
      if (now_ns() - t0 > 50000000ull) break;
    }
  }
}

// Arrive on an op's counter once this warp's units of it are done.  The
// CTA's last warp to arrive publishes for the CTA: after the o-projection it
// first adds the CTA's router-logit sums into the layer's global fixed-point
// sums (and clears them for the next layer).  Returns true (on every lane) for
// the warp whose arrival completed the LMHEAD op grid-wide; other ops' counters
// are bumped without waiting for the reply.
MK_INLINE bool arrive(Warp &w, int op, int type, int layer) {
  const Params &P = *w.P;
  __syncwarp();
  int cta_last = 0;
  if (w.lane == 0) {
    // The warp's results (ordered before this by __syncwarp) are released to
    // the CTA; the CTA's last warp acquires them here and releases them, with
    // its own, grid-wide through the counter (release is cumulative).
    const uint32_t old = atom_add_acq_rel_cta(&w.arrive[op], 1u);  // counts on over the launch's steps
    cta_last = (old % kConsumers == kConsumers - 1) ? 1 : 0;
  }
  cta_last = __shfl_sync(0xffffffffu, cta_last, 0);
  if (!cta_last) return false;
  if (type == OP_OPROJ && P.E > 0) {
    // the CTA's router-logit sums, added into the layer's global ones and
    // cleared for the next layer's o-projection
    long long *dst = P.racc + static_cast<size_t>(layer) * kMaxRows * P.e_ld;
    for (int i = w.lane; i < P.M * P.E; i += 32) {
      const int m = i / P.E, e = i - m * P.E;
      const long long sum = w.rsum[m * P.e_ld + e];
      if (sum != 0) red_add_fix(dst + m * P.e_ld + e, sum);
      w.rsum[m * P.e_ld + e] = 0;
    }
    __syncwarp();
  }
  int last = 0;
  if (w.lane == 0) {
    uint32_t *ctr = &P.counters[op * kCounterStride];
    if (type == OP_LMHEAD) {
      last = (atom_add_acq_rel(ctr, 1u) + 1 == w.epoch * static_cast<uint32_t>(P.n_cta)) ? 1 : 0;
    } else {
      red_add_release(ctr, 1u);
    }
  }
  last = __shfl_sync(0xffffffffu, last, 0);
  if (last) {
    // every lane observes the completed count before reading others' results
    (void)ld_acquire(&P.counters[op * kCounterStride]);
  }
  __syncwarp();
  return last != 0;
}

// Clear this warp's share of a layer's global router-logit sums once every CTA
// has read them (called after the dependency wait of a later op).
MK_INLINE void clear_router_sums(const Warp &w, int layer) {
  const Params &P = *w.P;
  if (P.E == 0) return;
  long long *buf = P.racc + static_cast<size_t>(layer) * kMaxRows * P.e_ld;
  const int n = P.M * P.e_ld;
  for (int i = w.slot * 32 + w.lane; i < n; i += w.nw * 32) buf[i] = 0;
}

// ---------------------------------------------------------------------------
// Activation sources (one lane, 8 consecutive columns, MJ rows)
// ---------------------------------------------------------------------------
// RMSNorm is applied as y = inv_rms * (W (h * g)): the per-row scalar is
// factored out of the dot product and multiplied in the epilogue.  At M > 1
// the gained rows h * g are written next to h by the op that produces h.
// Activation rows are stored panel-permuted: within each 256-column panel,
// columns 8g..8g+3 sit at 4g and columns 8g+4..8g+7 at 128 + 4g, so that the
// 32 lanes' float4 reads (lane g takes columns 8g..8g+7 of a panel) are 16
// bytes apart, free of shared-memory bank conflicts.  Every producer of an
// activation row writes it in this layout, so that a row is staged into shared
// memory by a plain bulk copy.
MK_INLINE int xs_pos4(int c4) {  // float4 slot of columns 4*c4 .. 4*c4+3
  return (c4 & ~63) | ((c4 & 1) << 5) | ((c4 & 63) >> 1);
}
MK_INLINE int xperm(int col) { return 4 * xs_pos4(col >> 2) + (col & 3); }

// The rows' addresses, resolved once per unit: rows past the unit's count
// repeat its first row (their sums are never stored), so every load is
// unconditional and the loads of all rows issue together.  Shared memory rows
// are held as 32-bit shared addresses, global ones as 32-bit offsets from one
// base, to keep the unit's loop light on registers.
MK_INLINE float4 lds_f4(uint32_t a) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
  return v;
}
template <int MJ, bool SH>
struct XPtrs {
  const float *base;  // global rows
  uint32_t ra[MJ];    // shared: byte address of row j; global: float offset of row j from base
  // rows J0 .. J0 + JN - 1
  template <int J0, int JN>
  MK_INLINE void load_part(int col, int K, float (&x)[JN][8]) const {
    if (col < K) {
      const int off = (col & ~(kPanel - 1)) + ((col & (kPanel - 1)) >> 1);
#pragma unroll
      for (int j = 0; j < JN; ++j) {
        float4 a, b;
        if constexpr (SH) {
          a = lds_f4(ra[J0 + j] + 4u * off);
          b = lds_f4(ra[J0 + j] + 4u * (off + kPanel / 2));
        } else {
          const float *pb = base + ra[J0 + j] + off;
          a = __ldca(reinterpret_cast<const float4 *>(pb));
          b = __ldca(reinterpret_cast<const float4 *>(pb + kPanel / 2));
        }
        x[j][0] = a.x; x[j][1] = a.y; x[j][2] = a.z; x[j][3] = a.w;
        x[j][4] = b.x; x[j][5] = b.y; x[j][6] = b.z; x[j][7] = b.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < JN; ++j)
#pragma unroll
        for (int k = 0; k < 8; ++k) x[j][k] = 0.f;
    }
  }
  MK_INLINE void load(int col, int K, float (&x)[MJ][8]) const { load_part<0, MJ>(col, K, x); }
};

// MJ activation rows (row[j] of src, stride ld, n of them), read 8
// consecutive columns per lane: from global memory through L1 (SH false) or
// from the CTA's staged copy in shared memory (SH true).
template <int MJ, bool SH>
struct XRows {
  const float *src;
  int ld;
  int row[MJ];
  int n;
  MK_INLINE XPtrs<MJ, SH> ptrs() const {
    XPtrs<MJ, SH> p;
    p.base = src;
#pragma unroll
    for (int j = 0; j < MJ; ++j) {
      const uint32_t r = static_cast<uint32_t>(j < n ? row[j] : row[0]) * static_cast<uint32_t>(ld);
      p.ra[j] = SH ? saddr(src) + 4u * r : r;
    }
    return p;
  }
};
template <int MJ>
using XPlain = XRows<MJ, false>;
template <int MJ>
using XSmem = XRows<MJ, true>;

// The CTA's staged row at batch 1 (one row) as an XSmem source.
MK_INLINE XSmem<1> staged_row(const float *xs) {
  XSmem<1> x;
  x.src = xs;
  x.ld = 0;
  x.row[0] = 0;
  x.n = 1;
  return x;
}

// Even and odd columns go to separate accumulators (acc, acc2): one packed FMA
// serves both, and each row has two independent FMA chains.
template <int MJ>
MK_INLINE void gemv_panel(const uint8_t *pan, float (&acc)[kRows * MJ], float (&acc2)[kRows * MJ],
                          const float (&x)[MJ][8]) {
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    // each (even, odd) column pair in one packed FMA: acc holds the even
    // columns' partial sums, acc2 the odd ones'
    const uint4 u = ld_shared_v4(pan + r * (kPanel * 2));
    const float2 wp[4] = {bf2(u.x), bf2(u.y), bf2(u.z), bf2(u.w)};
#pragma unroll
    for (int j = 0; j < MJ; ++j) {
      float2 ab = make_float2(acc[r * MJ + j], acc2[r * MJ + j]);
#pragma unroll
      for (int k = 0; k < 4; ++k) ab = fma2(wp[k], make_float2(x[j][2 * k], x[j][2 * k + 1]), ab);
      acc[r * MJ + j] = ab.x;
      acc2[r * MJ + j] = ab.y;
    }
  }
}

// One tile (4 rows x up to four boxes of 256 columns starting at colbase):
// acc[r*MJ + j] += W[r][cols] . x[j][cols] over this lane's columns.
template <int MJ, class XS>
MK_INLINE void gemv_tile(const uint8_t *slot, float (&acc)[kRows * MJ], float (&acc2)[kRows * MJ], int colbase,
                         int K, const XS &xs, int lane) {  // xs: an XPtrs
  const uint8_t *base = slot + lane * 16;
  if constexpr (MJ <= 2) {
    // every panel's activations first: one memory round trip per tile
    float x[kPanels][MJ][8];
#pragma unroll
    for (int p = 0; p < kPanels; ++p) xs.load(colbase + p * kPanel + lane * 8, K, x[p]);
#pragma unroll
    for (int p = 0; p < kPanels; ++p)
      if (colbase + p * kPanel < K) gemv_panel<MJ>(base + p * kBoxBytes, acc, acc2, x[p]);
  } else {
#pragma unroll
    for (int p = 0; p < kPanels; ++p) {
      const int pc = colbase + p * kPanel;
      if (pc >= K) break;
      float x[MJ][8];
      xs.load(pc + lane * 8, K, x);
      gemv_panel<MJ>(base + p * kBoxBytes, acc, acc2, x);
    }
  }
}

// Streams `ntiles` tiles of one unit through the ring into acc (not reduced).
template <int MJ, class XS>
MK_INLINE bool gemv_stream(Warp &w, int op, int ntiles, int col0, int K, const XS &xs, float (&acc)[kRows * MJ]) {
  float acc2[kRows * MJ];  // the odd columns' partial sums
#pragma unroll
  for (int q = 0; q < kRows * MJ; ++q) acc[q] = acc2[q] = 0.f;
  const auto xp = xs.ptrs();
  for (int t = 0; t < ntiles; ++t) {
    const uint8_t *slot = consume_begin(w, op);
    if (!slot) return false;
    gemv_tile<MJ>(slot, acc, acc2, col0 + t * kTileCols, K, xp, w.lane);
    consume_end(w);
  }
#pragma unroll
  for (int q = 0; q < kRows * MJ; ++q) acc[q] += acc2[q];
  return true;
}

// gemv_stream, then the cross-lane reduction: buf[r*MJ + j] = row r . x[j].
template <int MJ, class XS>
MK_INLINE bool gemv_unit(Warp &w, int op, int ntiles, int col0, int K, const XS &xs, float *buf) {
  float acc[kRows * MJ];
  if (!gemv_stream<MJ>(w, op, ntiles, col0, K, xs, acc)) return false;
  butterfly<kRows * MJ>(acc, w.lane);
  butterfly_store<kRows * MJ>(acc, buf, w.lane);
  __syncwarp();
  return true;
}

// A unit of `ngroups` groups of 4 rows over K columns, streamed box by box
// (nbx boxes of 256 columns per group, four boxes per tile); when a group is
// done its 4 x MJ sums are reduced across lanes into buf + g * 4 * MJ.  A
// tile whose four boxes lie in one group runs unrolled with its activations
// loaded first; a tile across two groups goes box by box.
template <int MJ>
MK_INLINE void group_done(float (&acc)[kRows * MJ], float (&acc2)[kRows * MJ], float *buf, int lane) {
#pragma unroll
  for (int q = 0; q < kRows * MJ; ++q) acc[q] += acc2[q];
  butterfly<kRows * MJ>(acc, lane);
  butterfly_store<kRows * MJ>(acc, buf, lane);
#pragma unroll
  for (int q = 0; q < kRows * MJ; ++q) acc[q] = acc2[q] = 0.f;
}

// Two 4-row groups with their boxes in column order: tile t holds (group 0,
// column 2t), (group 1, column 2t), (group 0, column 2t + 1), (group 1,
// column 2t + 1); each column's activations serve both groups.
template <int MJ, class XS>
MK_INLINE bool gemv_two_groups_by_column(Warp &w, int op, int K, const XS &xs, float *buf) {
  const int nbx = cdiv(K, kPanel);
  float a0[kRows * MJ], a0b[kRows * MJ], a1[kRows * MJ], a1b[kRows * MJ];
#pragma unroll
  for (int q = 0; q < kRows * MJ; ++q) a0[q] = a0b[q] = a1[q] = a1b[q] = 0.f;
  const auto xp = xs.ptrs();
  for (int c = 0; c < nbx; c += 2) {
    const uint8_t *slot = consume_begin(w, op);
    if (!slot) return false;
    const uint8_t *base = slot + w.lane * 16;
    float x0[MJ][8], x1[MJ][8];
    xp.load(c * kPanel + w.lane * 8, K, x0);
    const bool two = c + 1 < nbx;
    if (two) xp.load((c + 1) * kPanel + w.lane * 8, K, x1);
    gemv_panel<MJ>(base, a0, a0b, x0);
    gemv_panel<MJ>(base + kBoxBytes, a1, a1b, x0);
    if (two) {
      gemv_panel<MJ>(base + 2 * kBoxBytes, a0, a0b, x1);
      gemv_panel<MJ>(base + 3 * kBoxBytes, a1, a1b, x1);
    }
    consume_end(w);
  }
  group_done<MJ>(a0, a0b, buf, w.lane);
  group_done<MJ>(a1, a1b, buf + kRows * MJ, w.lane);
  __syncwarp();
  return true;
}

template <int MJ, class XS>
MK_INLINE bool gemv_groups(Warp &w, int op, int ngroups, int K, const XS &xs, float *buf) {
  if constexpr (MJ <= 2) {
    if (ngroups == 2 && w.P->down_cols) return gemv_two_groups_by_column<MJ>(w, op, K, xs, buf);
  }
  const int nbx = cdiv(K, kPanel), nb = ngroups * nbx;
  float acc[kRows * MJ], acc2[kRows * MJ];
#pragma unroll
  for (int q = 0; q < kRows * MJ; ++q) acc[q] = acc2[q] = 0.f;
  const auto xp = xs.ptrs();
  for (int b0 = 0; b0 < nb; b0 += kPanels) {
    const uint8_t *slot = consume_begin(w, op);
    if (!slot) return false;
    const uint8_t *base = slot + w.lane * 16;
    const int g0 = b0 / nbx, c0 = b0 - g0 * nbx;
    if (b0 + kPanels <= nb && c0 + kPanels <= nbx) {
      gemv_tile<MJ>(slot, acc, acc2, c0 * kPanel, K, xp, w.lane);
      if (c0 + kPanels == nbx) group_done<MJ>(acc, acc2, buf + g0 * kRows * MJ, w.lane);
    } else {
      for (int q = 0; q < kPanels && b0 + q < nb; ++q) {
        const int b = b0 + q, g = b / nbx, c = b - g * nbx;
        float x[MJ][8];
        xp.load(c * kPanel + w.lane * 8, K, x);
        gemv_panel<MJ>(base + q * kBoxBytes, acc, acc2, x);
        if (c == nbx - 1) group_done<MJ>(acc, acc2, buf + g * kRows * MJ, w.lane);
      }
    }
    consume_end(w);
  }
  __syncwarp();
  return true;
}

// ---------------------------------------------------------------------------
// Ops
// ---------------------------------------------------------------------------
// Lane 4m + r of a GEMV unit's epilogue holds output row r of activation row m.
static_assert(kRows == 4 && kMaxRows * kRows <= 32, "one lane per (row, residual row)");

// New residual rows of whole units, several units per pass when the rows
// leave lanes free: lane = 4 * (g * M + m) + r takes row r of activation row
// m of the pass's g-th unit, so that all of a pass's loads are in flight
// together.  Units are this warp's: slot, slot + nw, ...
template <class F>
MK_INLINE void residual_units(const Params &P, int lane, int slot, int nw, int dbg_layer, const __nv_bfloat16 *gx,
                              F val) {
  const int lanes_per_unit = kRows * P.M, per = 32 / lanes_per_unit;
  const int g = lane / lanes_per_unit, m = (lane / kRows) % P.M, r = lane % kRows;
  for (int base = slot; base < P.n_hb; base += per * nw) {
    const int unit = base + g * nw, row = unit * kRows + r;
    const bool live = g < per && unit < P.n_hb;
    float sq = 0.f;
    if (live && row < P.d) {
      const float hn = val(m, row);
      __stcg(P.h + static_cast<size_t>(m) * P.d + row, hn);
      __stcg(P.xg + static_cast<size_t>(m) * P.ldx + xperm(row), hn * __bfloat162float(gx[row]));
      sq = hn * hn;
      if (dbg_layer >= 0 && P.dbg_hidden)
        P.dbg_hidden[(static_cast<size_t>(dbg_layer) * P.max_rows + m) * P.d + row] = hn;
    }
    sq += __shfl_xor_sync(0xffffffffu, sq, 1);
    sq += __shfl_xor_sync(0xffffffffu, sq, 2);
    if (live && r == 0) red_add_fix(P.ssq + m, to_fix(sq));
  }
  __syncwarp();
}

MK_INLINE void op_embed(Warp &w) {
  const Params &P = *w.P;
  residual_units(P, w.lane, w.slot, w.nw, 0, P.norms[0], [&](int m, int row) {
    // step 0: the given tokens (may alias the argmax output); later steps:
    // the previous step's argmax
    int tok = w.step == 0 ? __ldcg(&P.tokens[m])
              : P.vpos ? __ldcg(&P.vtok[w.step * P.M + m]) : __ldcg(&P.argmax[(w.step - 1) * P.M + m]);
    if (tok < 0 || tok >= P.V) tok = 0;  // rejected at kernel start
    return __bfloat162float(P.embed[static_cast<size_t>(tok) * P.d + row]);
  });
}

// The residual entering the next layer, h = h_mid + the expert outputs'
// fixed-point sum (the routing weights are applied by the down units), its
// sum of squares and x = h * g of the next norm.
MK_INLINE void op_combine(Warp &w, int layer) {
  const Params &P = *w.P;
  const __nv_bfloat16 *gx = (layer + 1 < P.L) ? P.norms[2 * (layer + 1)] : P.final_norm;
  residual_units(P, w.lane, w.slot, w.nw, layer + 1, gx, [&](int m, int row) {
    const size_t i = static_cast<size_t>(m) * P.d + row;
    return __ldcg(P.hm + i) + from_fix(__ldcg(P.hacc + i));
  });
}

template <int MJ>
MK_INLINE void fill_all_rows(int (&row)[MJ], int M) {
#pragma unroll
  for (int j = 0; j < MJ; ++j) row[j] = j < M ? j : 0;
}

// Rows of a routed expert: row[q] = q-th row in `mask`; returns the count.
template <int MJ>
MK_INLINE int rows_of_mask(uint32_t mask, int (&row)[MJ]) {
  int n = 0;
#pragma unroll
  for (int q = 0; q < MJ; ++q) row[q] = 0;
#pragma unroll
  for (int m = 0; m < kMaxRows; ++m) {
    if (mask & (1u << m)) {
#pragma unroll
      for (int q = 0; q < MJ; ++q)
        if (q == n) row[q] = m;
      ++n;
    }
  }
  return n;
}

template <int MJ>
MK_INLINE int row_at(const int (&row)[MJ], int q) {
  int m = 0;
#pragma unroll
  for (int qq = 0; qq < MJ; ++qq)
    if (qq == q) m = row[qq];
  return m;
}

// Dense activations of an op: from the CTA's shared-memory copy (batch 1) or
// from global memory through L1 (more rows).
template <int MJ, bool XS, class Body>
MK_INLINE bool with_dense_x(Warp &w, int type, int layer, const float *xs, Body body) {
  const Params &P = *w.P;
  if constexpr (XS && MJ == 1) {
    return body(staged_row(xs));
  } else if constexpr (XS) {
    // the op's M rows, staged by the CTA with their global row strides
    XSmem<MJ> x;
    x.src = xs;
    x.ld = type == OP_OPROJ ? P.ldo : P.ldx;
    x.n = P.M;
    fill_all_rows<MJ>(x.row, P.M);
    return body(x);
  } else {
    // x = o, or h * g written with h by the op that produced it
    XPlain<MJ> xp;
    xp.src = type == OP_OPROJ ? P.o : P.xg;
    xp.ld = type == OP_OPROJ ? P.ldo : P.ldx;
    xp.n = P.M;
    fill_all_rows<MJ>(xp.row, P.M);
    return body(xp);
  }
}

// The o-projection unit's epilogue.  Lane 4m + r holds row row0 + r of the new
// residual of activation row m (h_mid = h + Wo o): it stores it (with x =
// h_mid * g_ffn, panel-permuted, for the expert GEMVs), its square into the
// sum-of-squares partials, and clears the expert-output accumulator's entry
// for the layer that follows.  With a router, the unit's last ring slot holds
// the router's 8 columns around these rows (all E rows): the unit adds its
// share of the router logits, u[m][e] += sum_r Wr[e][row0 + r] g[row0 + r]
// h_mid[m][row0 + r], into this warp's partial row in shared memory (lane l
// owns experts l, l + 32, ..., so the adds need no atomics and follow the
// warp's unit order).
template <int MJ>
MK_INLINE bool oproj_epilogue(Warp &w, int op, int layer, int unit, int row0, float h_old, float g_row,
                              const float *wb) {
  const Params &P = *w.P;
  const int m = w.lane / kRows, r = w.lane % kRows, row = row0 + r;
  const bool live = w.lane < kRows * P.M && row < P.d;
  float hn = 0.f, gx = 0.f, sq = 0.f;
  if (live) {
    hn = h_old + wb[r * MJ + m];
    gx = hn * g_row;
    const size_t i = static_cast<size_t>(m) * P.d + row;
    __stcg(P.hm + i, hn);
    __stcg(P.xg + static_cast<size_t>(m) * P.ldx + xperm(row), gx);
    __stcg(reinterpret_cast<unsigned long long *>(P.hacc) + i, 0ull);
    sq = hn * hn;
  }
  sq += __shfl_xor_sync(0xffffffffu, sq, 1);
  sq += __shfl_xor_sync(0xffffffffu, sq, 2);
  if (live && r == 0) red_add_fix(P.ssq + kMaxRows + m, to_fix(sq));
  if (P.E == 0) return true;
  const uint8_t *slot = consume_begin(w, op);
  if (!slot) return false;
  // lane l takes experts l, l + 32, ...: rows of 16 bytes, the unit's four
  // columns at byte (row0 & 4) * 2 of each
  const int ne = cdiv(P.E, 32);
#pragma unroll 1
  for (int i = 0; i < ne; ++i) {
    const int e = w.lane + 32 * i;
    const uint2 wr = (e < P.E) ? *reinterpret_cast<const uint2 *>(slot + e * 16 + (row0 & 4) * 2) : make_uint2(0u, 0u);
#pragma unroll
    for (int mm = 0; mm < MJ; ++mm) {
      if (mm >= P.M) break;
      const float x0 = __shfl_sync(0xffffffffu, gx, kRows * mm), x1 = __shfl_sync(0xffffffffu, gx, kRows * mm + 1);
      const float x2 = __shfl_sync(0xffffffffu, gx, kRows * mm + 2), x3 = __shfl_sync(0xffffffffu, gx, kRows * mm + 3);
      float u = bf_lo(wr.x) * x0;
      u = fmaf(bf_hi(wr.x), x1, u);
      u = fmaf(bf_lo(wr.y), x2, u);
      u = fmaf(bf_hi(wr.y), x3, u);
      // integer adds: the CTA's sum does not depend on the warps' order
      if (e < P.E) atomicAdd(reinterpret_cast<unsigned long long *>(&w.rsum[mm * P.e_ld + e]),
                             static_cast<unsigned long long>(to_fix(u)));
    }
  }
  consume_end(w);
  return true;
}

// One unit of a dense GEMV op over all M rows (QKV, OPROJ, LMHEAD).
template <int MMAX, bool XS>
MK_INLINE bool dense_unit(Warp &w, int op, int type, int layer, int unit, const float (&inv)[kMaxRows],
                          const float *xs, float &am_val, int &am_idx) {
  const Params &P = *w.P;
  constexpr int MJ = MMAX;
  float *wb = w.wbuf;
  int row0 = unit * kRows, N = 0, col0 = 0, ntiles = 0, K = P.d, qkv_half = 0;
  switch (type) {
    case OP_OPROJ: K = P.Hq * P.hd; ntiles = cdiv(K, kTileCols); N = P.d; break;
    case OP_QKV: {
      int half;
      qkv_unit(P, unit, row0, col0, ntiles, half);
      N = (P.Hq + 2 * P.Hkv) * P.hd;
      qkv_half = half;
      break;
    }
    default: ntiles = cdiv(P.d, kTileCols); N = P.V; break;
  }
  // lane 4m + r owns output (row0 + r, m); normed ops scale by inv_rms here
  const int m = w.lane / kRows, r = w.lane % kRows;
  const bool live = w.lane < kRows * P.M && row0 + r < N;
  // the o-projection's residual input, loaded before the stream so that its
  // latency hides behind the tiles
  const float h_old = (type == OP_OPROJ && live) ? __ldcg(P.h + static_cast<size_t>(m) * P.d + row0 + r) : 0.f;
  const float g_row = (type == OP_OPROJ && live) ? __bfloat162float(P.norms[2 * layer + 1][row0 + r]) : 0.f;
  const bool ok = with_dense_x<MJ, XS>(w, type, layer, xs, [&](const auto &x) {
    return gemv_unit<MJ>(w, op, ntiles, col0, K, x, wb);
  });
  if (!ok) return false;
  float im = 1.f;
#pragma unroll
  for (int mm = 0; mm < kMaxRows; ++mm)
    if (mm == m) im = inv[mm];
  switch (type) {
    case OP_QKV:
      if (live)
        __stcg(&P.qkv[(static_cast<size_t>(qkv_half) * kMaxRows + m) * (P.Hq + 2 * P.Hkv) * P.hd + row0 + r],
               im * wb[r * MJ + m]);
      break;
    case OP_LMHEAD: {
      const float v = im * wb[r * MJ + m];
      if (live) P.logits[static_cast<size_t>(m) * P.V + row0 + r] = v;
      // running argmax of row m over this warp's rows; lanes 4m..4m+3 hold
      // consecutive rows, so reduce them in row order before lane 4m keeps it
      float bv = live ? v : -INFINITY;
      int bi = live ? row0 + r : 0x7fffffff;
#pragma unroll
      for (int o = 1; o < kRows; o <<= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) {
          bv = ov;
          bi = oi;
        }
      }
      if (r == 0 && (bv > am_val || (bv == am_val && bi < am_idx))) {
        am_val = bv;
        am_idx = bi;
      }
      break;
    }
    case OP_OPROJ:
      if (!oproj_epilogue<MJ>(w, op, layer, unit, row0, h_old, g_row, wb)) return false;
      break;
    default: break;
  }
  __syncwarp();
  return true;
}

// Gate/up unit: 4 rows of the expert's gate and up projections for the rows
// routed to it (shared expert: all rows); writes act = silu(gate) * up.
template <int MJ, bool XS>
MK_INLINE bool gu_unit(Warp &w, int op, int type, int layer, int unit, const float (&inv)[kMaxRows],
                       const float *xs) {
  const Params &P = *w.P;
  XPlain<MJ> xn;  // x = h * g, written with h by the o-projection
  xn.src = P.xg;
  xn.ld = P.ldx;
  float *dst;
  int ld, f0;
  if (type == OP_ROUTED_GU) {
    const int nfb = P.F / kRows, j = unit / nfb;
    f0 = (unit % nfb) * kRows;
    xn.n = rows_of_mask<MJ>(w.rc->rowmask[j], xn.row);
    dst = P.act_routed + static_cast<size_t>(j) * kMaxRows * P.ldf;
    ld = P.ldf;
  } else {
    f0 = unit * kRows;
    xn.n = P.M;
    fill_all_rows<MJ>(xn.row, P.M);
    dst = P.act_shared;
    ld = P.ldfs;
  }
  const int half = cdiv(P.d, kTileCols);
  float *wb = w.wbuf;
  // gate rows, then up rows: one rolled loop, one copy of the stream code
  if constexpr (XS) {
    // the rows staged by SHARED_GU (all M rows, stride ldx)
    XSmem<MJ> x;
    x.src = xs;
    x.ld = P.ldx;
    x.n = xn.n;
#pragma unroll
    for (int j = 0; j < MJ; ++j) x.row[j] = xn.row[j];
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh)
      if (!gemv_unit<MJ>(w, op, half, 0, P.d, x, wb + hh * kRows * MJ)) return false;
  } else {
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh)
      if (!gemv_unit<MJ>(w, op, half, 0, P.d, xn, wb + hh * kRows * MJ)) return false;
  }
  const int q = w.lane / kRows, r = w.lane % kRows;
  if (w.lane < kRows * xn.n) {
    const int m = row_at<MJ>(xn.row, q);
    float im = 0.f;
#pragma unroll
    for (int mm = 0; mm < kMaxRows; ++mm)
      if (mm == m) im = inv[mm];
    const float g = im * wb[r * MJ + q], u = im * wb[kRows * MJ + r * MJ + q];
    __stcg(dst + static_cast<size_t>(m) * ld + xperm(f0 + r), silu(g) * u);
  }
  __syncwarp();
  return true;
}

// One down-projection unit: segment (routed expert j, or the shared expert
// when j == n_union) x 4 or 8 output rows, for every row m the segment serves.
template <int MJ, bool XS>
MK_INLINE bool down_unit(Warp &w, int op, int layer, int unit, const float *xsm) {
  const Params &P = *w.P;
  int seg, rb;
  down_unit_seg(w, unit, seg, rb);
  const int row0 = rb * kRows * P.down_groups;
  const int U = n_union(w);
  const RouteCache *rt = w.rc;
  XPlain<MJ> xs;
  int K;
  if (seg < U) {
    xs.src = P.act_routed + static_cast<size_t>(seg) * kMaxRows * P.ldf;
    xs.ld = P.ldf;
    xs.n = rows_of_mask<MJ>(rt->rowmask[seg], xs.row);
    K = P.F;
  } else {
    xs.src = P.act_shared;
    xs.ld = P.ldfs;
    xs.n = P.M;
    fill_all_rows<MJ>(xs.row, P.M);
    K = P.Fs;
  }
  float *wb = w.wbuf;
  bool ok;
  if constexpr (XS) {
    if (P.down_staged) {
      // the CTA staged its experts' activation rows: slot seg - dseg0 of the
      // staged block holds rows 0..M-1 of the segment at their global stride
      XSmem<MJ> xst;
      xst.src = xsm + (seg - w.dseg0) * P.M * panel_ld(max(P.F, P.Fs));
      xst.ld = xs.ld;
      xst.n = xs.n;
#pragma unroll
      for (int j = 0; j < MJ; ++j) xst.row[j] = xs.row[j];
      ok = gemv_groups<MJ>(w, op, P.down_groups, K, xst, wb);
    } else {
      ok = gemv_groups<MJ>(w, op, P.down_groups, K, xs, wb);
    }
  } else {
    ok = gemv_groups<MJ>(w, op, P.down_groups, K, xs, wb);
  }
  if (!ok) return false;
  // add w * y (w the row's routing weight, 1 for the shared expert) into the
  // fixed-point sum of the expert outputs of row m
  const int q = w.lane / kRows, r = w.lane % kRows;
  if (w.lane < kRows * xs.n) {
    const int m = row_at<MJ>(xs.row, q);
    const float wgt = (seg < U) ? rt->row_w[m][rt->kslot[seg][m]] : 1.f;
    long long *dst = P.hacc + static_cast<size_t>(m) * P.d + row0 + r;
    for (int g = 0; g < P.down_groups; ++g)
      if (row0 + g * kRows + r < P.d) red_add_fix(dst + g * kRows, to_fix(wgt * wb[(g * kRows + r) * MJ + q]));
  }
  __syncwarp();
  return true;
}

template <int MMAX, bool XS>
MK_INLINE bool routed_dispatch(Warp &w, int op, int type, int layer, int unit, const float (&inv)[kMaxRows],
                               const float *xs) {
  const Params &P = *w.P;
  int cnt;
  if (type == OP_ROUTED_GU) {
    cnt = __popc(w.rc->rowmask[unit / (P.F / kRows)]);
  } else if (type == OP_DOWN) {
    int seg, rb;
    down_unit_seg(w, unit, seg, rb);
    cnt = seg < n_union(w) ? __popc(w.rc->rowmask[seg]) : P.M;
  } else {
    cnt = P.M;  // shared gate/up
  }
#define MK_DISPATCH(MJ_)                                      \
  return (type == OP_DOWN) ? down_unit<MJ_, XS>(w, op, layer, unit, xs) \
                           : gu_unit<MJ_, XS>(w, op, type, layer, unit, inv, xs)
  if (cnt <= 1) {
    MK_DISPATCH(1);
  }
  if constexpr (MMAX >= 2) {
    if (cnt <= 2) {
      MK_DISPATCH(2);
    }
  }
  if constexpr (MMAX >= 4) {
    if (cnt <= 4) {
      MK_DISPATCH(4);
    }
  }
  if constexpr (MMAX >= 8) {
    MK_DISPATCH(8);
  }
#undef MK_DISPATCH
  return false;
}

// --- attention ---------------------------------------------------------------
// Lane layout of an attention warp: lane = 8 * pg + dl.  A tile is read in
// groups of four consecutive positions, pg picking one of them; dl owns the
// head dimensions [c*dl, c*dl + c) and [hd/2 + c*dl, hd/2 + c*dl + c) with
// c = hd / 16, which are exactly rotate-half RoPE pairs, so q's rotation stays
// in the lane.  A score is reduced over the 8 dl lanes only; the kQvp = 4
// query vectors of the item end up one per lane pair (query dl / 2).

// c consecutive bf16 values (c = 16, 8 or 4) from shared memory, as c / 2
// (even, odd) float pairs.
template <int C>
MK_INLINE void lds_bf16x2(const __nv_bfloat16 *p, float2 (&f)[C / 2]) {
  static_assert(C == 16 || C == 8 || C == 4, "8 or 16 values of a 64- or 128-wide head");
  if constexpr (C == 16) {
    const uint4 u = ld_shared_v4(p), u2 = ld_shared_v4(p + 8);
    f[0] = bf2(u.x);
    f[1] = bf2(u.y);
    f[2] = bf2(u.z);
    f[3] = bf2(u.w);
    f[4] = bf2(u2.x);
    f[5] = bf2(u2.y);
    f[6] = bf2(u2.z);
    f[7] = bf2(u2.w);
  } else if constexpr (C == 8) {
    const uint4 u = ld_shared_v4(p);
    f[0] = bf2(u.x);
    f[1] = bf2(u.y);
    f[2] = bf2(u.z);
    f[3] = bf2(u.w);
  } else {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    f[0] = bf2(u.x);
    f[1] = bf2(u.y);
  }
}

// Four partial scores (one per query) summed over the 8 dl lanes of a
// position: the lane keeps query dl / 2's full score.
MK_INLINE float reduce_scores8(const float (&p)[kQvp], int dl) {
  const bool up4 = (dl & 4) != 0, up2 = (dl & 2) != 0;
  float k0 = up4 ? p[2] : p[0], k1 = up4 ? p[3] : p[1];
  const float s0 = up4 ? p[0] : p[2], s1 = up4 ? p[1] : p[3];
  k0 += __shfl_xor_sync(0xffffffffu, s0, 4);
  k1 += __shfl_xor_sync(0xffffffffu, s1, 4);
  float k = up2 ? k1 : k0;
  k += __shfl_xor_sync(0xffffffffu, up2 ? k0 : k1, 2);
  k += __shfl_xor_sync(0xffffffffu, k, 1);
  return k;
}

// Shared-memory scratch of the attention items of one CTA.
struct AttnShared {
  float *o;           // [compute warps][kQvp][hd] partials (the staging row's space)
  float *q;           // [kQvp][hd] the item's query vectors, rotated and scaled
  __nv_bfloat16 *kn;  // [kMaxRows][hd] this step's new keys (rotated, bf16) inside the item's chunk
  __nv_bfloat16 *vn;  // [kMaxRows][hd] and values (bf16)
  float *ml;          // [compute warps][kQvp][2]
  uint32_t *rdv;      // rendezvous counter
  uint32_t *seq;      // this warp's rendezvous count
};

// One warp's share of an item: online softmax over its positions for the
// item's kQvp query vectors; the unnormalised o, the running max and the sum
// go to the CTA's scratch at warp slot wib.  The item's code runs once per
// layer, so its loops are kept rolled: fewer distinct instructions to fetch.
template <int HD>
MK_INLINE bool attn_warp(Warp &w, int op, int layer, const AttnItem &a, AttnShared &sh) {
  const Params &P = *w.P;
  constexpr int C = HD / 16, DL = 2 * C, HALF = HD / 2, QVP = kQvp;
  constexpr int NS = kKvBoxBytes / (2 * HD) / 4;  // groups of four positions per tile
  static_assert(QVP == 4, "one query vector per lane pair");
  const int G = P.Hq / P.Hkv;
  const int pos_b = seq_pos(P, a.b, w.step);
  const int lane = w.lane, pg = lane >> 3, dl = lane & 7, myq = dl >> 1;
  const int d0 = C * dl, d1 = HALF + C * dl;
  float m_run = -INFINITY, l_run = 0.f;
  constexpr int DP = DL / 2, CP = C / 2;  // float pairs per lane and per chunk
  // P.V runs on another lane layout: lane (vq, dc) = (lane >> 3, lane & 7)
  // accumulates query vq's output on dims [DL dc, DL dc + DL)
  const int vq = lane >> 3, dc = lane & 7;
  float2 ov[DP];
#pragma unroll
  for (int k = 0; k < DP; ++k) ov[k] = make_float2(0.f, 0.f);
  if (a.ntiles > 0) {
    // the item's query vectors, staged by the CTA: this lane's dimensions
    float2 q[QVP][DP];
#pragma unroll
    for (int v = 0; v < QVP; ++v) {
#pragma unroll
      for (int k = 0; k < CP; k += 2) {
        const float4 x1 = *reinterpret_cast<const float4 *>(sh.q + v * HD + d0 + 2 * k);
        const float4 x2 = *reinterpret_cast<const float4 *>(sh.q + v * HD + d1 + 2 * k);
        q[v][k] = make_float2(x1.x, x1.y);
        q[v][k + 1] = make_float2(x1.z, x1.w);
        q[v][CP + k] = make_float2(x2.x, x2.y);
        q[v][CP + k + 1] = make_float2(x2.z, x2.w);
      }
    }
    // last position query myq may see (-1: no such query vector)
    const int my_qv = a.qs * QVP + myq;
    const int lim = my_qv < G * P.T ? pos_b + my_qv / G : -1;
    const int end = a.pos0 + a.npos;
    for (int tt = 0; tt < a.ntiles; ++tt) {
      uint8_t *slot = const_cast<uint8_t *>(consume_begin(w, op));
      if (!slot) return false;
      const int pos0 = a.pos0 + tt * P.attn_ppt;
      __nv_bfloat16 *ks = reinterpret_cast<__nv_bfloat16 *>(slot);
      __nv_bfloat16 *vs = reinterpret_cast<__nv_bfloat16 *>(slot + kKvBoxBytes);
      // New positions of this step inside the tile: patch the tile with the
      // rotated, bf16-rounded rows the item staged (16 lanes per row each)
      const int lo = max(pos0, pos_b), hi = min(pos0 + P.attn_ppt, pos_b + P.T);
      for (int p = lo; p < hi; ++p) {
        const int t = p - pos_b, r = (p - pos0) * HD;
        constexpr int V16 = HD / 8;  // 16-byte pieces per row
        if (lane < 2 * V16) {
          const int j = lane % V16;
          const uint4 *srow = reinterpret_cast<const uint4 *>((lane < V16 ? sh.kn : sh.vn) + t * HD);
          reinterpret_cast<uint4 *>((lane < V16 ? ks : vs) + r)[j] = srow[j];
        }
      }
      if (lo < hi) fence_proxy_async_smem();
      __syncwarp();
      // scores, two groups of four positions per iteration: lane (pg, dl)
      // gets position pos0 + 4s + pg for query myq; results enter sc at the end
      float sc[NS];
#pragma unroll
      for (int s = 0; s < NS; s += 2) {
        float x[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const __nv_bfloat16 *kr = ks + (4 * (s + h) + pg) * HD;
          float2 k1[CP], k2[CP];
          lds_bf16x2<C>(kr + d0, k1);
          lds_bf16x2<C>(kr + d1, k2);
          float part[QVP];
#pragma unroll
          for (int v = 0; v < QVP; ++v) {
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < CP; ++k) acc = fma2(q[v][k], k1[k], acc);
#pragma unroll
            for (int k = 0; k < CP; ++k) acc = fma2(q[v][CP + k], k2[k], acc);
            part[v] = acc.x + acc.y;
          }
          x[h] = reduce_scores8(part, dl);
        }
#pragma unroll
        for (int r = 0; r + 2 < NS; ++r) sc[r] = sc[r + 2];
        sc[NS - 2] = x[0];
        sc[NS - 1] = x[1];
      }
      // online softmax over the tile (per query: the 4 pg lanes x NS groups)
      float mt = -INFINITY;
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        const int pos = pos0 + 4 * s + pg;
        if (!(pos <= lim && pos < end)) sc[s] = -INFINITY;
        mt = fmaxf(mt, sc[s]);
      }
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
      mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
      const float m_new = fmaxf(m_run, mt);
      const float alpha = (m_run == -INFINITY) ? 0.f : expf(m_run - m_new);
      float ps = 0.f;
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        sc[s] = (sc[s] == -INFINITY) ? 0.f : expf(sc[s] - m_new);
        ps += sc[s];
      }
      ps += __shfl_xor_sync(0xffffffffu, ps, 8);
      ps += __shfl_xor_sync(0xffffffffu, ps, 16);
      l_run = l_run * alpha + ps;
      m_run = m_new;
      // rescale query vq's output (alpha is the same on every lane of a query)
      const float av = __shfl_sync(0xffffffffu, alpha, 2 * vq);
      if (__any_sync(0xffffffffu, av != 1.f)) {
#pragma unroll
        for (int k = 0; k < DP; ++k) ov[k] = mul2(ov[k], make_float2(av, av));
      }
      // o[vq] += p(position, vq) * V[position]: position 4s + g's probability
      // for query vq sits on lane (g, 2 vq) in sc[s]
#pragma unroll
      for (int s2 = 0; s2 < NS; ++s2) {
#pragma unroll
        for (int g4 = 0; g4 < 4; ++g4) {
          const float pv = __shfl_sync(0xffffffffu, sc[s2], g4 * 8 + 2 * vq);
          const __nv_bfloat16 *vr = vs + (4 * s2 + g4) * HD + DL * dc;
          float2 vv[DP];
          lds_bf16x2<DL>(vr, vv);
          const float2 pp = make_float2(pv, pv);
#pragma unroll
          for (int k = 0; k < DP; ++k) ov[k] = fma2(pp, vv[k], ov[k]);
        }
      }
      consume_end(w);
    }
  }
  // this warp's share of query vq's output: dims [DL dc, DL dc + DL)
  float *so = sh.o + (w.wib * QVP + vq) * HD + DL * dc;
#pragma unroll
  for (int k = 0; k < DP; ++k) {
    so[2 * k] = ov[k].x;
    so[2 * k + 1] = ov[k].y;
  }
  if (pg == 0 && (dl & 1) == 0) {
    sh.ml[(w.wib * QVP + myq) * 2] = m_run;
    sh.ml[(w.wib * QVP + myq) * 2 + 1] = l_run;
  }
  return true;
}

MK_INLINE bool cta_rendezvous(Warp &w, uint32_t *cnt, uint32_t target, int op);

// Final merge of one query vector over the nch CTA partials of its group:
// o = sum_i e^(m_i - M) o_i / sum_i e^(m_i - M) l_i  (one lane per partial for
// (m, l); the o partials are read 8 at a time, all in flight together).
template <int DPL>
MK_INLINE void attn_final_merge(const Params &P, int lane, int grp, int v, int nch, int b, int g) {
  constexpr int hd = 32 * DPL, B = 16;  // partials loaded per batch, all in flight with (m, l)
  const int G = P.Hq / P.Hkv;
  const int qv = (grp % P.attn_qsplit) * kQvp + v;
  if (qv >= G * P.T) return;
  const float *mrow = P.attn_ml + (static_cast<size_t>(grp) * kQvp + v) * 2 * P.attn_nch_max;
  const float *obase = P.attn_o + (static_cast<size_t>(grp) * P.attn_nch_max * kQvp + v) * hd + lane * DPL;
  const size_t ostride = static_cast<size_t>(kQvp) * hd;  // one CTA partial to the next
  const float mi = lane < nch ? __ldcg(mrow + lane) : -INFINITY;
  const float li = lane < nch ? __ldcg(mrow + P.attn_nch_max + lane) : 0.f;
  float val[B][DPL];
#pragma unroll
  for (int k = 0; k < B; ++k)
#pragma unroll
    for (int dd = 0; dd < DPL; ++dd) val[k][dd] = (k < nch) ? __ldcg(obase + k * ostride + dd) : 0.f;
  const float M = warp_max(mi);
  const float wi = (lane < nch && mi != -INFINITY) ? expf(mi - M) : 0.f;
  const float L = warp_sum(wi * li);
  float acc[DPL];
#pragma unroll
  for (int dd = 0; dd < DPL; ++dd) acc[dd] = 0.f;
  for (int i0 = 0; i0 < nch; i0 += B) {
    if (i0 > 0) {
#pragma unroll
      for (int k = 0; k < B; ++k)
#pragma unroll
        for (int dd = 0; dd < DPL; ++dd) val[k][dd] = (i0 + k < nch) ? __ldcg(obase + (i0 + k) * ostride + dd) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < B; ++k) {
      const float wv = __shfl_sync(0xffffffffu, wi, (i0 + k) & 31);
#pragma unroll
      for (int dd = 0; dd < DPL; ++dd) acc[dd] = fmaf(wv, val[k][dd], acc[dd]);
    }
  }
  const int t = qv / G, head = g * G + qv % G, m = b * P.T + t;
  const float invl = 1.0f / L;
  // o is stored panel-permuted: this lane's DPL columns (2 or 4, aligned to
  // their count) stay together within one float4 slot
  const int col = head * hd + lane * DPL;
  float *dst = P.o + static_cast<size_t>(m) * P.ldo + xperm(col);
  if constexpr (DPL == 4) {
    __stcg(reinterpret_cast<float4 *>(dst), make_float4(acc[0] * invl, acc[1] * invl, acc[2] * invl, acc[3] * invl));
  } else {
#pragma unroll
    for (int dd = 0; dd < DPL; ++dd) __stcg(dst + dd, acc[dd] * invl);
  }
}

// One CTA-wide attention item: every warp computes its share, warp v (v < 4)
// merges the warps' shares of query vector v into the CTA's partial, and the
// warp that completes the count of (group, v) merges all CTA partials into o.
template <int DPL>
MK_INLINE bool attn_unit(Warp &w, int op, int layer, int item, AttnShared &sh) {
  const Params &P = *w.P;
  constexpr int hd = 32 * DPL;
  const AttnItem a = attn_item(P, w.attn_prefix, w.attn_nch, item, w.wib, w.step);
  {
    // the item's query vectors, once per CTA: warp v rotates (rotate-half
    // pairs (i, i + hd/2) over its lanes) and scales query vector v
    static_assert(kConsumers == kQvp, "one query vector per compute warp");
    constexpr int HALF = hd / 2;
    const int v = w.wib, qv = a.qs * kQvp + v, G = P.Hq / P.Hkv;
    float *dst = sh.q + v * hd;
    if (qv < G * P.T) {
      const int t = qv / G, head = a.g * G + qv % G, m = a.b * P.T + t, p = seq_pos(P, a.b, w.step) + t;
      const size_t src = static_cast<size_t>(m) * (P.Hq + 2 * P.Hkv) * hd + head * hd;
      const float scale = 1.0f / sqrtf(static_cast<float>(hd));
      float x1[HALF / 32], x2[HALF / 32];
      float2 cs[HALF / 32];
#pragma unroll
      for (int j = 0; j < HALF / 32; ++j) {
        const int i = w.lane + 32 * j;
        x1[j] = qkv_load(P, src + i);
        x2[j] = qkv_load(P, src + i + HALF);
        cs[j] = __ldg(&P.rope[static_cast<size_t>(p) * HALF + i]);
      }
#pragma unroll
      for (int j = 0; j < HALF / 32; ++j) {
        const int i = w.lane + 32 * j;
        dst[i] = (x1[j] * cs[j].x - x2[j] * cs[j].y) * scale;
        dst[i + HALF] = (x2[j] * cs[j].x + x1[j] * cs[j].y) * scale;
      }
    } else {
      for (int i = w.lane; i < hd; i += 32) dst[i] = 0.f;
    }
    // This step's new rows that fall in the item's chunk: rotate k, round k
    // and v to bf16, keep them for the tile patches and (one query group)
    // append them to the cache.  Warp v takes new rows v, v + 4, ...
    const int pos_b = seq_pos(P, a.b, w.step);
    const int c0 = a.c * P.attn_chunk * kConsumers;
    const int lo = max(c0, pos_b), hi = min(c0 + P.attn_chunk * kConsumers, pos_b + P.T);
    const int W3 = (P.Hq + 2 * P.Hkv) * hd;
    for (int p = lo + w.wib; p < hi; p += kConsumers) {
      const int t = p - pos_b, m = a.b * P.T + t;
      const size_t kq = static_cast<size_t>(m) * W3 + (P.Hq + a.g) * hd;
      const size_t vq = static_cast<size_t>(m) * W3 + (P.Hq + P.Hkv + a.g) * hd;
      float x1[HALF / 32], x2[HALF / 32], y1[HALF / 32], y2[HALF / 32];
      float2 cs[HALF / 32];
#pragma unroll
      for (int j = 0; j < HALF / 32; ++j) {  // every load of the row in flight at once
        const int i = w.lane + 32 * j;
        x1[j] = qkv_load(P, kq + i);
        x2[j] = qkv_load(P, kq + i + HALF);
        y1[j] = qkv_load(P, vq + i);
        y2[j] = qkv_load(P, vq + i + HALF);
        cs[j] = __ldg(&P.rope[static_cast<size_t>(p) * HALF + i]);
      }
      const size_t crow = (((static_cast<size_t>(layer) * P.Bmax + a.b) * P.Hkv + a.g) * P.cap + p) * hd;
#pragma unroll
      for (int j = 0; j < HALF / 32; ++j) {
        const int i = w.lane + 32 * j;
        const __nv_bfloat16 k1 = __float2bfloat16_rn(x1[j] * cs[j].x - x2[j] * cs[j].y);
        const __nv_bfloat16 k2 = __float2bfloat16_rn(x2[j] * cs[j].x + x1[j] * cs[j].y);
        const __nv_bfloat16 v1 = __float2bfloat16_rn(y1[j]), v2 = __float2bfloat16_rn(y2[j]);
        sh.kn[t * hd + i] = k1;
        sh.kn[t * hd + i + HALF] = k2;
        sh.vn[t * hd + i] = v1;
        sh.vn[t * hd + i + HALF] = v2;
        if (a.qs == 0) {
          P.kc[crow + i] = k1;
          P.kc[crow + i + HALF] = k2;
          P.vc[crow + i] = v1;
          P.vc[crow + i + HALF] = v2;
        }
      }
    }
    *sh.seq += kConsumers;
    if (!cta_rendezvous(w, sh.rdv, *sh.seq, op)) return false;
  }
  if (!attn_warp<hd>(w, op, layer, a, sh)) return false;
  *sh.seq += kConsumers;
  if (!cta_rendezvous(w, sh.rdv, *sh.seq, op)) return false;
  const int grp = (a.b * P.Hkv + a.g) * P.attn_qsplit + a.qs;
  if (w.wib < kQvp) {
    const int v = w.wib;
    float mw[kConsumers], M = -INFINITY;
#pragma unroll
    for (int k = 0; k < kConsumers; ++k) {
      mw[k] = sh.ml[(k * kQvp + v) * 2];
      M = fmaxf(M, mw[k]);
    }
    float L = 0.f, acc[DPL];
#pragma unroll
    for (int dd = 0; dd < DPL; ++dd) acc[dd] = 0.f;
#pragma unroll
    for (int k = 0; k < kConsumers; ++k) {
      const float e = (mw[k] == -INFINITY) ? 0.f : expf(mw[k] - M);
      L += e * sh.ml[(k * kQvp + v) * 2 + 1];
#pragma unroll
      for (int dd = 0; dd < DPL; ++dd) acc[dd] = fmaf(e, sh.o[(k * kQvp + v) * hd + w.lane * DPL + dd], acc[dd]);
    }
    float *dop = P.attn_o + ((static_cast<size_t>(grp) * P.attn_nch_max + a.c) * kQvp + v) * hd + w.lane * DPL;
#pragma unroll
    for (int dd = 0; dd < DPL; ++dd) __stcg(dop + dd, acc[dd]);
    if (w.lane == 0) {
      float *ml = P.attn_ml + (static_cast<size_t>(grp) * kQvp + v) * 2 * P.attn_nch_max;
      __stcg(ml + a.c, M);
      __stcg(ml + P.attn_nch_max + a.c, L);
    }
    // count this CTA's partial of query v; the warp that completes the
    // (group, v) count merges all of them into o and rewinds the counter.
    // Lane 0's acq_rel add releases the warp's partial (ordered before it by
    // __syncwarp) and, for the last arrival, acquires every other CTA's; the
    // second __syncwarp orders the other lanes' loads behind it.
    uint32_t *cnt = P.attn_cnt + static_cast<size_t>(grp) * kQvp + v;
    __syncwarp();
    int last = 0;
    if (w.lane == 0) last = (atom_add_acq_rel(cnt, 1u) + 1 == static_cast<uint32_t>(a.nch)) ? 1 : 0;
    last = __shfl_sync(0xffffffffu, last, 0);
    __syncwarp();
    if (last) {
      attn_final_merge<DPL>(P, w.lane, grp, v, a.nch, a.b, a.g);
      __syncwarp();
      if (w.lane == 0) *cnt = 0;
    }
  }
  // No CTA barrier here: a next item's query staging ends in one (before any
  // warp overwrites the partials), and the next op waits for every CTA's arrival.
  return true;
}

// --- the final argmax (run by the LMHEAD op's last arriving warp) -----------
__device__ __noinline__ void final_argmax(const Params &P, int lane, uint32_t epoch, int step) {
  for (int m = 0; m < P.M; ++m) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int s = lane; s < P.n_warps; s += 32) {
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
      const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == 0) P.argmax[step * P.M + m] = (bi == 0x7fffffff) ? 0 : bi;
  }
  __syncwarp();
  if (P.vpos) {
    // Verify step: sequence b (one lane each) accepts its block's drafts while
    // each equals the argmax of the row before it, plus one token; the next
    // block starts after the accepted tokens with the last of them, then the
    // drafts proposed for the positions that follow.
    const int T = P.T;
    const int *am = P.argmax + step * P.M;
    for (int b = lane; b < P.B; b += 32) {
      const int base = b * T;
      const int *blk = step == 0 ? P.tokens + base : P.vtok + step * P.M + base;
      int a = 1;
      while (a < T && __ldcg(&blk[a]) == __ldcg(&am[base + a - 1])) ++a;
      P.out_accepted[step * P.B + b] = a;
      for (int t = 0; t < T; ++t) P.out_tokens[step * P.M + base + t] = t < a ? __ldcg(&am[base + t]) : -1;
      const int p_next = __ldcg(&P.vpos[step * P.B + b]) + a, p0 = __ldg(&P.positions[b]);
      P.vpos[(step + 1) * P.B + b] = p_next;
      int *nb = P.vtok + (step + 1) * P.M + base;
      nb[0] = __ldcg(&am[base + a - 1]);
      for (int t = 1; t < T; ++t) {
        const int j = p_next - p0 + t;  // < draft_len: n_steps * T <= draft_len is checked by the host
        nb[t] = j < P.draft_len ? __ldg(&P.drafts[static_cast<size_t>(b) * P.draft_len + j]) : 0;
      }
    }
    __syncwarp();
  }
  if (lane < P.M) P.ssq[lane] = 0;  // the entering residual's sums, read by LMHEAD
  __syncwarp();
  if (lane == 0) {
    __threadfence();
    st_release(P.epoch, epoch);
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
// Bounded CTA-wide rendezvous on a shared-memory counter.  Not bar.sync: a
// warp that leaves on an error must not strand the others, and this wait ends
// on the timeout or on the error word.
MK_INLINE bool cta_rendezvous(Warp &w, uint32_t *cnt, uint32_t target, int op) {
  __syncwarp();
  if (w.lane == 0) {
    __threadfence_block();
    atomicAdd(cnt, 1u);
  }
  uint64_t t0 = 0;
  for (int it = 0;; ++it) {
    const uint32_t v = *reinterpret_cast<volatile uint32_t *>(cnt);
    if (__all_sync(0xffffffffu, v >= target)) break;
    if ((it & 31) == 31) {
      int bad = 0;
      if (w.lane == 0) {
        const uint64_t t = now_ns();
        if (t0 == 0) t0 = t;
        bad = (t - t0 > w.P->timeout_ns || *reinterpret_cast<volatile const int *>(w.P->error) != 0) ? 1 : 0;
      }
      if (__shfl_sync(0xffffffffu, bad, 0)) {
        set_error(w, -5, op);
        return false;
      }
    }
  }
  __threadfence_block();
  __syncwarp();
  return true;
}

// ---- batch 1: the op's activation row staged in shared memory --------------
// The rows live in global memory in the panel-permuted layout XSmem reads, so
// a CTA stages one with a plain bulk copy.  The first compute warp of the CTA
// past the op's dependency wait issues the copies (one mbarrier, expecting
// their bytes); every compute warp then waits for that barrier's phase.  The
// copies may overwrite shared memory that the previous staged op read: every
// op that stages waits (directly or through its dependencies) for the
// completion of the op that last used the row, so no warp of the CTA still
// reads it.
struct StageCtl {
  uint64_t bar;    // completes once per staging, when the copies have landed
  uint32_t elect;  // staging arrivals; the first of each kConsumers issues
};

MK_INLINE void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   saddr(dst)),
               "l"(src), "r"(bytes), "r"(saddr(bar))
               : "memory");
}

// Stage `n` rows: row i (bytes[i] bytes, a multiple of 16) from src[i] to
// xs + off[i] floats.  All four compute warps call it in the same order;
// w.xphase counts the stagings.
MK_INLINE bool stage_rows(Warp &w, StageCtl *sc, float *xs, const float *const *src, const uint32_t *bytes,
                          const int *off, int n, int op) {
  int issuer = 0;
  if (w.lane == 0) issuer = (atomicAdd(&sc->elect, 1u) % kConsumers) == 0 ? 1 : 0;
  issuer = __shfl_sync(0xffffffffu, issuer, 0);
  if (issuer && w.lane == 0) {
    // the rows were published by other SMs and acquired by this thread's
    // dependency wait (generic proxy); the bulk copies read them, and write
    // shared memory last read by generic loads, through the async proxy
    asm volatile("fence.proxy.async.global;" ::: "memory");
    fence_proxy_async_smem();
    uint32_t total = 0;
    for (int i = 0; i < n; ++i) total += bytes[i];
    mbar_arrive_expect_tx(&sc->bar, total);
    for (int i = 0; i < n; ++i) bulk_g2s(xs + off[i], src[i], bytes[i], &sc->bar);
  }
  const uint32_t par = w.xphase & 1u;
  w.xphase++;
  if (!__all_sync(0xffffffffu, mbar_try_wait(&sc->bar, par)) && !wait_slot_slow(&sc->bar, par, w.P->timeout_ns)) {
    set_error(w, -5, op);
    return false;
  }
  return true;
}

// The op's input row: x = h * g (QKV, LMHEAD: the residual entering the
// layer, or the final one, with the norm's gain; SHARED_GU, ROUTED_GU: the
// residual after the o-projection with the FFN norm's gain) or x = o
// (OPROJ).  Every producer of these rows writes them gained and permuted.
MK_INLINE bool stage_x(Warp &w, StageCtl *sc, int type, float *xs, int op) {
  const Params &P = *w.P;
  const bool oproj = type == OP_OPROJ;
  const float *src = oproj ? P.o : P.xg;
  // rows 0..M-1 are contiguous: one copy
  const uint32_t bytes = static_cast<uint32_t>(P.M * (oproj ? P.ldo : P.ldx) * sizeof(float));
  const int off = 0;
  return stage_rows(w, sc, xs, &src, &bytes, &off, 1, op);
}

// Staged down projection: the CTA copies the activation rows (rows 0..M-1) of
// the experts its unit range covers (routed experts first, then the shared
// one) into shared memory, one slot of M * panel_ld(max(F, Fs)) floats per
// expert from the range's first, each a single bulk copy.
MK_INLINE bool stage_down(Warp &w, StageCtl *sc, int layer, float *xs, int op) {
  const Params &P = *w.P;
  if (!route_cache(w, layer)) return false;
  const int U = n_union(w), total = op_total_units(w, OP_DOWN, layer);
  int c0, c1;
  down_cta_range(P, w.cta, total, c0, c1);
  w.dseg0 = c0 / P.n_db;
  const float *src[kMaxStageSegs];
  uint32_t bytes[kMaxStageSegs];
  int off[kMaxStageSegs];
  int n = 0;
  if (c1 > c0) {
    const int seg0 = c0 / P.n_db, seg1 = (c1 - 1) / P.n_db, slot = P.M * panel_ld(max(P.F, P.Fs));
    for (int sg = seg0; sg <= seg1 && n < kMaxStageSegs; ++sg, ++n) {
      src[n] = sg < U ? P.act_routed + static_cast<size_t>(sg) * kMaxRows * P.ldf : P.act_shared;
      bytes[n] = static_cast<uint32_t>(P.M * (sg < U ? P.ldf : P.ldfs) * sizeof(float));
      off[n] = (sg - seg0) * slot;
    }
  }
  return stage_rows(w, sc, xs, src, bytes, off, n, op);
}

// inv_rms of rows 0..M-1 from v, lane m's copy of the fixed-point sum of
// squares of row m (loaded by the caller ahead of time).
MK_INLINE float inv_rms_of(long long sum, const Params &P) {
  return 1.0f / sqrtf(static_cast<float>(static_cast<double>(sum) * 0x1p-32) / static_cast<float>(P.d) + P.eps);
}
template <int MMAX>
MK_INLINE void inv_from_ssq(const Params &P, long long v, float (&inv)[kMaxRows]) {
#pragma unroll
  for (int m = 0; m < MMAX; ++m) {
    const long long vm = __shfl_sync(0xffffffffu, v, m);
    inv[m] = m < P.M ? inv_rms_of(vm, P) : 0.f;  // rows past M: no work
  }
}

// Ops whose units scale by an inv_rms, and which residual's sums they use
// (0: entering the layer, 1: after the o-projection), else -1.
MK_INLINE int normed_ssq(int type) {
  return (type == OP_QKV || type == OP_LMHEAD) ? 0 : (type == OP_SHARED_GU || type == OP_ROUTED_GU) ? 1 : -1;
}

template <int MMAX, bool XS>
MK_INLINE bool run_tile_op(Warp &w, int op, int type, int layer, const float *xs, long long sqv, AttnShared &ash,
                           float &am_val, int &am_idx) {
  const Params &P = *w.P;
  if ((type == OP_ROUTED_GU || type == OP_DOWN) && !route_cache(w, layer)) return false;
  int u0, stride, n;
  op_units(w, op, type, layer, u0, stride, n);
  if (n == 0) return true;
  float inv[kMaxRows];
#pragma unroll
  for (int m = 0; m < kMaxRows; ++m) inv[m] = 0.f;
  if (normed_ssq(type) >= 0) inv_from_ssq<MMAX>(P, sqv, inv);
  for (int i = 0; i < n; ++i) {
    const int u = u0 + i * stride;
    bool ok;
    if (type == OP_ATTN) {
      ok = (P.hd == 64) ? attn_unit<2>(w, op, layer, u, ash) : attn_unit<4>(w, op, layer, u, ash);
    } else if (type == OP_ROUTED_GU || type == OP_DOWN || type == OP_SHARED_GU) {
      ok = routed_dispatch<MMAX, XS>(w, op, type, layer, u, inv, xs);
    } else {
      ok = dense_unit<MMAX, XS>(w, op, type, layer, u, inv, xs, am_val, am_idx);
    }
    if (!ok || w.failed) return false;
  }
  return true;
}

// Producer warp: keep its consumer's ring filled until every tile of the
// launch's ops (all its steps) has been issued, then wait for the last copies.
// The consumer's stream state stays in registers; the producer keeps its own
// per-step attention layout (it may be a step ahead of its consumer).
template <bool MULTI>
MK_INLINE void producer_run(const Params &P, Warp *feeds, int first, int lane, int *prefix, int *nch) {
  static_assert(kFeeds == 1, "one consumer per producer");
  Warp mine = feeds[first];
  mine.lane = lane;
  mine.attn_prefix = prefix;
  mine.attn_nch = nch;
  attn_layout(P, 0, prefix, nch, lane);
  mine.lstep = 0;
  uint64_t t_idle = 0;
  int idle_reason = 0, idle_op = 0;  // trace only
  uint64_t idle_t0 = 0;
  for (int it = 0;; ++it) {
    bool progress = false, all_done = true;
    int why = FEED_PROGRESS;
    if (!mine.done_issue && !mine.failed) why = feed_more<MULTI>(mine);
    progress = why == FEED_PROGRESS;
    if (kTrace && P.trace && lane == 0) {
      // the producer's idle episodes on its current op, by reason: a clock read
      // when one starts and when it ends, added to the consumer's record
      const int reason = progress ? 0 : (why == FEED_RING_FULL ? 11 : 10);
      if (reason != idle_reason) {
        const uint64_t t = now_ns();
        if (idle_reason && idle_op < P.op_end)
          P.trace[(static_cast<size_t>(idle_op) * mine.nw + mine.slot) * kTraceWords + idle_reason] += t - idle_t0;
        idle_reason = reason;
        idle_t0 = t;
        idle_op = mine.iop;
      }
    }
    all_done = mine.done_issue || mine.failed;
    if (all_done) break;
    int stop = 0;
    if (lane == 0) {
      // the error word is a global round trip: look at it every 16th pass only,
      // so that an idle producer polls its next dependency at a short interval
      if ((it & 15) == 15 && *reinterpret_cast<volatile const int *>(P.error) != 0) {
        stop = 1;
      } else if (progress) {
        t_idle = 0;
      } else {
        const uint64_t t = now_ns();
        if (t_idle == 0) t_idle = t;
        // consumers' own waits report a stall first (with the op that
        // stalled); this bound only guarantees the producer ends
        if (t - t_idle > 4 * P.timeout_ns) {
          stop = 2;
        } else if (it > 4) {
          __nanosleep(32);
        }
      }
    }
    stop = __shfl_sync(0xffffffffu, stop, 0);
    if (stop == 2) report_error(P, lane, -5, -1);
    if (stop) break;
  }
  drain_feed(mine);
  __syncwarp();
}

// MULTI: several steps per launch (P.n_steps); the single-step instance keeps
// the step index a compile-time zero.
template <int MMAX, bool XS, bool MULTI>
__global__ void __launch_bounds__(kThreads, 1) mk_step_kernel(const __grid_constant__ Params P) {
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ int s_attn_prefix[kWarpsPerCta][kMaxRows + 1];  // each warp's, for its step
  __shared__ int s_attn_nch[kWarpsPerCta][kMaxRows];
  __shared__ uint32_t s_stage;
  __shared__ RouteCache s_route;
  __shared__ float s_attn_ml[kConsumers * kQvp * 2];
  __shared__ Warp s_feed[kConsumers];  // each consumer's tile stream, as its producer keeps it
  __shared__ StageCtl s_xstage;        // batch 1: the staged activation row's copies
  const int wib = threadIdx.x >> 5;
  const bool consumer = wib < kConsumers;
  // dynamic shared memory: rings | activation row | full and empty barriers |
  // router-logit sums | epilogue scratch | per-op arrival counts
  constexpr int S = ring_slots(MMAX);
  float *xs = reinterpret_cast<float *>(smem + kConsumers * S * kSlotBytes);
  uint8_t *after_xs = reinterpret_cast<uint8_t *>(xs + P.xs_floats);
  uint64_t *fulls = reinterpret_cast<uint64_t *>(after_xs);
  uint64_t *empties = fulls + kConsumers * S;
  long long *rsum = reinterpret_cast<long long *>(empties + kConsumers * S);
  float *fbase = reinterpret_cast<float *>(rsum + MMAX * P.e_ld);
  uint32_t *arrive_cnt = reinterpret_cast<uint32_t *>(fbase + kConsumers * kWbuf);
  Warp w;
  w.P = &P;
  w.rc = &s_route;
  w.wib = wib;
  w.cta = blockIdx.x;
  w.lane = threadIdx.x & 31;
  w.nw = P.n_warps;
  w.slot = consumer ? wib * P.n_cta + blockIdx.x : -1;
  const int c = consumer ? wib : 0;  // producers reach their consumers' records through s_feed
  w.ring = smem + c * S * kSlotBytes;
  w.nslots = S;
  w.full = fulls + c * S;
  w.empty = empties + c * S;
  w.wbuf = fbase + c * kWbuf;
  w.arrive = arrive_cnt;
  w.rsum = rsum;
  w.attn_prefix = s_attn_prefix[wib];
  w.attn_nch = s_attn_nch[wib];
  w.step = 0;
  w.lstep = -1;
  w.phase = 0;
  w.cslot = 0;
  w.islot = 0;
  w.ephase = (1u << S) - 1u;  // a fresh barrier's previous phase counts as complete
  w.filled = 0;
  w.producer = false;
  w.dseg0 = 0;
  w.xphase = 0;
  w.failed = false;
  w.pol_w = policy_evict_first();
  w.pol_kv = policy_evict_normal();
  w.epoch = *reinterpret_cast<volatile const uint32_t *>(P.epoch) + 1u;
  w.iop = P.op_begin;
  w.iop_init = false;
  w.done_issue = false;
  w.iu0 = w.in_units = w.iu = w.it = w.iunit = 0;
  w.itype = w.ilayer = 0;
  w.istride = 1;
  w.in_tiles = -1;
  w.um = w.um2 = nullptr;
  w.urow0 = w.urow2 = w.ucol0 = w.uK = 0;
  w.uhalf = 1 << 30;
  w.tr_first = w.tr_last = w.tr_wait = 0;
  w.tr_n = 0;
  if (consumer && w.lane == 0) {
    for (int sl = 0; sl < S; ++sl) {
      mbar_init(&w.full[sl], 1);
      mbar_init(&w.empty[sl], 1);
    }
    fence_mbar_init();
    Warp f = w;
    f.producer = true;
    s_feed[wib] = f;
  }
  for (int i = threadIdx.x; i < P.n_ops; i += kThreads) arrive_cnt[i] = 0;
  for (int i = threadIdx.x; i < MMAX * P.e_ld; i += kThreads) rsum[i] = 0;
  if (threadIdx.x == 0) {
    s_stage = 0;
    s_route.ready_key = s_route.fill_key = 0;
    s_xstage.elect = 0;
    mbar_init(&s_xstage.bar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  // Reject bad positions / token ids before any memory is touched with them.
  // Every warp evaluates the same condition, so all exit together.
  bool bad = false;
  for (int b = 0; b < P.B; ++b) {
    const int p = __ldg(&P.positions[b]);
    if (p < 0 || p + P.T * P.n_steps > P.cap) bad = true;
  }
  for (int m = w.lane; m < P.M; m += 32) {
    const int t = __ldcg(&P.tokens[m]);
    if (t < 0 || t >= P.V) bad = true;
  }
  if (__any_sync(0xffffffffu, bad)) {
    if (wib == 0) set_error(w, -6, P.op_begin);
    return;
  }

  if (!consumer) {
    producer_run<MULTI>(P, s_feed, (wib - kConsumers) * kFeeds, w.lane, s_attn_prefix[wib], s_attn_nch[wib]);
    return;
  }

  uint32_t stage_seq = 0;
  __nv_bfloat16 *knew = reinterpret_cast<__nv_bfloat16 *>(xs + (kConsumers + 1) * kQvp * P.hd);
  AttnShared ash{xs, xs + kConsumers * kQvp * P.hd, knew, knew + kMaxRows * P.hd, s_attn_ml, &s_stage, &stage_seq};
  const uint32_t epoch0 = w.epoch;
  const int n_steps = MULTI ? P.n_steps : 1;
  for (int step = 0; step < n_steps && !w.failed; ++step) {
  if constexpr (MULTI) {
    w.step = step;
    w.epoch = epoch0 + static_cast<uint32_t>(step);
  }
  // a later step embeds the previous step's argmax (and, verifying, starts
  // where its acceptance left the sequence): wait for its publication
  if (MULTI && step > 0 && !wait_counter(w, P.epoch, w.epoch - 1u, P.op_begin)) break;
  attn_layout(P, w.step, w.attn_prefix, w.attn_nch, w.lane);
  float am_val = -INFINITY;
  int am_idx = 0x7fffffff;
  for (int op = P.op_begin; op < P.op_end && !w.failed; ++op) {
    const int type = op_type_of(op, P.L), layer = op_layer_of(op, P.L);
    int d0, d1;
    op_deps(op, P.L, &d0, &d1);
    // batch 1: SHARED_GU stages the normed row that ROUTED_GU reuses; a launch
    // that starts at ROUTED_GU stages it itself
    const bool stage = XS && (type == OP_QKV || type == OP_OPROJ || type == OP_SHARED_GU || type == OP_LMHEAD ||
                              (type == OP_ROUTED_GU && op == P.op_begin));
    if (type == OP_ATTN) {
      // the rotary rows of this step's new positions (read by the attention
      // items' staging), pulled into L2 while the QKV op finishes: lane 4r + i
      // takes 128-byte line i of new row r (row r = b * T + t)
      const int r = w.lane >> 2;
      if (r < P.M) {
        const int pos = seq_pos(P, r / P.T, w.step) + r % P.T;
        if (pos < P.cap && 128 * (w.lane & 3) < P.hd * 4)  // a row is hd/2 float2 = hd * 4 bytes
          prefetch_l2(reinterpret_cast<const char *>(P.rope + static_cast<size_t>(pos) * (P.hd / 2)) +
                      128 * (w.lane & 3));
      }
    }
    const uint32_t target = w.epoch * static_cast<uint32_t>(P.n_cta);
    const uint32_t extra = (op == P.inject_op) ? 1u : 0u;
    if (d0 >= 0 && !wait_counter(w, &P.counters[d0 * kCounterStride], target + extra, op)) break;
    if (d1 >= 0 && !wait_counter(w, &P.counters[d1 * kCounterStride], target, op)) break;
    if (kTrace && P.trace && w.lane == 0 && type != OP_ROUTED_GU)
      P.trace[(static_cast<size_t>(op) * w.nw + w.slot) * kTraceWords + 6] = now_ns();
    // a normed op's rows' sums of squares, loaded now so that the load overlaps
    // the staging (lane m holds row m's)
    const int which = normed_ssq(type);
    const long long sqv = (which >= 0 && w.lane < P.M) ? __ldcg(P.ssq + which * kMaxRows + w.lane) : 0ll;
    // The sums of squares are cleared once their readers are done: the
    // o-projection's (read by the routing and the expert GEMVs) at the next
    // QKV, the entering residual's (read by QKV) at the o-projection, and, for
    // the next step's embedding, by the final argmax.
    if (w.slot == 0 && w.lane < P.M) {
      if (type == OP_QKV) P.ssq[kMaxRows + w.lane] = 0;
      if (type == OP_OPROJ) P.ssq[w.lane] = 0;
    }
    // the previous layer's router sums have been read by every CTA (its down
    // projection is complete): clear them for the next step
    if (type == OP_OPROJ && layer > 0) clear_router_sums(w, layer - 1);
    if (type == OP_LMHEAD) clear_router_sums(w, P.L - 1);
    if constexpr (XS) {
      if (stage && !stage_x(w, &s_xstage, type, xs, op)) break;
      if (type == OP_DOWN && P.down_staged && !stage_down(w, &s_xstage, layer, xs, op)) break;
    }
    if (kTrace && P.trace && w.lane == 0 && type != OP_ROUTED_GU)
      P.trace[(static_cast<size_t>(op) * w.nw + w.slot) * kTraceWords + 7] = now_ns();
    if (kTrace && P.trace && w.lane == 0) P.trace[(static_cast<size_t>(op) * w.nw + w.slot) * kTraceWords] = now_ns();
    w.tr_first = w.tr_last = w.tr_wait = 0;
    w.tr_n = 0;
    bool ok = true;
    if (type == OP_EMBED) {
      op_embed(w);
    } else if (type == OP_COMBINE) {
      op_combine(w, layer);
    } else {
      ok = run_tile_op<MMAX, XS>(w, op, type, layer, xs, sqv, ash, am_val, am_idx);
    }
    if (!ok || w.failed) break;
    if (type == OP_LMHEAD && (w.lane % kRows) == 0 && w.lane / kRows < P.M) {
      // lane 4m holds this warp's best (value, index) of row m
      P.am_part[static_cast<size_t>(w.slot) * kMaxRows + w.lane / kRows] = ArgmaxPart{am_val, am_idx};
    }
    const bool last = arrive(w, op, type, layer);
    if (kTrace && P.trace && w.lane == 0) {
      unsigned long long *tr = P.trace + (static_cast<size_t>(op) * w.nw + w.slot) * kTraceWords;
      tr[1] = w.tr_first;
      tr[2] = w.tr_last;
      tr[3] = now_ns();
      tr[4] = w.tr_wait;
      tr[5] = static_cast<unsigned long long>(w.tr_n);
    }
    if (last && type == OP_LMHEAD) final_argmax(P, w.lane, w.epoch, w.step);
  }
  }  // steps
}

}  // namespace

#if !MK_TRACE
size_t step_smem_bytes(int n_ops, int xs_floats, int mmax, int e_ld) {
  const int S = ring_slots(mmax);
  return static_cast<size_t>(kConsumers) * S * kSlotBytes + static_cast<size_t>(xs_floats) * sizeof(float) +
         2 * kConsumers * S * sizeof(uint64_t) + static_cast<size_t>(mmax) * e_ld * sizeof(long long) +
         kConsumers * kWbuf * sizeof(float) + static_cast<size_t>(n_ops) * sizeof(uint32_t);
}

bool kernel_stages_x(int mmax) { return mmax <= 8; }
#endif

template <int MMAX, bool XS, bool MULTI>
static const void *kernel_ptr() {
  return reinterpret_cast<const void *>(&mk_step_kernel<MMAX, XS, MULTI>);
}

// Batch 1 stages its activation row in shared memory; more rows read it via L1.
static const void *kernel_for(int mmax, bool multi) {
  if (multi) {
    switch (mmax) {
      case 1: return kernel_ptr<1, true, true>();
      case 2: return kernel_ptr<2, true, true>();
      case 4: return kernel_ptr<4, true, true>();
      default: return kernel_ptr<8, true, true>();
    }
  }
  switch (mmax) {
    case 1: return kernel_ptr<1, true, false>();
    case 2: return kernel_ptr<2, true, false>();
    case 4: return kernel_ptr<4, true, false>();
    default: return kernel_ptr<8, true, false>();
  }
}

int MK_ENTRY(max_cta_per_sm)(int mmax, size_t smem) {
  int n_min = 1 << 30;
  for (int multi = 0; multi < 2; ++multi) {  // both forms, single- and multi-step
    const void *k = kernel_for(mmax, multi != 0);
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
      return -1;
    // Ask for the smallest shared-memory carve-out that fits, leaving the rest of
    // the SM's unified memory to L1 (activations are re-read through it by every warp).
    int max_sm = 0, dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&max_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev);
    if (max_sm > 0) {
      const int pct = static_cast<int>((smem * 100 + max_sm - 1) / max_sm);
      cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, pct > 100 ? 100 : pct);
    }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, kThreads, smem) != cudaSuccess) return -1;
    n_min = n < n_min ? n : n_min;
  }
  return n_min;
}

int MK_ENTRY(launch_step)(const Params &p, int mmax, bool cooperative, cudaStream_t stream) {
  const void *k = kernel_for(mmax, p.n_steps > 1);
  const size_t smem = step_smem_bytes(p.n_ops, p.xs_floats, mmax, p.e_ld);
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
