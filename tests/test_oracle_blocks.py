"""The oracle's blocks and whole step against closed forms and invariants.

Every expected value here is worked by hand (derivation in the test) or is an
invariant of the definition (router weights sum to one, a rotation keeps
norms and relative positions, ...).  These pins are chosen so that a plausible
slip -- an interleaved GQA mapping, a cache append at the wrong slot, rotation
after the cache store, a transposed projection, unnormalised routing weights --
fails at least one of them.
"""
import ctypes
import math

import numpy as np
import pytest

import oracle
from oracle import step as ostep


def bf(a):
    a = np.asarray(a, dtype=np.float32)
    bits = oracle.bf16_round(a)
    assert np.array_equal(oracle.bf16_to_f32(bits), a)
    return bits


class Cfg:
    """Minimal model description for hand-built cases."""

    def __init__(self, **kw):
        self.rope_theta = 1e4
        self.rms_eps = 1e-6
        self.__dict__.update(kw)


def _dims(cfg, max_seqs, cap):
    return ostep.dims_of(cfg, max_seqs, cap)


def test_attention_block_gqa_append_and_oproj(oracle_lib):
    """q = k = v = 0 for the new token; cached V is 1 on kv head 0 and 2 on kv
    head 1 over positions 0..2; the new token sits at position 3.

    Equal scores average the 4 attended values: heads of group 0 (q heads 0, 1)
    get 3/4 * 1, group 1 (q heads 2, 3) gets 3/4 * 2 -- contiguous grouping
    g = h / (Hq/Hkv).  Wo is the cyclic shift y[i] = o[(i+1) % 8], so
    h' = 1 + (.75,.75,.75,1.5,1.5,1.5,1.5,.75).  An interleaved mapping, an
    attended range that leaves out the new position, or a transposed Wo each
    changes the result.
    """
    cfg = Cfg(d_model=8, n_q_heads=4, n_kv_heads=2, head_dim=2, n_experts=2, top_k=1,
              expert_ffn=2, shared_ffn=0, vocab=4)
    cap = 8
    D = _dims(cfg, 1, cap)
    kc = np.zeros((1, 2, cap, 2), dtype=np.uint16)
    vc = np.zeros((1, 2, cap, 2), dtype=np.uint16)
    kc[0, :, :3, :] = bf(np.full((2, 3, 2), 0.5))
    vc[0, 0, :3, :] = bf(np.ones((3, 2)))
    vc[0, 1, :3, :] = bf(np.full((3, 2), 2.0))
    vc[0, :, 3:, :] = bf(np.full((2, cap - 3, 2), 7.0))  # beyond the append: never read
    wo = np.zeros((8, 8), dtype=np.float32)
    for i in range(8):
        wo[i, (i + 1) % 8] = 1.0
    h = np.ones((1, 8), dtype=np.float32)
    pos = np.array([3], dtype=np.int32)
    L = oracle.lib()
    L.or_attn_block(ctypes.byref(D), oracle.u16p(bf(np.ones(8))), oracle.u16p(bf(np.zeros((16, 8)))),
                    oracle.u16p(bf(wo)), oracle.u16p(kc), oracle.u16p(vc), ctypes.c_int(1),
                    ctypes.c_int(1), oracle.i32p(pos), oracle.f32p(h))
    want = 1 + np.array([.75, .75, .75, 1.5, 1.5, 1.5, 1.5, .75], dtype=np.float32)
    np.testing.assert_allclose(h[0], want, rtol=0, atol=1e-6)
    # the appended slot now holds bf16(+-0) for K and V; later slots are untouched
    assert np.all(oracle.bf16_to_f32(kc[0, :, 3]) == 0)
    assert np.all(oracle.bf16_to_f32(vc[0, :, 3]) == 0)
    assert np.all(oracle.bf16_to_f32(vc[0, :, 4:]) == 7.0)


def test_attention_block_rotates_keys_before_the_store(oracle_lib):
    """h = 1 (so x = 1/sqrt(1 + 1e-6) = 0.9999995), Wk row 0 = e0, row 1 = 0:
    k = (0.9999995, 0) at position 1.  Rotating pair 0 by 1 rad gives
    (0.5403020, 0.8414705); round-to-nearest-even bf16 gives (0.5390625,
    0.83984375) (neighbours 0.54296875 and 0.84375 are farther).  V gets the
    unrotated (0.9999995, 0) -> bf16 (1.0, 0).
    """
    cfg = Cfg(d_model=8, n_q_heads=1, n_kv_heads=1, head_dim=2, n_experts=2, top_k=1,
              expert_ffn=2, shared_ffn=0, vocab=4)
    cap = 4
    D = _dims(cfg, 1, cap)
    w = np.zeros((6, 8), dtype=np.float32)  # rows: q(2), k(2), v(2)
    w[2, 0] = 1.0
    w[4, 0] = 1.0
    kc = np.zeros((1, 1, cap, 2), dtype=np.uint16)
    vc = np.zeros((1, 1, cap, 2), dtype=np.uint16)
    h = np.ones((1, 8), dtype=np.float32)
    pos = np.array([1], dtype=np.int32)
    oracle.lib().or_attn_block(ctypes.byref(D), oracle.u16p(bf(np.ones(8))), oracle.u16p(bf(w)),
                               oracle.u16p(bf(np.zeros((8, 2)))), oracle.u16p(kc),
                               oracle.u16p(vc), ctypes.c_int(1), ctypes.c_int(1),
                               oracle.i32p(pos), oracle.f32p(h))
    np.testing.assert_array_equal(oracle.bf16_to_f32(kc[0, 0, 1]), [0.5390625, 0.83984375])
    np.testing.assert_array_equal(oracle.bf16_to_f32(vc[0, 0, 1]), [1.0, 0.0])
    assert np.all(kc[0, 0, 0] == 0) and np.all(kc[0, 0, 2:] == 0)


def test_router_dominant_row_and_weights(oracle_lib):
    """h = 1 -> y = 0.9999995 * 1; router row 2 = 0.5 gives logit 3.999998, the
    rest 0: top-2 = {2, 0} (lowest of the tied zeros) with weights
    e^4/(e^4+1) = 0.98201379, 1/(e^4+1) = 0.01798621."""
    cfg = Cfg(d_model=8, n_q_heads=1, n_kv_heads=1, head_dim=8, n_experts=4, top_k=2,
              expert_ffn=2, shared_ffn=0, vocab=4)
    D = _dims(cfg, 1, 4)
    wr = np.zeros((4, 8), dtype=np.float32)
    wr[2] = 0.5
    h = np.ones((1, 8), dtype=np.float32)
    y = np.empty_like(h)
    z = np.empty((1, 4), dtype=np.float32)
    ids = np.empty((1, 2), dtype=np.int32)
    w = np.empty((1, 2), dtype=np.float32)
    oracle.lib().or_ffn_route(ctypes.byref(D), oracle.u16p(bf(np.ones(8))), oracle.u16p(bf(wr)),
                              ctypes.c_int(1), oracle.f32p(h), oracle.f32p(y), oracle.f32p(z),
                              oracle.i32p(ids), oracle.f32p(w))
    assert list(ids[0]) == [2, 0]
    np.testing.assert_allclose(w[0], [0.9820137900379085, 0.01798620996209156], atol=2e-6)
    np.testing.assert_allclose(z[0], [0, 0, 4 / math.sqrt(1 + 1e-6), 0], atol=1e-6)


def _ffn_apply(cfg, y, w, experts, shared, h):
    D = _dims(cfg, 1, 4)
    M, k = w.shape
    Arr = ctypes.POINTER(ctypes.c_uint16) * (M * k)
    wg, wu, wd = Arr(), Arr(), Arr()
    for i, (g_, u_, d_) in enumerate(experts):
        wg[i], wu[i], wd[i] = oracle.u16p(g_), oracle.u16p(u_), oracle.u16p(d_)
    null = ctypes.POINTER(ctypes.c_uint16)()
    sg, su, sd = shared if shared else (None, None, None)
    oracle.lib().or_ffn_apply(ctypes.byref(D), ctypes.c_int(M), oracle.f32p(y), oracle.f32p(w),
                              wg, wu, wd, oracle.u16p(sg) if sg is not None else null,
                              oracle.u16p(su) if su is not None else null,
                              oracle.u16p(sd) if sd is not None else null, oracle.f32p(h))


def test_ffn_zero_gate_leaves_residual_unchanged(oracle_lib):
    """Wg = 0 -> silu(0) = 0 -> every expert outputs 0 -> h is unchanged."""
    cfg = Cfg(d_model=4, n_q_heads=1, n_kv_heads=1, head_dim=4, n_experts=2, top_k=2,
              expert_ffn=3, shared_ffn=0, vocab=4)
    rng = np.random.default_rng(0)
    z = bf(np.zeros((3, 4)))
    ex = [(z, bf(np.round(rng.normal(size=(3, 4)), 2).astype(np.float32) * 0 + 1),
           bf(np.ones((4, 3))))] * 2
    y = rng.normal(size=(1, 4)).astype(np.float32)
    h = np.array([[1, -2, 3, -4]], dtype=np.float32)
    _ffn_apply(cfg, y, np.array([[0.7, 0.3]], dtype=np.float32), ex, None, h)
    np.testing.assert_array_equal(h[0], [1, -2, 3, -4])


def test_ffn_combination_and_shared_expert(oracle_lib):
    """Hand-worked: d = 2, F = 2, y = (1, 2).  Expert A = the golden SwiGLU case
    (out (4.98530547, 3.52318831)); expert B has Wd = 0 (out 0).  Weights
    (0.25, 0.75): moe = 0.25 * A.  Shared expert = expert A again, weight 1.
    h' = h + 1.25 * A."""
    cfg = Cfg(d_model=2, n_q_heads=1, n_kv_heads=1, head_dim=2, n_experts=2, top_k=2,
              expert_ffn=2, shared_ffn=2, vocab=4)
    A = (bf([[1, 0], [0, 1]]), bf([[2, 0], [0, 1]]), bf([[1, 1], [0, 1]]))
    B = (A[0], A[1], bf(np.zeros((2, 2))))
    y = np.array([[1, 2]], dtype=np.float32)
    h = np.array([[10, 20]], dtype=np.float32)
    _ffn_apply(cfg, y, np.array([[0.25, 0.75]], dtype=np.float32), [A, B], A, h)
    a = np.array([4.985305469171539, 3.5231883119115293])
    np.testing.assert_allclose(h[0], [10, 20] + 1.25 * a, rtol=1e-6)


def test_whole_step_embedding_and_lm_head_orientation(oracle_lib):
    """One layer whose projections and experts are all zero: the step reduces to
    logits = Wlm (rms(embed[t]) * 1).  embed[t] = 4 e_t gives x = 2.828 e_t;
    Wlm row i = e_{(i+3) % 8}, so logits[i] = x[(i+3) % 8] peaks at
    i = (t + 5) % 8 (a transposed lm_head would peak at (t + 3) % 8)."""
    d, V = 8, 8
    cfg = Cfg(n_layers=1, d_model=d, n_q_heads=2, n_kv_heads=1, head_dim=4, n_experts=2,
              top_k=1, expert_ffn=2, shared_ffn=0, vocab=V)
    embed = np.zeros((V, d), dtype=np.float32)
    for t in range(V):
        embed[t, t] = 4.0
    lm = np.zeros((V, d), dtype=np.float32)
    for i in range(V):
        lm[i, (i + 3) % 8] = 1.0
    z = lambda *s: bf(np.zeros(s))  # noqa: E731
    layer = {"attn_norm": bf(np.ones(d)), "wqkv": z(16, d), "wo": z(d, 8),
             "ffn_norm": bf(np.ones(d)), "router": z(2, d), "w_gate": z(2, 2, d),
             "w_up": z(2, 2, d), "w_down": z(2, d, 2)}
    weights = {"embed": bf(embed), "final_norm": bf(np.ones(d)), "lm_head": bf(lm),
               "layers": [layer]}
    src = ostep.WeightSource(weights)
    for t in (1, 6):
        kc = np.zeros((1, 1, 1, 4, 4), dtype=np.uint16)
        vc = np.zeros_like(kc)
        r = ostep.decode_step(cfg, src, kc, vc, [t], [0], 1, 1)
        assert int(r.argmax[0]) == (t + 5) % 8
        np.testing.assert_allclose(r.logits[0, (t + 5) % 8], 4 / math.sqrt(2 + 1e-6), rtol=1e-6)


def test_router_invariants_random(oracle_lib):
    rng = np.random.default_rng(1)
    for E, k in ((8, 2), (64, 4), (128, 8)):
        for _ in range(50):
            z = rng.normal(size=E).astype(np.float32)
            ids, w = oracle.topk_softmax(z, k)
            assert len(set(ids.tolist())) == k
            assert abs(float(w.sum()) - 1.0) < 1e-6
            assert np.all(np.diff(w) <= 0)  # selection order is descending
            inside = z[ids].min()
            outside = np.delete(z, ids).max()
            assert inside >= outside
            # the renormalised weights equal a softmax over the selected logits
            zs = z[ids].astype(np.float64)
            ref = np.exp(zs - zs.max()) / np.exp(zs - zs.max()).sum()
            np.testing.assert_allclose(w, ref, rtol=1e-5)


def test_rope_invariants(oracle_lib):
    """A rotation keeps each pair's norm, and scores depend only on the offset."""
    rng = np.random.default_rng(2)
    hd = 16
    q = rng.normal(size=hd).astype(np.float32)
    k = rng.normal(size=hd).astype(np.float32)
    for p in (0, 1, 7, 1000, 4095):
        r = oracle.rope(q, p, 1e4)
        n0 = q[:8] ** 2 + q[8:] ** 2
        n1 = r[:8] ** 2 + r[8:] ** 2
        np.testing.assert_allclose(n1, n0, rtol=1e-5)
    for p, pk in ((5, 2), (300, 17), (4000, 3999)):
        base = float(np.dot(oracle.rope(q, p, 1e4), oracle.rope(k, pk, 1e4)))
        for s in (1, 13, 64):
            shifted = float(np.dot(oracle.rope(q, p + s, 1e4), oracle.rope(k, pk + s, 1e4)))
            assert abs(shifted - base) < 2e-4 * (1 + abs(base))


def test_attention_invariants(oracle_lib):
    """Adding a constant to every score (q . k shifted via an extra key
    component shared by all keys) leaves the softmax unchanged; permuting the
    cached positions permutes nothing in the output."""
    rng = np.random.default_rng(3)
    hd, n = 8, 9
    K = rng.normal(size=(n, hd)).astype(np.float32)
    V = rng.normal(size=(n, hd)).astype(np.float32)
    Kb, Vb = oracle.bf16_round(K), oracle.bf16_round(V)
    q = rng.normal(size=hd).astype(np.float32)
    out = oracle.attend(q, Kb, Vb)
    perm = rng.permutation(n)
    out_p = oracle.attend(q, Kb[perm], Vb[perm])
    np.testing.assert_allclose(out_p, out, rtol=1e-5, atol=1e-6)
    # output is a convex combination of the values
    Vf = oracle.bf16_to_f32(Vb)
    assert np.all(out <= Vf.max(axis=0) + 1e-6) and np.all(out >= Vf.min(axis=0) - 1e-6)
