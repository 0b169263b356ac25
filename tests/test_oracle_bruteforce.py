"""The oracle's incremental decode against brute force and against itself.

* Brute force: decode a sequence token by token from an empty cache with the
  oracle, and at every position recompute the whole prefix from scratch --
  full causal attention over freshly computed keys and values, no cache -- in
  float64 numpy.  The two must agree: this pins the cache append slot, the
  attended range, the rotary positions, GQA grouping, the routing and the
  residual plumbing of the incremental step.
* Verify block == sequential: T new tokens scored in one causal block equal T
  single-token steps.
* Batch == single rows: every sequence of a batched step equals its own B=1 step.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import step as ostep
from synthetic import ModelConfig, make_kv_cache, make_tokens, make_weights

BF = ModelConfig("bruteforce", n_layers=2, d_model=64, n_q_heads=4, n_kv_heads=2, head_dim=16,
                 n_experts=6, top_k=2, expert_ffn=32, shared_ffn=24, vocab=96, sigma=0.15)


def _f64(t):
    return t.float().double().numpy()


def _bf16_round64(x):
    """fp64 -> fp32 -> bf16 (round to nearest even) -> fp64, as the cache stores keys."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def full_sequence_logits(m: ModelConfig, w, tokens):
    """Float64 forward over the whole prefix with causal attention (no cache)."""
    n = len(tokens)
    Hq, Hkv, hd, d = m.n_q_heads, m.n_kv_heads, m.head_dim, m.d_model
    grp = Hq // Hkv

    def rms(H, g):
        return H / np.sqrt((H * H).mean(axis=1, keepdims=True) + m.rms_eps) * g

    half = hd // 2
    inv = m.rope_theta ** (-2.0 * np.arange(half) / hd)
    ang = np.arange(n)[:, None] * inv[None, :]
    cos, sin = np.cos(ang), np.sin(ang)

    def rot(X):  # X [n, heads, hd]
        a, b = X[..., :half], X[..., half:]
        c, s = cos[:, None, :], sin[:, None, :]
        return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)

    H = _f64(w["embed"])[tokens]
    routes = []
    for l in range(m.n_layers):
        lw = w["layers"][l]
        X = rms(H, _f64(lw["attn_norm"]))
        QKV = X @ _f64(lw["wqkv"]).T
        Q = rot(QKV[:, :Hq * hd].reshape(n, Hq, hd))
        K = _bf16_round64(rot(QKV[:, Hq * hd:(Hq + Hkv) * hd].reshape(n, Hkv, hd)))
        V = _bf16_round64(QKV[:, (Hq + Hkv) * hd:].reshape(n, Hkv, hd))
        O = np.empty((n, Hq, hd))
        causal = np.tril(np.ones((n, n), dtype=bool))
        for h in range(Hq):
            g = h // grp
            S = Q[:, h, :] @ K[:, g, :].T / np.sqrt(hd)
            S = np.where(causal, S, -np.inf)
            P = np.exp(S - S.max(axis=1, keepdims=True))
            P /= P.sum(axis=1, keepdims=True)
            O[:, h, :] = P @ V[:, g, :]
        H = H + O.reshape(n, Hq * hd) @ _f64(lw["wo"]).T
        Y = rms(H, _f64(lw["ffn_norm"]))
        Z = Y @ _f64(lw["router"]).T
        Pz = np.exp(Z - Z.max(axis=1, keepdims=True))
        Pz /= Pz.sum(axis=1, keepdims=True)
        moe = np.zeros_like(H)
        ids_l = []
        for r in range(n):
            sel = np.argsort(-Pz[r], kind="stable")[:m.top_k]
            ids_l.append(sorted(sel.tolist()))
            wsel = Pz[r, sel] / Pz[r, sel].sum()
            for e, we in zip(sel, wsel):
                g_ = _f64(lw["w_gate"][e]) @ Y[r]
                u_ = _f64(lw["w_up"][e]) @ Y[r]
                moe[r] += we * (_f64(lw["w_down"][e]) @ (g_ / (1 + np.exp(-g_)) * u_))
        sh = np.zeros_like(H)
        if m.shared_ffn:
            G = Y @ _f64(lw["ws_gate"]).T
            U = Y @ _f64(lw["ws_up"]).T
            sh = (G / (1 + np.exp(-G)) * U) @ _f64(lw["ws_down"]).T
        H = H + moe + sh
        routes.append(ids_l)
        zs = np.sort(Z, axis=1)[:, ::-1]
        routes[-1] = (ids_l, zs[:, m.top_k - 1] - zs[:, m.top_k])
    logits = rms(H, _f64(w["final_norm"])) @ _f64(w["lm_head"]).T
    return logits, routes


@pytest.fixture(scope="module")
def bf_model():
    return make_weights(BF, seed=11, device="cpu")


def test_incremental_equals_full_recompute(oracle_lib, bf_model):
    m = BF
    n = 14
    tokens = make_tokens(m.vocab, n, seed=12)
    src = ostep.WeightSource(bf_model)
    cap = 16
    kc = np.zeros((m.n_layers, 1, m.n_kv_heads, cap, m.head_dim), dtype=np.uint16)
    vc = np.zeros_like(kc)
    ref_logits, routes = full_sequence_logits(m, bf_model, tokens)
    for i in range(n):
        r = ostep.decode_step(m, src, kc, vc, [tokens[i]], [i], 1, 1)
        ref = ref_logits[i]
        err = np.abs(r.logits[0] - ref).max() / np.abs(ref).max()
        assert err < 2e-4, (i, err)
        for l in range(m.n_layers):
            ids_ref, margin = routes[l]
            if margin[i] > 1e-3:
                assert sorted(r.expert_ids[l, 0].tolist()) == ids_ref[i], (i, l)
        top2 = np.sort(ref)[-2:]
        if top2[1] - top2[0] > 1e-3:
            assert int(r.argmax[0]) == int(np.argmax(ref))


def test_verify_block_equals_sequential_steps(oracle_lib, bf_model):
    m = BF
    cap = 32
    k0, v0 = make_kv_cache(m, 1, cap, seed=13)
    kb = ostep._host_bits(k0).copy()
    vb = ostep._host_bits(v0).copy()
    ks, vs = kb.copy(), vb.copy()
    src = ostep.WeightSource(bf_model)
    toks = make_tokens(m.vocab, 5, seed=14)
    p0 = 9
    blk = ostep.decode_step(m, src, kb, vb, toks, [p0], 1, 5)
    for t in range(5):
        one = ostep.decode_step(m, src, ks, vs, [toks[t]], [p0 + t], 1, 1)
        np.testing.assert_allclose(blk.logits[t], one.logits[0], rtol=0, atol=1e-6)
        np.testing.assert_array_equal(blk.expert_ids[:, t], one.expert_ids[:, 0])
    np.testing.assert_array_equal(kb, ks)
    np.testing.assert_array_equal(vb, vs)


def test_batch_rows_equal_single_sequences(oracle_lib, bf_model):
    m = BF
    cap = 24
    B = 3
    k0, v0 = make_kv_cache(m, B, cap, seed=15)
    kb, vb = ostep._host_bits(k0).copy(), ostep._host_bits(v0).copy()
    src = ostep.WeightSource(bf_model)
    toks = make_tokens(m.vocab, B, seed=16)
    pos = [3, 17, 8]
    batch = ostep.decode_step(m, src, kb.copy(), vb.copy(), toks, pos, B, 1)
    for b in range(B):
        ks = np.ascontiguousarray(kb[:, b:b + 1])
        vs = np.ascontiguousarray(vb[:, b:b + 1])
        one = ostep.decode_step(m, src, ks, vs, [toks[b]], [pos[b]], 1, 1)
        np.testing.assert_allclose(batch.logits[b], one.logits[0], rtol=0, atol=1e-6)
        np.testing.assert_array_equal(batch.argmax[b], one.argmax[0])


def test_float64_restatement_agrees_on_tiny_shapes(oracle_lib):
    """Second opinion (not a pin): the fp64 restatement above and the C oracle
    agree on a random prefilled cache once the prefix is rebuilt the same way."""
    m = ModelConfig("t", 1, 32, 2, 1, 16, 4, 2, 16, 0, 40, sigma=0.2)
    w = make_weights(m, seed=21)
    toks = make_tokens(m.vocab, 6, seed=22)
    src = ostep.WeightSource(w)
    kc = np.zeros((1, 1, 1, 8, 16), dtype=np.uint16)
    vc = np.zeros_like(kc)
    ref, _ = full_sequence_logits(m, w, toks)
    for i, t in enumerate(toks):
        r = ostep.decode_step(m, src, kc, vc, [t], [i], 1, 1)
        assert np.abs(r.logits[0] - ref[i]).max() / np.abs(ref[i]).max() < 2e-4
