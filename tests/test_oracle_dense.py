"""The oracle's dense decoder (n_experts = 0: no router, the FFN held as the
shared expert) pinned to its MoE path: a MoE model whose routed experts all
have a zero down projection adds exactly nothing besides the shared expert, so
with the same attention, shared-expert and head weights both give the same
step bit for bit.  The MoE path itself is pinned by the other oracle tests."""
import dataclasses

import numpy as np
import torch

from oracle import step as ostep
from synthetic import (bf16_bits, make_context_lengths, make_kv_cache, make_tokens, make_weights,
                       workload)


def test_dense_step_equals_moe_step_with_silent_experts():
    wl = workload("tiny_dense")
    dense = wl.model
    moe = dataclasses.replace(dense, name="tiny_moe_silent", n_experts=4, top_k=2, expert_ffn=32)
    wd = make_weights(dense, wl.seed, "cpu")
    wm = make_weights(moe, wl.seed + 1, "cpu")
    for l in range(dense.n_layers):
        for name in ("attn_norm", "wqkv", "wo", "ffn_norm", "ws_gate", "ws_up", "ws_down"):
            wm["layers"][l][name] = wd["layers"][l][name].clone()
        wm["layers"][l]["w_down"].zero_()
    for name in ("embed", "final_norm", "lm_head"):
        wm[name] = wd[name].clone()

    cap = wl.kv_capacity()
    k, v = make_kv_cache(dense, 1, cap, wl.seed, "cpu")
    tokens = make_tokens(dense.vocab, 1, wl.seed)
    positions = make_context_lengths(wl)
    outs = []
    for model, w in ((dense, wd), (moe, wm)):
        kc, vc = bf16_bits(k).copy(), bf16_bits(v).copy()
        tok, pos = list(tokens), list(positions)
        steps = []
        for _ in range(3):
            r = ostep.decode_step(model, ostep.WeightSource(w), kc, vc, tok, pos, 1, 1)
            steps.append((r.logits.copy(), r.hidden.copy()))
            tok, pos = [int(r.argmax[0])], [pos[0] + 1]
        outs.append((steps, kc, vc))
    (sd, kd, vd), (sm, km, vm) = outs
    for (ld, hd), (lm, hm) in zip(sd, sm):
        assert np.array_equal(ld.view(np.uint32), lm.view(np.uint32))
        assert np.array_equal(hd.view(np.uint32), hm.view(np.uint32))
    assert np.array_equal(kd, km) and np.array_equal(vd, vm)
    # the experts really were consulted on the MoE side (so the test is not vacuous)
    r = ostep.decode_step(moe, ostep.WeightSource(wm), bf16_bits(k).copy(), bf16_bits(v).copy(),
                          tokens, positions, 1, 1)
    assert r.expert_ids.shape == (dense.n_layers, 1, 2)
    assert np.all(np.abs(r.expert_w.sum(-1) - 1.0) < 1e-5)


def test_dense_step_has_no_routing():
    wl = workload("tiny_dense")
    m = wl.model
    w = make_weights(m, wl.seed, "cpu")
    k, v = make_kv_cache(m, 1, wl.kv_capacity(), wl.seed, "cpu")
    r = ostep.decode_step(m, ostep.WeightSource(w), bf16_bits(k).copy(), bf16_bits(v).copy(),
                          make_tokens(m.vocab, 1, wl.seed), make_context_lengths(wl), 1, 1)
    assert r.router_logits.shape == (m.n_layers, 1, 0) and r.expert_ids.shape == (m.n_layers, 1, 0)
    assert np.isfinite(r.logits).all()
