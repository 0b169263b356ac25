"""Several greedy decode steps in one persistent launch (mk_decode_steps).

Each step of the launch runs the same schedule and arithmetic as a
single-step call, so N steps in one launch must give bit for bit the tokens,
final logits and appended KV rows of N single-step calls that feed each
step's argmax back as the next token.  The single-step path is checked
against the oracle elsewhere; here the launch's tokens are also compared with
the oracle's own greedy decode directly, up to its first near tie.
"""
import numpy as np
import pytest
import torch

import decode_megakernel_06_b200 as mk
from oracle import step as ostep
from synthetic import ModelConfig, Workload, make_context_lengths, make_tokens, workload

from parity import MARGIN, Session

pytestmark = pytest.mark.gpu

RAGGED = ModelConfig("ragged", n_layers=2, d_model=264, n_q_heads=6, n_kv_heads=2, head_dim=64,
                     n_experts=6, top_k=2, expert_ffn=48, shared_ffn=32, vocab=1000, sigma=0.05)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


def _single_steps(s: Session, tokens, positions, n):
    """n single-step calls, each step's argmax fed back on the device."""
    dev = s.dev
    tok = torch.tensor(tokens, dtype=torch.int32, device=dev)
    pos0 = torch.tensor(positions, dtype=torch.int32, device=dev)
    out = torch.empty((n, s.B), dtype=torch.int32, device=dev)
    logits = torch.empty((s.B, s.m.vocab), dtype=torch.float32, device=dev)
    for i in range(n):
        pos = pos0 + i
        rc = s.dec.step(tok if i == 0 else out[i - 1], pos, s.B, 1, s.k, s.v, logits, out[i])
        assert rc == mk.MK_OK, mk.mk_last_error()
    assert s.dec.status() == mk.MK_OK
    return out.cpu().numpy(), logits.cpu().numpy()


def _one_launch(s: Session, tokens, positions, n):
    dev = s.dev
    tok = torch.tensor(tokens, dtype=torch.int32, device=dev)
    pos = torch.tensor(positions, dtype=torch.int32, device=dev)
    out = torch.empty((n, s.B), dtype=torch.int32, device=dev)
    logits = torch.empty((s.B, s.m.vocab), dtype=torch.float32, device=dev)
    rc = s.dec.steps(tok, pos, s.B, n, s.k, s.v, logits, out)
    assert rc == mk.MK_OK, mk.mk_last_error()
    st = s.dec.status()
    assert st == mk.MK_OK, (st, mk.mk_last_error())
    return out.cpu().numpy(), logits.cpu().numpy()


def _workloads():
    return [
        ("tiny", workload("tiny"), None, 16),
        ("small", workload("small"), None, 6),
        ("ragged_b3", Workload("ragged_b3", RAGGED, 3, 1, context=None, context_range=(1, 60),
                               steps=8, seed=7), 96, 10),
        ("small_b4", workload("small_batch", 4), None, 4),
    ]


@pytest.mark.parametrize("name,wl,cap,n", _workloads(), ids=[w[0] for w in _workloads()])
def test_one_launch_equals_single_steps(name, wl, cap, n):
    cap = cap or wl.kv_capacity() + n
    s = Session(wl, capacity=cap)
    s.dec.set_debug(None, None, None)
    positions = make_context_lengths(wl)
    tokens = make_tokens(s.m.vocab, s.B, wl.seed)
    k0, v0 = s.k.clone(), s.v.clone()
    ref_tok, ref_logits = _single_steps(s, tokens, positions, n)
    k1, v1 = s.k.clone(), s.v.clone()
    s.k.copy_(k0)
    s.v.copy_(v0)
    got_tok, got_logits = _one_launch(s, tokens, positions, n)
    np.testing.assert_array_equal(got_tok, ref_tok)
    assert np.array_equal(got_logits.view(np.uint32), ref_logits.view(np.uint32)), "final logits differ"
    assert torch.equal(s.k.view(torch.int16), k1.view(torch.int16)), "K cache differs"
    assert torch.equal(s.v.view(torch.int16), v1.view(torch.int16)), "V cache differs"
    s.close()
    print(name, "tokens", got_tok[:, 0].tolist())


def test_tiny_launch_follows_the_oracle():
    """The launch's greedy tokens against the oracle's greedy decode, compared
    until the oracle meets its first argmax near tie."""
    wl = workload("tiny")
    n = 16
    s = Session(wl, capacity=wl.kv_capacity() + n)
    s.dec.set_debug(None, None, None)
    positions = make_context_lengths(wl)
    tokens = make_tokens(s.m.vocab, s.B, wl.seed)
    got_tok, _ = _one_launch(s, tokens, positions, n)
    checked = 0
    tok, pos = list(tokens), list(positions)
    for i in range(n):
        ref = s.oracle_step(tok, pos)
        top2 = np.sort(ref.logits[0])[-2:]
        if top2[1] - top2[0] <= MARGIN:
            break
        assert int(got_tok[i, 0]) == int(ref.argmax[0]), f"step {i}: {got_tok[i, 0]} vs {ref.argmax[0]}"
        checked += 1
        tok = [int(ref.argmax[0])]
        pos = [p + 1 for p in pos]
    s.close()
    assert checked >= 12, checked


def test_small_launch_follows_the_oracle():
    """The same on the small model (8 layers, d 2048, 64 experts top-4): one
    launch of 8 greedy steps against the oracle's greedy decode."""
    wl = workload("small")
    n = 8
    s = Session(wl, capacity=wl.kv_capacity() + n)
    s.dec.set_debug(None, None, None)
    positions = make_context_lengths(wl)
    tokens = make_tokens(s.m.vocab, s.B, wl.seed)
    got_tok, _ = _one_launch(s, tokens, positions, n)
    checked = 0
    tok, pos = list(tokens), list(positions)
    for i in range(n):
        ref = s.oracle_step(tok, pos)
        top2 = np.sort(ref.logits[0])[-2:]
        # stop at the first near tie of the argmax or of any layer's routing
        if top2[1] - top2[0] <= MARGIN or ostep.router_margins(ref.router_logits, s.m.top_k).min() <= MARGIN:
            break
        assert int(got_tok[i, 0]) == int(ref.argmax[0]), f"step {i}: {got_tok[i, 0]} vs {ref.argmax[0]}"
        checked += 1
        tok = [int(ref.argmax[0])]
        pos = [p + 1 for p in pos]
    s.close()
    assert checked >= 2, checked


def test_launch_rejects_bad_arguments():
    wl = workload("tiny")
    s = Session(wl, capacity=wl.kv_capacity() + 4)
    s.dec.set_debug(None, None, None)
    tok = torch.tensor(make_tokens(s.m.vocab, 1, wl.seed), dtype=torch.int32, device=s.dev)
    out = torch.empty((4, 1), dtype=torch.int32, device=s.dev)
    # host checks
    pos = torch.tensor([10], dtype=torch.int32, device=s.dev)
    assert s.dec.steps(tok, pos, 1, 0, s.k, s.v, None, out) == mk.MK_ERR_ARG
    # a launch that would run past the cache is stopped on the device, and the
    # handle keeps working afterwards
    pos = torch.tensor([s.cap - 2], dtype=torch.int32, device=s.dev)
    assert s.dec.steps(tok, pos, 1, 4, s.k, s.v, None, out) == mk.MK_OK
    assert s.dec.status() == mk.MK_ERR_DEVICE_CHECK
    pos = torch.tensor([10], dtype=torch.int32, device=s.dev)
    assert s.dec.steps(tok, pos, 1, 4, s.k, s.v, None, out) == mk.MK_OK
    assert s.dec.status() == mk.MK_OK
    s.close()
