"""Speculative verify with acceptance and rollback on the device
(mk_verify_steps): N blocks of T rows in one persistent launch.

Each step of the launch is the verify step of mk_decode_step, so N steps in
one launch must give bit for bit the accepted tokens, counts, final logits and
caches of N single-step calls with the acceptance done on the host.  With the
oracle's own greedy continuation as drafts every draft is accepted (outside
near ties), so the accepted tokens must be the oracle's greedy decode.
"""
import numpy as np
import pytest
import torch

import decode_megakernel_06_b200 as mk
from oracle import step as ostep
from synthetic import TINY, Workload, make_context_lengths, make_tokens, workload

from parity import MARGIN, Session

pytestmark = pytest.mark.gpu

T = 7


def _verify_workload(name):
    """Blocks of T rows for one sequence: the tiny model, or the small one."""
    if name == "tiny":
        return Workload("tiny_verify", TINY, 1, T, 127, steps=16, seed=0)
    return workload("verify", 1)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


def _host_loop(s: Session, first, p0, drafts, n):
    """n single-step verify calls, acceptance on the host."""
    dev = s.dev
    logits = torch.empty((T, s.m.vocab), dtype=torch.float32, device=dev)
    am = torch.empty(T, dtype=torch.int32, device=dev)
    last, p = first, p0
    toks, accs = [], []
    for _ in range(n):
        blk = [last] + [int(drafts[p - p0 + t]) for t in range(1, T)]
        rc = s.dec.step(torch.tensor(blk, dtype=torch.int32, device=dev),
                        torch.tensor([p], dtype=torch.int32, device=dev), 1, T, s.k, s.v, logits, am)
        assert rc == mk.MK_OK, mk.mk_last_error()
        row = am.cpu().numpy()
        a = 1
        while a < T and blk[a] == int(row[a - 1]):
            a += 1
        toks.append([int(row[t]) if t < a else -1 for t in range(T)])
        accs.append(a)
        last, p = int(row[a - 1]), p + a
    assert s.dec.status() == mk.MK_OK
    return np.array(toks), np.array(accs), logits.cpu().numpy()


def _launch(s: Session, first, p0, drafts, n):
    dev = s.dev
    blk = [first] + [int(drafts[t]) for t in range(1, T)]
    tok = torch.tensor(blk, dtype=torch.int32, device=dev)
    pos = torch.tensor([p0], dtype=torch.int32, device=dev)
    dr = torch.tensor(np.asarray(drafts)[None, :], dtype=torch.int32, device=dev)
    logits = torch.empty((T, s.m.vocab), dtype=torch.float32, device=dev)
    out = torch.empty((n, T), dtype=torch.int32, device=dev)
    acc = torch.empty((n, 1), dtype=torch.int32, device=dev)
    rc = s.dec.verify_steps(tok, pos, 1, T, n, dr, s.k, s.v, logits, out, acc)
    assert rc == mk.MK_OK, mk.mk_last_error()
    st = s.dec.status()
    assert st == mk.MK_OK, (st, mk.mk_last_error())
    return out.cpu().numpy(), acc.cpu().numpy()[:, 0], logits.cpu().numpy()


def _random_drafts(m, n, seed):
    """Uniform random drafts for n blocks (draft j for position p0 + j)."""
    return np.array(make_tokens(m.vocab, n * T + T, seed, name="drafts"), dtype=np.int64)


@pytest.mark.parametrize("name,n", [("tiny", 8), ("small", 4)])
def test_launch_equals_host_loop(name, n):
    wl = _verify_workload(name)
    s = Session(wl, capacity=wl.kv_capacity() + n * T + T)
    s.dec.set_debug(None, None, None)
    p0 = make_context_lengths(wl)[0]
    first = make_tokens(s.m.vocab, 1, wl.seed)[0]
    # drafts: random, except that a run of the host loop's own accepted tokens
    # is planted so that some steps accept several drafts
    drafts = _random_drafts(s.m, n, wl.seed)
    k0, v0 = s.k.clone(), s.v.clone()
    probe, _, _ = _host_loop(s, first, p0, drafts, 1)
    s.k.copy_(k0)
    s.v.copy_(v0)
    drafts[1] = probe[0][0]  # the first draft now matches the model's first prediction
    ref_tok, ref_acc, ref_logits = _host_loop(s, first, p0, drafts, n)
    k1, v1 = s.k.clone(), s.v.clone()
    s.k.copy_(k0)
    s.v.copy_(v0)
    got_tok, got_acc, got_logits = _launch(s, first, p0, drafts, n)
    np.testing.assert_array_equal(got_acc, ref_acc)
    np.testing.assert_array_equal(got_tok, ref_tok)
    assert np.array_equal(got_logits.view(np.uint32), ref_logits.view(np.uint32)), "final logits differ"
    assert torch.equal(s.k.view(torch.int16), k1.view(torch.int16)), "K cache differs"
    assert torch.equal(s.v.view(torch.int16), v1.view(torch.int16)), "V cache differs"
    assert ref_acc[0] >= 2, ref_acc
    s.close()
    print(name, "accepted", got_acc.tolist())


def test_oracle_drafts_are_all_accepted():
    """Drafts = the oracle's greedy continuation: every block is accepted in
    full, and the accepted tokens are the oracle's, up to its first near tie."""
    wl = _verify_workload("tiny")
    n = 5
    s = Session(wl, capacity=wl.kv_capacity() + n * T + T)
    s.dec.set_debug(None, None, None)
    p0 = make_context_lengths(wl)[0]
    first = make_tokens(s.m.vocab, 1, wl.seed)[0]
    # the oracle's greedy decode from (first, p0) on its own copy of the cache
    greedy = [first]
    tok, pos, tied = [first], [p0], None
    for i in range(n * T + 1):
        ref = ostep.decode_step(s.m, s.src, s.k_host, s.v_host, tok, pos, 1, 1)  # one row per step
        top2 = np.sort(ref.logits[0])[-2:]
        if tied is None and top2[1] - top2[0] <= MARGIN:
            tied = i
        tok, pos = [int(ref.argmax[0])], [pos[0] + 1]
        greedy.append(tok[0])
    drafts = np.array(greedy, dtype=np.int64)  # drafts[j] = the oracle's token at position p0 + j
    got_tok, got_acc, _ = _launch(s, first, p0, drafts, n)
    limit = n * T if tied is None else tied
    accepted = [t for row in got_tok for t in row if t >= 0]
    assert len(accepted) == int(got_acc.sum())
    assert accepted[:limit] == greedy[1:1 + min(limit, len(accepted))]
    if tied is None:
        assert got_acc.tolist() == [T] * n, got_acc
    s.close()


def _host_loop_batch(s: Session, firsts, p0s, drafts, n):
    """n single-step verify calls of B sequences, acceptance on the host."""
    dev, B = s.dev, len(firsts)
    logits = torch.empty((B * T, s.m.vocab), dtype=torch.float32, device=dev)
    am = torch.empty(B * T, dtype=torch.int32, device=dev)
    last, p = list(firsts), list(p0s)
    toks = np.full((n, B * T), -1, dtype=np.int64)
    accs = np.zeros((n, B), dtype=np.int64)
    for st in range(n):
        blk = []
        for b in range(B):
            blk += [last[b]] + [int(drafts[b][p[b] - p0s[b] + t]) for t in range(1, T)]
        rc = s.dec.step(torch.tensor(blk, dtype=torch.int32, device=dev),
                        torch.tensor(p, dtype=torch.int32, device=dev), B, T, s.k, s.v, logits, am)
        assert rc == mk.MK_OK, mk.mk_last_error()
        row = am.cpu().numpy()
        for b in range(B):
            a = 1
            while a < T and blk[b * T + a] == int(row[b * T + a - 1]):
                a += 1
            toks[st, b * T:b * T + a] = row[b * T:b * T + a]
            accs[st, b] = a
            last[b], p[b] = int(row[b * T + a - 1]), p[b] + a
    assert s.dec.status() == mk.MK_OK
    return toks, accs, logits.cpu().numpy()


@pytest.mark.parametrize("name,B,n", [("tiny", 2, 6), ("small", 8, 3)])
def test_wide_launch_equals_host_loop(name, B, n):
    """Blocks above 8 rows (2 x 7 on the tiny model, 8 x 7 on the small one):
    the tensor-core sequence with acceptance on the device, n blocks in one
    graph launch, against n single-step calls with host acceptance."""
    wl = Workload("tiny_verify_b2", TINY, B, T, 127, steps=16, seed=0) if name == "tiny" else workload("verify", B)
    s = Session(wl, capacity=wl.kv_capacity() + n * T + T)
    s.dec.set_debug(None, None, None)
    dev = s.dev
    p0s = make_context_lengths(wl)
    firsts = make_tokens(s.m.vocab, B, wl.seed)
    drafts = np.stack([np.array(make_tokens(s.m.vocab, n * T + T, wl.seed + b, name="drafts"), dtype=np.int64)
                       for b in range(B)])
    k0, v0 = s.k.clone(), s.v.clone()
    probe, _, _ = _host_loop_batch(s, firsts, p0s, drafts, 1)
    s.k.copy_(k0)
    s.v.copy_(v0)
    for b in range(B):  # each sequence's first draft matches the model's first prediction
        drafts[b][1] = probe[0][b * T]
    ref_tok, ref_acc, ref_logits = _host_loop_batch(s, firsts, p0s, drafts, n)
    k1, v1 = s.k.clone(), s.v.clone()
    s.k.copy_(k0)
    s.v.copy_(v0)
    blk = []
    for b in range(B):
        blk += [firsts[b]] + [int(drafts[b][t]) for t in range(1, T)]
    logits = torch.empty((B * T, s.m.vocab), dtype=torch.float32, device=dev)
    out = torch.empty((n, B * T), dtype=torch.int32, device=dev)
    acc = torch.empty((n, B), dtype=torch.int32, device=dev)
    rc = s.dec.verify_steps(torch.tensor(blk, dtype=torch.int32, device=dev),
                            torch.tensor(p0s, dtype=torch.int32, device=dev), B, T, n,
                            torch.tensor(drafts, dtype=torch.int32, device=dev), s.k, s.v, logits, out, acc)
    assert rc == mk.MK_OK, mk.mk_last_error()
    assert s.dec.status() == mk.MK_OK, mk.mk_last_error()
    np.testing.assert_array_equal(acc.cpu().numpy(), ref_acc)
    np.testing.assert_array_equal(out.cpu().numpy(), ref_tok)
    assert np.array_equal(logits.cpu().numpy().view(np.uint32), ref_logits.view(np.uint32)), "final logits differ"
    assert torch.equal(s.k.view(torch.int16), k1.view(torch.int16)), "K cache differs"
    assert torch.equal(s.v.view(torch.int16), v1.view(torch.int16)), "V cache differs"
    assert (ref_acc[0] >= 2).all(), ref_acc
    s.close()
    print(name, B, "accepted", acc.cpu().numpy().tolist())


def test_verify_launch_rejects_bad_arguments():
    wl = _verify_workload("tiny")
    s = Session(wl, capacity=wl.kv_capacity() + 64)
    s.dec.set_debug(None, None, None)
    dev = s.dev
    tok = torch.zeros(T, dtype=torch.int32, device=dev)
    pos = torch.tensor([20], dtype=torch.int32, device=dev)
    out = torch.empty((2, T), dtype=torch.int32, device=dev)
    acc = torch.empty((2, 1), dtype=torch.int32, device=dev)
    short = torch.zeros((1, T), dtype=torch.int32, device=dev)  # draft_len < n_steps * T
    assert s.dec.verify_steps(tok, pos, 1, T, 2, short, s.k, s.v, None, out, acc) == mk.MK_ERR_ARG
    ok = torch.zeros((1, 2 * T), dtype=torch.int32, device=dev)
    assert s.dec.verify_steps(tok[:1], pos, 1, 1, 2, ok, s.k, s.v, None, out, acc) == mk.MK_ERR_ARG
    assert s.dec.verify_steps(tok, pos, 1, T, 2, ok, s.k, s.v, None, out, acc) == mk.MK_OK
    assert s.dec.status() == mk.MK_OK
    s.close()
