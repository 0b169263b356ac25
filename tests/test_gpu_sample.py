"""Temperature / top-p sampling on the GPU against the oracle, through the C ABI.

mk_sample_top_p decides in exact fixed-point integers, as the oracle does, so
on the same logits and uniforms the tokens must agree exactly.  The only
freedom is the last ulp of the fp64 exponential (CUDA's and the host's), which
moves a mass by at most one fixed-point unit: draws whose oracle margin is
within 64 units of a boundary are not compared (none are expected).

mk_decode_step_sample is the decode step followed by the sampler: its tokens
must equal the sampler run on the step's own logits, and, where the oracle's
margin exceeds what the step's logits error can move, the oracle's draw on
the oracle's logits.
"""
import math

import numpy as np
import pytest
import torch

import decode_megakernel_06_b200 as mk
from oracle import sample as osample
from synthetic import TINY, Workload, make_context_lengths, make_logits, make_tokens, make_uniforms

from parity import Session, relerr

pytestmark = pytest.mark.gpu

FIXED_POINT_SLACK = 64


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


def _gpu_sample(logits: np.ndarray, T, top_p, u):
    dev = torch.device("cuda:0")
    lg = torch.from_numpy(np.ascontiguousarray(logits, np.float32)).to(dev)
    uu = None if u is None else torch.tensor(np.asarray(u, np.float64), device=dev)
    out = torch.full((lg.shape[0],), -7, dtype=torch.int32, device=dev)
    rc = mk.sample_top_p(lg, T, top_p, uu, out)
    assert rc == mk.MK_OK, mk.mk_last_error()
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _compare(logits, T, top_p, u):
    got = _gpu_sample(logits, T, top_p, u)
    checked = 0
    for r in range(logits.shape[0]):
        ref = osample.sample_top_p(logits[r], T, top_p, 0.0 if u is None else float(u[r]))
        if not ref.robust(FIXED_POINT_SLACK):
            continue
        assert int(got[r]) == ref.token, (r, T, top_p, int(got[r]), ref)
        checked += 1
    return checked


# (rows, vocab, sigma): the large and small models' vocabularies, ragged sizes,
# the largest row the sampler takes, fewer tokens than CTAs in a cluster, one token
CASES = [(1, 64000, 1.0), (3, 64000, 4.0), (8, 32000, 1.0), (2, 4099, 2.0), (4, 1001, 1.0),
         (1, 131072, 1.0), (5, 7, 1.0), (2, 1, 1.0), (3, 1024, 0.3)]


@pytest.mark.parametrize("rows,vocab,sigma", CASES, ids=[f"r{c[0]}_v{c[1]}_s{c[2]}" for c in CASES])
def test_sampler_matches_oracle(rows, vocab, sigma):
    logits = make_logits(rows, vocab, sigma, seed=31).numpy()
    total = checked = 0
    for i, (T, top_p) in enumerate([(t, p) for t in (0.0, 0.6, 1.0, 2.0) for p in (0.0, 0.5, 0.9, 1.0)]):
        u = make_uniforms(rows, seed=32 + i)
        checked += _compare(logits, T, top_p, u)
        total += rows
    assert checked >= total - max(1, total // 100), (checked, total)


def test_batch_of_64_rows():
    logits = make_logits(64, 64000, 1.0, seed=33).numpy()
    u = make_uniforms(64, seed=34)
    assert _compare(logits, 1.0, 0.9, u) >= 63


def test_edge_rows():
    V = 3000
    rng_rows = make_logits(6, V, 1.0, seed=35).numpy()
    rows = np.stack([
        np.zeros(V, np.float32),                              # all tied
        np.round(rng_rows[1] * 2) / 2,                        # many ties
        np.where(rng_rows[2] > 0, np.float32(0.0), np.float32(-0.0)),  # +0 and -0 only
        rng_rows[3] * 50.0,                                   # very peaked
        rng_rows[4] * 1e-3,                                   # nearly flat
        -np.abs(rng_rows[5]) - 1e4,                           # far from zero
    ]).astype(np.float32)
    for T, top_p in ((1.0, 0.5), (0.5, 0.9), (1.0, 5.0), (1.0, -1.0), (3.0, 0.999)):
        for u in ([0.0] * 6, [float(np.nextafter(1.0, 0.0))] * 6, make_uniforms(6, seed=36)):
            got = _gpu_sample(rows, T, top_p, u)
            for r in range(rows.shape[0]):
                ref = osample.sample_top_p(rows[r], T, top_p, u[r])
                assert int(got[r]) == ref.token, (r, T, top_p, u[r], int(got[r]), ref)


def test_greedy_without_uniforms():
    logits = make_logits(4, 5000, 1.0, seed=37).numpy()
    logits[2, 100] = logits[2, 4000] = logits[2].max() + 1.0  # tie at the top
    for T in (0.0, -1.0):
        got = _gpu_sample(logits, T, 0.9, None)
        for r in range(4):
            assert int(got[r]) == osample.greedy(logits[r])
    assert int(got[2]) == 100


def test_repeatable():
    logits = make_logits(8, 64000, 1.0, seed=38).numpy()
    u = make_uniforms(8, seed=39)
    a = _gpu_sample(logits, 0.8, 0.9, u)
    b = _gpu_sample(logits, 0.8, 0.9, u)
    assert np.array_equal(a, b)


def test_phase_stamped_sampler_draws_the_same_tokens():
    """mk_sample_top_p_phases is the same launch with the device clock written
    at its 12 phase boundaries: it draws the same tokens as mk_sample_top_p,
    and its stamps are in order."""
    dev = torch.device("cuda:0")
    logits = make_logits(8, 64000, 1.0, seed=40).numpy()
    u = make_uniforms(8, seed=41)
    ref = _gpu_sample(logits, 0.8, 0.9, u)
    lg = torch.from_numpy(np.ascontiguousarray(logits, np.float32)).to(dev)
    uu = torch.tensor(np.asarray(u, np.float64), device=dev)
    out = torch.full((8,), -7, dtype=torch.int32, device=dev)
    stamps = torch.zeros(mk.MK_SAMPLE_PHASES, dtype=torch.int64, device=dev)
    assert mk.sample_top_p_phases(lg, 0.8, 0.9, uu, out, stamps) == mk.MK_OK, mk.mk_last_error()
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), ref)
    t = stamps.cpu().tolist()
    assert t[0] > 0 and all(b >= a for a, b in zip(t, t[1:])), t
    assert t[-1] - t[0] < 10_000_000, t  # well under 10 ms for one 64000-wide row


def test_rejects_bad_arguments():
    dev = torch.device("cuda:0")
    lg = torch.zeros((2, 10), dtype=torch.float32, device=dev)
    u = torch.zeros(2, dtype=torch.float64, device=dev)
    out = torch.zeros(2, dtype=torch.int32, device=dev)
    s = torch.cuda.current_stream().cuda_stream
    assert mk.mk_sample_top_p(lg.data_ptr(), 0, 10, 1.0, 0.9, u.data_ptr(), out.data_ptr(), s) == mk.MK_ERR_ARG
    assert mk.mk_sample_top_p(lg.data_ptr(), 2, 0, 1.0, 0.9, u.data_ptr(), out.data_ptr(), s) == mk.MK_ERR_ARG
    assert mk.mk_sample_top_p(lg.data_ptr(), 2, 10, 1.0, float("nan"), u.data_ptr(), out.data_ptr(), s) == mk.MK_ERR_ARG
    assert mk.mk_sample_top_p(lg.data_ptr(), 2, 10, 1.0, 0.9, None, out.data_ptr(), s) == mk.MK_ERR_ARG
    assert mk.mk_sample_top_p(lg.data_ptr(), 2, 10, 1.0, 0.9, u.data_ptr(), None, s) == mk.MK_ERR_ARG
    assert mk.mk_sample_top_p(lg.data_ptr(), 1, 131073, 1.0, 0.9, u.data_ptr(), out.data_ptr(), s) == \
        mk.MK_ERR_UNSUPPORTED
    assert mk.mk_sample_top_p(lg.data_ptr(), 2, 10, 1.0, 0.9, u.data_ptr(), out.data_ptr(), s) == mk.MK_OK
    torch.cuda.synchronize()


def test_decode_step_sample_against_oracle():
    """The sampled step on the tiny model, 4 ragged sequences: equal to the
    sampler on the step's own logits, and to the oracle's draw on the oracle's
    logits wherever the logits' error cannot move the decision."""
    wl = Workload("tiny_b4_sample", TINY, 4, 1, context=None, context_range=(20, 120), steps=2, seed=21)
    s = Session(wl)
    s.dec.set_debug(None, None, None)
    positions = make_context_lengths(wl)
    tokens = make_tokens(s.m.vocab, 4, wl.seed)
    ref = s.oracle_step(tokens, positions)
    dev = s.dev
    tok = torch.tensor(tokens, dtype=torch.int32, device=dev)
    pos = torch.tensor(positions, dtype=torch.int32, device=dev)
    out = torch.empty(4, dtype=torch.int32, device=dev)
    again = torch.empty(4, dtype=torch.int32, device=dev)
    checked = total = 0
    for i, (T, top_p) in enumerate([(1.0, 0.9), (0.7, 0.5), (0.3, 0.95), (0.1, 0.8), (1.5, 1.0), (0.0, 0.9)]):
        for trial in range(4):
            u = torch.tensor(make_uniforms(4, seed=40 + 10 * i + trial), dtype=torch.float64, device=dev)
            rc = s.dec.step_sample(tok, pos, 4, 1, s.k, s.v, s.logits, T, top_p, u, out)
            assert rc == mk.MK_OK, mk.mk_last_error()
            assert s.dec.status() == mk.MK_OK
            assert mk.sample_top_p(s.logits, T, top_p, u, again) == mk.MK_OK
            torch.cuda.synchronize()
            assert torch.equal(out, again)
            logits = s.logits.cpu().numpy()
            err = relerr(logits, ref.logits)
            assert err <= 1e-5, err
            delta = err * float(np.abs(ref.logits).max())
            uh = u.cpu().numpy()
            for r in range(4):
                o = osample.sample_top_p(ref.logits[r], T, top_p, float(uh[r]))
                total += 1
                bound = 0 if T <= 0 else 2 * o.total_mass * math.expm1(2 * delta / T) + FIXED_POINT_SLACK
                if T > 0 and not o.robust(int(bound)):
                    continue
                if T <= 0 and np.sort(ref.logits[r])[-1] - np.sort(ref.logits[r])[-2] <= 2 * delta:
                    continue
                assert int(out[r]) == o.token, (T, top_p, r, int(out[r]), o)
                checked += 1
    s.close()
    assert checked >= total // 2, (checked, total)
    print("decode+sample checked", checked, "of", total)


def test_sampled_loop_equals_single_sampled_steps():
    """mk_decode_steps_sample (n sampled steps as one graph launch) against n
    mk_decode_step_sample calls, each fed the previous call's tokens: the same
    tokens, final logits and caches, bit for bit; the graph's replay too."""
    wl = Workload("tiny_b4_sample_loop", TINY, 4, 1, context=None, context_range=(20, 120), steps=8, seed=22)
    n, B = 6, 4
    s = Session(wl)
    s.dec.set_debug(None, None, None)
    dev = s.dev
    p0 = make_context_lengths(wl)
    tok0 = torch.tensor(make_tokens(s.m.vocab, B, wl.seed), dtype=torch.int32, device=dev)
    u = torch.tensor(make_uniforms(n * B, seed=77), dtype=torch.float64, device=dev).view(n, B)
    T, top_p = 0.8, 0.9
    k0, v0 = s.k.clone(), s.v.clone()
    ref = torch.empty((n, B), dtype=torch.int32, device=dev)
    tok = tok0.clone()
    for st in range(n):
        pos = torch.tensor([p + st for p in p0], dtype=torch.int32, device=dev)
        assert s.dec.step_sample(tok, pos, B, 1, s.k, s.v, s.logits, T, top_p, u[st].contiguous(), ref[st]) == mk.MK_OK
        tok = ref[st].clone()
    assert s.dec.status() == mk.MK_OK
    ref_logits = s.logits.clone()
    k1, v1 = s.k.clone(), s.v.clone()
    for rep in range(2):  # the first call records the graph, the second replays it
        s.k.copy_(k0)
        s.v.copy_(v0)
        out = torch.full((n, B), -7, dtype=torch.int32, device=dev)
        pos0 = torch.tensor(p0, dtype=torch.int32, device=dev)
        s.dec.stats(reset=True)
        assert s.dec.steps_sample(tok0, pos0, B, n, s.k, s.v, s.logits, T, top_p, u, out) == mk.MK_OK, mk.mk_last_error()
        assert s.dec.status() == mk.MK_OK
        st = s.dec.stats(reset=True)
        print("graph launches", st.graph_launches, "kernels", st.kernel_launches)
        assert torch.equal(out, ref), (rep, out, ref)
        assert torch.equal(s.logits.view(torch.int32), ref_logits.view(torch.int32)), "final logits differ"
        assert torch.equal(s.k.view(torch.int16), k1.view(torch.int16)), "K cache differs"
        assert torch.equal(s.v.view(torch.int16), v1.view(torch.int16)), "V cache differs"
    s.close()
