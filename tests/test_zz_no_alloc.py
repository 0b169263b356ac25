"""mk_decode_step_static (working memory in the library's fixed device array,
no allocation) against mk_decode_step on the same inputs, two steps in a row.

Each side appends to its own copy of the same prefilled cache, so both see the
same history.  Both calls launch the same kernel with the same plan, and every
sum in it has a fixed order (or is an exact fixed-point integer sum), so the
logits, argmax and the whole caches must be bitwise equal: a layout error in
the carved working memory that corrupts part of one buffer cannot hide inside
a tolerance.  This file is collected last on purpose: it must pass in a fresh
process and after every other GPU test.
"""
import ctypes
import dataclasses

import pytest
import torch

import decode_megakernel_06_b200 as mk
from synthetic import TINY, make_context_lengths, make_kv_cache, make_tokens, make_weights, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


def _run_pair(wl, null_logits: bool):
    m, B, T = wl.model, wl.batch, wl.tokens_per_step
    dev = torch.device("cuda:0")
    cap = wl.kv_capacity()
    w = make_weights(m, wl.seed, dev)
    k_a, v_a = make_kv_cache(m, B, cap, wl.seed, dev)
    k_b, v_b = k_a.clone(), v_a.clone()
    dec = mk.Decoder(m, w, max_rows=B * T, max_seqs=B, kv_capacity=cap, variant="megakernel")
    lengths = make_context_lengths(wl)
    toks = make_tokens(m.vocab, 2 * B * T, wl.seed, "no_alloc_tokens")
    M = B * T
    try:
        for step in range(2):
            pos = torch.tensor([n + step * T for n in lengths], dtype=torch.int32, device=dev)
            tok = torch.tensor(toks[step * M:(step + 1) * M], dtype=torch.int32, device=dev)
            logits_a = torch.empty((M, m.vocab), dtype=torch.float32, device=dev)
            logits_b = torch.empty_like(logits_a)
            am_a = torch.empty(M, dtype=torch.int32, device=dev)
            am_b = torch.empty_like(am_a)
            assert dec.step(tok, pos, B, T, k_a, v_a, logits_a, am_a) == mk.MK_OK, mk.mk_last_error()
            assert dec.status() == mk.MK_OK, mk.mk_last_error()
            rc = dec.step_static(tok, pos, B, T, k_b, v_b, None if null_logits else logits_b, am_b)
            assert rc == mk.MK_OK, mk.mk_last_error()
            assert dec.status() == mk.MK_OK, mk.mk_last_error()
            torch.cuda.synchronize()
            assert torch.equal(am_a, am_b), (step, am_a.tolist(), am_b.tolist())
            if not null_logits:
                assert torch.equal(logits_b, logits_a), step
            for b, n in enumerate(lengths):
                sl = slice(n + step * T, n + (step + 1) * T)
                for ca, cb in ((k_a, k_b), (v_a, v_b)):
                    assert torch.equal(cb[:, b, :, sl], ca[:, b, :, sl]), (step, b)
        # the caches agree everywhere else too (nothing outside the new rows moved)
        assert torch.equal(k_b, k_a) and torch.equal(v_b, v_a)
    finally:
        dec.close()


@pytest.mark.parametrize("kind,B", [("tiny", 1), ("small_batch", 4), ("verify", 1)])
def test_static_step_matches_decode_step(kind, B):
    _run_pair(workload(kind, B), null_logits=False)


def test_static_step_without_logits_buffer():
    """out_logits NULL: the logits live in the fixed array; argmax still agrees."""
    _run_pair(workload("small_batch", 2), null_logits=True)


def test_static_step_rejects_steps_beyond_the_array():
    """A step whose working memory exceeds MK_STATIC_SCRATCH_BYTES is refused on
    the host, before anything is launched, and the size it needs is named."""
    # the tiny model with one layer and a 1.1M-token vocabulary: 8 rows of
    # logits alone are 35 MB when the caller passes no logits buffer
    m = dataclasses.replace(TINY, name="wide_vocab", n_layers=1, vocab=1_100_000)
    dev = torch.device("cuda:0")
    w = make_weights(m, 0, dev)
    cap = 64
    k, v = make_kv_cache(m, 8, cap, 0, dev)
    dec = mk.Decoder(m, w, max_rows=8, max_seqs=8, kv_capacity=cap, variant="megakernel")
    try:
        tok = torch.zeros(8, dtype=torch.int32, device=dev)
        pos = torch.zeros(8, dtype=torch.int32, device=dev)
        am = torch.empty(8, dtype=torch.int32, device=dev)
        assert 8 * m.vocab * 4 > mk.MK_STATIC_SCRATCH_BYTES
        rc = dec.step_static(tok, pos, 8, 1, k, v, None, am)
        assert rc == mk.MK_ERR_CAPACITY
        msg = mk.mk_last_error()
        assert "static scratch" in msg and str(mk.MK_STATIC_SCRATCH_BYTES) in msg
    finally:
        dec.close()


def test_static_step_is_declared_with_its_limit():
    import os
    import re

    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "include", "mk.h")).read()
    got = re.search(r"#define MK_STATIC_SCRATCH_BYTES \((\d+)u << (\d+)\)", hdr)
    assert got and int(got.group(1)) << int(got.group(2)) == mk.MK_STATIC_SCRATCH_BYTES
    assert isinstance(mk.lib().mk_decode_step_static, ctypes._CFuncPtr)
