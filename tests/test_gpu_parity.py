"""CUDA decode step vs the CPU oracle on the workloads, through the C ABI.

Sizes the oracle finishes in seconds run several steps element by element;
the large model runs at full size with whole steps checked (the oracle fetches
only the experts each step routes to).
"""
import numpy as np
import pytest
import torch

import decode_megakernel_06_b200 as mk
from synthetic import ModelConfig, Workload, workload

from parity import Session, relerr, run_greedy, run_verify

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    torch.cuda.set_device(0)


@pytest.mark.parametrize("variant", ["megakernel", "multikernel", "multikernel_graph"])
def test_tiny_greedy_16_steps(variant):
    s = Session(workload("tiny"), variant=variant)
    rep = run_greedy(s, 16)
    s.close()
    assert rep.argmax_checked >= 14 and rep.expert_checked > 0
    print(variant, rep)


def test_small_bs1_greedy():
    s = Session(workload("small"))
    rep = run_greedy(s, 12)
    s.close()
    assert rep.argmax_checked >= 10
    print(rep)


@pytest.mark.parametrize("B", [2, 4, 8])
def test_small_batch_random_lengths(B):
    s = Session(workload("small_batch", B))
    rep = run_greedy(s, 4)
    s.close()
    print(B, rep)


def test_verify_block_t7():
    s = Session(workload("verify", 1))
    rep = run_verify(s, 4)
    s.close()
    print(rep)


# Shapes off the tile grid: d not a multiple of 256, vocab not a multiple of 16,
# fewer experts than a tile's rows, hd = 64, expert_ffn not a multiple of 256.
RAGGED = ModelConfig("ragged", n_layers=2, d_model=264, n_q_heads=6, n_kv_heads=2, head_dim=64,
                     n_experts=6, top_k=2, expert_ffn=48, shared_ffn=32, vocab=1000, sigma=0.05)


@pytest.mark.parametrize("B,T", [(1, 1), (3, 1), (8, 1), (2, 3), (1, 8)])
def test_ragged_shapes(B, T):
    wl = Workload(f"ragged_b{B}_t{T}", RAGGED, B, T, context=None, context_range=(1, 70),
                  steps=3, seed=7)
    s = Session(wl, capacity=96)
    rep = run_greedy(s, 3) if T == 1 else run_verify(s, 3)
    s.close()
    print(B, T, rep)


# Blocks of more than 8 rows take the tensor-core launch sequence: the
# speculative verify block of 8 sequences x 7 rows on the small model, and the
# ragged model (K = 264, F = 48, Fs = 32 off every 64-column tile) at 15, 64
# and 16 x 4 rows.
def test_verify_block_56_rows():
    s = Session(workload("verify", 8))
    rep = run_verify(s, 2)
    s.close()
    assert rep.rows_compared >= 56
    print(rep)


@pytest.mark.parametrize("B,T", [(3, 5), (8, 8), (16, 4)])
def test_ragged_wide_blocks(B, T):
    wl = Workload(f"ragged_wide_b{B}_t{T}", RAGGED, B, T, context=None, context_range=(1, 70), steps=3, seed=11)
    s = Session(wl, capacity=96)
    rep = run_greedy(s, 2) if T == 1 else run_verify(s, 2)
    s.close()
    assert rep.rows_compared >= B * T
    print(B, T, rep)


def test_wide_block_more_query_vectors_than_one_tile():
    """One sequence of 48 rows: 48 x 3 = 144 query vectors per KV head, more
    than one 128-row tile of the tensor-core attention, over contexts of
    several 128-position chunks."""
    wl = Workload("ragged_wide_b1_t48", RAGGED, 1, 48, context=None, context_range=(200, 330), steps=3, seed=13)
    s = Session(wl, capacity=512)
    rep = run_verify(s, 2)
    s.close()
    assert rep.rows_compared >= 48
    print(rep)


@pytest.mark.parametrize("B,T", [(8, 1), (2, 3), (1, 2)])
def test_tensorcore_variant_small_blocks(B, T):
    """MK_TENSORCORE: blocks of 2 to 8 rows on the tensor-core launch sequence
    (the ragged model), against the oracle."""
    wl = Workload(f"ragged_tc_b{B}_t{T}", RAGGED, B, T, context=None, context_range=(1, 70), steps=3, seed=14)
    s = Session(wl, variant="tensorcore", capacity=96)
    rep = run_greedy(s, 2) if T == 1 else run_verify(s, 2)
    s.close()
    assert rep.rows_compared >= B * T
    print(B, T, rep)


def test_wide_block_rejects_bad_inputs_on_device():
    wl = Workload("ragged_wide_bad", RAGGED, 4, 4, context=None, context_range=(1, 40), steps=1, seed=12)
    s = Session(wl, capacity=64)
    dev = s.dev
    tok = torch.full((16,), 3, dtype=torch.int32, device=dev)
    tok[5] = RAGGED.vocab
    pos = torch.tensor([10, 10, 10, 10], dtype=torch.int32, device=dev)
    assert s.dec.step(tok, pos, 4, 4, s.k, s.v, s.logits, s.argmax) == mk.MK_OK
    assert s.dec.status() == mk.MK_ERR_DEVICE_CHECK
    tok[5] = 1
    assert s.dec.step(tok, pos, 4, 4, s.k, s.v, s.logits, s.argmax) == mk.MK_OK
    assert s.dec.status() == mk.MK_OK
    s.close()


def test_empty_cache_and_full_capacity():
    """Position 0 (the token attends only itself) and a block ending exactly at
    the last cache slot."""
    wl = Workload("edge", RAGGED, 2, 1, context=None, context_range=(0, 0), steps=1, seed=9)
    s = Session(wl, capacity=64)
    rep = run_greedy(s, 2)
    from parity import compare_step, Report
    import numpy as np

    toks = [3, 5]
    pos = [0, 63]
    ref = s.oracle_step(toks, pos)
    got = s.gpu_step(toks, pos)
    compare_step(s, ref, got, Report(), np.ones(2, dtype=bool), pos)
    s.close()


def test_variants_agree_bitwise():
    """The three execution variants run the same math in the same order."""
    wl = workload("tiny")
    outs = []
    for variant in ("megakernel", "multikernel", "multikernel_graph"):
        s = Session(wl, variant=variant)
        pos = [wl.context]
        got = []
        for st in range(3):
            got.append(s.gpu_step([11 + st], [pos[0] + st])[0].copy())
        outs.append(got)
        s.close()
    for a, b in zip(outs[0], outs[1]):
        np.testing.assert_array_equal(a, b)
    for a, b in zip(outs[0], outs[2]):
        np.testing.assert_array_equal(a, b)


def test_invalid_inputs_are_rejected_on_device():
    wl = workload("tiny")
    s = Session(wl)
    dev = s.dev
    bad_tok = torch.tensor([wl.model.vocab], dtype=torch.int32, device=dev)
    pos = torch.tensor([wl.context], dtype=torch.int32, device=dev)
    assert s.dec.step(bad_tok, pos, 1, 1, s.k, s.v, s.logits, s.argmax) == mk.MK_OK
    assert s.dec.status() == mk.MK_ERR_DEVICE_CHECK
    ok_tok = torch.tensor([1], dtype=torch.int32, device=dev)
    bad_pos = torch.tensor([s.cap], dtype=torch.int32, device=dev)
    assert s.dec.step(ok_tok, bad_pos, 1, 1, s.k, s.v, s.logits, s.argmax) == mk.MK_OK
    assert s.dec.status() == mk.MK_ERR_DEVICE_CHECK
    # host-side capacity checks of the library itself (the torch wrapper would
    # already refuse the one-token buffer for B = 2)
    kv = mk.mk_kv_cache(s.k.data_ptr(), s.v.data_ptr())
    stream = torch.cuda.current_stream().cuda_stream
    rc = mk.mk_decode_step(s.dec.h, ok_tok.data_ptr(), pos.data_ptr(), 2, 1, kv, s.logits.data_ptr(),
                           s.argmax.data_ptr(), stream)
    assert rc == mk.MK_ERR_CAPACITY
    with pytest.raises(ValueError):
        s.dec.step(ok_tok, pos, 2, 1, s.k, s.v, s.logits, s.argmax)
    # and the handle still works
    rep = run_greedy(s, 2)
    s.close()


def test_bounded_wait_times_out_and_recovers():
    """An op waits for a count nothing will reach: the kernel gives up after
    the timeout, reports MK_ERR_TIMEOUT, and the next step is correct."""
    wl = workload("tiny")
    s = Session(wl)
    s.dec.set_timeout(20_000_000)  # 20 ms
    s.dec.inject(mk.MK_FAULT_UNREACHABLE_WAIT)
    t = torch.tensor([7], dtype=torch.int32, device=s.dev)
    p = torch.tensor([wl.context], dtype=torch.int32, device=s.dev)
    assert s.dec.step(t, p, 1, 1, s.k, s.v, s.logits, s.argmax) == mk.MK_OK
    assert s.dec.status() == mk.MK_ERR_TIMEOUT
    assert mk.mk_last_device_error_op(s.dec.h) >= 0
    # restore the cache the failed step may have touched, then run normally
    from synthetic import make_kv_cache

    k, v = make_kv_cache(wl.model, 1, s.cap, wl.seed, s.dev)
    s.k.copy_(k)
    s.v.copy_(v)
    rep = run_greedy(s, 2)
    s.close()


def test_host_buffer_entry_point_matches_device_entry_point():
    wl = workload("tiny")
    s = Session(wl)
    toks, pos = [42], [wl.context]
    logits_dev, am_dev = s.gpu_step(toks, pos)[:2]
    s2 = Session(wl)
    th = torch.tensor(toks, dtype=torch.int32).pin_memory()
    ph = torch.tensor(pos, dtype=torch.int32).pin_memory()
    out = torch.empty(1, dtype=torch.int32).pin_memory()
    rc = s2.dec.step_host(th, ph, 1, 1, s2.k, s2.v, out, logits=s2.logits)
    assert rc == mk.MK_OK, mk.mk_last_error()
    assert int(out[0]) == int(am_dev[0])
    np.testing.assert_array_equal(s2.logits.cpu().numpy(), logits_dev)
    s.close()
    s2.close()


@pytest.mark.parametrize("B", [1, 8])
def test_large_full_size(B):
    """The large model at full size (about 80 GB of bf16 weights), whole steps."""
    free, _ = torch.cuda.mem_get_info()
    if free < 90e9:
        pytest.skip("needs ~90 GB free device memory")
    s = Session(workload("large", B), cache_host_weights=False)
    rep = run_greedy(s, 2 if B == 1 else 1)
    s.close()
    del s
    torch.cuda.empty_cache()
    print(B, rep)
