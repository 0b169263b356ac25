"""The oracle's single ops against hand-worked closed-form cases.

The cases (tests/golden/ops_hand_worked.json) are derived by hand from each
op's definition; each carries its derivation and the passage it follows.
"""
import json
import os

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
with open(os.path.join(HERE, "golden", "ops_hand_worked.json")) as fh:
    GOLDEN = json.load(fh)


def bf(a):
    """Exact bf16 bits of small test values (all are bf16-representable)."""
    import oracle

    a = np.asarray(a, dtype=np.float32)
    bits = oracle.bf16_round(a)
    assert np.array_equal(oracle.bf16_to_f32(bits), a), "golden weights must be bf16-exact"
    return bits


@pytest.mark.parametrize("case", GOLDEN["cases"], ids=lambda c: f"{c['op']}:{c['name']}")
def test_golden(case, oracle_lib):
    o = oracle_lib
    op = case["op"]
    if op == "matvec":
        got = o.matvec(bf(case["W"]), case["x"])
        np.testing.assert_allclose(got, case["expected"], rtol=0, atol=case["tol"])
    elif op == "rmsnorm":
        got = o.rmsnorm(case["h"], bf(case["g"]), case["eps"])
        np.testing.assert_allclose(got, case["expected"], rtol=case["tol"], atol=case["tol"])
    elif op == "rope":
        got = o.rope(case["v"], case["pos"], case["theta"])
        np.testing.assert_allclose(got, case["expected"], rtol=0, atol=case["tol"])
    elif op == "attend":
        got = o.attend(case["q"], bf(case["K"]), bf(case["V"]))
        np.testing.assert_allclose(got, case["expected"], rtol=0, atol=case["tol"])
    elif op == "topk_softmax":
        ids, w = o.topk_softmax(case["z"], case["k"])
        assert list(ids) == case["expected_ids"]
        np.testing.assert_allclose(w, case["expected_w"], rtol=0, atol=case["tol"])
    elif op == "swiglu":
        got = o.swiglu(bf(case["Wg"]), bf(case["Wu"]), bf(case["Wd"]), case["y"])
        np.testing.assert_allclose(got, case["expected"], rtol=case["tol"], atol=case["tol"])
    elif op == "argmax":
        assert o.argmax(case["v"]) == case["expected"]
    else:
        raise AssertionError(f"unknown op {op}")


def test_bf16_rounding_is_nearest_even(oracle_lib):
    o = oracle_lib
    # 1 + 2^-8 lies exactly between bf16 neighbours 1 and 1 + 2^-7: ties to even -> 1.
    # 1 + 3*2^-8 lies between 1 + 2^-7 and 1 + 2^-6 (even): ties to even -> 1 + 2^-6.
    vals = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -8 + 2 ** -20, -2.5, 0.0],
                    dtype=np.float32)
    want = np.array([1.0, 1 + 2 ** -6, 1 + 2 ** -7, -2.5, 0.0], dtype=np.float32)
    np.testing.assert_array_equal(o.bf16_to_f32(o.bf16_round(vals)), want)
