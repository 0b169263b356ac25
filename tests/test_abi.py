"""The C ABI on the host: the library loads, exports every declared entry point,
validates descriptors and plans schedules -- all without a GPU."""
import ctypes
import os
import re

import pytest

import decode_megakernel_06_b200 as mk
from synthetic import LARGE, SMALL, TINY

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    if not os.path.exists(mk.LIB_PATH):
        from decode_megakernel_06_b200 import build

        build.build()
    return mk.lib()


def declared_symbols():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"MK_API\s+[\w\s\*]+?\b(mk_\w+)\s*\(", src)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(L):
    names = declared_symbols()
    assert "mk_create" in names and "mk_decode_step" in names
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/ but not exported"


def test_only_declared_symbols_are_exported(L):
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", mk.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l and l.split()[-1].startswith("mk_")}
    assert exported == set(declared_symbols())


def _desc(model=TINY, **kw):
    d = mk.make_desc(model, max_rows=kw.pop("max_rows", 8), max_seqs=kw.pop("max_seqs", 8),
                     kv_capacity=kw.pop("kv_capacity", 256))
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_validate_accepts_the_workload_models(L):
    for m in (TINY, SMALL, LARGE):
        assert mk.mk_validate_desc(_desc(m)) == mk.MK_OK, mk.mk_last_error()


@pytest.mark.parametrize("field,value,code", [
    ("n_layers", 0, mk.MK_ERR_ARG),
    ("d_model", 12, mk.MK_ERR_ARG),
    ("n_kv_heads", 3, mk.MK_ERR_ARG),
    ("head_dim", 96, mk.MK_ERR_UNSUPPORTED),
    ("n_experts", 300, mk.MK_ERR_UNSUPPORTED),
    ("top_k", 9, mk.MK_ERR_ARG),
    ("expert_ffn", 40, mk.MK_ERR_ARG),
    ("shared_ffn", 8, mk.MK_ERR_ARG),
    ("max_rows", 65, mk.MK_ERR_UNSUPPORTED),
    ("max_seqs", 0, mk.MK_ERR_ARG),
    ("variant", 4, mk.MK_ERR_ARG),
    ("rope_theta", 0.0, mk.MK_ERR_ARG),
])
def test_validate_rejects(L, field, value, code):
    assert mk.mk_validate_desc(_desc(**{field: value})) == code
    assert mk.mk_last_error() != "ok"


@pytest.mark.parametrize("B", [1, 2])
def test_schedule_is_a_dag_with_the_data_dependencies(L, B):
    """Every op waits only for earlier ops, and for each op the ops producing
    its inputs are reachable through its waits."""
    d = _desc(SMALL, kv_capacity=2112, max_seqs=B, max_rows=B)
    rc, info, ops = mk.mk_plan_describe(d, 148, B, 1)
    assert rc == mk.MK_OK, mk.mk_last_error()
    Lyr = SMALL.n_layers
    assert info.n_ops == len(ops) == 7 * Lyr + 2
    names = [mk.OP_NAMES[t] for t, *_ in ops]
    assert names[0] == "EMBED" and names[-1] == "LMHEAD"
    assert names[1:8] == ["QKV", "ATTN", "OPROJ", "SHARED_GU", "ROUTED_GU", "DOWN", "COMBINE"]
    idx = {(mk.OP_NAMES[t], l): i for i, (t, l, _, _) in enumerate(ops)}
    reach = []
    for i, (t, layer, d0, d1) in enumerate(ops):
        assert d0 < i and d1 < i
        r = set()
        for dep in (d0, d1):
            if dep >= 0:
                r |= {dep} | reach[dep]
        reach.append(r)
    end = "COMBINE"
    for l in range(Lyr):
        # the residual entering layer l: the embedding, or the previous layer's end
        prev_h = [idx[("EMBED", -1)]] if l == 0 else [idx[(end, l - 1)], idx[("OPROJ", l - 1)]]
        need = {
            "QKV": prev_h,
            "ATTN": [idx[("QKV", l)]],
            "OPROJ": [idx[("ATTN", l)], idx[("QKV", l)]],
            "SHARED_GU": [idx[("OPROJ", l)]],
            "ROUTED_GU": [idx[("OPROJ", l)]],  # router sums complete with the o-projection
            "DOWN": [idx[("SHARED_GU", l)], idx[("ROUTED_GU", l)], idx[("OPROJ", l)]],
            "COMBINE": [idx[("DOWN", l)]],
        }
        for name, deps in need.items():
            for dep in deps:
                assert dep in reach[idx[(name, l)]], (name, l, dep)
        # OPROJ rewrites h_mid and clears the expert-output sums: every reader of
        # the previous layer's (the staging of this QKV, or COMBINE) comes first
        assert idx[("QKV", l)] in reach[idx[("OPROJ", l)]]
        if l > 0:
            assert idx[(end, l - 1)] in reach[idx[("OPROJ", l)]]
    assert idx[(end, Lyr - 1)] in reach[idx[("LMHEAD", -1)]]


@pytest.mark.parametrize("model,B,T,cap", [(TINY, 1, 1, 256), (SMALL, 1, 1, 2112),
                                           (SMALL, 8, 1, 2112), (SMALL, 1, 7, 2560),
                                           (LARGE, 1, 1, 4160), (LARGE, 8, 1, 4160)])
def test_plan_shapes(L, model, B, T, cap):
    d = _desc(model, kv_capacity=cap, max_seqs=B, max_rows=B * T)
    rc, info, _ = mk.mk_plan_describe(d, 148, B, T)
    assert rc == mk.MK_OK, mk.mk_last_error()
    M = B * T
    assert info.mmax >= M and info.mmax in (1, 2, 4, 8)
    assert info.rows_per_tile == 4
    ppt = 2048 // model.head_dim
    assert info.attn_chunk % ppt == 0 and info.attn_chunk >= ppt
    assert -(-cap // (info.warps_per_cta * info.attn_chunk)) <= 32    # one merge level over CTA chunks
    G = model.n_q_heads // model.n_kv_heads
    assert info.attn_qsplit == -(-G * T // 4)
    assert info.smem_bytes <= 227 * 1024
    assert info.n_cta == 148 and 4 <= info.warps_per_cta <= 8   # compute warps (the rest issue TMA loads)


def test_plan_rejects_shapes_beyond_the_handle(L):
    d = _desc(TINY, max_rows=4, max_seqs=2)
    assert mk.mk_plan_describe(d, 148, 3, 1)[0] == mk.MK_ERR_CAPACITY
    assert mk.mk_plan_describe(d, 148, 2, 3)[0] == mk.MK_ERR_CAPACITY
    assert mk.mk_plan_describe(d, 148, 2, 2)[0] == mk.MK_OK


def test_create_fails_cleanly_without_a_gpu(L):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    d = _desc(TINY)
    lw = (mk.mk_layer_weights * TINY.n_layers)()
    for l in range(TINY.n_layers):
        lw[l] = mk.mk_layer_weights(*([16] * 8 + [None] * 3))
    w = mk.mk_weights(16, 16, 16, lw)
    h = ctypes.c_void_p()
    rc = L.mk_create(ctypes.byref(d), ctypes.byref(w), ctypes.byref(h))
    assert rc == mk.MK_ERR_CUDA and not h.value
    assert "cuda" in mk.mk_last_error().lower() or "device" in mk.mk_last_error().lower()


def test_null_arguments_are_rejected(L):
    assert L.mk_create(None, None, None) == mk.MK_ERR_ARG
    assert L.mk_get_device_status(None, None) == mk.MK_ERR_ARG
    assert L.mk_set_timeout(None, 5) == mk.MK_ERR_ARG
    kv = mk.mk_kv_cache(None, None)
    assert L.mk_decode_step(None, None, None, 1, 1, kv, None, None, None) == mk.MK_ERR_ARG
    L.mk_destroy(None)  # safe on NULL


def test_sampler_checks_its_arguments_on_the_host(L):
    """mk_sample_top_p rejects bad arguments before any CUDA call (the pointers
    below are never dereferenced)."""
    lg, u, out = 256, 512, 768  # stand-in addresses: every call here fails its host checks
    nan = float("nan")
    assert L.mk_sample_top_p(None, 1, 10, 1.0, 0.9, u, out, None) == mk.MK_ERR_ARG
    assert L.mk_sample_top_p(lg, 1, 10, 1.0, 0.9, u, None, None) == mk.MK_ERR_ARG
    assert L.mk_sample_top_p(lg, 0, 10, 1.0, 0.9, u, out, None) == mk.MK_ERR_ARG
    assert L.mk_sample_top_p(lg, 1, 0, 1.0, 0.9, u, out, None) == mk.MK_ERR_ARG
    assert L.mk_sample_top_p(lg, 1, 10, nan, 0.9, u, out, None) == mk.MK_ERR_ARG
    assert L.mk_sample_top_p(lg, 1, 10, 1.0, nan, u, out, None) == mk.MK_ERR_ARG
    assert L.mk_sample_top_p(lg, 1, 10, 0.7, 0.9, None, out, None) == mk.MK_ERR_ARG
    assert L.mk_sample_top_p(lg, 1, 131073, 1.0, 0.9, u, out, None) == mk.MK_ERR_UNSUPPORTED
    assert "131072" in mk.mk_last_error()
    st = 1024  # the phase-stamped form: the same checks, and its stamps
    assert L.mk_sample_top_p_phases(lg, 1, 10, 1.0, 0.9, u, out, None, None) == mk.MK_ERR_ARG
    assert "stamps" in mk.mk_last_error()
    assert L.mk_sample_top_p_phases(None, 1, 10, 1.0, 0.9, u, out, st, None) == mk.MK_ERR_ARG
    assert L.mk_sample_top_p_phases(lg, 1, 10, 0.7, 0.9, None, out, st, None) == mk.MK_ERR_ARG
    assert L.mk_sample_top_p_phases(lg, 1, 131073, 1.0, 0.9, u, out, st, None) == mk.MK_ERR_UNSUPPORTED
    kv = mk.mk_kv_cache(None, None)
    assert L.mk_decode_step_sample(None, None, None, 1, 1, kv, None, 1.0, 0.9, u, out, None) == mk.MK_ERR_ARG
    assert L.mk_decode_steps_sample(None, None, None, 1, 2, kv, None, 1.0, 0.9, u, out, None) == mk.MK_ERR_ARG


def test_torch_wrappers_check_tensors_before_any_launch():
    """The torch-tensor wrappers hand raw data pointers to the kernels, so they
    check dtype, layout, size and device first: a float32 or short uniforms
    vector, or a strided logits view, would otherwise be read past its end."""
    import torch

    lg = torch.zeros((4, 100), dtype=torch.float32)
    u = torch.zeros(4, dtype=torch.float64)
    out = torch.zeros(4, dtype=torch.int32)
    with pytest.raises(ValueError, match="dtype"):
        mk.sample_top_p(lg.double(), 1.0, 0.9, u, out)
    with pytest.raises(ValueError, match="2-D"):
        mk.sample_top_p(lg.view(-1), 1.0, 0.9, u, out)
    with pytest.raises(ValueError, match="contiguous"):
        mk.sample_top_p(lg.t(), 1.0, 0.9, u, out)
    with pytest.raises(ValueError, match="CUDA|cuda"):
        mk.sample_top_p(lg, 1.0, 0.9, u, out)  # CPU tensors never reach the library
    stamps = torch.zeros(mk.MK_SAMPLE_PHASES, dtype=torch.int64)
    with pytest.raises(ValueError, match="CUDA|cuda"):
        mk.sample_top_p_phases(lg, 1.0, 0.9, u, out, stamps)
    with pytest.raises(ValueError, match="dtype"):
        mk._need(stamps.int(), torch.int64, mk.MK_SAMPLE_PHASES, "stamps")
    with pytest.raises(ValueError, match="at least"):
        mk._need(stamps[:5], torch.int64, mk.MK_SAMPLE_PHASES, "stamps")
    with pytest.raises(ValueError, match="dtype"):
        mk._need(u.float(), torch.float64, 4, "uniforms")
    with pytest.raises(ValueError, match="at least 4"):
        mk._need(u[:3], torch.float64, 4, "uniforms")
    with pytest.raises(ValueError, match="dtype"):
        mk._need(out.long(), torch.int32, 4, "out_tokens")
