"""Python binding of ``libmk.so``, the fused MoE decode-step library for B200.

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of ``libmk.so``; PyTorch supplies device memory and streams.  The
ctypes functions carry the names of the C entry points in ``include/mk.h``;
``Decoder`` is a thin convenience wrapper that takes torch tensors.

There is no fallback: if ``libmk.so`` is missing or fails to load, every call
raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, List, Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmk.so")

MK_OK = 0
MK_ERR_ARG = -1
MK_ERR_CAPACITY = -2
MK_ERR_CUDA = -3
MK_ERR_LAUNCH = -4
MK_ERR_TIMEOUT = -5
MK_ERR_DEVICE_CHECK = -6
MK_ERR_UNSUPPORTED = -7

MK_MEGAKERNEL = 0
MK_MULTIKERNEL = 1
MK_MULTIKERNEL_GRAPH = 2
MK_TENSORCORE = 3
VARIANTS = {"megakernel": MK_MEGAKERNEL, "multikernel": MK_MULTIKERNEL,
            "multikernel_graph": MK_MULTIKERNEL_GRAPH, "tensorcore": MK_TENSORCORE}

MK_FAULT_NONE = 0
MK_FAULT_UNREACHABLE_WAIT = 1
MK_TRACE_WORDS = 12  # uint64 words per (op, warp) record of mk_set_trace
MK_SAMPLE_PHASES = 12  # phase stamps of mk_sample_top_p_phases
MK_STATIC_SCRATCH_BYTES = 32 << 20  # the fixed working array of mk_decode_step_static

OP_NAMES = ["EMBED", "QKV", "ATTN", "OPROJ", "SHARED_GU", "ROUTED_GU", "DOWN", "COMBINE", "LMHEAD"]


class mk_model_desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "n_layers", "d_model", "n_q_heads", "n_kv_heads", "head_dim",
        "n_experts", "top_k", "expert_ffn", "shared_ffn", "vocab")] + [
        ("rope_theta", ctypes.c_float), ("rms_eps", ctypes.c_float),
        ("max_rows", ctypes.c_int32), ("max_seqs", ctypes.c_int32),
        ("kv_capacity", ctypes.c_int32), ("variant", ctypes.c_int32)]


class mk_layer_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "attn_norm", "wqkv", "wo", "ffn_norm", "router", "w_gate", "w_up", "w_down",
        "ws_gate", "ws_up", "ws_down")]


class mk_weights(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("final_norm", ctypes.c_void_p),
                ("lm_head", ctypes.c_void_p), ("layers", ctypes.POINTER(mk_layer_weights))]


class mk_kv_cache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p)]


class mk_stats(ctypes.Structure):
    _fields_ = [("steps", ctypes.c_uint64), ("expert_union_total", ctypes.c_uint64),
                ("kernel_launches", ctypes.c_uint64), ("graph_launches", ctypes.c_uint64)]


class mk_plan_info(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "n_ops", "n_cta", "warps_per_cta", "rows_per_tile", "mmax", "attn_chunk",
        "attn_qsplit", "smem_bytes")] + [("scratch_bytes", ctypes.c_int64)]


class MkError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"mk error {code}: {msg}")
        self.code = code


_lib = None
_I32P = ctypes.POINTER(ctypes.c_int32)


def lib():
    """Load ``libmk.so``; raise if it is missing (no fallback exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with decode_megakernel_06_b200/build.py")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64
    sig = {
        "mk_create": (i32, [ctypes.POINTER(mk_model_desc), ctypes.POINTER(mk_weights), ctypes.POINTER(vp)]),
        "mk_decode_step": (i32, [vp, vp, vp, i32, i32, mk_kv_cache, vp, vp, vp]),
        "mk_decode_steps": (i32, [vp, vp, vp, i32, i32, mk_kv_cache, vp, vp, vp]),
        "mk_verify_steps": (i32, [vp, vp, vp, i32, i32, i32, vp, i32, mk_kv_cache, vp, vp, vp, vp]),
        "mk_decode_step_host": (i32, [vp, _I32P, _I32P, i32, i32, mk_kv_cache, vp, _I32P, vp]),
        "mk_decode_step_static": (i32, [vp, vp, vp, i32, i32, mk_kv_cache, vp, vp, vp]),
        "mk_sample_top_p": (i32, [vp, i32, i32, ctypes.c_float, ctypes.c_float, vp, vp, vp]),
        "mk_sample_top_p_phases": (i32, [vp, i32, i32, ctypes.c_float, ctypes.c_float, vp, vp, vp, vp]),
        "mk_decode_step_sample": (i32, [vp, vp, vp, i32, i32, mk_kv_cache, vp, ctypes.c_float,
                                        ctypes.c_float, vp, vp, vp]),
        "mk_decode_steps_sample": (i32, [vp, vp, vp, i32, i32, mk_kv_cache, vp, ctypes.c_float,
                                         ctypes.c_float, vp, vp, vp]),
        "mk_get_device_status": (i32, [vp, vp]),
        "mk_last_device_error_op": (i32, [vp]),
        "mk_last_error": (ctypes.c_char_p, []),
        "mk_destroy": (None, [vp]),
        "mk_set_variant": (i32, [vp, i32]),
        "mk_set_timeout": (i32, [vp, u64]),
        "mk_set_debug": (i32, [vp, vp, vp, vp]),
        "mk_debug_inject": (i32, [vp, i32]),
        "mk_set_trace": (i32, [vp, vp]),
        "mk_get_stats": (i32, [vp, ctypes.POINTER(mk_stats), i32]),
        "mk_hbm_read_probe": (i32, [vp, u64, i32, i32, ctypes.POINTER(ctypes.c_double), vp]),
        "mk_validate_desc": (i32, [ctypes.POINTER(mk_model_desc)]),
        "mk_plan_describe": (i32, [ctypes.POINTER(mk_model_desc), i32, i32, i32,
                                   ctypes.POINTER(mk_plan_info), _I32P, _I32P, _I32P, _I32P, i32]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def mk_last_error() -> str:
    return lib().mk_last_error().decode()


def _check(rc: int) -> int:
    if rc != MK_OK:
        raise MkError(rc, mk_last_error())
    return rc


# ---- same-named wrappers of the C entry points ---------------------------------

def mk_validate_desc(desc: mk_model_desc) -> int:
    return lib().mk_validate_desc(ctypes.byref(desc))


def mk_plan_describe(desc: mk_model_desc, n_sm: int, B: int, T: int):
    """Returns (rc, mk_plan_info, [(type, layer, dep0, dep1)] per op)."""
    info = mk_plan_info()
    n = 8 * desc.n_layers + 2  # an upper bound on the schedule's length
    arrs = [(ctypes.c_int32 * n)() for _ in range(4)]
    rc = lib().mk_plan_describe(ctypes.byref(desc), n_sm, B, T, ctypes.byref(info),
                                *[ctypes.cast(a, _I32P) for a in arrs], n)
    ops = list(zip(*[list(a)[:info.n_ops] for a in arrs])) if rc == MK_OK else []
    return rc, info, ops


def mk_create(desc: mk_model_desc, weights: mk_weights) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    _check(lib().mk_create(ctypes.byref(desc), ctypes.byref(weights), ctypes.byref(h)))
    return h


def mk_decode_steps(h, tokens: int, positions: int, B: int, n_steps: int, kv: mk_kv_cache,
                    out_logits: int, out_tokens: int, stream: int) -> int:
    """n_steps greedy steps in one launch (see include/mk.h)."""
    return lib().mk_decode_steps(h, tokens, positions, B, n_steps, kv, out_logits, out_tokens, stream)


def mk_verify_steps(h, tokens: int, positions: int, B: int, T: int, n_steps: int, drafts: int,
                    draft_len: int, kv: mk_kv_cache, out_logits: int, out_tokens: int,
                    out_accepted: int, stream: int) -> int:
    """n_steps speculative-verify steps in one launch (see include/mk.h)."""
    return lib().mk_verify_steps(h, tokens, positions, B, T, n_steps, drafts, draft_len, kv, out_logits,
                                 out_tokens, out_accepted, stream)


def mk_decode_step(h, tokens: int, positions: int, B: int, T: int, kv: mk_kv_cache,
                   out_logits: int, out_argmax: int, stream: int) -> int:
    return lib().mk_decode_step(h, tokens, positions, B, T, kv, out_logits, out_argmax, stream)


def mk_decode_step_host(h, tokens_host, positions_host, B: int, T: int, kv: mk_kv_cache,
                        out_logits: int, out_argmax_host, stream: int) -> int:
    return lib().mk_decode_step_host(h, tokens_host, positions_host, B, T, kv, out_logits,
                                     out_argmax_host, stream)


def mk_decode_step_static(h, tokens: int, positions: int, B: int, T: int, kv: mk_kv_cache,
                          out_logits: int, out_argmax: int, stream: int) -> int:
    return lib().mk_decode_step_static(h, tokens, positions, B, T, kv, out_logits, out_argmax,
                                       stream)


def mk_sample_top_p(logits: int, rows: int, vocab: int, temperature: float, top_p: float,
                    uniforms: int, out_tokens: int, stream: int) -> int:
    return lib().mk_sample_top_p(logits, rows, vocab, temperature, top_p, uniforms, out_tokens, stream)


def mk_sample_top_p_phases(logits: int, rows: int, vocab: int, temperature: float, top_p: float,
                           uniforms: int, out_tokens: int, stamps: int, stream: int = 0) -> int:
    return lib().mk_sample_top_p_phases(logits, rows, vocab, temperature, top_p, uniforms, out_tokens, stamps,
                                        stream)


def mk_decode_step_sample(h, tokens: int, positions: int, B: int, T: int, kv: mk_kv_cache,
                          out_logits: int, temperature: float, top_p: float, uniforms: int,
                          out_tokens: int, stream: int) -> int:
    return lib().mk_decode_step_sample(h, tokens, positions, B, T, kv, out_logits, temperature, top_p,
                                       uniforms, out_tokens, stream)


def mk_decode_steps_sample(h, tokens: int, positions: int, B: int, n_steps: int, kv: mk_kv_cache,
                           out_logits: int, temperature: float, top_p: float, uniforms: int,
                           out_tokens: int, stream: int) -> int:
    """n_steps sampled steps as one graph launch (see include/mk.h)."""
    return lib().mk_decode_steps_sample(h, tokens, positions, B, n_steps, kv, out_logits, temperature, top_p,
                                        uniforms, out_tokens, stream)


def _need(t, dtype, min_numel: int, name: str, device=None, dims: Optional[int] = None):
    """Check a tensor handed to a kernel by its data pointer: dtype, a
    contiguous layout with at least ``min_numel`` elements, optionally the
    number of dimensions, then that it lives on ``device`` (a CUDA device).
    A wrong tensor would otherwise make the kernel read or write past it."""
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if dims is not None and t.dim() != dims:
        raise ValueError(f"{name}: {t.dim()}-D, expected {dims}-D")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if t.numel() < min_numel:
        raise ValueError(f"{name}: {t.numel()} elements, at least {min_numel} needed")
    if t.device.type != "cuda" or (device is not None and t.device != device):
        raise ValueError(f"{name}: on {t.device}, expected " + (str(device) if device is not None else "a CUDA device"))


def sample_top_p(logits, temperature: float, top_p: float, uniforms, out_tokens, stream=None) -> int:
    """Torch-tensor form of mk_sample_top_p: logits fp32 [rows, vocab], uniforms
    fp64 [rows] (or None when temperature <= 0), out_tokens int32 [rows], all
    contiguous on one CUDA device (checked: ValueError otherwise).  Returns the
    launch status code."""
    import torch

    _need(logits, torch.float32, 1, "logits", dims=2)
    rows, vocab = logits.shape
    if uniforms is not None:
        _need(uniforms, torch.float64, rows, "uniforms", logits.device)
    _need(out_tokens, torch.int32, rows, "out_tokens", logits.device)
    s = stream if stream is not None else torch.cuda.current_stream()
    return mk_sample_top_p(logits.data_ptr(), rows, vocab, temperature, top_p, _ptr(uniforms),
                           out_tokens.data_ptr(), s.cuda_stream)


def sample_top_p_phases(logits, temperature: float, top_p: float, uniforms, out_tokens, stamps, stream=None) -> int:
    """sample_top_p, also writing the device clock (ns) at each of the
    MK_SAMPLE_PHASES phase boundaries of row 0 into ``stamps`` (int64 CUDA
    tensor of at least MK_SAMPLE_PHASES elements; see mk_sample_top_p_phases).
    The same checks as sample_top_p; returns the launch status code."""
    import torch

    _need(logits, torch.float32, 1, "logits", dims=2)
    rows, vocab = logits.shape
    if uniforms is not None:
        _need(uniforms, torch.float64, rows, "uniforms", logits.device)
    _need(out_tokens, torch.int32, rows, "out_tokens", logits.device)
    _need(stamps, torch.int64, MK_SAMPLE_PHASES, "stamps", logits.device)
    s = stream if stream is not None else torch.cuda.current_stream()
    return mk_sample_top_p_phases(logits.data_ptr(), rows, vocab, temperature, top_p, _ptr(uniforms),
                                  out_tokens.data_ptr(), stamps.data_ptr(), s.cuda_stream)


def hbm_read_probe(buf, form: int = 0, reps: int = 5, stream=None) -> float:
    """Read-only HBM bandwidth in GB/s over the CUDA tensor ``buf`` (16-byte
    aligned, >= 64 MiB; see mk_hbm_read_probe).  Raises on failure."""
    import torch

    if buf.device.type != "cuda" or not buf.is_contiguous():
        raise ValueError("buf must be a contiguous CUDA tensor")
    s = stream if stream is not None else torch.cuda.current_stream()
    out = ctypes.c_double(0.0)
    _check(lib().mk_hbm_read_probe(buf.data_ptr(), buf.numel() * buf.element_size(), form, reps,
                                   ctypes.byref(out), s.cuda_stream))
    return out.value


def mk_get_device_status(h, stream: int) -> int:
    return lib().mk_get_device_status(h, stream)


def mk_last_device_error_op(h) -> int:
    return lib().mk_last_device_error_op(h)


def mk_destroy(h) -> None:
    lib().mk_destroy(h)


def mk_set_variant(h, variant: int) -> int:
    return lib().mk_set_variant(h, variant)


def mk_set_timeout(h, ns: int) -> int:
    return lib().mk_set_timeout(h, ns)


def mk_set_debug(h, hidden: int, expert_ids: int, expert_w: int) -> int:
    return lib().mk_set_debug(h, hidden, expert_ids, expert_w)


def mk_set_trace(h, trace: int) -> int:
    return lib().mk_set_trace(h, trace)


def mk_debug_inject(h, fault: int) -> int:
    return lib().mk_debug_inject(h, fault)


def mk_get_stats(h, reset: bool = False) -> mk_stats:
    s = mk_stats()
    _check(lib().mk_get_stats(h, ctypes.byref(s), 1 if reset else 0))
    return s


# ---- convenience wrapper over torch tensors -------------------------------------

def make_desc(model, max_rows: int, max_seqs: int, kv_capacity: int,
              variant: int = MK_MEGAKERNEL) -> mk_model_desc:
    """Descriptor from any object with the decoder's dimension attributes."""
    return mk_model_desc(model.n_layers, model.d_model, model.n_q_heads, model.n_kv_heads,
                         model.head_dim, model.n_experts, model.top_k, model.expert_ffn,
                         model.shared_ffn, model.vocab, float(model.rope_theta),
                         float(model.rms_eps), max_rows, max_seqs, kv_capacity, variant)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


class Decoder:
    """A handle over torch-resident weights (dict as produced by the synthetic
    generator: embed, final_norm, lm_head, layers[...])."""

    def __init__(self, model, weights: Dict[str, object], max_rows: int, max_seqs: int,
                 kv_capacity: int, variant: str = "megakernel"):
        import torch

        self.model = model
        self.max_rows, self.max_seqs, self.kv_capacity = max_rows, max_seqs, kv_capacity
        self.desc = make_desc(model, max_rows, max_seqs, kv_capacity, VARIANTS[variant])
        layers = (mk_layer_weights * model.n_layers)()
        for l, lw in enumerate(weights["layers"]):
            layers[l] = mk_layer_weights(*[_ptr(lw.get(n)) for n in (
                "attn_norm", "wqkv", "wo", "ffn_norm", "router", "w_gate", "w_up", "w_down",
                "ws_gate", "ws_up", "ws_down")])
        self._layers = layers
        self._weights = weights
        self.w = mk_weights(_ptr(weights["embed"]), _ptr(weights["final_norm"]),
                            _ptr(weights["lm_head"]), layers)
        self.h = mk_create(self.desc, self.w)
        self._torch = torch

    def close(self):
        if self.h:
            mk_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_variant(self, variant: str):
        _check(mk_set_variant(self.h, VARIANTS[variant]))

    def set_timeout(self, ns: int):
        _check(mk_set_timeout(self.h, ns))

    def set_debug(self, hidden=None, expert_ids=None, expert_w=None):
        _check(mk_set_debug(self.h, _ptr(hidden), _ptr(expert_ids), _ptr(expert_w)))

    def set_trace(self, trace=None):
        _check(mk_set_trace(self.h, _ptr(trace)))

    def inject(self, fault: int):
        _check(mk_debug_inject(self.h, fault))

    def _io(self, tokens, positions, B: int, rows: int, k_cache, v_cache, logits=None):
        """The checks every device-tensor call shares (ValueError on a mismatch)."""
        t = self._torch
        _need(tokens, t.int32, rows, "tokens")
        dev = tokens.device
        _need(positions, t.int32, B, "positions", dev)
        kv_numel = (self.model.n_layers * self.max_seqs * self.model.n_kv_heads * self.kv_capacity
                    * self.model.head_dim)
        _need(k_cache, t.bfloat16, kv_numel, "k_cache", dev)
        _need(v_cache, t.bfloat16, kv_numel, "v_cache", dev)
        if logits is not None:
            _need(logits, t.float32, rows * self.model.vocab, "logits", dev)
        return dev

    def step(self, tokens, positions, B: int, T: int, k_cache, v_cache, logits, argmax,
             stream=None) -> int:
        """Enqueue one step (device tensors); returns the launch status code."""
        dev = self._io(tokens, positions, B, B * T, k_cache, v_cache, logits)
        _need(argmax, self._torch.int32, B * T, "argmax", dev)
        s = stream if stream is not None else self._torch.cuda.current_stream()
        kv = mk_kv_cache(k_cache.data_ptr(), v_cache.data_ptr())
        return mk_decode_step(self.h, tokens.data_ptr(), positions.data_ptr(), B, T, kv,
                              _ptr(logits), argmax.data_ptr(), s.cuda_stream)

    def step_sample(self, tokens, positions, B: int, T: int, k_cache, v_cache, logits, temperature: float,
                    top_p: float, uniforms, out_tokens, stream=None) -> int:
        """One step whose next tokens are sampled (temperature / top-p) from its
        logits with the given fp64 uniforms [B*T].  Returns the launch status code."""
        dev = self._io(tokens, positions, B, B * T, k_cache, v_cache, logits)
        if uniforms is not None:
            _need(uniforms, self._torch.float64, B * T, "uniforms", dev)
        _need(out_tokens, self._torch.int32, B * T, "out_tokens", dev)
        s = stream if stream is not None else self._torch.cuda.current_stream()
        kv = mk_kv_cache(k_cache.data_ptr(), v_cache.data_ptr())
        return mk_decode_step_sample(self.h, tokens.data_ptr(), positions.data_ptr(), B, T, kv,
                                     _ptr(logits), temperature, top_p, _ptr(uniforms),
                                     out_tokens.data_ptr(), s.cuda_stream)

    def steps_sample(self, tokens, positions, B: int, n_steps: int, k_cache, v_cache, logits,
                     temperature: float, top_p: float, uniforms, out_tokens, stream=None) -> int:
        """n_steps sampled steps as one graph launch; uniforms is fp64
        [n_steps, B] (None for greedy), out_tokens int32 [n_steps, B] on the
        device.  Returns the launch status code."""
        dev = self._io(tokens, positions, B, B, k_cache, v_cache, logits)
        if uniforms is not None:
            _need(uniforms, self._torch.float64, n_steps * B, "uniforms", dev)
        _need(out_tokens, self._torch.int32, n_steps * B, "out_tokens", dev)
        s = stream if stream is not None else self._torch.cuda.current_stream()
        kv = mk_kv_cache(k_cache.data_ptr(), v_cache.data_ptr())
        return mk_decode_steps_sample(self.h, tokens.data_ptr(), positions.data_ptr(), B, n_steps, kv,
                                      _ptr(logits), temperature, top_p, _ptr(uniforms),
                                      out_tokens.data_ptr(), s.cuda_stream)

    def steps(self, tokens, positions, B: int, n_steps: int, k_cache, v_cache, logits, out_tokens,
              stream=None) -> int:
        """Enqueue n_steps greedy steps as one launch; out_tokens is int32
        [n_steps, B] on the device.  Returns the launch status code."""
        dev = self._io(tokens, positions, B, B, k_cache, v_cache, logits)
        _need(out_tokens, self._torch.int32, n_steps * B, "out_tokens", dev)
        s = stream if stream is not None else self._torch.cuda.current_stream()
        kv = mk_kv_cache(k_cache.data_ptr(), v_cache.data_ptr())
        return mk_decode_steps(self.h, tokens.data_ptr(), positions.data_ptr(), B, n_steps, kv,
                               _ptr(logits), out_tokens.data_ptr(), s.cuda_stream)

    def verify_steps(self, tokens, positions, B: int, T: int, n_steps: int, drafts, k_cache, v_cache,
                     logits, out_tokens, out_accepted, stream=None) -> int:
        """Enqueue n_steps verify blocks of T rows as one launch; drafts is int32
        [B, draft_len] on the device, out_tokens [n_steps, B*T], out_accepted
        [n_steps, B].  Returns the launch status code."""
        dev = self._io(tokens, positions, B, B * T, k_cache, v_cache, logits)
        _need(drafts, self._torch.int32, B * drafts.shape[-1], "drafts", dev, dims=2)
        _need(out_tokens, self._torch.int32, n_steps * B * T, "out_tokens", dev)
        _need(out_accepted, self._torch.int32, n_steps * B, "out_accepted", dev)
        s = stream if stream is not None else self._torch.cuda.current_stream()
        kv = mk_kv_cache(k_cache.data_ptr(), v_cache.data_ptr())
        return mk_verify_steps(self.h, tokens.data_ptr(), positions.data_ptr(), B, T, n_steps,
                               drafts.data_ptr(), drafts.shape[-1], kv, _ptr(logits),
                               out_tokens.data_ptr(), out_accepted.data_ptr(), s.cuda_stream)

    def step_static(self, tokens, positions, B: int, T: int, k_cache, v_cache, logits, argmax,
                    stream=None) -> int:
        """Like ``step``, but the step's working memory is the library's fixed
        device array (no allocation; overlapping calls on one device race)."""
        dev = self._io(tokens, positions, B, B * T, k_cache, v_cache, logits)
        _need(argmax, self._torch.int32, B * T, "argmax", dev)
        s = stream if stream is not None else self._torch.cuda.current_stream()
        kv = mk_kv_cache(k_cache.data_ptr(), v_cache.data_ptr())
        return mk_decode_step_static(self.h, tokens.data_ptr(), positions.data_ptr(), B, T, kv,
                                     _ptr(logits), argmax.data_ptr(), s.cuda_stream)

    def step_host(self, tokens_host, positions_host, B: int, T: int, k_cache, v_cache,
                  argmax_host, logits=None, stream=None) -> int:
        """Host-buffer step: int32 CPU tensors in/out (pinned is fastest)."""
        s = stream if stream is not None else self._torch.cuda.current_stream()
        kv = mk_kv_cache(k_cache.data_ptr(), v_cache.data_ptr())
        cast = lambda t: ctypes.cast(t.data_ptr(), _I32P)  # noqa: E731
        return mk_decode_step_host(self.h, cast(tokens_host), cast(positions_host), B, T, kv,
                                   _ptr(logits), cast(argmax_host), s.cuda_stream)

    def status(self, stream=None) -> int:
        s = stream if stream is not None else self._torch.cuda.current_stream()
        return mk_get_device_status(self.h, s.cuda_stream)

    def stats(self, reset: bool = False) -> mk_stats:
        return mk_get_stats(self.h, reset)
