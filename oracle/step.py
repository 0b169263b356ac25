"""Whole decode steps of the CPU oracle, layer by layer.

TEST INFRASTRUCTURE ONLY.  The orchestration is the plain loop of the step's
definition: embed, then per layer the attention half, the router and the
expert half, then the final norm, lm_head and argmax.  Weights come from a
source object that hands out host bytes (uint16 views of bf16); experts are
fetched only once the router has chosen them, so a model larger than host
memory can still be checked.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

from . import Dims, _f32, _u16, f32p, i32p, lib, u16p


def dims_of(model, max_seqs: int, kv_capacity: int) -> Dims:
    return Dims(model.d_model, model.n_q_heads, model.n_kv_heads, model.head_dim,
                model.n_experts, model.top_k, model.expert_ffn, model.shared_ffn,
                model.vocab, max_seqs, kv_capacity, model.rms_eps, model.rope_theta)


def _host_bits(t) -> np.ndarray:
    """Host uint16 bits of a bf16 torch tensor (any device) or a uint16 array."""
    if isinstance(t, np.ndarray):
        return _u16(t)
    import torch  # plumbing only: device -> host copy of generator output

    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


class WeightSource:
    """Hands out host bytes of the weights.

    ``weights`` is the dict produced by the synthetic generator (torch tensors on
    any device) or the same structure holding uint16 numpy arrays.  With
    ``cache=True`` host copies are kept; otherwise each request copies afresh
    and experts are copied one at a time.
    """

    def __init__(self, weights: Dict[str, object], cache: bool = True):
        self.w = weights
        self.cache = cache
        self._memo: Dict[tuple, np.ndarray] = {}
        self.fetched_bytes = 0

    def _get(self, key, fetch):
        if key in self._memo:
            return self._memo[key]
        a = fetch()
        self.fetched_bytes += a.nbytes
        if self.cache:
            self._memo[key] = a
        return a

    def top(self, name: str) -> np.ndarray:
        return self._get((name,), lambda: _host_bits(self.w[name]))

    def layer(self, l: int, name: str) -> Optional[np.ndarray]:
        t = self.w["layers"][l].get(name)
        if t is None:
            return None
        return self._get((name, l), lambda: _host_bits(t))

    def expert(self, l: int, name: str, e: int) -> np.ndarray:
        t = self.w["layers"][l][name]
        return self._get((name, l, e), lambda: _host_bits(t[e]))


@dataclass
class StepResult:
    logits: np.ndarray                 # [M][V] fp32
    argmax: np.ndarray                 # [M] int32
    hidden: np.ndarray                 # [L+1][M][d] fp32 (embedding, then after each layer)
    router_logits: np.ndarray          # [L][M][E]
    expert_ids: np.ndarray             # [L][M][k] selection order
    expert_w: np.ndarray               # [L][M][k]
    extra: dict = field(default_factory=dict)


def decode_step(model, src: WeightSource, k_cache: np.ndarray, v_cache: np.ndarray,
                tokens, positions, B: int, T: int) -> StepResult:
    """One decode step of ``M = B*T`` rows; ``k_cache``/``v_cache`` are updated in place.

    ``k_cache``/``v_cache``: uint16 ``[L][max_seqs][Hkv][capacity][hd]``.
    ``tokens``: ``M`` ids, row ``m = b*T + t``.  ``positions``: ``B`` ints, the
    cache index of each sequence's first new token.
    """
    L, d, E, k, V = model.n_layers, model.d_model, model.n_experts, model.top_k, model.vocab
    M = B * T
    assert k_cache.dtype == np.uint16 and k_cache.flags.c_contiguous
    assert v_cache.dtype == np.uint16 and v_cache.flags.c_contiguous
    max_seqs, cap = k_cache.shape[1], k_cache.shape[3]
    D = dims_of(model, max_seqs, cap)
    Dp = ctypes.byref(D)
    lb = lib()
    tok = np.ascontiguousarray(tokens, dtype=np.int32)
    pos = np.ascontiguousarray(positions, dtype=np.int32)
    assert tok.size == M and pos.size == B
    assert all(0 <= int(p) and int(p) + T <= cap for p in pos)

    h = np.empty((M, d), dtype=np.float32)
    embed = src.top("embed")
    lb.or_embed(ctypes.c_int(d), u16p(embed), ctypes.c_int(M), i32p(tok), f32p(h))
    hidden = np.empty((L + 1, M, d), dtype=np.float32)
    hidden[0] = h
    router_logits = np.empty((L, M, E), dtype=np.float32)
    ids = np.empty((L, M, k), dtype=np.int32)
    wts = np.empty((L, M, k), dtype=np.float32)
    y = np.empty((M, d), dtype=np.float32)

    for l in range(L):
        kc = k_cache[l]
        vc = v_cache[l]
        lb.or_attn_block(Dp, u16p(src.layer(l, "attn_norm")), u16p(src.layer(l, "wqkv")),
                         u16p(src.layer(l, "wo")), u16p(kc), u16p(vc), ctypes.c_int(B),
                         ctypes.c_int(T), i32p(pos), f32p(h))
        lb.or_ffn_route(Dp, u16p(src.layer(l, "ffn_norm")), u16p(src.layer(l, "router")),
                        ctypes.c_int(M), f32p(h), f32p(y), f32p(router_logits[l]),
                        i32p(ids[l]), f32p(wts[l]))
        keep = []
        PtrArr = ctypes.POINTER(ctypes.c_uint16) * (M * k)
        wg, wu, wd = PtrArr(), PtrArr(), PtrArr()
        for m in range(M):
            for j in range(k):
                e = int(ids[l, m, j])
                g_, u_, d_ = (src.expert(l, "w_gate", e), src.expert(l, "w_up", e),
                              src.expert(l, "w_down", e))
                keep += [g_, u_, d_]
                wg[m * k + j], wu[m * k + j], wd[m * k + j] = u16p(g_), u16p(u_), u16p(d_)
        sg, su, sd = (src.layer(l, "ws_gate"), src.layer(l, "ws_up"), src.layer(l, "ws_down"))
        null = ctypes.POINTER(ctypes.c_uint16)()
        lb.or_ffn_apply(Dp, ctypes.c_int(M), f32p(y), f32p(wts[l]), wg, wu, wd,
                        u16p(sg) if sg is not None else null,
                        u16p(su) if su is not None else null,
                        u16p(sd) if sd is not None else null, f32p(h))
        del keep
        hidden[l + 1] = h

    logits = np.empty((M, V), dtype=np.float32)
    am = np.empty(M, dtype=np.int32)
    lb.or_final(Dp, u16p(src.top("final_norm")), u16p(src.top("lm_head")), ctypes.c_int(M),
                f32p(h), f32p(logits), i32p(am))
    return StepResult(logits, am, hidden, router_logits, ids, wts)


def router_margins(router_logits: np.ndarray, k: int) -> np.ndarray:
    """Gap between the k-th and (k+1)-th largest router logits, per [layer][row]."""
    z = -np.sort(-router_logits, axis=-1)
    if z.shape[-1] <= k:
        return np.full(z.shape[:-1], np.inf, dtype=np.float32)
    return z[..., k - 1] - z[..., k]


def argmax_margins(logits: np.ndarray) -> np.ndarray:
    """Gap between the two largest logits, per row."""
    top2 = -np.partition(-logits, 1, axis=-1)[..., :2]
    return top2[..., 0] - top2[..., 1]
