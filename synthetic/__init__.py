"""Seeded synthetic inputs for the layered MoE decode step.

This module draws random numbers and nothing else: model dimensions, bf16
weights, prefilled KV caches, context lengths and token ids.  It holds none of
the decode step's arithmetic, so both the CUDA path (through its benchmark and
tests) and the CPU oracle can take their inputs from here without sharing any
of the method's code.

Recipe (the workloads the megakernel pages describe are single-stream and
small-batch MoE decode, plus a speculative verify block; the pages print no
weights, so the weights are random):

* every weight tensor is drawn as N(0, sigma) in fp32 and rounded to bf16
  (round-to-nearest-even, ``Tensor.to(torch.bfloat16)``); norm gains are 1.0;
* each tensor has its own ``torch.Generator`` seeded by
  ``tensor_seed(seed, name, layer)`` (CRC-32 based, stable across processes);
  tensors whose leading dimension is the expert index are drawn one expert at a
  time from that generator, so no fp32 temporary larger than one expert exists;
* the prefilled KV cache is N(0, 1) in bf16 (keys count as already rotated);
* token ids are uniform in ``[0, vocab)``; per-sequence context lengths are
  either fixed or uniform in ``[512, 2048]``.

The values depend on the device the generator runs on (torch's CPU and CUDA
generators differ); every comparison reads the same bytes on both sides.
"""
from __future__ import annotations

import dataclasses
import zlib
from typing import Dict, List, Optional

import torch


@dataclasses.dataclass(frozen=True)
class ModelConfig:
    """Dimensions of one synthetic decoder (the symbols used throughout)."""

    name: str
    n_layers: int          # L
    d_model: int           # d
    n_q_heads: int         # Hq
    n_kv_heads: int        # Hkv
    head_dim: int          # hd
    n_experts: int         # E
    top_k: int             # k
    expert_ffn: int        # F
    shared_ffn: int        # Fs (0 = no shared expert)
    vocab: int             # V
    rope_theta: float = 1e4
    rms_eps: float = 1e-6
    sigma: float = 0.02    # weight standard deviation


@dataclasses.dataclass(frozen=True)
class Workload:
    """A decode workload: a model plus batch shape, context and step count."""

    name: str
    model: ModelConfig
    batch: int             # B sequences
    tokens_per_step: int   # T (1, or 7 for a verify block)
    context: Optional[int]  # prefilled positions per sequence; None = U[lo, hi]
    context_range: tuple = (512, 2048)
    steps: int = 16
    seed: int = 0

    @property
    def rows(self) -> int:
        return self.batch * self.tokens_per_step

    def kv_capacity(self) -> int:
        """Cache slots per sequence: the longest context plus every step's tokens."""
        longest = self.context if self.context is not None else self.context_range[1]
        need = longest + self.steps * self.tokens_per_step
        return (need + 63) // 64 * 64


TINY = ModelConfig("tiny", 2, 256, 4, 2, 64, 8, 2, 512, 0, 1024)
SMALL = ModelConfig("small", 8, 2048, 16, 4, 128, 64, 4, 1024, 1024, 32000)
LARGE = ModelConfig("large", 16, 4096, 32, 8, 128, 128, 8, 1536, 1536, 64000, sigma=0.015)

# The large model's dimensions with 2 layers and 16 experts (about 2.5 GB of
# weights): the same per-op shapes, small enough for a full profiler capture.
PROFILE = ModelConfig("profile", 2, 4096, 32, 8, 128, 16, 8, 1536, 1536, 64000, sigma=0.015)

# The small model's attention, dense and vocab shapes with 16 experts (about
# 2.2 GB of weights): the wide-block path's kernels at their verify-block
# shapes, small enough for a full profiler capture.
SMALL_PROFILE = ModelConfig("small_profile", 8, 2048, 16, 4, 128, 16, 4, 1024, 1024, 32000)

# Dense decoders (no router; one SwiGLU FFN per layer, held as the shared
# expert): the tiny model's shapes, and the large model's attention, vocab and
# a Llama-3-8B-sized FFN (about 7.5 GB read per step, like the large MoE's
# active bytes).
TINY_DENSE = ModelConfig("tiny_dense", 2, 256, 4, 2, 64, 0, 0, 16, 512, 1024)
DENSE = ModelConfig("dense", 16, 4096, 32, 8, 128, 0, 0, 16, 14336, 64000, sigma=0.015)

MODELS = {m.name: m for m in (TINY, SMALL, LARGE, PROFILE, SMALL_PROFILE, TINY_DENSE, DENSE)}


def workload(kind: str, batch: int = 1) -> Workload:
    """The named workloads: tiny / small / small_batch / verify / large / profile,
    and the dense decoders tiny_dense / dense."""
    if kind == "tiny":
        return Workload("tiny_bs1", TINY, 1, 1, 127, steps=16, seed=0)
    if kind == "small":
        return Workload("small_bs1", SMALL, 1, 1, 2047, steps=64, seed=1)
    if kind == "small_batch":
        return Workload(f"small_bs{batch}", SMALL, batch, 1, None, steps=64, seed=2)
    if kind == "verify":
        return Workload(f"verify_b{batch}_t7", SMALL, batch, 7, 2048, steps=64, seed=3)
    if kind == "large":
        return Workload(f"large_bs{batch}", LARGE, batch, 1, 4095, steps=32, seed=4)
    if kind == "profile":
        return Workload(f"profile_bs{batch}", PROFILE, batch, 1, 4095, steps=8, seed=5)
    if kind == "tiny_dense":
        return Workload("tiny_dense_bs1", TINY_DENSE, 1, 1, 127, steps=16, seed=6)
    if kind == "dense":
        return Workload(f"dense_bs{batch}", DENSE, batch, 1, 4095, steps=32, seed=7)
    raise ValueError(f"unknown workload {kind!r}")


def tensor_seed(seed: int, name: str, layer: int = -1) -> int:
    """Stable 63-bit seed for one named tensor."""
    h = zlib.crc32(f"{seed}:{name}:{layer}".encode())
    return (seed * 1_000_003 + h * 7919 + (layer + 1) * 104_729) & ((1 << 63) - 1)


def _normal_bf16(shape, sigma: float, gen: torch.Generator, device) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    x.mul_(sigma)
    return x.to(torch.bfloat16)


def _draw(shape, sigma, seed, name, layer, device, per_expert=False) -> torch.Tensor:
    gen = torch.Generator(device=device)
    gen.manual_seed(tensor_seed(seed, name, layer))
    if not per_expert:
        return _normal_bf16(shape, sigma, gen, device)
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    for e in range(shape[0]):
        out[e] = _normal_bf16(shape[1:], sigma, gen, device)
    return out


LAYER_TENSORS = ("attn_norm", "wqkv", "wo", "ffn_norm", "router",
                 "w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down")


def layer_shapes(m: ModelConfig) -> Dict[str, tuple]:
    """Row-major shapes ``[out, in]`` of one layer's tensors (experts leading)."""
    qkv_rows = (m.n_q_heads + 2 * m.n_kv_heads) * m.head_dim
    shapes = {
        "attn_norm": (m.d_model,),
        "wqkv": (qkv_rows, m.d_model),
        "wo": (m.d_model, m.n_q_heads * m.head_dim),
        "ffn_norm": (m.d_model,),
        "router": (m.n_experts, m.d_model),
        "w_gate": (m.n_experts, m.expert_ffn, m.d_model),
        "w_up": (m.n_experts, m.expert_ffn, m.d_model),
        "w_down": (m.n_experts, m.d_model, m.expert_ffn),
    }
    if m.shared_ffn > 0:
        shapes["ws_gate"] = (m.shared_ffn, m.d_model)
        shapes["ws_up"] = (m.shared_ffn, m.d_model)
        shapes["ws_down"] = (m.d_model, m.shared_ffn)
    return shapes


def make_weights(m: ModelConfig, seed: int, device="cpu") -> Dict[str, object]:
    """All weights of model ``m`` as bf16 tensors on ``device``.

    Returns ``{"embed", "final_norm", "lm_head", "layers": [dict per layer]}``.
    """
    dev = torch.device(device)
    w: Dict[str, object] = {
        "embed": _draw((m.vocab, m.d_model), m.sigma, seed, "embed", -1, dev),
        "final_norm": torch.ones(m.d_model, dtype=torch.bfloat16, device=dev),
        "lm_head": _draw((m.vocab, m.d_model), m.sigma, seed, "lm_head", -1, dev),
    }
    layers: List[Dict[str, torch.Tensor]] = []
    for l in range(m.n_layers):
        lw = {}
        for name, shape in layer_shapes(m).items():
            if name.endswith("_norm"):
                lw[name] = torch.ones(shape, dtype=torch.bfloat16, device=dev)
            else:
                lw[name] = _draw(shape, m.sigma, seed, name, l, dev,
                                 per_expert=(len(shape) == 3))
        layers.append(lw)
    w["layers"] = layers
    return w


def make_kv_cache(m: ModelConfig, max_seqs: int, capacity: int, seed: int,
                  device="cpu"):
    """Prefilled bf16 K and V caches, each ``[L][max_seqs][Hkv][capacity][hd]``, N(0,1)."""
    dev = torch.device(device)
    shape = (m.n_layers, max_seqs, m.n_kv_heads, capacity, m.head_dim)
    out = []
    for name in ("k_cache", "v_cache"):
        gen = torch.Generator(device=dev)
        gen.manual_seed(tensor_seed(seed, name))
        t = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        for l in range(m.n_layers):
            t[l] = torch.randn(shape[1:], generator=gen, device=dev,
                               dtype=torch.float32).to(torch.bfloat16)
        out.append(t)
    return out[0], out[1]


def make_context_lengths(wl: Workload) -> List[int]:
    """Prefilled length per sequence (fixed, or uniform in ``context_range``)."""
    if wl.context is not None:
        return [wl.context] * wl.batch
    gen = torch.Generator()
    gen.manual_seed(tensor_seed(wl.seed, "context_lengths"))
    lo, hi = wl.context_range
    return [int(v) for v in torch.randint(lo, hi + 1, (wl.batch,), generator=gen)]


def make_tokens(vocab: int, count: int, seed: int, name: str = "tokens") -> List[int]:
    """``count`` token ids uniform in ``[0, vocab)``."""
    gen = torch.Generator()
    gen.manual_seed(tensor_seed(seed, name))
    return [int(v) for v in torch.randint(0, vocab, (count,), generator=gen)]


def bf16_bits(t: torch.Tensor):
    """Raw uint16 bit pattern of a bf16 tensor as a numpy array (on the host)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def make_logits(rows: int, vocab: int, sigma: float, seed: int) -> torch.Tensor:
    """fp32 ``[rows][vocab]`` logits, N(0, sigma), on the host: the sampler's
    stand-alone input (a decode step's own logits are the other)."""
    gen = torch.Generator()
    gen.manual_seed(tensor_seed(seed, "logits", vocab))
    return torch.randn((rows, vocab), generator=gen, dtype=torch.float32).mul_(sigma)


def make_uniforms(count: int, seed: int, name: str = "uniforms") -> List[float]:
    """``count`` fp64 uniforms in [0, 1): the random numbers a sampler draws,
    passed to it as inputs."""
    gen = torch.Generator()
    gen.manual_seed(tensor_seed(seed, name))
    return [float(v) for v in torch.rand((count,), generator=gen, dtype=torch.float64)]
