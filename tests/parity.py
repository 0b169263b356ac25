"""Teacher-forced parity of the CUDA decode step against the CPU oracle.

Both sides start from the same generator bytes (weights, prefilled KV cache,
initial tokens).  Each step the oracle runs on its own host copy of the cache
and the GPU on the device cache; the next step's tokens are the ORACLE's
argmax (and, for verify blocks, the oracle's acceptance), so no oracle input
ever comes from the CUDA path.

Bars (max|diff| / max|ref| per tensor): final logits <= 2e-2, per-layer
hidden states <= 1e-2; selected expert sets and argmax tokens bit-exact
wherever the oracle's margin exceeds 1e-3 (router: gap between the k-th and
(k+1)-th router logits; argmax: gap between the top two logits).  A row whose
expert set differs at a near tie is flagged and dropped from the rest of the
run (its cache history differs from then on).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np
import torch

import decode_megakernel_06_b200 as mk
from oracle import step as ostep
from synthetic import (Workload, bf16_bits, make_context_lengths, make_kv_cache, make_tokens,
                       make_weights)

LOGITS_TOL = 2e-2
HIDDEN_TOL = 1e-2
MARGIN = 1e-3


def relerr(got, ref) -> float:
    ref = np.asarray(ref, dtype=np.float64)
    got = np.asarray(got, dtype=np.float64)
    den = np.abs(ref).max()
    return float(np.abs(got - ref).max() / den) if den > 0 else float(np.abs(got).max())


@dataclasses.dataclass
class Report:
    steps: int = 0
    rows_compared: int = 0
    max_logits_err: float = 0.0
    max_hidden_err: float = 0.0
    argmax_checked: int = 0
    argmax_near_ties: int = 0
    expert_checked: int = 0
    expert_near_ties: int = 0
    flagged_rows: int = 0
    kv_max_ulps: float = 0.0


class Session:
    """Weights, caches and a decoder handle for one workload on cuda:0."""

    def __init__(self, wl: Workload, variant="megakernel", cache_host_weights=True,
                 model=None, capacity: Optional[int] = None, weights=None):
        self.wl = wl
        self.m = model or wl.model
        self.dev = torch.device("cuda:0")
        self.B, self.T = wl.batch, wl.tokens_per_step
        self.cap = capacity or wl.kv_capacity()
        self.w = weights if weights is not None else make_weights(self.m, wl.seed, self.dev)
        self.k, self.v = make_kv_cache(self.m, self.B, self.cap, wl.seed, self.dev)
        self.k_host = bf16_bits(self.k).copy()
        self.v_host = bf16_bits(self.v).copy()
        self.src = ostep.WeightSource(self.w, cache=cache_host_weights)
        self.dec = mk.Decoder(self.m, self.w, max_rows=self.B * self.T, max_seqs=self.B,
                              kv_capacity=self.cap, variant=variant)
        M, L, d, k = self.B * self.T, self.m.n_layers, self.m.d_model, self.m.top_k
        self.hidden = torch.zeros((L + 1, M, d), dtype=torch.float32, device=self.dev)
        self.ids = torch.zeros((L, M, k), dtype=torch.int32, device=self.dev)
        self.ew = torch.zeros((L, M, k), dtype=torch.float32, device=self.dev)
        self.dec.set_debug(self.hidden, self.ids, self.ew)
        self.logits = torch.empty((M, self.m.vocab), dtype=torch.float32, device=self.dev)
        self.argmax = torch.empty(M, dtype=torch.int32, device=self.dev)

    def close(self):
        self.dec.close()

    def gpu_step(self, tokens: List[int], positions: List[int]):
        t = torch.tensor(tokens, dtype=torch.int32, device=self.dev)
        p = torch.tensor(positions, dtype=torch.int32, device=self.dev)
        rc = self.dec.step(t, p, self.B, self.T, self.k, self.v, self.logits, self.argmax)
        assert rc == mk.MK_OK, mk.mk_last_error()
        st = self.dec.status()
        assert st == mk.MK_OK, (st, mk.mk_last_error())
        return (self.logits.cpu().numpy(), self.argmax.cpu().numpy(), self.hidden.cpu().numpy(),
                self.ids.cpu().numpy(), self.ew.cpu().numpy())

    def oracle_step(self, tokens, positions):
        return ostep.decode_step(self.m, self.src, self.k_host, self.v_host, tokens, positions,
                                 self.B, self.T)


def compare_step(s: Session, ref, got, rep: Report, alive: np.ndarray, positions):
    logits, am, hidden, ids, ew = got
    M, T = s.B * s.T, s.T
    k = s.m.top_k
    rmarg = ostep.router_margins(ref.router_logits, k)  # [L][M]
    dead = ~alive
    for l in range(s.m.n_layers):
        for m in range(M):
            if dead[m // T]:
                continue
            a = sorted(ids[l, m].tolist())
            b = sorted(ref.expert_ids[l, m].tolist())
            if rmarg[l, m] > MARGIN:
                rep.expert_checked += 1
                assert a == b, f"expert set mismatch layer {l} row {m}: {a} vs {b} (margin {rmarg[l, m]:.2e})"
                np.testing.assert_allclose(
                    np.sort(ew[l, m]), np.sort(ref.expert_w[l, m]), rtol=0, atol=1e-4)
            else:
                rep.expert_near_ties += 1
                if a != b:
                    dead[m // T] = True  # this sequence's history now differs
    rows = [m for m in range(M) if not dead[m // T]]
    if rows:
        rep.rows_compared += len(rows)
        e = relerr(logits[rows], ref.logits[rows])
        rep.max_logits_err = max(rep.max_logits_err, e)
        assert e <= LOGITS_TOL, f"logits rel err {e}"
        for l in range(s.m.n_layers + 1):
            he = relerr(hidden[l][rows], ref.hidden[l][rows])
            rep.max_hidden_err = max(rep.max_hidden_err, he)
            assert he <= HIDDEN_TOL, f"hidden[{l}] rel err {he}"
        amarg = ostep.argmax_margins(ref.logits)
        for m in rows:
            if amarg[m] > MARGIN:
                rep.argmax_checked += 1
                assert int(am[m]) == int(ref.argmax[m]), f"argmax row {m}: {am[m]} vs {ref.argmax[m]}"
            else:
                rep.argmax_near_ties += 1
    # appended cache entries: same bar as the per-layer states (max|d|/max|ref|);
    # the largest bf16 ulp difference is reported (near-zero entries can differ
    # by several ulps from fp32 summation order alone)
    for cache, host in ((s.k, s.k_host), (s.v, s.v_host)):
        cd = cache.view(torch.int16)
        for b in range(s.B):
            if dead[b]:
                continue
            p0 = positions[b]
            got_k = cd[:, b, :, p0:p0 + T].cpu().numpy().view(np.uint16)
            ref_k = host[:, b, :, p0:p0 + T]
            ulps = np.abs(got_k.astype(np.int32) - ref_k.astype(np.int32)).max()
            rep.kv_max_ulps = max(rep.kv_max_ulps, float(ulps))
            import oracle

            e = relerr(oracle.bf16_to_f32(got_k), oracle.bf16_to_f32(ref_k))
            assert e <= HIDDEN_TOL, f"appended cache entries rel err {e}"
    alive &= ~dead
    rep.flagged_rows = int((~alive).sum())


def run_greedy(s: Session, steps: int, rep: Optional[Report] = None) -> Report:
    """Greedy decode (T == 1), teacher-forced by the oracle's tokens."""
    assert s.T == 1
    rep = rep or Report()
    positions = make_context_lengths(s.wl)
    tokens = make_tokens(s.m.vocab, s.B, s.wl.seed)
    alive = np.ones(s.B, dtype=bool)
    for _ in range(steps):
        ref = s.oracle_step(tokens, positions)
        got = s.gpu_step(tokens, positions)
        compare_step(s, ref, got, rep, alive, positions)
        rep.steps += 1
        tokens = [int(t) for t in ref.argmax]
        positions = [p + 1 for p in positions]
    assert alive.mean() >= 0.5, "too many rows lost to router near-ties"
    return rep


def run_verify(s: Session, steps: int, rep: Optional[Report] = None) -> Report:
    """Verify blocks of T rows (last accepted token + T-1 random drafts); the
    oracle's greedy acceptance advances the positions of both sides."""
    rep = rep or Report()
    T = s.T
    positions = make_context_lengths(s.wl)
    last = make_tokens(s.m.vocab, s.B, s.wl.seed)
    alive = np.ones(s.B, dtype=bool)
    for st in range(steps):
        drafts = make_tokens(s.m.vocab, s.B * (T - 1), s.wl.seed, name=f"drafts{st}")
        tokens = []
        for b in range(s.B):
            tokens += [last[b]] + drafts[b * (T - 1):(b + 1) * (T - 1)]
        ref = s.oracle_step(tokens, positions)
        got = s.gpu_step(tokens, positions)
        compare_step(s, ref, got, rep, alive, positions)
        rep.steps += 1
        for b in range(s.B):
            row = ref.argmax[b * T:(b + 1) * T]
            acc = 1
            while acc < T and tokens[b * T + acc] == int(row[acc - 1]):
                acc += 1
            positions[b] += acc
            last[b] = int(row[acc - 1])
    return rep
