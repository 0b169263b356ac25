"""Temperature / top-p (nucleus) sampling of one token per logits row.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU legs are the only callers; the product path never imports this module.

The megakernel pages name the sampler only: their larger pipeline generates
either greedily or with temperature and top-p (tpu-megakernels README, section
on the serving demos).  This module is the plain definition those two words
have (Holtzman et al., "The Curious Case of Neural Text Degeneration", 2020,
section 3.1), with the steps the pages leave open fixed as follows:

1. temperature: p_i = exp((l_i - max_j l_j) / T) for T > 0, computed in fp64
   from the fp32 logits (so the largest p is exactly 1); T <= 0 means greedy:
   the argmax, lowest token id on ties;
2. masses are quantised once, q_i = round_half_even(p_i * 2**46), and every
   later sum is an exact integer sum of the q_i, so the decisions below do not
   depend on the order of any summation (the CUDA sampler decides in the same
   fixed point; with V <= 2**17 no sum overflows 64 bits);
3. the nucleus is the smallest prefix of the tokens sorted by probability,
   descending, ties by lower token id first (a stable sort), whose mass reaches
   need = max(1, ceil(top_p * Q)), Q the total mass; top_p <= 0 keeps the single
   most probable token, top_p >= 1 keeps every token with non-zero mass;
4. the draw takes one uniform u in [0, 1) per row as an input (the random
   number is not drawn here): y = min(S - 1, floor(u * S)) with S the nucleus
   mass, and the token is the first one, in token-id order, among the nucleus
   whose cumulative mass exceeds y.  Each nucleus token t is therefore drawn
   for a share q_t / S of the u interval: the renormalised nucleus
   distribution.

Steps 3 and 4 compute ceil(top_p * Q) and floor(u * S) in IEEE fp64 from the
fp64 values of the integers (round to nearest), as the CUDA sampler does.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

MASS_SCALE = 2.0 ** 46  # fixed-point unit of a probability mass
MAX_VOCAB = 1 << 17     # largest row the 64-bit mass sums cover without overflow


@dataclass
class Sample:
    token: int
    nucleus: int         # tokens in the nucleus (1 for greedy)
    nucleus_mass: int    # S, fixed point
    total_mass: int      # Q, fixed point
    need: int            # mass the nucleus had to reach
    y: int               # the draw's point in [0, S)
    draw_margin: int     # distance of y from the ends of the drawn token's interval
    nucleus_margin: int  # distance of the prefix sums from need at the nucleus boundary
                         # (unbounded where no rounding can move the boundary)
    boundary_mass: int   # largest mass that could enter or leave at that boundary

    def robust(self, slack: int) -> bool:
        """True when no change of the masses' sums by at most ``slack`` units can
        change the token: the draw is clear of its interval's ends, and the
        nucleus boundary either cannot move or, if it does, shifts the draw's
        point and interval ends by less than the draw's distance to them."""
        if self.total_mass == 0:
            return True  # greedy
        if self.draw_margin <= slack:
            return False
        return self.nucleus_margin > slack or self.draw_margin > self.boundary_mass + 2 * slack

    @property
    def margin(self) -> int:
        return min(self.draw_margin, self.nucleus_margin)


UNBOUNDED = 1 << 80


def probabilities(logits: np.ndarray, temperature: float) -> np.ndarray:
    """p_i = exp((l_i - max l) / T) in fp64 (step 1)."""
    l = np.asarray(logits, dtype=np.float32).astype(np.float64)
    inv_t = 1.0 / float(np.float32(temperature))
    return np.exp((l - l.max()) * inv_t)


def masses(logits: np.ndarray, temperature: float) -> np.ndarray:
    """Fixed-point masses q_i (step 2), uint64."""
    return np.rint(probabilities(logits, temperature) * MASS_SCALE).astype(np.uint64)


def greedy(logits: np.ndarray) -> int:
    """The argmax, lowest token id on ties."""
    l = np.asarray(logits, dtype=np.float32)
    return int(np.flatnonzero(l == l.max())[0])


def nucleus_need(total: int, top_p: float) -> int:
    """need = max(1, ceil(top_p * Q)) in fp64 (step 3)."""
    n = int(np.ceil(np.float64(np.float32(top_p)) * np.float64(total)))
    return max(1, min(n, total))


def draw_point(nucleus_mass: int, u: float) -> int:
    """y = min(S - 1, floor(u * S)) in fp64 (step 4)."""
    y = int(np.floor(np.float64(u) * np.float64(nucleus_mass)))
    return min(nucleus_mass - 1, max(0, y))


def sample_top_p(logits: np.ndarray, temperature: float, top_p: float, u: float) -> Sample:
    """One token from one logits row: the definition, step by step."""
    l = np.asarray(logits, dtype=np.float32)
    if l.ndim != 1 or l.size == 0 or l.size > MAX_VOCAB:
        raise ValueError("one row of 1 .. 2**17 logits")
    if not np.isfinite(l).all():
        raise ValueError("logits must be finite")
    if not (0.0 <= u < 1.0):
        raise ValueError("u must lie in [0, 1)")
    if float(np.float32(temperature)) <= 0.0:
        t = greedy(l)
        return Sample(t, 1, 0, 0, 0, 0, UNBOUNDED, UNBOUNDED, 0)
    q = masses(l, temperature)
    total = int(q.sum(dtype=np.uint64))
    need = nucleus_need(total, top_p)
    # step 3: stable descending sort by probability (= by logit), ties by id
    order = np.argsort(-l.astype(np.float64), kind="stable")
    cum = np.cumsum(q[order], dtype=np.uint64)
    k = int(np.searchsorted(cum, np.uint64(need), side="left")) + 1  # nucleus size
    members = order[:k]
    s = int(cum[k - 1])
    # step 4: inverse CDF over the nucleus in token-id order
    ids = np.sort(members)
    acum = np.cumsum(q[ids], dtype=np.uint64)
    assert int(acum[-1]) == s
    y = draw_point(s, u)
    j = int(np.searchsorted(acum, np.uint64(y), side="right"))  # first acum > y
    token = int(ids[j])
    before = int(acum[j - 1]) if j > 0 else 0
    draw_margin = min(y - before, int(acum[j]) - 1 - y)
    # the nucleus boundary: need = 1 keeps the top token whatever the rounding;
    # the nucleus cannot grow once it holds every token with mass
    nucleus_margin, boundary = UNBOUNDED, 0
    if need > 1:
        below = int(cum[k - 2]) if k > 1 else 0
        nucleus_margin = need - 1 - below
        boundary = int(q[order[k - 1]])
        if k < int(np.count_nonzero(q)):
            nucleus_margin = min(nucleus_margin, int(cum[k - 1]) - need)
            boundary = max(boundary, int(q[order[k]]))
    return Sample(token, k, s, total, need, y, draw_margin, nucleus_margin, boundary)
