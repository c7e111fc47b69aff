"""Exact-arithmetic checks of a salient-column selection (test helpers).

The salience score of the Spark card's Tier A ("Semantic Channel Salience
Ranking") is the L2 norm of a rotated weight column times the channel's
activation scale, and the salient set is the top-12.5 % of the columns by
that score.  Any fp64 evaluation of the sum of squares rounds, so a column
whose exact score lies within the rounding error of the boundary may land on
either side of it.  These helpers judge a selection against the EXACT scores
(rational arithmetic on the fp64 rotated weights and FP32 scales), with a
stated relative error bound, independently of the summation order that the
oracle and the GPU share.

Also here: a BF16 weight matrix whose rotated columns come in exact ties
that straddle 16-row chunk boundaries, so that which tied columns win is
decided by fp64 rounding.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np
import torch

U64 = 2.0 ** -53


def tree_error_bound(M: int, depth_extra: int = 4) -> float:
    """Relative error bound of a score a * sqrt(sum of M squares) evaluated in
    fp64 by any summation tree of depth at most M (each square, add, the
    square root and the product rounded once): gamma_(M + depth_extra)."""
    d = M + depth_extra
    return d * U64 / (1.0 - d * U64)


def _exact_sq_score(col: np.ndarray, a: float) -> Fraction:
    """a^2 * sum(col^2) as an exact rational (fp64 entries, FP32 scale)."""
    s = Fraction(0)
    for v in col:
        if v != 0.0:
            f = Fraction(float(v))
            s += f * f
    fa = Fraction(float(a))
    return fa * fa * s


def check_selection_valid(W_rot: np.ndarray, act: np.ndarray, sal: np.ndarray, n_sal: int,
                          rel: float | None = None) -> dict:
    """Assert that ``sal`` is a valid top-n_sal set of the exact scores.

    With E_k the n_sal-th largest exact score and rel the relative error
    bound of a computed score: every column whose exact score exceeds
    E_k (1 + rel)^2 / (1 - rel)^2 must be selected, and every selected
    column must score at least E_k (1 - rel)^2 / (1 + rel)^2.  Scores are
    compared squared.  Returns counts for the caller's own assertions.
    """
    W_rot = np.asarray(W_rot, dtype=np.float64)
    act = np.asarray(act, dtype=np.float32).astype(np.float64)
    M, K = W_rot.shape
    sal = np.asarray(sal, dtype=np.int64)
    assert sal.size == n_sal and np.all(np.diff(sal) > 0), "not n_sal ascending indices"
    if n_sal == 0:
        return dict(band=0, exact_ties=0)
    if rel is None:
        rel = tree_error_bound(M)
    approx = act * act * np.einsum("ij,ij->j", W_rot, W_rot)     # squared scores
    kth = np.sort(approx)[::-1][n_sal - 1]
    # columns within 1e-9 of the boundary are judged exactly; elsewhere the
    # approximation (error ~1e-13) cannot change the comparison
    band = np.abs(approx - kth) <= 1e-9 * max(kth, 1e-300)
    idx_band = np.nonzero(band)[0]
    exact = {int(j): _exact_sq_score(W_rot[:, j], act[j]) for j in idx_band}
    n_above = int(np.sum(approx > kth * (1 + 1e-9)))
    ranked = sorted(exact.values(), reverse=True)
    Ek = ranked[n_sal - n_above - 1]
    hi = Ek * Fraction((1 + rel) ** 2) / Fraction((1 - rel) ** 2)
    lo = Ek * Fraction((1 - rel) ** 2) / Fraction((1 + rel) ** 2)
    chosen = set(int(j) for j in sal)
    for j in range(K):
        if band[j]:
            e = exact[j]
            if e > hi:
                assert j in chosen, f"column {j} clearly above the boundary was not selected"
            if j in chosen:
                assert e >= lo, f"selected column {j} is clearly below the boundary"
        else:
            if approx[j] > kth:
                assert j in chosen, f"column {j} clearly above the boundary was not selected"
            else:
                assert j not in chosen, f"selected column {j} is clearly below the boundary"
    ties = sum(1 for e in exact.values() if e == Ek)
    return dict(band=int(band.sum()), exact_ties=ties)


def near_tie_weight(seed: int = 0, M: int = 64, K: int = 512, b: int = 256):
    """BF16 W [M][K] whose rotated columns tie exactly across chunk boundaries.

    Every row has one value w1_i at offset 0 of each Hadamard block, so every
    rotated column of the block receives (w1_i / sqrt b)^2 from row i.  Three
    row pairs (7, 8), (15, 16) and (47, 48) share w1 and add w2 at offsets
    d = 1, 2 / 4, 8 / 16, 32: rotated column j then holds w1 + s w2 in one row
    of the pair and w1 + s' w2 in the other, with s, s' = +-1 given by bits of
    j.  Columns with (s, s') = (+, -) and (-, +) have equal exact energies,
    but their squares sit in different 16-row chunks for pairs (15, 16) and
    (47, 48), so the fp64 chunk sums round differently.

    The pairs' w2 magnitudes (about 2^-2, 2^-10 and 2^-29 of w1) decide the
    energy order pair by pair, and the third pair's w1 +- w2 has about 38
    significant bits, so its squares round in fp64.  Returns (W as torch.bfloat16, n_sal): n_sal = 16 puts the
    selection boundary inside the tie class of the third pair (top class:
    the 8 columns with (+, +) in every pair; then 16 tied columns for 8
    places).
    """
    g = np.random.Generator(np.random.PCG64(seed))
    W = np.zeros((M, K), dtype=np.float32)
    # rows outside the pairs span 2^-30..1, except rows 32..46 (the chunk that
    # ends with row 47), which are about 2^5: the third pair's squares are
    # added to a large partial sum in one chunk and a small one in the next,
    # so the two tied patterns round differently
    w1 = (g.uniform(0.5, 1.0, size=M) * 2.0 ** -g.integers(0, 31, size=M)).astype(np.float32)
    w1[32:47] = g.uniform(0.5, 1.0, size=15).astype(np.float32) * np.float32(32.0)
    pairs = ((7, 8, 1, 2, 0.25), (15, 16, 4, 8, 2.0 ** -10), (47, 48, 16, 32, 2.0 ** -29))
    w2 = {}
    for r0, r1, d0, d1, mag in pairs:
        w1[r0] = w1[r1] = np.float32(g.uniform(0.5, 1.0))
        v = np.float32(mag * g.uniform(0.5, 1.0))
        w2[r0], w2[r1] = (d0, v), (d1, v)
    for kb in range(K // b):
        for i in range(M):
            W[i, kb * b] = w1[i]
            if i in w2:
                d, v = w2[i]
                W[i, kb * b + d] = v
    Wt = torch.from_numpy(W).to(torch.bfloat16)
    return Wt, 16
