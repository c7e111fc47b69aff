"""Pins for the fp64 oracle: each check rests on the pages or on mathematics,
never on the oracle re-running its own formula.

Sources: "MiniCPM5-2B-Hadamard-GSQ" model card, Mathematical Foundations §1
(Sylvester Hadamard, rotation invariance, dispersion bound) and §2 (INT4
group RTN, Q.s dequant, truncated SVD A = U sqrt(S), B = sqrt(S) V^T, runtime
equation); "Spark-X2.5-4B-Hadamard-GSQ" model card, Tier A/B/C and the
Empirical Scorecard.
"""
import math
import os
import re
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import dvssq_oracle as O
from mixed_precision_weight_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_vals(a):
    """Round an fp32/fp64 array to BF16 values via torch (RNE) -> fp64."""
    t = torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return O.torch_bf16_to_f64(t)


def _read_kv(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            for part in line.split():
                if "=" in part:
                    k, v = part.split("=")
                    out[k.strip()] = v.strip()
            if " = " in line:
                k, v = line.split(" = ")
                out[k.strip()] = v.strip()
    return out


# ---------------------------------------------------------------- Hadamard ---

@pytest.mark.parametrize("b", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_sylvester_matches_closed_form(b):
    # Sylvester's matrix has the closed form S[i, j] = (-1)^popcount(i & j).
    S = O.sylvester(b)
    i, j = np.meshgrid(np.arange(b), np.arange(b), indexing="ij")
    pc = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    assert np.array_equal(S, np.where(pc % 2 == 0, 1, -1))


@pytest.mark.parametrize("b", [128, 256])
def test_hadamard_orthogonal_symmetric(b):
    S = O.sylvester(b)
    assert np.array_equal(S @ S.T, b * np.eye(b, dtype=np.int64))   # exact, integers
    assert np.array_equal(S, S.T)
    H = O.hadamard(b)
    assert np.abs(H @ H.T - np.eye(b)).max() < 1e-14
    assert O.hadamard_scale(256) == 1.0 / 16.0
    # c_128 is the correctly rounded 1/sqrt(128)
    c = Fraction(O.hadamard_scale(128))
    assert abs(c * c - Fraction(1, 128)) < Fraction(1, 128) * Fraction(1, 2 ** 51)


def test_rotation_equals_block_diagonal_matmul():
    # W . H_K with H_K = diag(H_b, ..., H_b) built explicitly (Tier B equation).
    from scipy.linalg import block_diag
    rng = np.random.default_rng(3)
    for b, K in ((256, 512), (128, 384)):
        x = _bf16_vals(rng.standard_normal((5, K)))
        HK = block_diag(*([O.hadamard(b)] * (K // b)))
        assert np.abs(O.rotate(x, b) - x @ HK).max() < 1e-12


def test_rotation_invariance_and_parseval():
    # Y' = X'W'^T = X H H^T W^T = X W^T  (Mathematical Foundations §1)
    rng = np.random.default_rng(0)
    for b in (128, 256):
        K = 2 * b
        W = _bf16_vals(0.02 * rng.standard_normal((33, K)))
        x = _bf16_vals(rng.standard_normal((7, K)))
        y = x @ W.T
        y2 = O.rotate(x, b) @ O.rotate(W, b).T
        assert np.abs(y - y2).max() <= 1e-12 * np.abs(y).max()
        xr = O.rotate(x, b)
        assert np.allclose(np.linalg.norm(xr, axis=1), np.linalg.norm(x, axis=1),
                           rtol=1e-14)


def test_outlier_dispersion_bound():
    # max_j |X'_j| <= (1/sqrt(d)) sum_i |X_i| per rotated block (§1)
    rng = np.random.default_rng(1)
    b = 256
    x = rng.standard_normal((20, b))
    x[:, 7] *= 50.0
    x = _bf16_vals(x)
    xr = O.rotate(x, b)
    assert np.all(np.abs(xr).max(axis=1) <= np.abs(x).sum(axis=1) / math.sqrt(b) * (1 + 1e-15))
    # special cases: a one-hot block spreads to +-c; an all-ones block concentrates
    e = np.zeros((1, b)); e[0, 5] = 1.0
    assert np.allclose(np.abs(O.rotate(e, b)), 1 / 16)
    ones = np.ones((1, b))
    r = O.rotate(ones, b)
    assert r[0, 0] == 16.0 and np.all(r[0, 1:] == 0.0)


def test_rotation_is_exact_vs_rational_arithmetic():
    rng = np.random.default_rng(2)
    S = O.sylvester(128)
    for _ in range(3):
        row = _bf16_vals(rng.standard_normal(128) * np.exp(rng.uniform(-8, 8, 128)))
        exact = [sum((Fraction(float(v)) if S[j, l] > 0 else -Fraction(float(v)))
                     for l, v in enumerate(row)) for j in range(128)]
        want = np.array([float(e) for e in exact]) * O.hadamard_scale(128)
        got = O.rotate(row[None, :], 128)[0]
        assert np.array_equal(got, want)


def test_rotation_wide_exponent_spread_takes_exact_path():
    b = 256
    row = np.zeros(b)
    row[0], row[1], row[2] = 1.0, 2.0 ** -60, -1.0
    row = _bf16_vals(row)
    assert O.rotation_inexact_blocks(row[None, :], b) == 1
    got = O.rotate(row[None, :], b)[0]
    S = O.sylvester(b)
    want = np.array([float(sum(Fraction(float(row[l])) * int(S[j, l]) for l in range(3)))
                     for j in range(b)]) / 16.0
    assert np.array_equal(got, want)
    assert got[0] == 2.0 ** -64
    # a left-to-right fp64 sum loses the small term: (1 + 2^-60) - 1 == 0
    naive = 0.0
    for v in row[:3]:
        naive += v
    assert naive == 0.0


# ------------------------------------------------------------- BF16 rounding --

def _bf16_neighbours(x):
    f = np.float32(x)
    bits = int(np.array(f).view(np.uint32)) >> 16
    cands = []
    for d in range(-2, 3):
        bb = (bits + d) & 0xFFFF
        v = float(np.array(bb << 16, dtype=np.uint32).view(np.float32))
        if np.isfinite(v):
            cands.append((v, bb))
    return cands


def test_rn_bf16_brute_force():
    rng = np.random.default_rng(5)
    xs = np.concatenate([rng.standard_normal(2000) * np.exp(rng.uniform(-30, 30, 2000)),
                         rng.standard_normal(200) * 1e-39])
    got = O.rn_bf16(xs)
    for x, g in zip(xs, got):
        c = _bf16_neighbours(x)
        dist = [abs(v - x) for v, _ in c]
        dmin = min(dist)
        best = [(v, bb) for (v, bb), d in zip(c, dist) if d == dmin]
        if len(best) > 1:
            best = [t for t in best if t[1] % 2 == 0]
        assert g == best[0][0], (x, g, best)


def test_rn_bf16_ties_to_even():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7 -> even significand (1.0)
    assert O.rn_bf16(1.0 + 2.0 ** -8) == 1.0
    assert O.rn_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2 * 2.0 ** -7
    # a value just above a midpoint rounds up: no double rounding through fp32
    assert O.rn_bf16(1.0 + 2.0 ** -8 + 2.0 ** -40) == 1.0 + 2.0 ** -7


# ------------------------------------------------------------------ INT4/INT8 -

def _rtn_brute(w, s, lo, hi):
    best, bq = None, None
    for q in range(lo, hi + 1):
        d = abs(Fraction(float(w)) - q * Fraction(float(s)))
        if best is None or d < best or (d == best and q % 2 == 0):
            best, bq = d, q
    return bq


def test_int4_rtn_brute_force():
    rng = np.random.default_rng(7)
    W = _bf16_vals(0.02 * rng.standard_normal((4, 128)))
    Wr = O.rotate(W, 128)
    q, s4 = O.quantize_int4(Wr, np.array([], dtype=np.int32))
    for i in range(4):
        for g in range(2):
            grp = Wr[i, 64 * g:64 * g + 64]
            s = O.rn_bf16(np.abs(grp).max() / 7.0)
            assert s4[i, g] == s
            for j in range(64):
                assert q[i, 64 * g + j] == _rtn_brute(grp[j], s, -8, 7)


def test_int4_grid_round_trip():
    # W_rot = Q . s with one +-7 per group and BF16-exact scales -> exact Q, s back
    rng = np.random.default_rng(11)
    M, K = 6, 256
    Q = rng.integers(-7, 8, size=(M, K))
    for i in range(M):
        for g in range(K // 64):
            Q[i, 64 * g + rng.integers(64)] = rng.choice([-7, 7])
    s = O.rn_bf16(np.exp(rng.uniform(-8, 2, (M, K // 64))))
    Wr = (Q.reshape(M, K // 64, 64) * s[..., None]).reshape(M, K)
    q, s4 = O.quantize_int4(Wr, np.array([], dtype=np.int32))
    assert np.array_equal(q, Q) and np.array_equal(s4, s)
    # packing round trip, low nibble = even column
    p = O.pack_int4(q)
    assert np.array_equal(O.unpack_int4(p), q)
    assert p[0, 0] == ((int(q[0, 0]) & 15) | ((int(q[0, 1]) & 15) << 4))


def test_int4_special_groups():
    M, K = 3, 128
    Wr = np.zeros((M, K))
    Wr[1, 3] = -0.5          # a single nonzero -> code -7 at scale 0.5/7
    sal = np.array([64 + j for j in range(64)], dtype=np.int32)
    Wr[2, 64:] = 9.0         # a group made only of salient columns
    q, s4 = O.quantize_int4(Wr, sal)
    assert np.all(q[0] == 0) and np.all(s4[0] == 0)          # all-zero group
    assert q[1, 3] == -7 and s4[1, 0] == O.rn_bf16(0.5 / 7)
    assert np.all(q[2, 64:] == 0) and s4[2, 1] == 0          # salient-only group
    assert q.min() >= -8 and q.max() <= 7


def test_int8_brute_force_and_grid():
    rng = np.random.default_rng(13)
    Wr = O.rotate(_bf16_vals(0.02 * rng.standard_normal((5, 256))), 256)
    sal = np.sort(rng.choice(256, 32, replace=False)).astype(np.int32)
    q8, s8 = O.quantize_int8(Wr, sal)
    for i in range(5):
        s = O.rn_bf16(np.abs(Wr[i, sal]).max() / 127.0)
        assert s8[i] == s
        for k, j in enumerate(sal):
            assert q8[i, k] == _rtn_brute(Wr[i, j], s, -128, 127)
    Q = rng.integers(-127, 128, size=(4, 40)); Q[:, 0] = 127
    s = O.rn_bf16(np.exp(rng.uniform(-6, 0, 4)))
    Wg = np.zeros((4, 128)); idx = np.arange(0, 120, 3)[:40]
    Wg[:, idx] = Q * s[:, None]
    q8, s8 = O.quantize_int8(Wg, idx)
    assert np.array_equal(q8, Q) and np.array_equal(s8, s)


def test_int8_step_finer_than_int4():
    # Tier A: INT8 (256 levels) vs INT4 (16 bins): 16x more levels; the step of
    # a symmetric absmax quantiser shrinks by 127/7 ~= 18.
    kv = _read_kv("salient_counts.txt")
    assert int(kv["int8_levels"]) // int(kv["int4_levels"]) == 16
    rng = np.random.default_rng(17)
    w = rng.standard_normal(64)
    s4 = O.rn_bf16(np.abs(w).max() / 7.0)
    s8 = O.rn_bf16(np.abs(w).max() / 127.0)
    assert 17.0 < s4 / s8 < 19.5


# -------------------------------------------------------------- selection ----

def test_topk_brute_force_and_ties():
    rng = np.random.default_rng(19)
    score = rng.integers(0, 6, size=80).astype(np.float64)    # many exact ties
    sal = O.select_salient(score, 10)
    ranked = sorted(range(80), key=lambda j: (-score[j], j))[:10]
    assert list(sal) == sorted(ranked)
    assert np.all(np.diff(sal) > 0)


def test_salient_counts_match_pages():
    pairs = []
    with open(os.path.join(GOLDEN, "salient_counts.txt")) as f:
        for line in f:
            m = re.match(r"K=(\d+) n_sal=(\d+)", line.strip())
            if m:
                pairs.append((int(m.group(1)), int(m.group(2))))
    assert pairs == [(2560, 320), (10240, 1280)]
    for K, n in pairs:
        assert K // O.SAL_DEN == n
        W = np.random.default_rng(K).standard_normal((3, K))
        assert O.select_salient(O.salience(W, np.ones(K, np.float32)), K // 8).size == n


def test_column_ssq_order_definition():
    # The chunked order is a fixed summation tree of the exact sum of squares:
    # the result lies within a few ulps of the rational sum.
    rng = np.random.default_rng(23)
    Wr = O.rotate(_bf16_vals(0.02 * rng.standard_normal((150, 256))), 256)
    ssq = O.column_ssq(Wr)
    for j in (0, 17, 255):
        exact = sum(Fraction(float(v)) ** 2 for v in Wr[:, j])
        assert abs(Fraction(float(ssq[j])) - exact) <= exact * Fraction(1, 2 ** 45)
    # planted column energies decide the ranking
    act = np.ones(256, dtype=np.float32)
    Wr2 = Wr.copy(); Wr2[:, [5, 99]] *= 10
    sal = O.select_salient(O.salience(Wr2, act), 2)
    assert list(sal) == [5, 99]


# -------------------------------------------------------------------- SVD ----

def test_svd_eckart_young_and_monotone():
    rng = np.random.default_rng(29)
    R = rng.standard_normal((60, 90)) @ np.diag(np.linspace(2, 0.1, 90)) * 0.01
    prev = np.inf
    for r in (0, 2, 4, 8, 16):
        A, B, S = O.svd_factors(R, r, round_bf16=False)
        err = np.linalg.norm(R - A @ B) ** 2
        assert abs(err - (S[r:] ** 2).sum()) <= 1e-10 * (S ** 2).sum()
        Ab, Bb, _ = O.svd_factors(R, r)
        errb = np.linalg.norm(R - Ab @ Bb)
        assert errb < prev
        prev = errb
    A, B, S = O.svd_factors(R, 4, round_bf16=False)
    U, S2, Vt = np.linalg.svd(R)
    assert np.allclose(A @ B, U[:, :4] @ np.diag(S2[:4]) @ Vt[:4], atol=1e-12)
    assert np.allclose(np.linalg.norm(A, axis=0), np.sqrt(S[:4]))


# ---------------------------------------------------------------- forward ----

def test_forward_matches_dense_reconstruction():
    wl = synth.WORKLOADS["tiny"]
    W = O.torch_bf16_to_f64(wl.weight())
    a = wl.act_scale().numpy()
    enc = O.encode(W, a, wl.block, wl.rank)
    x = O.torch_bf16_to_f64(wl.activations(4))
    bias = _bf16_vals(0.1 * np.random.default_rng(3).standard_normal(wl.M))
    y = O.forward(enc, x, bias)
    y_dense = x @ O.dense_effective_weight(enc).T + bias
    assert np.abs(y - y_dense).max() <= 1e-12 * np.abs(y).max()
    # the compressed layer approximates the BF16 layer: INT4 G=64 RTN leaves
    # ~8 % weight error in the rotated domain; the x outlier channels (x30)
    # weight that error unevenly, so the output error is larger
    Wr = enc["W_rot"]
    W_hat = O.dense_effective_weight(enc)
    assert np.linalg.norm(W_hat - W) / np.linalg.norm(W) < 0.1
    rel = np.linalg.norm(y - bias - x @ W.T) / np.linalg.norm(x @ W.T)
    assert rel < 0.3


def test_encode_invariants_tiny():
    wl = synth.WORKLOADS["tiny"]
    W = O.torch_bf16_to_f64(wl.weight())
    enc = O.encode(W, wl.act_scale().numpy(), wl.block, wl.rank)
    assert enc["sal_idx"].size == 64 and np.all(np.diff(enc["sal_idx"]) > 0)
    assert enc["q4"].shape == (256, 256) and enc["q8"].shape == (256, 64)
    assert np.all(enc["q"][:, enc["sal_idx"]] == 0)
    assert enc["inexact_blocks"] == 0
    # every scale is a BF16 value
    O.f64_to_bf16_bits(enc["s4"]); O.f64_to_bf16_bits(enc["s8"])
    O.f64_to_bf16_bits(enc["U"]); O.f64_to_bf16_bits(enc["V"])
    # residual error falls with rank
    errs = []
    for r in (0, 4, 8, 16):
        A, B, _ = O.svd_factors(enc["R"], r)
        errs.append(np.linalg.norm(enc["R"] - A @ B))
    assert all(e1 > e2 for e1, e2 in zip(errs, errs[1:]))


def test_salient_rows_dominate_with_planted_outliers():
    # outlier input columns get large rotated norms in their block; the 4
    # outlier columns x20 of the tiny workload raise their blocks' energy
    wl = synth.WORKLOADS["tiny"]
    W = O.torch_bf16_to_f64(wl.weight())
    enc = O.encode(W, np.ones(wl.K, np.float32), wl.block, 0, with_svd=False)
    s = enc["score"]
    assert s[enc["sal_idx"]].min() >= np.delete(s, enc["sal_idx"]).max()


# ---------------------------------------------------------- storage layout ---

def test_footprint_dense_layout_matches_scorecard():
    kv = _read_kv("spark_scorecard.txt")
    bf16_total = int(kv["bf16_total_bytes"])
    dv_total = int(kv["dvssq_total_bytes"])
    fp = O.spark_model_footprint()
    non_mlp = bf16_total - fp["mlp_bf16"]
    implied_mlp = dv_total - non_mlp
    rel = abs(fp["mlp_dvssq"] - implied_mlp) / implied_mlp
    assert rel < 0.01, rel
    # the compact layout (INT4 on the 87.5 % background columns only) is far off
    compact = fp["mlp_dvssq"] - 36 * 3 * 10240 * 2560 // 2 // 8
    assert abs(compact - implied_mlp) / implied_mlp > 0.05
    assert abs(bf16_total / dv_total - float(kv["compression_ratio"])) < 1e-3


def test_packed_bytes_spark_down():
    assert O.packed_bytes(2560, 10240, 16) == 17623040
    assert O.packed_bytes(10240, 2560, 16) == 17634560


def test_oracle_is_independent_of_library():
    import oracle.dvssq_oracle as mod
    src = open(mod.__file__).read()
    assert "mixed_precision_weight_b200" not in src and "ctypes" not in src


# ------------------------------------------------------------- R10 MLP block --

def test_gelu_closed_forms():
    # gelu(v) = v * Phi(v): Phi(0) = 1/2, Phi(1) and Phi(-2) from the normal table
    assert O.gelu(np.array([0.0]))[0] == 0.0
    assert abs(O.gelu(np.array([1.0]))[0] - 0.8413447460685429) < 1e-15
    assert abs(O.gelu(np.array([-2.0]))[0] - (-2.0 * 0.022750131948179195)) < 1e-15
    v = np.linspace(-6, 6, 97)
    # Phi(v) + Phi(-v) = 1  =>  gelu(v) - gelu(-v) = v
    assert np.allclose(O.gelu(v) - O.gelu(-v), v, rtol=0, atol=1e-14)
    assert np.all(O.gelu(np.array([40.0])) == 40.0)
    # deep negative tail: Phi(-10) = 7.619853024160527e-24 (normal table)
    assert abs(O.gelu(np.array([-10.0]))[0] / (-10.0 * 7.619853024160527e-24) - 1) < 1e-12


def test_gelu_mul_rounds_once_to_bf16():
    rng = np.random.default_rng(4)
    g = O.rn_bf16(rng.normal(size=257))
    u = O.rn_bf16(rng.normal(size=257))
    h = O.gelu_mul(g, u)
    assert np.array_equal(h, O.rn_bf16(h))                  # already BF16
    exact = O.gelu(g) * u
    # BF16 spacing at |v| in [2^e, 2^(e+1)) is 2^(e-7); RN errs by at most half
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact), 1e-30))) - 7)
    assert np.all(np.abs(h - exact) <= 0.5 * ulp)


def test_mlp_block_matches_dense_composition():
    # the block on the packed form equals the composition written with each
    # layer's effective dense weight, with the same BF16 rounding points
    rng = np.random.default_rng(5)
    H, I = 256, 512
    encs = []
    for (M, K), seed in (((I, H), 1), ((I, H), 2), ((H, I), 3)):
        W = O.rn_bf16(rng.normal(scale=0.05, size=(M, K)))
        act = np.abs(rng.normal(size=K)) + 0.1
        encs.append(O.encode(W, act, 256, 4))
    x = O.rn_bf16(rng.normal(size=(2, H)))
    y = O.mlp_block(*encs, x)
    Wg, Wu, Wd = (O.dense_effective_weight(e) for e in encs)
    g = O.rn_bf16(x @ Wg.T)
    u = O.rn_bf16(x @ Wu.T)
    h = O.rn_bf16(O.gelu(g) * u)
    ref = O.rn_bf16(h @ Wd.T)
    # identical up to fp64 rounding of the two summation orders: BF16 values
    # may differ only where a sum lands within ~1e-12 of a rounding boundary
    assert np.mean(y == ref) > 0.99
    assert np.max(np.abs(y - ref)) <= 2.0 ** -7 * np.max(np.abs(ref))


# ------------------------------------------- planted pins (independent) -----

def _HK(K, b):
    """H_K = diag(H_b, ...) from scipy's Sylvester Hadamard, divided by sqrt(b)
    (for b = 256 the division by 16 is exact)."""
    from scipy.linalg import block_diag, hadamard
    Hb = hadamard(b).astype(np.float64) / math.sqrt(b)
    return block_diag(*([Hb] * (K // b)))


def test_salience_activation_factor_planted():
    # Tier A salience on the ROTATED weights times the activation scale of
    # the rotated column: six planted rotated columns with exact norms n and
    # scales a.  a*n = (8, 7, 4, 8, 2, 12) selects {0, 3, 5}; each plausible
    # mistake selects another set: a^2*n {0, 2, 5}, sqrt(a)*n {0, 1, 3},
    # n alone {0, 3, 4}, a*n^2 {0, 1, 3}, n/a {0, 3, 4}.  Scoring the
    # unrotated W (all of whose columns have equal norms here) would select
    # by a alone.
    b, K, M = 256, 256, 6
    n = np.array([8.0, 7.0, 2.0, 8.0, 8.0, 3.0])
    a = np.array([1.0, 1.0, 2.0, 1.0, 0.25, 4.0], dtype=np.float32)
    pos = np.array([3, 40, 77, 130, 200, 251])
    W_rot = np.zeros((M, K))
    for c in range(6):
        W_rot[c, pos[c]] = n[c]                 # one nonzero per row: exact norms
    W = W_rot @ _HK(K, b)                       # original domain, every entry +-n/16
    assert np.array_equal(W, O.rn_bf16(W))      # BF16 values, as the encoder takes
    act = np.full(K, 3.0, dtype=np.float32)     # columns with zero norm score 0
    act[pos] = a
    enc = O.encode(W, act, b, 0, n_sal=3, with_svd=False)
    assert list(enc["sal_idx"]) == [3, 130, 251]
    assert list(enc["score"][pos]) == [8.0, 7.0, 4.0, 8.0, 2.0, 12.0]


def _planted_grid(seed, M=8, K=512, b=256, n_sal=64):
    """Rotated-domain weights on the INT4/INT8 grids: W_rot = Q s4 outside the
    salient set P and Q8 s8 on it, every group with a +-7 (so s4 comes back)
    and every row with a +-127 in P (so s8 comes back); |Q8| >= 64 keeps P
    the top n_sal columns by norm for activation scales in [1, 1.5]."""
    rng = np.random.default_rng(seed)
    P = np.sort(rng.choice(K, n_sal, replace=False))
    nonsal = np.setdiff1d(np.arange(K), P)
    s4 = 2.0 ** rng.integers(-12, -7, size=(M, K // 64))
    s8 = 2.0 ** rng.integers(-4, -1, size=M)
    Q = rng.integers(-6, 7, size=(M, K))
    Q[:, P] = 0
    for i in range(M):
        for g in range(K // 64):
            cols = nonsal[(nonsal >= 64 * g) & (nonsal < 64 * g + 64)]
            Q[i, rng.choice(cols)] = rng.choice([-7, 7])
    Q8 = rng.integers(64, 128, size=(M, n_sal)) * rng.choice([-1, 1], size=(M, n_sal))
    Q8[np.arange(M), rng.integers(0, n_sal, size=M)] = 127
    W_rot = (Q.reshape(M, K // 64, 64) * s4[..., None]).reshape(M, K)
    W_rot[:, P] = Q8 * s8[:, None]
    return dict(P=P, Q=Q, s4=s4, Q8=Q8, s8=s8, W_rot=W_rot)


def test_grid_round_trip_encode_and_forward():
    # W = (Q s4 + scatter(Q8 s8)) H_K built with scipy's Hadamard: encode
    # must return exactly the planted salient set, codes and scales, a zero
    # residual, and forward must equal the dense W x (MiniCPM card §2 runtime
    # equation; rotation invariance of §1) to fp64 rounding.
    b, K, M = 256, 512, 8
    pl = _planted_grid(3, M, K, b)
    HK = _HK(K, b)
    W = pl["W_rot"] @ HK
    act = (1.0 + 0.5 * np.random.default_rng(4).random(K)).astype(np.float32)
    enc = O.encode(W, act, b, 0, n_sal=64)
    assert np.array_equal(enc["sal_idx"], pl["P"])
    assert np.array_equal(enc["q"], pl["Q"])
    assert np.array_equal(enc["s4"], pl["s4"])
    assert np.array_equal(enc["q8"].astype(np.int64), pl["Q8"])
    assert np.array_equal(enc["s8"], pl["s8"])
    assert not np.any(enc["R"])                                  # residual exactly zero
    rng = np.random.default_rng(5)
    x = O.rn_bf16(rng.standard_normal((3, K)))
    bias = O.rn_bf16(rng.standard_normal(M))
    z = (np.zeros((M, 0)), np.zeros((0, K)))
    y = O.forward(enc, x, bias, U=z[0], V=z[1])
    ref = x @ W.T + bias
    assert np.abs(y - ref).max() <= 1e-12 * np.abs(ref).max()
    # the rank-r term acts on the rotated activations: W_eff = (W_rot + U V) H_K
    U = O.rn_bf16(0.01 * rng.standard_normal((M, 4)))
    V = O.rn_bf16(0.01 * rng.standard_normal((4, K)))
    y = O.forward(enc, x, U=U, V=V)
    ref = x @ ((pl["W_rot"] + U @ V) @ HK).T
    assert np.abs(y - ref).max() <= 1e-12 * np.abs(ref).max()


def test_residual_excludes_salient_columns_and_is_the_rounding_error():
    # Tier C: R = W_bg - What_bg, W_bg with the salient columns removed.  Off
    # the grid, R at a salient column is 0 (neither W_bg nor What4 holds it)
    # and elsewhere it is w - q s4 with q the brute-force nearest code.
    b, K, M = 256, 512, 8
    pl = _planted_grid(6, M, K, b)
    rng = np.random.default_rng(7)
    W_rot = pl["W_rot"].copy()
    nonsal = np.setdiff1d(np.arange(K), pl["P"])
    jitter = rng.uniform(-0.4, 0.4, size=(M, nonsal.size)) * np.repeat(pl["s4"], 64, axis=1)[:, nonsal]
    W_rot[:, nonsal] += jitter                  # the +-7 anchors stay the group maxima
    W = W_rot @ _HK(K, b)
    enc = O.encode(W, np.ones(K, np.float32), b, 0, n_sal=64)
    assert np.array_equal(enc["sal_idx"], pl["P"])
    R = enc["R"]
    assert not np.any(R[:, pl["P"]])
    Wr = enc["W_rot"]
    for i, j in ((0, nonsal[0]), (3, nonsal[100]), (7, nonsal[-1])):
        s = enc["s4"][i, j // 64]
        q = _rtn_brute(Wr[i, j], s, -8, 7)
        assert R[i, j] == Wr[i, j] - q * s
    assert np.abs(R[:, nonsal]).max() <= 0.5 * enc["s4"].max()


def test_svd_recovers_planted_rank_r():
    # Tier C / §2: a residual of exact rank r with distinct singular values
    # sigma is returned as A B = R; the split is A = U sqrt(S), B = sqrt(S) V^T;
    # truncation to r' < r keeps the planted leading terms.
    rng = np.random.default_rng(31)
    M, K, r = 40, 70, 4
    U0, _ = np.linalg.qr(rng.standard_normal((M, r)))
    V0, _ = np.linalg.qr(rng.standard_normal((K, r)))
    sigma = np.array([5.0, 3.0, 2.0, 0.5])
    R = U0 @ np.diag(sigma) @ V0.T
    A, B, S = O.svd_factors(R, r, round_bf16=False)
    assert np.allclose(S[:r], sigma, rtol=0, atol=1e-13)
    assert np.all(S[r:] < 1e-13)
    assert np.abs(A @ B - R).max() < 1e-13
    assert np.allclose(np.linalg.norm(A, axis=0), np.sqrt(sigma), atol=1e-13)
    assert np.allclose(np.linalg.norm(B, axis=1), np.sqrt(sigma), atol=1e-13)
    A2, B2, _ = O.svd_factors(R, 2, round_bf16=False)
    assert np.abs(A2 @ B2 - U0[:, :2] @ np.diag(sigma[:2]) @ V0[:, :2].T).max() < 1e-13


def test_column_ssq_tree_on_exactly_summable_inputs():
    # Where every partial sum is exact (small dyadic values), any summation
    # order gives the same bits: the fixed tree equals a plain row-ascending
    # sum and the exact integer sum.
    rng = np.random.default_rng(37)
    Wr = rng.integers(-20, 21, size=(333, 64)).astype(np.float64) / 8.0
    tree = O.column_ssq(Wr)
    seq = np.zeros(64)
    for i in range(Wr.shape[0]):
        seq = seq + Wr[i] * Wr[i]
    exact = (np.rint(Wr * 8).astype(np.int64) ** 2).sum(axis=0) / 64.0
    assert np.array_equal(tree, seq) and np.array_equal(tree, exact)


@pytest.mark.parametrize("seed", [0, 4])
def test_selection_valid_against_exact_scores_near_ties(seed):
    # Planted exact ties whose squares straddle 16-row chunk boundaries: the
    # fp64 rounding decides which tied columns make the top n_sal.  The
    # oracle's fixed tree and a plain sequential sum both yield a valid
    # top-n_sal set of the EXACT scores (rational arithmetic), though not the
    # same set: the tree's shape is a reading (R3), not a fact of the pages.
    import exact_topk as X
    W, n_sal = X.near_tie_weight(seed)
    Wf = O.torch_bf16_to_f64(W)
    assert O.rotation_inexact_blocks(Wf, 256) == 0
    act = np.ones(Wf.shape[1], np.float32)
    Wr = O.rotate(Wf, 256)
    score = O.salience(Wr, act)
    sal = O.select_salient(score, n_sal)
    info = X.check_selection_valid(Wr, act, sal, n_sal)
    assert info["exact_ties"] == 16                 # the boundary sits in a 16-way tie
    tied = np.argsort(-score, kind="stable")[8:24]
    assert len(set(score[tied])) > 1                # ... which rounding splits
    seq = np.zeros(Wr.shape[1])
    for i in range(Wr.shape[0]):
        seq = seq + Wr[i] * Wr[i]
    sal_seq = O.select_salient(np.sqrt(seq), n_sal)
    X.check_selection_valid(Wr, act, sal_seq, n_sal)
    assert not np.array_equal(sal, sal_seq)


# ------------------------------------------------------------- R11 KV-BSS ---

def test_bss_reduces_to_plain_softmax_attention():
    # tau = 1 and the haze truncation off: standard scaled dot-product
    # attention, checked against scipy's softmax
    from scipy.special import softmax
    rng = np.random.default_rng(8)
    B, Hq, Hkv, L, d = 2, 4, 2, 37, 16
    q, k, v = (rng.standard_normal(s) for s in ((B, Hq, d), (B, Hkv, L, d), (B, Hkv, L, d)))
    out = O.bss_attention(q, k, v, tau=1.0, haze=0.0)
    for b in range(B):
        for h in range(Hq):
            p = softmax(k[b, h // 2] @ q[b, h] / 4.0)
            assert np.allclose(out[b, h], p @ v[b, h // 2], rtol=0, atol=1e-13)


def test_bss_focus_factor_scales_the_logits():
    # tau multiplies the logits: tau = 2 equals tau = 1 on a doubled query
    rng = np.random.default_rng(9)
    q, k, v = rng.standard_normal((1, 2, 8)), rng.standard_normal((1, 1, 20, 8)), \
        rng.standard_normal((1, 1, 20, 8))
    assert np.allclose(O.bss_attention(q, k, v, tau=2.0, haze=0.0),
                       O.bss_attention(2.0 * q, k, v, tau=1.0, haze=0.0), atol=1e-14)


def test_bss_haze_truncation_planted():
    # logits (after scaling) planted at 0, -5, -11.9, -12.1 and -30 nats below
    # the maximum: the last two are masked, the rest keep exp(-gap) weights;
    # exp(-12) = 6.14e-6 (the pages' figure)
    assert abs(math.exp(-12.0) - 6.14e-6) < 0.01e-6
    d = 4
    gaps = np.array([0.0, 5.0, 11.9, 12.1, 30.0])
    q = np.zeros((1, 1, d)); q[0, 0, 0] = 1.0
    tau = 1.10
    k = np.zeros((1, 1, 5, d))
    k[0, 0, :, 0] = (20.0 - gaps) * math.sqrt(d) / tau        # logits 20 - gap
    v = np.zeros((1, 1, 5, d)); v[0, 0, :, 1] = np.arange(5) + 1.0
    out = O.bss_attention(q, k, v, tau=tau, haze=12.0)[0, 0]
    w = np.exp(-gaps[:3])
    assert abs(out[1] - (w @ (np.arange(3) + 1.0)) / w.sum()) < 1e-14
    # without the truncation the two far keys count
    full = O.bss_attention(q, k, v, tau=tau, haze=0.0)[0, 0]
    w5 = np.exp(-gaps)
    assert abs(full[1] - (w5 @ (np.arange(5) + 1.0)) / w5.sum()) < 1e-14
    assert out[1] != full[1]


def test_bss_single_dominant_binding_returns_its_value():
    # one key 13 nats above every other: all others are truncated and the
    # output is exactly that key's value
    rng = np.random.default_rng(10)
    d, L = 8, 50
    q = rng.standard_normal((1, 1, d))
    k = 0.01 * rng.standard_normal((1, 1, L, d))
    k[0, 0, 17] = q[0, 0] * (13.5 * math.sqrt(d) / 1.10 / (q[0, 0] @ q[0, 0]))
    v = rng.standard_normal((1, 1, L, d))
    out = O.bss_attention(q, k, v)
    assert np.array_equal(out[0, 0], v[0, 0, 17])


def test_bss_defaults_are_the_pages_constants():
    import inspect
    g = _read_kv("kv_bss.txt")
    sig = inspect.signature(O.bss_attention)
    assert sig.parameters["tau"].default == float(g["tau_focus"])
    assert sig.parameters["haze"].default == float(g["haze_nats"])
    assert abs(math.exp(-float(g["haze_nats"])) - float(g["exp_minus_haze"])) < 0.01e-6
    # tau = 1.00 (KV-BSS off) with the haze off is plain attention: the same
    # output as tau = 1.10 applied to a query scaled by 1 / 1.10
    rng = np.random.default_rng(12)
    q, k, v = rng.standard_normal((1, 2, 8)), rng.standard_normal((1, 1, 30, 8)), \
        rng.standard_normal((1, 1, 30, 8))
    off = O.bss_attention(q, k, v, tau=float(g["tau_off"]), haze=0.0)
    assert np.allclose(off, O.bss_attention(q / float(g["tau_focus"]), k, v, haze=0.0), atol=1e-14)
