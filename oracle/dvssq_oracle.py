"""fp64 CPU oracle of the DV-SSQ compressed linear layer.

TEST INFRASTRUCTURE ONLY.  This module is the plain, slow, obviously-correct
reference that the CUDA library is checked against.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it; the library itself never does, and this module imports nothing from the
library (it shares no code, table or constant with it).

Every quantity is computed in IEEE fp64 with numpy; BLAS matmul, LAPACK SVD
and numpy sort serve as library steps.  Sources, cited by page and section:

* [Spark] "Spark-X2.5-4B-Hadamard-GSQ" model card (F-Labs), section
  "Architectural Pillars / 1. DV-SSQ": Tier A (column-energy salience, top
  12.5 % kept as INT8 with clip to [-128, 127]), Tier B (W_rot = W_bg . H_K,
  H_K = diag(H_256, ...), INT4 group-wise, G = 64), Tier C (R = W_bg - What_bg
  ~= U_r S_r V_r^T = A . B, stored in BF16); "Empirical Scorecard" (weight
  footprint).
* [MiniCPM] "MiniCPM5-2B-Hadamard-GSQ" model card (F-Labs), section
  "Mathematical Foundations": §1 (Sylvester normalised orthogonal Hadamard,
  rotation-invariance equation Y' = X'W'^T = XW^T, outlier-dispersion bound),
  §2 (s_g = max|W|/7, Q = clip(round(W/s_g), -8, 7), What = Q.s, R = W - What
  ~= A.B with A = U_r sqrt(S_r), B = sqrt(S_r) V_r^T, runtime equation
  Y = X.What^T + (X.B^T).A^T).

Readings taken where the pages leave a step open (each is listed in the
design notes of the repository):

R1  H_b = S_b / sqrt(b) with S_b the Sylvester +-1 matrix; c_b = RN64(sqrt(1/b)).
R2  W_rot[i, kb+j] = RN64(c_b * RN64(sum_l S_b[j,l] W[i, kb+l])): the +-1 sum
    is taken exactly and the scale is applied once, after the sum.
R3  Salience follows the task's fixed choice: the L2 norm of each *rotated*
    column times a per-channel activation scale a_j (indexed by rotated
    column).  The column sum of squares uses a fixed summation tree: rows in
    chunks of SSQ_CHUNK, within a chunk acc = acc + w*w (product and sum each
    rounded); chunk sums added in order within groups of SSQ_GROUP chunks;
    group sums added in ascending order.
R4  Top-k: n_sal largest scores, ties broken toward the lower column index;
    returned ascending.
R5  INT4 groups are 64 contiguous rotated columns over the full K ("dense"
    layout, salient positions coded 0); s4 = RN_bf16(RN64(absmax / 7)),
    q = clip(rint(w * RN64(1 / s4)), -8, 7), rint = half-to-even; s4 = 0 gives
    q = 0.
R6  INT8 salient tier: one BF16 scale per row, s8 = RN_bf16(RN64(m / 127)) with
    m the row's largest |W_rot| over the salient columns; q8 likewise.
R7  Residual R = W_bg - What4 in the rotated domain (Tier C's W_bg - What_bg);
    A, B from LAPACK SVD, each rounded to BF16.
R8  Forward: y = sum_j (q_ij s4_ig) xr_j + s8_i sum_k q8_ik xr_{sal_k}
    + sum_p A_ip (sum_j B_pj xr_j) (+ bias), xr = H_K x, evaluated in fp64 and
    not rounded.
R9  Nibble packing: two's-complement 4-bit codes, two per byte, the even
    rotated column in the low nibble.
R10 MLP block of the Spark shape ("Myric/Spark-X2.5-4B-GGUF", "The model":
    GELU FFN, 36 layers; "Spark-X2.5-4B-ASHQ1-GGUF", "Architecture":
    ffn_gate / ffn_up / ffn_down): x_next = down(GELU(gate x) * up x) with
    the exact erf GELU, no norm or residual, and hidden states rounded to
    BF16 after every projection and after the gated product.
R11 KV-BSS attention ([Spark] "2. KV-BSS"): logits q.k tau / sqrt(d), tau =
    1.10; a logit more than `haze` = 12 nats below the query's largest logit
    (over the keys it attends) is masked to -inf before the softmax.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

SSQ_CHUNK = 16          # R3: rows per fixed-order partial of the column sum of squares
SSQ_GROUP = 8           # R3: chunk sums per second-level partial
GROUP = 64              # Tier B / §2: group size G = 64
SAL_DEN = 8             # Tier A: top 12.5 % = 1/8 of the input channels

# ---------------------------------------------------------------------------
# BF16 <-> fp64 helpers (storage format of weights, scales and factors)
# ---------------------------------------------------------------------------


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode BF16 bit patterns (uint16) to fp64 values (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def rn_bf16(x) -> np.ndarray:
    """Round fp64 values to the nearest BF16 value, ties to even (as fp64).

    BF16 keeps 8 significand bits and the fp32 exponent range; below 2^-126 the
    quantum is 2^-133 (subnormals).  Written from the format definition:
    x = m * 2^e with 0.5 <= |m| < 1, the kept significand is rint(m * 2^8).
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    fin = np.isfinite(x)
    m, e = np.frexp(np.where(fin, x, 0.0))
    normal = np.abs(x) >= 2.0 ** -126
    q_norm = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    q_sub = np.ldexp(np.rint(np.ldexp(np.where(fin, x, 0.0), 133)), -133)
    out = np.where(normal, q_norm, q_sub)
    # overflow past the largest finite BF16 (0x7F7F = (2 - 2^-7) * 2^127)
    big = (2.0 - 2.0 ** -8) * 2.0 ** 127
    out = np.where(np.abs(x) >= big, np.copysign(np.inf, x), out)
    out = np.where(fin, out, x)
    return out


def f64_to_bf16_bits(x) -> np.ndarray:
    """fp64 values that are exactly BF16 -> their uint16 bit patterns."""
    v = np.asarray(x, dtype=np.float64)
    f = v.astype(np.float32)
    if not np.array_equal(f.astype(np.float64), v, equal_nan=True):
        raise ValueError("value not representable in BF16")
    bits = f.view(np.uint32)
    if np.any(bits & 0xFFFF):
        raise ValueError("value not representable in BF16")
    return (bits >> 16).astype(np.uint16)


def torch_bf16_to_f64(t) -> np.ndarray:
    """torch.bfloat16 tensor -> fp64 numpy array (exact)."""
    import torch
    return bf16_bits_to_f64(t.contiguous().view(torch.int16).numpy().view(np.uint16))


# ---------------------------------------------------------------------------
# [MiniCPM] Mathematical Foundations §1: Walsh-Hadamard rotation
# ---------------------------------------------------------------------------


def sylvester(b: int) -> np.ndarray:
    """Sylvester +-1 matrix S_b by the doubling construction S_2n = [[S, S], [S, -S]]."""
    if b < 1 or b & (b - 1):
        raise ValueError("Hadamard size must be a power of two")
    S = np.ones((1, 1), dtype=np.int64)
    while S.shape[0] < b:
        S = np.block([[S, S], [S, -S]])
    return S


def hadamard_scale(b: int) -> float:
    """c_b = RN64(1/sqrt(b)) (R1); 1/b is exact for powers of two."""
    return float(np.sqrt(np.float64(1.0) / np.float64(b)))


def hadamard(b: int) -> np.ndarray:
    """Normalised H_b = c_b * S_b (entries rounded once)."""
    return sylvester(b).astype(np.float64) * hadamard_scale(b)


def _bf16_exponent_lsb(v: np.ndarray):
    """(exponent, log2 of the last significand bit) of nonzero BF16 values.

    The exponent is floor(log2|v|) for normal values and -127 for subnormal
    ones (an upper bound, so the exactness test stays sufficient).
    """
    e = np.maximum(np.floor(np.log2(np.abs(v))).astype(np.int64), -127)
    lsb = np.maximum(e - 7, -133)
    return e, lsb


def block_sum_is_exact(Wblk: np.ndarray) -> np.ndarray:
    """Sufficient test that every +-1 partial sum of each row-block is exact in fp64.

    ``Wblk`` is [..., b] of BF16 values.  All partial sums are integer multiples
    of 2^Lmin (the smallest last-bit among the block's nonzeros) bounded by
    b * 2^(Emax+1); they fit fp64's 53-bit significand when
    Emax + 1 + log2(b) - Lmin <= 53.
    """
    b = Wblk.shape[-1]
    nz = Wblk != 0
    safe = np.where(nz, Wblk, 1.0)
    e, lsb = _bf16_exponent_lsb(safe)
    emax = np.where(nz, e, -10 ** 6).max(axis=-1)
    lmin = np.where(nz, lsb, 10 ** 6).min(axis=-1)
    span = emax + 1 + int(math.log2(b)) - lmin
    return (~nz.any(axis=-1)) | (span <= 53)


def _exact_block_sums(row: np.ndarray, S: np.ndarray) -> np.ndarray:
    """Exact +-1 sums of one row-block with rational arithmetic, rounded once to fp64."""
    fr = [Fraction(float(v)) for v in row]
    out = np.empty(S.shape[0], dtype=np.float64)
    for j in range(S.shape[0]):
        acc = Fraction(0)
        for l in range(S.shape[1]):
            acc += fr[l] if S[j, l] > 0 else -fr[l]
        out[j] = float(acc)   # Fraction -> float rounds to nearest, ties even
    return out


def rotate(W: np.ndarray, b: int) -> np.ndarray:
    """R2: blockwise W . H_K along the last axis, each +-1 sum exact, then x c_b.

    ``W`` holds BF16 values as fp64, shape [..., K] with K % b == 0.  Row-blocks
    whose sums are provably exact go through one BLAS matmul with S_b; the rest
    are summed exactly with rational arithmetic.
    """
    W = np.asarray(W, dtype=np.float64)
    K = W.shape[-1]
    if K % b:
        raise ValueError("K must be a multiple of the Hadamard block")
    S = sylvester(b).astype(np.float64)
    lead = W.shape[:-1]
    blk = W.reshape(-1, K // b, b)
    sums = blk @ S                       # S is symmetric: W . S == (S . W^T)^T
    exact = block_sum_is_exact(blk)
    if not exact.all():
        Si = sylvester(b)
        for i, kb in zip(*np.nonzero(~exact)):
            sums[i, kb] = _exact_block_sums(blk[i, kb], Si)
    return (sums * hadamard_scale(b)).reshape(*lead, K)


def rotation_inexact_blocks(W: np.ndarray, b: int) -> int:
    """Number of row-blocks that fail the fp64 exact-sum test (diagnostic)."""
    W = np.asarray(W, dtype=np.float64)
    blk = W.reshape(-1, W.shape[-1] // b, b)
    return int((~block_sum_is_exact(blk)).sum())


def fwht(x: np.ndarray, b: int) -> np.ndarray:
    """Activation rotation x_rot = H_K x per token (same definition as ``rotate``)."""
    return rotate(x, b)


# ---------------------------------------------------------------------------
# [Spark] Tier A: salience and top-12.5 % selection
# ---------------------------------------------------------------------------


def column_ssq(W_rot: np.ndarray, chunk: int = SSQ_CHUNK, group: int = SSQ_GROUP) -> np.ndarray:
    """R3: per-column sum of squares in the fixed three-level order."""
    M, K = W_rot.shape
    chunk_sums = []
    for c0 in range(0, M, chunk):
        part = np.zeros(K, dtype=np.float64)
        for i in range(c0, min(c0 + chunk, M)):
            w = W_rot[i]
            part = part + w * w
        chunk_sums.append(part)
    total = np.zeros(K, dtype=np.float64)
    for g0 in range(0, len(chunk_sums), group):
        gsum = np.zeros(K, dtype=np.float64)
        for part in chunk_sums[g0:g0 + group]:
            gsum = gsum + part
        total = total + gsum
    return total


def salience(W_rot: np.ndarray, act_scale: np.ndarray) -> np.ndarray:
    """score_j = a_j * sqrt(sum_i W_rot[i, j]^2) (Tier A equation, R3)."""
    a = np.asarray(act_scale, dtype=np.float32).astype(np.float64)
    return a * np.sqrt(column_ssq(W_rot))


def select_salient(score: np.ndarray, n_sal: int) -> np.ndarray:
    """R4: indices of the n_sal largest scores (ties -> lower index), ascending."""
    score = np.asarray(score, dtype=np.float64)
    if np.isnan(score).any():
        raise ValueError("NaN salience score")
    idx = np.arange(score.size)
    order = np.lexsort((idx, -score))     # primary: score desc, secondary: index asc
    return np.sort(order[:n_sal]).astype(np.int32)


# ---------------------------------------------------------------------------
# [Spark] Tier B + [MiniCPM] §2: INT4 group RTN;  [Spark] Tier A: INT8
# ---------------------------------------------------------------------------


def quantize_int4(W_rot: np.ndarray, sal_idx: np.ndarray, group: int = GROUP):
    """R5: returns (q int8 [M][K] in [-8,7], s4 fp64 [M][K/group] BF16 values)."""
    M, K = W_rot.shape
    Wbg = W_rot.copy()
    Wbg[:, np.asarray(sal_idx, dtype=np.int64)] = 0.0
    g = Wbg.reshape(M, K // group, group)
    absmax = np.abs(g).max(axis=-1)
    s4 = rn_bf16(absmax / 7.0)
    with np.errstate(divide="ignore"):
        inv = np.where(s4 > 0, 1.0 / np.where(s4 > 0, s4, 1.0), 0.0)
    q = np.clip(np.rint(g * inv[..., None]), -8, 7)
    q = np.where(s4[..., None] > 0, q, 0.0)
    return q.reshape(M, K).astype(np.int8), s4


def quantize_int8(W_rot: np.ndarray, sal_idx: np.ndarray):
    """R6: returns (q8 int8 [M][n_sal], s8 fp64 [M] BF16 values)."""
    sal = np.asarray(sal_idx, dtype=np.int64)
    Ws = W_rot[:, sal]
    M = W_rot.shape[0]
    if sal.size == 0:
        return np.zeros((M, 0), np.int8), np.zeros(M)
    m = np.abs(Ws).max(axis=1)
    s8 = rn_bf16(m / 127.0)
    inv = np.where(s8 > 0, 1.0 / np.where(s8 > 0, s8, 1.0), 0.0)
    q8 = np.clip(np.rint(Ws * inv[:, None]), -128, 127)
    q8 = np.where(s8[:, None] > 0, q8, 0.0)
    return q8.astype(np.int8), s8


def pack_int4(q: np.ndarray) -> np.ndarray:
    """R9: [M][K] codes in [-8, 7] -> uint8 [M][K/2], even column in the low nibble."""
    u = (np.asarray(q, dtype=np.int64) & 0xF).astype(np.uint8)
    return (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)


def unpack_int4(p: np.ndarray) -> np.ndarray:
    p = np.asarray(p, dtype=np.uint8).astype(np.int64)
    lo, hi = p & 0xF, p >> 4
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    q = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.int8)
    q[:, 0::2], q[:, 1::2] = lo, hi
    return q


def dequant_int4(q: np.ndarray, s4: np.ndarray, group: int = GROUP) -> np.ndarray:
    """What4 = Q . s ([MiniCPM] §2), fp64 [M][K]."""
    M, K = q.shape
    return (q.astype(np.float64).reshape(M, K // group, group) * s4[..., None]).reshape(M, K)


# ---------------------------------------------------------------------------
# [Spark] Tier C / [MiniCPM] §2: low-rank residual compensation
# ---------------------------------------------------------------------------


def residual(W_rot: np.ndarray, sal_idx: np.ndarray, q: np.ndarray, s4: np.ndarray):
    """R7: R = W_bg - What4 in the rotated domain (fp64)."""
    Wbg = W_rot.copy()
    Wbg[:, np.asarray(sal_idx, dtype=np.int64)] = 0.0
    return Wbg - dequant_int4(q, s4)


def svd_factors(R: np.ndarray, r: int, round_bf16: bool = True):
    """Truncated SVD R ~= A.B, A = U_r sqrt(S_r), B = sqrt(S_r) V_r^T (LAPACK gesdd).

    Returns (A [M][r], B [r][K], singular values); A and B rounded to BF16
    values unless ``round_bf16`` is False.
    """
    U, S, Vt = np.linalg.svd(R, full_matrices=False)
    sq = np.sqrt(S[:r])
    A = U[:, :r] * sq[None, :]
    B = sq[:, None] * Vt[:r]
    if round_bf16:
        A, B = rn_bf16(A), rn_bf16(B)
    return A, B, S


# ---------------------------------------------------------------------------
# The whole encoder and the runtime forward
# ---------------------------------------------------------------------------


def encode(W: np.ndarray, act_scale: np.ndarray, block: int, rank: int,
           n_sal: int | None = None, with_svd: bool = True) -> dict:
    """Offline half: rotation, salience, INT8 tier, INT4 tier, packing, SVD.

    ``W`` holds BF16 values as fp64 [M][K]; ``act_scale`` is FP32 [K].
    """
    W = np.asarray(W, dtype=np.float64)
    M, K = W.shape
    if n_sal is None:
        n_sal = K // SAL_DEN
    W_rot = rotate(W, block)
    score = salience(W_rot, act_scale)
    sal = select_salient(score, n_sal)
    q, s4 = quantize_int4(W_rot, sal)
    q8, s8 = quantize_int8(W_rot, sal)
    out = dict(M=M, K=K, block=block, rank=rank, n_sal=n_sal, W_rot=W_rot,
               score=score, sal_idx=sal, q=q, q4=pack_int4(q), s4=s4, q8=q8,
               s8=s8, inexact_blocks=rotation_inexact_blocks(W, block))
    if with_svd:
        R = residual(W_rot, sal, q, s4)
        A, B, S = svd_factors(R, rank)
        out.update(R=R, U=A, V=B, sigma=S)
    return out


def forward(enc: dict, x: np.ndarray, bias: np.ndarray | None = None,
            U: np.ndarray | None = None, V: np.ndarray | None = None) -> np.ndarray:
    """R8 / [MiniCPM] §2 runtime equation on the packed form, fp64 [T][M].

    ``x`` holds BF16 values as fp64 [T][K].  ``U``/``V`` default to the
    encoder's BF16 SVD factors (A, B); pass them to use other factors.
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    xr = rotate(x, enc["block"])
    W4 = dequant_int4(unpack_int4(enc["q4"]), enc["s4"])
    y = xr @ W4.T
    sal = enc["sal_idx"].astype(np.int64)
    if sal.size:
        y = y + (xr[:, sal] @ enc["q8"].astype(np.float64).T) * enc["s8"][None, :]
    U = enc.get("U") if U is None else U
    V = enc.get("V") if V is None else V
    if U is not None and V is not None and U.shape[1] > 0:
        y = y + (xr @ np.asarray(V, np.float64).T) @ np.asarray(U, np.float64).T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y


def dense_effective_weight(enc: dict, U=None, V=None) -> np.ndarray:
    """W_eff in the original domain: (What4 + scatter(What8) + A.B) . H_K^T."""
    M, K, b = enc["M"], enc["K"], enc["block"]
    Wr = dequant_int4(unpack_int4(enc["q4"]), enc["s4"])
    sal = enc["sal_idx"].astype(np.int64)
    Wr[:, sal] += enc["q8"].astype(np.float64) * enc["s8"][:, None]
    U = enc.get("U") if U is None else U
    V = enc.get("V") if V is None else V
    if U is not None and V is not None:
        Wr = Wr + np.asarray(U, np.float64) @ np.asarray(V, np.float64)
    H = hadamard(b)
    return (Wr.reshape(M, K // b, b) @ H.T).reshape(M, K)


# ---------------------------------------------------------------------------
# Storage arithmetic ([Spark] Empirical Scorecard)
# ---------------------------------------------------------------------------


def packed_bytes(M: int, K: int, rank: int, n_sal: int | None = None,
                 group: int = GROUP) -> int:
    """Bytes of one encoded matrix: q4 + s4 + q8 + s8 + sal_idx + U + V."""
    if n_sal is None:
        n_sal = K // SAL_DEN
    return (M * K // 2 + M * (K // group) * 2 + M * n_sal + M * 2 + n_sal * 4
            + M * rank * 2 + rank * K * 2)


def spark_model_footprint(hubs=(3, 7, 11, 15, 19, 23, 27, 31, 35), layers=36,
                          hidden=2560, inter=10240, r_std=16, r_hub=32,
                          with_sal_idx=False) -> dict:
    """Predicted MLP bytes of the Spark release under the dense layout (R5).

    Returns the DV-SSQ MLP bytes and the BF16 MLP bytes, so that the pages'
    total footprint can be compared by difference (non-MLP tensors are BF16
    on both sides).
    """
    mlp = 0
    bf16 = 0
    for l in range(layers):
        r = r_hub if l in hubs else r_std
        for (M, K) in ((inter, hidden), (inter, hidden), (hidden, inter)):
            n_sal = K // SAL_DEN
            b = packed_bytes(M, K, r, n_sal)
            if not with_sal_idx:
                b -= n_sal * 4
            mlp += b
            bf16 += M * K * 2
    return dict(mlp_dvssq=mlp, mlp_bf16=bf16)


# ---------------------------------------------------------------------------
# Gated MLP stack (per layer: down(GELU(gate x) * up x)), exact erf GELU
# ---------------------------------------------------------------------------


def gelu(v: np.ndarray) -> np.ndarray:
    """Exact (erf) GELU, v * Phi(v), in fp64.

    Phi(v) = erfc(-v / sqrt 2) / 2 -- the same function as (1 + erf(v/sqrt 2))/2,
    written so that it keeps its relative accuracy for negative v (1 + erf
    cancels to 0 in fp64 below v ~ -8).
    """
    from scipy.special import erfc
    v = np.asarray(v, dtype=np.float64)
    return 0.5 * v * erfc(-v / math.sqrt(2.0))


def gelu_mul(g: np.ndarray, u: np.ndarray) -> np.ndarray:
    """R10: h = RN_bf16(gelu(g) * u) for BF16 g, u held as fp64."""
    return rn_bf16(gelu(np.asarray(g, np.float64)) * np.asarray(u, np.float64))


def mlp_block(enc_gate: dict, enc_up: dict, enc_down: dict, x: np.ndarray) -> np.ndarray:
    """R10: one Spark-shaped MLP block on the packed form, BF16 between steps.

    g = RN_bf16(gate x), u = RN_bf16(up x), h = RN_bf16(gelu(g) u),
    x_next = RN_bf16(down h); every projection is forward() in fp64.
    """
    g = rn_bf16(forward(enc_gate, x))
    u = rn_bf16(forward(enc_up, x))
    h = gelu_mul(g, u)
    return rn_bf16(forward(enc_down, h))


# ---------------------------------------------------------------------------
# KV-BSS attention ([Spark] "2. KV-BSS: Key-Value Binding Softmax
# Sharpening"; forum post "Architectural Proposal: KV-BSS", implementation
# notes): focus factor and attention haze truncation
# ---------------------------------------------------------------------------


def bss_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, tau: float = 1.10,
                  haze: float = 12.0) -> np.ndarray:
    """Attention of the query tokens over their whole context with KV-BSS.

    q [B][Hq][d], k and v [B][Hkv][L][d] (BF16 values as fp64), Hq a multiple
    of Hkv (grouped-query attention: query head h reads KV head h // (Hq/Hkv)).
    Per query head, in fp64:
      s_l = (q . k_l) * tau / sqrt(d)           (focus factor scaling)
      s_l -> -inf where s_l < max_l s_l - haze  (attention haze truncation;
                                                 haze <= 0 or inf disables it)
      p = softmax(s),  out = sum_l p_l v_l.
    Reading R11: the threshold is taken on the scaled logits over the keys the
    query attends (the whole context here), as the implementation notes apply
    it to attn_weights before the softmax.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    grp = Hq // Hkv
    out = np.empty((B, Hq, d))
    scale = tau / math.sqrt(d)
    for b in range(B):
        for h in range(Hq):
            kh = h // grp
            s = (k[b, kh] @ q[b, h]) * scale
            m = s.max()
            keep = np.ones_like(s, dtype=bool)
            if 0 < haze < np.inf:
                keep = s >= m - haze
            p = np.where(keep, np.exp(s - m), 0.0)
            out[b, h] = (p @ v[b, kh]) / p.sum()
    return out
