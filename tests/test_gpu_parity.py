"""CUDA path vs the fp64 oracle, through the C ABI.

Bit-exact: INT4 bytes, BF16 scales, salient indices, INT8 codes, residual.
Tolerance (the forward, FP32 output): relative L2 <= 1e-3 and max abs error
<= 1e-2 * max|y| against the fp64 oracle.  dvssq_fwht: relative L2 <= 1e-6.
"""
import numpy as np
import pytest
import torch

from oracle import dvssq_oracle as O
from mixed_precision_weight_b200 import synth

pytestmark = pytest.mark.gpu

REL_L2 = 1e-3
MAX_ABS = 1e-2


@pytest.fixture(scope="module")
def dv():
    import mixed_precision_weight_b200 as pkg
    return pkg.binding


def bits16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f64(t):
    return O.torch_bf16_to_f64(t.cpu())


def assert_y_close(y, ref, rel=REL_L2, mx=MAX_ABS):
    y = np.asarray(y, dtype=np.float64)
    err = y - ref
    r = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300)
    m = np.abs(err).max() / max(np.abs(ref).max(), 1e-300)
    assert r <= rel and m <= mx, (r, m)
    return r, m


def gpu_encode(dv, W, act, block, rank, n_sal=None, resid=False, U=None, V=None):
    M, K = W.shape
    shape = dv.Shape.make(M, K, block, rank, n_sal)
    packed = dv.PackedWeights.empty(shape, "cuda", U=U, V=V)
    R = torch.empty((M, K), dtype=torch.float32, device="cuda") if resid else None
    info = dv.dvssq_encode(shape, W.cuda(), act.cuda(), packed, resid=R, want_info=True)
    torch.cuda.synchronize()
    return shape, packed, info, R


def check_codes(shape, packed, enc, R=None):
    n = shape.n_sal
    assert np.array_equal(packed.q4.cpu().numpy(), enc["q4"])
    assert np.array_equal(bits16(packed.s4), O.f64_to_bf16_bits(enc["s4"]))
    assert np.array_equal(bits16(packed.s8), O.f64_to_bf16_bits(enc["s8"]))
    if n:
        assert np.array_equal(packed.sal_idx[:n].cpu().numpy(), enc["sal_idx"])
        assert np.array_equal(packed.q8[:, :n].cpu().numpy(), enc["q8"])
    if R is not None:
        ref = O.residual(enc["W_rot"], enc["sal_idx"], enc["q"], enc["s4"]).astype(np.float32)
        assert np.array_equal(R.cpu().numpy(), ref)


class Layer:
    """A workload's layer encoded by the oracle (with SVD) and by the GPU."""

    def __init__(self, dv, wl, n_sal=None, rank=None, act=None, W=None):
        self.wl = wl
        self.W = wl.weight() if W is None else W
        self.act = wl.act_scale() if act is None else act
        self.rank = wl.rank if rank is None else rank
        self.n_sal = wl.n_sal if n_sal is None else n_sal
        self.enc = O.encode(f64(self.W), self.act.numpy(), wl.block, self.rank, n_sal=self.n_sal)
        self.U = torch.from_numpy(self.enc["U"].astype(np.float32)).to(torch.bfloat16).cuda()
        self.V = torch.from_numpy(self.enc["V"].astype(np.float32)).to(torch.bfloat16).cuda()
        self.shape, self.packed, self.info, self.R = gpu_encode(
            dv, self.W, self.act, wl.block, self.rank, self.n_sal, resid=True,
            U=self.U.contiguous(), V=self.V.contiguous())


_cache = {}


def layer(dv, name, **kw):
    key = (name, tuple(sorted(kw.items())))
    if key not in _cache:
        _cache[key] = Layer(dv, synth.WORKLOADS[name], **kw)
    return _cache[key]


# ------------------------------------------------------------------ fwht ----

@pytest.mark.parametrize("block,rows,cols", [(256, 5, 512), (128, 7, 384), (256, 1, 10240),
                                             (128, 333, 2048)])
def test_fwht_parity(dv, block, rows, cols):
    x = synth.activations(rows, cols, seed=block + rows, n_outlier=3, outlier_scale=25.0)
    y = dv.dvssq_fwht(x.cuda(), block)
    ref = O.fwht(f64(x), block)
    err = np.linalg.norm(y.cpu().numpy() - ref) / np.linalg.norm(ref)
    assert err <= 1e-6, err


# ---------------------------------------------------------------- encoder ---

@pytest.mark.parametrize("name", ["tiny", "minicpm_k", "spark_down", "minicpm_up"])
def test_encode_bit_exact(dv, name):
    L = layer(dv, name)
    check_codes(L.shape, L.packed, L.enc, L.R)
    assert L.info["inexact_rotation_blocks"] == L.enc["inexact_blocks"] == 0
    assert L.info["nonfinite_scores"] == 0


@pytest.mark.parametrize("M,K,block,n_sal", [(200, 512, 256, 64), (1000, 384, 128, 48),
                                             (77, 256, 256, 0), (64, 1024, 128, 1024)])
def test_encode_ragged_and_degenerate(dv, M, K, block, n_sal):
    W = synth.weight(M, K, seed=M + K, n_outlier_cols=2, outlier_scale=20.0)
    act = synth.act_scale(K, seed=M)
    enc = O.encode(f64(W), act.numpy(), block, 0, n_sal=n_sal, with_svd=False)
    shape, packed, info, R = gpu_encode(dv, W, act, block, 0, n_sal, resid=True)
    check_codes(shape, packed, enc, R)


def test_encode_tied_scores_pick_lowest_indices(dv):
    M, K = 128, 512
    W = synth.weight(M, K, seed=5)
    act = torch.zeros(K, dtype=torch.float32)          # every score is 0: a 512-way tie
    act[100] = 1.0
    enc = O.encode(f64(W), act.numpy(), 256, 0, with_svd=False)
    assert list(enc["sal_idx"][:3]) == [0, 1, 2] and 100 in enc["sal_idx"]
    shape, packed, info, _ = gpu_encode(dv, W, act, 256, 0)
    check_codes(shape, packed, enc)


def test_encode_zero_rows_and_wide_exponent_spread(dv):
    M, K = 64, 512
    Wn = synth.weight(M, K, seed=9).float()
    Wn[3] = 0.0                                         # all-zero row: s4 = s8 = 0
    Wn[7, 0] = 1.0
    Wn[7, 1] = 2.0 ** -60                               # fp64 butterfly would round
    Wn[20, 300] = 2.0 ** 40                             # a second chunk and block
    Wn[20, 301] = -(2.0 ** -30)
    Wn[20, 302] = 2.0 ** -120                           # BF16 subnormal-adjacent tail
    Wn[40, 256:512] = 0.0
    Wn[40, 260] = 3.0 * 2.0 ** -133                     # BF16 subnormals only
    Wn[40, 261] = -(2.0 ** -130)
    W = Wn.to(torch.bfloat16)
    act = synth.act_scale(K, seed=2)
    enc = O.encode(f64(W), act.numpy(), 256, 0, with_svd=False)
    assert enc["inexact_blocks"] >= 2
    shape, packed, info, R = gpu_encode(dv, W, act, 256, 0, resid=True)
    assert info["inexact_rotation_blocks"] == enc["inexact_blocks"]
    # every row, the flagged ones included, bit for bit (codes, scales, salient
    # set, residual)
    check_codes(shape, packed, enc, R)
    assert np.all(packed.q4.cpu().numpy()[3] == 0) and bits16(packed.s8)[3] == 0


@pytest.mark.parametrize("seed", [0, 4])
def test_encode_near_ties_bit_exact_and_valid(dv, seed):
    # exact ties across 16-row chunk boundaries, split by fp64 rounding: the
    # GPU's salient set equals the oracle's (same summation tree) and is a
    # valid top-n_sal set of the exact rational scores
    import exact_topk as X
    W, n_sal = X.near_tie_weight(seed)
    act = torch.ones(W.shape[1], dtype=torch.float32)
    enc = O.encode(f64(W), act.numpy(), 256, 0, n_sal=n_sal, with_svd=False)
    shape, packed, info, R = gpu_encode(dv, W, act, 256, 0, n_sal, resid=True)
    check_codes(shape, packed, enc, R)
    got = packed.sal_idx[:n_sal].cpu().numpy()
    X.check_selection_valid(enc["W_rot"], act.numpy(), got, n_sal)


# ---------------------------------------------------------------- forward ---

@pytest.mark.parametrize("name,T", [("tiny", 4), ("tiny", 1), ("spark_down", 1),
                                    ("spark_down", 2), ("spark_down", 16), ("minicpm_k", 1),
                                    ("minicpm_k", 8), ("minicpm_up", 1), ("minicpm_up", 2),
                                    ("minicpm_up", 8), ("minicpm_up", 16),
                                    ("spark_up_prefill", 1), ("spark_up_prefill", 16)])
def test_forward_decode_parity(dv, name, T):
    L = layer(dv, name)
    x = L.wl.activations(T)
    bias = synth.activations(1, L.wl.M, seed=T)[0] * 0.1
    ref = O.forward(L.enc, f64(x), f64(bias))
    y = dv.dvssq_linear_forward(L.shape, L.packed, x.cuda(), bias.cuda(), path=dv.PATH_DECODE)
    assert_y_close(y.cpu().numpy(), ref)


@pytest.mark.parametrize("name,T", [("tiny", 4), ("tiny", 300), ("minicpm_k", 64),
                                    ("minicpm_up", 64), ("spark_down", 17), ("spark_down", 16)])
def test_forward_prefill_parity(dv, name, T):
    L = layer(dv, name)
    x = L.wl.activations(T)
    ref = O.forward(L.enc, f64(x))
    y = dv.dvssq_linear_forward(L.shape, L.packed, x.cuda(), path=dv.PATH_PREFILL)
    assert_y_close(y.cpu().numpy(), ref)


def test_forward_prefill_full_config(dv):
    # Spark up_proj 10240 x 2560, r = 16, 4096 tokens: the tensor-core workload
    L = layer(dv, "spark_up_prefill")
    x = L.wl.activations(4096)
    ref = O.forward(L.enc, f64(x))
    y = dv.dvssq_linear_forward(L.shape, L.packed, x.cuda())
    r, m = assert_y_close(y.cpu().numpy(), ref)
    check_codes(L.shape, L.packed, L.enc)


def test_forward_bf16_output_and_paths_agree(dv):
    L = layer(dv, "tiny")
    x = L.wl.activations(16)
    y32d = dv.dvssq_linear_forward(L.shape, L.packed, x.cuda(), path=dv.PATH_DECODE)
    y16d = dv.dvssq_linear_forward(L.shape, L.packed, x.cuda(), path=dv.PATH_DECODE, y_dtype=dv.Y_BF16)
    assert torch.equal(y16d, y32d.to(torch.bfloat16))        # BF16 = RN of the FP32 result
    y32p = dv.dvssq_linear_forward(L.shape, L.packed, x.cuda(), path=dv.PATH_PREFILL)
    ref = O.forward(L.enc, f64(x))
    assert_y_close(y32p.cpu().numpy(), ref)
    assert_y_close(y32d.cpu().numpy(), ref)
    y16p = dv.dvssq_linear_forward(L.shape, L.packed, x.cuda(), path=dv.PATH_PREFILL, y_dtype=dv.Y_BF16)
    assert torch.equal(y16p, y32p.to(torch.bfloat16))


@pytest.mark.parametrize("path", [1, 2])
def test_forward_rank0_nsal0_ragged(dv, path):
    M, K, block = 200, 384, 128
    W = synth.weight(M, K, seed=31)
    act = synth.act_scale(K, seed=3)
    for n_sal in (0, 48):
        enc = O.encode(f64(W), act.numpy(), block, 0, n_sal=n_sal, with_svd=False)
        shape, packed, info, _ = gpu_encode(dv, W, act, block, 0, n_sal)
        check_codes(shape, packed, enc)
        for T in (1, 3, 16):
            x = synth.activations(T, K, seed=T)
            y = dv.dvssq_linear_forward(shape, packed, x.cuda(), path=path)
            assert_y_close(y.cpu().numpy(), O.forward(enc, f64(x), U=np.zeros((M, 0)),
                                                      V=np.zeros((0, K))))


def test_forward_deterministic(dv):
    L = layer(dv, "spark_down")
    x = L.wl.activations(16).cuda()
    y1 = dv.dvssq_linear_forward(L.shape, L.packed, x)
    y2 = dv.dvssq_linear_forward(L.shape, L.packed, x)
    assert torch.equal(y1, y2)


def test_no_device_errors(dv):
    torch.cuda.synchronize()
    assert dv.dvssq_device_error(clear=True) == 0
