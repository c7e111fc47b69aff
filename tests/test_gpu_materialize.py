"""dvssq_materialize against the fp64 oracle's dense effective weight.

The Spark card's materialize_weights() ("Quickstart & Inference Guide")
turns the packed layer back into plain BF16.  The oracle's
dense_effective_weight forms (What4 + scatter(What8) + U V) . H_K in fp64;
the GPU evaluates it in FP32 and rounds once to BF16.

Tolerance, from the GPU's arithmetic: an output is a b-term +-1 sum (times
1/sqrt b) of v = q s4 (+ q8 s8) + (U V), with U V accumulated over r terms
in FP32 on the tensor cores and the sum formed by log2 b FP32 butterfly
stages.  Its FP32 error is at most about (log2 b + 4) 2^-24 sum_l |v_l| /
sqrt(b) (|v_l| taken with |U| |V| for the rank term): tiny next to the
output except where the b terms cancel.  So a BF16 result may differ from
RN_bf16 of the exact value by one BF16 step plus that bound; and at least
99.9 % of the values are equal bit for bit.  Checked on the configs'
shapes, a ragged odd-M shape, rank 0 and no salient columns.
"""
import numpy as np
import pytest
import torch

from oracle import dvssq_oracle as O
from mixed_precision_weight_b200 import synth

from test_gpu_parity import check_codes, f64, gpu_encode, layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dv():
    import mixed_precision_weight_b200 as pkg
    return pkg.binding


def bf16_step(v):
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -140)))
    return 2.0 ** np.maximum(e - 7, -133)


def fp32_bound(enc, U=None, V=None):
    """Per-output bound of the FP32 evaluation error (see the module text)."""
    M, K, b = enc["M"], enc["K"], enc["block"]
    v = np.abs(O.dequant_int4(O.unpack_int4(enc["q4"]), enc["s4"]))
    sal = enc["sal_idx"].astype(np.int64)
    v[:, sal] += np.abs(enc["q8"].astype(np.float64) * enc["s8"][:, None])
    U = enc.get("U") if U is None else U
    V = enc.get("V") if V is None else V
    if U is not None and V is not None and np.asarray(U).shape[1] > 0:
        v += np.abs(np.asarray(U, np.float64)) @ np.abs(np.asarray(V, np.float64))
    blk = v.reshape(M, K // b, b).sum(axis=-1) / np.sqrt(b)
    gamma = (np.log2(b) + 4) * 2.0 ** -24
    return np.repeat(gamma * blk, b, axis=1)


def check_materialized(W_gpu, enc, U=None, V=None):
    ref = O.rn_bf16(O.dense_effective_weight(enc, U=U, V=V))
    got = f64(W_gpu)
    eq = float(np.mean(got == ref))
    far = np.abs(got - ref) > bf16_step(ref) * 1.0000001 + fp32_bound(enc, U, V)
    assert not far.any(), (int(far.sum()), np.argwhere(far)[:5])
    assert eq >= 0.999, eq
    return eq


@pytest.mark.parametrize("name", ["tiny", "minicpm_k", "spark_down", "minicpm_up"])
def test_materialize_matches_oracle(dv, name):
    L = layer(dv, name)
    W = dv.dvssq_materialize(L.shape, L.packed)
    torch.cuda.synchronize()
    check_materialized(W, L.enc)
    assert dv.dvssq_device_error(clear=True) == 0


@pytest.mark.parametrize("M,K,block,n_sal,rank", [(201, 384, 128, 48, 8), (77, 512, 256, 0, 0),
                                                  (64, 1024, 128, 1024, 16)])
def test_materialize_ragged_and_degenerate(dv, M, K, block, n_sal, rank):
    W = synth.weight(M, K, seed=M + K, n_outlier_cols=2, outlier_scale=20.0)
    act = synth.act_scale(K, seed=M)
    enc = O.encode(f64(W), act.numpy(), block, rank, n_sal=n_sal)
    U = V = None
    if rank:
        U = torch.from_numpy(enc["U"].astype(np.float32)).to(torch.bfloat16).cuda().contiguous()
        V = torch.from_numpy(enc["V"].astype(np.float32)).to(torch.bfloat16).cuda().contiguous()
    shape, packed, _, _ = gpu_encode(dv, W, act, block, rank, n_sal, U=U, V=V)
    check_codes(shape, packed, enc)
    Wg = dv.dvssq_materialize(shape, packed)
    torch.cuda.synchronize()
    if rank == 0:
        check_materialized(Wg, enc, U=np.zeros((M, 0)), V=np.zeros((0, K)))
    else:
        check_materialized(Wg, enc)


def test_materialized_weight_reproduces_the_forward(dv):
    # W_eff x (BF16 weights, fp64 product) against the packed forward: the only
    # difference is the BF16 rounding of W_eff (relative 2^-9 per weight)
    L = layer(dv, "spark_down")
    W = f64(dv.dvssq_materialize(L.shape, L.packed))
    x = f64(L.wl.activations(4))
    y = x @ W.T
    ref = O.forward(L.enc, x)
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) < 4e-3


def test_materialize_rejects_bad_arguments(dv):
    L = layer(dv, "tiny")
    wc = L.packed._c(L.shape)
    import ctypes
    buf = torch.empty(L.wl.M * L.wl.K + 8, dtype=torch.bfloat16, device="cuda")
    assert dv.lib.dvssq_materialize(ctypes.byref(L.shape), ctypes.byref(wc),
                                    ctypes.c_void_p(buf.data_ptr() + 2), None) == 3   # MISALIGNED
    assert dv.lib.dvssq_materialize(ctypes.byref(L.shape), ctypes.byref(wc), None, None) == 1
