"""The one-launch MLP stack (dvssq_mlp_stack_forward) against the fp64 oracle
and against the chain of single-layer GPU calls.

- Reduced Spark-shaped stacks (hidden 512, intermediate 1024, b = 256) encoded
  by the GPU encoder with the oracle's SVD factors, two ranks: the fused
  output against the oracle's mlp_block applied layer after layer
  (reading R10), and against the GPU chain gate / up / gelu_mul / down.
- The same with the MiniCPM Hadamard block (b = 128) and without the rank-r
  term (rank 0).
- Full Spark shapes (hidden 2560, intermediate 10240, rank 16 and 24): the
  fused output against the GPU chain of the same packed layers.
Both sides round g, u, h and each block output to BF16; the fused kernel
differs from the chain only in FP32 summation order and in forming the
rank-r input as (V H) x, so outputs agree up to BF16 rounding flips.
"""
import numpy as np
import pytest
import torch

from oracle import dvssq_oracle as O
from mixed_precision_weight_b200 import synth

from test_gpu_parity import check_codes, f64, gpu_encode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dv():
    import mixed_precision_weight_b200 as pkg
    return pkg.binding


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def chain(dv, layers, x):
    cur = x
    for (sg, pg), (su, pu), (sd, pd) in layers:
        g = dv.dvssq_linear_forward(sg, pg, cur, y_dtype=dv.Y_BF16)
        u = dv.dvssq_linear_forward(su, pu, cur, y_dtype=dv.Y_BF16)
        cur = dv.dvssq_linear_forward(sd, pd, dv.dvssq_gelu_mul(g, u), y_dtype=dv.Y_BF16)
    return cur


def small_stack(dv, L, H, I, ranks, seed, block=256):
    layers, encs = [], []
    for l in range(L):
        mats, es = [], []
        for which, (M, K) in enumerate(((I, H), (I, H), (H, I))):
            s = seed + 10 * l + which
            W = synth.weight(M, K, seed=s, n_outlier_cols=2, outlier_scale=15.0)
            act = synth.act_scale(K, seed=s)
            enc = O.encode(f64(W), act.numpy(), block, ranks[l])
            U = V = None
            if ranks[l] > 0:
                U = torch.from_numpy(enc["U"].astype(np.float32)).to(torch.bfloat16).cuda().contiguous()
                V = torch.from_numpy(enc["V"].astype(np.float32)).to(torch.bfloat16).cuda().contiguous()
            shape, packed, _, _ = gpu_encode(dv, W, act, block, ranks[l], U=U, V=V)
            check_codes(shape, packed, enc)
            mats.append((shape, packed))
            es.append(enc)
        layers.append(tuple(mats))
        encs.append(es)
    return layers, encs


@pytest.mark.parametrize("ranks", [(8, 16), (16, 8)])
def test_stack_matches_oracle_and_chain(dv, ranks):
    H, I = 512, 1024
    layers, encs = small_stack(dv, 2, H, I, ranks, seed=31 + ranks[0])
    x = synth.activations(1, H, seed=9, n_outlier=3, outlier_scale=25.0)
    stack = dv.MlpStack(layers)
    y = stack.forward(x.cuda())
    torch.cuda.synchronize()
    assert dv.dvssq_device_error(clear=True) == 0
    ref = f64(x)
    for eg, eu, ed in encs:
        ref = O.rn_bf16(O.mlp_block(eg, eu, ed, ref))
    got = f64(y)
    assert rel_l2(got, ref) <= 3e-2, rel_l2(got, ref)
    ch = f64(chain(dv, layers, x.cuda()))
    assert rel_l2(got, ch) <= 1e-2, rel_l2(got, ch)
    # repeatable: the same inputs give the same bits
    assert torch.equal(stack.forward(x.cuda()), y)


@pytest.mark.parametrize("block,ranks", [(128, (24, 8)), (256, (0, 0))])
def test_stack_block128_and_rank0(dv, block, ranks):
    # the MiniCPM Hadamard block (H_128) and a stack without the rank-r term
    H, I = 512, 1024
    layers, encs = small_stack(dv, 2, H, I, ranks, seed=51 + ranks[0], block=block)
    x = synth.activations(1, H, seed=13, n_outlier=3, outlier_scale=25.0)
    y = dv.MlpStack(layers).forward(x.cuda())
    torch.cuda.synchronize()
    assert dv.dvssq_device_error(clear=True) == 0
    ref = f64(x)
    for eg, eu, ed in encs:       # rank 0: the oracle's factors are [M][0] and [0][K]
        ref = O.rn_bf16(O.mlp_block(eg, eu, ed, ref))
    assert rel_l2(f64(y), ref) <= 3e-2, rel_l2(f64(y), ref)
    ch = f64(chain(dv, layers, x.cuda()))
    assert rel_l2(f64(y), ch) <= 1e-2, rel_l2(f64(y), ch)


def test_stack_output_may_alias_input(dv):
    H, I = 512, 1024
    layers, _ = small_stack(dv, 1, H, I, (8,), seed=77)
    stack = dv.MlpStack(layers)
    x = synth.activations(1, H, seed=4).cuda()
    y = stack.forward(x)
    xx = x.clone()
    stack.forward(xx, y=xx)
    assert torch.equal(xx, y)


def test_stack_full_spark_shapes_match_chain(dv):
    H, I = 2560, 10240
    layers = []
    for l in range(2):
        r = (16, 24)[l]
        mats = []
        for which, (M, K) in enumerate(((I, H), (I, H), (H, I))):
            seed = synth.layer_seed(1, l, which)
            shape = dv.Shape.make(M, K, 256, r)
            W = synth.weight_device(M, K, seed, "cuda", n_outlier_cols=max(1, K // 1000),
                                    outlier_scale=15.0)
            act = synth.act_scale(K, seed).cuda()
            U, V = synth.lowrank_factors(M, K, r, seed=seed + 17)
            packed = dv.PackedWeights.empty(shape, "cuda", U=U.cuda(), V=V.cuda())
            dv.dvssq_encode(shape, W, act, packed)
            mats.append((shape, packed))
        layers.append(tuple(mats))
    x = synth.activations(1, H, seed=3, n_outlier=13, outlier_scale=25.0).cuda()
    stack = dv.MlpStack(layers)
    y = stack.forward(x)
    torch.cuda.synchronize()
    assert dv.dvssq_device_error(clear=True) == 0
    ch = chain(dv, layers, x)
    assert rel_l2(f64(y), f64(ch)) <= 1e-2, rel_l2(f64(y), f64(ch))


def test_stack_rejects_bad_layers(dv):
    H, I = 512, 1024
    layers, _ = small_stack(dv, 1, H, I, (8,), seed=5)
    (sg, pg), (su, pu), (sd, pd) = layers[0]
    bad = [((sd, pd), (su, pu), (sg, pg))]           # gate / down swapped
    with pytest.raises(dv.DvssqError):
        dv.dvssq_mlp_stack_workspace_size(bad)
    with pytest.raises(dv.DvssqError):
        dv.dvssq_mlp_stack_workspace_size([])


def _full_block(dv, l, r, base=7):
    """One Spark-shaped block (hidden 2560, intermediate 10240, rank r), encoded
    by the oracle and by the GPU (codes checked bit for bit); stand-in BF16
    factors U, V shared by both sides."""
    H, I = 2560, 10240
    mats, encs = [], []
    for which, (M, K) in enumerate(((I, H), (I, H), (H, I))):
        seed = synth.layer_seed(base, l, which)
        W = synth.weight(M, K, seed, n_outlier_cols=max(1, K // 1000), outlier_scale=15.0)
        act = synth.act_scale(K, seed)
        U, V = synth.lowrank_factors(M, K, r, seed=seed + 17)
        enc = O.encode(f64(W), act.numpy(), 256, r, with_svd=False)
        enc["U"], enc["V"] = f64(U), f64(V)
        shape, packed, _, _ = gpu_encode(dv, W, act, 256, r, U=U.cuda().contiguous(),
                                         V=V.cuda().contiguous())
        check_codes(shape, packed, enc)
        mats.append((shape, packed))
        encs.append(enc)
    return tuple(mats), encs


def test_stack_full_spark_shapes_teacher_forced_oracle(dv):
    # Each block of a two-layer Spark stack (rank 16, then 24) runs as a
    # one-layer stack fed the ORACLE's input for that block, and its BF16
    # output is held to the oracle's block (reading R10: BF16 after gate, up,
    # the gated product and down).  The two computations round at the same
    # four points; their pre-rounding values differ by the GPU's FP32 error,
    # so a fraction of the BF16 values sit one step apart.
    x = f64(synth.activations(1, 2560, seed=21, n_outlier=13, outlier_scale=25.0))
    for l, r in enumerate((16, 24)):
        mats, (eg, eu, ed) = _full_block(dv, l, r)
        ref = O.mlp_block(eg, eu, ed, x)
        xin = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).cuda()
        y = dv.MlpStack([mats]).forward(xin)
        torch.cuda.synchronize()
        assert dv.dvssq_device_error(clear=True) == 0
        got = f64(y)[None, :]
        rl = rel_l2(got, ref)
        mx = float(np.abs(got - ref).max() / np.abs(ref).max())
        eq = float(np.mean(got == ref))
        print(f"block {l} r={r}: rel-L2 {rl:.3e}, max-abs/max|y| {mx:.3e}, equal {eq:.4f}")
        assert rl <= 3e-3 and mx <= 1e-2, (rl, mx)
        assert eq >= 0.80, eq
        x = ref[0]                                       # teacher forcing: the oracle's output
