"""GPU vs the fp64 oracle for the MLP-block glue and the decode edge paths.

- dvssq_gelu_mul against oracle.gelu_mul (reading R10): at least 99% of the
  BF16 values equal, and none more than one BF16 step apart (the GPU
  evaluates erfc and the product in FP32).
- One Spark-shaped MLP block (reduced sizes), teacher-forced: every GPU step
  is fed the oracle's input for that step.
- A layer whose salient columns are all contiguous (so a few slabs carry
  every salient entry): the decode kernels' salient staging overflows and
  takes their global-memory path.
"""
import numpy as np
import pytest
import torch

from oracle import dvssq_oracle as O
from mixed_precision_weight_b200 import synth

from test_gpu_parity import assert_y_close, check_codes, f64, gpu_encode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dv():
    import mixed_precision_weight_b200 as pkg
    return pkg.binding


def bf16_step(v):
    """Spacing of BF16 values at |v| (2^-133 throughout the subnormal range)."""
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -140)))
    return 2.0 ** np.maximum(e - 7, -133)


def test_gelu_mul_matches_oracle(dv):
    gen = torch.Generator().manual_seed(11)
    n = 10007                                   # not a multiple of 8: the tail path too
    g = (torch.randn(n, generator=gen) * 3).to(torch.bfloat16)
    u = torch.randn(n, generator=gen).to(torch.bfloat16)
    g[:4] = torch.tensor([0.0, -0.0, 30.0, -30.0])
    h = dv.dvssq_gelu_mul(g.cuda(), u.cuda()).cpu()
    ref = O.gelu_mul(f64(g), f64(u))
    got = f64(h)
    # FP32 evaluation of erfc and of the product can move a value across a
    # BF16 rounding boundary (most often in the tails, where erfc amplifies
    # the rounding of its argument); it can never move it by more than one step
    assert np.mean(got == ref) > 0.99
    assert np.all(np.abs(got - ref) <= bf16_step(ref) * 1.0000001)


def test_gelu_mul_rejects_bad_arguments(dv):
    x = torch.zeros(8, dtype=torch.bfloat16, device="cuda")
    assert dv.lib.dvssq_gelu_mul(None, None, None, 8, None) == 1          # INVALID_ARG
    assert dv.lib.dvssq_gelu_mul(x.data_ptr() + 2, x.data_ptr(), x.data_ptr(), 4, None) == 3
    assert dv.lib.dvssq_gelu_mul(None, None, None, 0, None) == 0          # n = 0: no-op


class _Block:
    def __init__(self, dv, H=512, I=1024, rank=8, seed=21):
        self.encs, self.layers = [], []
        for (M, K), s in (((I, H), seed), ((I, H), seed + 1), ((H, I), seed + 2)):
            W = synth.weight(M, K, seed=s, n_outlier_cols=2, outlier_scale=15.0)
            act = synth.act_scale(K, seed=s)
            enc = O.encode(f64(W), act.numpy(), 256, rank)
            U = torch.from_numpy(enc["U"].astype(np.float32)).to(torch.bfloat16).cuda().contiguous()
            V = torch.from_numpy(enc["V"].astype(np.float32)).to(torch.bfloat16).cuda().contiguous()
            shape, packed, _, _ = gpu_encode(dv, W, act, 256, rank, U=U, V=V)
            check_codes(shape, packed, enc)
            self.encs.append(enc)
            self.layers.append((shape, packed))


@pytest.mark.parametrize("T", [1, 2, 5])
def test_mlp_block_teacher_forced(dv, T):
    blk = _Block(dv)
    (sg, pg), (su, pu), (sd, pd) = blk.layers
    eg, eu, ed = blk.encs
    x = synth.activations(T, 512, seed=T)
    xo = f64(x)
    # gate and up, FP32 outputs against the fp64 oracle
    yg = dv.dvssq_linear_forward(sg, pg, x.cuda())
    yu = dv.dvssq_linear_forward(su, pu, x.cuda())
    assert_y_close(yg.cpu().numpy(), O.forward(eg, xo))
    assert_y_close(yu.cpu().numpy(), O.forward(eu, xo))
    # BF16 outputs are the RN of the FP32 ones
    g16 = dv.dvssq_linear_forward(sg, pg, x.cuda(), y_dtype=dv.Y_BF16)
    assert torch.equal(g16, yg.to(torch.bfloat16))
    # gated product on the oracle's g and u
    go = O.rn_bf16(O.forward(eg, xo))
    uo = O.rn_bf16(O.forward(eu, xo))
    ho = O.gelu_mul(go, uo)
    h = dv.dvssq_gelu_mul(torch.from_numpy(go).to(torch.bfloat16).cuda(),
                          torch.from_numpy(uo).to(torch.bfloat16).cuda())
    assert np.all(np.abs(f64(h) - ho) <= bf16_step(ho) * 1.0000001)
    # down on the oracle's h
    hd = torch.from_numpy(ho).to(torch.bfloat16).cuda()
    yd = dv.dvssq_linear_forward(sd, pd, hd)
    assert_y_close(yd.cpu().numpy(), O.forward(ed, ho))
    # the chained GPU block drifts from the oracle's only by BF16 roundings
    g_gpu = dv.dvssq_linear_forward(sg, pg, x.cuda(), y_dtype=dv.Y_BF16)
    u_gpu = dv.dvssq_linear_forward(su, pu, x.cuda(), y_dtype=dv.Y_BF16)
    y_gpu = dv.dvssq_linear_forward(sd, pd, dv.dvssq_gelu_mul(g_gpu, u_gpu), y_dtype=dv.Y_BF16)
    ref = O.mlp_block(eg, eu, ed, xo)
    err = np.linalg.norm(f64(y_gpu) - ref) / np.linalg.norm(ref)
    assert err <= 2e-2, err


@pytest.mark.parametrize("T", [1, 4])
def test_decode_contiguous_salient_columns(dv, T):
    # activation scales that make the first n_sal rotated columns salient:
    # every salient entry falls in the first two slabs
    M, K, n_sal = 4096, 4096, 512
    W = synth.weight(M, K, seed=41)
    act = torch.full((K,), 0.1)
    act[:n_sal] = 1000.0
    enc = O.encode(f64(W), act.numpy(), 256, 0, n_sal=n_sal, with_svd=False)
    assert list(enc["sal_idx"]) == list(range(n_sal))
    shape, packed, _, _ = gpu_encode(dv, W, act, 256, 0, n_sal)
    check_codes(shape, packed, enc)
    x = synth.activations(T, K, seed=5)
    y = dv.dvssq_linear_forward(shape, packed, x.cuda(), path=dv.PATH_DECODE)
    assert_y_close(y.cpu().numpy(), O.forward(enc, f64(x), U=np.zeros((M, 0)), V=np.zeros((0, K))))
    torch.cuda.synchronize()
    assert dv.dvssq_device_error(clear=True) == 0
