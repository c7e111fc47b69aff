"""KV-BSS decode attention (dvssq_bss_attention) against the fp64 oracle.

Spark card, "2. KV-BSS": logits scaled by tau / sqrt(d) (tau = 1.10) and
every logit more than 12 nats below the row maximum masked before the
softmax (reading R11).  Inputs are seeded and planted so the truncation
matters: per KV-head group, two binding keys carry the largest logits of
the group's first query head, about 40 % of the context sits 12.5 nats
below that maximum (masked) and about 40 % at 11.5 (kept); with that mass
the output moves by about 1.5 % between truncation on and off.

Tolerance from the arithmetic: the GPU forms each logit as an FP32 dot
product of d BF16 pairs (error about d 2^-24 sum |q_i k_i| tau / sqrt(d),
below 1e-4 nats here) and exp/sums in FP32; a weight's relative error
equals its logit's absolute error, so outputs agree to about 1e-4 and keys
within that distance of the threshold can flip at a cost of e^-12 each.
Checked: relative L2 <= 1e-3 and max abs <= 2e-3 max|out| against the
truncated oracle, and a clear miss against the untruncated one.
"""
import math

import numpy as np
import pytest
import torch

from oracle import dvssq_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dv():
    import mixed_precision_weight_b200 as pkg
    return pkg.binding


def bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def planted(B, Hq, Hkv, d, L, seed, tau=1.10):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, Hq, d))
    k = g.standard_normal((B, Hkv, L, d))
    v = g.standard_normal((B, Hkv, L, d))
    G = Hq // Hkv
    scale = tau / math.sqrt(d)
    for b in range(B):
        for kh in range(Hkv):
            h0 = kh * G
            u = q[b, h0] / np.linalg.norm(q[b, h0])
            qn = np.linalg.norm(q[b, h0])
            # logit of h0 for key c u + e: scale (c qn + q.e)
            targets = np.empty(L)
            targets[:] = 0.0
            sel = g.permutation(L)
            nb = int(0.4 * L)
            targets[sel[:nb]] = 20.0 - 12.5 + g.uniform(-0.3, 0.3, nb)          # masked band
            targets[sel[nb:2 * nb]] = 20.0 - 11.5 + g.uniform(-0.3, 0.3, nb)    # kept band
            targets[sel[2 * nb]] = 20.0                                          # bindings
            targets[sel[2 * nb + 1]] = 18.0
            planted_keys = sel[:2 * nb + 2]
            e = 0.05 * g.standard_normal((planted_keys.size, d))
            e -= np.outer(e @ u, u)
            k[b, kh, planted_keys] = np.outer(targets[planted_keys] / (scale * qn), u) + e
    return bf16(q), bf16(k), bf16(v)


def f64(t):
    return O.torch_bf16_to_f64(t.cpu())


@pytest.mark.parametrize("B,Hq,Hkv,d,L", [(2, 16, 4, 256, 300), (1, 16, 4, 256, 4096),
                                          (2, 16, 2, 128, 1000), (1, 8, 4, 256, 17),
                                          (1, 8, 2, 128, 2050)])
def test_bss_attention_matches_oracle(dv, B, Hq, Hkv, d, L):
    q, k, v = planted(B, Hq, Hkv, d, L, seed=B * 100 + L)
    out = dv.dvssq_bss_attention(q.cuda(), k.cuda(), v.cuda())
    torch.cuda.synchronize()
    qf, kf, vf = f64(q), f64(k), f64(v)
    ref = O.bss_attention(qf, kf, vf, tau=1.10, haze=12.0)
    got = out.double().cpu().numpy()
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    mx = np.abs(got - ref).max() / np.abs(ref).max()
    full = O.bss_attention(qf, kf, vf, tau=1.10, haze=0.0)
    miss = np.linalg.norm(got - full) / np.linalg.norm(full)
    print(f"B={B} Hq={Hq} Hkv={Hkv} d={d} L={L}: rel-L2 {rel:.2e}, max {mx:.2e}, "
          f"vs untruncated {miss:.2e}")
    assert rel <= 1e-3 and mx <= 2e-3, (rel, mx)
    if L >= 300:
        assert miss > 10 * rel, (miss, rel)       # the truncation is what the GPU applied


def test_bss_attention_without_truncation_and_tau_one(dv):
    q, k, v = planted(1, 16, 4, 256, 777, seed=3)
    out = dv.dvssq_bss_attention(q.cuda(), k.cuda(), v.cuda(), tau=1.0, haze=0.0)
    ref = O.bss_attention(f64(q), f64(k), f64(v), tau=1.0, haze=0.0)
    got = out.double().cpu().numpy()
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 1e-3


def test_bss_attention_deterministic_and_rejects_bad_shapes(dv):
    q, k, v = planted(1, 8, 4, 256, 512, seed=4)
    a = dv.dvssq_bss_attention(q.cuda(), k.cuda(), v.cuda())
    b = dv.dvssq_bss_attention(q.cuda(), k.cuda(), v.cuda())
    assert torch.equal(a, b)
    for B, Hq, Hkv, d in ((1, 8, 3, 256), (1, 8, 8, 256), (1, 16, 2, 256), (1, 8, 4, 64)):
        shape = dv.AttnShape(B, Hq, Hkv, d, 16, 1.1, 12.0)
        with pytest.raises(dv.DvssqError):
            dv.dvssq_bss_attention_workspace_size(shape)
    assert dv.dvssq_device_error(clear=True) == 0
