"""The encoder's exact +-1 Hadamard sum (csrc/exact_sum.cuh), built for the
host and checked against rational arithmetic.

The encoder's codes are defined on RN64 of the exact sum sum_l S_b[o, l] w_l
(MiniCPM5-2B-Hadamard-GSQ model card, Mathematical Foundations §1, with the
scale applied once afterwards).  Row-blocks whose BF16 exponents are spread
too widely for an exact fp64 butterfly take this integer path on the GPU;
here the same routine runs on the CPU against Python's Fraction, whose float()
conversion rounds to nearest, ties to even.
"""
import os
import random
import shutil
import subprocess
from fractions import Fraction

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "mixed_precision_weight_b200", "csrc")


@pytest.fixture(scope="module")
def exe(tmp_path_factory):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no host C++ compiler")
    out = str(tmp_path_factory.mktemp("exact") / "exact_sum_host")
    subprocess.run([cxx, "-O2", "-std=c++17", "-I", CSRC,
                    os.path.join(ROOT, "tests", "exact_sum_host.cpp"), "-o", out], check=True)
    return out


def bf16_value(bits):
    e, m, s = (bits >> 7) & 0xFF, bits & 0x7F, bits >> 15
    v = Fraction(m, 1 << 7) * Fraction(2) ** -126 if e == 0 else \
        Fraction(128 + m, 128) * Fraction(2) ** (e - 127)
    return -v if s else v


def exact(bits, o):
    acc = Fraction(0)
    for l, w in enumerate(bits):
        v = bf16_value(w)
        acc += -v if bin(o & l).count("1") & 1 else v
    return float(acc)


def random_block(rng, b, lo_exp, hi_exp, zeros=0.0):
    out = []
    for _ in range(b):
        if rng.random() < zeros:
            out.append(rng.choice([0x0000, 0x8000]))
            continue
        e = rng.randint(lo_exp, hi_exp)          # biased exponent 0..254
        out.append((rng.randint(0, 1) << 15) | (e << 7) | rng.randint(0, 127))
    return out


def run(exe, cases):
    text = "".join(f"{len(w)} {o} " + " ".join(f"{v:x}" for v in w) + "\n" for w, o in cases)
    res = subprocess.run([exe], input=text, capture_output=True, text=True, check=True)
    return [float.fromhex(t) for t in res.stdout.split()]


def test_exact_sum_matches_rational_arithmetic(exe):
    rng = random.Random(0)
    cases = []
    for b in (128, 256):
        for lo, hi in ((1, 254), (0, 40), (100, 160), (120, 130), (0, 254)):
            for _ in range(6):
                w = random_block(rng, b, lo, hi, zeros=0.2)
                cases.append((w, rng.randrange(b)))
        # planted cancellations: x, tiny, -x leaves exactly the tiny value
        w = [0] * b
        w[0], w[1], w[2] = 0x3F80, 0x2180, 0xBF80          # 1, 2^-60, -1
        cases += [(w, 0), (w, 1), (w, 3), (w, b - 1)]
        # a round-to-even tie: 1 + 2^-53 (as +1 and +2^-53) rounds down to 1
        w = [0] * b
        w[0], w[1] = 0x3F80, 0x2500                          # 1, 2^-53
        cases += [(w, 0), (w, 2)]
        # 1 + 2^-53 + 2^-80: above the tie, rounds up
        w = [0] * b
        w[0], w[1], w[2] = 0x3F80, 0x2500, 0x1780
        cases += [(w, 0)]
        # subnormal BF16 inputs only, and an all-zero block
        cases += [([rng.randint(0, 0x7F) | (rng.randint(0, 1) << 15) for _ in range(b)], 5),
                  ([0] * b, 7)]
    got = run(exe, cases)
    want = [exact(w, o) for w, o in cases]
    assert len(got) == len(want)
    for g, wv, (w, o) in zip(got, want, cases):
        assert g == wv and (g != 0.0 or np.copysign(1.0, g) == 1.0), (g, wv, o)
    assert 1.0 in got and 2.0 ** -60 in got                  # the planted cases are live
