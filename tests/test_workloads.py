"""The synthetic workloads' shapes against the numbers the model cards print
(tests/golden/): the inputs stand in for the cards' layers, so their sizes,
Hadamard blocks and ranks must be the cards'."""
import os

from mixed_precision_weight_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if " = " in line:
                k, v = line.split(" = ")
                out[k.strip()] = v.strip()
    return out


def test_minicpm_workloads_follow_the_card():
    g = _read("minicpm_arch.txt")
    d, b = int(g["hidden"]), int(g["hadamard_block"])
    assert d == 2 ** 11 and d % b == 0
    k, up = synth.WORKLOADS["minicpm_k"], synth.WORKLOADS["minicpm_up"]
    for w in (k, up):
        assert w.K == d and w.block == b
    assert k.rank == int(g["rank_k_proj"])              # the doubled k_proj rank
    assert up.rank == int(g["rank_circuits"])           # a circuit layer (14-28)
    assert int(g["rank_k_proj"]) == 2 * int(g["rank_base"])
    # the attention heads the KV-BSS tests use: head_dim = hidden / query heads
    assert d // int(g["q_heads"]) == 128 and int(g["q_heads"]) % int(g["kv_heads"]) == 0


def test_spark_workloads_follow_the_card():
    g = _read("spark_scorecard.txt")
    H, I = int(g["hidden"]), int(g["intermediate"])
    down, gate = synth.WORKLOADS["spark_down"], synth.WORKLOADS["spark_gate"]
    up = synth.WORKLOADS["spark_up_prefill"]
    assert (down.M, down.K) == (H, I)
    assert (gate.M, gate.K) == (I, H) and (up.M, up.K) == (I, H)
    for w in (down, gate, up):
        assert w.block == int(g["hadamard_block"]) and w.rank == int(g["rank_standard"])
        assert w.n_sal == w.K // 8
