"""The MLP-stack entry points' host-side checks, without a GPU.

The layer table (gate, up, down per block) is validated on the host before
any device work: every projection's shape against the stack's hidden and
intermediate sizes, one Hadamard block size, hidden and intermediate sizes
that are multiples of 512, ranks that are multiples of 8 and at most 32, salient
counts that are multiples of 32, and 16-byte aligned buffers.  The workspace
query answers on the host.  The buffers here are host tensors: these calls
read only their addresses.
"""
import pytest
import torch

OK, INVALID_ARG, UNSUPPORTED_SHAPE, MISALIGNED = 0, 1, 2, 3


@pytest.fixture(scope="module")
def dv():
    import mixed_precision_weight_b200 as pkg
    return pkg.binding


def _mat(dv, M, K, r, block=256, n_sal=None):
    shape = dv.Shape.make(M, K, block, r, n_sal=n_sal)
    U = torch.empty((M, max(r, 1)), dtype=torch.bfloat16)
    V = torch.empty((max(r, 1), K), dtype=torch.bfloat16)
    return shape, dv.PackedWeights.empty(shape, device="cpu", U=U, V=V)


def _layer(dv, H, I, ranks=(8, 8, 8), blocks=(256, 256, 256), n_sal=(None, None, None)):
    dims = ((I, H), (I, H), (H, I))
    return tuple(_mat(dv, M, K, r, b, n) for (M, K), r, b, n in zip(dims, ranks, blocks, n_sal))


def _status(dv, layers):
    try:
        dv.dvssq_mlp_stack_workspace_size(layers)
    except dv.DvssqError as e:
        return e.status
    return OK


def test_workspace_query_answers_on_the_host(dv):
    H, I = 512, 1024
    one = dv.dvssq_mlp_stack_workspace_size([_layer(dv, H, I)])
    two = dv.dvssq_mlp_stack_workspace_size([_layer(dv, H, I), _layer(dv, H, I)])
    ranked = dv.dvssq_mlp_stack_workspace_size([_layer(dv, H, I, ranks=(32, 32, 32))])
    # holds at least (V H) in FP32 for every matrix and the BF16 intermediate h
    vh = lambda r: 4 * (r * H + r * H + r * I)
    assert one >= vh(8) + 2 * I
    assert two - one >= vh(8)               # a second layer adds its (V H) at least
    assert ranked - one >= vh(32) - vh(8)
    assert _status(dv, [_layer(dv, 2560, 10240, ranks=(16, 16, 24))]) == OK


@pytest.mark.parametrize("case,expected", [
    ("empty", INVALID_ARG),
    ("gate_down_swapped", UNSUPPORTED_SHAPE),
    ("hidden_not_512_multiple", UNSUPPORTED_SHAPE),
    ("second_layer_other_width", UNSUPPORTED_SHAPE),
    ("mixed_blocks", UNSUPPORTED_SHAPE),
    ("rank_above_32", UNSUPPORTED_SHAPE),
    ("rank_not_multiple_of_8", UNSUPPORTED_SHAPE),
    ("n_sal_not_multiple_of_32", UNSUPPORTED_SHAPE),
    ("misaligned_q4", MISALIGNED),
])
def test_rejects_bad_layer_tables(dv, case, expected):
    H, I = 512, 1024
    if case == "empty":
        layers = []
    elif case == "gate_down_swapped":
        g, u, d = _layer(dv, H, I)
        layers = [(d, u, g)]
    elif case == "hidden_not_512_multiple":
        layers = [_layer(dv, 768, 1536)]
    elif case == "second_layer_other_width":
        layers = [_layer(dv, H, I), _layer(dv, H, 2048)]
    elif case == "mixed_blocks":
        layers = [_layer(dv, H, I, blocks=(128, 256, 256))]
    elif case == "rank_above_32":
        layers = [_layer(dv, H, I, ranks=(8, 40, 8))]
    elif case == "rank_not_multiple_of_8":
        layers = [_layer(dv, H, I, ranks=(8, 8, 12))]
    elif case == "n_sal_not_multiple_of_32":
        layers = [_layer(dv, H, I, n_sal=(48, None, None))]
    else:
        g, u, d = _layer(dv, H, I)
        shape, packed = g
        base = torch.empty(packed.q4.numel() + 16, dtype=torch.uint8)
        off = (16 - base.data_ptr() % 16) % 16 + 1          # one byte past a 16-byte boundary
        packed.q4 = base[off:off + packed.q4.numel()].view(packed.q4.shape)
        layers = [((shape, packed), u, d)]
    assert _status(dv, layers) == expected


def test_plan_query_for_the_spark_stack(dv):
    # 36 Spark blocks (hidden 2560, intermediate 10240, n_sal = K / 8; ranks
    # 16 and 24 as in the bench's stack) on a B200's 148 SMs
    layers = [_layer(dv, 2560, 10240, ranks=(r, r, r)) for r in [16] * 14 + [24] * 15 + [16] * 7]
    p = dv.dvssq_mlp_stack_plan_query(layers, 148)
    assert p["ctas"] == 148 and p["threads"] == 512
    # gate/up rows are 1280 + 80 + 320 + 2 r bytes: ten of them per slot; down
    # rows 6768 bytes at r = 24: two per slot, inside the same slot size
    assert p["rows_per_tile_gate_up"] == 10 and p["rows_per_tile_down"] == 2
    assert p["slot_bytes"] >= 10 * (1280 + 80 + 320 + 2 * 24)
    assert p["slot_bytes"] >= 2 * (5120 + 320 + 1280 + 2 * 24)
    assert p["ring_slots"] >= 2
    assert p["ring_slots"] * p["slot_bytes"] < p["smem_bytes"] <= 232448   # 227 KB opt-in
    # the plan does not depend on the SM count up to the limit, and stops there
    assert dv.dvssq_mlp_stack_plan_query(layers, 160)["ring_slots"] == p["ring_slots"]
    for sm, status in ((161, UNSUPPORTED_SHAPE), (0, INVALID_ARG)):
        with pytest.raises(dv.DvssqError) as e:
            dv.dvssq_mlp_stack_plan_query(layers, sm)
        assert e.value.status == status


def test_plan_query_rejects_what_the_workspace_query_rejects(dv):
    g, u, d = _layer(dv, 512, 1024)
    assert dv.dvssq_mlp_stack_plan_query([(g, u, d)], 148)["ring_slots"] >= 2
    with pytest.raises(dv.DvssqError) as e:
        dv.dvssq_mlp_stack_plan_query([(d, u, g)], 148)
    assert e.value.status == UNSUPPORTED_SHAPE
