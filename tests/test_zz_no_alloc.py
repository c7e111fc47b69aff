"""The allocation-free decode forward, dvssq_linear_forward_static.

It serves callers that cannot allocate device memory for a workspace (a host
program with no device allocator of its own, or a plug-in host that forbids
allocation): its scratch is a fixed array inside the library.  It must give
the same result as the workspace entry point -- the same kernels on the same
inputs, so the same bits -- also on the second of two calls in a row, when
the array still holds the first call's contents, and a warm call must leave
the device's allocated memory unchanged.

This file is collected last on purpose, so that a run stopping at the first
failure has run every other test before it.
"""
import pytest
import torch

from mixed_precision_weight_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dv():
    import mixed_precision_weight_b200 as pkg
    return pkg.binding


def _layer(dv, name):
    wl = synth.WORKLOADS[name]
    shape = dv.Shape.make(wl.M, wl.K, wl.block, wl.rank)
    U, V = synth.lowrank_factors(wl.M, wl.K, wl.rank, seed=wl.seed)
    packed = dv.PackedWeights.empty(shape, "cuda", U=U.cuda(), V=V.cuda())
    dv.dvssq_encode(shape, wl.weight().cuda(), wl.act_scale().cuda(), packed)
    return wl, shape, packed


@pytest.mark.parametrize("name", ["spark_down", "tiny"])
def test_static_scratch_matches_workspace_entry_point(dv, name):
    wl, shape, packed = _layer(dv, name)
    bias = (synth.activations(1, wl.M, seed=3)[0] * 0.1).cuda()
    # calls in a row: each later call finds the previous call's data in the array
    for T, seed in ((16, 0), (1, 1), (16, 2)):
        x = wl.activations(T, seed_offset=100 + seed).cuda()
        y_static = dv.dvssq_linear_forward_static(shape, packed, x, bias)
        y_ref = dv.dvssq_linear_forward(shape, packed, x, bias, path=dv.PATH_DECODE)
        torch.cuda.synchronize()
        assert torch.equal(y_static, y_ref)
    assert dv.dvssq_device_error() == 0


def test_static_scratch_call_allocates_nothing(dv):
    wl, shape, packed = _layer(dv, "spark_down")
    x = wl.activations(16, seed_offset=7).cuda()
    y = torch.empty((16, wl.M), dtype=torch.float32, device="cuda")
    dv.dvssq_linear_forward_static(shape, packed, x, y=y)          # warm: set-up done
    torch.cuda.synchronize()
    torch_before = torch.cuda.memory_allocated()
    free_before, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        dv.dvssq_linear_forward_static(shape, packed, x, y=y)
    torch.cuda.synchronize()
    free_after, _ = torch.cuda.mem_get_info()
    assert torch.cuda.memory_allocated() == torch_before
    assert free_after == free_before
    assert torch.equal(y, dv.dvssq_linear_forward(shape, packed, x, path=dv.PATH_DECODE))


def test_static_scratch_rejects_oversized_shapes(dv):
    big = dv.Shape.make(262144, 8192, 256, 16)
    need = dv.dvssq_forward_workspace_size(big, 16, dv.PATH_DECODE)
    assert need > dv.STATIC_SCRATCH_BYTES
    x = torch.zeros((16, 8), dtype=torch.bfloat16, device="cuda")   # never read
    empty = dv.PackedWeights(*(torch.zeros(16, dtype=torch.uint8, device="cuda"),) * 5)
    with pytest.raises(dv.DvssqError, match="exceeds the static scratch"):
        dv.dvssq_linear_forward_static(big, empty, x)
    wl, shape, packed = _layer(dv, "tiny")
    with pytest.raises(dv.DvssqError, match="unsupported shape"):
        dv.dvssq_linear_forward_static(shape, packed, torch.zeros((17, wl.K), dtype=torch.bfloat16,
                                                                  device="cuda"))
