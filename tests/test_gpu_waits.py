"""Bounded waits run out cleanly: with a short wait limit, a warp that waits
on an mbarrier nobody arrives at, or on a grid-barrier counter nobody
increments, gives up, sets its bit of the device error word and returns.
The call returns OK, the error word reports the timeout, and the context
stays usable (a forward afterwards matches the oracle).  Nothing faults or
traps: the wait itself simply ends."""
import numpy as np
import pytest
import torch

from oracle import dvssq_oracle as O
from mixed_precision_weight_b200 import synth

from test_gpu_parity import assert_y_close, f64, layer

pytestmark = pytest.mark.gpu

ERR_WAIT_MBARRIER = 1 << 0
ERR_WAIT_GRID = 1 << 3


@pytest.fixture(scope="module")
def dv():
    import mixed_precision_weight_b200 as pkg
    return pkg.binding


@pytest.mark.parametrize("which,bit", [(0, ERR_WAIT_MBARRIER), (1, ERR_WAIT_GRID)])
def test_wait_runs_out_and_reports(dv, which, bit):
    torch.cuda.synchronize()
    assert dv.dvssq_device_error(clear=True) == 0
    dv.dvssq_set_wait_limit(2_000_000)             # about 1 ms at the boost clock
    try:
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        dv.dvssq_selftest_wait(which)
        ev1.record()
        torch.cuda.synchronize()
        ms = ev0.elapsed_time(ev1)
    finally:
        dv.dvssq_set_wait_limit(0)                 # back to the default limit
    assert dv.dvssq_device_error(clear=True) == bit
    assert ms < 1000.0, ms                          # it gave up after the short limit
    # the context still works
    L = layer(dv, "tiny")
    x = L.wl.activations(4)
    y = dv.dvssq_linear_forward(L.shape, L.packed, x.cuda())
    assert_y_close(y.cpu().numpy(), O.forward(L.enc, f64(x)))
    assert dv.dvssq_device_error(clear=True) == 0


def test_selftest_rejects_unknown_kind(dv):
    with pytest.raises(dv.DvssqError):
        dv.dvssq_selftest_wait(2)
