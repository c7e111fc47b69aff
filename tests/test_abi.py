"""The C ABI without a GPU: the library loads, exports every symbol that
include/dvssq.h declares, sizes workspaces and rejects bad arguments on the
host before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def dv():
    import mixed_precision_weight_b200 as pkg
    return pkg.binding


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "dvssq.h")).read()
    return sorted(set(re.findall(r"DVSSQ_API\s+[\w\s\*]+?\b(dvssq_\w+)\s*\(", src)))


def test_header_declares_the_documented_entry_points():
    syms = _declared_symbols()
    for name in ("dvssq_fwht", "dvssq_encode", "dvssq_linear_forward",
                 "dvssq_encode_workspace_size", "dvssq_forward_workspace_size"):
        assert name in syms


def test_library_exports_every_declared_symbol(dv):
    for name in _declared_symbols():
        assert hasattr(dv.lib, name), name
    assert set(_declared_symbols()) == set(dv.EXPORTED_SYMBOLS)
    assert dv.lib.dvssq_abi_version() == 1


def test_status_strings(dv):
    for s in range(7):
        assert dv.lib.dvssq_status_string(s)
    assert dv.lib.dvssq_status_string(0) == b"ok"


def _shape(dv, **kw):
    base = dict(M=256, K=512, block=256, group=64, n_sal=64, rank=8)
    base.update(kw)
    return dv.Shape(**base)


def test_workspace_sizes(dv):
    s = _shape(dv)
    assert dv.dvssq_encode_workspace_size(s) > 0
    big = _shape(dv, M=2560, K=10240, n_sal=1280, rank=16)
    # one fp64 partial per column and 8-chunk group (128 rows): 20 x K doubles
    assert dv.dvssq_encode_workspace_size(big) >= 20 * 10240 * 8
    d1 = dv.dvssq_forward_workspace_size(big, 1, dv.PATH_AUTO)
    d16 = dv.dvssq_forward_workspace_size(big, 16, dv.PATH_AUTO)
    assert 0 < d1 < d16
    p = dv.dvssq_forward_workspace_size(big, 4096, dv.PATH_AUTO)
    assert p >= 4096 * (10240 + 1280 + 64) * 2
    with pytest.raises(dv.DvssqError):
        dv.dvssq_forward_workspace_size(big, 17, dv.PATH_DECODE)


@pytest.mark.parametrize("kw,status", [
    (dict(block=64), 2), (dict(group=32), 2), (dict(K=500), 2), (dict(K=384, block=256), 2),
    (dict(n_sal=65), 2), (dict(n_sal=1024), 2), (dict(rank=65), 2), (dict(M=0), 2),
    (dict(rank=-1), 2), (dict(rank=12), 2), (dict(K=131072), 2),
])
def test_bad_shapes_rejected(dv, kw, status):
    n = ctypes.c_size_t(0)
    assert dv.lib.dvssq_encode_workspace_size(ctypes.byref(_shape(dv, **kw)), ctypes.byref(n)) == status


def test_null_and_misaligned_buffers_rejected_before_launch(dv):
    s = _shape(dv)
    w = dv._Weights(256, 256, 256, 256, 256, 256, 256)
    P = ctypes.c_void_p
    # NULL weight pointer
    assert dv.lib.dvssq_encode(ctypes.byref(s), None, P(256), ctypes.byref(w), None, None,
                               P(256), 1 << 20, None) == 1
    # misaligned W
    assert dv.lib.dvssq_encode(ctypes.byref(s), P(258), P(256), ctypes.byref(w), None, None,
                               P(256), 1 << 20, None) == 3
    # workspace not 256-byte aligned
    assert dv.lib.dvssq_encode(ctypes.byref(s), P(256), P(256), ctypes.byref(w), None, None,
                               P(272), 1 << 20, None) == 3
    # workspace too small
    assert dv.lib.dvssq_encode(ctypes.byref(s), P(256), P(256), ctypes.byref(w), None, None,
                               P(256), 16, None) == 4
    # forward: bad y dtype, bad path, decode with T > 16, misaligned x
    args = lambda x, T, yd, path, ws: (ctypes.byref(s), ctypes.byref(w), P(x), T, None, P(256),
                                       yd, path, P(256), ws, None)
    assert dv.lib.dvssq_linear_forward(*args(256, 4, 7, 0, 1 << 30)) == 1
    assert dv.lib.dvssq_linear_forward(*args(256, 4, 0, 9, 1 << 30)) == 1
    assert dv.lib.dvssq_linear_forward(*args(256, 17, 0, dv.PATH_DECODE, 1 << 30)) == 2
    assert dv.lib.dvssq_linear_forward(*args(260, 4, 0, 0, 1 << 30)) == 3
    assert dv.lib.dvssq_linear_forward(*args(256, 4, 0, 0, 8)) == 4
    # T == 0 is a no-op that succeeds without a device
    assert dv.lib.dvssq_linear_forward(*args(256, 0, 0, 0, 0)) == 0
    # rank > 0 needs U and V
    w2 = dv._Weights(256, 256, 256, 256, 256, None, None)
    assert dv.lib.dvssq_linear_forward(ctypes.byref(s), ctypes.byref(w2), P(256), 4, None, P(256),
                                       0, 0, P(256), 1 << 30, None) == 1


def test_fwht_argument_checks(dv):
    P = ctypes.c_void_p
    assert dv.lib.dvssq_fwht(P(256), P(256), 4, 500, 256, None) == 2
    assert dv.lib.dvssq_fwht(P(256), P(256), 4, 512, 64, None) == 2
    assert dv.lib.dvssq_fwht(P(256), P(256), -1, 512, 256, None) == 1
    assert dv.lib.dvssq_fwht(P(256), P(256), 0, 512, 256, None) == 0
    assert dv.lib.dvssq_fwht(P(264), P(256), 4, 512, 256, None) == 3


def test_profile_api_without_launches(dv):
    dv.dvssq_profile_reset()
    dv.dvssq_profile_enable(True)
    dv.dvssq_profile_collect()
    assert dv.dvssq_profile_read() == {}
    dv.dvssq_profile_enable(False)


def test_no_cpu_fallback_in_product_path():
    # the binding never imports the oracle and has no torch fallback for compute
    src = open(os.path.join(ROOT, "mixed_precision_weight_b200", "binding.py")).read()
    assert "oracle" not in src.replace("oracle/", "")
    for mod in ("binding.py", "__init__.py", "synth.py"):
        s = open(os.path.join(ROOT, "mixed_precision_weight_b200", mod)).read()
        assert "import oracle" not in s and "from oracle" not in s
