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


def test_gelu_mul_argument_checks(dv):
    P = ctypes.c_void_p
    assert dv.lib.dvssq_gelu_mul(P(256), P(256), P(256), -1, None) == 1
    assert dv.lib.dvssq_gelu_mul(P(256), P(256), P(256), 0, None) == 0   # no-op, no device
    assert dv.lib.dvssq_gelu_mul(None, P(256), P(256), 8, None) == 1
    assert dv.lib.dvssq_gelu_mul(P(256), P(264), P(256), 8, None) == 3


def test_materialize_argument_checks(dv):
    P = ctypes.c_void_p
    s = _shape(dv)
    w = dv._Weights(256, 256, 256, 256, 256, 256, 256)
    assert dv.lib.dvssq_materialize(ctypes.byref(_shape(dv, block=64)), ctypes.byref(w), P(256), None) == 2
    assert dv.lib.dvssq_materialize(ctypes.byref(s), None, P(256), None) == 1
    assert dv.lib.dvssq_materialize(ctypes.byref(s), ctypes.byref(w), None, None) == 1
    assert dv.lib.dvssq_materialize(ctypes.byref(s), ctypes.byref(w), P(264), None) == 3
    no_uv = dv._Weights(256, 256, 256, 256, 256, None, None)          # rank 8 needs U and V
    assert dv.lib.dvssq_materialize(ctypes.byref(s), ctypes.byref(no_uv), P(256), None) == 1
    no_sal = dv._Weights(256, 256, None, None, 256, 256, 256)         # n_sal 64 needs sal_idx, q8
    assert dv.lib.dvssq_materialize(ctypes.byref(s), ctypes.byref(no_sal), P(256), None) == 1
    bad_q4 = dv._Weights(264, 256, 256, 256, 256, 256, 256)
    assert dv.lib.dvssq_materialize(ctypes.byref(s), ctypes.byref(bad_q4), P(256), None) == 3


def test_lowrank_argument_checks(dv):
    P = ctypes.c_void_p
    n = ctypes.c_size_t(0)
    assert dv.lib.dvssq_lowrank_workspace_size(2560, 10240, 16, ctypes.byref(n)) == 0
    small = n.value
    assert small > 0
    assert dv.lib.dvssq_lowrank_workspace_size(2560, 10240, 32, ctypes.byref(n)) == 0
    assert n.value > small                                            # p = r + 16 columns
    for M, K, r in ((2560, 10240, 4), (2560, 10240, 72), (2560, 10240, 12), (24, 10240, 16),
                    (0, 10240, 16)):
        assert dv.lib.dvssq_lowrank_workspace_size(M, K, r, ctypes.byref(n)) == 2, (M, K, r)
    assert dv.lib.dvssq_lowrank_workspace_size(2560, 10240, 16, None) == 1
    call = lambda R, it, ws, wsb: dv.lib.dvssq_lowrank(P(R), 2560, 10240, 16, it, 1, P(256), P(256),
                                                       None, P(ws), wsb, None)
    assert call(256, 65, 256, small) == 1                             # iterations 0..64
    assert call(0, 4, 256, small) == 1                                # no residual
    assert call(264, 4, 256, small) == 3                              # misaligned residual
    assert call(256, 4, 272, small) == 3                              # workspace not 256-aligned
    assert call(256, 4, 256, small - 16) == 4                         # workspace too small


def test_bss_attention_argument_checks(dv):
    P = ctypes.c_void_p
    n = ctypes.c_size_t(0)
    spark = dv.AttnShape(1, 16, 4, 256, 32768, 1.10, 12.0)
    minicpm = dv.AttnShape(2, 16, 2, 128, 1000, 1.10, 12.0)
    for sh in (spark, minicpm):
        assert dv.lib.dvssq_bss_attention_workspace_size(ctypes.byref(sh), ctypes.byref(n)) == 0
        assert n.value > 0
    assert dv.lib.dvssq_bss_attention_workspace_size(ctypes.byref(spark), ctypes.byref(n)) == 0
    need = n.value
    bad = [dv.AttnShape(1, 12, 4, 256, 100, 1.1, 12.0),               # 3 query heads per KV head
           dv.AttnShape(1, 16, 4, 64, 100, 1.1, 12.0),                # head_dim 64
           dv.AttnShape(1, 16, 5, 128, 100, 1.1, 12.0),               # q_heads % kv_heads
           dv.AttnShape(1, 16, 4, 256, 0, 1.1, 12.0)]                 # empty context
    for sh in bad:
        assert dv.lib.dvssq_bss_attention_workspace_size(ctypes.byref(sh), ctypes.byref(n)) == 2
    for tau, haze in ((0.0, 12.0), (-1.0, 12.0), (1.1, float("nan"))):
        sh = dv.AttnShape(1, 16, 4, 256, 100, tau, haze)
        assert dv.lib.dvssq_bss_attention_workspace_size(ctypes.byref(sh), ctypes.byref(n)) == 1
    call = lambda q, ws, wsb: dv.lib.dvssq_bss_attention(ctypes.byref(spark), P(q), P(256), P(256),
                                                         P(256), P(ws), wsb, None)
    assert call(0, 256, need) == 1
    assert call(264, 256, need) == 3
    assert call(256, 272, need) == 3
    assert call(256, 256, need - 16) == 4


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
