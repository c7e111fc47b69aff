"""ctypes binding of libdvssq.so, the sm_100a DV-SSQ compressed linear layer.

Argument marshalling only: every step of the encoder and of the forward runs
in the CUDA kernels of the library; this module passes device pointers,
sizes and the current CUDA stream through ctypes, allocates outputs and
workspaces with PyTorch, and raises ``DvssqError`` on a non-OK status.  There
is no CPU or PyTorch fallback: if the library is missing this import fails.

Functions keep the C names (see include/dvssq.h):
    dvssq_fwht, dvssq_encode_workspace_size, dvssq_encode,
    dvssq_forward_workspace_size, dvssq_linear_forward, dvssq_device_error,
    dvssq_mlp_stack_workspace_size, dvssq_mlp_stack_prepare,
    dvssq_mlp_stack_forward, dvssq_profile_* .
``DvssqLinear`` bundles one encoded layer with its workspaces; ``MlpStack``
bundles a stack of gated-GELU MLP blocks with its prepared workspace.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

__all__ = [
    "DvssqError", "Shape", "PackedWeights", "DvssqLinear", "lib", "library_path",
    "dvssq_fwht", "dvssq_gelu_mul", "dvssq_encode_workspace_size", "dvssq_encode",
    "dvssq_forward_workspace_size", "dvssq_linear_forward", "dvssq_linear_forward_static",
    "dvssq_materialize", "dvssq_lowrank_workspace_size", "dvssq_lowrank", "AttnShape",
    "dvssq_bss_attention_workspace_size", "dvssq_bss_attention", "dvssq_device_error", "STATIC_SCRATCH_BYTES", "MlpStack",
    "dvssq_mlp_stack_workspace_size", "dvssq_mlp_stack_plan_query", "dvssq_mlp_stack_prepare",
    "dvssq_mlp_stack_forward", "dvssq_profile_enable", "dvssq_profile_collect", "dvssq_profile_read",
    "dvssq_profile_reset", "dvssq_set_wait_limit", "dvssq_selftest_wait",
    "Y_F32", "Y_BF16", "PATH_AUTO", "PATH_DECODE", "PATH_PREFILL",
    "EXPORTED_SYMBOLS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.environ.get("DVSSQ_LIBRARY", os.path.join(_HERE, "libdvssq.so"))

if not os.path.exists(library_path):
    raise ImportError(
        f"libdvssq.so not found at {library_path}; build it with "
        "`python -m mixed_precision_weight_b200.build` (nvcc, sm_100a)")

lib = ctypes.CDLL(library_path)

Y_F32, Y_BF16 = 0, 1
PATH_AUTO, PATH_DECODE, PATH_PREFILL = 0, 1, 2

EXPORTED_SYMBOLS = (
    "dvssq_abi_version", "dvssq_status_string", "dvssq_last_error", "dvssq_fwht",
    "dvssq_gelu_mul",
    "dvssq_encode_workspace_size", "dvssq_encode", "dvssq_forward_workspace_size",
    "dvssq_linear_forward", "dvssq_linear_forward_static", "dvssq_materialize",
    "dvssq_lowrank_workspace_size", "dvssq_lowrank", "dvssq_bss_attention_workspace_size",
    "dvssq_bss_attention", "dvssq_device_error", "dvssq_mlp_stack_workspace_size",
    "dvssq_mlp_stack_plan_query", "dvssq_mlp_stack_prepare", "dvssq_mlp_stack_forward",
    "dvssq_profile_enable",
    "dvssq_profile_collect", "dvssq_profile_count", "dvssq_profile_get",
    "dvssq_profile_reset", "dvssq_set_wait_limit", "dvssq_selftest_wait",
)


class Shape(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int32), ("K", ctypes.c_int32), ("block", ctypes.c_int32),
                ("group", ctypes.c_int32), ("n_sal", ctypes.c_int32), ("rank", ctypes.c_int32)]

    @classmethod
    def make(cls, M, K, block, rank, n_sal=None, group=64):
        return cls(M, K, block, group, K // 8 if n_sal is None else n_sal, rank)

    def __repr__(self):
        return (f"Shape(M={self.M}, K={self.K}, block={self.block}, group={self.group}, "
                f"n_sal={self.n_sal}, rank={self.rank})")


class _Weights(ctypes.Structure):
    _fields_ = [("q4", ctypes.c_void_p), ("s4", ctypes.c_void_p), ("sal_idx", ctypes.c_void_p),
                ("q8", ctypes.c_void_p), ("s8", ctypes.c_void_p), ("U", ctypes.c_void_p),
                ("V", ctypes.c_void_p)]


class _MlpLayer(ctypes.Structure):
    _fields_ = [("shape", Shape * 3), ("w", _Weights * 3)]


class _StackPlan(ctypes.Structure):
    _fields_ = [("ctas", ctypes.c_int32), ("threads", ctypes.c_int32),
                ("ring_slots", ctypes.c_int32), ("slot_bytes", ctypes.c_int32),
                ("rows_per_tile_gate_up", ctypes.c_int32), ("rows_per_tile_down", ctypes.c_int32),
                ("smem_bytes", ctypes.c_int32)]


class AttnShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("q_heads", ctypes.c_int32),
                ("kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("ctx", ctypes.c_int32), ("tau", ctypes.c_float), ("haze", ctypes.c_float)]


class _EncodeInfo(ctypes.Structure):
    _fields_ = [("inexact_rotation_blocks", ctypes.c_int64),
                ("fp16_unsafe_scales", ctypes.c_int64),
                ("nonfinite_scores", ctypes.c_int64)]


_P = ctypes.c_void_p
_sig = {
    "dvssq_abi_version": (ctypes.c_int32, []),
    "dvssq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "dvssq_last_error": (ctypes.c_char_p, []),
    "dvssq_fwht": (ctypes.c_int, [_P, _P, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, _P]),
    "dvssq_gelu_mul": (ctypes.c_int, [_P, _P, _P, ctypes.c_int64, _P]),
    "dvssq_encode_workspace_size": (ctypes.c_int, [ctypes.POINTER(Shape), ctypes.POINTER(ctypes.c_size_t)]),
    "dvssq_encode": (ctypes.c_int, [ctypes.POINTER(Shape), _P, _P, ctypes.POINTER(_Weights), _P,
                                    ctypes.POINTER(_EncodeInfo), _P, ctypes.c_size_t, _P]),
    "dvssq_forward_workspace_size": (ctypes.c_int, [ctypes.POINTER(Shape), ctypes.c_int64,
                                                    ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]),
    "dvssq_linear_forward": (ctypes.c_int, [ctypes.POINTER(Shape), ctypes.POINTER(_Weights), _P,
                                            ctypes.c_int64, _P, _P, ctypes.c_int32, ctypes.c_int32,
                                            _P, ctypes.c_size_t, _P]),
    "dvssq_linear_forward_static": (ctypes.c_int, [ctypes.POINTER(Shape), ctypes.POINTER(_Weights),
                                                   _P, ctypes.c_int64, _P, _P, ctypes.c_int32, _P]),
    "dvssq_materialize": (ctypes.c_int, [ctypes.POINTER(Shape), ctypes.POINTER(_Weights), _P, _P]),
    "dvssq_bss_attention_workspace_size": (ctypes.c_int, [ctypes.POINTER(AttnShape),
                                                          ctypes.POINTER(ctypes.c_size_t)]),
    "dvssq_bss_attention": (ctypes.c_int, [ctypes.POINTER(AttnShape), _P, _P, _P, _P, _P,
                                           ctypes.c_size_t, _P]),
    "dvssq_lowrank_workspace_size": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                    ctypes.POINTER(ctypes.c_size_t)]),
    "dvssq_lowrank": (ctypes.c_int, [_P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_int32, ctypes.c_uint64, _P, _P, _P, _P,
                                     ctypes.c_size_t, _P]),
    "dvssq_device_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int32]),
    "dvssq_mlp_stack_workspace_size": (ctypes.c_int, [ctypes.POINTER(_MlpLayer), ctypes.c_int32,
                                                      ctypes.POINTER(ctypes.c_size_t)]),
    "dvssq_mlp_stack_plan_query": (ctypes.c_int, [ctypes.POINTER(_MlpLayer), ctypes.c_int32,
                                                  ctypes.c_int32, ctypes.POINTER(_StackPlan)]),
    "dvssq_mlp_stack_prepare": (ctypes.c_int, [ctypes.POINTER(_MlpLayer), ctypes.c_int32, _P,
                                               ctypes.c_size_t, _P]),
    "dvssq_mlp_stack_forward": (ctypes.c_int, [ctypes.POINTER(_MlpLayer), ctypes.c_int32, _P, _P,
                                               _P, ctypes.c_size_t, _P]),
    "dvssq_profile_enable": (ctypes.c_int, [ctypes.c_int32]),
    "dvssq_profile_collect": (ctypes.c_int, []),
    "dvssq_profile_count": (ctypes.c_int32, []),
    "dvssq_profile_get": (ctypes.c_int, [ctypes.c_int32, ctypes.POINTER(ctypes.c_char_p),
                                         ctypes.POINTER(ctypes.c_int64),
                                         ctypes.POINTER(ctypes.c_double)]),
    "dvssq_profile_reset": (ctypes.c_int, []),
    "dvssq_set_wait_limit": (ctypes.c_int, [ctypes.c_int64]),
    "dvssq_selftest_wait": (ctypes.c_int, [ctypes.c_int32, _P]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class DvssqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.dvssq_status_string(status).decode()
        detail = lib.dvssq_last_error().decode()
        super().__init__(f"{where}: {msg}" + (f" ({detail})" if detail and status in (4, 5) else ""))


def _check(status: int, where: str):
    if status != 0:
        raise DvssqError(status, where)


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("tensors passed to libdvssq must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _bits(t):
    """BF16 tensors travel as their 16-bit patterns; the pointer is the same."""
    return t


@dataclasses.dataclass
class PackedWeights:
    """Device tensors of one encoded layer (layouts of dvssq_weights)."""
    q4: torch.Tensor
    s4: torch.Tensor
    sal_idx: torch.Tensor
    q8: torch.Tensor
    s8: torch.Tensor
    U: torch.Tensor | None = None
    V: torch.Tensor | None = None

    @classmethod
    def empty(cls, shape: Shape, device="cuda", U=None, V=None):
        M, K, n = shape.M, shape.K, shape.n_sal
        return cls(q4=torch.empty((M, K // 2), dtype=torch.uint8, device=device),
                   s4=torch.empty((M, K // 64), dtype=torch.bfloat16, device=device),
                   sal_idx=torch.empty((max(n, 1),), dtype=torch.int32, device=device),
                   q8=torch.empty((M, max(n, 1)), dtype=torch.int8, device=device),
                   s8=torch.empty((M,), dtype=torch.bfloat16, device=device), U=U, V=V)

    def _c(self, shape: Shape) -> _Weights:
        has_sal = shape.n_sal > 0
        return _Weights(self.q4.data_ptr(), self.s4.data_ptr(),
                        self.sal_idx.data_ptr() if has_sal else None,
                        self.q8.data_ptr() if has_sal else None, self.s8.data_ptr(),
                        self.U.data_ptr() if self.U is not None and shape.rank > 0 else None,
                        self.V.data_ptr() if self.V is not None and shape.rank > 0 else None)


def dvssq_gelu_mul(gate: torch.Tensor, up: torch.Tensor, h: torch.Tensor | None = None,
                   stream=None):
    """h = RN_bf16(gelu(gate) * up) elementwise, BF16 in and out."""
    if gate.dtype != torch.bfloat16 or up.dtype != torch.bfloat16 or gate.shape != up.shape:
        raise TypeError("gate and up must be bfloat16 tensors of one shape")
    if h is None:
        h = torch.empty_like(gate)
    _check(lib.dvssq_gelu_mul(_ptr(gate), _ptr(up), _ptr(h), gate.numel(), _stream(stream)),
           "dvssq_gelu_mul")
    return h


def dvssq_fwht(x: torch.Tensor, block: int, y: torch.Tensor | None = None, stream=None):
    """y = H_K x (fp32) for BF16 x [rows][cols]."""
    if x.dtype != torch.bfloat16:
        raise TypeError("x must be bfloat16")
    rows, cols = (x.shape[0], x.shape[1]) if x.dim() == 2 else (1, x.shape[-1])
    if y is None:
        y = torch.empty(x.shape, dtype=torch.float32, device=x.device)
    _check(lib.dvssq_fwht(_ptr(x), _ptr(y), rows, cols, block, _stream(stream)), "dvssq_fwht")
    return y


def dvssq_encode_workspace_size(shape: Shape) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.dvssq_encode_workspace_size(ctypes.byref(shape), ctypes.byref(n)),
           "dvssq_encode_workspace_size")
    return n.value


def dvssq_encode(shape: Shape, W: torch.Tensor, act_scale: torch.Tensor, out: PackedWeights,
                 resid: torch.Tensor | None = None, want_info: bool = False,
                 workspace: torch.Tensor | None = None, stream=None):
    """Encode BF16 W [M][K] into ``out``; returns the info dict when asked."""
    if workspace is None:
        workspace = torch.empty(dvssq_encode_workspace_size(shape), dtype=torch.uint8,
                                device=W.device)
    info = _EncodeInfo()
    w = out._c(shape)
    _check(lib.dvssq_encode(ctypes.byref(shape), _ptr(W), _ptr(act_scale), ctypes.byref(w),
                            _ptr(resid), ctypes.byref(info) if want_info else None,
                            _ptr(workspace), workspace.numel(), _stream(stream)), "dvssq_encode")
    if want_info:
        return dict(inexact_rotation_blocks=info.inexact_rotation_blocks,
                    fp16_unsafe_scales=info.fp16_unsafe_scales,
                    nonfinite_scores=info.nonfinite_scores)
    return None


def dvssq_forward_workspace_size(shape: Shape, T: int, path: int = PATH_AUTO) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.dvssq_forward_workspace_size(ctypes.byref(shape), T, path, ctypes.byref(n)),
           "dvssq_forward_workspace_size")
    return n.value


def dvssq_linear_forward(shape: Shape, w: PackedWeights, x: torch.Tensor,
                         bias: torch.Tensor | None = None, y: torch.Tensor | None = None,
                         y_dtype: int = Y_F32, path: int = PATH_AUTO,
                         workspace: torch.Tensor | None = None, stream=None):
    """y [T][M] = DV-SSQ forward of BF16 x [T][K] on the packed layer."""
    T = x.shape[0]
    if y is None:
        y = torch.empty((T, shape.M), dtype=torch.float32 if y_dtype == Y_F32 else torch.bfloat16,
                        device=x.device)
    if workspace is None:
        workspace = torch.empty(max(1, dvssq_forward_workspace_size(shape, T, path)),
                                dtype=torch.uint8, device=x.device)
    wc = w._c(shape)
    _check(lib.dvssq_linear_forward(ctypes.byref(shape), ctypes.byref(wc), _ptr(x), T, _ptr(bias),
                                    _ptr(y), y_dtype, path, _ptr(workspace), workspace.numel(),
                                    _stream(stream)), "dvssq_linear_forward")
    return y


def dvssq_linear_forward_static(shape: Shape, w: PackedWeights, x: torch.Tensor,
                                bias: torch.Tensor | None = None, y: torch.Tensor | None = None,
                                y_dtype: int = Y_F32, stream=None):
    """The decode forward (T <= 16) using the library's fixed internal scratch.

    For callers that cannot allocate a workspace; see dvssq.h for the size
    limit and the rule that overlapping calls must be serialised.
    """
    T = x.shape[0]
    if y is None:
        y = torch.empty((T, shape.M), dtype=torch.float32 if y_dtype == Y_F32 else torch.bfloat16,
                        device=x.device)
    wc = w._c(shape)
    _check(lib.dvssq_linear_forward_static(ctypes.byref(shape), ctypes.byref(wc), _ptr(x), T,
                                           _ptr(bias), _ptr(y), y_dtype, _stream(stream)),
           "dvssq_linear_forward_static")
    return y


STATIC_SCRATCH_BYTES = 8 * 1024 * 1024


def dvssq_bss_attention_workspace_size(shape: AttnShape) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.dvssq_bss_attention_workspace_size(ctypes.byref(shape), ctypes.byref(n)),
           "dvssq_bss_attention_workspace_size")
    return n.value


def dvssq_bss_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, tau: float = 1.10,
                        haze: float = 12.0, out: torch.Tensor | None = None,
                        workspace: torch.Tensor | None = None, stream=None):
    """KV-BSS decode attention: q [B][Hq][d], k/v [B][Hkv][L][d] (BF16) -> FP32 [B][Hq][d]."""
    B, Hq, d = q.shape
    Hkv, L = k.shape[1], k.shape[2]
    shape = AttnShape(B, Hq, Hkv, d, L, tau, haze)
    if out is None:
        out = torch.empty((B, Hq, d), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(dvssq_bss_attention_workspace_size(shape), dtype=torch.uint8,
                                device=q.device)
    _check(lib.dvssq_bss_attention(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                   _ptr(workspace), workspace.numel(), _stream(stream)),
           "dvssq_bss_attention")
    return out


def dvssq_lowrank_workspace_size(M: int, K: int, rank: int) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.dvssq_lowrank_workspace_size(M, K, rank, ctypes.byref(n)),
           "dvssq_lowrank_workspace_size")
    return n.value


def dvssq_lowrank(R: torch.Tensor, rank: int, iters: int = 4, seed: int = 0,
                  U: torch.Tensor | None = None, V: torch.Tensor | None = None,
                  sigma: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                  stream=None):
    """BF16 rank-r factors (U [M][r], V [r][K]) of the FP32 residual R [M][K]."""
    if R.dtype != torch.float32 or R.dim() != 2:
        raise TypeError("R must be a float32 matrix")
    M, K = R.shape
    if U is None:
        U = torch.empty((M, rank), dtype=torch.bfloat16, device=R.device)
    if V is None:
        V = torch.empty((rank, K), dtype=torch.bfloat16, device=R.device)
    if workspace is None:
        workspace = torch.empty(dvssq_lowrank_workspace_size(M, K, rank), dtype=torch.uint8,
                                device=R.device)
    _check(lib.dvssq_lowrank(_ptr(R), M, K, rank, iters, seed & (2 ** 64 - 1), _ptr(U), _ptr(V),
                             _ptr(sigma), _ptr(workspace), workspace.numel(), _stream(stream)),
           "dvssq_lowrank")
    return U, V


def dvssq_materialize(shape: Shape, w: PackedWeights, out: torch.Tensor | None = None,
                      stream=None):
    """Dense BF16 W_eff [M][K] in the original domain (materialize_weights)."""
    if out is None:
        out = torch.empty((shape.M, shape.K), dtype=torch.bfloat16, device=w.q4.device)
    wc = w._c(shape)
    _check(lib.dvssq_materialize(ctypes.byref(shape), ctypes.byref(wc), _ptr(out),
                                 _stream(stream)), "dvssq_materialize")
    return out


def _mlp_layers(layers) -> ctypes.Array:
    """[(gate, up, down)] of (Shape, PackedWeights) -> the C array of dvssq_mlp_layer."""
    arr = (_MlpLayer * len(layers))()
    for l, mats in enumerate(layers):
        if len(mats) != 3:
            raise ValueError("each layer is (gate, up, down)")
        for mi, (shape, packed) in enumerate(mats):
            arr[l].shape[mi] = shape
            arr[l].w[mi] = packed._c(shape)
    return arr


def dvssq_mlp_stack_workspace_size(layers) -> int:
    arr = _mlp_layers(layers)
    n = ctypes.c_size_t(0)
    _check(lib.dvssq_mlp_stack_workspace_size(arr, len(layers), ctypes.byref(n)),
           "dvssq_mlp_stack_workspace_size")
    return n.value


def dvssq_mlp_stack_plan_query(layers, sm_count: int) -> dict:
    """The forward's launch plan for these layers on a device of sm_count SMs
    (host only): CTAs, threads per CTA, weight-ring slots and their bytes, weight
    rows per slot for gate/up and for down, dynamic shared memory per CTA."""
    arr = _mlp_layers(layers)
    plan = _StackPlan()
    _check(lib.dvssq_mlp_stack_plan_query(arr, len(layers), int(sm_count), ctypes.byref(plan)),
           "dvssq_mlp_stack_plan_query")
    return {name: getattr(plan, name) for name, _ in _StackPlan._fields_}


def dvssq_mlp_stack_prepare(layers, workspace: torch.Tensor, stream=None):
    arr = _mlp_layers(layers)
    _check(lib.dvssq_mlp_stack_prepare(arr, len(layers), _ptr(workspace), workspace.numel(),
                                       _stream(stream)), "dvssq_mlp_stack_prepare")


def dvssq_mlp_stack_forward(layers, x: torch.Tensor, workspace: torch.Tensor,
                            y: torch.Tensor | None = None, stream=None, _arr=None):
    """y = one BF16 token [hidden] through the prepared stack."""
    arr = _mlp_layers(layers) if _arr is None else _arr
    if y is None:
        y = torch.empty_like(x)
    _check(lib.dvssq_mlp_stack_forward(arr, len(layers), _ptr(x), _ptr(y), _ptr(workspace),
                                       workspace.numel(), _stream(stream)),
           "dvssq_mlp_stack_forward")
    return y


class MlpStack:
    """A stack of gated-GELU MLP blocks with its prepared workspace."""

    def __init__(self, layers, device="cuda", stream=None):
        self.layers = [tuple(m) for m in layers]
        self._arr = _mlp_layers(self.layers)
        self.workspace = torch.empty(dvssq_mlp_stack_workspace_size(self.layers),
                                     dtype=torch.uint8, device=device)
        dvssq_mlp_stack_prepare(self.layers, self.workspace, stream=stream)

    def forward(self, x: torch.Tensor, y: torch.Tensor | None = None, stream=None):
        return dvssq_mlp_stack_forward(self.layers, x, self.workspace, y=y, stream=stream,
                                       _arr=self._arr)


def dvssq_device_error(clear: bool = True) -> int:
    word = ctypes.c_uint32(0)
    _check(lib.dvssq_device_error(ctypes.byref(word), 1 if clear else 0), "dvssq_device_error")
    return word.value


def dvssq_set_wait_limit(cycles: int = 0):
    """Wait limit of the kernels' bounded waits (cycles; <= 0: the default)."""
    _check(lib.dvssq_set_wait_limit(int(cycles)), "dvssq_set_wait_limit")


def dvssq_selftest_wait(which: int, stream=None):
    """One warp waits on something never signalled (0: mbarrier, 1: grid counter)."""
    _check(lib.dvssq_selftest_wait(int(which), _stream(stream)), "dvssq_selftest_wait")


def dvssq_profile_enable(on: bool = True):
    _check(lib.dvssq_profile_enable(1 if on else 0), "dvssq_profile_enable")


def dvssq_profile_collect():
    _check(lib.dvssq_profile_collect(), "dvssq_profile_collect")


def dvssq_profile_reset():
    _check(lib.dvssq_profile_reset(), "dvssq_profile_reset")


def dvssq_profile_read() -> dict:
    """{kernel name: (launches, total_ms)} accumulated since the last reset."""
    out = {}
    for i in range(lib.dvssq_profile_count()):
        name, n, ms = ctypes.c_char_p(), ctypes.c_int64(), ctypes.c_double()
        _check(lib.dvssq_profile_get(i, ctypes.byref(name), ctypes.byref(n), ctypes.byref(ms)),
               "dvssq_profile_get")
        out[name.value.decode()] = (n.value, ms.value)
    return out


class DvssqLinear:
    """One DV-SSQ linear layer on the GPU: encode once, run the forward.

    Public end-to-end API: tensors may live on the host (copied to the device
    inside the call) or on the device.
    """

    def __init__(self, shape: Shape, packed: PackedWeights, bias: torch.Tensor | None = None):
        self.shape, self.packed, self.bias = shape, packed, bias
        self._ws = {}

    @classmethod
    def from_weight(cls, W, act_scale, U, V, block, bias=None, n_sal=None, device="cuda",
                    stream=None):
        W = W.to(device, non_blocking=True)
        act_scale = act_scale.to(device, non_blocking=True)
        M, K = W.shape
        r = 0 if U is None else U.shape[1]
        shape = Shape.make(M, K, block, r, n_sal)
        packed = PackedWeights.empty(shape, device,
                                     U=None if U is None else U.to(device, non_blocking=True).contiguous(),
                                     V=None if V is None else V.to(device, non_blocking=True).contiguous())
        dvssq_encode(shape, W, act_scale, packed, stream=stream)
        if bias is not None:
            bias = bias.to(device, non_blocking=True)
        return cls(shape, packed, bias)

    def workspace(self, T: int, path: int = PATH_AUTO, device="cuda"):
        key = (T, path)
        if key not in self._ws:
            n = max(1, dvssq_forward_workspace_size(self.shape, T, path))
            self._ws[key] = torch.empty(n, dtype=torch.uint8, device=device)
        return self._ws[key]

    def __call__(self, x, y_dtype: int = Y_F32, path: int = PATH_AUTO, stream=None, out=None):
        dev = self.packed.q4.device
        x = x.to(dev, non_blocking=True)
        return dvssq_linear_forward(self.shape, self.packed, x, self.bias, y=out, y_dtype=y_dtype,
                                    path=path, workspace=self.workspace(x.shape[0], path, dev),
                                    stream=stream)
