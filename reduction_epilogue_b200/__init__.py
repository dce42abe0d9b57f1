"""Python binding for libfle: fused fp32 Linear + epilogue on B200 (sm_100a).

Argument marshalling only.  Every step of the computation runs in the CUDA
library behind ``include/fle.h``; PyTorch supplies device memory and streams.
There is no fallback: if the library is missing, or the device is not a
B200, the calls raise.

    import reduction_epilogue_b200 as fle
    out = fle.linear_epilogue(x, W, b, "scale_hardtanh_gelu", precision="tf32")
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "EPI_SCALE_HARDTANH_GELU", "EPI_SWISH_SCALE", "EPI_AVGPOOL_GELU_SCALE_ROWMAX", "EPI_NONE",
    "PREC_3XTF32", "PREC_TF32", "EpilogueDesc", "FleError", "desc_for", "forward",
    "workspace_size", "workspace_size_min", "device_status", "plan_string", "plan_units", "pool_weights",
    "workspace_size_pooled", "forward_pooled", "linear_epilogue", "library_path", "load",
    "PROBLEMS",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
# FLE_BUILD=check selects the barrier-checking build of the same sources
# (-DFLE_CHECK_BARRIERS: protocol checks record FLE_ERR_PROTOCOL); tests only.
_CHECK = os.environ.get("FLE_BUILD", "") == "check"
_LIB = os.path.join(_PKG, "lib", "libfle_check.so" if _CHECK else "libfle.so")

# Values mirror include/fle.h.
EPI_SCALE_HARDTANH_GELU = 0
EPI_SWISH_SCALE = 1
EPI_AVGPOOL_GELU_SCALE_ROWMAX = 2
EPI_NONE = 3
PREC_3XTF32 = 0
PREC_TF32 = 1
FLAG_GELU_TANH = 1
FLAG_FOLD_SCALE = 2

FLE_OK = 0
STATUS_NAMES = {
    0: "FLE_OK", 1: "FLE_ERR_NULL", 2: "FLE_ERR_SHAPE", 3: "FLE_ERR_ALIGN", 4: "FLE_ERR_DESC",
    5: "FLE_ERR_WORKSPACE", 6: "FLE_ERR_ARCH", 7: "FLE_ERR_CUDA", 8: "FLE_ERR_TIMEOUT",
    9: "FLE_ERR_UNSUPPORTED", 10: "FLE_ERR_PROTOCOL",
}

# The pages' three problems: epilogue kind and constants.
PROBLEMS = {
    "scale_hardtanh_gelu": dict(kind=EPI_SCALE_HARDTANH_GELU, scale=0.5, clamp_lo=-2.0, clamp_hi=2.0),
    "swish_scale": dict(kind=EPI_SWISH_SCALE, scale=2.0),
    "avgpool_gelu_scale_rowmax": dict(kind=EPI_AVGPOOL_GELU_SCALE_ROWMAX, scale=2.0, pool_k=16),
    "none": dict(kind=EPI_NONE),
}


class EpilogueDesc(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int32),
        ("precision", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("clamp_lo", ctypes.c_float),
        ("clamp_hi", ctypes.c_float),
        ("pool_k", ctypes.c_int32),
        ("pool_stride", ctypes.c_int32),
        ("flags", ctypes.c_int32),
    ]


class FleError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        name = STATUS_NAMES.get(status, str(status))
        super().__init__(f"{what}: {name} ({_status_text(status)})" if what else f"{name} ({_status_text(status)})")


_lib = None


def library_path() -> str:
    return _LIB


def load():
    """Loads libfle.so (built in-tree by reduction_epilogue_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB):
        raise FileNotFoundError(
            f"{_LIB} is missing; build it with `python -m reduction_epilogue_b200.build`")
    from . import build as _build
    if _build.sources_present() and _build.built_hash(_LIB) != _build.source_hash(_CHECK):
        raise RuntimeError(
            f"{_LIB} was not built from the sources beside it; rebuild it with "
            "`python -m reduction_epilogue_b200.build`")
    lib = ctypes.CDLL(_LIB)
    i64, vp, sz = ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t
    lib.fle_forward.argtypes = [vp, vp, vp, i64, i64, i64, ctypes.POINTER(EpilogueDesc), vp, vp, sz, vp]
    lib.fle_forward.restype = ctypes.c_int
    lib.fle_workspace_size.argtypes = [i64, i64, i64, ctypes.POINTER(EpilogueDesc)]
    lib.fle_workspace_size.restype = sz
    lib.fle_workspace_size_min.argtypes = [i64, i64, i64, ctypes.POINTER(EpilogueDesc)]
    lib.fle_workspace_size_min.restype = sz
    lib.fle_status_string.argtypes = [ctypes.c_int]
    lib.fle_status_string.restype = ctypes.c_char_p
    lib.fle_device_status.argtypes = [vp]
    lib.fle_device_status.restype = ctypes.c_int
    lib.fle_plan_string.argtypes = [i64, i64, i64, ctypes.POINTER(EpilogueDesc), ctypes.c_char_p, sz]
    lib.fle_plan_string.restype = ctypes.c_int
    lib.fle_version.argtypes = []
    lib.fle_version.restype = ctypes.c_int
    lib.fle_plan_units.argtypes = [i64, i64, i64, ctypes.POINTER(EpilogueDesc), ctypes.c_int, ctypes.c_int,
                                   vp, ctypes.c_int, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]
    lib.fle_plan_units.restype = ctypes.c_int
    lib.fle_pool_weights.argtypes = [vp, vp, i64, i64, ctypes.c_int32, vp, vp, vp]
    lib.fle_pool_weights.restype = ctypes.c_int
    lib.fle_workspace_size_pooled.argtypes = [i64, i64, i64, ctypes.POINTER(EpilogueDesc)]
    lib.fle_workspace_size_pooled.restype = sz
    lib.fle_forward_pooled.argtypes = [vp, vp, vp, i64, i64, i64, ctypes.POINTER(EpilogueDesc), vp, vp, sz, vp]
    lib.fle_forward_pooled.restype = ctypes.c_int
    lib.fle_source_hash.argtypes = []
    lib.fle_source_hash.restype = ctypes.c_char_p
    lib.fle_test_bounded_wait.argtypes = [ctypes.c_uint32, vp]
    lib.fle_test_bounded_wait.restype = ctypes.c_int
    lib.fle_test_set_finisher.argtypes = [ctypes.c_int32]
    lib.fle_test_set_finisher.restype = ctypes.c_int
    lib.fle_test_finisher_counts.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int32, vp]
    lib.fle_test_finisher_counts.restype = ctypes.c_int
    _lib = lib
    return lib


def _status_text(status: int) -> str:
    try:
        return load().fle_status_string(int(status)).decode()
    except Exception:
        return "?"


def desc_for(problem: str | None = None, precision: str | int = "tf32", gelu: str = "erf",
             fold_scale: bool = False, **overrides) -> EpilogueDesc:
    """Builds an EpilogueDesc from a page problem name and/or explicit fields.
    gelu="tanh" selects FLE_FLAG_GELU_TANH; fold_scale selects
    FLE_FLAG_FOLD_SCALE."""
    f = dict(kind=EPI_NONE, scale=1.0, clamp_lo=-2.0, clamp_hi=2.0, pool_k=16)
    if problem is not None:
        f.update(PROBLEMS[problem])
    f.update(overrides)
    if isinstance(precision, str):
        precision = {"tf32": PREC_TF32, "3xtf32": PREC_3XTF32}[precision.lower()]
    if gelu not in ("erf", "tanh"):
        raise ValueError("gelu must be 'erf' or 'tanh'")
    flags = int(f.get("flags", 0)) | (FLAG_GELU_TANH if gelu == "tanh" else 0) | (FLAG_FOLD_SCALE if fold_scale else 0)
    pk = int(f["pool_k"])
    return EpilogueDesc(int(f["kind"]), int(precision), float(f["scale"]), float(f["clamp_lo"]),
                        float(f["clamp_hi"]), pk, int(f.get("pool_stride", pk)), flags)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream_handle(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check_tensor(name, t, shape):
    import torch
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous float32 CUDA tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def workspace_size(M: int, K: int, N: int, desc: EpilogueDesc) -> int:
    return int(load().fle_workspace_size(M, K, N, ctypes.byref(desc)))


def workspace_size_min(M: int, K: int, N: int, desc: EpilogueDesc) -> int:
    return int(load().fle_workspace_size_min(M, K, N, ctypes.byref(desc)))


def plan_string(M: int, K: int, N: int, desc: EpilogueDesc) -> str:
    buf = ctypes.create_string_buffer(512)
    st = load().fle_plan_string(M, K, N, ctypes.byref(desc), buf, 512)
    if st != FLE_OK:
        raise FleError(st, "fle_plan_string")
    return buf.value.decode()


def plan_units(M: int, K: int, N: int, desc: EpilogueDesc, num_sms: int, cta: int):
    """(grid, [unit rows]) that CTA `cta` would run; see fle_plan_units."""
    import numpy as np
    lib = load()
    n = ctypes.c_int(0)
    g = ctypes.c_int(0)
    st = lib.fle_plan_units(M, K, N, ctypes.byref(desc), num_sms, cta, None, 0, ctypes.byref(n), ctypes.byref(g))
    if st != FLE_OK:
        raise FleError(st, "fle_plan_units")
    rows = np.zeros((max(n.value, 1), 12), dtype=np.int32)
    st = lib.fle_plan_units(M, K, N, ctypes.byref(desc), num_sms, cta, rows.ctypes.data, n.value,
                            ctypes.byref(n), ctypes.byref(g))
    if st != FLE_OK:
        raise FleError(st, "fle_plan_units")
    return g.value, rows[: n.value]


def device_status(stream=None) -> int:
    return int(load().fle_device_status(_stream_handle(stream)))


def forward(x, W, b, out, desc: EpilogueDesc, workspace=None, workspace_bytes: int | None = None,
            stream=None, M: int | None = None, K: int | None = None, N: int | None = None) -> None:
    """Calls fle_forward.  x, W, b, out, workspace are torch CUDA tensors (or
    raw device addresses as ints, then M, K, N must be given)."""
    lib = load()
    if M is None:
        M, K = x.shape
        N = W.shape[0]
        _check_tensor("x", x, (M, K))
        _check_tensor("W", W, (N, K))
        _check_tensor("b", b, (N,))
        _check_tensor("out", out, (M,) if desc.kind == EPI_AVGPOOL_GELU_SCALE_ROWMAX else (M, N))
    if workspace_bytes is None:
        if workspace is None:
            workspace_bytes = 0
        elif isinstance(workspace, int):
            raise ValueError("give workspace_bytes with a raw workspace address")
        else:
            workspace_bytes = workspace.numel() * workspace.element_size()
    st = lib.fle_forward(_ptr(x), _ptr(W), _ptr(b), int(M), int(K), int(N), ctypes.byref(desc), _ptr(out),
                         _ptr(workspace), int(workspace_bytes), _stream_handle(stream))
    if st != FLE_OK:
        raise FleError(st, "fle_forward")


def pool_weights(W, b, pool_k: int = 16, W_pooled=None, b_pooled=None, stream=None):
    """fle_pool_weights: (W_pooled [N/k, K], b_pooled [N/k] or None)."""
    import torch
    N, K = W.shape
    P = N // pool_k
    if W_pooled is None:
        W_pooled = torch.empty(P, K, dtype=torch.float32, device=W.device)
    if b is not None and b_pooled is None:
        b_pooled = torch.empty(P, dtype=torch.float32, device=W.device)
    st = load().fle_pool_weights(_ptr(W), _ptr(b), N, K, int(pool_k), _ptr(W_pooled),
                                 _ptr(b_pooled) if b is not None else None, _stream_handle(stream))
    if st != FLE_OK:
        raise FleError(st, "fle_pool_weights")
    return W_pooled, (b_pooled if b is not None else None)


def workspace_size_pooled(M: int, K: int, N: int, desc: EpilogueDesc) -> int:
    return int(load().fle_workspace_size_pooled(M, K, N, ctypes.byref(desc)))


def forward_pooled(x, W, b, out, desc: EpilogueDesc, workspace=None, workspace_bytes: int | None = None,
                   stream=None) -> None:
    """fle_forward_pooled: epilogue (c) through pooled weights in one call."""
    M, K = x.shape
    N = W.shape[0]
    _check_tensor("x", x, (M, K))
    _check_tensor("W", W, (N, K))
    _check_tensor("b", b, (N,))
    _check_tensor("out", out, (M,))
    if workspace_bytes is None:
        workspace_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = load().fle_forward_pooled(_ptr(x), _ptr(W), _ptr(b), M, K, N, ctypes.byref(desc), _ptr(out),
                                   _ptr(workspace), int(workspace_bytes), _stream_handle(stream))
    if st != FLE_OK:
        raise FleError(st, "fle_forward_pooled")


def linear_epilogue(x, W, b, problem: str = "scale_hardtanh_gelu", precision: str = "tf32",
                    out=None, stream=None, **overrides):
    """Allocates the output (and workspace, if the plan needs one) with torch
    and runs one fused call.  Returns out."""
    import torch
    desc = desc_for(problem, precision, **overrides)
    M, K = x.shape
    N = W.shape[0]
    if out is None:
        shape = (M,) if desc.kind == EPI_AVGPOOL_GELU_SCALE_ROWMAX else (M, N)
        out = torch.empty(shape, dtype=torch.float32, device=x.device)
    ws_bytes = workspace_size(M, K, N, desc)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=x.device) if ws_bytes else None
    forward(x, W, b, out, desc, workspace=ws, workspace_bytes=ws_bytes, stream=stream)
    return out


def forward_noalloc(x, W, b, out, desc: EpilogueDesc, stream=None) -> None:
    """Calls fle_forward_noalloc: fle_forward with the library's own static
    scratch instead of a caller workspace, for callers that cannot allocate
    device memory where they run the layer.  Calls that overlap on the GPU
    share that scratch and must be serialised."""
    lib = load()
    fn = lib.fle_forward_noalloc
    vp = ctypes.c_void_p
    fn.argtypes = [vp, vp, vp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                   ctypes.POINTER(EpilogueDesc), vp, vp]
    fn.restype = ctypes.c_int
    M, K = x.shape
    N = W.shape[0]
    _check_tensor("x", x, (M, K))
    _check_tensor("W", W, (N, K))
    _check_tensor("b", b, (N,))
    _check_tensor("out", out, (M,) if desc.kind == EPI_AVGPOOL_GELU_SCALE_ROWMAX else (M, N))
    st = fn(_ptr(x), _ptr(W), _ptr(b), int(M), int(K), int(N), ctypes.byref(desc), _ptr(out),
            _stream_handle(stream))
    if st != FLE_OK:
        raise FleError(st, "fle_forward_noalloc")
