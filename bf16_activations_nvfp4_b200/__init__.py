"""bf16 activations x NVFP4 weights (mm_bf16_fp4) for NVIDIA B200 (sm_100a).

A thin ctypes binding over the C-ABI library ``libfi_nvfp4.so`` (declared in
``include/fi_nvfp4.h``). This module only marshals arguments: every step of the
computation runs in the library's CUDA kernels. torch supplies device memory and the
current CUDA stream. There is no CPU fallback: if the library is missing, every call
raises.

    Wq, Ws, g = pack_weights(W)                # W: fp32 [n, k] on cuda
    out = mm_bf16_fp4(A, Wq, Ws, g)            # A: bf16 [m, k] on cuda -> bf16 [m, n]
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import threading

import torch

__all__ = [
    "FiError", "KIND_GEMV", "KIND_MMA", "TACTIC_DEFAULT", "make_tactic", "tactic_fields",
    "pack_weights", "mm_bf16_fp4", "splitk_reduce", "resolve_tactic", "default_tactic",
    "list_tactics", "workspace_bytes", "set_workspace", "last_error", "version", "library",
    "library_path", "get_device_error", "debug_set", "DEBUG_STALL_PRODUCER", "DEBUG_WAIT_TIMEOUT_NS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libfi_nvfp4.so"

KIND_GEMV = 0
KIND_MMA = 1
TACTIC_DEFAULT = -1
# output element types of fi_mm_bf16_fp4_out / fi_splitk_reduce_out
_DTYPES = {torch.bfloat16: 0, torch.float16: 1}

_STATUS = {0: "FI_OK", -1: "FI_ERR_INVALID_ARG", -2: "FI_ERR_UNSUPPORTED_SHAPE",
           -3: "FI_ERR_UNSUPPORTED_ARCH", -4: "FI_ERR_WORKSPACE", -5: "FI_ERR_CUDA"}


class FiError(RuntimeError):
    """A library call returned a non-zero fi_status."""

    def __init__(self, status: int, where: str, message: str):
        self.status = status
        super().__init__(f"{where}: {_STATUS.get(status, status)}: {message}")


class TacticInfo(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("splits", ctypes.c_int32),
                ("ctas_per_sm", ctypes.c_int32), ("variant", ctypes.c_int32),
                ("grid_x", ctypes.c_int32), ("grid_y", ctypes.c_int32),
                ("threads", ctypes.c_int32), ("smem_bytes", ctypes.c_int32),
                ("workspace_bytes", ctypes.c_int64)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def library() -> ctypes.CDLL:
    """Load libfi_nvfp4.so (built by ``python -m bf16_activations_nvfp4_b200.build``)."""
    global _lib
    lib = _lib
    if lib is not None:  # loaded: no lock on the per-call path
        return lib
    with _lock:
        if _lib is not None:
            return _lib
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(
                f"{path} is missing: build it with `python -m bf16_activations_nvfp4_b200.build` "
                "(there is no fallback implementation)")
        lib = ctypes.CDLL(path)
        vp, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
        lib.fi_nvfp4_pack_weights.argtypes = [vp, i64, i64, vp, vp, vp, vp]
        lib.fi_mm_bf16_fp4.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp]
        lib.fi_mm_bf16_fp4_ex.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp, sz, vp]
        lib.fi_mm_bf16_fp4_noalloc.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i64, vp]
        lib.fi_splitk_reduce.argtypes = [vp, i64, i64, i64, vp, vp, vp]
        lib.fi_mm_bf16_fp4_out.argtypes = [vp, vp, vp, vp, vp, ctypes.c_int, i64, i64, i64, i64, vp, sz, vp]
        lib.fi_splitk_reduce_out.argtypes = [vp, i64, i64, i64, vp, vp, ctypes.c_int, vp]
        lib.fi_resolve_tactic.argtypes = [i64, i64, i64, i64, ctypes.c_int, ctypes.POINTER(TacticInfo)]
        lib.fi_default_tactic.argtypes = [i64, i64, i64, ctypes.c_int]
        lib.fi_default_tactic.restype = i64
        lib.fi_list_tactics.argtypes = [i64, i64, i64, ctypes.c_int, ctypes.POINTER(i64), ctypes.c_int]
        lib.fi_mm_workspace_bytes.argtypes = [i64, i64, i64, i64, ctypes.c_int]
        lib.fi_mm_workspace_bytes.restype = sz
        lib.fi_set_workspace.argtypes = [vp, sz]
        lib.fi_last_error.argtypes = []
        lib.fi_last_error.restype = ctypes.c_char_p
        lib.fi_version.argtypes = []
        lib.fi_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint)]
        lib.fi_debug_set.argtypes = [ctypes.c_int, i64]
        for name in ("fi_nvfp4_pack_weights", "fi_mm_bf16_fp4", "fi_mm_bf16_fp4_ex", "fi_mm_bf16_fp4_noalloc",
                     "fi_splitk_reduce", "fi_mm_bf16_fp4_out", "fi_splitk_reduce_out",
                     "fi_resolve_tactic", "fi_list_tactics", "fi_set_workspace", "fi_version",
                     "fi_get_device_error", "fi_debug_set"):
            getattr(lib, name).restype = ctypes.c_int
        _lib = lib
        return lib


def last_error() -> str:
    return library().fi_last_error().decode()


def version() -> int:
    return library().fi_version()


def _check(status: int, where: str) -> None:
    if status != 0:
        raise FiError(status, where, last_error())


DEBUG_STALL_PRODUCER = 1
DEBUG_WAIT_TIMEOUT_NS = 2


def get_device_error() -> int:
    """Read and clear the current device's sticky kernel error word (0 = no error)."""
    code = ctypes.c_uint(0)
    _check(library().fi_get_device_error(ctypes.byref(code)), "fi_get_device_error")
    return int(code.value)


def debug_set(key: int, value: int) -> None:
    """Test hooks of fi_debug_set (stall the producer of the next launches, wait limit)."""
    _check(library().fi_debug_set(int(key), int(value)), "fi_debug_set")


# ------------------------------------------------------------------------- tactics

def make_tactic(kind: int, splits: int = 0, ctas_per_sm: int = 0, variant: int = 0) -> int:
    """FI_TACTIC(kind, splits, ctas_per_sm, variant) from include/fi_nvfp4.h."""
    return (kind << 24) | (splits << 12) | (ctas_per_sm << 8) | variant


def tactic_fields(t: int) -> dict:
    return {"kind": (t >> 24) & 0xF, "splits": (t >> 12) & 0xFFF, "ctas_per_sm": (t >> 8) & 0xF,
            "variant": t & 0xFF}


def resolve_tactic(m: int, n: int, k: int, tactic: int = TACTIC_DEFAULT, num_sms: int = 0) -> dict:
    info = TacticInfo()
    _check(library().fi_resolve_tactic(m, n, k, tactic, num_sms, ctypes.byref(info)), "fi_resolve_tactic")
    return info.as_dict()


def default_tactic(m: int, n: int, k: int, num_sms: int = 0) -> int:
    t = library().fi_default_tactic(m, n, k, num_sms)
    if t < 0:
        raise FiError(int(t), "fi_default_tactic", last_error())
    return int(t)


def list_tactics(m: int, n: int, k: int, num_sms: int = 0) -> list[int]:
    lib = library()
    count = lib.fi_list_tactics(m, n, k, num_sms, None, 0)
    if count < 0:
        raise FiError(count, "fi_list_tactics", last_error())
    buf = (ctypes.c_int64 * max(count, 1))()
    lib.fi_list_tactics(m, n, k, num_sms, buf, count)
    return [int(buf[i]) for i in range(count)]


def workspace_bytes(m: int, n: int, k: int, tactic: int = TACTIC_DEFAULT, num_sms: int = 0) -> int:
    return int(library().fi_mm_workspace_bytes(m, n, k, tactic, num_sms))


def set_workspace(buf: torch.Tensor | None) -> None:
    """Register a caller-owned split-K workspace (a CUDA tensor) for the current device.
    The caller must keep `buf` alive while calls may use it; None unregisters it."""
    if buf is None:
        _check(library().fi_set_workspace(None, 0), "fi_set_workspace")
    else:
        _check(library().fi_set_workspace(buf.data_ptr(), buf.numel() * buf.element_size()),
               "fi_set_workspace")


# ---------------------------------------------------------------------- the op

def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _require(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {ndim}-d tensor")


def _same_device(ref: torch.Tensor, **tensors) -> None:
    d = ref.get_device()
    for name, t in tensors.items():
        if t is not None and t.get_device() != d:
            raise ValueError(f"{name} is on {t.device}, the operands on {ref.device}")


def _pack_out_check(W: torch.Tensor, out: tuple) -> tuple:
    """The caller's (Wq, Wscale, gscale) buffers for W [n, k], checked against W's shape,
    dtype and device (the kernel writes n*k/2, n*k/16 and 1 elements there)."""
    n, k = W.shape
    if len(out) != 3:
        raise ValueError("out must be (Wq, Wscale, gscale)")
    Wq, Ws, g = out
    for name, t, dtype, shape in (("Wq", Wq, torch.uint8, (n, k // 2)), ("Wscale", Ws, torch.uint8, (n, k // 16)),
                                  ("gscale", g, torch.float32, (1,))):
        if not isinstance(t, torch.Tensor) or t.dtype != dtype or tuple(t.shape) != shape or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {shape}")
    _same_device(W, Wq=Wq, Wscale=Ws, gscale=g)
    return Wq, Ws, g


def _mm_shapes(A: torch.Tensor, Wq: torch.Tensor, Wscale: torch.Tensor, gscale: torch.Tensor,
               out: torch.Tensor | None) -> tuple:
    """(m, n, k) of an mm call, after checking that the operands' shapes agree, that `out` is
    [m, n] and that every operand is on A's device."""
    m, k = A.shape
    n, kq = Wq.shape
    if kq * 2 != k or Wscale.shape != (n, k // 16):
        raise ValueError(f"shape mismatch: A {tuple(A.shape)}, Wq {tuple(Wq.shape)}, Wscale {tuple(Wscale.shape)}")
    if gscale.shape != (1,):
        raise ValueError(f"gscale must hold one element, got shape {tuple(gscale.shape)}")
    if out is not None and out.shape != (m, n):
        raise ValueError(f"out must be [{m}, {n}], got {tuple(out.shape)}")
    d = A.get_device()
    if Wq.get_device() != d or Wscale.get_device() != d or gscale.get_device() != d or (
            out is not None and out.get_device() != d):
        _same_device(A, Wq=Wq, Wscale=Wscale, gscale=gscale, out=out)
    return m, n, k


def pack_weights(W: torch.Tensor, out: tuple | None = None):
    """Quantise fp32 W [n, k] (CUDA) to NVFP4 -> (Wq uint8 [n, k/2], Wscale uint8 [n, k/16],
    gscale fp32 [1]), all on W's device."""
    _require(W, "W", torch.float32, 2)
    n, k = W.shape
    if out is None:
        Wq = torch.empty((n, k // 2), dtype=torch.uint8, device=W.device)
        Ws = torch.empty((n, k // 16), dtype=torch.uint8, device=W.device)
        g = torch.empty(1, dtype=torch.float32, device=W.device)
    else:
        Wq, Ws, g = _pack_out_check(W, out)
    with torch.cuda.device(W.device):
        _check(library().fi_nvfp4_pack_weights(W.data_ptr(), n, k, Wq.data_ptr(), Ws.data_ptr(),
                                               g.data_ptr(), _stream(W.device)), "fi_nvfp4_pack_weights")
    return Wq, Ws, g


def _out_dtype(out: torch.Tensor | None, out_dtype: torch.dtype | None) -> torch.dtype:
    dtype = out.dtype if out is not None else (out_dtype or torch.bfloat16)
    if dtype not in _DTYPES or (out_dtype is not None and out_dtype != dtype):
        raise ValueError(f"the output is bf16 or f16 (out_dtype {out_dtype}, out {None if out is None else out.dtype})")
    return dtype


def mm_bf16_fp4(A: torch.Tensor, Wq: torch.Tensor, Wscale: torch.Tensor, gscale: torch.Tensor,
                tactic: int = TACTIC_DEFAULT, out: torch.Tensor | None = None,
                workspace: torch.Tensor | None = None, out_dtype: torch.dtype | None = None) -> torch.Tensor:
    """out[m, n] = A[m, k] . dequant(W)^T (CUDA tensors on one device), bf16 out unless
    out_dtype (or the dtype of `out`) is torch.float16.

    `workspace` (optional CUDA tensor) is passed to fi_mm_bf16_fp4_ex; without it the call
    uses the per-device workspace of fi_mm_bf16_fp4. An f16 output goes through
    fi_mm_bf16_fp4_out.
    """
    _require(A, "A", torch.bfloat16, 2)
    _require(Wq, "Wq", torch.uint8, 2)
    _require(Wscale, "Wscale", torch.uint8, 2)
    _require(gscale, "gscale", torch.float32, 1)
    dtype = _out_dtype(out, out_dtype)
    if out is not None:
        _require(out, "out", dtype, 2)
    if workspace is not None:
        if not isinstance(workspace, torch.Tensor) or not workspace.is_cuda or not workspace.is_contiguous():
            raise ValueError("workspace must be a contiguous CUDA tensor")
        _same_device(A, workspace=workspace)
    m, n, k = _mm_shapes(A, Wq, Wscale, gscale, out)
    if out is None:
        out = torch.empty((m, n), dtype=dtype, device=A.device)
    lib = library()
    dev = A.device
    # the library works on the current device: switch only when A lives on another one
    ctx = torch.cuda.device(dev) if dev.index != torch.cuda.current_device() else contextlib.nullcontext()
    with ctx:
        s = torch.cuda.current_stream(dev).cuda_stream
        if dtype != torch.bfloat16:
            ws_ptr, ws_bytes = (0, 0) if workspace is None else (workspace.data_ptr(),
                                                                  workspace.numel() * workspace.element_size())
            st = lib.fi_mm_bf16_fp4_out(A.data_ptr(), Wq.data_ptr(), Wscale.data_ptr(), gscale.data_ptr(),
                                        out.data_ptr(), _DTYPES[dtype], m, n, k, tactic, ws_ptr or None, ws_bytes, s)
            if st:
                _check(st, "fi_mm_bf16_fp4_out")
        elif workspace is None:
            st = lib.fi_mm_bf16_fp4(A.data_ptr(), Wq.data_ptr(), Wscale.data_ptr(), gscale.data_ptr(),
                                    out.data_ptr(), m, n, k, tactic, s)
            if st:
                _check(st, "fi_mm_bf16_fp4")
        else:
            st = lib.fi_mm_bf16_fp4_ex(A.data_ptr(), Wq.data_ptr(), Wscale.data_ptr(), gscale.data_ptr(),
                                       out.data_ptr(), m, n, k, tactic, workspace.data_ptr(),
                                       workspace.numel() * workspace.element_size(), s)
            if st:
                _check(st, "fi_mm_bf16_fp4_ex")
    return out


def splitk_reduce(partials: torch.Tensor, gscale: torch.Tensor, out: torch.Tensor | None = None,
                  out_dtype: torch.dtype | None = None) -> torch.Tensor:
    """round(gscale * fixed-order sum over dim 0) of fp32 partials [S, m, n] to bf16 (default)
    or f16 (out_dtype, or the dtype of `out`)."""
    _require(partials, "partials", torch.float32, 3)
    _require(gscale, "gscale", torch.float32, 1)
    S, m, n = partials.shape
    if gscale.numel() != 1:
        raise ValueError(f"gscale must hold one element, got {gscale.numel()}")
    dtype = _out_dtype(out, out_dtype)
    if out is None:
        out = torch.empty((m, n), dtype=dtype, device=partials.device)
    else:
        _require(out, "out", dtype, 2)
        if tuple(out.shape) != (m, n):
            raise ValueError(f"out must be [{m}, {n}], got {tuple(out.shape)}")
    _same_device(partials, gscale=gscale, out=out)
    with torch.cuda.device(partials.device):
        _check(library().fi_splitk_reduce_out(partials.data_ptr(), S, m, n, gscale.data_ptr(), out.data_ptr(),
                                              _DTYPES[dtype], _stream(partials.device)), "fi_splitk_reduce_out")
    return out
