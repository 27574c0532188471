"""CPU oracle for mm_bf16_fp4 (bf16 activations x NVFP4 weights).

TEST INFRASTRUCTURE ONLY: the slow, plain reference the CUDA library is checked against.
Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import it. It shares no code with the CUDA library and never imports it.

The arithmetic lives in ``nvfp4_oracle.c`` (plain C, fp32 quantiser, fp64 dequantise and
matmul); this module compiles it with gcc on first use and marshals numpy arrays.
Every function is pinned by ``tests/test_oracle_*.py`` against closed forms, an
independent library decoder, brute force on tiny shapes and hand-worked cases.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile nvfp4_oracle.c into oracle/_liboracle.so (gcc, OpenMP, strict IEEE fp)."""
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-frounding-math", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        u8p = ctypes.POINTER(ctypes.c_uint8)
        f32p = ctypes.POINTER(ctypes.c_float)
        f64p = ctypes.POINTER(ctypes.c_double)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i64 = ctypes.c_int64
        lib.orc_e2m1_decode.argtypes = [ctypes.c_uint32]
        lib.orc_e2m1_decode.restype = ctypes.c_double
        lib.orc_e4m3_decode.argtypes = [ctypes.c_uint32]
        lib.orc_e4m3_decode.restype = ctypes.c_double
        lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
        lib.orc_e4m3_encode.restype = ctypes.c_uint32
        lib.orc_e2m1_encode.argtypes = [ctypes.c_float]
        lib.orc_e2m1_encode.restype = ctypes.c_uint32
        lib.orc_f32_to_f16.argtypes = [ctypes.c_float]
        lib.orc_f32_to_f16.restype = ctypes.c_uint16
        lib.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.orc_f32_to_bf16.restype = ctypes.c_uint16
        lib.orc_global_scale.argtypes = [f32p, i64]
        lib.orc_global_scale.restype = ctypes.c_float
        lib.orc_nvfp4_pack.argtypes = [f32p, i64, i64, u8p, u8p, f32p]
        lib.orc_nvfp4_pack.restype = ctypes.c_int
        lib.orc_dequant_row.argtypes = [u8p, u8p, ctypes.c_float, i64, f64p]
        lib.orc_dequant_row.restype = None
        lib.orc_mm.argtypes = [u16p, u8p, u8p, ctypes.c_float, i64, i64, i64, i64p, i64, f64p]
        lib.orc_mm.restype = ctypes.c_int
        lib.orc_splitk_reduce.argtypes = [f32p, i64, i64, ctypes.c_float, ctypes.c_int, u16p]
        lib.orc_splitk_reduce.restype = None
        lib.orc_num_threads.argtypes = []
        lib.orc_num_threads.restype = ctypes.c_int
        lib.orc_set_num_threads.argtypes = [ctypes.c_int]
        lib.orc_set_num_threads.restype = None
        _lib = lib
        return lib


def _ptr(a: np.ndarray, ctype):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctype))


# ------------------------------------------------------------------ element formats

def e2m1_decode(code: int) -> float:
    """Value of a 4-bit E2M1 code (OCP MX v1.0 FP4: bias 1, subnormal 0/0.5, max 6)."""
    return _load().orc_e2m1_decode(int(code))


def e4m3_decode(code: int) -> float:
    """Value of an 8-bit E4M3 code (OCP OFP8: bias 7, max 448, 0x7F/0xFF NaN)."""
    return _load().orc_e4m3_decode(int(code))


def e4m3_encode(x: float) -> int:
    """fp32 -> E4M3 code, round to nearest even, saturating to +-448."""
    return _load().orc_e4m3_encode(float(np.float32(x)))


def e2m1_encode(x: float) -> int:
    """fp32 -> E2M1 code, round to nearest even, saturating to +-6; sign bit follows x."""
    return _load().orc_e2m1_encode(float(np.float32(x)))


def f32_to_bf16_bits(x: float) -> int:
    """fp32 -> bf16 bit pattern, round to nearest even."""
    return _load().orc_f32_to_bf16(float(np.float32(x)))


def f32_to_f16_bits(x: float) -> int:
    """fp32 -> IEEE binary16 bit pattern, round to nearest even, overflow to +-inf."""
    return _load().orc_f32_to_f16(float(np.float32(x)))


def round_out(v: np.ndarray, out_dtype: str = "bf16") -> np.ndarray:
    """fp32 values -> output bits (uint16) of out_dtype ("bf16" or "f16"), round to nearest even."""
    f = f32_to_f16_bits if out_dtype == "f16" else f32_to_bf16_bits
    v = np.asarray(v, np.float32)
    return np.array([f(x) for x in v.ravel()], np.uint16).reshape(v.shape)


# ---------------------------------------------------------------------- quantise

def global_scale(W: np.ndarray) -> np.float32:
    """gscale = amax(|W|) / (448 * 6), one fp32 division."""
    W = np.ascontiguousarray(W, dtype=np.float32)
    return np.float32(_load().orc_global_scale(_ptr(W, ctypes.c_float), W.size))


def pack(W: np.ndarray):
    """Quantise fp32 W [n, k] to NVFP4.

    Returns (Wq uint8 [n, k/2], Wscale uint8 [n, k/16], gscale float32). Byte j of a Wq row
    holds code 2j in its low nibble and code 2j+1 in its high nibble; Wscale is row-major.
    """
    W = np.ascontiguousarray(W, dtype=np.float32)
    n, k = W.shape
    if k % 16:
        raise ValueError("k must be a multiple of 16")
    Wq = np.zeros((n, k // 2), np.uint8)
    Ws = np.zeros((n, k // 16), np.uint8)
    g = np.zeros(1, np.float32)
    rc = _load().orc_nvfp4_pack(_ptr(W, ctypes.c_float), n, k, _ptr(Wq, ctypes.c_uint8),
                                _ptr(Ws, ctypes.c_uint8), _ptr(g, ctypes.c_float))
    if rc != 0:
        raise RuntimeError(f"orc_nvfp4_pack failed ({rc})")
    return Wq, Ws, np.float32(g[0])


# ----------------------------------------------------------------- dequant, matmul

def dequant(Wq: np.ndarray, Wscale: np.ndarray, gscale) -> np.ndarray:
    """dequant(W) in fp64 [n, k] (exact): e2m1(code) * e4m3(scale) * gscale."""
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    Wscale = np.ascontiguousarray(Wscale, dtype=np.uint8)
    n, kh = Wq.shape
    k = kh * 2
    out = np.zeros((n, k), np.float64)
    lib = _load()
    for j in range(n):
        row = out[j]
        lib.orc_dequant_row(_ptr(Wq[j], ctypes.c_uint8), _ptr(Wscale[j], ctypes.c_uint8),
                            float(np.float32(gscale)), k, _ptr(row, ctypes.c_double))
    return out


def mm(A_bits: np.ndarray, Wq: np.ndarray, Wscale: np.ndarray, gscale, cols=None) -> np.ndarray:
    """ref[r, c] = sum_i A[r, i] * dequant(W)[cols[c], i] in fp64, natural i order.

    A_bits is the bf16 bit pattern as uint16 [m, k]. cols selects weight rows (output
    columns); None means all n. Returns float64 [m, len(cols)] (unrounded).
    """
    A_bits = np.ascontiguousarray(A_bits, dtype=np.uint16)
    Wq = np.ascontiguousarray(Wq, dtype=np.uint8)
    Wscale = np.ascontiguousarray(Wscale, dtype=np.uint8)
    m, k = A_bits.shape
    n = Wq.shape[0]
    if Wq.shape[1] * 2 != k or Wscale.shape != (n, k // 16):
        raise ValueError("shape mismatch between A, Wq and Wscale")
    if cols is None:
        cptr, ncols = None, n
    else:
        cols = np.ascontiguousarray(cols, dtype=np.int64)
        cptr, ncols = _ptr(cols, ctypes.c_int64), cols.size
    ref = np.zeros((m, ncols), np.float64)
    rc = _load().orc_mm(_ptr(A_bits, ctypes.c_uint16), _ptr(Wq, ctypes.c_uint8),
                        _ptr(Wscale, ctypes.c_uint8), float(np.float32(gscale)), m, n, k,
                        cptr, ncols, _ptr(ref, ctypes.c_double))
    if rc != 0:
        raise RuntimeError(f"orc_mm failed ({rc})")
    return ref


def splitk_reduce(partials: np.ndarray, gscale, out_dtype: str = "bf16") -> np.ndarray:
    """Bits of round(gscale * (((p0 + p1) + p2) + ...)), all in fp32, rounded to nearest even
    into out_dtype ("bf16", or "f16" for the optional fp16 output).

    partials is float32 [S, m, n]; returns uint16 [m, n].
    """
    if out_dtype not in ("bf16", "f16"):
        raise ValueError("out_dtype must be 'bf16' or 'f16'")
    partials = np.ascontiguousarray(partials, dtype=np.float32)
    S = partials.shape[0]
    mn = partials[0].size
    out = np.zeros(partials.shape[1:], np.uint16)
    _load().orc_splitk_reduce(_ptr(partials, ctypes.c_float), S, mn, float(np.float32(gscale)),
                              1 if out_dtype == "f16" else 0, _ptr(out, ctypes.c_uint16))
    return out


def num_threads() -> int:
    return _load().orc_num_threads()


def set_num_threads(t: int) -> None:
    _load().orc_set_num_threads(int(t))


# ------------------------------------------------------------------ tolerance

def within_tolerance(out: np.ndarray, ref: np.ndarray, rtol: float = 1e-2, rrms: float = 1e-2):
    """Elementwise check |out - ref| <= rtol*|ref| + rrms*rms(ref row).

    out and ref are [m, n]; returns a boolean array of the same shape.
    """
    out = np.asarray(out, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True))
    return np.abs(out - ref) <= rtol * np.abs(ref) + rrms * rms
