"""CPU oracle for the W8A8 int8-dynamic linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference leg may import this package.  It shares no
code with the CUDA library and never imports it.

The arithmetic lives in ``w8a8_oracle.c`` (plain C, one IEEE binary32 operation
at a time, OpenMP over rows); this module only marshals numpy arrays.  bf16
values travel as their uint16 bit patterns.

Functions and the passages they follow (see the C file for the full text):

* ``quant_rows``      per-row symmetric int8 quantization, s = max|x|/127,
                      q = clamp(rint(x/s), -127, 127), ties to even -- the
                      dynamic per-token activation scheme of "Issue 5 probe:
                      int8 quantized DiT serve paths on the RTX 3090 (24 GB)",
                      section "Round two ... W8A8 int8-dynamic"; applied to
                      weight rows it is the per-output-channel weight scheme
                      of the same section and of "Qwen-Image-2.1: TE
                      AutoRound-AWQ on GPU + all-resident single-3090 stack",
                      section "Whole-pipeline follow-up".
* ``gemm_i32``        exact int8 x int8 -> int32 product (int64 sums, checked).
* ``epilogue``        y32 = ((float)acc * s_a) * s_w + bias, then bf16 (RNE);
                      the x act_scale factor is the one the "Round two" section
                      warns a reference must not drop.
* ``linear``          the three steps above for one layer call.

Every function is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py``; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is not None:
        return _lib
    path = _build.build()
    lib = ctypes.CDLL(path)
    i64, vp = ctypes.c_int64, ctypes.c_void_p
    lib.w8a8_oracle_quant_rows.argtypes = [vp, i64, i64, i64, vp, i64, vp]
    lib.w8a8_oracle_quant_rows.restype = ctypes.c_int
    lib.w8a8_oracle_gemm_i32.argtypes = [vp, i64, i64, vp, i64, i64, i64, vp, i64]
    lib.w8a8_oracle_gemm_i32.restype = i64
    lib.w8a8_oracle_epilogue.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, i64, vp, i64]
    lib.w8a8_oracle_epilogue.restype = ctypes.c_int
    lib.w8a8_oracle_linear.argtypes = [vp, i64, i64, i64, vp, vp, vp, i64, vp, vp, vp, vp, vp]
    lib.w8a8_oracle_linear.restype = i64
    lib.w8a16_oracle_linear.argtypes = [vp, i64, i64, i64, vp, vp, vp, i64, vp, vp, vp, vp]
    lib.w8a16_oracle_linear.restype = ctypes.c_int
    lib.w8a8_oracle_pack_int32.argtypes = [vp, i64, i64, vp]
    lib.w8a8_oracle_pack_int32.restype = None
    lib.w8a8_oracle_unpack_int32.argtypes = [vp, i64, i64, vp]
    lib.w8a8_oracle_unpack_int32.restype = None
    lib.w8a8_oracle_f32_to_bf16.argtypes = [ctypes.c_float]
    lib.w8a8_oracle_f32_to_bf16.restype = ctypes.c_uint16
    lib.w8a8_oracle_set_threads.argtypes = [ctypes.c_int]
    lib.w8a8_oracle_set_threads.restype = None
    lib.w8a8_oracle_threads.argtypes = []
    lib.w8a8_oracle_threads.restype = ctypes.c_int
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _as_c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return np.ascontiguousarray(a)


def set_threads(n: int) -> None:
    """Set the OpenMP thread count the oracle uses."""
    _load().w8a8_oracle_set_threads(int(n))


def threads() -> int:
    """OpenMP thread count the oracle will use."""
    return int(_load().w8a8_oracle_threads())


def f32_to_bf16_bits(v: float) -> int:
    return int(_load().w8a8_oracle_f32_to_bf16(ctypes.c_float(v)))


def quant_rows(x_bits: np.ndarray):
    """Per-row symmetric int8 quantization of bf16 rows (uint16 bits, [R, C]).

    Returns (q int8 [R, C], s float32 [R])."""
    x = _as_c(x_bits, np.uint16)
    if x.ndim != 2:
        raise ValueError("x must be 2-D")
    R, C = x.shape
    q = np.empty((R, C), np.int8)
    s = np.empty((R,), np.float32)
    rc = _load().w8a8_oracle_quant_rows(_ptr(x), R, C, C, _ptr(q), C, _ptr(s))
    if rc != 0:
        raise RuntimeError("oracle quant_rows rejected its arguments")
    return q, s


# Weight quantization is the same rule applied to the rows of W [N, K].
quantize_weights = quant_rows


def gemm_i32(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Exact acc[m, n] = sum_k a[m, k] * b[n, k] for int8 a [M, K], b [N, K]."""
    a = _as_c(a, np.int8)
    b = _as_c(b, np.int8)
    M, K = a.shape
    N, K2 = b.shape
    if K != K2:
        raise ValueError("inner dimensions differ")
    acc = np.empty((M, N), np.int32)
    ov = _load().w8a8_oracle_gemm_i32(_ptr(a), M, K, _ptr(b), N, K, K, _ptr(acc), N)
    if ov != 0:
        raise OverflowError(f"{ov} accumulators do not fit int32")
    return acc


def epilogue(acc: np.ndarray, s_a: np.ndarray, s_w: np.ndarray, bias_bits=None):
    """y32 = ((float)acc * s_a[m]) * s_w[n] (+ bias[n]); returns (y32, y_bits)."""
    acc = _as_c(acc, np.int32)
    s_a = _as_c(s_a, np.float32)
    s_w = _as_c(s_w, np.float32)
    M, N = acc.shape
    if s_a.shape != (M,) or s_w.shape != (N,):
        raise ValueError("scale shapes do not match acc")
    b = None
    if bias_bits is not None:
        b = _as_c(bias_bits, np.uint16)
        if b.shape != (N,):
            raise ValueError("bias must be [N]")
    y32 = np.empty((M, N), np.float32)
    y = np.empty((M, N), np.uint16)
    rc = _load().w8a8_oracle_epilogue(
        _ptr(acc), M, N, N, _ptr(s_a), _ptr(s_w), _ptr(b) if b is not None else None,
        _ptr(y32), N, _ptr(y), N)
    if rc != 0:
        raise RuntimeError("oracle epilogue rejected its arguments")
    return y32, y


def linear(x_bits: np.ndarray, wq: np.ndarray, s_w: np.ndarray, bias_bits=None) -> dict:
    """Whole layer: quantize x rows, exact int32 GEMM against wq, fp32 epilogue.

    Returns dict(q, s_a, acc, y32, y) with y as bf16 bits."""
    x = _as_c(x_bits, np.uint16)
    wq = _as_c(wq, np.int8)
    s_w = _as_c(s_w, np.float32)
    M, K = x.shape
    N, K2 = wq.shape
    if K != K2 or s_w.shape != (N,):
        raise ValueError("shape mismatch")
    b = None
    if bias_bits is not None:
        b = _as_c(bias_bits, np.uint16)
        if b.shape != (N,):
            raise ValueError("bias must be [N]")
    q = np.empty((M, K), np.int8)
    s_a = np.empty((M,), np.float32)
    acc = np.empty((M, N), np.int32)
    y32 = np.empty((M, N), np.float32)
    y = np.empty((M, N), np.uint16)
    ov = _load().w8a8_oracle_linear(
        _ptr(x), M, K, K, _ptr(wq), _ptr(s_w), _ptr(b) if b is not None else None, N,
        _ptr(q), _ptr(s_a), _ptr(acc), _ptr(y32), _ptr(y))
    if ov < 0:
        raise RuntimeError("oracle linear rejected its arguments")
    if ov > 0:
        raise OverflowError(f"{ov} accumulators do not fit int32")
    return {"q": q, "s_a": s_a, "acc": acc, "y32": y32, "y": y}


def w8a16_linear(x_bits: np.ndarray, wq: np.ndarray, s_w: np.ndarray, bias_bits=None) -> dict:
    """Weight-only int8 layer on bf16 activations: y = bf16(acc32 * s_w + bias)
    with acc32 = the exact sum_k x * q rounded once to fp32.  Returns acc32,
    abs_sum (sum_k |x * q|, for summation-order bounds), y32 and y (bf16 bits)."""
    x_bits = _as_c(x_bits, np.uint16)
    wq = _as_c(wq, np.int8)
    s_w = _as_c(s_w, np.float32)
    M, K = x_bits.shape
    N = wq.shape[0]
    if wq.shape[1] != K or s_w.shape[0] != N:
        raise ValueError("shape mismatch")
    b = None if bias_bits is None else _as_c(bias_bits, np.uint16)
    out = {k: np.empty((M, N), np.float32) for k in ("acc32", "abs_sum", "y32")}
    out["y"] = np.empty((M, N), np.uint16)
    st = _load().w8a16_oracle_linear(_ptr(x_bits), M, K, K, _ptr(wq), _ptr(s_w),
                                     None if b is None else _ptr(b), N, _ptr(out["acc32"]),
                                     _ptr(out["abs_sum"]), _ptr(out["y32"]), _ptr(out["y"]))
    if st != 0:
        raise ValueError("w8a16_oracle_linear: bad arguments")
    return out


def pack_int32(wq: np.ndarray) -> np.ndarray:
    """int8 [N, K] codes -> int32 [N, K/4] words: each code + 128 as a byte,
    four consecutive codes per word, the first in the least significant byte
    (the serialized weight storage; the order inside a word is this module's
    reading of the pages)."""
    wq = _as_c(wq, np.int8)
    N, K = wq.shape
    if K % 4:
        raise ValueError("K must be a multiple of 4")
    out = np.empty((N, K // 4), np.int32)
    _load().w8a8_oracle_pack_int32(_ptr(wq), N, K, _ptr(out))
    return out


def unpack_int32(packed: np.ndarray, K: int) -> np.ndarray:
    """int32 [N, K/4] words -> int8 [N, K] codes (inverse of pack_int32)."""
    packed = _as_c(packed, np.int32)
    N = packed.shape[0]
    if packed.shape[1] * 4 != K:
        raise ValueError("packed must be [N, K/4]")
    out = np.empty((N, K), np.int8)
    _load().w8a8_oracle_unpack_int32(_ptr(packed), N, K, _ptr(out))
    return out


def library_path() -> str:
    return _build.LIB


__all__ = [
    "quant_rows", "quantize_weights", "gemm_i32", "epilogue", "linear",
    "set_threads", "threads", "f32_to_bf16_bits", "library_path",
]
