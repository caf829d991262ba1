"""ctypes binding of libw8a8.so -- argument marshalling only.

Two layers:
  * the C-ABI functions under their C names (``w8a8_linear_fused(...)`` etc.),
    taking raw pointers and sizes exactly as include/w8a8.h declares them;
  * torch-tensor helpers (``quantize_weights``, ``quant_act``, ``linear``,
    ``linear_fused``, ...) that check dtypes/devices/strides, allocate outputs
    with torch, and call the C-ABI on the current CUDA stream.

Every step of the layer runs in the library's CUDA kernels.  There is no CPU
or PyTorch fallback: if libw8a8.so is missing this module raises on first use.
"""
from __future__ import annotations

import contextlib
import ctypes
import functools
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libw8a8.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "w8a8.h")

W8A8_OK = 0
W8A8_ERR_INVALID_ARG = 1
W8A8_ERR_UNSUPPORTED_SHAPE = 2
W8A8_ERR_MISALIGNED = 3
W8A8_ERR_WORKSPACE = 4
W8A8_ERR_CUDA = 5
W8A8_ERR_DEVICE_TIMEOUT = 6
W8A8_ERR_UNSUPPORTED_DEVICE = 7

VARIANT_AUTO = 0
VARIANT_GEMV = 1
VARIANT_GEMM_BN128 = 2
VARIANT_GEMM_BN256 = 3
VARIANT_GEMM_PAIR = 4
VARIANT_GEMM_BN64 = 5
VARIANT_GEMV_TC = 6
VARIANT_NAMES = {0: "auto", 1: "gemv", 2: "gemm_bn128", 3: "gemm_bn256", 4: "gemm_pair",
                 5: "gemm_bn64", 6: "gemv_tc"}


class W8A8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class Plan(ctypes.Structure):
    _fields_ = [("variant", ctypes.c_int32), ("tile_m", ctypes.c_int32),
                ("tile_n", ctypes.c_int32), ("num_tiles", ctypes.c_int32),
                ("grid", ctypes.c_int32), ("waves_x100", ctypes.c_int32),
                ("split_tiles", ctypes.c_int32), ("split_kblocks_per_pair", ctypes.c_int32),
                ("tail_tiles_nsplit", ctypes.c_int32), ("quant_in_gemm_launch", ctypes.c_int32),
                ("k_split", ctypes.c_int32)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_}


_lib = None
_vp, _i64, _i32, _int, _sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int,
                              ctypes.c_size_t)

_SIGNATURES = {
    "w8a8_status_string": ([_int], ctypes.c_char_p),
    "w8a8_version": ([], ctypes.c_char_p),
    "w8a8_quantize_weights": ([_vp, _i64, _i64, _i64, _vp, _vp, _vp], _int),
    "w8a8_quant_act": ([_vp, _i64, _i64, _i64, _vp, _vp, _vp], _int),
    "w8a8_unpack_int32_weights": ([_vp, _i64, _i64, _vp, _vp], _int),
    "w8a8_workspace_size": ([_i64, _i64, _i64, ctypes.POINTER(_sz)], _int),
    "w8a8_workspace_size_ex": ([_i64, _i64, _i64, _int, ctypes.POINTER(_sz)], _int),
    "w8a8_linear": ([_vp, _vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _i64, _vp, _vp, _sz, _vp],
                    _int),
    "w8a8_linear_ex": ([_vp, _vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _i64, _vp, _int, _vp,
                        _sz, _vp], _int),
    "w8a8_linear_fused": ([_vp, _i64, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _i64, _vp, _vp,
                           _vp, _sz, _vp], _int),
    "w8a8_linear_fused_ex": ([_vp, _i64, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _i64, _vp, _vp,
                              _vp, _sz, _int, _vp], _int),
    "w8a8_linear_fused_host": ([_vp, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _vp, _sz,
                                _vp], _int),
    "w8a8_linear_fused_noalloc": ([_vp, _i64, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _i64, _vp],
                                  _int),
    "w8a16_linear": ([_vp, _i64, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _i64, _vp], _int),
    "w8a8_select": ([_i64, _i64, _i64, _i32, _int, ctypes.POINTER(Plan)], _int),
    "w8a8_last_device_error": ([_vp], _int),
    "w8a8_selftest_bounded_wait": ([_i64, _vp], _int),
    "w8a8_selftest_quant_exhaustive": ([_vp, _vp], _int),
    "w8a8_debug_peek_tag": ([ctypes.POINTER(ctypes.c_uint64)], _int),
    "w8a8_bench_mma_i8_peak": ([_i64, _i32, _vp], _int),
}


def header_functions() -> list[str]:
    """Names of the functions include/w8a8.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"W8A8_API\s+[^;(]*?\b(w8a(?:8|16)_\w+)\s*\(", text)))


def lib() -> ctypes.CDLL:
    """Load libw8a8.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m w8a8_int8_dynamic_token_b200.build`"
                " (there is no fallback implementation)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.argtypes = args
            fn.restype = res
        _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().w8a8_status_string(int(status)).decode()


def version() -> str:
    return lib().w8a8_version().decode()


def _check(status: int, where: str) -> None:
    if status != W8A8_OK:
        raise W8A8Error(status, where)


# ------------------------------------------------------------------ raw C ABI

def w8a8_quantize_weights(W, N, K, ldw, Wq, s_w, stream) -> int:
    return lib().w8a8_quantize_weights(W, N, K, ldw, Wq, s_w, stream)


def w8a8_unpack_int32_weights(packed, N, K, Wq, stream) -> int:
    return lib().w8a8_unpack_int32_weights(packed, N, K, Wq, stream)


def w8a8_quant_act(x, M, K, ldx, q, s_a, stream) -> int:
    return lib().w8a8_quant_act(x, M, K, ldx, q, s_a, stream)


def w8a8_workspace_size(M, N, K) -> tuple[int, int]:
    out = ctypes.c_size_t(0)
    st = lib().w8a8_workspace_size(M, N, K, ctypes.byref(out))
    return st, int(out.value)


def w8a8_workspace_size_ex(M, N, K, variant) -> tuple[int, int]:
    out = ctypes.c_size_t(0)
    st = lib().w8a8_workspace_size_ex(M, N, K, variant, ctypes.byref(out))
    return st, int(out.value)


def w8a8_linear(q, s_a, M, K, Wq, s_w, bias, N, y, ldy, acc_debug, workspace, ws_bytes,
                stream) -> int:
    return lib().w8a8_linear(q, s_a, M, K, Wq, s_w, bias, N, y, ldy, acc_debug, workspace,
                             ws_bytes, stream)


def w8a8_linear_ex(q, s_a, M, K, Wq, s_w, bias, N, y, ldy, acc_debug, variant, workspace,
                   ws_bytes, stream) -> int:
    return lib().w8a8_linear_ex(q, s_a, M, K, Wq, s_w, bias, N, y, ldy, acc_debug, variant,
                                workspace, ws_bytes, stream)


def w8a8_linear_fused(x, M, K, ldx, Wq, s_w, bias, N, y, ldy, q_out, s_a_out, workspace,
                      ws_bytes, stream) -> int:
    return lib().w8a8_linear_fused(x, M, K, ldx, Wq, s_w, bias, N, y, ldy, q_out, s_a_out,
                                   workspace, ws_bytes, stream)


def w8a8_linear_fused_ex(x, M, K, ldx, Wq, s_w, bias, N, y, ldy, q_out, s_a_out, workspace,
                         ws_bytes, options, stream) -> int:
    return lib().w8a8_linear_fused_ex(x, M, K, ldx, Wq, s_w, bias, N, y, ldy, q_out, s_a_out,
                                      workspace, ws_bytes, options, stream)


FUSED_ONE_LAUNCH = 1


def w8a8_linear_fused_host(x_host, M, K, Wq, s_w, bias, N, y_host, x_dev, y_dev, workspace,
                           ws_bytes, stream) -> int:
    return lib().w8a8_linear_fused_host(x_host, M, K, Wq, s_w, bias, N, y_host, x_dev, y_dev,
                                        workspace, ws_bytes, stream)


def w8a8_linear_fused_noalloc(x, M, K, ldx, Wq, s_w, bias, N, y, ldy, stream) -> int:
    return lib().w8a8_linear_fused_noalloc(x, M, K, ldx, Wq, s_w, bias, N, y, ldy, stream)


def w8a16_linear_raw(x, M, K, ldx, Wq, s_w, bias, N, y, ldy, stream) -> int:
    return lib().w8a16_linear(x, M, K, ldx, Wq, s_w, bias, N, y, ldy, stream)


def w8a8_select(M, N, K, num_sms=148, variant=VARIANT_AUTO) -> tuple[int, Plan]:
    plan = Plan()
    st = lib().w8a8_select(M, N, K, num_sms, variant, ctypes.byref(plan))
    return st, plan


def w8a8_last_device_error(stream) -> int:
    return lib().w8a8_last_device_error(stream)


def w8a8_selftest_bounded_wait(limit_ns, stream) -> int:
    return lib().w8a8_selftest_bounded_wait(limit_ns, stream)


# ------------------------------------------------------------------ torch helpers

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if isinstance(stream, int):  # a raw handle (see _OnCurrent)
        return ctypes.c_void_p(stream)
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype, ndim):
    """dtype, rank and unit inner stride (checked before the device, so shape
    errors surface the same way on any device)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-D")
    if t.numel() > 0 and t.stride(-1) != 1:
        raise ValueError(f"{name} must have unit stride in its last dimension")


def _shape(t, name, shape):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _on_one_device(**tensors):
    """The CUDA device every given tensor lives on (all must share it)."""
    dev = None
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, expected {dev}")
    return dev


class _OnCurrent:
    """The common case of _launching: the tensors' device is already current
    and no stream is given, so nothing needs switching; yields that device's
    current stream as a raw handle."""
    __slots__ = ("handle",)

    def __init__(self, handle):
        self.handle = handle

    def __enter__(self):
        return self.handle

    def __exit__(self, *exc):
        return False


def _launching(dev, stream=None):
    """Run a call on the tensors' device: the library reads the current device
    (its properties, and the allocation-free scratch), so that device is made
    current.  The call is enqueued on `stream`, or on that device's current
    stream; tensors allocated inside belong to that stream, so the caching
    allocator never hands their memory to other work while the call may still
    use it.  When the device is current already and no stream is given,
    nothing is switched (a few microseconds of host time per call less)."""
    if stream is None and dev.index == torch.cuda.current_device():
        return _OnCurrent(torch._C._cuda_getCurrentRawStream(dev.index))
    return _switching(dev, stream)


@contextlib.contextmanager
def _switching(dev, stream):
    with torch.cuda.device(dev):
        if stream is None:
            yield torch.cuda.current_stream()
        else:
            if stream.device != dev:
                raise ValueError(f"stream is on {stream.device}, the tensors on {dev}")
            with torch.cuda.stream(stream):
                yield stream


@functools.lru_cache(maxsize=1024)
def workspace_size(M: int, N: int, K: int, variant: int = VARIANT_AUTO) -> int:
    st, n = w8a8_workspace_size_ex(M, N, K, variant)
    _check(st, "w8a8_workspace_size_ex")
    return n


def select(M: int, N: int, K: int, num_sms: int = 148, variant: int = VARIANT_AUTO) -> dict:
    st, plan = w8a8_select(M, N, K, num_sms, variant)
    _check(st, "w8a8_select")
    d = plan.as_dict()
    d["variant_name"] = VARIANT_NAMES[d["variant"]]
    return d


def quantize_weights(W: torch.Tensor, stream=None):
    """bf16 W [N, K] -> (Wq int8 [N, K], s_w fp32 [N]) on W's device."""
    _need(W, "W", torch.bfloat16, 2)
    dev = _on_one_device(W=W)
    N, K = W.shape
    with _launching(dev, stream) as s:
        Wq = torch.empty((N, K), dtype=torch.int8, device=dev)
        s_w = torch.empty((N,), dtype=torch.float32, device=dev)
        _check(w8a8_quantize_weights(_ptr(W), N, K, W.stride(0), _ptr(Wq), _ptr(s_w), _stream(s)),
               "w8a8_quantize_weights")
    return Wq, s_w


def unpack_int32_weights(packed: torch.Tensor, stream=None) -> torch.Tensor:
    """Packed int32 [N, K/4] weight storage (codes + 128, four per word, first
    code in the low byte) -> Wq int8 [N, K] on packed's device."""
    _need(packed, "packed", torch.int32, 2)
    if not packed.is_contiguous():
        raise ValueError("packed must be dense row-major")
    dev = _on_one_device(packed=packed)
    N, K = packed.shape[0], packed.shape[1] * 4
    with _launching(dev, stream) as s:
        Wq = torch.empty((N, K), dtype=torch.int8, device=dev)
        _check(w8a8_unpack_int32_weights(_ptr(packed), N, K, _ptr(Wq), _stream(s)),
               "w8a8_unpack_int32_weights")
    return Wq


def quant_act(x: torch.Tensor, stream=None):
    """bf16 x [M, K] -> (q int8 [M, K], s_a fp32 [M])."""
    _need(x, "x", torch.bfloat16, 2)
    dev = _on_one_device(x=x)
    M, K = x.shape
    with _launching(dev, stream) as s:
        q = torch.empty((M, K), dtype=torch.int8, device=dev)
        s_a = torch.empty((M,), dtype=torch.float32, device=dev)
        _check(w8a8_quant_act(_ptr(x), M, K, x.stride(0), _ptr(q), _ptr(s_a), _stream(s)),
               "w8a8_quant_act")
    return q, s_a


def _workspace_for(M, N, K, workspace, dev, variant=VARIANT_AUTO):
    """(tensor, pointer, bytes): the caller's workspace, or a fresh one of
    workspace_size(M, N, K, variant) bytes when `workspace` is None (allocated
    on the launching stream, inside _launching).  The caller keeps the returned
    tensor alive until the launch has been enqueued: the device memory must
    not return to the allocator before then, or an output allocated
    afterwards could share it."""
    need = workspace_size(M, N, K, variant)
    if workspace is None:
        if need == 0:
            return None, None, 0
        workspace = torch.empty((need,), dtype=torch.uint8, device=dev)
    return workspace, _ptr(workspace), workspace.numel() * workspace.element_size()


def _check_layer_args(M, N, K, bias, out):
    if bias is not None:
        _need(bias, "bias", torch.bfloat16, 1)
        _shape(bias, "bias", (N,))
    if out is not None:
        _need(out, "out", torch.bfloat16, 2)
        _shape(out, "out", (M, N))


def linear(q, s_a, Wq, s_w, bias=None, out=None, acc_debug=False, variant=VARIANT_AUTO,
           workspace=None, split=True, stream=None):
    """y = bf16(((float)(q @ Wq^T) * s_a) * s_w + bias); with acc_debug=True the raw
    int32 accumulators [M, N] are returned instead.  split=False runs the pair
    kernel without its K-split tail (no workspace is passed)."""
    _need(q, "q", torch.int8, 2)
    _need(s_a, "s_a", torch.float32, 1)
    _need(Wq, "Wq", torch.int8, 2)
    _need(s_w, "s_w", torch.float32, 1)
    M, K = q.shape
    N = Wq.shape[0]
    if Wq.shape[1] != K or s_a.shape[0] != M or s_w.shape[0] != N:
        raise ValueError("shape mismatch between q, s_a, Wq, s_w")
    if not (q.is_contiguous() and Wq.is_contiguous()):
        raise ValueError("q and Wq must be dense row-major")
    _check_layer_args(M, N, K, bias, None if acc_debug else out)
    dev = _on_one_device(q=q, s_a=s_a, Wq=Wq, s_w=s_w, bias=bias,
                         out=None if acc_debug else out, workspace=workspace)
    with _launching(dev, stream) as s:
        ws, ws_ptr, ws_bytes = (_workspace_for(M, N, K, workspace, dev, variant) if split
                                else (None, None, 0))
        if acc_debug:
            acc = torch.empty((M, N), dtype=torch.int32, device=dev)
            _check(w8a8_linear_ex(_ptr(q), _ptr(s_a), M, K, _ptr(Wq), _ptr(s_w), _ptr(bias), N,
                                  None, N, _ptr(acc), variant, ws_ptr, ws_bytes, _stream(s)),
                   "w8a8_linear_ex")
            del ws  # enqueued on s: later allocations on s are ordered after the launch
            return acc
        y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        _check(w8a8_linear_ex(_ptr(q), _ptr(s_a), M, K, _ptr(Wq), _ptr(s_w), _ptr(bias), N,
                              _ptr(y), y.stride(0), None, variant, ws_ptr, ws_bytes, _stream(s)),
               "w8a8_linear_ex")
        del ws
    return y


def linear_fused(x, Wq, s_w, bias=None, out=None, workspace=None, return_intermediates=False,
                 stream=None):
    """Whole layer from bf16 x [M, K]: per-token quantization, int8 GEMM, fused
    epilogue.  Returns y [M, N] (and (q, s_a) with return_intermediates=True)."""
    _need(x, "x", torch.bfloat16, 2)
    _need(Wq, "Wq", torch.int8, 2)
    _need(s_w, "s_w", torch.float32, 1)
    M, K = x.shape
    N = Wq.shape[0]
    if Wq.shape[1] != K or s_w.shape[0] != N or not Wq.is_contiguous():
        raise ValueError("shape mismatch between x, Wq, s_w")
    _check_layer_args(M, N, K, bias, out)
    dev = _on_one_device(x=x, Wq=Wq, s_w=s_w, bias=bias, out=out, workspace=workspace)
    with _launching(dev, stream) as s:
        y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        q = s_a = None
        if return_intermediates:
            q = torch.empty((M, K), dtype=torch.int8, device=dev)
            s_a = torch.empty((M,), dtype=torch.float32, device=dev)
        ws, ws_ptr, ws_bytes = _workspace_for(M, N, K, workspace, dev)
        _check(w8a8_linear_fused(_ptr(x), M, K, x.stride(0), _ptr(Wq), _ptr(s_w), _ptr(bias), N,
                                 _ptr(y), y.stride(0), _ptr(q), _ptr(s_a), ws_ptr, ws_bytes,
                                 _stream(s)), "w8a8_linear_fused")
        del ws
    if return_intermediates:
        return y, q, s_a
    return y


def w8a16_linear(x, Wq, s_w, bias=None, out=None, stream=None):
    """Weight-only int8 layer on bf16 x [M, K]: y = bf16((x @ Wq^T) * s_w + bias),
    fp32 accumulation on the tensor cores."""
    _need(x, "x", torch.bfloat16, 2)
    _need(Wq, "Wq", torch.int8, 2)
    _need(s_w, "s_w", torch.float32, 1)
    M, K = x.shape
    N = Wq.shape[0]
    if Wq.shape[1] != K or s_w.shape[0] != N or not Wq.is_contiguous():
        raise ValueError("shape mismatch between x, Wq, s_w")
    _check_layer_args(M, N, K, bias, out)
    dev = _on_one_device(x=x, Wq=Wq, s_w=s_w, bias=bias, out=out)
    with _launching(dev, stream) as s:
        y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        _check(w8a16_linear_raw(_ptr(x), M, K, x.stride(0), _ptr(Wq), _ptr(s_w), _ptr(bias), N,
                                _ptr(y), y.stride(0), _stream(s)), "w8a16_linear")
    return y


def linear_fused_host(x_host, Wq, s_w, bias, y_host, x_dev, y_dev, workspace, stream=None):
    """End-to-end call on host buffers: copy x in, run the layer, copy y out
    (all enqueued on the stream; synchronize before reading y_host)."""
    M, K = x_host.shape
    N = Wq.shape[0]
    if tuple(y_host.shape) != (M, N) or tuple(x_dev.shape) != (M, K) or tuple(y_dev.shape) != (M, N):
        raise ValueError("x_host / x_dev must be [M, K] and y_host / y_dev [M, N]")
    dev = _on_one_device(Wq=Wq, s_w=s_w, bias=bias, x_dev=x_dev, y_dev=y_dev, workspace=workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with _launching(dev, stream) as s:
        _check(w8a8_linear_fused_host(_ptr(x_host), M, K, _ptr(Wq), _ptr(s_w), _ptr(bias), N,
                                      _ptr(y_host), _ptr(x_dev), _ptr(y_dev), _ptr(workspace),
                                      ws_bytes, _stream(s)), "w8a8_linear_fused_host")
    return y_host


def last_device_error(stream=None) -> int:
    return w8a8_last_device_error(_stream(stream))


def selftest_bounded_wait(limit_ns: int, stream=None) -> int:
    return w8a8_selftest_bounded_wait(int(limit_ns), _stream(stream))


def w8a8_selftest_quant_exhaustive(counts_dev, stream) -> int:
    return lib().w8a8_selftest_quant_exhaustive(counts_dev, stream)


def selftest_quant_exhaustive(stream=None) -> tuple[int, int]:
    """(pairs checked, pairs whose code differs from the IEEE-division path)."""
    counts = torch.zeros(2, dtype=torch.int64, device="cuda")
    _check(w8a8_selftest_quant_exhaustive(_ptr(counts), _stream(stream)),
           "w8a8_selftest_quant_exhaustive")
    torch.cuda.current_stream().synchronize() if stream is None else stream.synchronize()
    c = counts.cpu().tolist()
    return int(c[0]), int(c[1])


PEAK_OPS_PER_PAIR_ITERATION = 4 * 2 * 256 * 256 * 32


def bench_mma_i8_peak(iterations: int, pairs: int, stream=None) -> None:
    """Enqueue the int8 tensor-core peak loop (pairs * iterations *
    PEAK_OPS_PER_PAIR_ITERATION operations); time it with CUDA events."""
    _check(lib().w8a8_bench_mma_i8_peak(int(iterations), int(pairs), _stream(stream)),
           "w8a8_bench_mma_i8_peak")


def debug_peek_tag() -> int:
    """The launch tag the next call using arrival counters will draw."""
    out = ctypes.c_uint64(0)
    _check(lib().w8a8_debug_peek_tag(ctypes.byref(out)), "w8a8_debug_peek_tag")
    return int(out.value)
