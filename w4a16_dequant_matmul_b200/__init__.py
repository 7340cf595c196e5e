"""Python binding of libwq, the B200 (sm_100a) library for round-to-nearest group-wise INT4
weight quantization and the W4A16 dequant-matmul.

Argument marshalling only: every function forwards device pointers of torch tensors to the
C ABI declared in include/wq.h, on the current CUDA stream; all arithmetic runs in the
library's kernels. There is no CPU path: without libwq.so or a CUDA device the calls raise.

Functions carry the C names:
    wq_quantize_rtn_g128(W, w_bit=4, group=128, zero_point=True) -> (packed, S, Z)
    wq_quantize_rtn_per_tensor(W) -> (packed, S, Z)
    wq_pack_int4(codes) -> packed
    wq_dequant(packed, S, Z, group, out_dtype) -> W_hat
    wq_w4a16_gemm(X, packed, S, Z, group) -> Y
    wq_w8a16_gemm(X, codes, S) -> Y
    wq_channel_stat(A, stat) -> float32 [cols]      (WQ_STAT_ABSMAX / WQ_STAT_ABSMEAN)
    wq_smooth_scales(xmax, wmax, alpha) -> s
    wq_awq_scales(a_mag, alpha) -> s
    wq_quantize_rtn_scaled(W, s, group=128, zero_point=True) -> (packed, S, Z)
    wq_scale_activations(X, s) -> X / s
    wq_quantize_gptq(W, X, group=128, zero_point=True, damp=0.01) -> (packed, S, Z)
    wq_get_status() -> int
S and Z are returned as torch.float16 tensors (binary16 bit patterns in the C ABI).
"""
from __future__ import annotations

import contextlib
import ctypes
import os

from ._build import LIB_PATH, build_library  # noqa: F401  (build_library re-exported)

__all__ = [
    "WQError", "lib", "status_name",
    "wq_version", "wq_status_string", "wq_quantize_rtn_g128", "wq_quantize_rtn_per_tensor",
    "wq_quantize_per_tensor_workspace_bytes", "wq_quantize_rtn_per_tensor_noalloc",
    "wq_pack_int4", "wq_dequant", "wq_w4a16_gemm",
    "wq_w8a16_gemm", "wq_get_status", "wq_selftest_bounded_wait",
    "wq_channel_stat", "wq_smooth_scales", "wq_awq_scales", "wq_quantize_rtn_scaled",
    "wq_scale_activations", "wq_quantize_gptq", "wq_gptq_workspace_bytes",
    "WQ_F32", "WQ_BF16", "WQ_F16", "WQ_U8", "WQ_I8", "WQ_STAT_ABSMAX", "WQ_STAT_ABSMEAN",
]

WQ_F32, WQ_BF16, WQ_F16, WQ_U8, WQ_I8 = 0, 1, 2, 3, 4
WQ_STAT_ABSMAX, WQ_STAT_ABSMEAN = 0, 1
STATUS_NAMES = {
    0: "WQ_OK", 1: "WQ_ERR_NULL", 2: "WQ_ERR_SHAPE", 3: "WQ_ERR_ALIGN", 4: "WQ_ERR_DTYPE",
    5: "WQ_ERR_UNSUPPORTED", 6: "WQ_ERR_CUDA", 7: "WQ_ERR_NONFINITE", 8: "WQ_ERR_TIMEOUT",
    9: "WQ_ERR_RANGE", 10: "WQ_ERR_NODEVICE", 11: "WQ_ERR_DEVICE",
}


class WQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_name(status)} ({_raw_status_string(status)})")


class _QParams(ctypes.Structure):
    _fields_ = [("w_bit", ctypes.c_int32), ("group", ctypes.c_int32),
                ("zero_point", ctypes.c_int32)]


_LIB = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32

_SIGNATURES = {
    "wq_version": (_I32, []),
    "wq_status_string": (ctypes.c_char_p, [_I32]),
    "wq_quantize_rtn_g128": (_I32, [_P, _I32, _I64, _I64, _I64, ctypes.POINTER(_QParams), _P, _P,
                                    _P, _P]),
    "wq_quantize_per_tensor_workspace_bytes": (ctypes.c_size_t, [_I64, _I64]),
    "wq_quantize_rtn_per_tensor": (_I32, [_P, _I32, _I64, _I64, _I64, _P, _P, _P, _P,
                                          ctypes.c_size_t, _P]),
    "wq_quantize_rtn_per_tensor_noalloc": (_I32, [_P, _I32, _I64, _I64, _I64, _P, _P, _P, _P]),
    "wq_pack_int4": (_I32, [_P, _I64, _I64, _P, _P]),
    "wq_dequant": (_I32, [_P, _P, _P, _I64, _I64, _I32, _P, _I32, _P]),
    "wq_w4a16_gemm": (_I32, [_P, _I64, _I64, _P, _P, _P, _I64, _I64, _I32, _P, _I64, _P]),
    "wq_w8a16_gemm": (_I32, [_P, _I64, _I64, _P, _P, _I64, _I64, _P, _I64, _P]),
    "wq_get_status": (_I32, [_P]),
    "wq_channel_stat": (_I32, [_P, _I32, _I64, _I64, _I64, _I32, _P, _P]),
    "wq_smooth_scales": (_I32, [_P, _P, _I64, ctypes.c_float, _P, _P]),
    "wq_awq_scales": (_I32, [_P, _I64, ctypes.c_float, _P, _P]),
    "wq_quantize_rtn_scaled": (_I32, [_P, _I32, _I64, _I64, _I64, _P, ctypes.POINTER(_QParams),
                                      _P, _P, _P, _P]),
    "wq_scale_activations": (_I32, [_P, _I64, _I64, _I64, _P, _P, _I64, _P]),
    "wq_gptq_workspace_bytes": (ctypes.c_size_t, [_I64, _I64]),
    "wq_quantize_gptq": (_I32, [_P, _I32, _I64, _I64, _I64, _P, _I64, _I64, ctypes.c_double,
                                ctypes.POINTER(_QParams), _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "wq_selftest_bounded_wait": (_I32, [ctypes.c_uint64, _I32, _P]),
}


def lib() -> ctypes.CDLL:
    """The loaded libwq.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m w4a16_dequant_matmul_b200._build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = handle
    return _LIB


def status_name(status: int) -> str:
    return STATUS_NAMES.get(int(status), f"status {status}")


def _raw_status_string(status: int) -> str:
    try:
        return lib().wq_status_string(int(status)).decode()
    except Exception:  # the library itself may be what failed to load
        return "?"


def _check(status: int, where: str) -> None:
    if status != 0:
        raise WQError(status, where)


def _stream(stream=None):
    import torch

    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


_RAW_STREAM = None


def _stream_handle(t, stream=None) -> int:
    """cudaStream_t (as an int) of `stream`, or of the current stream of t's device; the
    raw accessor avoids building a Stream object per call on the decode hot path."""
    global _RAW_STREAM
    if stream is not None:
        return stream.cuda_stream
    if _RAW_STREAM is None:
        import torch

        _RAW_STREAM = getattr(torch._C, "_cuda_getCurrentRawStream", None) or (
            lambda dev: torch.cuda.current_stream(dev).cuda_stream)
    dev = t.get_device()
    if dev < 0:  # a host tensor: the library rejects it; any stream will do
        import torch

        dev = torch.cuda.current_device()
    return _RAW_STREAM(dev)


_GET_DEVICE = None


def _on_device(t):
    """A context that makes the CUDA device holding tensor t current for the call (the C
    library works on the current device and rejects other devices' memory); a no-op when
    it already is current, or when t is not a CUDA tensor."""
    global _GET_DEVICE
    d = t.get_device()
    if d < 0:
        return contextlib.nullcontext()
    import torch

    if _GET_DEVICE is None:
        _GET_DEVICE = getattr(torch._C, "_cuda_getDevice", None) or torch.cuda.current_device
    if _GET_DEVICE() == d:
        return contextlib.nullcontext()
    return torch.cuda.device(d)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _rows(t, name):
    if t.dim() != 2 or (t.shape[1] > 1 and t.stride(1) != 1):
        raise ValueError(f"{name} must be a 2-D tensor with unit column stride")
    return t.stride(0) if t.shape[0] > 1 else max(t.shape[1], t.stride(0))


def _w_dtype(t):
    import torch

    if t.dtype == torch.float32:
        return WQ_F32
    if t.dtype == torch.bfloat16:
        return WQ_BF16
    raise TypeError("W must be float32 or bfloat16")


def wq_version() -> int:
    return int(lib().wq_version())


def wq_status_string(status: int) -> str:
    return _raw_status_string(status)


def wq_quantize_rtn_g128(W, w_bit: int = 4, group: int = 128, zero_point: bool = True,
                         packed=None, S=None, Z=None, stream=None):
    """Round-to-nearest quantization of W [N, K]. INT4 asymmetric ({4, g, True}) returns
    (packed uint8 [N, K/2], S fp16 [N, K/g], Z fp16 [N, K/g]); INT4 symmetric
    ({4, g, False}) the same, with codes q + 8 and every Z = 8; INT8 symmetric per channel
    ({8, K, False}) returns (codes int8 [N, K], S fp16 [N], None)."""
    import torch

    N, K = W.shape
    ldw = _rows(W, "W")
    dev = W.device
    if w_bit == 4:
        packed = torch.empty((N, K // 2), dtype=torch.uint8, device=dev) if packed is None else packed
        G = K // group if group else 1
        S = torch.empty((N, G), dtype=torch.float16, device=dev) if S is None else S
        Z = torch.empty((N, G), dtype=torch.float16, device=dev) if Z is None else Z
    else:
        packed = torch.empty((N, K), dtype=torch.int8, device=dev) if packed is None else packed
        S = torch.empty((N,), dtype=torch.float16, device=dev) if S is None else S
    p = _QParams(w_bit, group, 1 if zero_point else 0)
    with _on_device(W):
        st = lib().wq_quantize_rtn_g128(_ptr(W), _w_dtype(W), N, K, ldw, ctypes.byref(p),
                                        _ptr(packed), _ptr(S), _ptr(Z), _stream(stream))
    _check(st, "wq_quantize_rtn_g128")
    return packed, S, Z


def wq_quantize_per_tensor_workspace_bytes(N: int, K: int) -> int:
    return int(lib().wq_quantize_per_tensor_workspace_bytes(N, K))


def wq_quantize_rtn_per_tensor(W, workspace=None, stream=None):
    """Per-tensor asymmetric INT4: returns (packed [N, K/2], S fp16 [1], Z fp16 [1])."""
    import torch

    N, K = W.shape
    ldw = _rows(W, "W")
    dev = W.device
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    S = torch.empty((1,), dtype=torch.float16, device=dev)
    Z = torch.empty((1,), dtype=torch.float16, device=dev)
    nbytes = wq_quantize_per_tensor_workspace_bytes(N, K)
    if workspace is None:
        workspace = torch.empty((nbytes,), dtype=torch.uint8, device=dev)
    with _on_device(W):
        st = lib().wq_quantize_rtn_per_tensor(_ptr(W), _w_dtype(W), N, K, ldw, _ptr(packed),
                                              _ptr(S), _ptr(Z), _ptr(workspace),
                                              workspace.numel() * workspace.element_size(),
                                              _stream(stream))
    _check(st, "wq_quantize_rtn_per_tensor")
    return packed, S, Z


def wq_quantize_rtn_per_tensor_noalloc(W, stream=None):
    """Per-tensor asymmetric INT4 without a workspace (for callers that cannot allocate
    device memory); the library's own fixed scratch array is used. Returns
    (packed [N, K/2], S fp16 [1], Z fp16 [1]). Output tensors are allocated here by torch
    only for convenience; C callers pass their own."""
    import torch

    N, K = W.shape
    ldw = _rows(W, "W")
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=W.device)
    S = torch.empty((1,), dtype=torch.float16, device=W.device)
    Z = torch.empty((1,), dtype=torch.float16, device=W.device)
    with _on_device(W):
        st = lib().wq_quantize_rtn_per_tensor_noalloc(_ptr(W), _w_dtype(W), N, K, ldw,
                                                      _ptr(packed), _ptr(S), _ptr(Z),
                                                      _stream(stream))
    _check(st, "wq_quantize_rtn_per_tensor_noalloc")
    return packed, S, Z


def wq_pack_int4(codes, packed=None, stream=None):
    """codes uint8 [N, K] in [0, 15] -> packed uint8 [N, K/2]."""
    import torch

    N, K = codes.shape
    if not codes.is_contiguous():
        raise ValueError("codes must be contiguous")
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=codes.device) if packed is None else packed
    with _on_device(codes):
        st = lib().wq_pack_int4(_ptr(codes), N, K, _ptr(packed), _stream(stream))
    _check(st, "wq_pack_int4")
    return packed


def wq_dequant(packed, S, Z, group: int = 128, out_dtype=None, out=None, stream=None):
    """W_hat = S'(q - Z) as float32 (exact) or bfloat16 [N, K]."""
    import torch

    out_dtype = torch.float32 if out_dtype is None else out_dtype
    N, K2 = packed.shape
    K = 2 * K2
    code = WQ_F32 if out_dtype == torch.float32 else WQ_BF16 if out_dtype == torch.bfloat16 else -1
    out = torch.empty((N, K), dtype=out_dtype, device=packed.device) if out is None else out
    with _on_device(packed):
        st = lib().wq_dequant(_ptr(packed), _ptr(S), _ptr(Z), N, K, group, _ptr(out), code,
                              _stream(stream))
    _check(st, "wq_dequant")
    return out


_GEMM = None


def wq_w4a16_gemm(X, packed, S, Z, group: int = 128, Y=None, stream=None):
    """Y [M, N] bf16 = X [M, K] bf16 @ W_hat^T, fp32 accumulation. (The decode hot path:
    raw integer pointers and a cached function handle keep the per-call host cost low.)"""
    global _GEMM
    if _GEMM is None:
        _GEMM = lib().wq_w4a16_gemm
    M, K = X.shape
    N = packed.shape[0]
    ldx = _rows(X, "X")
    if Y is None:
        import torch

        Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    ldy = _rows(Y, "Y")
    with _on_device(X):
        st = _GEMM(X.data_ptr(), M, ldx, packed.data_ptr(), S.data_ptr(), Z.data_ptr(), N, K,
                   group, Y.data_ptr(), ldy, _stream_handle(X, stream))
    if st != 0:
        raise WQError(st, "wq_w4a16_gemm")
    return Y


def wq_w8a16_gemm(X, codes, S, Y=None, stream=None):
    """Y [M, N] bf16 = X [M, K] bf16 @ (s' q)^T with INT8 per-channel weights."""
    import torch

    M, K = X.shape
    N = codes.shape[0]
    ldx = _rows(X, "X")
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device) if Y is None else Y
    ldy = _rows(Y, "Y")
    with _on_device(X):
        st = lib().wq_w8a16_gemm(_ptr(X), M, ldx, _ptr(codes), _ptr(S), N, K, _ptr(Y), ldy,
                                 _stream(stream))
    _check(st, "wq_w8a16_gemm")
    return Y


def wq_channel_stat(A, stat: int = WQ_STAT_ABSMAX, out=None, stream=None):
    """Per-column max |A_ij| (WQ_STAT_ABSMAX) or mean |A_ij| (WQ_STAT_ABSMEAN) of A [rows,
    cols] (float32 or bfloat16) -> float32 [cols]."""
    import torch

    rows, cols = A.shape
    lda = _rows(A, "A")
    out = torch.empty((cols,), dtype=torch.float32, device=A.device) if out is None else out
    with _on_device(A):
        st = lib().wq_channel_stat(_ptr(A), _w_dtype(A), rows, cols, lda, int(stat), _ptr(out),
                                   _stream(stream))
    _check(st, "wq_channel_stat")
    return out


def wq_smooth_scales(xmax, wmax, alpha: float = 0.5, out=None, stream=None):
    """SmoothQuant factors s_j = xmax_j^alpha / wmax_j^(1 - alpha), float32 [K]."""
    import torch

    K = xmax.shape[0]
    out = torch.empty((K,), dtype=torch.float32, device=xmax.device) if out is None else out
    with _on_device(xmax):
        st = lib().wq_smooth_scales(_ptr(xmax), _ptr(wmax), K, float(alpha), _ptr(out),
                                    _stream(stream))
    _check(st, "wq_smooth_scales")
    return out


def wq_awq_scales(a_mag, alpha: float, out=None, stream=None):
    """AWQ factors a_j^alpha / sqrt(max * min), float32 [K]."""
    import torch

    K = a_mag.shape[0]
    out = torch.empty((K,), dtype=torch.float32, device=a_mag.device) if out is None else out
    with _on_device(a_mag):
        st = lib().wq_awq_scales(_ptr(a_mag), K, float(alpha), _ptr(out), _stream(stream))
    _check(st, "wq_awq_scales")
    return out


def wq_quantize_rtn_scaled(W, s, group: int = 128, zero_point: bool = True, packed=None,
                           S=None, Z=None, stream=None):
    """RTN INT4 of W diag(s) (W [N, K] float32 or bfloat16, s float32 [K]): returns
    (packed uint8 [N, K/2], S fp16 [N, K/g], Z fp16 [N, K/g]) as wq_quantize_rtn_g128."""
    import torch

    N, K = W.shape
    ldw = _rows(W, "W")
    dev = W.device
    G = K // group if group else 1
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=dev) if packed is None else packed
    S = torch.empty((N, G), dtype=torch.float16, device=dev) if S is None else S
    Z = torch.empty((N, G), dtype=torch.float16, device=dev) if Z is None else Z
    p = _QParams(4, group, 1 if zero_point else 0)
    with _on_device(W):
        st = lib().wq_quantize_rtn_scaled(_ptr(W), _w_dtype(W), N, K, ldw, _ptr(s),
                                          ctypes.byref(p), _ptr(packed), _ptr(S), _ptr(Z),
                                          _stream(stream))
    _check(st, "wq_quantize_rtn_scaled")
    return packed, S, Z


def wq_scale_activations(X, s, out=None, stream=None):
    """X / s per column (X [M, K] bfloat16, s float32 [K]) -> bfloat16 [M, K]; out may be
    X itself."""
    import torch

    M, K = X.shape
    ldx = _rows(X, "X")
    out = torch.empty((M, K), dtype=torch.bfloat16, device=X.device) if out is None else out
    ldo = _rows(out, "out")
    with _on_device(X):
        st = lib().wq_scale_activations(_ptr(X), M, K, ldx, _ptr(s), _ptr(out), ldo,
                                        _stream(stream))
    _check(st, "wq_scale_activations")
    return out


def wq_gptq_workspace_bytes(N: int, K: int) -> int:
    return int(lib().wq_gptq_workspace_bytes(N, K))


def wq_quantize_gptq(W, X, group: int = 128, zero_point: bool = True, damp: float = 0.01,
                     workspace=None, stream=None):
    """GPTQ of W [N, K] (float32 or bfloat16) on calibration activations X [T, K] (bfloat16):
    returns (packed uint8 [N, K/2], S fp16 [N, K/g], Z fp16 [N, K/g]) in the RTN format."""
    import torch

    N, K = W.shape
    T = X.shape[0]
    ldw = _rows(W, "W")
    ldx = _rows(X, "X")
    dev = W.device
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    S = torch.empty((N, K // group), dtype=torch.float16, device=dev)
    Z = torch.empty((N, K // group), dtype=torch.float16, device=dev)
    nbytes = wq_gptq_workspace_bytes(N, K)
    if workspace is None:
        workspace = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=dev)
    p = _QParams(4, group, 1 if zero_point else 0)
    with _on_device(W):
        st = lib().wq_quantize_gptq(_ptr(W), _w_dtype(W), N, K, ldw, _ptr(X), T, ldx,
                                    float(damp), ctypes.byref(p), _ptr(packed), _ptr(S), _ptr(Z),
                                    _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream))
    _check(st, "wq_quantize_gptq")
    return packed, S, Z


def wq_selftest_bounded_wait(limit_ns: int = 20_000_000, spin: bool = True, stream=None) -> None:
    """Launch the failure-detection self-test (a bounded wait that runs out); the next
    wq_get_status() then returns WQ_ERR_TIMEOUT (8)."""
    _check(lib().wq_selftest_bounded_wait(int(limit_ns), 1 if spin else 0, _stream(stream)),
           "wq_selftest_bounded_wait")


def wq_get_status(stream=None) -> int:
    """Synchronize the stream and return (and clear) the device status word."""
    return int(lib().wq_get_status(_stream(stream)))
