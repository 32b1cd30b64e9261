"""ctypes binding of libw8a8 (include/w8a8.h) over torch CUDA tensors.

Argument marshalling only: every function here checks tensor dtypes/shapes,
passes raw device pointers, sizes and the current CUDA stream to the C entry
point of the same name, and raises W8A8Error when it returns a non-OK status.
All compute runs in the library's kernels; there is no fallback. If
libw8a8.so is missing or cannot load, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_PATH = os.path.join(HERE, "libw8a8.so")
HEADER = os.path.join(ROOT, "include", "w8a8.h")

OK = 0
BF16, FP32, I32 = 0, 1, 2
DECODE_MAX_M = 64  # calls with at most this many tokens take the weight-streaming decode kernel
STATUS_NAMES = {}


class W8A8Error(RuntimeError):
    def __init__(self, fn, status, msg):
        super().__init__(f"{fn} failed: {msg} ({status})")
        self.status = status


_lock = threading.Lock()
_lib = None

_P, _I64, _I32, _SZ, _F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
_SIGNATURES = {
    "w8a8_status_string": (ctypes.c_char_p, [_I32]),
    "w8a8_quant_weight_per_channel": (_I32, [_P, _I32, _I64, _I64, _I64, _P, _P, _P, _P]),
    "w8a8_calibrate_static": (_I32, [_P, _I32, _I64, _I64, _I64, _P, _P, _P, _P]),
    "w8a8_quant_per_token": (_I32, [_P, _I64, _I64, _I64, _P, _P, _P]),
    "w8a8_quant_per_tensor": (_I32, [_P, _I64, _I64, _I64, _P, _P, _P, _P]),
    "w8a8_dequant_per_tensor": (_I32, [_P, _I64, _I64, _I64, _P, _P, _P, _I32, _P]),
    "w8a8_gemm_dequant": (_I32, [_P, _P, _I32, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _I32, _P, _SZ, _P]),
    "w8a8_gemm_workspace_size": (_SZ, [_I64, _I64, _I64]),
    "w8a8_linear_static": (_I32, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _I64, _P, _I32, _P, _SZ, _P]),
    "w8a8_gemm_requant": (_I32, [_P, _P, _I32, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P, _P, _P]),
    "w8a8_linear_static_requant": (_I32, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _I64, _P, _P, _P, _P,
                                          _SZ, _P]),
    "w8a8_linear_static_noalloc": (_I32, [_P, _I64, _I64, _I64, _P, _P, _P, _P, _P, _P, _P, _I64, _P, _I32, _P]),
    "int8_outlier_split": (_I32, [_P, _I64, _I64, _I64, _F, _I32, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "int8_outlier_split_workspace_size": (_SZ, [_I64]),
    "int8_mixed_decomp_gemm": (_I32, [_P, _P, _P, _P, _P, _I32, _P, _P, _P, _I64, _P, _I64, _I64, _I64, _P, _I32, _P]),
    "w8a8_check_device_error": (_I32, [_P, _P]),
    "w8a8_debug_wait_timeout_selftest": (_I32, [ctypes.c_uint64, _P]),
}


def header_symbols() -> list[str]:
    """Names of the functions include/w8a8.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)


def lib() -> ctypes.CDLL:
    """Load libw8a8.so (once) and declare every entry point's signature."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m int8_gemm_token_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().w8a8_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != OK:
        raise W8A8Error(fn, status, status_string(status))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dt(dtype) -> int:
    return {torch.bfloat16: BF16, torch.float32: FP32, torch.int32: I32}[dtype]


def _ld(t: torch.Tensor) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with contiguous rows")
    return t.stride(0)


def _expect(t: torch.Tensor, dtype, shape, what: str):
    """Raise before the C call when a tensor the C side takes as a raw
    pointer of a fixed type and dense layout is not that."""
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{what}: expected a contiguous {dtype} tensor of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)}")


# --------------------------------------------------------------------------
# Entry points (same names as the C ABI)
# --------------------------------------------------------------------------

def w8a8_quant_weight_per_channel(W: torch.Tensor, Wq=None, s_w=None, colsum=None, stream=None):
    """W [K, N] bf16/fp32 -> (Wq int8 [N, K], s_w fp32 [N], colsum int32 [N])."""
    K, N = W.shape
    dev = W.device
    Wq = torch.empty((N, K), dtype=torch.int8, device=dev) if Wq is None else Wq
    s_w = torch.empty((N,), dtype=torch.float32, device=dev) if s_w is None else s_w
    colsum = torch.empty((N,), dtype=torch.int32, device=dev) if colsum is None else colsum
    _check("w8a8_quant_weight_per_channel", lib().w8a8_quant_weight_per_channel(
        _ptr(W), _dt(W.dtype), K, N, _ld(W), _ptr(Wq), _ptr(s_w), _ptr(colsum), _stream(stream)))
    return Wq, s_w, colsum


def w8a8_calibrate_static(Xcal: torch.Tensor, S=None, r=None, Z=None, stream=None):
    """MinMax calibration over Xcal [T, K] -> device scalars (S, r, Z)."""
    T, K = Xcal.shape
    dev = Xcal.device
    S = torch.empty((1,), dtype=torch.float32, device=dev) if S is None else S
    r = torch.empty((1,), dtype=torch.float32, device=dev) if r is None else r
    Z = torch.empty((1,), dtype=torch.int32, device=dev) if Z is None else Z
    _check("w8a8_calibrate_static", lib().w8a8_calibrate_static(
        _ptr(Xcal), _dt(Xcal.dtype), T, K, _ld(Xcal), _ptr(S), _ptr(r), _ptr(Z), _stream(stream)))
    return S, r, Z


def w8a8_quant_per_token(X: torch.Tensor, Xq=None, S_x=None, stream=None):
    """bf16 X [M, K] -> (Xq int8 [M, K], S_x fp32 [M])."""
    M, K = X.shape
    Xq = torch.empty((M, K), dtype=torch.int8, device=X.device) if Xq is None else Xq
    S_x = torch.empty((M,), dtype=torch.float32, device=X.device) if S_x is None else S_x
    _check("w8a8_quant_per_token", lib().w8a8_quant_per_token(
        _ptr(X), M, K, _ld(X), _ptr(Xq), _ptr(S_x), _stream(stream)))
    return Xq, S_x


def w8a8_quant_per_tensor(X: torch.Tensor, r: torch.Tensor, Z: torch.Tensor, Xq=None, stream=None):
    M, K = X.shape
    Xq = torch.empty((M, K), dtype=torch.int8, device=X.device) if Xq is None else Xq
    _check("w8a8_quant_per_tensor", lib().w8a8_quant_per_tensor(
        _ptr(X), M, K, _ld(X), _ptr(r), _ptr(Z), _ptr(Xq), _stream(stream)))
    return Xq


def w8a8_dequant_per_tensor(Xq: torch.Tensor, S: torch.Tensor, Z: torch.Tensor, out=None, out_dtype=torch.bfloat16,
                            stream=None):
    """int8 Xq [M, K] -> S * (Xq - Z) as bf16 or fp32 [M, K]."""
    M, K = Xq.shape
    if Xq.dtype != torch.int8:
        raise ValueError(f"Xq: expected int8 codes, got {Xq.dtype}")
    out = torch.empty((M, K), dtype=out_dtype, device=Xq.device) if out is None else out
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError(f"out: expected bfloat16 or float32, got {out.dtype}")
    _expect(out, out.dtype, (M, K), "out")
    _check("w8a8_dequant_per_tensor", lib().w8a8_dequant_per_tensor(
        _ptr(Xq), M, K, _ld(Xq), _ptr(S), _ptr(Z), _ptr(out), _dt(out.dtype),
        _stream(stream)))
    return out


def w8a8_gemm_workspace_size(M: int, N: int, K: int) -> int:
    return int(lib().w8a8_gemm_workspace_size(M, N, K))


def new_workspace(M: int, N: int, K: int, device=None) -> torch.Tensor | None:
    """A workspace for w8a8_linear_static of this shape (None when the shape
    needs none). It needs no initial contents; calls on one stream may share it."""
    n = w8a8_gemm_workspace_size(M, N, K)
    if n == 0:
        return None
    return torch.empty((n,), dtype=torch.uint8, device=device or torch.device("cuda"))


def _workspace(n: int, dev, ws):
    if n == 0:
        return None, 0
    if ws is None:
        ws = torch.empty((n,), dtype=torch.uint8, device=dev)
    return ws, ws.numel() * ws.element_size()


def w8a8_gemm_dequant(Xq, S_x, Wq, s_w, colsum=None, Z=None, bias=None, out=None,
                      out_dtype=torch.bfloat16, workspace=None, stream=None):
    """out [M, N] = S_x * s_w * (Xq Wq^T - Z * colsum) + bias.

    S_x is [M] (per token) or a 1-element tensor (per tensor)."""
    M, K = Xq.shape
    N = Wq.shape[0]
    out = torch.empty((M, N), dtype=out_dtype, device=Xq.device) if out is None else out
    if S_x.numel() not in (1, M):
        raise ValueError("S_x holds one scale per row or a single per-tensor scale")
    per_row = 1 if S_x.numel() == M else 0
    ws, nbytes = (None, 0) if workspace is None else (workspace, workspace.numel() * workspace.element_size())
    _check("w8a8_gemm_dequant", lib().w8a8_gemm_dequant(
        _ptr(Xq), _ptr(S_x), per_row, _ptr(Z), _ptr(Wq), _ptr(s_w), _ptr(colsum), _ptr(bias),
        M, N, K, _ptr(out), _dt(out.dtype), _ptr(ws), nbytes, _stream(stream)))
    return out


def w8a8_linear_static(X, S, r, Z, Wq, s_w, colsum, bias=None, out=None, out_dtype=torch.bfloat16,
                       workspace=None, stream=None):
    """Fused Decode linear with static per-tensor quantization of bf16 X."""
    M, K = X.shape
    N = Wq.shape[0]
    out = torch.empty((M, N), dtype=out_dtype, device=X.device) if out is None else out
    ws, nbytes = _workspace(w8a8_gemm_workspace_size(M, N, K), X.device, workspace)
    _check("w8a8_linear_static", lib().w8a8_linear_static(
        _ptr(X), M, K, _ld(X), _ptr(S), _ptr(r), _ptr(Z), _ptr(Wq), _ptr(s_w), _ptr(colsum),
        _ptr(bias), N, _ptr(out), _dt(out.dtype), _ptr(ws), nbytes, _stream(stream)))
    return out


def w8a8_gemm_requant(Xq, S_x, Wq, s_w, r_out, Z_out, colsum=None, Z=None, bias=None, out=None, stream=None):
    """w8a8_gemm_dequant whose bf16 result is quantized at once with the next
    linear's static r_out, Z_out: returns int8 [M, N] (M <= 64)."""
    M, K = Xq.shape
    N = Wq.shape[0]
    _expect(Xq, torch.int8, (M, K), "Xq")
    _expect(Wq, torch.int8, (N, K), "Wq")
    out = torch.empty((M, N), dtype=torch.int8, device=Xq.device) if out is None else out
    _expect(out, torch.int8, (M, N), "out")
    if S_x.numel() not in (1, M):
        raise ValueError("S_x holds one scale per row or a single per-tensor scale")
    per_row = 1 if S_x.numel() == M else 0
    _check("w8a8_gemm_requant", lib().w8a8_gemm_requant(
        _ptr(Xq), _ptr(S_x), per_row, _ptr(Z), _ptr(Wq), _ptr(s_w), _ptr(colsum), _ptr(bias), M, N, K,
        _ptr(r_out), _ptr(Z_out), _ptr(out), _stream(stream)))
    return out


def w8a8_linear_static_requant(X, S, r, Z, Wq, s_w, colsum, r_out, Z_out, bias=None, out=None, workspace=None,
                               stream=None):
    """Decode linear whose bf16 result is quantized at once with the next
    linear's static r_out, Z_out: returns int8 [M, N] (M <= 64)."""
    M, K = X.shape
    N = Wq.shape[0]
    if X.dtype != torch.bfloat16:
        raise ValueError(f"X: expected bfloat16, got {X.dtype}")
    _expect(Wq, torch.int8, (N, K), "Wq")
    out = torch.empty((M, N), dtype=torch.int8, device=X.device) if out is None else out
    _expect(out, torch.int8, (M, N), "out")
    ws, nbytes = _workspace(w8a8_gemm_workspace_size(M, N, K), X.device, workspace)
    _check("w8a8_linear_static_requant", lib().w8a8_linear_static_requant(
        _ptr(X), M, K, _ld(X), _ptr(S), _ptr(r), _ptr(Z), _ptr(Wq), _ptr(s_w), _ptr(colsum), _ptr(bias), N,
        _ptr(r_out), _ptr(Z_out), _ptr(out), _ptr(ws), nbytes, _stream(stream)))
    return out


def w8a8_linear_static_noalloc(X, S, r, Z, Wq, s_w, colsum, bias=None, out=None, out_dtype=torch.bfloat16,
                               stream=None):
    """w8a8_linear_static with the library's own fixed scratch instead of a
    caller workspace (M <= 32, N <= 32768, K <= 16384)."""
    M, K = X.shape
    N = Wq.shape[0]
    out = torch.empty((M, N), dtype=out_dtype, device=X.device) if out is None else out
    _check("w8a8_linear_static_noalloc", lib().w8a8_linear_static_noalloc(
        _ptr(X), M, K, _ld(X), _ptr(S), _ptr(r), _ptr(Z), _ptr(Wq), _ptr(s_w), _ptr(colsum), _ptr(bias), N,
        _ptr(out), _dt(out.dtype), _stream(stream)))
    return out


def int8_outlier_split(X, threshold: float = 6.0, cap: int = 64, Xq=None, S_x=None, idx=None,
                       n_out=None, Xo=None, workspace=None, stream=None):
    """LLM.int8() split -> (Xq, S_x, outlier_idx [cap], n_out [1], Xo [M, cap])."""
    M, K = X.shape
    dev = X.device
    Xq = torch.empty((M, K), dtype=torch.int8, device=dev) if Xq is None else Xq
    S_x = torch.empty((M,), dtype=torch.float32, device=dev) if S_x is None else S_x
    idx = torch.empty((max(cap, 1),), dtype=torch.int32, device=dev) if idx is None else idx
    n_out = torch.empty((1,), dtype=torch.int32, device=dev) if n_out is None else n_out
    Xo = torch.empty((M, max(cap, 1)), dtype=torch.bfloat16, device=dev) if Xo is None else Xo
    ws, nbytes = _workspace(int(lib().int8_outlier_split_workspace_size(K)), dev, workspace)
    _check("int8_outlier_split", lib().int8_outlier_split(
        _ptr(X), M, K, _ld(X), float(threshold), int(cap), _ptr(Xq), _ptr(S_x), _ptr(idx), _ptr(n_out),
        _ptr(Xo), _ptr(ws), nbytes, _stream(stream)))
    return Xq, S_x, idx, n_out, Xo


def int8_mixed_decomp_gemm(Xq, S_x, Xo, idx, n_out, cap: int, Wq, s_w, W, bias=None, out=None,
                           out_dtype=torch.bfloat16, stream=None):
    """INT8 vector-wise product + bf16 outlier side product, summed in the epilogue."""
    M, K = Xq.shape
    N = Wq.shape[0]
    out = torch.empty((M, N), dtype=out_dtype, device=Xq.device) if out is None else out
    _check("int8_mixed_decomp_gemm", lib().int8_mixed_decomp_gemm(
        _ptr(Xq), _ptr(S_x), _ptr(Xo), _ptr(idx), _ptr(n_out), int(cap), _ptr(Wq), _ptr(s_w), _ptr(W),
        _ld(W), _ptr(bias), M, N, K, _ptr(out), _dt(out.dtype), _stream(stream)))
    return out


def w8a8_check_device_error(stream=None) -> int:
    """Synchronize the stream, return and clear the device status word."""
    st = ctypes.c_int32(0)
    _check("w8a8_check_device_error", lib().w8a8_check_device_error(_stream(stream), ctypes.byref(st)))
    return int(st.value)


def w8a8_debug_wait_timeout_selftest(limit_ns: int = 5_000_000, stream=None):
    _check("w8a8_debug_wait_timeout_selftest",
           lib().w8a8_debug_wait_timeout_selftest(int(limit_ns), _stream(stream)))
