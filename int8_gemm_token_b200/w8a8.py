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
    "int8_mixed_decomp_gemm_tc": (_I32, [_P, _P, _P, _P, _P, _I32, _P, _P, _P, _I64, _P, _I64, _I64, _I64, _P, _I32,
                                         _P, _SZ, _P]),
    "int8_mixed_decomp_gemm_tc_workspace_size": (_SZ, [_I64, _I64, _I32]),
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
    if t.dim() != 2 or (t.shape[1] > 1 and t.stride(1) != 1):
        raise ValueError("expected a 2-D tensor with contiguous rows")
    return t.stride(0)


def _expect(t: torch.Tensor, dtype, shape, what: str):
    """Raise before the C call when a tensor the C side takes as a raw
    pointer of a fixed type and dense layout is not that."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what}: expected a tensor, got {type(t).__name__}")
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{what}: expected a contiguous {dtype} tensor of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)}")


def _rows(t: torch.Tensor, dtype, what: str, shape=None) -> int:
    """A 2-D matrix of `dtype` whose rows are contiguous (any row stride);
    returns the row stride in elements."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what}: expected a tensor, got {type(t).__name__}")
    if t.dtype != dtype:
        raise ValueError(f"{what}: expected {dtype}, got {t.dtype}")
    if t.dim() != 2 or (t.shape[1] > 1 and t.stride(1) != 1):
        raise ValueError(f"{what}: expected a 2-D tensor with contiguous rows, got shape {tuple(t.shape)} "
                         f"strides {tuple(t.stride())}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{what}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.stride(0)


def _vec(t, dtype, n: int, what: str, optional: bool = False):
    """A dense vector of n elements (n = 1: a device scalar, shape (1,) or ())."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{what}: required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what}: expected a tensor, got {type(t).__name__}")
    if t.dtype != dtype or t.numel() != n or not t.is_contiguous() or t.dim() > 1:
        raise ValueError(f"{what}: expected a contiguous {dtype} vector of {n} element(s), "
                         f"got {t.dtype} {tuple(t.shape)}")


def _on_one_gpu(*ts):
    """Every tensor a CUDA tensor on the same device (checked after the
    shapes, so shape errors are reported first)."""
    devs = {t.device for t in ts if t is not None}
    if any(d.type != "cuda" for d in devs) or len(devs) > 1:
        raise ValueError(f"expected CUDA tensors on one device, got {sorted(str(d) for d in devs)}")


def _out(out, dtype, shape, dev, allowed, what="out"):
    if out is None:
        if dtype not in allowed:
            raise ValueError(f"{what}: dtype must be one of {allowed}, got {dtype}")
        return torch.empty(shape, dtype=dtype, device=dev)
    if out.dtype not in allowed:
        raise ValueError(f"{what}: dtype must be one of {allowed}, got {out.dtype}")
    _expect(out, out.dtype, shape, what)
    return out


_GEMM_OUT = (torch.bfloat16, torch.float32, torch.int32)


# --------------------------------------------------------------------------
# Entry points (same names as the C ABI)
# --------------------------------------------------------------------------

def w8a8_quant_weight_per_channel(W: torch.Tensor, Wq=None, s_w=None, colsum=None, stream=None):
    """W [K, N] bf16/fp32 -> (Wq int8 [N, K], s_w fp32 [N], colsum int32 [N])."""
    if W.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError(f"W: expected bfloat16 or float32, got {W.dtype}")
    ldw = _rows(W, W.dtype, "W")
    K, N = W.shape
    dev = W.device
    Wq = torch.empty((N, K), dtype=torch.int8, device=dev) if Wq is None else Wq
    s_w = torch.empty((N,), dtype=torch.float32, device=dev) if s_w is None else s_w
    colsum = torch.empty((N,), dtype=torch.int32, device=dev) if colsum is None else colsum
    _expect(Wq, torch.int8, (N, K), "Wq")
    _vec(s_w, torch.float32, N, "s_w")
    _vec(colsum, torch.int32, N, "colsum")
    _on_one_gpu(W, Wq, s_w, colsum)
    _check("w8a8_quant_weight_per_channel", lib().w8a8_quant_weight_per_channel(
        _ptr(W), _dt(W.dtype), K, N, ldw, _ptr(Wq), _ptr(s_w), _ptr(colsum), _stream(stream)))
    return Wq, s_w, colsum


def w8a8_calibrate_static(Xcal: torch.Tensor, S=None, r=None, Z=None, stream=None):
    """MinMax calibration over Xcal [T, K] -> device scalars (S, r, Z)."""
    if Xcal.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError(f"Xcal: expected bfloat16 or float32, got {Xcal.dtype}")
    ldx = _rows(Xcal, Xcal.dtype, "Xcal")
    T, K = Xcal.shape
    dev = Xcal.device
    S = torch.empty((1,), dtype=torch.float32, device=dev) if S is None else S
    r = torch.empty((1,), dtype=torch.float32, device=dev) if r is None else r
    Z = torch.empty((1,), dtype=torch.int32, device=dev) if Z is None else Z
    _vec(S, torch.float32, 1, "S")
    _vec(r, torch.float32, 1, "r")
    _vec(Z, torch.int32, 1, "Z")
    _on_one_gpu(Xcal, S, r, Z)
    _check("w8a8_calibrate_static", lib().w8a8_calibrate_static(
        _ptr(Xcal), _dt(Xcal.dtype), T, K, ldx, _ptr(S), _ptr(r), _ptr(Z), _stream(stream)))
    return S, r, Z


def w8a8_quant_per_token(X: torch.Tensor, Xq=None, S_x=None, stream=None):
    """bf16 X [M, K] -> (Xq int8 [M, K], S_x fp32 [M])."""
    ldx = _rows(X, torch.bfloat16, "X")
    M, K = X.shape
    Xq = torch.empty((M, K), dtype=torch.int8, device=X.device) if Xq is None else Xq
    S_x = torch.empty((M,), dtype=torch.float32, device=X.device) if S_x is None else S_x
    _expect(Xq, torch.int8, (M, K), "Xq")
    _vec(S_x, torch.float32, M, "S_x")
    _on_one_gpu(X, Xq, S_x)
    _check("w8a8_quant_per_token", lib().w8a8_quant_per_token(
        _ptr(X), M, K, ldx, _ptr(Xq), _ptr(S_x), _stream(stream)))
    return Xq, S_x


def w8a8_quant_per_tensor(X: torch.Tensor, r: torch.Tensor, Z: torch.Tensor, Xq=None, stream=None):
    """bf16 X [M, K] -> int8 codes clamp(rne(X r) + Z) [M, K]."""
    ldx = _rows(X, torch.bfloat16, "X")
    M, K = X.shape
    Xq = torch.empty((M, K), dtype=torch.int8, device=X.device) if Xq is None else Xq
    _expect(Xq, torch.int8, (M, K), "Xq")
    _vec(r, torch.float32, 1, "r")
    _vec(Z, torch.int32, 1, "Z")
    _on_one_gpu(X, Xq, r, Z)
    _check("w8a8_quant_per_tensor", lib().w8a8_quant_per_tensor(
        _ptr(X), M, K, ldx, _ptr(r), _ptr(Z), _ptr(Xq), _stream(stream)))
    return Xq


def w8a8_dequant_per_tensor(Xq: torch.Tensor, S: torch.Tensor, Z: torch.Tensor, out=None, out_dtype=torch.bfloat16,
                            stream=None):
    """int8 Xq [M, K] -> S * (Xq - Z) as bf16 or fp32 [M, K]."""
    if Xq.dtype != torch.int8:
        raise ValueError(f"Xq: expected int8 codes, got {Xq.dtype}")
    ldq = _rows(Xq, torch.int8, "Xq")
    M, K = Xq.shape
    out = _out(out, out_dtype, (M, K), Xq.device, (torch.bfloat16, torch.float32))
    _vec(S, torch.float32, 1, "S")
    _vec(Z, torch.int32, 1, "Z")
    _on_one_gpu(Xq, out, S, Z)
    _check("w8a8_dequant_per_tensor", lib().w8a8_dequant_per_tensor(
        _ptr(Xq), M, K, ldq, _ptr(S), _ptr(Z), _ptr(out), _dt(out.dtype),
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
    if ws is None:
        if n == 0:
            return None, 0
        ws = torch.empty((n,), dtype=torch.uint8, device=dev)
    if not ws.is_contiguous():
        raise ValueError("workspace: expected a contiguous tensor")
    return ws, ws.numel() * ws.element_size()


def _weight_operands(Wq, s_w, colsum, bias, K):
    """Wq int8 [N, K] dense, s_w fp32 [N], colsum int32 [N] (optional), bias fp32 [N] (optional)."""
    if Wq.dtype != torch.int8 or Wq.dim() != 2:
        raise ValueError(f"Wq: expected a 2-D int8 tensor, got {Wq.dtype} {tuple(Wq.shape)}")
    N = Wq.shape[0]
    _expect(Wq, torch.int8, (N, K), "Wq")
    _vec(s_w, torch.float32, N, "s_w")
    _vec(colsum, torch.int32, N, "colsum", optional=True)
    _vec(bias, torch.float32, N, "bias", optional=True)
    return N


def _scales(S_x, M):
    if S_x is None or S_x.numel() not in (1, M):
        raise ValueError("S_x holds one scale per row or a single per-tensor scale")
    _vec(S_x, torch.float32, S_x.numel(), "S_x")
    return 1 if S_x.numel() == M else 0  # M == 1: both readings give the same single scale


def w8a8_gemm_dequant(Xq, S_x, Wq, s_w, colsum=None, Z=None, bias=None, out=None,
                      out_dtype=torch.bfloat16, workspace=None, stream=None):
    """out [M, N] = S_x * s_w * (Xq Wq^T - Z * colsum) + bias.

    S_x is [M] (per token) or a 1-element tensor (per tensor)."""
    if Xq.dtype != torch.int8 or Xq.dim() != 2:
        raise ValueError(f"Xq: expected a 2-D int8 tensor, got {Xq.dtype} {tuple(Xq.shape)}")
    M, K = Xq.shape
    _expect(Xq, torch.int8, (M, K), "Xq")
    N = _weight_operands(Wq, s_w, colsum, bias, K)
    per_row = _scales(S_x, M)
    _vec(Z, torch.int32, 1, "Z", optional=True)
    if Z is not None and colsum is None:
        raise ValueError("colsum: required with a zero point Z")
    out = _out(out, out_dtype, (M, N), Xq.device, _GEMM_OUT)
    ws, nbytes = (None, 0) if workspace is None else _workspace(0, Xq.device, workspace)
    _on_one_gpu(Xq, S_x, Wq, s_w, colsum, Z, bias, out, ws)
    _check("w8a8_gemm_dequant", lib().w8a8_gemm_dequant(
        _ptr(Xq), _ptr(S_x), per_row, _ptr(Z), _ptr(Wq), _ptr(s_w), _ptr(colsum), _ptr(bias),
        M, N, K, _ptr(out), _dt(out.dtype), _ptr(ws), nbytes, _stream(stream)))
    return out


def _static_inputs(X, S, r, Z, Wq, s_w, colsum, bias):
    ldx = _rows(X, torch.bfloat16, "X")
    M, K = X.shape
    N = _weight_operands(Wq, s_w, colsum, bias, K)
    if colsum is None:
        raise ValueError("colsum: required (the zero-point correction)")
    _vec(S, torch.float32, 1, "S")
    _vec(r, torch.float32, 1, "r")
    _vec(Z, torch.int32, 1, "Z")
    return ldx, M, K, N


def w8a8_linear_static(X, S, r, Z, Wq, s_w, colsum, bias=None, out=None, out_dtype=torch.bfloat16,
                       workspace=None, stream=None):
    """Fused Decode linear with static per-tensor quantization of bf16 X."""
    ldx, M, K, N = _static_inputs(X, S, r, Z, Wq, s_w, colsum, bias)
    out = _out(out, out_dtype, (M, N), X.device, _GEMM_OUT)
    ws, nbytes = _workspace(w8a8_gemm_workspace_size(M, N, K), X.device, workspace)
    _on_one_gpu(X, S, r, Z, Wq, s_w, colsum, bias, out, ws)
    _check("w8a8_linear_static", lib().w8a8_linear_static(
        _ptr(X), M, K, ldx, _ptr(S), _ptr(r), _ptr(Z), _ptr(Wq), _ptr(s_w), _ptr(colsum),
        _ptr(bias), N, _ptr(out), _dt(out.dtype), _ptr(ws), nbytes, _stream(stream)))
    return out


def w8a8_gemm_requant(Xq, S_x, Wq, s_w, r_out, Z_out, colsum=None, Z=None, bias=None, out=None, stream=None):
    """w8a8_gemm_dequant whose bf16 result is quantized at once with the next
    linear's static r_out, Z_out: returns int8 [M, N] (M <= 64)."""
    if Xq.dtype != torch.int8 or Xq.dim() != 2:
        raise ValueError(f"Xq: expected a 2-D int8 tensor, got {Xq.dtype} {tuple(Xq.shape)}")
    M, K = Xq.shape
    _expect(Xq, torch.int8, (M, K), "Xq")
    N = _weight_operands(Wq, s_w, colsum, bias, K)
    per_row = _scales(S_x, M)
    _vec(Z, torch.int32, 1, "Z", optional=True)
    if Z is not None and colsum is None:
        raise ValueError("colsum: required with a zero point Z")
    _vec(r_out, torch.float32, 1, "r_out")
    _vec(Z_out, torch.int32, 1, "Z_out")
    out = _out(out, torch.int8, (M, N), Xq.device, (torch.int8,))
    _on_one_gpu(Xq, S_x, Wq, s_w, colsum, Z, bias, r_out, Z_out, out)
    _check("w8a8_gemm_requant", lib().w8a8_gemm_requant(
        _ptr(Xq), _ptr(S_x), per_row, _ptr(Z), _ptr(Wq), _ptr(s_w), _ptr(colsum), _ptr(bias), M, N, K,
        _ptr(r_out), _ptr(Z_out), _ptr(out), _stream(stream)))
    return out


def w8a8_linear_static_requant(X, S, r, Z, Wq, s_w, colsum, r_out, Z_out, bias=None, out=None, workspace=None,
                               stream=None):
    """Decode linear whose bf16 result is quantized at once with the next
    linear's static r_out, Z_out: returns int8 [M, N] (M <= 64)."""
    ldx, M, K, N = _static_inputs(X, S, r, Z, Wq, s_w, colsum, bias)
    _vec(r_out, torch.float32, 1, "r_out")
    _vec(Z_out, torch.int32, 1, "Z_out")
    out = _out(out, torch.int8, (M, N), X.device, (torch.int8,))
    ws, nbytes = _workspace(w8a8_gemm_workspace_size(M, N, K), X.device, workspace)
    _on_one_gpu(X, S, r, Z, Wq, s_w, colsum, bias, r_out, Z_out, out, ws)
    _check("w8a8_linear_static_requant", lib().w8a8_linear_static_requant(
        _ptr(X), M, K, ldx, _ptr(S), _ptr(r), _ptr(Z), _ptr(Wq), _ptr(s_w), _ptr(colsum), _ptr(bias), N,
        _ptr(r_out), _ptr(Z_out), _ptr(out), _ptr(ws), nbytes, _stream(stream)))
    return out


def w8a8_linear_static_noalloc(X, S, r, Z, Wq, s_w, colsum, bias=None, out=None, out_dtype=torch.bfloat16,
                               stream=None):
    """w8a8_linear_static with the library's own fixed scratch instead of a
    caller workspace (M <= 32, N <= 32768, K <= 16384)."""
    ldx, M, K, N = _static_inputs(X, S, r, Z, Wq, s_w, colsum, bias)
    out = _out(out, out_dtype, (M, N), X.device, _GEMM_OUT)
    _on_one_gpu(X, S, r, Z, Wq, s_w, colsum, bias, out)
    _check("w8a8_linear_static_noalloc", lib().w8a8_linear_static_noalloc(
        _ptr(X), M, K, ldx, _ptr(S), _ptr(r), _ptr(Z), _ptr(Wq), _ptr(s_w), _ptr(colsum), _ptr(bias), N,
        _ptr(out), _dt(out.dtype), _stream(stream)))
    return out


def int8_outlier_split(X, threshold: float = 6.0, cap: int = 64, Xq=None, S_x=None, idx=None,
                       n_out=None, Xo=None, workspace=None, stream=None):
    """LLM.int8() split -> (Xq, S_x, outlier_idx [cap], n_out [1], Xo [M, cap])."""
    ldx = _rows(X, torch.bfloat16, "X")
    M, K = X.shape
    cap = int(cap)
    dev = X.device
    Xq = torch.empty((M, K), dtype=torch.int8, device=dev) if Xq is None else Xq
    S_x = torch.empty((M,), dtype=torch.float32, device=dev) if S_x is None else S_x
    idx = torch.empty((max(cap, 1),), dtype=torch.int32, device=dev) if idx is None else idx
    n_out = torch.empty((1,), dtype=torch.int32, device=dev) if n_out is None else n_out
    Xo = torch.empty((M, max(cap, 1)), dtype=torch.bfloat16, device=dev) if Xo is None else Xo
    _expect(Xq, torch.int8, (M, K), "Xq")
    _vec(S_x, torch.float32, M, "S_x")
    _vec(n_out, torch.int32, 1, "n_out")
    if idx.dtype != torch.int32 or idx.numel() < cap or not idx.is_contiguous():
        raise ValueError(f"idx: expected a contiguous int32 tensor of at least {cap} elements")
    _expect(Xo, torch.bfloat16, (M, max(cap, 1)), "Xo")
    ws, nbytes = _workspace(int(lib().int8_outlier_split_workspace_size(K)), dev, workspace)
    _on_one_gpu(X, Xq, S_x, idx, n_out, Xo, ws)
    _check("int8_outlier_split", lib().int8_outlier_split(
        _ptr(X), M, K, ldx, float(threshold), cap, _ptr(Xq), _ptr(S_x), _ptr(idx), _ptr(n_out),
        _ptr(Xo), _ptr(ws), nbytes, _stream(stream)))
    return Xq, S_x, idx, n_out, Xo


def _mixed(fn, Xq, S_x, Xo, idx, n_out, cap, Wq, s_w, W, bias, out, out_dtype, stream, workspace=None):
    if Xq.dtype != torch.int8 or Xq.dim() != 2:
        raise ValueError(f"Xq: expected a 2-D int8 tensor, got {Xq.dtype} {tuple(Xq.shape)}")
    M, K = Xq.shape
    cap = int(cap)
    _expect(Xq, torch.int8, (M, K), "Xq")
    N = _weight_operands(Wq, s_w, None, bias, K)
    _vec(S_x, torch.float32, M, "S_x")
    _expect(Xo, torch.bfloat16, (M, max(cap, 1)), "Xo")
    if idx.dtype != torch.int32 or idx.numel() < cap or not idx.is_contiguous():
        raise ValueError(f"idx: expected a contiguous int32 tensor of at least {cap} elements")
    _vec(n_out, torch.int32, 1, "n_out")
    ldw = _rows(W, torch.bfloat16, "W", shape=(K, N))
    out = _out(out, out_dtype, (M, N), Xq.device, (torch.bfloat16, torch.float32))
    args = [_ptr(Xq), _ptr(S_x), _ptr(Xo), _ptr(idx), _ptr(n_out), cap, _ptr(Wq), _ptr(s_w), _ptr(W),
            ldw, _ptr(bias), M, N, K, _ptr(out), _dt(out.dtype)]
    ws = None
    if fn == "int8_mixed_decomp_gemm_tc":
        ws, nbytes = _workspace(int(lib().int8_mixed_decomp_gemm_tc_workspace_size(M, N, cap)), Xq.device, workspace)
        args += [_ptr(ws), nbytes]
    _on_one_gpu(Xq, S_x, Xo, idx, n_out, Wq, s_w, W, bias, out, ws)
    _check(fn, getattr(lib(), fn)(*args, _stream(stream)))
    return out


def int8_mixed_decomp_gemm(Xq, S_x, Xo, idx, n_out, cap: int, Wq, s_w, W, bias=None, out=None,
                           out_dtype=torch.bfloat16, stream=None):
    """INT8 vector-wise product + bf16 outlier side product (fixed-order fmaf
    chain on CUDA cores), summed in the epilogue."""
    return _mixed("int8_mixed_decomp_gemm", Xq, S_x, Xo, idx, n_out, cap, Wq, s_w, W, bias, out, out_dtype, stream)


def int8_mixed_decomp_gemm_tc(Xq, S_x, Xo, idx, n_out, cap: int, Wq, s_w, W, bias=None, out=None,
                              out_dtype=torch.bfloat16, workspace=None, stream=None):
    """The same decomposition with the bf16 side product on the tensor cores
    (kind::f16 MMAs into a second TMEM accumulator); `workspace` (allocated
    when None) holds the padded side operands."""
    return _mixed("int8_mixed_decomp_gemm_tc", Xq, S_x, Xo, idx, n_out, cap, Wq, s_w, W, bias, out, out_dtype,
                  stream, workspace)


def w8a8_check_device_error(stream=None) -> int:
    """Synchronize the stream, return and clear the device status word."""
    st = ctypes.c_int32(0)
    _check("w8a8_check_device_error", lib().w8a8_check_device_error(_stream(stream), ctypes.byref(st)))
    return int(st.value)


def w8a8_debug_wait_timeout_selftest(limit_ns: int = 5_000_000, stream=None):
    _check("w8a8_debug_wait_timeout_selftest",
           lib().w8a8_debug_wait_timeout_selftest(int(limit_ns), _stream(stream)))
