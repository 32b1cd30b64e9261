"""CPU oracle for the W8A8 linear layer (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline / reference arm import this package. The product library in
``int8_gemm_token_b200`` never imports it, and it imports nothing from there.

The arithmetic lives in ``w8a8_oracle.c`` (plain loops, fixed fp32 order,
round-half-even, int64 accumulation). This module only builds that file with
gcc, loads it with ctypes and moves numpy arrays in and out. Arrays of bf16
values are carried as ``numpy.uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "w8a8_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fopenmp", "-Wall", "-Wextra"]

DT_BF16 = 0
DT_FP32 = 1

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` with gcc."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # ORACLE_LIB_OVERRIDE lets the mutation test load a deliberately
            # broken build of the same source; nothing else sets it.
            lib = ctypes.CDLL(os.environ.get("ORACLE_LIB_OVERRIDE") or build())
            P, I64, I32, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float
            sig = {
                "oracle_quant_per_token": (None, [P, ctypes.c_int, I64, I64, I64, P, P]),
                "oracle_quant_weight_per_channel": (None, [P, ctypes.c_int, I64, I64, I64, P, P, P]),
                "oracle_calibrate_static": (None, [P, ctypes.c_int, I64, I64, I64, P, P, P]),
                "oracle_quant_per_tensor": (None, [P, ctypes.c_int, I64, I64, I64, F, I32, P]),
                "oracle_dequant_per_tensor": (None, [P, I64, I64, F, I32, ctypes.c_int, P]),
                "oracle_gemm_i64": (None, [P, P, I64, I64, I64, P]),
                "oracle_epilogue": (ctypes.c_int, [P, I64, I64, P, ctypes.c_int, P, P, P, P, P, P]),
                "oracle_f32_to_bf16_array": (None, [P, I64, P]),
                "oracle_outlier_split": (ctypes.c_int, [P, I64, I64, I64, F, I32, P, P, P, P, P]),
                "oracle_outlier_side": (None, [P, I64, I32, I32, P, P, I64, I64, P]),
                "oracle_round_mode_ok": (ctypes.c_int, []),
                "oracle_num_threads": (ctypes.c_int, []),
                "oracle_set_num_threads": (None, [ctypes.c_int]),
                "oracle_bf16_to_f32": (ctypes.c_float, [ctypes.c_uint16]),
                "oracle_f32_to_bf16": (ctypes.c_uint16, [ctypes.c_float]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            if not lib.oracle_round_mode_ok():
                raise RuntimeError("oracle requires round-to-nearest-even")
            _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return DT_BF16
    if a.dtype == np.float32:
        return DT_FP32
    raise TypeError(f"oracle takes bf16 bits (uint16) or float32, got {a.dtype}")


def _c(a: np.ndarray) -> np.ndarray:
    return np.ascontiguousarray(a)


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32 (a 16-bit shift)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(y: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even) in the oracle's C code."""
    y = _c(np.asarray(y, dtype=np.float32))
    out = np.empty(y.shape, dtype=np.uint16)
    _load().oracle_f32_to_bf16_array(_ptr(y), y.size, _ptr(out))
    return out


def quant_per_token(X: np.ndarray):
    """Per-token symmetric absmax quantization of X [M, K] -> (Xq int8 [M, K], S_x f32 [M])."""
    X = _c(X)
    M, K = X.shape
    Xq = np.empty((M, K), dtype=np.int8)
    S = np.empty((M,), dtype=np.float32)
    _load().oracle_quant_per_token(_ptr(X), _dtype_code(X), M, K, K, _ptr(Xq), _ptr(S))
    return Xq, S


def quant_weight_per_channel(W: np.ndarray):
    """W [K, N] (bf16 bits or f32) -> (Wq int8 [N, K], s_w f32 [N], colsum int32 [N])."""
    W = _c(W)
    K, N = W.shape
    Wq = np.empty((N, K), dtype=np.int8)
    s = np.empty((N,), dtype=np.float32)
    cs = np.empty((N,), dtype=np.int32)
    _load().oracle_quant_weight_per_channel(_ptr(W), _dtype_code(W), K, N, N, _ptr(Wq), _ptr(s), _ptr(cs))
    return Wq, s, cs


def calibrate_static(Xcal: np.ndarray):
    """MinMax calibration over all of Xcal [T, K] -> (S, r, Z) as numpy scalars."""
    Xcal = _c(Xcal)
    T, K = Xcal.shape
    S = np.zeros(1, np.float32)
    r = np.zeros(1, np.float32)
    Z = np.zeros(1, np.int32)
    _load().oracle_calibrate_static(_ptr(Xcal), _dtype_code(Xcal), T, K, K, _ptr(S), _ptr(r), _ptr(Z))
    return S[0], r[0], Z[0]


def quant_per_tensor(X: np.ndarray, r, Z):
    """Static asymmetric quantization q = clamp(rne(x*r) + Z, -128, 127)."""
    X = _c(X)
    M, K = X.shape
    Xq = np.empty((M, K), dtype=np.int8)
    _load().oracle_quant_per_tensor(_ptr(X), _dtype_code(X), M, K, K, float(np.float32(r)), int(Z), _ptr(Xq))
    return Xq


def dequant_per_tensor(Xq: np.ndarray, S, Z, out_dtype: int = DT_BF16) -> np.ndarray:
    """Static dequantization x = S * (q - Z): bf16 bits (DT_BF16) or float32."""
    Xq = _c(np.asarray(Xq, dtype=np.int8))
    M, K = Xq.shape
    out = np.empty((M, K), dtype=np.uint16 if out_dtype == DT_BF16 else np.float32)
    _load().oracle_dequant_per_tensor(_ptr(Xq), M, K, float(np.float32(S)), int(Z), int(out_dtype), _ptr(out))
    return out


def gemm_i64(Xq: np.ndarray, Wq: np.ndarray) -> np.ndarray:
    """acc[m, n] = sum_k Xq[m, k] * Wq[n, k] in int64."""
    Xq, Wq = _c(Xq), _c(Wq)
    M, K = Xq.shape
    N, K2 = Wq.shape
    assert K == K2
    acc = np.empty((M, N), dtype=np.int64)
    _load().oracle_gemm_i64(_ptr(Xq), _ptr(Wq), M, N, K, _ptr(acc))
    return acc


def epilogue(acc, S_x, s_w, colsum=None, Z=None, bias=None, side=None) -> np.ndarray:
    """fp32 y = fmaf(float(acc - Z*colsum), S_x*s_w, side + bias) in the fixed order."""
    acc = _c(np.asarray(acc, dtype=np.int64))
    M, N = acc.shape
    S_x = _c(np.atleast_1d(np.asarray(S_x, dtype=np.float32)))
    if S_x.size not in (1, M):
        raise ValueError("S_x is a scalar or one scale per row")
    per_row = 1 if S_x.size == M else 0
    s_w = _c(np.asarray(s_w, dtype=np.float32))
    z = None if Z is None else np.array([Z], dtype=np.int32)
    cs = None if colsum is None else _c(np.asarray(colsum, dtype=np.int32))
    if z is not None and cs is None:
        raise ValueError("a zero point needs colsum")
    b = None if bias is None else _c(np.asarray(bias, dtype=np.float32))
    sd = None if side is None else _c(np.asarray(side, dtype=np.float32))
    y = np.empty((M, N), dtype=np.float32)
    rc = _load().oracle_epilogue(_ptr(acc), M, N, _ptr(S_x), per_row, _ptr(z), _ptr(cs), _ptr(s_w),
                                 _ptr(b), _ptr(sd), _ptr(y))
    if rc != 0:
        raise OverflowError("corrected accumulator leaves the int32 range")
    return y


def outlier_split(X: np.ndarray, threshold: float = 6.0, cap: int = 64):
    """LLM.int8() outlier split of X [M, K] (bf16 bits).

    Returns (Xq int8 [M, K], S_x f32 [M], idx int32 [n_stored], n_out, Xo bf16 [M, cap]).
    """
    X = _c(np.asarray(X, dtype=np.uint16))
    M, K = X.shape
    Xq = np.empty((M, K), dtype=np.int8)
    S = np.empty((M,), dtype=np.float32)
    idx = np.full((max(cap, 1),), -1, dtype=np.int32)
    n = np.zeros(1, np.int32)
    Xo = np.zeros((M, max(cap, 1)), dtype=np.uint16)
    rc = _load().oracle_outlier_split(_ptr(X), M, K, K, float(threshold), int(cap), _ptr(Xq), _ptr(S),
                                      _ptr(idx), _ptr(n), _ptr(Xo))
    if rc == -3:
        raise MemoryError
    n_out = int(n[0])
    return Xq, S, idx[:min(n_out, cap)].copy(), n_out, Xo[:, :cap]


def outlier_side(Xo: np.ndarray, idx: np.ndarray, W: np.ndarray) -> np.ndarray:
    """side[m, n] = fmaf chain over ascending j of Xo[m, j] * W[idx[j], n]."""
    Xo = _c(np.asarray(Xo, dtype=np.uint16))
    W = _c(np.asarray(W, dtype=np.uint16))
    idx = _c(np.asarray(idx, dtype=np.int32))
    M, cap = Xo.shape
    K, N = W.shape
    side = np.empty((M, N), dtype=np.float32)
    _load().oracle_outlier_side(_ptr(Xo), M, int(idx.size), int(cap), _ptr(idx), _ptr(W), N, N, _ptr(side))
    return side


# --------------------------------------------------------------------------
# The whole layer, step by step, in the pages' order.
# --------------------------------------------------------------------------

def linear_prefill(X, Wq, s_w, bias=None):
    """PDMIX prefill: per-token symmetric quant, INT8 GEMM, dequant epilogue.

    Returns (Xq, S_x, acc, y_f32)."""
    Xq, S_x = quant_per_token(X)
    acc = gemm_i64(Xq, Wq)
    y = epilogue(acc, S_x, s_w, bias=bias)
    return Xq, S_x, acc, y


def linear_decode(X, r, Z, S, Wq, s_w, colsum, bias=None):
    """PDMIX decode: per-tensor static asymmetric quant, INT8 GEMM, zero-point
    corrected dequant. Returns (Xq, acc, y_f32)."""
    Xq = quant_per_tensor(X, r, Z)
    acc = gemm_i64(Xq, Wq)
    y = epilogue(acc, np.float32(S), s_w, colsum=colsum, Z=Z, bias=bias)
    return Xq, acc, y


def linear_decode_requant(X, r, Z, S, Wq, s_w, colsum, r_out, Z_out, bias=None):
    """PDMIX decode linear whose bf16 result is quantized for the next linear
    with that linear's static r_out, Z_out (PDMIX glossary §2.3 eq. Q_decode
    applied to the next layer's input). The result passes between layers as
    bf16, so the code is taken from the bf16-rounded value.

    Returns (Xq, acc, y_f32, y_bf16, Xq_out)."""
    Xq, acc, y = linear_decode(X, r, Z, S, Wq, s_w, colsum, bias=bias)
    y_bf16 = f32_to_bf16(y)
    Xq_out = quant_per_tensor(y_bf16, r_out, Z_out)
    return Xq, acc, y, y_bf16, Xq_out


def linear_mixed(X, W_bf16, Wq, s_w, threshold=6.0, cap=64, bias=None):
    """LLM.int8() vector-wise INT8 path plus the 16-bit outlier side path.

    Returns (Xq, S_x, idx, n_out, Xo, acc, side, y_f32)."""
    Xq, S_x, idx, n_out, Xo = outlier_split(X, threshold, cap)
    acc = gemm_i64(Xq, Wq)
    side = outlier_side(Xo[:, :max(cap, 1)], idx, W_bf16)
    y = epilogue(acc, S_x, s_w, bias=bias, side=side)
    return Xq, S_x, idx, n_out, Xo, acc, side, y

