"""The C ABI on a host without a GPU: the library loads, exports every symbol
include/w8a8.h declares, and rejects bad arguments on the host before any
CUDA call (fake pointers are never dereferenced)."""
import ctypes
import subprocess

import pytest
import torch

from int8_gemm_token_b200 import w8a8

GOOD = 0x10000  # a 16-byte aligned fake device address (never dereferenced)
ODD = 0x10008


@pytest.fixture(scope="module")
def L():
    return w8a8.lib()


def test_every_declared_symbol_is_exported(L):
    names = w8a8.header_symbols()
    assert len(names) >= 13
    out = subprocess.run(["nm", "-D", "--defined-only", w8a8.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(L, n)
    assert set(w8a8._SIGNATURES) == set(names)


def test_status_strings(L):
    for code, name in [(0, "W8A8_OK"), (1, "W8A8_ERR_INVALID_ARG"), (2, "W8A8_ERR_MISALIGNED"),
                       (3, "W8A8_ERR_UNSUPPORTED_SHAPE"), (4, "W8A8_ERR_UNSUPPORTED_DTYPE"),
                       (6, "W8A8_ERR_DEVICE_TIMEOUT"), (7, "W8A8_ERR_OUTLIER_OVERFLOW"),
                       (9, "W8A8_ERR_WORKSPACE"), (10, "W8A8_ERR_NO_DEVICE"), (1234, "W8A8_ERR_UNKNOWN")]:
        assert w8a8.status_string(code) == name


def test_quant_per_token_host_checks(L):
    f = L.w8a8_quant_per_token
    assert f(GOOD, 4, 15, 16, GOOD, GOOD, None) == 3          # K not a multiple of 16
    assert f(GOOD, 4, 65536 + 16, 65552, GOOD, GOOD, None) == 3
    assert f(GOOD, 4, 0, 16, GOOD, GOOD, None) == 1
    assert f(GOOD, -1, 16, 16, GOOD, GOOD, None) == 1
    assert f(GOOD, 4, 32, 16, GOOD, GOOD, None) == 1          # ldx < K
    assert f(None, 4, 32, 32, GOOD, GOOD, None) == 1
    assert f(ODD, 4, 32, 32, GOOD, GOOD, None) == 2
    assert f(GOOD, 4, 32, 36, GOOD, GOOD, None) == 2          # rows not 16-byte aligned
    assert f(GOOD, 4, 32, 32, None, GOOD, None) == 1
    assert f(GOOD, 0, 32, 32, None, None, None) == 0          # empty: nothing to do


def test_gemm_host_checks(L):
    f = L.w8a8_gemm_dequant
    args = dict(Xq=GOOD, S_x=GOOD, per_row=1, Z=None, Wq=GOOD, s_w=GOOD, colsum=None, bias=None,
                M=8, N=8, K=64, out=GOOD, dt=0, ws=None, wsb=0, stream=None)

    def call(**kw):
        a = dict(args, **kw)
        return f(*a.values())
    assert call(K=40) == 3
    assert call(dt=7) == 4
    assert call(Wq=None) == 1
    assert call(Z=GOOD, colsum=None) == 1
    assert call(out=ODD) == 2
    assert call(bias=ODD) == 2
    assert call(M=0) == 0 and call(N=0) == 0
    assert call(M=-2) == 1


def test_linear_static_workspace_check(L):
    f = L.w8a8_linear_static
    # X, M, K, ldx, S, r, Z, Wq, s_w, colsum, bias, N, out, dt, ws, wsb, stream
    # more than 32 tokens: the quantized activation needs M*K bytes of workspace
    assert f(GOOD, 40, 64, 64, GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, None, 8, GOOD, 0, None, 0, None) == 9
    assert f(GOOD, 40, 64, 64, GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, None, 8, GOOD, 0, GOOD, 40 * 64 - 1, None) == 9
    assert f(GOOD, 4, 64, 64, GOOD, GOOD, None, GOOD, GOOD, GOOD, None, 8, GOOD, 0, GOOD, 4096, None) == 1


def test_requant_entry_points_host_checks(L):
    f = L.w8a8_linear_static_requant
    # X, M, K, ldx, S, r, Z, Wq, s_w, colsum, bias, N, r_out, Z_out, Xq_out, ws, wsb, stream
    base = [GOOD, 8, 64, 64, GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, None, 8, GOOD, GOOD, GOOD, None, 0, None]

    def call(**kw):
        a = list(base)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return f(*a)
    assert call(a1=65) == 3                      # Decode-shaped only: M <= 64
    assert call(a1=0) == 0 and call(a11=0) == 0
    assert call(a12=None) == 1 and call(a13=None) == 1 and call(a14=None) == 1
    assert call(a14=ODD) == 2
    assert call(a1=40) == 9                      # 40 tokens: the workspace holds the quantized activation
    g = L.w8a8_gemm_requant
    # Xq, S_x, per_row, Z, Wq, s_w, colsum, bias, M, N, K, r_out, Z_out, Xq_out, stream
    assert g(GOOD, GOOD, 0, GOOD, GOOD, GOOD, GOOD, None, 65, 8, 64, GOOD, GOOD, GOOD, None) == 3
    assert g(GOOD, GOOD, 0, GOOD, GOOD, GOOD, GOOD, None, 8, 8, 40, GOOD, GOOD, GOOD, None) == 3
    assert g(GOOD, GOOD, 0, GOOD, GOOD, GOOD, GOOD, None, 8, 8, 64, None, GOOD, GOOD, None) == 1
    assert g(GOOD, GOOD, 0, GOOD, GOOD, GOOD, None, None, 8, 8, 64, GOOD, GOOD, GOOD, None) == 1  # Z without colsum
    assert g(GOOD, GOOD, 0, GOOD, GOOD, GOOD, GOOD, None, 8, 8, 64, GOOD, GOOD, ODD, None) == 2
    assert g(GOOD, GOOD, 0, GOOD, GOOD, GOOD, GOOD, None, 0, 8, 64, GOOD, GOOD, GOOD, None) == 0


def test_other_entry_points_host_checks(L):
    assert L.w8a8_quant_weight_per_channel(GOOD, 5, 64, 8, 8, GOOD, GOOD, GOOD, None) == 4
    assert L.w8a8_quant_weight_per_channel(GOOD, 1, 64, 8, 4, GOOD, GOOD, GOOD, None) == 1
    assert L.w8a8_quant_weight_per_channel(GOOD + 1, 0, 64, 3, 3, GOOD, GOOD, GOOD, None) == 2  # odd bf16 address
    assert L.w8a8_quant_weight_per_channel(GOOD, 0, 64, 3, 3, GOOD + 4, GOOD, GOOD, None) == 2  # Wq rows
    assert L.w8a8_calibrate_static(GOOD, 0, 0, 16, 16, GOOD, GOOD, GOOD, None) == 1
    assert L.w8a8_calibrate_static(GOOD, 3, 4, 16, 16, GOOD, GOOD, GOOD, None) == 4
    assert L.w8a8_quant_per_tensor(GOOD, 4, 64, 64, None, GOOD, GOOD, None) == 1
    # Xq, M, K, ldq, S, Z, out, out_dtype, stream
    assert L.w8a8_dequant_per_tensor(GOOD, 4, 40, 48, GOOD, GOOD, GOOD, 0, None) == 3    # K not a multiple of 16
    assert L.w8a8_dequant_per_tensor(GOOD, 4, 64, 48, GOOD, GOOD, GOOD, 0, None) == 1    # ldq < K
    assert L.w8a8_dequant_per_tensor(GOOD, 4, 64, 72, GOOD, GOOD, GOOD, 0, None) == 2    # rows not 16-byte aligned
    assert L.w8a8_dequant_per_tensor(GOOD, 4, 64, 64, GOOD, GOOD, GOOD, 2, None) == 4    # no int32 output
    assert L.w8a8_dequant_per_tensor(GOOD, 4, 64, 64, None, GOOD, GOOD, 0, None) == 1
    assert L.w8a8_dequant_per_tensor(GOOD, 4, 64, 64, GOOD, GOOD, ODD, 1, None) == 2
    assert L.w8a8_dequant_per_tensor(None, 0, 64, 64, None, None, None, 0, None) == 0
    assert L.int8_mixed_decomp_gemm(GOOD, GOOD, GOOD, GOOD, GOOD, 8, GOOD, GOOD, GOOD, 8, None,
                                    8, 8, 64, GOOD, 2, None) == 4  # int32 output not offered here
    assert L.int8_mixed_decomp_gemm(GOOD, GOOD, GOOD, GOOD, GOOD, 5000, GOOD, GOOD, GOOD, 8, None,
                                    8, 8, 64, GOOD, 0, None) == 1
    # X, M, K, ldx, S, r, Z, Wq, s_w, colsum, bias, N, out, dt, stream
    assert L.w8a8_linear_static_noalloc(GOOD, 33, 64, 64, GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, None, 8, GOOD, 0, None) == 3
    assert L.w8a8_linear_static_noalloc(GOOD, 4, 16400, 16400, GOOD, GOOD, GOOD, GOOD, GOOD, GOOD, None, 8, GOOD, 0, None) == 3
    assert L.w8a8_linear_static_noalloc(GOOD, 4, 64, 64, GOOD, GOOD, None, GOOD, GOOD, GOOD, None, 8, GOOD, 0, None) == 1
    assert L.w8a8_debug_wait_timeout_selftest(10, None) == 1
    st = ctypes.c_int32(0)
    assert L.w8a8_check_device_error(None, None) == 1


def test_valid_call_without_a_gpu_reports_no_device(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert L.w8a8_quant_per_token(GOOD, 4, 32, 32, GOOD, GOOD, None) == 10
    assert L.w8a8_gemm_requant(GOOD, GOOD, 0, GOOD, GOOD, GOOD, GOOD, None, 8, 8, 64, GOOD, GOOD, GOOD, None) == 10
    assert w8a8.w8a8_gemm_workspace_size(4, 8, 64) == 0  # one kernel: quantized inside the GEMM
    assert w8a8.w8a8_gemm_workspace_size(32, 4096, 64) == 0
    assert w8a8.w8a8_gemm_workspace_size(32, 4104, 64) >= 32 * 64  # quantization kernel first
    assert w8a8.w8a8_gemm_workspace_size(48, 100, 64) >= 48 * 64  # 33..64 tokens: quantization kernel first
    assert w8a8.w8a8_gemm_workspace_size(64, 8, 64) >= 64 * 64
    assert w8a8.lib().int8_outlier_split_workspace_size(8192) >= 8192 // 8


def test_binding_rejects_wrong_output_types_before_the_c_call():
    """The requantizing and dequantizing entry points take raw int8 / bf16 /
    fp32 pointers; the binding refuses a tensor of another type or shape
    before calling into the library (CPU tensors: nothing reaches a GPU)."""
    import torch
    Xq = torch.zeros((4, 32), dtype=torch.int8)
    Wq = torch.zeros((8, 32), dtype=torch.int8)
    s = torch.ones(1)
    z = torch.zeros(1, dtype=torch.int32)
    with pytest.raises(ValueError):
        w8a8.w8a8_gemm_requant(Xq, s, Wq, torch.ones(8), s, z, out=torch.zeros((4, 8), dtype=torch.float32))
    with pytest.raises(ValueError):
        w8a8.w8a8_gemm_requant(Xq, s, Wq, torch.ones(8), s, z, out=torch.zeros((4, 9), dtype=torch.int8))
    with pytest.raises(ValueError):
        w8a8.w8a8_gemm_requant(Xq.float(), s, Wq, torch.ones(8), s, z)
    with pytest.raises(ValueError):
        w8a8.w8a8_linear_static_requant(torch.zeros((4, 32)), s, s, z, Wq, torch.ones(8), torch.zeros(8), s, z)
    with pytest.raises(ValueError):
        w8a8.w8a8_dequant_per_tensor(Xq.to(torch.int32), s, z)
    with pytest.raises(ValueError):
        w8a8.w8a8_dequant_per_tensor(Xq, s, z, out=torch.zeros((4, 32), dtype=torch.int32))


def _decode_args(M=4, N=8, K=32):
    """Well-formed CPU tensors for the Decode linear (shapes and dtypes only)."""
    return dict(X=torch.zeros((M, K), dtype=torch.bfloat16), S=torch.ones(1), r=torch.ones(1),
                Z=torch.zeros(1, dtype=torch.int32), Wq=torch.zeros((N, K), dtype=torch.int8),
                s_w=torch.ones(N), colsum=torch.zeros(N, dtype=torch.int32), bias=torch.zeros(N))


@pytest.mark.parametrize("fn", ["w8a8_linear_static", "w8a8_linear_static_noalloc"])
@pytest.mark.parametrize("bad,what", [
    (dict(out=torch.zeros((4, 7), dtype=torch.bfloat16)), "out"),       # out smaller than [M, N]
    (dict(out=torch.zeros((4, 8), dtype=torch.float16)), "out"),        # dtype the C side has no code for
    (dict(s_w=torch.ones(7)), "s_w"),                                   # shorter than N
    (dict(colsum=torch.zeros(8, dtype=torch.int64)), "colsum"),
    (dict(colsum=torch.zeros(7, dtype=torch.int32)), "colsum"),
    (dict(bias=torch.zeros(7)), "bias"),
    (dict(bias=torch.zeros(8, dtype=torch.float64)), "bias"),
    (dict(X=torch.zeros((4, 32), dtype=torch.float32)), "X"),
    (dict(X=torch.zeros((32, 4), dtype=torch.bfloat16).t()), "X"),     # rows not contiguous
    (dict(Wq=torch.zeros((8, 16), dtype=torch.int8)), "Wq"),           # K differs from X's
    (dict(Wq=torch.zeros((8, 32), dtype=torch.uint8)), "Wq"),
    (dict(S=torch.ones(2)), "S"),
    (dict(r=torch.ones(1, dtype=torch.float64)), "r"),
    (dict(Z=torch.zeros(1, dtype=torch.int64)), "Z"),
])
def test_binding_rejects_bad_tensors_before_the_c_call(fn, bad, what):
    """Every tensor the C side takes as a raw pointer of a fixed type and
    extent is checked in the binding: a wrong shape or dtype raises
    ValueError naming the argument, before anything is launched."""
    a = _decode_args()
    bad = dict(bad)
    out = bad.pop("out", None)
    a.update(bad)
    with pytest.raises(ValueError, match=what):
        getattr(w8a8, fn)(a["X"], a["S"], a["r"], a["Z"], a["Wq"], a["s_w"], a["colsum"], bias=a["bias"], out=out)


def test_binding_rejects_host_tensors_and_bad_gemm_operands():
    a = _decode_args()
    with pytest.raises(ValueError, match="CUDA"):   # well-formed, but host memory
        w8a8.w8a8_linear_static(a["X"], a["S"], a["r"], a["Z"], a["Wq"], a["s_w"], a["colsum"])
    Xq = torch.zeros((4, 32), dtype=torch.int8)
    with pytest.raises(ValueError, match="S_x"):
        w8a8.w8a8_gemm_dequant(Xq, torch.ones(3), a["Wq"], a["s_w"])
    with pytest.raises(ValueError, match="colsum"):
        w8a8.w8a8_gemm_dequant(Xq, torch.ones(4), a["Wq"], a["s_w"], Z=a["Z"])
    with pytest.raises(ValueError, match="out"):
        w8a8.w8a8_gemm_dequant(Xq, torch.ones(4), a["Wq"], a["s_w"], out=torch.zeros((4, 8), dtype=torch.int8))
    with pytest.raises(ValueError, match="W"):
        w8a8.int8_mixed_decomp_gemm(Xq, torch.ones(4), torch.zeros((4, 16), dtype=torch.bfloat16),
                                    torch.zeros(16, dtype=torch.int32), torch.zeros(1, dtype=torch.int32), 16,
                                    a["Wq"], a["s_w"], torch.zeros((32, 7), dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="Xo"):
        w8a8.int8_outlier_split(a["X"], 6.0, 16, Xo=torch.zeros((4, 8), dtype=torch.bfloat16))
