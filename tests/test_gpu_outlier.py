"""LLM.int8() mode on the GPU vs the CPU oracle: the outlier split (codes, row
scales, outlier indices and count, gathered 16-bit values: all bit for bit)
and the mixed-decomposition GEMM (bf16 and fp32 outputs compared exactly; the
epilogue and the 16-bit side product use the oracle's fp32 operations in the
oracle's order)."""
import numpy as np
import pytest
import torch

import oracle
from int8_gemm_token_b200 import synth
from int8_gemm_token_b200 import w8a8 as W
from tests.gpu_util import dev, dev_bf16, diff_report, host, host_bf16

pytestmark = pytest.mark.gpu


def assert_same(gpu, ref, what):
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    eq = (gpu.view(np.uint32) == ref.view(np.uint32)) if gpu.dtype == np.float32 else (gpu == ref)
    assert eq.all(), f"{what}: " + diff_report(gpu, ref)


def planted(M, K, cols, seed, lo=20.0, hi=100.0, clip=None):
    """N(0,1) [M, K] (optionally clipped to +-clip, so that only the planted
    columns can exceed a threshold above it) with `cols` replaced by random
    sign x U(lo, hi)."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    if clip is not None:
        x = np.clip(x, -clip, clip)
    mag = rng.uniform(lo, hi, size=(M, len(cols))).astype(np.float32)
    sign = np.where(rng.random((M, len(cols))) < 0.5, -1.0, 1.0).astype(np.float32)
    x[:, cols] = sign * mag
    return synth.bf16_bits(x)


def check_split(X, threshold, cap, ld_pad=0):
    M, K = X.shape
    Xd = dev_bf16(np.pad(X, ((0, 0), (0, ld_pad))))[:, :K]
    Xq, S_x, idx, n_out, Xo = W.int8_outlier_split(Xd, threshold, cap)
    st = W.w8a8_check_device_error()
    rq, rS, ridx, rn, rXo = oracle.outlier_split(X, threshold, cap)
    assert int(host(n_out)[0]) == rn
    nuse = min(rn, cap)
    assert_same(host(idx)[:nuse], ridx[:nuse], "outlier_idx")
    assert_same(host(Xq), rq, "Xq")
    assert_same(host(S_x), rS, "S_x")
    assert_same(host_bf16(Xo)[:, :nuse], rXo[:, :nuse], "Xo")
    return rn, st


@pytest.mark.parametrize("M,K", [(40, 4096), (300, 8192), (12, 2048)])
def test_split_tiny_rows(M, K):
    """Rows whose masked absmax is below 127/FLT_MAX (tiny values everywhere
    but in the outlier columns) quantize as zero rows, as in the oracle."""
    rng = np.random.default_rng(M + K)
    Xf = np.clip(rng.standard_normal((M, K), dtype=np.float32), -5.5, 5.5)
    tiny = np.array([1e-38, -1e-38, 3e-39, -9.2e-41, 0.0, -0.0, 2e-40, -5e-39], np.float32)
    Xf[2:6] = rng.choice(tiny, size=(4, K))
    cols = [3, K // 2 + 1, K - 1]
    Xf[:, cols] = 20.0
    X = synth.bf16_bits(Xf)
    n, st = check_split(X, 6.0, 16)
    assert n == len(cols) and st == 0


@pytest.mark.parametrize("M,K,cols,ld_pad", [
    (3, 16, [2, 9], 0), (16, 256, [7, 100, 255], 8), (300, 4112, [0, 33, 4095, 4111], 0),
    (129, 1024, [], 0), (2, 65536, [5, 65535], 0), (4096, 8192, [11, 512, 777, 4000, 6001, 8191], 0),
    (7, 24576, [100, 24575], 0), (1500, 16384, [3, 9000], 16), (20000, 512, [0, 511], 0)])
def test_outlier_split_bit_exact(M, K, cols, ld_pad):
    X = planted(M, K, cols, seed=M + K)
    n, st = check_split(X, 6.0, 64, ld_pad)
    assert n >= len(cols) and st == 0


@pytest.mark.parametrize("M,K", [(300, 4112), (4096, 8192), (7, 24576)])
def test_outlier_split_reuses_a_dirty_workspace(M, K):
    """The call clears its column bitmap itself: a workspace filled with ones,
    then two back-to-back splits with different outlier columns on that same
    workspace (the second launched while the first may still run), each equal
    to the oracle -- no flag may leak from the garbage or from the first call."""
    cols_a, cols_b = [0, 33, K - 1], [5, K // 2 + 1]
    Xa = planted(M, K, cols_a, seed=M + 1, clip=5.5)
    Xb = planted(M, K, cols_b, seed=M + 2, clip=5.5)
    cap = 8
    ws = torch.full((int(W.lib().int8_outlier_split_workspace_size(K)),), 255, dtype=torch.uint8, device="cuda")
    outs = [W.int8_outlier_split(dev_bf16(X), 6.0, cap, workspace=ws) for X in (Xa, Xb)]
    assert W.w8a8_check_device_error() == 0
    for X, cols, (Xq, S_x, idx, n_out, Xo) in zip((Xa, Xb), (cols_a, cols_b), outs):
        rq, rS, ridx, rn, rXo = oracle.outlier_split(X, 6.0, cap)
        assert rn == len(cols) and int(host(n_out)[0]) == rn
        assert_same(host(idx)[:rn], ridx[:rn], "outlier_idx")
        assert_same(host(Xq), rq, "Xq")
        assert_same(host(S_x), rS, "S_x")
        assert_same(host_bf16(Xo)[:, :rn], rXo[:, :rn], "Xo")


def test_outlier_split_thresholds_and_overflow():
    X = planted(64, 512, [3, 70, 300], seed=1)
    n, st = check_split(X, float("inf"), 16)
    assert n == 0 and st == 0
    n, st = check_split(X, 0.0, 512)       # every column with a nonzero entry
    assert n == 512 and st == 0
    n, st = check_split(X, 2.0, 8)         # more outlier columns than cap
    assert n > 8 and st == 7              # W8A8_ERR_OUTLIER_OVERFLOW recorded, then cleared
    assert W.w8a8_check_device_error() == 0
    # exactly-at-threshold values stay in the INT8 path (strict "exceeds")
    x = np.zeros((4, 32), np.float32)
    x[1, 5] = 6.0
    x[2, 9] = -6.5
    n, st = check_split(synth.bf16_bits(x), 6.0, 8)
    assert n == 1 and st == 0


@pytest.mark.parametrize("M,K,N,cols", [(16, 256, 512, [3, 200]), (300, 400, 520, [0, 399]),
                                        (129, 1024, 257, [17, 18, 19, 700, 1000, 1023]), (5, 128, 128, []),
                                        (32, 4096, 4096, [1, 2000, 4000]),
                                        (520, 400, 5400, [5, 6, 390]),
                                        # CTA-pair tiles past the 16 staged outlier rows: an odd N (row
                                        # stride not a multiple of 8 elements) and 17 at a ragged N
                                        (300, 1024, 1001, list(range(3, 1000, 50))),
                                        (260, 512, 520, [7 * i + 1 for i in range(17)]),
                                        # the same past 16 outliers in the single-CTA kernel (65..255 tokens)
                                        (100, 1024, 1001, list(range(5, 1000, 50)))])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_mixed_decomp_gemm_bit_exact(M, K, N, cols, out_dtype):
    X = planted(M, K, cols, seed=3 * M + K)
    Wb = synth.bf16_bits(synth.weight(np.random.default_rng(N + K), K, N))
    bias = synth.bias(np.random.default_rng(5), N)
    cap = 16 if len(cols) <= 16 else 32
    Wd = dev_bf16(Wb)
    Wq, s_w, _ = W.w8a8_quant_weight_per_channel(Wd)
    Xq, S_x, idx, n_out, Xo = W.int8_outlier_split(dev_bf16(X), 6.0, cap)
    out = W.int8_mixed_decomp_gemm(Xq, S_x, Xo, idx, n_out, cap, Wq, s_w, Wd, bias=dev(bias), out_dtype=out_dtype)
    rwq, rws, _ = oracle.quant_weight_per_channel(Wb)
    *_, y = oracle.linear_mixed(X, Wb, rwq, rws, threshold=6.0, cap=cap, bias=bias)
    if out_dtype == torch.bfloat16:
        assert_same(host_bf16(out), oracle.f32_to_bf16(y), "out")
    else:
        assert_same(host(out), y, "out")
    assert W.w8a8_check_device_error() == 0


def test_llm_int8_full_size():
    """X [4096, 8192] with 6-8 planted outlier columns, W bf16 [8192, 8192]:
    the split and every element of the mixed GEMM's output compared with the
    oracle (the INT8 product, the 16-bit side product and the epilogue over
    the whole layer)."""
    case = synth.llm_int8(0)
    cap = 64
    Wd = dev_bf16(case.W)
    Wq, s_w, _ = W.w8a8_quant_weight_per_channel(Wd)
    Xq, S_x, idx, n_out, Xo = W.int8_outlier_split(dev_bf16(case.X), case.threshold, cap)
    out = W.int8_mixed_decomp_gemm(Xq, S_x, Xo, idx, n_out, cap, Wq, s_w, Wd)
    rq, rS, ridx, rn, rXo = oracle.outlier_split(case.X, case.threshold, cap)
    assert rn >= len(case.cols) and set(case.cols.tolist()) <= set(ridx.tolist())
    assert int(host(n_out)[0]) == rn
    assert_same(host(idx)[:rn], ridx, "outlier_idx")
    assert_same(host(Xq), rq, "Xq")
    assert_same(host(S_x), rS, "S_x")
    assert_same(host_bf16(Xo)[:, :rn], rXo[:, :rn], "Xo")
    rwq, rws, _ = oracle.quant_weight_per_channel(case.W)
    assert_same(host(Wq), rwq, "Wq")
    assert_same(host(s_w), rws, "s_w")
    side = oracle.outlier_side(rXo, ridx, case.W)
    y = oracle.epilogue(oracle.gemm_i64(rq, rwq), rS, rws, side=side)
    assert_same(host_bf16(out), oracle.f32_to_bf16(y), "out")
    assert W.w8a8_check_device_error() == 0


# ------------------------------------------------------------ tensor-core side product
U = 2.0 ** -23  # one fp32 ulp at 1.0 (an upper bound on the unit roundoff under any rounding rule)


def side_tolerance(Xo_bits, idx, W_bits, side_ref, bias, y_ref):
    """Per-element bound on |y_tc - y_oracle| when only the summation order of
    the side product differs. The products Xo[m, j] W[idx[j], n] are exact
    in fp32, and any order of n additions in fp32 is within
    (n - 1) u sum_j |products| of the exact sum, so two orders differ by at
    most 2 n u S_abs (S_abs = sum_j |product|, in float64 here). The
    epilogue then rounds side + bias once and the fma once, which moves y by
    at most one ulp of each of those results more."""
    n = len(idx)
    xo = np.abs(oracle.bf16_to_f32(Xo_bits[:, :n]).astype(np.float64))
    w = np.abs(oracle.bf16_to_f32(W_bits[idx]).astype(np.float64))
    s_abs = xo @ w
    b = 0.0 if bias is None else np.abs(bias.astype(np.float64))[None, :]
    return U * (2 * n * s_abs + np.abs(side_ref) + b + 2 * np.abs(y_ref)) + 1e-30, s_abs


@pytest.mark.parametrize("M,K,N,n_cols,cap,with_bias", [
    (300, 1024, 520, 0, 16, True),      # no outlier: the side accumulator is never read
    (300, 1024, 520, 8, 8, True),       # one side k-block, mostly padding
    (129, 2048, 1000, 64, 64, False),   # exactly one full side k-block
    (520, 2048, 777, 65, 70, True),     # two k-blocks, Xo rows not 16-byte multiples (cap 70)
    (512, 2048, 1024, 512, 512, True),  # eight k-blocks through the double-buffered side ring
    (256, 8192, 512, 4096, 4096, False),  # the largest cap
    (16, 512, 300, 40, 48, True),       # fewer tokens than one pair tile
])
def test_mixed_decomp_gemm_tc_within_derived_bound(M, K, N, n_cols, cap, with_bias):
    rng = np.random.default_rng(M + K + n_cols)
    cols = np.sort(rng.choice(K, n_cols, replace=False)) if n_cols else np.array([], np.int64)
    X = planted(M, K, cols.tolist(), seed=7 * M + n_cols, clip=5.5)  # exactly the planted columns exceed 6
    Wb = synth.bf16_bits(synth.weight(np.random.default_rng(N + n_cols), K, N))
    bias = synth.bias(np.random.default_rng(9), N) if with_bias else None
    Wd = dev_bf16(Wb)
    Wq, s_w, _ = W.w8a8_quant_weight_per_channel(Wd)
    Xq, S_x, idx, n_out, Xo = W.int8_outlier_split(dev_bf16(X), 6.0, cap)
    b = None if bias is None else dev(bias)
    y32 = W.int8_mixed_decomp_gemm_tc(Xq, S_x, Xo, idx, n_out, cap, Wq, s_w, Wd, bias=b, out_dtype=torch.float32)
    y16 = W.int8_mixed_decomp_gemm_tc(Xq, S_x, Xo, idx, n_out, cap, Wq, s_w, Wd, bias=b)
    assert W.w8a8_check_device_error() == 0
    rq, rS, ridx, rn, rXo = oracle.outlier_split(X, 6.0, cap)
    assert rn == n_cols and int(host(n_out)[0]) == rn
    rwq, rws, _ = oracle.quant_weight_per_channel(Wb)
    side = oracle.outlier_side(rXo, ridx, Wb)
    y_ref = oracle.epilogue(oracle.gemm_i64(rq, rwq), rS, rws, bias=bias, side=side)
    got = host(y32)
    # the bf16 result is the fp32 result rounded once (same kernel, same order)
    assert_same(host_bf16(y16), oracle.f32_to_bf16(got), "bf16 out vs the fp32 out rounded")
    if n_cols == 0:  # no side product at all: the fixed-order epilogue, bit for bit
        assert_same(got, y_ref, "out")
        return
    tol, s_abs = side_tolerance(rXo, ridx, Wb, side, bias, y_ref)
    err = np.abs(got.astype(np.float64) - y_ref.astype(np.float64))
    bad = np.argwhere(err > tol)
    assert bad.size == 0, f"{len(bad)} elements outside the bound; first {bad[:3].tolist()}: " \
                          f"{[(got[tuple(i)], y_ref[tuple(i)], tol[tuple(i)]) for i in bad[:3]]}"
    # the target's 1e-3 relative error per element, wherever the side sum is
    # well conditioned (2 n u S_abs <= 1e-4 |y|); near cancellation no fp32
    # summation order, the oracle's included, is that close to the exact sum
    wc = 2 * n_cols * U * s_abs <= 1e-4 * np.abs(y_ref)
    assert (err[wc] <= 1e-3 * np.abs(y_ref[wc])).all()


def test_llm_int8_full_size_tensor_core_side():
    """The LLM.int8() workload (4096 x 8192 -> 8192, 6-8 outlier columns)
    through the tensor-core side product: every output element within the
    derived bound of the oracle."""
    case = synth.llm_int8(0)
    cap = 64
    Wd = dev_bf16(case.W)
    Wq, s_w, _ = W.w8a8_quant_weight_per_channel(Wd)
    Xq, S_x, idx, n_out, Xo = W.int8_outlier_split(dev_bf16(case.X), case.threshold, cap)
    y32 = W.int8_mixed_decomp_gemm_tc(Xq, S_x, Xo, idx, n_out, cap, Wq, s_w, Wd, out_dtype=torch.float32)
    assert W.w8a8_check_device_error() == 0
    rq, rS, ridx, rn, rXo = oracle.outlier_split(case.X, case.threshold, cap)
    rwq, rws, _ = oracle.quant_weight_per_channel(case.W)
    side = oracle.outlier_side(rXo, ridx, case.W)
    y_ref = oracle.epilogue(oracle.gemm_i64(rq, rwq), rS, rws, side=side)
    tol, _ = side_tolerance(rXo, ridx, case.W, side, None, y_ref)
    err = np.abs(host(y32).astype(np.float64) - y_ref.astype(np.float64))
    assert (err <= tol).all(), f"{int((err > tol).sum())} elements outside the bound"
