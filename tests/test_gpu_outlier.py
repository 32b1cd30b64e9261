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


def planted(M, K, cols, seed, lo=20.0, hi=100.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
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


@pytest.mark.parametrize("M,K,cols,ld_pad", [
    (3, 16, [2, 9], 0), (16, 256, [7, 100, 255], 8), (300, 4112, [0, 33, 4095, 4111], 0),
    (129, 1024, [], 0), (2, 65536, [5, 65535], 0), (4096, 8192, [11, 512, 777, 4000, 6001, 8191], 0),
    (7, 24576, [100, 24575], 0), (1500, 16384, [3, 9000], 16), (20000, 512, [0, 511], 0)])
def test_outlier_split_bit_exact(M, K, cols, ld_pad):
    X = planted(M, K, cols, seed=M + K)
    n, st = check_split(X, 6.0, 64, ld_pad)
    assert n >= len(cols) and st == 0


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
                                        (520, 400, 5400, [5, 6, 390])])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_mixed_decomp_gemm_bit_exact(M, K, N, cols, out_dtype):
    X = planted(M, K, cols, seed=3 * M + K)
    Wb = synth.bf16_bits(synth.weight(np.random.default_rng(N + K), K, N))
    bias = synth.bias(np.random.default_rng(5), N)
    cap = 16
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


def test_llm_int8_full_size_sampled():
    """X [4096, 8192] with 6-8 planted outlier columns, W bf16 [8192, 8192]:
    the split is compared in full, the output on 96 x 96 sampled elements
    computed one by one by the oracle."""
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
    rng = np.random.default_rng(7)
    rows = np.sort(rng.choice(4096, 96, replace=False))
    cols = np.sort(rng.choice(8192, 96, replace=False))
    Wsub = np.ascontiguousarray(case.W[:, cols])
    rwq, rws, _ = oracle.quant_weight_per_channel(Wsub)   # per-channel: columns are independent
    acc = oracle.gemm_i64(rq[rows], rwq)
    side = oracle.outlier_side(rXo[rows], ridx, Wsub)
    y = oracle.epilogue(acc, rS[rows], rws, side=side)
    assert_same(host_bf16(out)[np.ix_(rows, cols)], oracle.f32_to_bf16(y), "sampled out")
    assert W.w8a8_check_device_error() == 0
