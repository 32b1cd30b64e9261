"""Seeded random shapes across the kernels' dispatch ranges, compared with the
oracle bit for bit.

The hand-picked cases elsewhere sit on tile edges and on the switches between
kernels; these draw their sizes instead: the Prefill linear (per-token
quantization, then the INT8 GEMM with its dequant epilogue) for 1 to 600 rows,
which spans the Decode-shaped, the 1-CTA and the CTA-pair kernels; the Decode
linear with static quantization for 1 to 64 rows (the one-kernel and the
two-kernel forms); the LLM.int8() split followed by the CUDA-core mixed GEMM
with 0 to 20 outlier columns; and the tensor-core side product with 0 to 100,
held to its derived per-element bound.
"""
import numpy as np
import pytest
import torch

import oracle
from int8_gemm_token_b200 import synth
from int8_gemm_token_b200 import w8a8 as W
from tests.gpu_util import dev, dev_bf16, diff_report, host, host_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_status():
    yield
    assert W.w8a8_check_device_error() == 0


def assert_same(gpu, ref, what):
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    if gpu.dtype == np.float32:
        eq = gpu.view(np.uint32) == ref.view(np.uint32)
    else:
        eq = gpu == ref
    assert eq.all(), f"{what}: " + diff_report(gpu, ref)


def draw(seed, m_hi, n_hi, k_hi):
    """(rng, M, N, K): M in [1, m_hi], N in [1, n_hi], K a multiple of 16 in [16, k_hi]."""
    rng = np.random.default_rng(7000 + seed)
    M = int(rng.integers(1, m_hi + 1))
    N = int(rng.integers(1, n_hi + 1))
    K = 16 * int(rng.integers(1, k_hi // 16 + 1))
    return rng, M, N, K


@pytest.mark.parametrize("seed", range(12))
def test_prefill_linear_random_shape(seed):
    rng, M, N, K = draw(seed, 600, 1500, 2048)
    X = synth.activations(rng, M, K, with_outliers=K >= 64)
    Wf = synth.weight(rng, K, N)
    b = synth.bias(rng, N)
    Wq, s_w, _ = W.w8a8_quant_weight_per_channel(dev(Wf))
    Xq, S_x = W.w8a8_quant_per_token(dev_bf16(X))
    out = W.w8a8_gemm_dequant(Xq, S_x, Wq, s_w, bias=dev(b))
    rwq, rws, _ = oracle.quant_weight_per_channel(Wf)
    rxq, rS, _, y = oracle.linear_prefill(X, rwq, rws, bias=b)
    assert_same(host(Wq), rwq, f"Wq {M}x{N}x{K}")
    assert_same(host(Xq), rxq, f"Xq {M}x{N}x{K}")
    assert_same(host(S_x), rS, f"S_x {M}x{N}x{K}")
    assert_same(host_bf16(out), oracle.f32_to_bf16(y), f"out {M}x{N}x{K}")


@pytest.mark.parametrize("seed", range(10))
def test_decode_linear_random_shape(seed):
    rng, M, N, K = draw(100 + seed, 64, 3000, 4096)
    case = synth.decode_static(M=M, N=N, K=K, seed=seed)
    S, r, Z = W.w8a8_calibrate_static(dev_bf16(case.Xcal))
    Wq, s_w, cs = W.w8a8_quant_weight_per_channel(dev(case.W))
    out = W.w8a8_linear_static(dev_bf16(case.X), S, r, Z, Wq, s_w, cs)
    rS, rr, rZ = oracle.calibrate_static(case.Xcal)
    rwq, rws, rwc = oracle.quant_weight_per_channel(case.W)
    _, _, y = oracle.linear_decode(case.X, rr, rZ, rS, rwq, rws, rwc)
    assert_same(host_bf16(out), oracle.f32_to_bf16(y), f"out {M}x{N}x{K}")


@pytest.mark.parametrize("seed", range(8))
def test_llm_int8_random_shape(seed):
    rng, M, N, K = draw(200 + seed, 400, 1200, 2048)
    n_cols = int(rng.integers(0, min(20, K) + 1))
    cols = np.sort(rng.choice(K, size=n_cols, replace=False))
    x = np.clip(rng.standard_normal((M, K)).astype(np.float32), -5.5, 5.5)
    x[:, cols] = (np.where(rng.random((M, n_cols)) < 0.5, -1.0, 1.0) * rng.uniform(20, 100, (M, n_cols))).astype(np.float32)
    X = synth.bf16_bits(x)
    Wb = synth.bf16_bits(synth.weight(rng, K, N))
    bias = synth.bias(rng, N)
    cap = 32
    Wd = dev_bf16(Wb)
    Wq, s_w, _ = W.w8a8_quant_weight_per_channel(Wd)
    Xq, S_x, idx, n_out, Xo = W.int8_outlier_split(dev_bf16(X), 6.0, cap)
    out = W.int8_mixed_decomp_gemm(Xq, S_x, Xo, idx, n_out, cap, Wq, s_w, Wd, bias=dev(bias))
    rq, rS, ridx, rn, _ = oracle.outlier_split(X, 6.0, cap)
    assert int(host(n_out)[0]) == rn == n_cols
    assert_same(host(idx)[:rn], ridx[:rn], f"outlier_idx {M}x{K}")
    assert_same(host(Xq), rq, f"Xq {M}x{K}")
    assert_same(host(S_x), rS, f"S_x {M}x{K}")
    rwq, rws, _ = oracle.quant_weight_per_channel(Wb)
    *_, y = oracle.linear_mixed(X, Wb, rwq, rws, threshold=6.0, cap=cap, bias=bias)
    assert_same(host_bf16(out), oracle.f32_to_bf16(y), f"out {M}x{N}x{K}")


@pytest.mark.parametrize("seed", range(8))
def test_llm_int8_tensor_core_side_random_shape(seed):
    """The tensor-core side product at random shapes and outlier counts (0 to
    100 columns, any cap above them), held to the same per-element bound as
    its hand-picked cases (the fp32 side sums differ from the oracle's only
    in their order)."""
    from tests.test_gpu_outlier import side_tolerance

    rng, M, N, K = draw(300 + seed, 600, 1500, 2048)
    n_cols = int(rng.integers(0, min(100, K) + 1))
    cap = n_cols + int(rng.integers(0, 40)) if n_cols else int(rng.integers(1, 40))
    cols = np.sort(rng.choice(K, size=n_cols, replace=False))
    x = np.clip(rng.standard_normal((M, K)).astype(np.float32), -5.5, 5.5)
    x[:, cols] = (np.where(rng.random((M, n_cols)) < 0.5, -1.0, 1.0) * rng.uniform(20, 100, (M, n_cols))).astype(np.float32)
    X = synth.bf16_bits(x)
    Wb = synth.bf16_bits(synth.weight(rng, K, N))
    bias = synth.bias(rng, N) if rng.random() < 0.5 else None
    Wd = dev_bf16(Wb)
    Wq, s_w, _ = W.w8a8_quant_weight_per_channel(Wd)
    Xq, S_x, idx, n_out, Xo = W.int8_outlier_split(dev_bf16(X), 6.0, cap)
    y32 = W.int8_mixed_decomp_gemm_tc(Xq, S_x, Xo, idx, n_out, cap, Wq, s_w, Wd,
                                      bias=None if bias is None else dev(bias), out_dtype=torch.float32)
    rq, rS, ridx, rn, rXo = oracle.outlier_split(X, 6.0, cap)
    assert rn == n_cols and int(host(n_out)[0]) == rn
    rwq, rws, _ = oracle.quant_weight_per_channel(Wb)
    side = oracle.outlier_side(rXo, ridx, Wb)
    y_ref = oracle.epilogue(oracle.gemm_i64(rq, rwq), rS, rws, bias=bias, side=side)
    got = host(y32)
    if n_cols == 0:
        assert_same(got, y_ref, f"out {M}x{N}x{K}")
        return
    tol, _ = side_tolerance(rXo, ridx, Wb, side, bias, y_ref)
    err = np.abs(got.astype(np.float64) - y_ref.astype(np.float64))
    assert (err <= tol).all(), f"{M}x{N}x{K}, {n_cols} columns: {int((err > tol).sum())} elements outside the bound"
