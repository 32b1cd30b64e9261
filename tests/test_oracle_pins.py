"""Pins for the CPU oracle, checked against things other than the oracle.

Each test ties one part of the oracle to the pages' worked examples, to a
closed form, to an invariant, or to an independent library routine (numpy,
torch), so that a dropped term, a wrong sign or index or a transposed operand
in ``oracle/w8a8_oracle.c`` fails at least one of them.
"""
import numpy as np
import pytest
import torch

import oracle
from int8_gemm_token_b200 import synth

F32 = np.float32


def bf(a):
    return synth.bf16_bits(np.asarray(a, dtype=np.float32))


def f32(bits):
    return synth.bits_to_f32(bits)


# ---------------------------------------------------------------------------
# Symmetric absmax quantizer (per-token rows, per-channel weight columns)
# ---------------------------------------------------------------------------

def test_worked_example_row_constant(golden):
    """LLM.int8() summary, architecture figure step (1)-(2): row [2,-1,1] has C_x = 2."""
    g = golden("absmax_worked_example.txt")
    row = np.array([float(v) for v in g["row"][0]], dtype=np.float32)
    cx = float(g["C_x"][0][0])
    codes = np.array([int(v) for v in g["codes"][0]], dtype=np.int8)
    Xq, S = oracle.quant_per_token(bf(row[None, :]))
    assert S[0] == F32(cx) / F32(127.0)
    assert np.array_equal(Xq[0], codes)
    # the same vector as one output channel of W [K, N] (one column) gives the same codes
    Wq, s_w, colsum = oracle.quant_weight_per_channel(row[:, None].astype(np.float32))
    assert np.array_equal(Wq[0], codes) and s_w[0] == S[0] and colsum[0] == int(codes.astype(np.int64).sum())


@pytest.mark.parametrize("row, codes", [
    ([254, 1, -1, 3], [127, 0, 0, 2]),      # r = 0.5: 0.5 -> 0, -0.5 -> 0, 1.5 -> 2
    ([254, 5, -5, 7], [127, 2, -2, 4]),     # 2.5 -> 2, -2.5 -> -2, 3.5 -> 4
    ([-254, 9, 11, -13], [-127, 4, 6, -6]),  # 4.5 -> 4, 5.5 -> 6, -6.5 -> -6
])
def test_ties_round_half_to_even(row, codes):
    """Exact ties (r = 127/254 = 0.5 exactly) round half to even (IEEE default)."""
    Xq, S = oracle.quant_per_token(bf(np.array([row], dtype=np.float32)))
    assert np.array_equal(Xq[0], np.array(codes, dtype=np.int8))
    assert S[0] == F32(2.0)


def test_absmax_roundtrip_bound_and_extremes():
    """|x - S q| <= S/2 (plus fp32 slack), the absmax element maps to +-127,
    signs are kept, and codes stay in [-127, 127]."""
    rng = np.random.default_rng(3)
    X = synth.activations(rng, 64, 200, with_outliers=True)
    Xq, S = oracle.quant_per_token(X)
    x = f32(X).astype(np.float64)
    q = Xq.astype(np.float64)
    s = S.astype(np.float64)[:, None]
    err = np.abs(x - s * q)
    assert np.all(err <= s * (0.5 + 1e-5))
    amax = np.abs(x).max(axis=1)
    assert np.allclose(s[:, 0], amax / 127.0, rtol=1e-6, atol=0)
    arg = np.abs(x).argmax(axis=1)
    assert np.all(np.abs(Xq[np.arange(64), arg]) == 127)
    assert Xq.min() >= -127 and Xq.max() <= 127
    assert np.all((np.sign(q) == np.sign(x)) | (q == 0))


def test_float64_brute_force_codes():
    """Against an exact float64 rendering of round(127 x / a): codes differ by
    at most one, and only where 127x/a sits within fp32 rounding of a .5 tie."""
    rng = np.random.default_rng(11)
    X = synth.activations(rng, 8, 8)
    Xq, _ = oracle.quant_per_token(X)
    x = f32(X).astype(np.float64)
    a = np.abs(x).max(axis=1, keepdims=True)
    t = 127.0 * x / a
    q64 = np.clip(np.round(t), -127, 127)  # numpy rounds half to even
    diff = np.abs(q64 - Xq)
    near_tie = np.abs(np.abs(t - np.floor(t)) - 0.5) < 1e-5 * np.maximum(1, np.abs(t))
    assert np.all(diff <= 1) and np.all((diff == 0) | near_tie)


def test_zero_row_gives_zero_scale_and_codes():
    X = bf(np.zeros((2, 32), np.float32))
    Xq, S = oracle.quant_per_token(X)
    assert np.all(Xq == 0) and np.all(S == 0)


def test_tiny_vectors_quantize_as_zero():
    """A row (or weight column) whose absmax a is below 127/FLT_MAX, where
    127/a overflows fp32 (bf16 subnormals, tiny normals), is quantized as a
    zero vector: S = 0 and all codes 0. Just above that bound the scale is
    finite and the row's extreme values take codes +-127; a calibration range
    whose 255/d overflows is treated like an empty one (S = r = 1, Z = 0)."""
    fmax = float(np.finfo(np.float32).max)
    tiny = np.array([1e-38, -1e-38, 3e-39, -9.2e-41, 0.0, -0.0, 2e-40, -5e-39], np.float32)
    edge = np.array([4e-37, -4e-37, 1e-37, 0.0], np.float32)
    X = bf(np.stack([tiny, tiny[::-1], np.zeros(8, np.float32), np.resize(edge, 8)]))
    xf = f32(X)
    a = np.abs(xf).max(axis=1)
    assert np.all(a[:2] < 127.0 / fmax) and np.all(a[:2] > 0) and a[3] > 127.0 / fmax
    Xq, S = oracle.quant_per_token(X)
    assert np.all(Xq[:3] == 0) and np.all(S[:3] == 0)
    assert S[3] > 0 and Xq[3, 0] == 127 and Xq[3, 1] == -127 and Xq[3, 3] == 0
    Wq, s_w, colsum = oracle.quant_weight_per_channel(bf(np.stack([tiny, tiny[::-1]], axis=1)))
    assert np.all(Wq == 0) and np.all(s_w == 0) and np.all(colsum == 0)
    S, r, Z = oracle.calibrate_static(bf(tiny.reshape(2, 4)))
    assert (S, r, Z) == (1.0, 1.0, 0)
    S, r, Z = oracle.calibrate_static(bf(edge.reshape(1, 4) * 4))
    assert 0 < r < fmax and -128 <= Z <= 127


def test_weight_per_channel_pins():
    """One scale per output channel n over all K; colsum is the column sum of
    the int8 codes (numpy); round-trip bound per column."""
    rng = np.random.default_rng(5)
    W = synth.weight(rng, 96, 40)
    W[:, 3] = 0.0
    Wq, s_w, colsum = oracle.quant_weight_per_channel(W)
    assert Wq.shape == (40, 96)
    assert np.array_equal(colsum, Wq.astype(np.int64).sum(axis=1).astype(np.int32))
    w = W.astype(np.float64).T
    err = np.abs(w - s_w[:, None].astype(np.float64) * Wq)
    assert np.all(err <= s_w[:, None] * (0.5 + 1e-5))
    amax = np.abs(W).max(axis=0)
    nz = amax > 0
    assert np.allclose(s_w[nz], amax[nz] / 127.0, rtol=1e-6)
    assert s_w[3] == 0 and np.all(Wq[3] == 0)
    # bf16 weights take the same path as their exact fp32 values
    Wb = bf(W)
    Wq2, s2, c2 = oracle.quant_weight_per_channel(Wb)
    Wq3, s3, c3 = oracle.quant_weight_per_channel(f32(Wb))
    assert np.array_equal(Wq2, Wq3) and np.array_equal(s2, s3) and np.array_equal(c2, c3)


# ---------------------------------------------------------------------------
# Asymmetric MinMax calibration and the static quantizer (PDMIX decode)
# ---------------------------------------------------------------------------

def test_calibration_one_sided_range_gives_min_zero_point():
    """ReLU-shifted calibration data (all >= 0.5): the range starts at real 0,
    so the zero point is the lowest code and 0 maps to it exactly."""
    rng = np.random.default_rng(1)
    Xcal = synth.calibration_tokens(rng, 64, 128)
    S, r, Z = oracle.calibrate_static(Xcal)
    hi = f32(Xcal).max()
    assert Z == -128
    assert abs(float(S) * 255.0 - float(hi)) <= 2e-7 * float(hi)
    q = oracle.quant_per_tensor(bf(np.array([[0.0, hi]], np.float32)), r, Z)
    assert q[0, 0] == -128 and q[0, 1] == 127


def test_calibration_signed_range_closed_forms():
    """Signed data: q(lo) = -128, q(hi) = 127, q(0) = Z, and every in-range x
    satisfies |x - S (q - Z)| <= S/2 (+ fp32 slack)."""
    rng = np.random.default_rng(2)
    Xcal = synth.activations(rng, 96, 64)
    x = f32(Xcal)
    S, r, Z = oracle.calibrate_static(Xcal)
    lo, hi = float(x.min()), float(x.max())
    assert -128 < Z < 127
    assert abs(float(S) * 255.0 - (hi - lo)) <= 1e-6 * (hi - lo)
    ends = oracle.quant_per_tensor(bf(np.array([[lo, 0.0, hi]], np.float32)), r, Z)
    assert list(ends[0]) == [-128, int(Z), 127]
    q = oracle.quant_per_tensor(Xcal, r, Z).astype(np.float64)
    err = np.abs(x.astype(np.float64) - float(S) * (q - float(Z)))
    assert np.all(err <= float(S) * (0.5 + 1e-4))


def test_static_quant_saturates_outside_range():
    """Glossary §2.4: out-of-distribution decode values saturate at the ends."""
    rng = np.random.default_rng(4)
    Xcal = synth.calibration_tokens(rng, 32, 64)
    S, r, Z = oracle.calibrate_static(Xcal)
    hi = float(f32(Xcal).max())
    X = bf(np.array([[2 * hi, -hi, hi + 2 * float(S), -3 * float(S), 1e30, -1e30]], np.float32))
    q = oracle.quant_per_tensor(X, r, Z)
    assert list(q[0]) == [127, -128, 127, -128, 127, -128]


def test_static_dequant_inverts_the_static_quantizer():
    """x = S (q - Z), the inverse of eq. Q_decode (the INT8 KV cache's read
    side). Hand values: S = 0.5, Z = -128 maps codes -128, 0, 127 to 0, 64,
    127.5. q = Z gives exactly 0. Every code equals the exact real product
    (float64 holds it) rounded once to fp32, and bf16 output is torch's
    rounding of that. Codes of calibrated values come back within S/2."""
    hand = np.zeros((1, 16), np.int8)
    hand[0, :3] = [-128, 0, 127]
    y = oracle.dequant_per_tensor(hand, F32(0.5), -128, oracle.DT_FP32)
    assert y[0, :3].tolist() == [0.0, 64.0, 127.5]
    codes = np.arange(-128, 128).astype(np.int8)[None, :]
    for S, Z in [(F32(0.5), -128), (F32(0.013), 7), (F32(3.0e-3), 127), (F32(250.0), -5)]:
        y = oracle.dequant_per_tensor(codes, S, Z, oracle.DT_FP32)
        exact = (float(S) * (codes.astype(np.float64) - Z)).astype(np.float32)
        assert np.array_equal(y, exact)
        assert y[0, Z + 128] == 0.0
        assert np.array_equal(oracle.dequant_per_tensor(codes, S, Z), bf(exact))
    rng = np.random.default_rng(12)
    Xcal = synth.activations(rng, 32, 64)
    S, r, Z = oracle.calibrate_static(Xcal)
    q = oracle.quant_per_tensor(Xcal, r, Z)
    back = oracle.dequant_per_tensor(q, S, Z, oracle.DT_FP32).astype(np.float64)
    assert np.all(np.abs(f32(Xcal).astype(np.float64) - back) <= float(S) * (0.5 + 1e-4))


def test_calibration_all_zero_is_identity_scale():
    S, r, Z = oracle.calibrate_static(bf(np.zeros((4, 16), np.float32)))
    assert (S, r, Z) == (1.0, 1.0, 0)


# ---------------------------------------------------------------------------
# Integer GEMM, zero-point correction, epilogue
# ---------------------------------------------------------------------------

def test_gemm_matches_numpy_int64():
    rng = np.random.default_rng(6)
    for M, N, K in [(7, 5, 33), (1, 1, 1), (16, 9, 256)]:
        Xq = rng.integers(-128, 128, (M, K), dtype=np.int8)
        Wq = rng.integers(-127, 128, (N, K), dtype=np.int8)
        Xq[0, :] = -128
        acc = oracle.gemm_i64(Xq, Wq)
        assert np.array_equal(acc, Xq.astype(np.int64) @ Wq.astype(np.int64).T)


def test_gemm_k1_is_outer_product():
    x = np.array([[3], [-2], [127]], np.int8)
    w = np.array([[5], [-128 + 1], [0], [7]], np.int8)
    assert np.array_equal(oracle.gemm_i64(x, w), np.outer(x[:, 0].astype(np.int64), w[:, 0].astype(np.int64)))


def test_zero_point_correction_equals_explicit_subtraction():
    """LLM.int8() summary §一.2 four-term expansion with zp_b = 0:
    acc - Z*colsum[n] == sum_k (Xq - Z) * Wq, computed explicitly with numpy."""
    rng = np.random.default_rng(7)
    M, N, K = 6, 10, 48
    Xq = rng.integers(-128, 128, (M, K), dtype=np.int8)
    Wq = rng.integers(-127, 128, (N, K), dtype=np.int8)
    colsum = Wq.astype(np.int64).sum(axis=1).astype(np.int32)
    for Z in (-128, -37, 0, 5, 127):
        acc = oracle.gemm_i64(Xq, Wq)
        y = oracle.epilogue(acc, np.float32(1.0), np.ones(N, np.float32), colsum=colsum, Z=Z)
        explicit = (Xq.astype(np.int64) - Z) @ Wq.astype(np.int64).T
        assert np.array_equal(y.astype(np.int64), explicit)  # |values| < 2^24: exact in fp32


def test_exact_when_scales_are_powers_of_two():
    """Rows/columns whose absmax is 127 (or 254, with even entries) get scale
    1 (or 2): quantization is exact, so the layer output equals the float64
    product X @ W + bias exactly."""
    rng = np.random.default_rng(8)
    M, K, N = 5, 64, 12
    X = rng.integers(-60, 61, (M, K)).astype(np.float32) * 2
    X[:, 0] = 254.0
    X[2] = 0.0
    W = rng.integers(-127, 128, (K, N)).astype(np.float32)
    W[1, :] = 127.0
    b = rng.integers(-8, 9, N).astype(np.float32)
    Wq, s_w, _ = oracle.quant_weight_per_channel(W)
    assert np.all(s_w == 1.0)
    Xq, S_x, acc, y = oracle.linear_prefill(bf(X), Wq, s_w, bias=b)
    ref = X.astype(np.float64) @ W.astype(np.float64) + b
    assert np.array_equal(y.astype(np.float64), ref)


def test_layer_error_within_quantization_bound():
    """Closed-form bound vs the float64 product of the unquantized inputs:
    |y - (X W + b)| <= sum_k (|x_k| s_w/2 + |w_k| S_x/2 + S_x s_w/4) + epilogue
    rounding. A transposed scale or operand breaks it by orders of magnitude."""
    case = synth.prefill_small(0)
    Wq, s_w, _ = oracle.quant_weight_per_channel(case.W)
    Xq, S_x, acc, y = oracle.linear_prefill(case.X, Wq, s_w, bias=case.bias)
    x = f32(case.X).astype(np.float64)
    W = case.W.astype(np.float64)
    ref = x @ W + case.bias
    Sx = S_x.astype(np.float64)[:, None]
    sw = s_w.astype(np.float64)[None, :]
    bound = (np.abs(x).sum(1, keepdims=True) * sw / 2 + Sx * np.abs(W).sum(0, keepdims=True) / 2
             + x.shape[1] * Sx * sw / 4)
    bound += 1e-6 * np.abs(ref) + 1e-7
    assert np.all(np.abs(y - ref) <= bound)
    # and the dequant equals acc * (c_x (x) c_w) / 127^2 of the summary's step (4)
    cx = S_x.astype(np.float64) * 127
    cw = s_w.astype(np.float64) * 127
    step4 = acc * np.outer(cx, cw) / (127.0 * 127.0) + case.bias
    assert np.allclose(y, step4, rtol=1e-5, atol=1e-6)


def test_decode_layer_error_bound():
    """Decode path (static S, Z): output vs float64 X W within the same bound
    with S in place of S_x, for tokens inside the calibrated range."""
    rng = np.random.default_rng(9)
    Xcal = synth.calibration_tokens(rng, 64, 128)
    X = synth.calibration_tokens(rng, 4, 128)
    W = synth.weight(rng, 128, 24)
    S, r, Z = oracle.calibrate_static(Xcal)
    x = f32(X).astype(np.float64)
    assert x.max() <= f32(Xcal).max()
    Wq, s_w, colsum = oracle.quant_weight_per_channel(W)
    Xq, acc, y = oracle.linear_decode(X, r, Z, S, Wq, s_w, colsum)
    ref = x @ W.astype(np.float64)
    sw = s_w.astype(np.float64)[None, :]
    bound = (np.abs(x).sum(1, keepdims=True) * sw / 2 + float(S) * np.abs(W).sum(0, keepdims=True) / 2
             + 128 * float(S) * sw / 4 + 1e-6 * np.abs(ref) + 1e-7)
    assert np.all(np.abs(y - ref) <= bound)


def test_decode_requant_of_a_hand_worked_layer():
    """Static requantization for the next linear, worked by hand. With S = 1,
    r = 1, Z = 0 the activation codes are the integers of X; one channel of
    ones over the first three inputs gives y = 127 + 127 + 7 = 261. bf16 keeps
    8 significant bits, so 261 is stored as 260; with r_out = 1, Z_out = -200
    the code is 260 - 200 = 60 (quantizing the fp32 value would give 61, and
    dropping Z_out would saturate at 127). A second channel of -1s gives
    y = -261 -> bf16 -260 -> -460, saturated to -128."""
    K = 16
    X = np.zeros((1, K), np.float32)
    X[0, :3] = [127.0, 127.0, 7.0]
    Wq = np.zeros((2, K), np.int8)
    Wq[0, :3] = 1
    Wq[1, :3] = -1
    s_w = np.ones(2, np.float32)
    colsum = Wq.astype(np.int32).sum(1).astype(np.int32)
    _, acc, y, y_bf16, q = oracle.linear_decode_requant(bf(X), F32(1.0), 0, F32(1.0), Wq, s_w, colsum,
                                                        F32(1.0), -200)
    assert acc.tolist() == [[261, -261]] and y.tolist() == [[261.0, -261.0]]
    assert f32(y_bf16).tolist() == [[260.0, -260.0]]
    assert q.tolist() == [[60, -128]]
    # a scaled case: r_out = 0.25 maps bf16 260 to 65 exactly; Z_out = 3 shifts it
    q2 = oracle.linear_decode_requant(bf(X), F32(1.0), 0, F32(1.0), Wq, s_w, colsum, F32(0.25), 3)[4]
    assert q2.tolist() == [[68, -62]]


def test_epilogue_fixed_order():
    """fmaf(float(c), S_x*s_w, side + bias) with single roundings, checked
    against float64 evaluation of the same expression rounded once."""
    acc = np.array([[16777217, -3, 0]], np.int64)  # 2^24 + 1 rounds to 2^24 in fp32
    S_x = np.array([0.1], np.float32)
    s_w = np.array([0.3, 0.7, 1.0], np.float32)
    bias = np.array([0.25, -0.5, 0.0], np.float32)
    y = oracle.epilogue(acc, S_x, s_w, bias=bias)
    sc = (S_x[0] * s_w).astype(np.float32)
    f = acc[0].astype(np.float32).astype(np.float64)
    expect = (f * sc.astype(np.float64) + bias.astype(np.float64)).astype(np.float32)
    assert np.array_equal(y[0], expect)
    assert float(np.float32(16777217)) == 16777216.0


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(10)
    y = (rng.standard_normal(20000) * 10 ** rng.uniform(-3, 3, 20000)).astype(np.float32)
    ties = np.array([1.00390625, 1.01171875, -1.00390625, 3.0e38, 1e-40], np.float32)
    y = np.concatenate([y, ties])
    ours = oracle.f32_to_bf16(y)
    ref = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert ours[-5] == 0x3F80 and ours[-4] == 0x3F82


# ---------------------------------------------------------------------------
# LLM.int8() outlier decomposition
# ---------------------------------------------------------------------------

def test_outlier_columns_of_the_figure(golden):
    g = golden("outlier_columns_example.txt")
    thr = float(g["threshold"][0][0])
    X = np.array([[float(v) for v in r] for r in g["row"]], np.float32)
    want = [int(v) for v in g["outlier_columns"][0]]
    Xq, S_x, idx, n_out, Xo = oracle.outlier_split(bf(X), thr, cap=8)
    assert list(idx) == want and n_out == len(want)
    assert np.all(Xq[:, want] == 0)
    assert np.array_equal(f32(Xo[:, :n_out]), X[:, want])
    # row scales come from the normal columns only: row 1 -> max(|6|, |-3|) = 6
    assert S_x[1] == F32(6.0) / F32(127.0)


def test_threshold_infinity_is_plain_vector_wise():
    case = synth.prefill_small(1)
    Xq0, S0 = oracle.quant_per_token(case.X)
    Xq, S_x, idx, n_out, _ = oracle.outlier_split(case.X, float("inf"), cap=8)
    assert n_out == 0 and np.array_equal(Xq, Xq0) and np.array_equal(S_x, S0)


def test_threshold_zero_routes_everything_to_the_side_path():
    """Threshold 0 and no zero column: every column is an outlier, the INT8
    path is all zeros and the output is the fp32 GEMM of the bf16 inputs."""
    rng = np.random.default_rng(12)
    M, K, N = 6, 24, 10
    xf = rng.standard_normal((M, K)).astype(np.float32) + 3.0
    X = bf(xf)
    W = bf(rng.standard_normal((K, N)).astype(np.float32))
    Wq, s_w, _ = oracle.quant_weight_per_channel(W)
    Xq, S_x, idx, n_out, Xo, acc, side, y = oracle.linear_mixed(X, W, Wq, s_w, threshold=0.0, cap=K)
    assert n_out == K and np.all(Xq == 0) and np.all(S_x == 0)
    ref = f32(X).astype(np.float64) @ f32(W).astype(np.float64)
    tol = K * 2.0 ** -23 * (np.abs(f32(X)).astype(np.float64) @ np.abs(f32(W)).astype(np.float64))
    assert np.all(np.abs(y - ref) <= tol)


def test_mixed_layer_error_bound():
    """Decomposed layer vs float64 X W: only the normal columns carry
    quantization error; the outlier columns are carried in fp32 (bf16 inputs)."""
    rng = np.random.default_rng(13)
    M, K, N = 12, 64, 16
    xf = rng.standard_normal((M, K)).astype(np.float32)
    cols = [5, 40]
    xf[:, cols] = rng.uniform(20, 100, (M, 2)).astype(np.float32) * np.sign(rng.standard_normal((M, 2))).astype(np.float32)
    X = bf(xf)
    W = bf(synth.weight(rng, K, N))
    Wq, s_w, _ = oracle.quant_weight_per_channel(W)
    Xq, S_x, idx, n_out, Xo, acc, side, y = oracle.linear_mixed(X, W, Wq, s_w)
    assert list(idx) == cols
    x = f32(X).astype(np.float64)
    w = f32(W).astype(np.float64)
    ref = x @ w
    xn = x.copy()
    xn[:, cols] = 0
    wn = w.copy()
    wn[cols, :] = 0
    Sx = S_x.astype(np.float64)[:, None]
    sw = s_w.astype(np.float64)[None, :]
    bound = (np.abs(xn).sum(1, keepdims=True) * sw / 2 + Sx * np.abs(wn).sum(0, keepdims=True) / 2
             + K * Sx * sw / 4 + 1e-5 * (np.abs(x) @ np.abs(w)) + 1e-7)
    assert np.all(np.abs(y - ref) <= bound)


def test_outlier_exactly_at_threshold_stays_int8_and_cap_overflow():
    X = bf(np.array([[6.0, 1.0, -7.0, 0.5, 9.0]], np.float32))
    _, _, idx, n_out, _ = oracle.outlier_split(X, 6.0, cap=8)
    assert list(idx) == [2, 4]
    _, _, idx, n_out, _ = oracle.outlier_split(X, 0.75, cap=2)
    assert n_out == 4 and list(idx) == [0, 1]
