"""Randomized properties of the CPU oracle (hypothesis), each checked
against a closed form or a float64 / numpy evaluation rather than against
the oracle itself: shapes, magnitudes and signs beyond the fixed seeds of
the pins. CPU only; bounded to a few seconds."""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from int8_gemm_token_b200 import synth

SETTINGS = dict(max_examples=40, deadline=None)


def _bf16_matrix(seed, M, K, scale):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K), dtype=np.float32) * np.float32(scale)
    x[rng.random((M, K)) < 0.05] = 0.0
    return synth.bf16_bits(x)


@settings(**SETTINGS)
@given(seed=st.integers(0, 2**31 - 1), M=st.integers(1, 9), K16=st.integers(1, 8),
       scale=st.sampled_from([1e-30, 1e-3, 1.0, 60.0, 1e30]))
def test_per_token_codes_bound_and_extremes(seed, M, K16, scale):
    """PDMIX glossary eq. Q_prefill with the reading r = 127/a: every code is
    within [-127, 127], |x - S q| <= S/2 (fp32 slack), the row maximum maps
    to +-127 and S = a/127 rounded once."""
    X = _bf16_matrix(seed, M, 16 * K16, scale)
    Xq, S = oracle.quant_per_token(X)
    x = synth.bits_to_f32(X).astype(np.float64)
    a = np.abs(x).max(axis=1)
    assert Xq.min() >= -127 and Xq.max() <= 127
    for m in range(M):
        if a[m] == 0:
            assert S[m] == 0 and not Xq[m].any()
            continue
        assert S[m] == np.float32(np.float32(a[m]) / np.float32(127.0))
        s = float(S[m])
        assert np.all(np.abs(x[m] - s * Xq[m]) <= s * (0.5 + 1e-5))
        assert np.abs(Xq[m, np.abs(x[m]).argmax()]) == 127


@settings(**SETTINGS)
@given(seed=st.integers(0, 2**31 - 1), T=st.integers(1, 6), K16=st.integers(1, 6),
       shift=st.sampled_from([-3.0, 0.0, 0.5, 4.0]))
def test_static_codes_round_trip_inside_the_calibrated_range(seed, T, K16, shift):
    """PDMIX glossary eq. Q_decode: for x in the calibrated range,
    |x - S (q - Z)| <= S/2 (fp32 slack); 0 maps to Z exactly; the range ends
    map to -128 and 127 (the MinMax range includes 0)."""
    Xcal = synth.bf16_bits(synth.bits_to_f32(_bf16_matrix(seed, T, 16 * K16, 1.0)) + np.float32(shift))
    S, r, Z = oracle.calibrate_static(Xcal)
    x = synth.bits_to_f32(Xcal)
    lo, hi = min(0.0, float(x.min())), max(0.0, float(x.max()))
    if hi == lo:
        assert (S, r, Z) == (1.0, 1.0, 0)
        return
    q = oracle.quant_per_tensor(Xcal, r, Z).astype(np.float64)
    assert np.all(np.abs(x.astype(np.float64) - float(S) * (q - float(Z))) <= float(S) * (0.5 + 1e-4))
    ends = oracle.quant_per_tensor(synth.bf16_bits(np.array([[lo, 0.0, hi]], np.float32)), r, Z)[0]
    assert ends[1] == Z
    assert ends[0] == -128 or lo == 0.0 and Z == -128
    assert ends[2] == 127


@settings(**SETTINGS)
@given(seed=st.integers(0, 2**31 - 1), M=st.integers(1, 5), N=st.integers(1, 7), K16=st.integers(1, 4),
       Z=st.integers(-128, 127))
def test_corrected_accumulator_is_the_zero_point_shifted_product(seed, M, N, K16, Z):
    """acc - Z*colsum == sum_k (Xq - Z) Wq (numpy int64), for any zero point;
    the int32 output mode of the epilogue is that integer."""
    rng = np.random.default_rng(seed)
    K = 16 * K16
    Xq = rng.integers(-128, 128, (M, K), dtype=np.int8)
    Wq = rng.integers(-127, 128, (N, K), dtype=np.int8)
    colsum = Wq.astype(np.int64).sum(axis=1).astype(np.int32)
    acc = oracle.gemm_i64(Xq, Wq)
    assert np.array_equal(acc, Xq.astype(np.int64) @ Wq.astype(np.int64).T)
    y = oracle.epilogue(acc, np.float32(1.0), np.ones(N, np.float32), colsum=colsum, Z=Z)
    explicit = (Xq.astype(np.int64) - Z) @ Wq.astype(np.int64).T
    assert np.array_equal(y.astype(np.int64), explicit)  # |values| < 2^24: exact in fp32


@settings(**SETTINGS)
@given(seed=st.integers(0, 2**31 - 1), M=st.integers(1, 6), K16=st.integers(1, 6),
       planted=st.lists(st.integers(0, 95), max_size=5), threshold=st.sampled_from([0.5, 3.0, 6.0]))
def test_outlier_split_definition(seed, M, K16, planted, threshold):
    """LLM.int8() summary, mixed-precision decomposition steps 1-2: the
    outlier set is exactly the columns with some |x| > threshold (ascending),
    their codes are 0, the row scale is the absmax of the other columns / 127,
    and Xo holds the original values of the outlier columns."""
    K = 16 * K16
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K), dtype=np.float32)
    for k in planted:
        if k < K:
            x[rng.integers(0, M), k] = np.float32(20.0)
    X = synth.bf16_bits(x)
    xf = synth.bits_to_f32(X)
    Xq, S_x, idx, n_out, Xo = oracle.outlier_split(X, threshold, cap=K)
    want = np.flatnonzero((np.abs(xf) > threshold).any(axis=0))
    assert n_out == want.size and np.array_equal(idx, want)
    normal = np.ones(K, bool)
    normal[want] = False
    assert not Xq[:, ~normal].any()
    for m in range(M):
        a = np.abs(xf[m, normal]).max() if normal.any() else np.float32(0.0)
        assert S_x[m] == (np.float32(a) / np.float32(127.0) if a > 0 else 0.0)
    assert np.array_equal(Xo[:, :n_out], X[:, want])
