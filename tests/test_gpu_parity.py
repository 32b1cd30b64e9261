"""CUDA path vs the CPU oracle, element by element, on seeded inputs.

Integers (codes, zero points, column sums, int32 accumulators) and scales
must match bit for bit. Outputs must match too: the epilogue performs the
same fp32 operations in the same order as the oracle (int->float RN,
S_x*s_w RN, one fmaf, bf16 RNE), so bf16 and fp32 outputs are compared for
exact equality -- stricter than the 1e-3 relative bound the layer is held to.
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
        eq = (gpu.view(np.uint32) == ref.view(np.uint32))
    else:
        eq = gpu == ref
    assert eq.all(), f"{what}: " + diff_report(gpu, ref)


# ------------------------------------------------------------ quantizers
@pytest.mark.parametrize("M,K,ld_pad", [(16, 256, 0), (1, 16, 0), (3, 48, 8), (130, 4096, 0),
                                        (7, 4112, 0), (33, 11008, 16), (5, 65536, 0), (2, 8192 + 16, 0)])
def test_quant_per_token_bit_exact(M, K, ld_pad):
    rng = np.random.default_rng(M * 7 + K)
    X = synth.activations(rng, M, K, with_outliers=K >= 64)
    if M > 2:
        X[1] = 0  # an all-zero token
    Xd_full = dev_bf16(np.pad(X, ((0, 0), (0, ld_pad))))
    Xd = Xd_full[:, :K]
    Xq, S = W.w8a8_quant_per_token(Xd)
    rq, rS = oracle.quant_per_token(X)
    assert_same(host(Xq), rq, "Xq")
    assert_same(host(S), rS, "S_x")


def test_quant_per_token_ties():
    X = synth.bf16_bits(np.array([[254, 1, -1, 3, 5, -5, 7, 9] + [0] * 8], np.float32))
    Xq, S = W.w8a8_quant_per_token(dev_bf16(X))
    assert list(host(Xq)[0, :8]) == [127, 0, 0, 2, 2, -2, 4, 4]


TINY = np.array([1e-38, -1e-38, 3e-39, -9.2e-41, 0.0, -0.0, 2e-40, -5e-39], np.float32)
EDGE = np.array([4e-37, -4e-37, 1e-37, 0.0, -3e-38, 2e-39], np.float32)


@pytest.mark.parametrize("M,K", [(6, 48), (6, 4096), (40, 11008), (300, 8192)])
def test_quant_per_token_tiny_rows(M, K):
    """Rows whose absmax is below 127/FLT_MAX (bf16 subnormals and tiny
    normals) between ordinary rows quantize as zero rows (127/a overflows
    fp32); a row just above that bound has a finite scale. Bit for bit as in
    the oracle."""
    rng = np.random.default_rng(K + 1)
    X = synth.activations(rng, M, K)
    X[1:4] = synth.bf16_bits(rng.choice(TINY, size=(3, K)))
    X[4] = synth.bf16_bits(rng.choice(EDGE, size=K))
    X[M - 1] = synth.bf16_bits(rng.choice(TINY[4:], size=K))
    Xq, S = W.w8a8_quant_per_token(dev_bf16(X))
    rq, rS = oracle.quant_per_token(X)
    assert np.all(rq[1:4] == 0) and np.all(rS[1:4] == 0) and rS[4] > 0
    assert_same(host(Xq), rq, "Xq")
    assert_same(host(S), rS, "S_x")


def test_calibrate_tiny_range():
    """A calibration range whose 255/d overflows fp32 counts as empty
    (S = r = 1, Z = 0); one just above it has a finite r."""
    for Xf in (np.resize(TINY, (4, 64)), np.resize(EDGE * 4, (4, 64))):
        X = synth.bf16_bits(Xf)
        S, r, Z = W.w8a8_calibrate_static(dev_bf16(X))
        rS, rr, rZ = oracle.calibrate_static(X)
        assert host(S)[0] == rS and host(r)[0] == rr and host(Z)[0] == rZ


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_weight_quant_tiny_columns(dtype):
    rng = np.random.default_rng(3)
    Wf = synth.weight(rng, 256, 40)
    Wf[:, 5:9] = rng.choice(TINY, size=(256, 4))
    Wf[:, 11] = rng.choice(EDGE, size=256)
    Wh = synth.bf16_bits(Wf) if dtype == "bf16" else Wf
    Wq, s_w, cs = W.w8a8_quant_weight_per_channel(dev_bf16(Wh) if dtype == "bf16" else dev(Wh))
    rq, rs, rc = oracle.quant_weight_per_channel(Wh)
    assert_same(host(Wq), rq, "Wq")
    assert_same(host(s_w), rs, "s_w")
    assert_same(host(cs), rc, "colsum")


@pytest.mark.parametrize("M,K", [(1, 4096), (32, 4096), (4096, 4096), (5, 48)])
def test_calibrate_and_quant_per_tensor_bit_exact(M, K):
    case = synth.decode_static(M=min(M, 64), N=16, K=K, seed=M)
    S, r, Z = W.w8a8_calibrate_static(dev_bf16(case.Xcal))
    rS, rr, rZ = oracle.calibrate_static(case.Xcal)
    assert host(S)[0] == rS and host(r)[0] == rr and host(Z)[0] == rZ
    X = case.X if M <= 64 else synth.calibration_tokens(np.random.default_rng(5), M, K)
    Xq = W.w8a8_quant_per_tensor(dev_bf16(X), r, Z)
    assert_same(host(Xq), oracle.quant_per_tensor(X, rr, rZ), "Xq")


def test_calibrate_signed_fp32_and_zero():
    rng = np.random.default_rng(9)
    Xcal = synth.bits_to_f32(synth.activations(rng, 100, 200, with_outliers=True))
    S, r, Z = W.w8a8_calibrate_static(dev(Xcal))
    assert (host(S)[0], host(r)[0], host(Z)[0]) == oracle.calibrate_static(Xcal)
    S, r, Z = W.w8a8_calibrate_static(dev(np.zeros((3, 50), np.float32)))
    assert (host(S)[0], host(r)[0], host(Z)[0]) == (1.0, 1.0, 0)


@pytest.mark.parametrize("K,N,dtype", [(256, 512, "f32"), (4096, 520, "f32"), (400, 33, "bf16"),
                                       (16, 8, "bf16"), (11008, 96, "f32")])
def test_weight_quant_bit_exact(K, N, dtype):
    rng = np.random.default_rng(K + N)
    Wf = synth.weight(rng, K, N)
    Wf[:, 1] = 0.0
    if dtype == "bf16":
        Wh = synth.bf16_bits(Wf)
        Wd = dev_bf16(Wh)
    else:
        Wh = Wf
        Wd = dev(Wf)
    Wq, s_w, cs = W.w8a8_quant_weight_per_channel(Wd)
    rq, rs, rc = oracle.quant_weight_per_channel(Wh)
    assert_same(host(Wq), rq, "Wq")
    assert_same(host(s_w), rs, "s_w")
    assert_same(host(cs), rc, "colsum")


# ------------------------------------------------------------ GEMM
def _rand_case(M, N, K, seed):
    rng = np.random.default_rng(seed)
    X = synth.activations(rng, M, K, with_outliers=True)
    Wf = synth.weight(rng, K, N)
    b = synth.bias(rng, N)
    return X, Wf, b


# 32 < M < 256 takes the 1-CTA kernel (128 x 256 tiles), with ragged edges.
@pytest.mark.parametrize("M,N,K", [(16, 512, 256), (128, 256, 128), (300, 520, 400), (1, 40, 16),
                                   (257, 1000, 4096), (129, 257, 144), (520, 5400, 400), (520, 5000, 144),
                                   (200, 11008, 256), (100, 2000, 400), (250, 40000, 128)])
def test_gemm_int32_accumulator_bit_exact(M, N, K):
    X, Wf, b = _rand_case(M, N, K, M + N + K)
    rq, rS = oracle.quant_per_token(X)
    wq, ws, wc = oracle.quant_weight_per_channel(Wf)
    acc = W.w8a8_gemm_dequant(dev(rq), dev(rS), dev(wq), dev(ws), out_dtype=torch.int32)
    assert_same(host(acc), oracle.gemm_i64(rq, wq).astype(np.int32), "acc")


# M >= 256 takes the CTA-pair kernel: ragged last row and column tiles, K not a
# multiple of the 128-byte k-block. (2048, 20480, 512) has 8 x 80 = 640 pair
# tiles, more than the GPU has clusters, so every cluster walks several tiles
# through both TMEM accumulator slots and their phase flips; (1000, 18000, 208)
# does the same with ragged edges.
@pytest.mark.parametrize("M,N,K", [(16, 512, 256), (300, 520, 400), (200, 264, 512), (520, 5000, 400),
                                   (520, 5400, 256), (520, 5800, 272), (200, 11008, 512), (100, 2000, 400),
                                   (2048, 20480, 512), (1000, 18000, 208),
                                   # the dispatch edges: Decode kernel up to 64 rows, 1-CTA up to 255, pair from 256
                                   (64, 1000, 512), (65, 1000, 512), (255, 520, 400), (256, 520, 400),
                                   # CTA-pair tiles: rows of bf16 output that are not 16-byte multiples
                                   # (direct stores), and one tile whose only valid 64-column box is partial
                                   (260, 1001, 272), (300, 40, 128)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_prefill_linear_bit_exact(M, N, K, out_dtype):
    X, Wf, b = _rand_case(M, N, K, 3 * M + N)
    Wq, s_w, cs = W.w8a8_quant_weight_per_channel(dev(Wf))
    Xq, S_x = W.w8a8_quant_per_token(dev_bf16(X))
    out = W.w8a8_gemm_dequant(Xq, S_x, Wq, s_w, bias=dev(b), out_dtype=out_dtype)
    rwq, rws, _ = oracle.quant_weight_per_channel(Wf)
    _, _, _, y = oracle.linear_prefill(X, rwq, rws, bias=b)
    if out_dtype == torch.bfloat16:
        assert_same(host_bf16(out), oracle.f32_to_bf16(y), "out")
    else:
        assert_same(host(out), y, "out")


def test_zero_point_path_and_raw_corrected_accumulator():
    M, N, K = 40, 300, 256
    case = synth.decode_static(M=M, N=N, K=K, seed=3)
    rS, rr, rZ = oracle.calibrate_static(case.Xcal)
    rxq = oracle.quant_per_tensor(case.X, rr, rZ)
    rwq, rws, rwc = oracle.quant_weight_per_channel(case.W)
    S, r, Z = W.w8a8_calibrate_static(dev_bf16(case.Xcal))
    Xq = W.w8a8_quant_per_tensor(dev_bf16(case.X), r, Z)
    Wq, s_w, cs = W.w8a8_quant_weight_per_channel(dev(case.W))
    c = W.w8a8_gemm_dequant(Xq, S, Wq, s_w, colsum=cs, Z=Z, out_dtype=torch.int32)
    acc = oracle.gemm_i64(rxq, rwq)
    assert_same(host(c), (acc - int(rZ) * rwc.astype(np.int64)[None, :]).astype(np.int32), "acc - Z colsum")
    y = W.w8a8_gemm_dequant(Xq, S, Wq, s_w, colsum=cs, Z=Z, out_dtype=torch.float32)
    assert_same(host(y), oracle.epilogue(acc, rS, rws, colsum=rwc, Z=rZ), "y")


@pytest.mark.parametrize("M", [1, 4, 16, 32])
@pytest.mark.parametrize("N", [4096, 11008])
def test_decode_linear_static_bit_exact(M, N):
    case = synth.decode_static(M=M, N=N, seed=0)
    S, r, Z = W.w8a8_calibrate_static(dev_bf16(case.Xcal))
    Wq, s_w, cs = W.w8a8_quant_weight_per_channel(dev(case.W))
    out = W.w8a8_linear_static(dev_bf16(case.X), S, r, Z, Wq, s_w, cs)
    rS, rr, rZ = oracle.calibrate_static(case.Xcal)
    rwq, rws, rwc = oracle.quant_weight_per_channel(case.W)
    rxq, _, y = oracle.linear_decode(case.X, rr, rZ, rS, rwq, rws, rwc)
    assert (rxq == 127).any() and (rxq == -128).any()  # the 1% pushed past the range saturates
    assert_same(host_bf16(out), oracle.f32_to_bf16(y), "out")


def test_prefill_7b_full_size():
    """The full 2048 x 4096 x 11008 workload in the launch configuration the
    benchmark uses (the CTA-pair kernel, 8 x 43 = 344 pair tiles over the
    GPU's clusters, so every cluster runs several tiles through both
    accumulator slots): codes, scales, weight and every output element
    compared with the oracle."""
    case = synth.prefill_7b(0)
    Wq, s_w, cs = W.w8a8_quant_weight_per_channel(dev(case.W))
    Xq, S_x = W.w8a8_quant_per_token(dev_bf16(case.X))
    out = W.w8a8_gemm_dequant(Xq, S_x, Wq, s_w, bias=dev(case.bias))
    rxq, rS = oracle.quant_per_token(case.X)
    rwq, rws, rwc = oracle.quant_weight_per_channel(case.W)
    assert_same(host(Xq), rxq, "Xq")
    assert_same(host(S_x), rS, "S_x")
    assert_same(host(Wq), rwq, "Wq")
    assert_same(host(s_w), rws, "s_w")
    assert_same(host(cs), rwc, "colsum")
    y = oracle.epilogue(oracle.gemm_i64(rxq, rwq), rS, rws, bias=case.bias)
    assert_same(host_bf16(out), oracle.f32_to_bf16(y), "out")


def test_pdmix_block_full_size():
    """The PDMIX block workload at full size, in the launch configuration the
    benchmark times: for each of the four linears (QKV, O, gate+up, down), one
    INT8 weight serves a 4096-token Prefill (per-token quant + GEMM) and
    Decode steps of 32 tokens (static calibration + one call). Weights,
    calibration scalars, Prefill codes, scales and every Prefill output
    element, and every Decode output element of the first and last step, are
    compared with the oracle."""
    for L_ in synth.pdmix_block(seed=0):
        what = f"{L_.name} {L_.K}->{L_.N}"
        Wf = L_.weight()
        Wq, s_w, cs = W.w8a8_quant_weight_per_channel(dev(Wf))
        rwq, rws, rwc = oracle.quant_weight_per_channel(Wf)
        del Wf
        assert_same(host(Wq), rwq, what + " Wq")
        assert_same(host(s_w), rws, what + " s_w")
        assert_same(host(cs), rwc, what + " colsum")
        # Prefill, 4096 tokens
        Xp = L_.prefill_input(4096)
        Xq, S_x = W.w8a8_quant_per_token(dev_bf16(Xp))
        out = W.w8a8_gemm_dequant(Xq, S_x, Wq, s_w)
        rxq, rS = oracle.quant_per_token(Xp)
        assert_same(host(Xq), rxq, what + " Xq")
        assert_same(host(S_x), rS, what + " S_x")
        y = oracle.epilogue(oracle.gemm_i64(rxq, rwq), rS, rws)
        assert_same(host_bf16(out), oracle.f32_to_bf16(y), what + " prefill out")
        del Xp, Xq, S_x, out, rxq, y
        # Decode: calibration, then two of the 64 steps
        cal = L_.calibration()
        S, r, Z = W.w8a8_calibrate_static(dev_bf16(cal))
        rS_t, rr, rZ = oracle.calibrate_static(cal)
        assert (host(S)[0], host(r)[0], host(Z)[0]) == (rS_t, rr, rZ), what
        work = W.new_workspace(32, L_.N, L_.K)
        for step in (0, 63):
            xd = L_.decode_input(step, 32)
            o = W.w8a8_linear_static(dev_bf16(xd), S, r, Z, Wq, s_w, cs, workspace=work)
            _, _, yd = oracle.linear_decode(xd, rr, rZ, rS_t, rwq, rws, rwc)
            assert_same(host_bf16(o), oracle.f32_to_bf16(yd), f"{what} decode step {step}")


# ------------------------------------------------------------ failure path
def test_bounded_wait_reports_timeout_and_device_stays_usable():
    W.w8a8_debug_wait_timeout_selftest(2_000_000)
    assert W.w8a8_check_device_error() == 6  # W8A8_ERR_DEVICE_TIMEOUT
    assert W.w8a8_check_device_error() == 0  # cleared
    X = synth.activations(np.random.default_rng(0), 4, 64)
    Xq, S = W.w8a8_quant_per_token(dev_bf16(X))
    assert_same(host(Xq), oracle.quant_per_token(X)[0], "Xq after timeout")


# ------------------------------------------------------------ decode kernel (M <= 32)
@pytest.mark.parametrize("M,N,K", [(1, 128, 128), (5, 300, 400), (16, 4096, 4096), (17, 520, 1024),
                                   (32, 11008, 4096), (3, 40, 16), (32, 4096, 11008), (32, 22016, 4096),
                                   (32, 131072, 512), (16, 131072, 256), (32, 1024, 4096), (8, 256, 2048),
                                   (32, 5376, 4096), (16, 6272, 2048), (7, 7552, 1552), (32, 2816, 4096),
                                   (33, 11008, 4096), (48, 4096, 1552), (64, 22016, 512), (64, 520, 4096)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.int32])
def test_decode_gemm_int8_input_bit_exact(M, N, K, out_dtype):
    """Small-M GEMM (K split over a cluster of 1..8 CTAs per 128 output
    channels; the shapes reach every cluster size and a ragged last k-block)
    with per-token scales."""
    X, Wf, b = _rand_case(M, N, K, 7 * M + N + K)
    rq, rS = oracle.quant_per_token(X)
    rwq, rws, rwc = oracle.quant_weight_per_channel(Wf)
    out = W.w8a8_gemm_dequant(dev(rq), dev(rS), dev(rwq), dev(rws), bias=dev(b), out_dtype=out_dtype)
    acc = oracle.gemm_i64(rq, rwq)
    if out_dtype == torch.int32:
        assert_same(host(out), acc.astype(np.int32), "acc")
    else:
        assert_same(host_bf16(out), oracle.f32_to_bf16(oracle.epilogue(acc, rS, rws, bias=b)), "out")


@pytest.mark.parametrize("M,N,K,ld_pad", [(3, 200, 400, 8), (32, 384, 2048, 0), (9, 12288, 4096, 0),
                                          (32, 22016, 4096, 0), (32, 4096, 11008, 0), (32, 131072, 512, 0),
                                          (12, 65536, 1024, 24), (32, 5376, 4096, 0), (7, 7552, 1552, 8),
                                          (64, 11008, 4096, 0), (40, 300, 400, 8)])
def test_decode_fused_static_ragged_and_block_shapes(M, N, K, ld_pad):
    case = synth.decode_static(M=M, N=N, K=K, seed=M + N)
    S, r, Z = W.w8a8_calibrate_static(dev_bf16(case.Xcal))
    Wq, s_w, cs = W.w8a8_quant_weight_per_channel(dev(case.W))
    bias = synth.bias(np.random.default_rng(1), N)
    Xd = dev_bf16(np.pad(case.X, ((0, 0), (0, ld_pad))))[:, :K]
    ws = W.new_workspace(M, N, K)
    outs = [W.w8a8_linear_static(Xd, S, r, Z, Wq, s_w, cs, bias=dev(bias), workspace=ws) for _ in range(2)]
    rS, rr, rZ = oracle.calibrate_static(case.Xcal)
    rwq, rws, rwc = oracle.quant_weight_per_channel(case.W)
    _, _, y = oracle.linear_decode(case.X, rr, rZ, rS, rwq, rws, rwc, bias=bias)
    for o in outs:  # the second call reuses the first call's workspace
        assert_same(host_bf16(o), oracle.f32_to_bf16(y), "out")


def test_decode_fp32_output_and_zero_point():
    M, N, K = 7, 1000, 512
    case = synth.decode_static(M=M, N=N, K=K, seed=21)
    S, r, Z = W.w8a8_calibrate_static(dev_bf16(case.Xcal))
    Wq, s_w, cs = W.w8a8_quant_weight_per_channel(dev(case.W))
    out = W.w8a8_linear_static(dev_bf16(case.X), S, r, Z, Wq, s_w, cs, out_dtype=torch.float32)
    rS, rr, rZ = oracle.calibrate_static(case.Xcal)
    rwq, rws, rwc = oracle.quant_weight_per_channel(case.W)
    _, _, y = oracle.linear_decode(case.X, rr, rZ, rS, rwq, rws, rwc)
    assert_same(host(out), y, "out")


@pytest.mark.parametrize("graph", [False, True])
def test_decode_back_to_back_calls_overlap_safely(graph):
    """Consecutive Decode linears on one stream, with no synchronization
    between them, as a Decode step issues them: each GEMM may start streaming
    its weight while the previous kernels still run, and the calls share one
    workspace. Every output must still equal the oracle's, eagerly and when
    the calls are replayed from a CUDA graph."""
    shapes = [(32, 11008, 4096), (32, 4096, 11008), (8, 4096, 4096), (32, 12288, 4096), (1, 520, 1024),
              (32, 4096, 4096)]
    layers, refs = [], []
    for i, (M, N, K) in enumerate(shapes):
        case = synth.decode_static(M=M, N=N, K=K, seed=100 + i)
        S, r, Z = W.w8a8_calibrate_static(dev_bf16(case.Xcal))
        Wq, s_w, cs = W.w8a8_quant_weight_per_channel(dev(case.W))
        Xq_in = W.w8a8_quant_per_tensor(dev_bf16(case.X), r, Z)
        layers.append((dev_bf16(case.X), S, r, Z, Wq, s_w, cs, Xq_in,
                       torch.empty((M, N), dtype=torch.bfloat16, device="cuda"),
                       torch.empty((M, N), dtype=torch.bfloat16, device="cuda")))
        rS, rr, rZ = oracle.calibrate_static(case.Xcal)
        rwq, rws, rwc = oracle.quant_weight_per_channel(case.W)
        _, _, y = oracle.linear_decode(case.X, rr, rZ, rS, rwq, rws, rwc)
        refs.append(oracle.f32_to_bf16(y))
    ws = W.new_workspace(32, 12288, 11008)

    def step():
        for X, S, r, Z, Wq, s_w, cs, Xq_in, out_a, out_b in layers:
            W.w8a8_linear_static(X, S, r, Z, Wq, s_w, cs, out=out_a, workspace=ws)
            W.w8a8_gemm_dequant(Xq_in, S, Wq, s_w, colsum=cs, Z=Z, out=out_b)

    torch.cuda.synchronize()
    if graph:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            step()
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        for Ly in layers:  # the replay must rewrite every output
            Ly[8].fill_(float("nan"))
            Ly[9].fill_(float("nan"))
        g.replay()
        g.replay()
    else:
        step()
        step()
    torch.cuda.synchronize()
    for (X, S, r, Z, Wq, s_w, cs, Xq_in, out_a, out_b), ref in zip(layers, refs):
        assert_same(host_bf16(out_a), ref, "linear_static")
        assert_same(host_bf16(out_b), ref, "gemm_dequant")


def _all_finite_bf16(rows):
    """Every finite bf16 bit pattern (65,280 of them) as [rows, K], K the next
    multiple of 16, the tail padded with +0."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    bits = bits[(bits & 0x7F80) != 0x7F80]
    K = -(-bits.size // rows // 16) * 16
    out = np.zeros(rows * K, dtype=np.uint16)
    out[:bits.size] = bits
    return out.reshape(rows, K)


@pytest.mark.parametrize("r,Z", [(1.0, 0), (0.013, -128), (127.0 / 3.5, 7), (1e-30, 127), (3.0e38, -5),
                                 (1000.0, -17)])
def test_quant_per_tensor_every_finite_bf16_value(r, Z):
    """q = clamp(rne(x * r) + Z, -128, 127) for every finite bf16 x: ties to
    even, values that overflow x * r, subnormals and signed zeros."""
    X = _all_finite_bf16(510)
    rd = torch.tensor([r], dtype=torch.float32, device="cuda")
    Zd = torch.tensor([Z], dtype=torch.int32, device="cuda")
    got = host(W.w8a8_quant_per_tensor(dev_bf16(X), rd, Zd))
    assert_same(got, oracle.quant_per_tensor(X, np.float32(r), Z), "Xq")


@pytest.mark.parametrize("M,N", [(32, 1000), (16, 1000), (24, 5000)])
def test_decode_linear_static_every_finite_bf16_activation(M, N):
    """Feed the Decode linear every finite bf16 value as its activation (rows
    of K = 2048, 4080 or 2720) and compare the outputs with the oracle's
    quantize -> GEMM -> epilogue: the first two shapes quantize inside the GEMM
    kernel, the third with the separate quantization kernel."""
    X = _all_finite_bf16(M)
    K = X.shape[1]
    case = synth.decode_static(M=M, N=N, K=K, seed=5)
    S, r, Z = W.w8a8_calibrate_static(dev_bf16(case.Xcal))
    Wq, s_w, cs = W.w8a8_quant_weight_per_channel(dev(case.W))
    out = W.w8a8_linear_static(dev_bf16(X), S, r, Z, Wq, s_w, cs, out_dtype=torch.float32)
    rS, rr, rZ = oracle.calibrate_static(case.Xcal)
    rwq, rws, rwc = oracle.quant_weight_per_channel(case.W)
    _, _, y = oracle.linear_decode(X, rr, rZ, rS, rwq, rws, rwc)
    assert_same(host(out), y, "out")


# ------------------------------------------------------------ static requantization for the next linear


def _next_linear_params(y_bf16, shrink=0.7):
    """The next linear's static (S, r, Z): the oracle's MinMax over this
    layer's bf16 result, the range narrowed so that both ends saturate."""
    yf = oracle.bf16_to_f32(y_bf16)
    cal = oracle.f32_to_bf16(np.clip(yf, shrink * yf.min(), shrink * yf.max()))
    return oracle.calibrate_static(cal)


@pytest.mark.parametrize("M,N,K,ld_pad", [(1, 4096, 4096, 0), (16, 11008, 4096, 0), (32, 4096, 4096, 0),
                                          (32, 11008, 4096, 0), (3, 1001, 400, 8), (48, 300, 400, 8),
                                          (64, 520, 2048, 0), (24, 5000, 1024, 0), (33, 4104, 512, 0)])
def test_decode_requant_bit_exact(M, N, K, ld_pad):
    """w8a8_linear_static_requant: the next linear's int8 codes of this
    linear's bf16 result equal the oracle's, in the one-kernel form (M <= 16,
    or M <= 32 with N <= 4096) and with the separate quantization kernel, on
    ragged N (rows of Xq_out not 8-byte aligned) and padded activation rows."""
    case = synth.decode_static(M=M, N=N, K=K, seed=3 * M + N)
    rS, rr, rZ = oracle.calibrate_static(case.Xcal)
    rwq, rws, rwc = oracle.quant_weight_per_channel(case.W)
    bias = synth.bias(np.random.default_rng(2), N)
    _, _, _, y_bf16, _ = oracle.linear_decode_requant(case.X, rr, rZ, rS, rwq, rws, rwc, np.float32(1), 0,
                                                      bias=bias)
    _, r2, Z2 = _next_linear_params(y_bf16)
    q_ref = oracle.linear_decode_requant(case.X, rr, rZ, rS, rwq, rws, rwc, r2, Z2, bias=bias)[4]
    assert (q_ref == 127).any() and (q_ref == -128).any()

    S, r, Z = W.w8a8_calibrate_static(dev_bf16(case.Xcal))
    Wq, s_w, cs = W.w8a8_quant_weight_per_channel(dev(case.W))
    Xd = dev_bf16(np.pad(case.X, ((0, 0), (0, ld_pad))))[:, :K]
    r2d = torch.tensor([r2], dtype=torch.float32, device="cuda")
    Z2d = torch.tensor([Z2], dtype=torch.int32, device="cuda")
    ws = W.new_workspace(M, N, K)
    q = W.w8a8_linear_static_requant(Xd, S, r, Z, Wq, s_w, cs, r2d, Z2d, bias=dev(bias), workspace=ws)
    assert q.dtype == torch.int8 and tuple(q.shape) == (M, N)
    assert_same(host(q), q_ref, "Xq_out")
    if N % 16 == 0:  # the same as the two calls it replaces (quantization rows are multiples of 16)
        out = W.w8a8_linear_static(Xd, S, r, Z, Wq, s_w, cs, bias=dev(bias), workspace=ws)
        assert torch.equal(q, W.w8a8_quant_per_tensor(out, r2d, Z2d))


@pytest.mark.parametrize("graph", [False, True])
def test_decode_requant_chain_of_linears(graph):
    """Three Decode linears chained on one stream with no synchronization:
    linear 1 quantizes bf16 X and hands int8 codes to linear 2
    (w8a8_linear_static_requant), linear 2 takes codes and hands codes on
    (w8a8_gemm_requant), linear 3 takes codes and writes bf16
    (w8a8_gemm_dequant), each with its own static S, Z. Each kernel may start its weight stream while the previous
    one runs; every result must equal the oracle's chain."""
    M, widths = 32, [2048, 4096, 1024, 3000]
    rng = np.random.default_rng(44)
    Xcal = synth.calibration_tokens(rng, 256, widths[0])
    X = synth.calibration_tokens(rng, M, widths[0])
    Ws = [synth.weight(np.random.default_rng(50 + i), widths[i], widths[i + 1]) for i in range(3)]
    # oracle chain; each next linear calibrated on the previous one's bf16 result
    S1, r1, Z1 = oracle.calibrate_static(Xcal)
    qs = [oracle.quant_weight_per_channel(w) for w in Ws]
    y1 = oracle.linear_decode_requant(X, r1, Z1, S1, *qs[0], np.float32(1), 0)[3]
    S2, r2, Z2 = _next_linear_params(y1, 0.8)
    q1 = oracle.linear_decode_requant(X, r1, Z1, S1, *qs[0], r2, Z2)[4]
    acc2 = oracle.gemm_i64(q1, qs[1][0])
    y2 = oracle.f32_to_bf16(oracle.epilogue(acc2, np.float32(S2), qs[1][1], colsum=qs[1][2], Z=Z2))
    S3, r3, Z3 = _next_linear_params(y2, 0.8)
    q2 = oracle.quant_per_tensor(y2, r3, Z3)
    y3 = oracle.f32_to_bf16(oracle.epilogue(oracle.gemm_i64(q2, qs[2][0]), np.float32(S3), qs[2][1],
                                            colsum=qs[2][2], Z=Z3))

    def scal(v, dt):
        return torch.tensor([v], dtype=dt, device="cuda")
    Xd = dev_bf16(X)
    S1d, r1d, Z1d = W.w8a8_calibrate_static(dev_bf16(Xcal))
    S2d, r2d, Z2d = scal(S2, torch.float32), scal(r2, torch.float32), scal(Z2, torch.int32)
    S3d, r3d, Z3d = scal(S3, torch.float32), scal(r3, torch.float32), scal(Z3, torch.int32)
    wd = [W.w8a8_quant_weight_per_channel(dev(w)) for w in Ws]
    ws = W.new_workspace(M, max(widths), max(widths))
    q1d = torch.empty((M, widths[1]), dtype=torch.int8, device="cuda")
    q2d = torch.empty((M, widths[2]), dtype=torch.int8, device="cuda")
    y3d = torch.empty((M, widths[3]), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()

    def step():
        W.w8a8_linear_static_requant(Xd, S1d, r1d, Z1d, *wd[0], r2d, Z2d, out=q1d, workspace=ws)
        W.w8a8_gemm_requant(q1d, S2d, wd[1][0], wd[1][1], r3d, Z3d, colsum=wd[1][2], Z=Z2d, out=q2d)
        W.w8a8_gemm_dequant(q2d, S3d, wd[2][0], wd[2][1], colsum=wd[2][2], Z=Z3d, out=y3d)

    if graph:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            step()
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        q1d.fill_(-99)  # the replay must rewrite every output
        q2d.fill_(-99)
        y3d.fill_(float("nan"))
        g.replay()
        g.replay()
    else:
        step()
        step()
    torch.cuda.synchronize()
    assert_same(host(q1d), q1, "codes for linear 2")
    assert_same(host(q2d), q2, "codes for linear 3")
    assert_same(host_bf16(y3d), y3, "linear 3")


def test_gemm_requant_per_token_scales_and_bias():
    """w8a8_gemm_requant with one scale per token (a per-token quantized
    activation), no zero point and a bias: the codes equal the oracle's
    epilogue -> bf16 -> static quantization, on a ragged N."""
    M, N, K = 20, 1000, 512
    rng = np.random.default_rng(31)
    X = synth.activations(rng, M, K, with_outliers=True)
    Wf = synth.weight(rng, K, N)
    bias = synth.bias(rng, N)
    rxq, rS = oracle.quant_per_token(X)
    rwq, rws, _ = oracle.quant_weight_per_channel(Wf)
    y_bf16 = oracle.f32_to_bf16(oracle.epilogue(oracle.gemm_i64(rxq, rwq), rS, rws, bias=bias))
    _, r2, Z2 = _next_linear_params(y_bf16)
    q_ref = oracle.quant_per_tensor(y_bf16, r2, Z2)
    Xq, S_x = W.w8a8_quant_per_token(dev_bf16(X))
    Wq, s_w, _ = W.w8a8_quant_weight_per_channel(dev(Wf))
    r2d = torch.tensor([r2], dtype=torch.float32, device="cuda")
    Z2d = torch.tensor([Z2], dtype=torch.int32, device="cuda")
    q = W.w8a8_gemm_requant(Xq, S_x, Wq, s_w, r2d, Z2d, bias=dev(bias))
    assert_same(host(q), q_ref, "Xq_out")


# ------------------------------------------------------------ static dequantization (INT8 KV cache)


@pytest.mark.parametrize("S,Z", [(0.5, -128), (0.013, 7), (3.0e-3, 127), (250.0, -5)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_dequant_every_code(S, Z, out_dtype):
    """x = S (q - Z) for every int8 code, in rows with a padded stride."""
    codes = np.tile(np.arange(-128, 128).astype(np.int8), (5, 2))  # [5, 512]
    Xd = dev(np.pad(codes, ((0, 0), (0, 32))))[:, :512]
    Sd = torch.tensor([S], dtype=torch.float32, device="cuda")
    Zd = torch.tensor([Z], dtype=torch.int32, device="cuda")
    got = W.w8a8_dequant_per_tensor(Xd, Sd, Zd, out_dtype=out_dtype)
    if out_dtype == torch.bfloat16:
        assert_same(host_bf16(got), oracle.dequant_per_tensor(codes, np.float32(S), Z), "bf16")
    else:
        assert_same(host(got), oracle.dequant_per_tensor(codes, np.float32(S), Z, oracle.DT_FP32), "fp32")


@pytest.mark.parametrize("M,K", [(1, 16), (7, 4112), (4096, 4096), (333, 1024)])
def test_kv_cache_round_trip(M, K):
    """A KV-cache tensor quantized with the Decode scheme and read back:
    the GPU's codes and bf16 values equal the oracle's."""
    rng = np.random.default_rng(M + K)
    cal = synth.activations(rng, 64, K, with_outliers=True)
    X = synth.activations(rng, M, K, with_outliers=True)
    S, r, Z = W.w8a8_calibrate_static(dev_bf16(cal))
    q = W.w8a8_quant_per_tensor(dev_bf16(X), r, Z)
    back = W.w8a8_dequant_per_tensor(q, S, Z)
    rS, rr, rZ = oracle.calibrate_static(cal)
    rq = oracle.quant_per_tensor(X, rr, rZ)
    assert_same(host(q), rq, "codes")
    assert_same(host_bf16(back), oracle.dequant_per_tensor(rq, rS, rZ), "values")


@pytest.mark.parametrize("M,K", [(4099, 1040), (2048, 2048)])
def test_static_quant_and_dequant_stream_path_bit_exact(M, K):
    """Dense tensors of 4M elements or more take the kernels that stream
    16 KiB tiles through shared memory with bulk copies: codes and values
    equal the oracle's, with every finite bf16 value in the input and a
    total size (4099 x 1040) that is not a whole number of tiles."""
    finite = _all_finite_bf16(1).reshape(-1)
    reps = -(-(M * K) // finite.size)
    X = np.tile(finite, reps)[:M * K].reshape(M, K)
    case = synth.decode_static(M=1, N=16, K=K, seed=M)
    S, r, Z = W.w8a8_calibrate_static(dev_bf16(case.Xcal))
    rS, rr, rZ = oracle.calibrate_static(case.Xcal)
    q = W.w8a8_quant_per_tensor(dev_bf16(X), r, Z)
    rq = oracle.quant_per_tensor(X, rr, rZ)
    assert_same(host(q), rq, "codes")
    assert_same(host_bf16(W.w8a8_dequant_per_tensor(q, S, Z)), oracle.dequant_per_tensor(rq, rS, rZ), "bf16 values")
    assert_same(host(W.w8a8_dequant_per_tensor(q, S, Z, out_dtype=torch.float32)),
                oracle.dequant_per_tensor(rq, rS, rZ, oracle.DT_FP32), "fp32 values")
