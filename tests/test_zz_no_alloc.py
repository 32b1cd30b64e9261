"""w8a8_linear_static_noalloc -- the Decode linear for callers that cannot
allocate device memory when they run a step: a plug-in inside a runtime that
owns every byte of device memory, or a latency-critical step that cannot take
the device-wide synchronization an allocation may cause.

It must give exactly what w8a8_linear_static gives (every output here is held
to bit equality with it, and with the oracle), on consecutive calls that share
the library's one scratch array. Called through the C ABI with raw device
pointers. This file is collected last and shares no state with the other test
files, so it passes alone in a fresh process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from int8_gemm_token_b200 import synth
from int8_gemm_token_b200 import w8a8 as W

pytestmark = pytest.mark.gpu

_CODES = {torch.bfloat16: W.BF16, torch.float32: W.FP32, torch.int32: W.I32}


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _noalloc_call(X, S, r, Z, Wq, s_w, colsum, bias, out, stream):
    M, K = X.shape
    N = Wq.shape[0]
    return W.lib().w8a8_linear_static_noalloc(
        X.data_ptr(), M, K, X.stride(0), S.data_ptr(), r.data_ptr(), Z.data_ptr(), Wq.data_ptr(),
        s_w.data_ptr(), colsum.data_ptr(), None if bias is None else bias.data_ptr(), N, out.data_ptr(),
        _CODES[out.dtype], ctypes.c_void_p(stream.cuda_stream))


def _synthetic_layer(M, N, K, seed):
    """Seeded Decode inputs (bf16 bits), their static calibration and weight."""
    case = synth.decode_static(M=M, N=N, K=K, seed=seed)
    bias = synth.bias(np.random.default_rng(seed), N)
    return case, bias


def _bits(t):
    return t.view({torch.bfloat16: torch.int16, torch.float32: torch.int32, torch.int32: torch.int32}[t.dtype])


@pytest.mark.parametrize("M,N,K,ld_pad,with_bias", [(32, 11008, 4096, 0, True), (5, 1000, 512, 0, True),
                                                    (1, 4096, 4096, 0, True), (32, 32768, 16384, 0, True),
                                                    (7, 520, 1040, 24, False)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32, torch.int32])
def test_noalloc_matches_linear_static_on_consecutive_calls(M, N, K, ld_pad, with_bias, out_dtype):
    case, bias_h = _synthetic_layer(M, N, K, seed=M + N + K)
    S, r, Z = W.w8a8_calibrate_static(_bf16(case.Xcal))
    Wq, s_w, colsum = W.w8a8_quant_weight_per_channel(torch.from_numpy(case.W).cuda())
    bias = torch.from_numpy(bias_h).cuda() if with_bias else None
    X = _bf16(np.pad(case.X, ((0, 0), (0, ld_pad))))[:, :K]  # rows of stride K + ld_pad
    stream = torch.cuda.current_stream()
    ref = W.w8a8_linear_static(X, S, r, Z, Wq, s_w, colsum, bias=bias, out_dtype=out_dtype)
    for call in range(2):  # the second call reuses the scratch the first one left behind
        out = torch.full((M, N), -7, dtype=out_dtype, device="cuda")
        assert _noalloc_call(X, S, r, Z, Wq, s_w, colsum, bias, out, stream) == W.OK
        torch.cuda.synchronize()
        assert torch.equal(_bits(out), _bits(ref)), f"call {call}: differs from w8a8_linear_static"
    # and both equal the oracle's Decode linear
    rS, rr, rZ = oracle.calibrate_static(case.Xcal)
    rwq, rws, rwc = oracle.quant_weight_per_channel(case.W)
    rxq, acc, y = oracle.linear_decode(case.X, rr, rZ, rS, rwq, rws, rwc, bias=bias_h if with_bias else None)
    got = out.cpu().numpy() if out_dtype != torch.bfloat16 else out.view(torch.int16).cpu().numpy().view(np.uint16)
    if out_dtype == torch.int32:
        want = (acc - int(rZ) * rwc.astype(np.int64)[None, :]).astype(np.int32)
    elif out_dtype == torch.float32:
        want = y
        got, want = got.view(np.uint32), want.view(np.uint32)
    else:
        want = oracle.f32_to_bf16(y)
    assert np.array_equal(got, want), "differs from the oracle"
    assert W.w8a8_check_device_error() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    case, _ = _synthetic_layer(4, 64, 128, seed=1)
    S, r, Z = W.w8a8_calibrate_static(_bf16(case.Xcal))
    Wq, s_w, colsum = W.w8a8_quant_weight_per_channel(torch.from_numpy(case.W).cuda())
    X = _bf16(case.X)
    out = torch.empty((4, 64), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()
    L = W.lib()
    args = [X.data_ptr(), 4, 128, 128, S.data_ptr(), r.data_ptr(), Z.data_ptr(), Wq.data_ptr(), s_w.data_ptr(),
            colsum.data_ptr(), None, 64, out.data_ptr(), W.BF16, ctypes.c_void_p(stream.cuda_stream)]
    too_many_tokens = list(args)
    too_many_tokens[1] = 33
    assert L.w8a8_linear_static_noalloc(*too_many_tokens) == 3  # W8A8_ERR_UNSUPPORTED_SHAPE
    too_wide = list(args)
    too_wide[11] = 32768 + 128
    assert L.w8a8_linear_static_noalloc(*too_wide) == 3
    too_deep = list(args)
    too_deep[2] = too_deep[3] = 16384 + 16
    assert L.w8a8_linear_static_noalloc(*too_deep) == 3
    assert L.w8a8_linear_static_noalloc(*args) == W.OK
    torch.cuda.synchronize()
    assert W.w8a8_check_device_error() == 0
