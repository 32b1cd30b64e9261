"""w8a8_linear_static_noalloc -- the Decode linear for callers that cannot
allocate device memory (a graph under capture, a plug-in in a runtime that
owns the memory, a step that cannot afford an allocation's synchronization).

It must give exactly what w8a8_linear_static gives (the tests here hold every
output to bit equality), on consecutive calls that share the library's one
scratch array. Called through the C ABI with raw device pointers. This file
is collected last and has no state shared with the other test files, so it
passes alone in a fresh process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

from int8_gemm_token_b200 import synth
from int8_gemm_token_b200 import w8a8 as W

pytestmark = pytest.mark.gpu


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _noalloc_call(X, S, r, Z, Wq, s_w, colsum, bias, out, stream):
    M, K = X.shape
    N = Wq.shape[0]
    return W.lib().w8a8_linear_static_noalloc(
        X.data_ptr(), M, K, X.stride(0), S.data_ptr(), r.data_ptr(), Z.data_ptr(), Wq.data_ptr(),
        s_w.data_ptr(), colsum.data_ptr(), None if bias is None else bias.data_ptr(), N, out.data_ptr(),
        W.BF16 if out.dtype == torch.bfloat16 else W.FP32, ctypes.c_void_p(stream.cuda_stream))


def _synthetic_layer(M, N, K, seed):
    """Calibrated static S, r, Z and a per-channel INT8 weight, made on the GPU."""
    case = synth.decode_static(M=M, N=16, K=K, seed=seed)
    S, r, Z = W.w8a8_calibrate_static(_bf16(case.Xcal))
    g = torch.Generator(device="cuda").manual_seed(seed)
    Wf = torch.randn((K, N), generator=g, device="cuda", dtype=torch.float32) * 0.02
    Wq, s_w, colsum = W.w8a8_quant_weight_per_channel(Wf)
    bias = torch.randn((N,), generator=g, device="cuda", dtype=torch.float32) * 0.01
    return _bf16(case.X), S, r, Z, Wq, s_w, colsum, bias


@pytest.mark.parametrize("M,N,K", [(32, 11008, 4096), (5, 1000, 512), (1, 4096, 4096), (32, 32768, 16384)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_noalloc_matches_linear_static_on_consecutive_calls(M, N, K, out_dtype):
    X, S, r, Z, Wq, s_w, colsum, bias = _synthetic_layer(M, N, K, seed=M + N + K)
    stream = torch.cuda.current_stream()
    ref = W.w8a8_linear_static(X, S, r, Z, Wq, s_w, colsum, bias=bias, out_dtype=out_dtype)
    for call in range(2):  # the second call reuses the scratch the first one left behind
        out = torch.full((M, N), float("nan"), dtype=out_dtype, device="cuda")
        assert _noalloc_call(X, S, r, Z, Wq, s_w, colsum, bias, out, stream) == W.OK
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32),
                           ref.view(torch.int16 if out_dtype == torch.bfloat16 else torch.int32)), f"call {call}"
    assert W.w8a8_check_device_error() == 0


def test_noalloc_rejects_shapes_beyond_its_scratch():
    X, S, r, Z, Wq, s_w, colsum, bias = _synthetic_layer(4, 64, 128, seed=1)
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
    assert L.w8a8_linear_static_noalloc(*args) == W.OK
    torch.cuda.synchronize()
    assert W.w8a8_check_device_error() == 0
