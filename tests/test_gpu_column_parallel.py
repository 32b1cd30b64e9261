"""The column-parallel layer on one GPU through its default CUDA operations:
with a single process (a group of one) its Prefill and Decode outputs must
equal the library's own calls and the oracle, bit for bit. The sharding and
the gather across ranks are covered on CPU with gloo ranks."""
import numpy as np
import pytest
import torch

import oracle
from int8_gemm_token_b200 import synth
from int8_gemm_token_b200 import w8a8 as W
from int8_gemm_token_b200.column_parallel import ColumnParallelW8A8Linear
from tests.gpu_util import dev_bf16, host_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,N", [(300, 512, 1000), (24, 256, 4096)])
def test_single_gpu_layer_matches_the_library_and_the_oracle(M, K, N):
    rng = np.random.default_rng(M + K + N)
    X = synth.activations(rng, M, K, with_outliers=True)
    Wf = synth.weight(rng, K, N)
    b = synth.bias(rng, N)
    cal = synth.calibration_tokens(rng, 64, K)
    layer = ColumnParallelW8A8Linear.from_weight(torch.from_numpy(Wf).cuda(), torch.from_numpy(b).cuda())
    assert (layer.n0, layer.n1, layer.world) == (0, N, 1)
    Xd = dev_bf16(X)
    # Prefill
    y = layer.prefill(Xd, gather=True)
    Xq, S_x = W.w8a8_quant_per_token(Xd)
    y_lib = W.w8a8_gemm_dequant(Xq, S_x, layer.Wq, layer.s_w, bias=layer.bias)
    assert torch.equal(y.view(torch.int16), y_lib.view(torch.int16))
    rwq, rws, rwc = oracle.quant_weight_per_channel(Wf)
    _, _, _, yr = oracle.linear_prefill(X, rwq, rws, bias=b)
    assert np.array_equal(host_bf16(y), oracle.f32_to_bf16(yr))
    # Decode with the static scales of the calibration tokens
    S, r, Z = W.w8a8_calibrate_static(dev_bf16(cal))
    yd = layer.decode(Xd[:16].contiguous(), S, r, Z, gather=True)
    rS, rr, rZ = oracle.calibrate_static(cal)
    _, _, ydr = oracle.linear_decode(X[:16], rr, rZ, rS, rwq, rws, rwc, bias=b)
    assert np.array_equal(host_bf16(yd), oracle.f32_to_bf16(ydr))
    assert W.w8a8_check_device_error() == 0
