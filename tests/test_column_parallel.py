"""Column-parallel (N-sharded) W8A8 linear: the partition and the gather, on
CPU with gloo ranks.

The product class runs its per-rank compute on the CUDA library; here the
same five calls are answered by the oracle (on CPU tensors) so that the
sharding logic -- which columns each rank quantizes and computes, and how
the slices are gathered -- is checked without a GPU: every rank's slice and
the gathered output must equal the oracle's unsharded layer bit for bit.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from int8_gemm_token_b200.column_parallel import SHARD_ALIGN, shard_range, shard_width  # noqa: E402


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


class OracleOps:
    """The layer's five calls answered by the CPU oracle (test only)."""

    def __init__(self):
        import oracle
        self.o = oracle

    def quant_weight_per_channel(self, W):
        Wn = W.numpy() if W.dtype == torch.float32 else _bits(W)
        q, s, c = self.o.quant_weight_per_channel(Wn)
        return torch.from_numpy(q), torch.from_numpy(s), torch.from_numpy(c)

    def quant_per_token(self, X):
        q, s = self.o.quant_per_token(_bits(X))
        return torch.from_numpy(q), torch.from_numpy(s)

    def gemm_dequant(self, Xq, S_x, Wq, s_w, bias):
        acc = self.o.gemm_i64(Xq.numpy(), Wq.numpy())
        y = self.o.epilogue(acc, S_x.numpy(), s_w.numpy(), bias=None if bias is None else bias.numpy())
        return _bf16(self.o.f32_to_bf16(y))

    def linear_static(self, X, S, r, Z, Wq, s_w, colsum, bias):
        _, _, y = self.o.linear_decode(_bits(X), r.numpy()[0], Z.numpy()[0], S.numpy()[0], Wq.numpy(),
                                       s_w.numpy(), colsum.numpy(), bias=None if bias is None else bias.numpy())
        return _bf16(self.o.f32_to_bf16(y))

    def empty_out(self, M, N, like):
        return torch.empty((M, N), dtype=torch.bfloat16)


def _layer(M, K, N, seed):
    from int8_gemm_token_b200 import synth
    rng = np.random.default_rng(seed)
    X = synth.activations(rng, M, K, with_outliers=True)
    W = synth.weight(rng, K, N)
    b = synth.bias(rng, N)
    cal = synth.calibration_tokens(rng, 64, K)
    return X, W, b, cal


CASES = [(24, 256, 1000), (5, 128, 100)]  # N = 100 over 2 ranks: rank 1's shard is empty


def _rank_main(rank, world, port, q):
    import torch.distributed as dist

    import oracle
    from int8_gemm_token_b200.column_parallel import ColumnParallelW8A8Linear
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        res = []
        for i, (M, K, N) in enumerate(CASES):
            X, W, b, cal = _layer(M, K, N, seed=i)
            layer = ColumnParallelW8A8Linear.from_weight(torch.from_numpy(W), torch.from_numpy(b), ops=OracleOps())
            local = layer.prefill(_bf16(X))
            full = layer.prefill(_bf16(X), gather=True)
            S, r, Z = oracle.calibrate_static(cal)
            dec_full = layer.decode(_bf16(X), torch.tensor([S]), torch.tensor([r]), torch.tensor([Z]), gather=True)
            res.append((layer.n0, layer.n1, _bits(local), _bits(full), _bits(dec_full),
                        None if layer.Wq is None else layer.Wq.numpy(), None if layer.s_w is None else layer.s_w.numpy()))
        dist.barrier()
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_shard_columns_and_gather_exactly():
    import oracle
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        while len(got) < world:
            try:
                rank, res = q.get(timeout=5)
                got[rank] = res
            except Exception:
                assert all(p.exitcode in (None, 0) for p in procs), "a rank failed"
    finally:
        for p in procs:
            p.join(60)
            if p.exitcode is None:
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    for i, (M, K, N) in enumerate(CASES):
        X, W, b, cal = _layer(M, K, N, seed=i)
        wq, sw, cs = oracle.quant_weight_per_channel(W)
        _, _, _, y = oracle.linear_prefill(X, wq, sw, bias=b)
        want = oracle.f32_to_bf16(y)
        S, r, Z = oracle.calibrate_static(cal)
        _, _, yd = oracle.linear_decode(X, r, Z, S, wq, sw, cs, bias=b)
        want_dec = oracle.f32_to_bf16(yd)
        covered = []
        for rank in range(world):
            n0, n1, local, full, dec_full, Wq_r, sw_r = got[rank][i]
            assert (n0, n1) == shard_range(N, world, rank)
            covered.extend(range(n0, n1))
            assert np.array_equal(local, want[:, n0:n1]), f"case {i} rank {rank}: local slice"
            assert np.array_equal(full, want), f"case {i} rank {rank}: gathered prefill output"
            assert np.array_equal(dec_full, want_dec), f"case {i} rank {rank}: gathered decode output"
            if n1 > n0:  # quantizing a column slice = slicing the full quantization
                assert np.array_equal(Wq_r, wq[n0:n1]) and np.array_equal(sw_r, sw[n0:n1])
        assert covered == list(range(N))


@pytest.mark.parametrize("N", [0, 1, 100, 128, 1000, 4096, 11008, 22016, 12345])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_ranges_partition_the_columns(N, world):
    ranges = [shard_range(N, world, r) for r in range(world)]
    width = shard_width(N, world)
    pos = 0
    for n0, n1 in ranges:
        assert n0 == pos and n0 <= n1 and n1 - n0 <= width
        assert n0 % SHARD_ALIGN == 0 or n0 == N  # slices start on a weight-tile boundary
        pos = n1
    assert pos == N


def test_single_process_layer_needs_no_group():
    from int8_gemm_token_b200.column_parallel import ColumnParallelW8A8Linear
    import oracle
    X, W, b, _ = _layer(6, 128, 300, seed=5)
    layer = ColumnParallelW8A8Linear.from_weight(torch.from_numpy(W), torch.from_numpy(b), ops=OracleOps())
    assert (layer.n0, layer.n1, layer.world) == (0, 300, 1)
    wq, sw, _ = oracle.quant_weight_per_channel(W)
    _, _, _, y = oracle.linear_prefill(X, wq, sw, bias=b)
    assert np.array_equal(_bits(layer.prefill(_bf16(X), gather=True)), oracle.f32_to_bf16(y))
