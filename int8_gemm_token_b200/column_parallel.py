"""Column-parallel W8A8 linear across the GPUs of one node (N-sharding).

The output channels n of the layer are split into contiguous ranges, one per
rank. Because every quantity of the layer that depends on n -- the weight's
per-channel scale s_w[n], its codes Wq[n, :], colsum[n], bias[n] and the
output column out[:, n] -- is computed from that channel alone, each rank can
quantize only its own columns of W at load time and compute only its own
output columns, with no exchange at all:

  * Prefill: every rank holds the whole activation X [M, K] and computes the
    per-token scales S_x itself (identical on every rank: the absmax of a
    token row does not depend on N), then its [M, n1 - n0] slice of the
    output (PDMIX glossary §2.3 eq. Q_prefill; LLM.int8() summary steps
    (3)-(4): the rescale is the outer product S_x[m] s_w[n], so a column
    slice of the output needs only the matching slice of s_w).
  * Decode: the static S, r, Z are scalars of the whole tensor, shared by all
    ranks (eq. Q_decode), and each rank runs the Decode linear on its slice.

Only when a caller asks for the full output is there a collective: one
all-gather of the output slices over the process group (NCCL over NVLink /
NVSwitch between GPUs). Every kernel reads only its own GPU's memory; no
tensor map or library kernel is given another GPU's memory.

The compute calls go through `ops`, by default the CUDA library
(`CudaOps`, the C ABI of include/w8a8.h). There is no CPU path in this
module: the argument exists so that tests can drive the sharding and gather
logic with another implementation of the same five calls.

The pages' one multi-GPU remark (LLM.int8() summary §三: BLOOM-176B fits on
4 instead of 8 A100s with 8-bit weights) concerns memory, not a partition;
the N-split is the partition under which the method stays exact.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

# Shard boundaries fall on multiples of this many output channels, so each
# slice of Wq, s_w, colsum and bias starts 16-byte aligned (and on a 128-row
# weight tile of the kernels whenever N allows it).
SHARD_ALIGN = 128


def shard_range(N: int, world: int, rank: int, align: int = SHARD_ALIGN) -> tuple[int, int]:
    """Columns [n0, n1) of output rank `rank` of `world`: equal widths of
    ceil(N / world) rounded up to `align`, the last shard ragged (possibly
    empty when N is small)."""
    if world <= 0 or not 0 <= rank < world or N < 0:
        raise ValueError(f"bad shard request N={N} world={world} rank={rank}")
    per = -(-N // world)
    per = -(-per // align) * align if per > 0 else 0
    n0 = min(N, rank * per)
    n1 = min(N, n0 + per)
    return n0, n1


def shard_width(N: int, world: int, align: int = SHARD_ALIGN) -> int:
    """The padded width every rank contributes to the all-gather."""
    return shard_range(N, world, 0, align)[1] if N else 0


class CudaOps:
    """The five calls of the layer, on the CUDA library (include/w8a8.h)."""

    def __init__(self):
        from . import w8a8
        self.W = w8a8
        w8a8.lib()  # fail loudly now if the library is missing

    def quant_weight_per_channel(self, W):
        return self.W.w8a8_quant_weight_per_channel(W)

    def quant_per_token(self, X):
        return self.W.w8a8_quant_per_token(X)

    def gemm_dequant(self, Xq, S_x, Wq, s_w, bias):
        return self.W.w8a8_gemm_dequant(Xq, S_x, Wq, s_w, bias=bias)

    def linear_static(self, X, S, r, Z, Wq, s_w, colsum, bias):
        return self.W.w8a8_linear_static(X, S, r, Z, Wq, s_w, colsum, bias=bias)

    def empty_out(self, M, N, like):
        return torch.empty((M, N), dtype=torch.bfloat16, device=like.device)


class ColumnParallelW8A8Linear:
    """One W8A8 linear layer whose output channels are split over the ranks
    of `group` (the default process group when None; a single process works
    as a group of one)."""

    def __init__(self, N: int, K: int, n0: int, n1: int, Wq, s_w, colsum, bias, group=None, ops=None):
        self.N, self.K, self.n0, self.n1 = N, K, n0, n1
        self.Wq, self.s_w, self.colsum, self.bias = Wq, s_w, colsum, bias
        self.group = group
        self.ops = ops if ops is not None else CudaOps()
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0

    @classmethod
    def from_weight(cls, W: torch.Tensor, bias: torch.Tensor | None = None, group=None, ops=None):
        """Quantize this rank's columns of the full weight W [K, N] (the
        same tensor on every rank, or at least the same columns). Per-channel
        quantization of a column slice equals the slice of the full
        quantization, so no rank needs the others' columns."""
        world = dist.get_world_size(group) if dist.is_initialized() else 1
        rank = dist.get_rank(group) if dist.is_initialized() else 0
        K, N = W.shape
        n0, n1 = shard_range(N, world, rank)
        ops = ops if ops is not None else CudaOps()
        if n1 > n0:
            Wq, s_w, colsum = ops.quant_weight_per_channel(W[:, n0:n1].contiguous())
            b = None if bias is None else bias[n0:n1].contiguous()
        else:
            Wq = s_w = colsum = b = None
        return cls(N, K, n0, n1, Wq, s_w, colsum, b, group=group, ops=ops)

    @property
    def local_width(self) -> int:
        return self.n1 - self.n0

    def prefill(self, X: torch.Tensor, gather: bool = False) -> torch.Tensor:
        """Per-token dynamic quantization of the whole X [M, K] on this rank,
        then this rank's output columns [M, n1 - n0] (bf16); with gather=True
        the full [M, N] output, all-gathered from every rank."""
        M = X.shape[0]
        if self.local_width > 0:
            Xq, S_x = self.ops.quant_per_token(X)
            out = self.ops.gemm_dequant(Xq, S_x, self.Wq, self.s_w, self.bias)
        else:
            out = self.ops.empty_out(M, 0, X)
        return self.all_gather(out) if gather else out

    def decode(self, X: torch.Tensor, S, r, Z, gather: bool = False) -> torch.Tensor:
        """The Decode linear with the layer's static per-tensor S, r, Z (the
        same scalars on every rank) on this rank's columns."""
        M = X.shape[0]
        if self.local_width > 0:
            out = self.ops.linear_static(X, S, r, Z, self.Wq, self.s_w, self.colsum, self.bias)
        else:
            out = self.ops.empty_out(M, 0, X)
        return self.all_gather(out) if gather else out

    def all_gather(self, out_local: torch.Tensor) -> torch.Tensor:
        """Full [M, N] output from every rank's [M, n1 - n0] slice: each rank
        pads its slice to the common shard width, one all-gather of
        [world, M, width], then the slices are laid side by side."""
        M = out_local.shape[0]
        if self.world == 1:
            return out_local
        width = shard_width(self.N, self.world)  # a multiple of SHARD_ALIGN: even
        send = out_local.new_zeros((M, width))
        send[:, :self.local_width] = out_local
        # exchanged as raw 32-bit words (two bf16 values each): the bits move as they are
        words = send.view(torch.int32) if send.element_size() == 2 else send
        parts = [torch.empty_like(words) for _ in range(self.world)]
        dist.all_gather(parts, words, group=self.group)
        full = torch.cat([p_.view(send.dtype) for p_ in parts], dim=1)[:, :self.N].contiguous()
        return full
