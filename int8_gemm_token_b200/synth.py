"""Seeded synthetic inputs for the W8A8 linear layer.

These generators stand in for LLM activations and weights (no dataset or
trained weights are used). They only draw random numbers and arrange them;
none of the layer's arithmetic (scales, rounding, zero points, GEMM) lives
here, so the same bytes can feed both the CUDA path and the CPU oracle.

Distributions follow the workloads the pages describe:
  - activations: N(0, 1) with each row scaled by exp(N(0, 0.5)) (row-scaled,
    per-token dynamic range), optionally with a few fixed feature channels
    multiplied by 60 -- the emergent outlier features of the LLM.int8()
    summary (§二, about six hidden dimensions far above the rest);
  - weights: N(0, 0.02); bias: N(0, 0.01);
  - decode calibration data: ReLU of the row-scaled activations plus 0.5, so
    that its range is one-sided and the zero point is far from 0;
  - LLM.int8() decomposition input: N(0, 1) with 6-8 fixed outlier columns
    whose entries are a random sign times U(20, 100).

bf16 values are returned as numpy uint16 bit patterns, made by torch's
float32 -> bfloat16 cast (round to nearest even). Float32 arrays stay float32.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

OUTLIER_GAIN = 60.0


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 array -> bf16 bit patterns (uint16), rounded by torch's cast."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 (exact widening)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def row_scaled_normal(rng: np.random.Generator, M: int, K: int) -> np.ndarray:
    """N(0,1) [M, K] with each row multiplied by exp(N(0, 0.5)) (float32)."""
    z = rng.standard_normal((M, K), dtype=np.float32)
    row = np.exp(rng.normal(0.0, 0.5, size=(M, 1))).astype(np.float32)
    return z * row


def outlier_channels(K: int, count: int = 6, seed: int = 12345) -> np.ndarray:
    """Fixed feature-channel indices for a layer input of width K."""
    return np.sort(np.random.default_rng(seed + K).choice(K, count, replace=False)).astype(np.int64)


def activations(rng: np.random.Generator, M: int, K: int, with_outliers: bool = False) -> np.ndarray:
    """Row-scaled activations as bf16 bits; optional x60 outlier channels."""
    x = row_scaled_normal(rng, M, K)
    if with_outliers:
        x[:, outlier_channels(K)] *= OUTLIER_GAIN
    return bf16_bits(x)


def weight(rng: np.random.Generator, K: int, N: int) -> np.ndarray:
    """W [K, N] float32 ~ N(0, 0.02)."""
    return (rng.standard_normal((K, N), dtype=np.float32) * np.float32(0.02)).astype(np.float32)


def bias(rng: np.random.Generator, N: int) -> np.ndarray:
    return (rng.standard_normal((N,), dtype=np.float32) * np.float32(0.01)).astype(np.float32)


def calibration_tokens(rng: np.random.Generator, T: int, K: int) -> np.ndarray:
    """ReLU(row-scaled N(0,1)) + 0.5 as bf16 bits: one-sided, shifted range."""
    x = np.maximum(row_scaled_normal(rng, T, K), np.float32(0.0)) + np.float32(0.5)
    return bf16_bits(x)


def push_past_range(rng: np.random.Generator, x_bits: np.ndarray, hi: float, frac: float = 0.01) -> np.ndarray:
    """Replace `frac` of the entries (seeded positions): half by 2*hi, half by
    -hi, where hi is the largest calibration value. Both ends then fall
    outside any range calibrated on that data."""
    x = bits_to_f32(x_bits).copy().reshape(-1)
    n = max(2, int(round(frac * x.size)))
    pos = rng.choice(x.size, n, replace=False)
    x[pos[: n // 2]] = np.float32(2.0 * hi)
    x[pos[n // 2:]] = np.float32(-hi)
    return bf16_bits(x.reshape(x_bits.shape))


# --------------------------------------------------------------------------
# The five workloads.
# --------------------------------------------------------------------------

@dataclass
class PrefillCase:
    X: np.ndarray          # bf16 bits [M, K]
    W: np.ndarray          # float32 [K, N]
    bias: np.ndarray | None


def prefill_small(seed: int = 0) -> PrefillCase:
    """Single linear, prefill: X [16, 256] row-scaled, W [256, 512], bias."""
    rng = np.random.default_rng(seed)
    X = activations(rng, 16, 256)
    W = weight(rng, 256, 512)
    b = bias(rng, 512)
    return PrefillCase(X, W, b)


def prefill_7b(seed: int = 0, M: int = 2048, K: int = 4096, N: int = 11008) -> PrefillCase:
    """Prefill at 7B shapes: X [2048, 4096] with 6 x60 channels, W [4096, 11008], bias."""
    rng = np.random.default_rng(seed)
    X = activations(rng, M, K, with_outliers=True)
    W = weight(rng, K, N)
    b = bias(rng, N)
    return PrefillCase(X, W, b)


@dataclass
class DecodeCase:
    Xcal: np.ndarray       # bf16 bits [512, K]
    X: np.ndarray          # bf16 bits [M, K] with 1% pushed past the range
    W: np.ndarray          # float32 [K, N]


def decode_static(M: int, N: int, K: int = 4096, seed: int = 0, T: int = 512) -> DecodeCase:
    """Decode with a static per-tensor scale: calibration tokens (seed + 1),
    decode tokens of the same distribution (seed), 1% pushed past the range."""
    rng_cal = np.random.default_rng(seed + 1)
    Xcal = calibration_tokens(rng_cal, T, K)
    hi = float(bits_to_f32(Xcal).max())
    rng = np.random.default_rng(seed)
    X = push_past_range(rng, calibration_tokens(rng, M, K), hi)
    W = weight(np.random.default_rng(seed + 7 + N), K, N)
    return DecodeCase(Xcal, X, W)


BLOCK_LINEARS = (("qkv", 4096, 12288), ("o", 4096, 4096), ("gate_up", 4096, 22016), ("down", 11008, 4096))


@dataclass
class BlockLinear:
    name: str
    K: int
    N: int
    seed: int

    def weight(self) -> np.ndarray:
        return weight(np.random.default_rng(self.seed), self.K, self.N)

    def calibration(self, T: int = 512) -> np.ndarray:
        return activations(np.random.default_rng(self.seed + 1), T, self.K, with_outliers=True)

    def prefill_input(self, M: int = 4096) -> np.ndarray:
        return activations(np.random.default_rng(self.seed + 2), M, self.K, with_outliers=True)

    def decode_input(self, step: int, M: int = 32) -> np.ndarray:
        return activations(np.random.default_rng(1000 + step + 100000 * self.seed), M, self.K, with_outliers=True)


def pdmix_block(seed: int = 0) -> list[BlockLinear]:
    """Llama-7B-like block linears; each has its own weight and inputs."""
    return [BlockLinear(name, K, N, seed * 10 + i) for i, (name, K, N) in enumerate(BLOCK_LINEARS)]


@dataclass
class MixedCase:
    X: np.ndarray          # bf16 bits [M, K]
    W: np.ndarray          # bf16 bits [K, N]
    cols: np.ndarray       # planted outlier columns
    threshold: float = 6.0


def llm_int8(seed: int = 0, M: int = 4096, K: int = 8192, N: int = 8192) -> MixedCase:
    """X ~ N(0,1) with 6-8 fixed outlier columns of sign * U(20, 100); W bf16 N(0, 0.02)."""
    rng = np.random.default_rng(seed)
    n_cols = int(rng.choice([6, 7, 8]))
    cols = np.sort(rng.choice(K, n_cols, replace=False)).astype(np.int64)
    x = rng.standard_normal((M, K), dtype=np.float32)
    mag = rng.uniform(20.0, 100.0, size=(M, n_cols)).astype(np.float32)
    sign = np.where(rng.random((M, n_cols)) < 0.5, np.float32(-1.0), np.float32(1.0))
    x[:, cols] = sign * mag
    W = bf16_bits(weight(rng, K, N))
    return MixedCase(bf16_bits(x), W, cols)
