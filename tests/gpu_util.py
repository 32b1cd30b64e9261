"""Helpers for the GPU parity tests: move seeded numpy inputs to the device
and bring results back as numpy arrays in the oracle's representation."""
import numpy as np
import torch


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    """bf16 bit patterns (uint16) -> CUDA bfloat16 tensor with the same bits."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.cuda()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_bf16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().numpy()


def diff_report(a: np.ndarray, b: np.ndarray, limit: int = 5) -> str:
    bad = np.argwhere(a != b)
    rows = [f"{tuple(i)}: gpu={a[tuple(i)]} oracle={b[tuple(i)]}" for i in bad[:limit]]
    return f"{len(bad)} mismatches; first: " + "; ".join(rows)
