"""Host <-> device helpers for the GPU parity tests (BF16 kept as uint16 bits on the host)."""

import numpy as np
import torch


def dev():
    return torch.device("cuda", 0)


def to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev())


def bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def i32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev())


def f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev())


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def max_rel_err(got_bits: np.ndarray, ref_bits: np.ndarray) -> float:
    """Largest |g - r| / |r| over elements (|g| itself where r == 0)."""
    g = bf16_to_f32(got_bits).astype(np.float64)
    r = bf16_to_f32(ref_bits).astype(np.float64)
    err = np.abs(g - r)
    den = np.abs(r)
    rel = np.where(den > 0, err / np.where(den > 0, den, 1), err)
    return float(rel.max(initial=0.0))


COMBINE_TOL = 2.0 ** -7   # max relative error per element, the contract for combine
