"""Helpers shared by the GPU parity tests: device transfer of bit patterns and the tolerance checks."""
import numpy as np
import torch

import oracle

# Block and projection outputs (bf16): max|d| / max|ref| <= 2e-2 and mean|d| / mean|ref| <= 3e-3.
MAX_REL = 2e-2
MEAN_REL = 3e-3


def dev(a: np.ndarray) -> torch.Tensor:
    """numpy (uint16 bf16 bits, uint8 codes, float32, int32) -> contiguous CUDA tensor with the same bytes."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        t = torch.from_numpy(a.view(np.int16))
    else:
        t = torch.from_numpy(a)
    return t.cuda()


def bits(t: torch.Tensor) -> np.ndarray:
    """CUDA tensor holding bf16 bit patterns -> numpy uint16."""
    return t.cpu().numpy().view(np.uint16)


def as_f64(t: torch.Tensor) -> np.ndarray:
    return oracle.bf16_to_f64(bits(t))


def assert_close(got: np.ndarray, ref: np.ndarray, max_rel: float = MAX_REL, mean_rel: float = MEAN_REL, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    d = np.abs(got - ref)
    mx = d.max() / max(np.abs(ref).max(), 1e-30)
    mn = d.mean() / max(np.abs(ref).mean(), 1e-30)
    assert mx <= max_rel and mn <= mean_rel, f"{what}: max-rel {mx:.3e} (<= {max_rel}), mean-rel {mn:.3e} (<= {mean_rel})"
    return mx, mn


def empty_bf16(*shape) -> torch.Tensor:
    return torch.empty(*shape, dtype=torch.int16, device="cuda")


def workspace(nbytes: int) -> torch.Tensor:
    """Device scratch filled with 0xFF bytes (NaN in every 16- and 32-bit float format), so that a
    kernel reading scratch it has not written shows up as a non-finite output."""
    return torch.full((max(int(nbytes), 256),), 0xFF, dtype=torch.uint8, device="cuda")


def poisoned_like(t: torch.Tensor) -> torch.Tensor:
    """An output buffer of t's shape filled with 0xFF bytes (NaN as bf16, f16 and fp32)."""
    out = torch.empty_like(t)
    out.view(torch.uint8).fill_(0xFF)
    return out
