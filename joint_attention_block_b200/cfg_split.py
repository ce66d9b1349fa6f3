"""A denoising step with the two guidance branches on two GPUs.

The conditional and the unconditional branch of a step use separate weights (Ideogram 4 deep
dive, section 4-4: asymmetric CFG with a separate unconditional DiT; section 4-6: both DiTs run
at every step), so they split across two ranks with no sharing of weights or activations.  Per
step each rank runs its own branch on the same latent z, the two velocities are exchanged once
(an all-gather of [batch, n_img, d] bf16 per rank), and both ranks apply the same CFG + Euler
update, so z stays identical on both without a second exchange.

    rank 0: v_c = stack_cond  ([text_cond;   bf16(z)])[image rows]
    rank 1: v_u = stack_uncond([text_uncond; bf16(z)])[image rows]
    both:   (v_c, v_u) = all_gather(v_rank);  z = z + dt (v_u + gw (v_c - v_u))

``SplitStep`` holds the exchange and its ordering; the compute is passed in, so the same logic
runs with the CUDA library (``gpu_branch`` and ``gpu_update``, NCCL) and, in tests, with plain
CPU functions over gloo.
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch
import torch.distributed as dist

COND, UNCOND = 0, 1


class SplitStep:
    """One rank's side of the two-rank split.  Rank 0 runs the conditional branch, rank 1 the
    unconditional one; every collective is issued by both ranks in the same order."""

    def __init__(self, group=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if self.world != 2:
            raise ValueError(f"the CFG-branch split runs on exactly 2 ranks, got {self.world}")
        self.branch = COND if self.rank == 0 else UNCOND

    def exchange(self, v: torch.Tensor):
        """(v_cond, v_uncond) on both ranks from this rank's velocity (contiguous, same shape on both)."""
        v = v.contiguous()
        raw = v.reshape(-1).view(torch.uint8)  # raw bytes: every backend gathers uint8 (gloo has no 16-bit ints)
        parts = [torch.empty_like(raw) for _ in range(2)]
        dist.all_gather(parts, raw, group=self.group)
        return tuple(p.view(v.dtype).view(v.shape) for p in (parts[COND], parts[UNCOND]))

    def run(self, z: torch.Tensor, branch_velocity: Callable[[torch.Tensor, int], torch.Tensor],
            update: Callable[[torch.Tensor, torch.Tensor, torch.Tensor, float, float], None],
            guidance: Sequence[float], dts: Sequence[float]) -> torch.Tensor:
        """len(guidance) steps; ``branch_velocity(z, branch)`` returns this branch's velocity,
        ``update(z, v_c, v_u, gw, dt)`` applies the CFG + Euler step to z in place."""
        if len(guidance) != len(dts):
            raise ValueError("one dt per guidance weight")
        for gw, dt in zip(guidance, dts):
            v = branch_velocity(z, self.branch)
            v_c, v_u = self.exchange(v)
            update(z, v_c, v_u, float(gw), float(dt))
        return z


def gpu_branch(cfg, weights, text, n_text: int, grid_h: int, grid_w: int, x: torch.Tensor, out: torch.Tensor,
               workspace: torch.Tensor, stream=None) -> Callable[[torch.Tensor, int], torch.Tensor]:
    """This rank's branch through the CUDA library: tokens from the latent, the block stack, and
    the image rows of its output (batch 1, so they are one contiguous slice)."""
    from . import _abi as ops

    def run(z: torch.Tensor, branch: int) -> torch.Tensor:
        if z.shape[0] != 1:
            raise ValueError("gpu_branch exchanges one contiguous image-row slice: batch 1")
        ops.tokens_from_latent(z, text, x, stream=stream)
        ops.dit_stack_forward(cfg, weights, x, out, n_text, grid_h, grid_w, workspace, stream=stream)
        return out[0, n_text:]

    return run


def gpu_update(stream=None) -> Callable[[torch.Tensor, torch.Tensor, torch.Tensor, float, float], None]:
    """The CFG + Euler update through euler_cfg_step (flat fp32 latent, bf16 velocities)."""
    from . import _abi as ops

    def run(z, v_c, v_u, gw, dt):
        ops.euler_cfg_step(z.view(-1), v_c.reshape(-1), v_u.reshape(-1), gw, dt, stream=stream)

    return run
