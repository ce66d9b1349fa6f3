"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke run.

This module only draws random numbers and packs them into the storage formats
the block consumes (bf16 bit patterns, e4m3 bytes with a per-output-row fp32
scale).  It holds none of the block's arithmetic: positions, norms, rotary
angles, attention and the Euler update are computed separately by the CUDA
path and by the fp64 oracle.

Shapes and distributions follow the workloads the Ideogram 4 pages describe:
a 13 x 4096 concatenated text-encoder feature per token (SimpleTuner Ideogram 4
quickstart, "Text Embed Cache"), a 64 x 64 latent grid of 128-channel tokens at
1024 px (Ideogram 4 deep dive, section 4-5 on the VAE and 2x2 patching), FP8
e4m3 weights with a per-output-channel ``weight_scale`` (unsloth
diffusion_ideogram4.py commit log, fp8 loader commit) and the fused
``attention.qkv.weight`` of shape [3*hidden, hidden].

Seeds are ``1000 * config_index + tensor_id``; every tensor has its own PCG64
stream so any one of them can be regenerated alone.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Tuple

import numpy as np
import torch

E4M3_MAX = 448.0


@dataclasses.dataclass(frozen=True)
class BlockShape:
    """Sizes of one single-stream DiT block workload."""

    name: str
    index: int
    batch: int
    n_text: int
    grid_h: int
    grid_w: int
    d_model: int
    n_heads: int
    head_dim: int
    d_mlp: int
    rope_sections: Tuple[int, int, int]  # rotary pairs per axis (t, h, w)
    rope_theta: float = 10000.0
    eps: float = 1e-6
    gelu_tanh: int = 0

    @property
    def n_img(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def seq(self) -> int:
        return self.n_text + self.n_img

    def flops(self) -> float:
        """Dense algorithmic FLOPs of one block forward (GEMMs + attention)."""
        s, d, f = self.seq, self.d_model, self.d_mlp
        return float(self.batch) * (2.0 * s * (3 * d * d + d * d + 2 * d * f) + 4.0 * s * s * d)


@dataclasses.dataclass(frozen=True)
class CondShape:
    """Sizes of the frozen llm_cond_norm / llm_cond_proj projection."""

    name: str
    index: int
    n_tok: int
    n_layers: int
    hidden: int
    d_out: int
    eps: float = 1e-6

    @property
    def k(self) -> int:
        return self.n_layers * self.hidden

    def flops(self) -> float:
        return 2.0 * self.n_tok * self.k * self.d_out


# The five workloads.  Sections count rotary PAIRS and sum to head_dim / 2.
TINY = BlockShape("tiny", 0, 1, 16, 8, 8, 256, 4, 64, 1024, (8, 12, 12))
COND = CondShape("cond", 1, 512, 13, 4096, 4096)
C1024 = BlockShape("c1024", 2, 1, 512, 64, 64, 4096, 32, 128, 16384, (24, 20, 20))
UNCOND1024 = BlockShape("uncond1024", 3, 1, 32, 64, 64, 4096, 32, 128, 16384, (24, 20, 20))
C2048 = BlockShape("c2048", 4, 1, 512, 128, 128, 4096, 32, 128, 16384, (24, 20, 20))
LATENT_CHANNELS = 128
CFG_GUIDANCE = 4.0
CFG_DT = -1.0 / 50.0

BLOCKS: Dict[str, BlockShape] = {b.name: b for b in (TINY, C1024, UNCOND1024, C2048)}


def rng(config_index: int, tensor_id: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(1000 * config_index + tensor_id))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32/fp64 values to bf16 (round-to-nearest-even) and return the uint16 bits."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def quantize_rows_e4m3(w: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per-output-row e4m3 quantisation of a synthetic weight [out, in].

    scale_row = amax_row / 448 in fp32 (rows that are all zero get scale 1), and
    the stored byte is e4m3(w / scale_row) rounded to nearest even and clamped
    to +-448.  Only the bytes and scales reach the block.
    """
    w = np.asarray(w, dtype=np.float32)
    amax = np.abs(w).max(axis=1).astype(np.float32)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    q = np.clip(w / scale[:, None], -E4M3_MAX, E4M3_MAX).astype(np.float32)
    codes = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, scale


def normal(config_index: int, tensor_id: int, shape, std: float = 1.0, mean: float = 0.0) -> np.ndarray:
    return (rng(config_index, tensor_id).standard_normal(size=shape, dtype=np.float32) * std + mean).astype(np.float32)


def block_inputs(shape: BlockShape, *, zero_text: bool = False) -> Dict[str, np.ndarray]:
    """Activations, FP8 weights + scales and gains of one block.

    Tensor ids: 0 x; 1-4 w_qkv, w_o, w_up, w_down; 5-8 g_norm1, g_norm2, g_q, g_k.
    x ~ N(0, 1) bf16 [batch, seq, d] (text rows first); weights ~ N(0, 0.02)
    quantised per output row; gains ~ 1 + N(0, 0.05) bf16.
    """
    c, d, f, hd = shape.index, shape.d_model, shape.d_mlp, shape.head_dim
    x = normal(c, 0, (shape.batch, shape.seq, d))
    if zero_text:
        x[:, : shape.n_text, :] = 0.0
    out = {"x": to_bf16_bits(x)}
    for tid, (name, rows, cols) in enumerate(
        (("w_qkv", 3 * d, d), ("w_o", d, d), ("w_up", f, d), ("w_down", d, f)), start=1
    ):
        codes, scale = quantize_rows_e4m3(normal(c, tid, (rows, cols), std=0.02))
        out[name] = codes
        out["s_" + name[2:]] = scale
    for tid, (name, n) in enumerate((("g_norm1", d), ("g_norm2", d), ("g_q", hd), ("g_k", hd)), start=5):
        out[name] = to_bf16_bits(normal(c, tid, (n,), std=0.05, mean=1.0))
    return out


def cond_inputs(shape: CondShape = COND, n_tok: int | None = None) -> Dict[str, np.ndarray]:
    """Raw 13-layer text features [n_tok, 13*4096] bf16 ~ N(0, 1), gain, FP8 projection weight.

    Tensor ids: 0 feats, 1 w, 2 g.
    """
    n = shape.n_tok if n_tok is None else n_tok
    c = shape.index
    feats = to_bf16_bits(normal(c, 0, (n, shape.k)))
    codes, scale = quantize_rows_e4m3(normal(c, 1, (shape.d_out, shape.k), std=0.02))
    g = to_bf16_bits(normal(c, 2, (shape.k,), std=0.05, mean=1.0))
    return {"feats": feats, "w": codes, "scale": scale, "g": g}


def euler_inputs(n: int, config_index: int = 3) -> Dict[str, np.ndarray]:
    """Latent state x fp32 ~ N(0, 1) and the two velocities bf16 ~ N(0, 1).

    Tensor ids: 10 x, 11 v_cond, 12 v_uncond.
    """
    return {
        "x": normal(config_index, 10, (n,)),
        "v_cond": to_bf16_bits(normal(config_index, 11, (n,))),
        "v_uncond": to_bf16_bits(normal(config_index, 12, (n,))),
    }


def block_weights_device(shape: BlockShape, seed: int, device) -> Dict[str, "torch.Tensor"]:
    """FP8 weights, scales and gains of one block drawn directly on a CUDA device (torch's own
    generator, so not the numpy streams above): for throughput runs that cycle through many
    distinct weight sets, where drawing hundreds of MB on the host would dominate.  Same
    distributions and the same per-output-row quantisation as ``block_inputs``; bf16 gains are
    returned as int16 bit patterns, like the host path's uint16 arrays on the device."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    d, f, hd = shape.d_model, shape.d_mlp, shape.head_dim
    out = {}
    for name, rows, cols in (("w_qkv", 3 * d, d), ("w_o", d, d), ("w_up", f, d), ("w_down", d, f)):
        w = torch.randn((rows, cols), generator=gen, device=device, dtype=torch.float32) * 0.02
        amax = w.abs().amax(dim=1)
        scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
        q = (w / scale[:, None]).clamp_(-E4M3_MAX, E4M3_MAX)
        out[name] = q.to(torch.float8_e4m3fn).view(torch.uint8).contiguous()
        out["s_" + name[2:]] = scale.contiguous()
        del w, q
    for name, n in (("g_norm1", d), ("g_norm2", d), ("g_q", hd), ("g_k", hd)):
        g = 1.0 + 0.05 * torch.randn((n,), generator=gen, device=device, dtype=torch.float32)
        out[name] = g.to(torch.bfloat16).view(torch.int16).contiguous()
    return out


def bf16_normal_device(shape, seed: int, device, std: float = 1.0) -> "torch.Tensor":
    """bf16 ~ N(0, std^2) activations drawn on the device (int16 bit patterns)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return (torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std).to(
        torch.bfloat16).view(torch.int16)
