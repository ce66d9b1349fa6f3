"""Plain fp64 CPU oracle of the Ideogram 4 single-stream DiT block hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The CUDA library never
calls it, and it shares no code with the CUDA path: inputs arrive as raw bf16
bit patterns, e4m3 bytes and fp32 scales, and every decode, norm, rotation and
product below is written out here in float64 with numpy.  A library matmul is
used as the contraction step; nothing is blocked, fused or reordered beyond
what each definition states.

Sources, by page and section:

* unsloth ``diffusion_ideogram4.py`` commit log, fp8 loader commit: weights are
  float8_e4m3 (range +-448) with a per-output-channel ``weight_scale``; the real
  weight is ``fp8.float() * weight_scale[:, None]``; attention is stored fused as
  ``attention.qkv.weight`` [3*hidden, hidden] with Q, K, V rows stacked in that
  order, plus ``attention.o.weight``.
* Ideogram 4.0 announcement thread (digg.com): a single-stream DiT with
  self-attention, QK-RMSNorm and 3D multimodal RoPE placing text and image
  tokens in one positional frame; 13 hidden states concatenated on features.
* Ideogram 4 deep dive (ai-news-5min-kr), section 4-2: text and image tokens are
  one sequence through the same self-attention; section 6-3: ``mrope_section =
  (24, 20, 20)``; section 4-6: the CFG combine ``gw*v_cond + (1-gw)*v_uncond``
  and the Euler update ``z + v*(s - t)``.
* SimpleTuner Ideogram 4 quickstart (Japanese), "Text Embed Cache": the frozen
  ``llm_cond_norm`` / ``llm_cond_proj`` project 13 * 4096 = 53,248 raw features
  per token.

Readings where the pages are silent (each is also a runtime parameter):
RMSNorm is ``x / sqrt(mean(x^2) + eps) * g`` with eps = 1e-6; rotary sections
count frequency pairs and are laid out contiguously (t, then h, then w);
``inv_freq_i = fp32(theta^(-2i/hd))``, theta = 1e4, rotate-half pairing
(i, i + hd/2); text token j sits at (j, j, j) and image cell (r, c) at
(t_img, r, c) with t_img = n_text; softmax scale 1/sqrt(hd); the block is
sequential pre-norm ``x1 = x + Attn(RMSNorm(x))``, ``y = x1 + MLP(RMSNorm(x1))``
with no biases and an exact-erf GELU MLP.  The W8A8 variant (not on the pages) rounds the two
pre-norm outputs to e4m3 per token (scale amax / 448) and q, k (taken from their f16 storage, after
the QK-norm and the rotations) to e4m3 with one static scale each, sqrt(hd) * max|g| / 448.
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np
from scipy.special import erf

# ---------------------------------------------------------------- decoding


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns: bf16 is the top half of an IEEE binary32."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    """Exact value of OCP float8 e4m3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits).

    Exponent field 0 is subnormal (m/8 * 2^-6); there is no infinity; S.1111.111 is
    NaN, so the largest finite magnitude is 1.75 * 2^8 = 448 (the +-448 range the
    fp8 loader commit quotes).
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c & 0x80) != 0, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    val = sign * np.where(e == 0, sub, normal)
    return np.where((e == 0xF) & ((c & 0x7) == 0x7), np.nan, val)


def e4m3_round(v: np.ndarray) -> np.ndarray:
    """Nearest e4m3 value (ties to even), saturating at +-448, written from the format: a finite
    magnitude in [2^e, 2^(e+1)) with e >= -6 has 3 fraction bits, so the spacing there is
    2^(e-3); below 2^-6 the subnormal spacing is 2^-9; 448 = 1.75 * 2^8 is the largest value."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    _, ex = np.frexp(a)  # a = m * 2^ex with m in [0.5, 1), so the binary exponent is ex - 1
    e = np.maximum(ex - 1, -6)
    step = np.exp2(e.astype(np.float64) - 3.0)
    q = np.round(a / step) * step  # numpy rounds halves to even; a / step is exact in fp64
    return np.sign(v) * np.minimum(q, 448.0)


def quantize_rows_act(h: np.ndarray):
    """Per-token e4m3 quantisation of activations [rows, cols]: scale_row = fp32(amax_row / 448)
    (1 for an all-zero row), values e4m3_round(h / scale_row).  Returns (dequantised values, scales);
    the product of a code and its scale is exact in fp64."""
    h = np.asarray(h, dtype=np.float64)
    amax = np.abs(h).max(axis=-1, keepdims=True)
    scale = np.where(amax > 0, amax / 448.0, 1.0).astype(np.float32).astype(np.float64)
    return e4m3_round(h / scale) * scale, scale[..., 0]


def qk_e4m3_scale(g: np.ndarray, head_dim: int) -> float:
    """Static e4m3 scale of the normalised, rotated q (or k) of the W8A8 variant: after the per-head
    RMSNorm a head vector has Euclidean norm at most sqrt(hd) * max|g| (its mean square before the
    gain is at most 1), and each rotation of a pair (i, i + hd/2) keeps that norm, so no component
    exceeds it.  Dividing by sqrt(hd) * max|g| / 448 therefore never leaves the e4m3 range.  Each
    step is rounded to fp32: the scale is an fp32 number the kernels share."""
    s = np.float32(np.sqrt(np.float32(head_dim)))
    s = np.float32(s * np.float32(np.abs(np.asarray(g, dtype=np.float64)).max()))
    return float(np.float32(s / np.float32(448.0)))


def quantize_qk(x: np.ndarray, scale: float) -> np.ndarray:
    """q or k of the W8A8 variant as the attention product sees them: e4m3_round(x / scale) * scale."""
    return e4m3_round(np.asarray(x, dtype=np.float64) / scale) * scale


def dequant(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """Real weight = fp8 value * weight_scale[:, None] (scale indexed by output row)."""
    return e4m3_to_f64(codes) * np.asarray(scale, dtype=np.float32).astype(np.float64)[:, None]


# ---------------------------------------------------------------- pieces


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * g."""
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * g


def gelu(x: np.ndarray, tanh: bool = False) -> np.ndarray:
    """GELU: x * Phi(x) with the exact erf (default), or the tanh approximation."""
    if tanh:
        return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def mrope_positions(n_text: int, grid_h: int, grid_w: int, t_img: Optional[int] = None) -> np.ndarray:
    """(t, h, w) per token of the joint sequence [text; image].

    Text token j gets (j, j, j); image cell (r, c), stored in raster order r*grid_w + c
    after the text rows, gets (t_img, r, c) with t_img = n_text unless given.
    """
    if t_img is None or t_img < 0:
        t_img = n_text
    pos = np.zeros((n_text + grid_h * grid_w, 3), dtype=np.int64)
    j = np.arange(n_text)
    pos[:n_text] = j[:, None]
    r, c = np.divmod(np.arange(grid_h * grid_w), grid_w)
    pos[n_text:, 0] = t_img
    pos[n_text:, 1] = r
    pos[n_text:, 2] = c
    return pos


def inv_freq(head_dim: int, theta: float) -> np.ndarray:
    """Rotary inverse frequencies theta^(-2i/hd), i < hd/2, held in fp32 as the loader keeps them."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return (theta ** (-2.0 * i / head_dim)).astype(np.float32).astype(np.float64)


def mrope_angles(pos: np.ndarray, head_dim: int, sections: Sequence[int], theta: float) -> np.ndarray:
    """Angle [S, hd/2]: pair i takes the position of its axis (t, h or w, by contiguous sections)."""
    s_t, s_h, s_w = sections
    assert s_t + s_h + s_w == head_dim // 2, "rotary sections must sum to head_dim/2 pairs"
    axis = np.array([0] * s_t + [1] * s_h + [2] * s_w)
    p = np.asarray(pos, dtype=np.float64)[:, axis]  # [S, hd/2]
    return p * inv_freq(head_dim, theta)[None, :]


def mrope(x: np.ndarray, pos: np.ndarray, sections: Sequence[int], theta: float) -> np.ndarray:
    """Rotate x [S, H, hd] pairwise: pair (i, i + hd/2) by the angle of pair i."""
    hd = x.shape[-1]
    half = hd // 2
    ang = mrope_angles(pos, hd, sections, theta)[:, None, :]  # [S, 1, hd/2]
    cos, sin = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * cos - x2 * sin, x2 * cos + x1 * sin], axis=-1)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, key_valid: Optional[np.ndarray] = None) -> np.ndarray:
    """Bidirectional softmax attention per head; q [Sq, H, hd], k/v [S, H, hd] -> [Sq, H, hd].

    ``key_valid`` (bool [S]), when given, removes the other keys (padding) from every row's
    softmax: their logits are -inf, so they get weight exactly 0."""
    hd = q.shape[-1]
    out = np.empty((q.shape[0], q.shape[1], v.shape[-1]), dtype=np.float64)
    for h in range(q.shape[1]):
        s = q[:, h, :] @ k[:, h, :].T / math.sqrt(hd)
        if key_valid is not None:
            s = np.where(np.asarray(key_valid, dtype=bool)[None, :], s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ v[:, h, :]
    return out


# ---------------------------------------------------------------- the three calls


def dit_block_forward(
    cfg,
    w: Dict[str, np.ndarray],
    x_bits: np.ndarray,
    n_text: int,
    grid_h: int,
    grid_w: int,
    t_img: Optional[int] = None,
    rows: Optional[np.ndarray] = None,
    pos: Optional[np.ndarray] = None,
    text_lens: Optional[Sequence[int]] = None,
    w8a8: bool = False,
) -> np.ndarray:
    """One single-stream DiT block forward, fp64, for x [B, S, d] (bf16 bits) -> [B, S, d].

    ``w8a8`` quantises the inputs of the QKV and MLP-up projections (the two pre-norm outputs)
    to e4m3 per token (quantize_rows_act) before the FP8-weight products, as an FP8-activation
    pipeline would, and the normalised, rotated q and k to e4m3 with one static scale each
    (qk_e4m3_scale, quantize_qk) before q k^T, taken from q and k as the QKV product stores them
    (f16); P V and the other products keep 16-bit activations.

    ``cfg`` carries d_model, n_heads, head_dim, d_mlp, rope_sections, rope_theta,
    eps, gelu_tanh.  ``w`` holds e4m3 codes w_qkv [3d, d], w_o [d, d], w_up [F, d],
    w_down [d, F], fp32 scales s_qkv, s_o, s_up, s_down and bf16 gains g_norm1,
    g_norm2 [d], g_q, g_k [hd].  With ``rows`` given only those query rows are
    computed (K and V still cover every token) and the result is [B, len(rows), d].

    ``text_lens`` (one per batch element, each <= n_text) makes a padded batch of prompts of
    different lengths: element b holds its text_lens[b] text rows, then its grid_h*grid_w image
    rows, then n_text - text_lens[b] rows of padding at the end.  Each element is positioned as
    if alone (text j at (j, j, j), image cell (r, c) at (text_lens[b], r, c) unless t_img is
    given), padding rows are excluded as keys, and their own outputs are not defined (returned
    as computed).
    """
    d, nh, hd = cfg.d_model, cfg.n_heads, cfg.head_dim
    eps = cfg.eps
    x_all = bf16_to_f64(x_bits)
    S = n_text + grid_h * grid_w
    assert x_all.shape[1] == S and x_all.shape[2] == d
    if pos is None:
        pos = mrope_positions(n_text, grid_h, grid_w, t_img)
    W_qkv = dequant(w["w_qkv"], w["s_qkv"])
    W_o = dequant(w["w_o"], w["s_o"])
    W_up = dequant(w["w_up"], w["s_up"])
    W_dn = dequant(w["w_down"], w["s_down"])
    g1, g2 = bf16_to_f64(w["g_norm1"]), bf16_to_f64(w["g_norm2"])
    gq, gk = bf16_to_f64(w["g_q"]), bf16_to_f64(w["g_k"])
    sel = np.arange(S) if rows is None else np.asarray(rows)
    outs = []
    for b in range(x_all.shape[0]):
        x = x_all[b]
        key_valid = None
        pos_b = pos
        if text_lens is not None:
            L = int(text_lens[b])
            assert 0 <= L <= n_text
            n_valid = L + grid_h * grid_w
            key_valid = np.arange(S) < n_valid
            pos_b = np.zeros((S, 3), dtype=np.int64)
            pos_b[:n_valid] = mrope_positions(L, grid_h, grid_w, L if t_img is None else t_img)
        h = rmsnorm(x, g1, eps)
        if w8a8:
            h = quantize_rows_act(h)[0]
        # K and V for every token, Q only for the requested rows.
        k = (h @ W_qkv[d : 2 * d].T).reshape(S, nh, hd)
        v = (h @ W_qkv[2 * d :].T).reshape(S, nh, hd)
        q = (h[sel] @ W_qkv[:d].T).reshape(len(sel), nh, hd)
        if w8a8:
            # the variant rounds q and k to e4m3 after the QK-norm; it takes them from the
            # 16-bit (f16, round to nearest even) values its QKV product stores
            q = q.astype(np.float16).astype(np.float64)
            k = k.astype(np.float16).astype(np.float64)
        q = rmsnorm(q, gq, eps)
        k = rmsnorm(k, gk, eps)
        q = mrope(q, pos_b[sel], cfg.rope_sections, cfg.rope_theta)
        k = mrope(k, pos_b, cfg.rope_sections, cfg.rope_theta)
        if w8a8:
            q = quantize_qk(q, qk_e4m3_scale(gq, hd))
            k = quantize_qk(k, qk_e4m3_scale(gk, hd))
        o = attention(q, k, v, key_valid).reshape(len(sel), d)
        x1 = x[sel] + o @ W_o.T
        h2 = rmsnorm(x1, g2, eps)
        if w8a8:
            h2 = quantize_rows_act(h2)[0]
        u = gelu(h2 @ W_up.T, tanh=bool(cfg.gelu_tanh))
        outs.append(x1 + u @ W_dn.T)
    return np.stack(outs)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round values to bf16 (nearest, ties to even) and return the bit patterns.

    Goes through binary32 (round to nearest even), then keeps the top 16 bits with
    round-to-nearest-even on the dropped half; NaN stays NaN.
    """
    b = np.asarray(x, dtype=np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    r = ((b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float64))
    return np.where(nan, np.uint16(0x7FC0), r).astype(np.uint16)


def dit_stack_forward(
    cfg,
    ws: Sequence[Dict[str, np.ndarray]],
    x_bits: np.ndarray,
    n_text: int,
    grid_h: int,
    grid_w: int,
    t_img: Optional[int] = None,
    pos: Optional[np.ndarray] = None,
) -> np.ndarray:
    """Blocks applied in order, each taking the previous block's output as its bf16 input
    (the DiT stacks 34 single-stream blocks: Ideogram 4.0 announcement thread; a block's
    input and output are bf16 tensors).  Returns the last block's fp64 output."""
    cur = np.asarray(x_bits, dtype=np.uint16)
    out = None
    for i, w in enumerate(ws):
        out = dit_block_forward(cfg, w, cur, n_text, grid_h, grid_w, t_img=t_img, pos=pos)
        if i + 1 < len(ws):
            cur = f64_to_bf16_bits(out)
    return out


def cond_proj_forward(feats_bits: np.ndarray, g_bits: np.ndarray, eps: float, codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    """llm_cond_norm then llm_cond_proj: RMSNorm over the 13*4096 concatenated features, then the FP8 projection."""
    n = rmsnorm(bf16_to_f64(feats_bits), bf16_to_f64(g_bits), eps)
    return n @ dequant(codes, scale).T


def euler_cfg_step(x: np.ndarray, v_cond_bits: np.ndarray, v_uncond_bits: np.ndarray, guidance: float, dt: float) -> np.ndarray:
    """Dual-branch CFG then one Euler step: x + dt * (gw*v_c + (1-gw)*v_u), dt = s - t."""
    vc, vu = bf16_to_f64(v_cond_bits), bf16_to_f64(v_uncond_bits)
    v = guidance * vc + (1.0 - guidance) * vu
    return np.asarray(x, dtype=np.float64) + v * dt


def denoise_steps(
    cfg,
    ws_cond: Sequence[Dict[str, np.ndarray]],
    ws_uncond: Sequence[Dict[str, np.ndarray]],
    text_cond_bits: np.ndarray,
    text_uncond_bits: np.ndarray,
    z: np.ndarray,
    grid_h: int,
    grid_w: int,
    guidance: Sequence[float],
    dts: Sequence[float],
) -> np.ndarray:
    """Denoising steps with dual-branch CFG (Ideogram 4 deep dive, section 4-6 pseudocode):
    per step, v_c from the conditional stack on [text_cond; z], v_u from the unconditional stack
    on [text_uncond; z], then z + dt * (gw * v_c + (1 - gw) * v_u).

    The pages give neither the latent-to-token map nor the final projection, so both are the
    identity: z [B, grid_h*grid_w, d] holds the image tokens; it enters each branch as bf16 rows
    after that branch's text rows (a block's input is a bf16 tensor), and a branch's velocity is
    the image rows of its stack output rounded to bf16 (a block's output is a bf16 tensor).
    Returns z after the steps (fp64)."""
    z = np.asarray(z, dtype=np.float64)
    lc, lu = text_cond_bits.shape[1], text_uncond_bits.shape[1]
    for gw, dt in zip(guidance, dts):
        zb = f64_to_bf16_bits(z)
        xc = np.concatenate([text_cond_bits, zb], axis=1)
        xu = np.concatenate([text_uncond_bits, zb], axis=1)
        vc = f64_to_bf16_bits(dit_stack_forward(cfg, ws_cond, xc, lc, grid_h, grid_w)[:, lc:])
        vu = f64_to_bf16_bits(dit_stack_forward(cfg, ws_uncond, xu, lu, grid_h, grid_w)[:, lu:])
        z = euler_cfg_step(z, vc, vu, gw, dt)
    return z

