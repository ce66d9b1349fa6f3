"""Per-kernel parity of the CUDA path against the fp64 oracle (needs a B200)."""
import math

import numpy as np
import pytest
import torch

import oracle
from joint_attention_block_b200 import ops, synth
from gpu_util import as_f64, assert_close, bits, dev, empty_bf16, workspace

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_errors():
    yield
    assert ops.poll_error() == 0, "a kernel recorded a device-side error"


def test_e4m3_to_bf16_every_code_bit_exact():
    codes = np.tile(np.arange(256, dtype=np.uint8), 17)[: 256 * 16 + 7]  # ragged tail
    out = empty_bf16(codes.size)
    ops.e4m3_to_bf16(dev(codes), out)
    got = bits(out)
    ref = oracle.e4m3_to_f64(codes)
    fin = ~np.isnan(ref)
    want = (ref[fin].astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(got[fin], want)
    # the two NaN codes come out as +-480 (no FP8 checkpoint holds NaN)
    assert set(oracle.bf16_to_f64(got[~fin]).tolist()) == {480.0, -480.0}


@pytest.mark.parametrize("rows,cols", [(3, 256), (5, 4096), (2, 8200), (3, 53248)])
def test_rmsnorm_rows(rows, cols):
    x = synth.to_bf16_bits(synth.normal(7, rows, (rows, cols), std=2.0))
    g = synth.to_bf16_bits(synth.normal(7, 100 + rows, (cols,), std=0.05, mean=1.0))
    y = empty_bf16(rows, cols)
    ops.rmsnorm_rows(dev(x), dev(g), y, 1e-6)
    ref = oracle.rmsnorm(oracle.bf16_to_f64(x), oracle.bf16_to_f64(g), 1e-6)
    got = as_f64(y)
    # one bf16 rounding of an fp32 result: |d| <= 2^-8 |ref|
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-30)


@pytest.mark.parametrize("n_text,gh,gw,t_img", [(16, 8, 8, -1), (512, 64, 64, -1), (0, 3, 5, -1), (1, 1, 1, 7), (4, 0, 0, -1)])
def test_positions_bit_exact(n_text, gh, gw, t_img):
    S = n_text + gh * gw
    out = torch.empty(S, 3, dtype=torch.int32, device="cuda")
    ops.mrope_positions(n_text, gh, gw, t_img, out)
    assert np.array_equal(out.cpu().numpy(), oracle.mrope_positions(n_text, gh, gw, None if t_img < 0 else t_img))


@pytest.mark.parametrize("n", [4096 * 128, 4096 * 128 + 5, 16384 * 128, 3])
def test_euler_cfg(n):
    e = synth.euler_inputs(n)
    g, dt = 4.0, float(np.float32(-1.0 / 50))
    x = dev(e["x"])
    ops.euler_cfg_step(x, dev(e["v_cond"]), dev(e["v_uncond"]), g, dt)
    ref = oracle.euler_cfg_step(e["x"], e["v_cond"], e["v_uncond"], g, dt)
    got = x.cpu().numpy().astype(np.float64)
    vc, vu = oracle.bf16_to_f64(e["v_cond"]), oracle.bf16_to_f64(e["v_uncond"])
    # three fp32 roundings (difference, guidance fma, Euler fma)
    bound = 2.0 ** -23 * (np.abs(ref) + abs(dt) * (abs(g) * np.abs(vc - vu) + np.abs(vu) + np.abs(vu + g * (vc - vu))))
    assert np.all(np.abs(got - ref) <= bound + 1e-30)


def _gemm_case(M, N, K, seed):
    r = np.random.default_rng(seed)
    a = synth.to_bf16_bits(r.standard_normal((M, K)).astype(np.float32))
    codes, scale = synth.quantize_rows_e4m3((r.standard_normal((N, K)) * 0.02).astype(np.float32))
    res = synth.to_bf16_bits(r.standard_normal((M, N)).astype(np.float32))
    return a, codes, scale, res


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (200, 512, 256), (37, 768, 1024), (300, 288, 528)])
@pytest.mark.parametrize("epi", [0, 1, 2])
def test_gemm_w8a16(M, N, K, epi):
    a, codes, scale, res = _gemm_case(M, N, K, seed=M + N + K + epi)
    y = empty_bf16(M, N)
    ops.gemm_w8a16(dev(a), dev(codes), dev(scale), y, residual=dev(res) if epi == 2 else None, epilogue=epi)
    ref = oracle.bf16_to_f64(a) @ oracle.dequant(codes, scale).T
    if epi == 1:
        ref = oracle.gelu(ref)
    if epi == 2:
        ref = ref + oracle.bf16_to_f64(res)
    got = as_f64(y)
    # fp32 accumulation of exact products, one bf16 rounding at the end
    assert_close(got, ref, max_rel=8e-3, mean_rel=3e-3, what=f"gemm {M}x{N}x{K} epi{epi}")


def test_gemm_dequant_is_exact_inside_the_mma():
    """A = identity, scale = 1: Y[m, n] = W8[n, m] exactly, for every finite code incl. subnormals."""
    K = N = 256
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    codes = np.resize(finite, (N, K)).astype(np.uint8)
    a = synth.to_bf16_bits(np.eye(K, dtype=np.float32))
    y = empty_bf16(K, N)
    ops.gemm_w8a16(dev(a), dev(codes), dev(np.ones(N, dtype=np.float32)), y)
    want = oracle.e4m3_to_f64(codes).T
    assert np.array_equal(as_f64(y), want)


def _tiny_qkv(shape, seed=3, n_text=None, gh=None, gw=None, batch=1):
    n_text = shape.n_text if n_text is None else n_text
    gh = shape.grid_h if gh is None else gh
    gw = shape.grid_w if gw is None else gw
    S = n_text + gh * gw
    qkv = synth.to_bf16_bits(np.random.default_rng(seed).standard_normal((batch, S, 3 * shape.d_model)).astype(np.float32))
    return qkv, n_text, gh, gw, S


@pytest.mark.parametrize("shape", [synth.TINY, synth.C1024], ids=["tiny", "hd128"])
def test_qknorm_mrope(shape):
    import ctypes
    cfg = ops.make_config(shape)
    if shape is synth.C1024:
        qkv_np, n_text, gh, gw, S = _tiny_qkv(shape, n_text=37, gh=9, gw=11)
    else:
        qkv_np, n_text, gh, gw, S = _tiny_qkv(shape)
    w = synth.block_inputs(synth.TINY) if shape is synth.TINY else None
    r = np.random.default_rng(5)
    gq = synth.to_bf16_bits(1 + 0.05 * r.standard_normal(shape.head_dim))
    gk = synth.to_bf16_bits(1 + 0.05 * r.standard_normal(shape.head_dim))
    qkv = dev(qkv_np)
    ops.qknorm_mrope(qkv, cfg, n_text, gh, gw, dev(gq), dev(gk), workspace(2 * S * shape.head_dim * 4 + 1024))
    got = oracle.bf16_to_f64(bits(qkv)).reshape(1, S, 3, shape.n_heads, shape.head_dim)
    x = oracle.bf16_to_f64(qkv_np).reshape(1, S, 3, shape.n_heads, shape.head_dim)
    pos = oracle.mrope_positions(n_text, gh, gw)
    for which, g in ((0, gq), (1, gk)):
        ref = oracle.mrope(oracle.rmsnorm(x[0, :, which], oracle.bf16_to_f64(g), shape.eps), pos, shape.rope_sections, shape.rope_theta)
        assert np.max(np.abs(got[0, :, which] - ref)) <= 2.0 ** -7 * np.abs(ref).max()
    assert np.array_equal(bits(qkv).reshape(1, S, 3, -1)[:, :, 2], qkv_np.reshape(1, S, 3, -1)[:, :, 2])


@pytest.mark.parametrize("S,H,hd,batch", [(80, 4, 64, 1), (300, 2, 128, 1), (1, 2, 128, 1), (129, 1, 64, 2), (640, 2, 128, 1)])
def test_joint_attention(S, H, hd, batch):
    d = H * hd
    r = np.random.default_rng(S * 7 + H)
    qkv_np = synth.to_bf16_bits((r.standard_normal((batch, S, 3 * d)) * 1.5).astype(np.float32))
    out = empty_bf16(batch, S, d)
    ops.joint_attention(dev(qkv_np), out, H, hd)
    x = oracle.bf16_to_f64(qkv_np).reshape(batch, S, 3, H, hd)
    got = as_f64(out).reshape(batch, S, H, hd)
    for b in range(batch):
        ref = oracle.attention(x[b, :, 0], x[b, :, 1], x[b, :, 2])
        assert_close(got[b], ref, max_rel=2e-2, mean_rel=3e-3, what=f"attention S={S} H={H} hd={hd}")


def test_bounded_wait_timeout_is_not_hit_in_normal_runs():
    ops.set_wait_timeout_ms(2000)
    assert ops.poll_error() == 0
