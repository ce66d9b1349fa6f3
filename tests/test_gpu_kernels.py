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
    st = ops.poll_error()
    assert st == 0, f"a kernel recorded a device-side error: status {st}, word {ops.last_device_error():#x}"


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


@pytest.mark.parametrize("rows,cols", [(3, 256), (5, 4096), (2, 8200), (3, 53248), (2, 57344), (1, 57352)])
@pytest.mark.parametrize("x_fmt,y_fmt", [(0, 0), (0, 1), (2, 1), (2, 0)], ids=["bf16-bf16", "bf16-f16", "f32-f16", "f32-bf16"])
def test_rmsnorm_rows(rows, cols, x_fmt, y_fmt):
    xf = synth.normal(7, rows, (rows, cols), std=2.0)
    g = synth.to_bf16_bits(synth.normal(7, 100 + rows, (cols,), std=0.05, mean=1.0))
    if x_fmt == 0:
        x_np = synth.to_bf16_bits(xf)
        x_val = oracle.bf16_to_f64(x_np)
    else:
        x_np = xf.astype(np.float32)
        x_val = x_np.astype(np.float64)
    y = torch.empty(rows, cols, dtype=torch.int16 if y_fmt == 0 else torch.float16, device="cuda")
    ops.rmsnorm_rows(dev(x_np), dev(g), y, 1e-6, x_fmt=x_fmt, y_fmt=y_fmt)
    ref = oracle.rmsnorm(x_val, oracle.bf16_to_f64(g), 1e-6)
    got = as_f64(y) if y_fmt == 0 else y.cpu().numpy().astype(np.float64)
    # one 16-bit rounding of an fp32 result: |d| <= 2^-8 |ref| (bf16), 2^-11 |ref| (f16)
    ulp = 2.0 ** -8 if y_fmt == 0 else 2.0 ** -11
    assert np.all(np.abs(got - ref) <= ulp * np.abs(ref) + 1e-7)


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


def _fmt_tensor(vals: np.ndarray, fmt: int) -> torch.Tensor:
    if fmt == 0:
        return dev(synth.to_bf16_bits(vals))
    if fmt == 1:
        return torch.from_numpy(vals.astype(np.float16)).cuda()
    return torch.from_numpy(vals.astype(np.float32)).cuda()


def _fmt_values(t: torch.Tensor, fmt: int) -> np.ndarray:
    return as_f64(t) if fmt == 0 else t.cpu().numpy().astype(np.float64)


def _fmt_empty(shape, fmt: int) -> torch.Tensor:
    return torch.empty(*shape, dtype=(torch.int16, torch.float16, torch.float32)[fmt], device="cuda")


@pytest.mark.parametrize("M,N,K", [(128, 256, 64), (200, 512, 256), (37, 768, 1024), (300, 288, 528),
                                   (4500, 2080, 256)])
@pytest.mark.parametrize("a_fmt,y_fmt,act,res_fmt", [
    (0, 0, 0, None), (0, 0, 1, None), (0, 0, 0, 0),  # bf16 in / out
    (1, 1, 0, None), (1, 2, 0, 0), (1, 1, 1, None), (1, 0, 0, 2),  # the block's four GEMMs
], ids=["bf16", "bf16-gelu", "bf16-res", "qkv", "oproj", "up-gelu", "down"])
def test_gemm_w8a16(M, N, K, a_fmt, y_fmt, act, res_fmt):
    r = np.random.default_rng(M + N + K + 10 * a_fmt + y_fmt + act)
    a_vals = r.standard_normal((M, K)).astype(np.float32)
    codes, scale = synth.quantize_rows_e4m3((r.standard_normal((N, K)) * 0.02).astype(np.float32))
    a_t = _fmt_tensor(a_vals, a_fmt)
    a_exact = _fmt_values(a_t, a_fmt)
    res_t = None if res_fmt is None else _fmt_tensor(r.standard_normal((M, N)).astype(np.float32), res_fmt)
    y = _fmt_empty((M, N), y_fmt)
    ops.gemm_w8a16(a_t, dev(codes), dev(scale), y, residual=res_t, act=act, a_fmt=a_fmt, y_fmt=y_fmt,
                   res_fmt=0 if res_fmt is None else res_fmt)
    ref = a_exact @ oracle.dequant(codes, scale).T
    if act == 1:
        ref = oracle.gelu(ref)
    if res_t is not None:
        ref = ref + _fmt_values(res_t, res_fmt)
    got = _fmt_values(y, y_fmt)
    # fp32 accumulation of exact products, one rounding to the output format
    assert_close(got, ref, max_rel=8e-3, mean_rel=2e-3, what=f"gemm {M}x{N}x{K}")


def test_gemm_fp32_out_with_fp32_residual_many_units():
    """fp32 output plus fp32 residual (one output box per epilogue warp) over more work
    units than CTA pairs (each pair walks several 256 x 512 tiles, ragged in M and N)."""
    M, N, K = 4500, 2080, 512
    r = np.random.default_rng(29)
    a_t = _fmt_tensor(r.standard_normal((M, K)).astype(np.float32), 1)
    codes, scale = synth.quantize_rows_e4m3((r.standard_normal((N, K)) * 0.02).astype(np.float32))
    res_t = _fmt_tensor(r.standard_normal((M, N)).astype(np.float32), 2)
    y = _fmt_empty((M, N), 2)
    ops.gemm_w8a16(a_t, dev(codes), dev(scale), y, residual=res_t, a_fmt=1, y_fmt=2, res_fmt=2)
    ref = _fmt_values(a_t, 1) @ oracle.dequant(codes, scale).T + _fmt_values(res_t, 2)
    assert_close(_fmt_values(y, 2), ref, max_rel=8e-3, mean_rel=2e-3, what="gemm f32 out + f32 residual")


def test_gemm_dequant_is_exact_inside_the_mma():
    """A = identity, scale = 1: Y[m, n] = W8[n, m] exactly, for every finite code incl. subnormals."""
    K = N = 256
    finite = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    codes = np.resize(finite, (N, K)).astype(np.uint8)
    want = oracle.e4m3_to_f64(codes).T
    for a_fmt in (0, 1):
        a = _fmt_tensor(np.eye(K, dtype=np.float32), a_fmt)
        y = _fmt_empty((K, N), 2)
        ops.gemm_w8a16(a, dev(codes), dev(np.ones(N, dtype=np.float32)), y, a_fmt=a_fmt, y_fmt=2)
        assert np.array_equal(_fmt_values(y, 2), want), f"a_fmt={a_fmt}"


@pytest.mark.parametrize("gelu_tanh", [0, 1], ids=["erf", "tanh"])
def test_gemm_gelu_epilogue_accuracy(gelu_tanh):
    """W8 = identity, scale = 1: Y = GELU(A) on 131,072 f16 values across [-12, 12] plus extremes.

    The accumulator is exact here, so what is left is the epilogue's GELU against the
    oracle's: fp32 evaluation with an erf (or tanh) approximation good to ~1e-7.
    """
    M, K = 512, 256
    vals = np.linspace(-12.0, 12.0, M * K).astype(np.float16)
    vals[:6] = np.array([-65504.0, 65504.0, -300.0, 300.0, 0.0, -0.0], dtype=np.float16)
    a = torch.from_numpy(vals.reshape(M, K)).cuda()
    eye = np.zeros((K, K), dtype=np.uint8)
    eye[np.arange(K), np.arange(K)] = 0x38  # e4m3 code of 1.0
    y = _fmt_empty((M, K), 2)
    ops.gemm_w8a16(a, dev(eye), dev(np.ones(K, dtype=np.float32)), y, act=1, gelu_tanh=gelu_tanh, a_fmt=1, y_fmt=2)
    x = vals.astype(np.float64).reshape(M, K)
    ref = oracle.gelu(x, tanh=bool(gelu_tanh))
    got = _fmt_values(y, 2)
    err = np.abs(got - ref) / np.maximum(1.0, np.abs(x))
    assert np.all(np.isfinite(got)) and err.max() <= 5e-7, f"max scaled error {err.max():.3e}"


def _tiny_qkv(shape, seed=3, n_text=None, gh=None, gw=None, batch=1):
    n_text = shape.n_text if n_text is None else n_text
    gh = shape.grid_h if gh is None else gh
    gw = shape.grid_w if gw is None else gw
    S = n_text + gh * gw
    qkv = synth.to_bf16_bits(np.random.default_rng(seed).standard_normal((batch, S, 3 * shape.d_model)).astype(np.float32))
    return qkv, n_text, gh, gw, S


@pytest.mark.parametrize("shape", [synth.TINY, synth.C1024], ids=["tiny", "hd128"])
@pytest.mark.parametrize("fmt", [0, 1], ids=["bf16", "f16"])
def test_qknorm_mrope(shape, fmt):
    cfg = ops.make_config(shape)
    if shape is synth.C1024:
        qkv_np, n_text, gh, gw, S = _tiny_qkv(shape, n_text=37, gh=9, gw=11)
    else:
        qkv_np, n_text, gh, gw, S = _tiny_qkv(shape)
    r = np.random.default_rng(5)
    gq = synth.to_bf16_bits(1 + 0.05 * r.standard_normal(shape.head_dim))
    gk = synth.to_bf16_bits(1 + 0.05 * r.standard_normal(shape.head_dim))
    vals = oracle.bf16_to_f64(qkv_np).astype(np.float32)
    qkv = _fmt_tensor(vals, fmt)
    before = qkv.clone()
    ops.qknorm_mrope(qkv, cfg, n_text, gh, gw, dev(gq), dev(gk), workspace(2 * S * shape.head_dim * 4 + 1024), fmt=fmt)
    got = _fmt_values(qkv, fmt).reshape(1, S, 3, shape.n_heads, shape.head_dim)
    x = _fmt_values(before, fmt).reshape(1, S, 3, shape.n_heads, shape.head_dim)
    pos = oracle.mrope_positions(n_text, gh, gw)
    for which, g in ((0, gq), (1, gk)):
        ref = oracle.mrope(oracle.rmsnorm(x[0, :, which], oracle.bf16_to_f64(g), shape.eps), pos, shape.rope_sections, shape.rope_theta)
        assert np.max(np.abs(got[0, :, which] - ref)) <= 2.0 ** -7 * np.abs(ref).max()
    assert torch.equal(qkv.view(1, S, 3, -1)[:, :, 2], before.view(1, S, 3, -1)[:, :, 2])


# (129, 160, 64, 1) and (200, 48, 128, 2): more work items (batch, head, 512 queries) than SM pairs,
# so each persistent CTA pair walks several items, each ending in a ragged key block.
@pytest.mark.parametrize("S,H,hd,batch", [(80, 4, 64, 1), (300, 2, 128, 1), (1, 2, 128, 1), (129, 1, 64, 2), (640, 2, 128, 1),
                                          (129, 160, 64, 1), (200, 48, 128, 2)])
@pytest.mark.parametrize("fmt", [0, 1], ids=["bf16", "f16"])
def test_joint_attention(S, H, hd, batch, fmt):
    d = H * hd
    r = np.random.default_rng(S * 7 + H)
    qkv = _fmt_tensor((r.standard_normal((batch, S, 3 * d)) * 1.5).astype(np.float32), fmt)
    out = _fmt_empty((batch, S, d), fmt)
    ops.joint_attention(qkv, out, H, hd, fmt=fmt)
    x = _fmt_values(qkv, fmt).reshape(batch, S, 3, H, hd)
    got = _fmt_values(out, fmt).reshape(batch, S, H, hd)
    for b in range(batch):
        ref = oracle.attention(x[b, :, 0], x[b, :, 1], x[b, :, 2])
        assert_close(got[b], ref, max_rel=2e-2, mean_rel=3e-3, what=f"attention S={S} H={H} hd={hd}")


@pytest.mark.parametrize("fmt", [0, 1], ids=["bf16", "f16"])
def test_joint_attention_running_max_rises(fmt):
    """Rows whose running max rises by ~8.5 log2 units after many keys already carry weight.

    Query row i looks along feature i % 4; along each feature a group of keys has logit 3
    and four later keys logit 8.9 (natural units): inside key block 0 at chunk 1 (keys
    32-35) and chunk 3 (keys 100-103), in block 2 (keys 300-303), and in the partial last
    block (keys 580-583 of 600).  The earlier keys keep ~6-30 % of the mass, so a kernel
    that skips rescaling O, the row sum or the P values of the block already written is
    off by a factor of up to 2^8.5 (an emulation without either rescale errs by >3 in
    max-rel).
    """
    S, H, hd = 600, 1, 128
    r = np.random.default_rng(11)
    q = 0.3 * r.standard_normal((S, hd))
    k = 0.3 * r.standard_normal((S, hd))
    v = r.standard_normal((S, hd))
    q[:, :4] = 0.0
    k[:, :4] = 0.0
    q[np.arange(S), np.arange(S) % 4] = 8.0
    groups = {0: (range(0, 32), range(32, 36)), 1: (range(0, 96), range(100, 104)),
              2: (range(0, 128), range(300, 304)), 3: (range(0, 200), range(580, 584))}
    for g, (base, late) in groups.items():
        k[list(base), g] = 3.0 * np.sqrt(hd) / 8.0
        k[list(late), g] = 8.9 * np.sqrt(hd) / 8.0
    qkv = _fmt_tensor(np.concatenate([q, k, v], axis=1)[None].astype(np.float32), fmt)
    out = _fmt_empty((1, S, hd), fmt)
    ops.joint_attention(qkv, out, H, hd, fmt=fmt)
    x = _fmt_values(qkv, fmt).reshape(S, 3, hd)
    ref = oracle.attention(x[:, 0][:, None], x[:, 1][:, None], x[:, 2][:, None])[:, 0]
    got = _fmt_values(out, fmt).reshape(S, hd)
    assert_close(got, ref, max_rel=2e-2, mean_rel=3e-3, what="attention with rising maxima")


def test_bounded_wait_timeout_is_not_hit_in_normal_runs():
    ops.set_wait_timeout_ms(2000)
    assert ops.poll_error() == 0


def test_bounded_wait_gives_up_and_context_survives():
    """A wait that nothing completes times out, is reported, and the next kernels still run."""
    ops.set_wait_timeout_ms(100)
    try:
        ops.wait_selftest()
        assert ops.poll_error() == 5  # DIT_ERR_TIMEOUT
        assert ops.last_device_error() & 0xFFF == 0x1F0
        assert ops.poll_error() == 0  # the error word was cleared
    finally:
        ops.set_wait_timeout_ms(2000)
    # the context is still usable: a real kernel after the timeout is exact
    codes = np.arange(256, dtype=np.uint8)
    out = empty_bf16(256)
    ops.e4m3_to_bf16(dev(codes), out)
    ref = oracle.e4m3_to_f64(codes)
    fin = ~np.isnan(ref)
    assert np.array_equal(bits(out)[fin], (ref[fin].astype(np.float32).view(np.uint32) >> 16).astype(np.uint16))
