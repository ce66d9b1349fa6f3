"""The W8A8 variant (e4m3 activations into the QKV and MLP-up projections, e4m3 q and k into
q k^T) against the oracle (needs a B200).

The FP8 GEMM is checked on its own (e4m3 x e4m3 products are exact in fp32, so only the fp32
accumulation differs from fp64), the RMSNorm-to-e4m3 kernel code by code (a code may differ only
where the fp32 and fp64 quotients fall on opposite sides of a rounding tie), and the whole block
against oracle.dit_block_forward(..., w8a8=True): at the block tolerances on the small shapes, at
its own (mean 6e-3, reasons at the test) on the 1024 px block.  The e4m3 QK-norm is checked code by
code and the e4m3 attention against the oracle on seeded codes.  The variant's own error against
the 16-bit pipeline is reported, not bounded by the 16-bit tolerances.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from joint_attention_block_b200 import ops, synth
from gpu_util import as_f64, assert_close, dev, poisoned_like, workspace

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clean_errors():
    yield
    st = ops.poll_error()
    assert st == 0, f"a kernel recorded a device-side error: status {st}, word {ops.last_device_error():#x}"


def _codes(rng, shape):
    c = rng.integers(0, 256, size=shape).astype(np.uint8)
    c[(c & 0x7F) == 0x7F] = 0x3C  # no NaN codes
    return c


@pytest.mark.parametrize("M,N,K", [(300, 544, 512), (4608, 512, 4096), (1, 32, 16)])
def test_gemm_w8a8_fp32_out(M, N, K):
    rng = np.random.default_rng(90 + M)
    a8, w8 = _codes(rng, (M, K)), _codes(rng, (N, K))
    sa = (rng.uniform(0.5, 2.0, M) * 1e-3).astype(np.float32)
    sw = (rng.uniform(0.5, 2.0, N) * 1e-3).astype(np.float32)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    ops.gemm_w8a8(dev(a8), dev(sa), dev(w8), dev(sw), y, y_fmt=ops.FMT_F32)
    torch.cuda.synchronize()
    a = oracle.e4m3_to_f64(a8) * sa.astype(np.float64)[:, None]
    ref = a @ oracle.dequant(w8, sw).T
    # products of e4m3 codes are exact in fp32; what remains is the tensor core's fp32 accumulation
    assert_close(y.cpu().numpy(), ref, max_rel=1e-5, mean_rel=5e-6, what=f"w8a8 {M}x{N}x{K}")


def test_gemm_w8a8_gelu_f16():
    rng = np.random.default_rng(95)
    M, N, K = 260, 1024, 1024
    a8, w8 = _codes(rng, (M, K)), _codes(rng, (N, K))
    sa = np.full(M, 1.0 / 448.0, np.float32)
    sw = (rng.uniform(0.5, 2.0, N) * 2e-4).astype(np.float32)
    for tanh in (0, 1):
        y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        ops.gemm_w8a8(dev(a8), dev(sa), dev(w8), dev(sw), y, act=1, gelu_tanh=tanh, y_fmt=ops.FMT_F16)
        torch.cuda.synchronize()
        pre = (oracle.e4m3_to_f64(a8) * sa.astype(np.float64)[:, None]) @ oracle.dequant(w8, sw).T
        ref = oracle.gelu(pre, tanh=bool(tanh))
        assert_close(y.float().cpu().numpy(), ref, max_rel=2e-3, mean_rel=1e-3, what=f"w8a8 GELU tanh={tanh}")


@pytest.mark.parametrize("x_fmt", [ops.FMT_BF16, ops.FMT_F32])
def test_rmsnorm_e4m3_codes_and_scales(x_fmt):
    rng = np.random.default_rng(96)
    rows, cols = 37, 4096
    xf = rng.standard_normal((rows, cols)) * rng.uniform(0.1, 10.0, (rows, 1))
    xf[5] = 0.0
    g = synth.to_bf16_bits(1.0 + 0.05 * rng.standard_normal(cols))
    if x_fmt == ops.FMT_BF16:
        xb = synth.to_bf16_bits(xf)
        x, xv = dev(xb), oracle.bf16_to_f64(xb)
    else:
        x32 = xf.astype(np.float32)
        x, xv = dev(x32), x32.astype(np.float64)
    y8 = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    ys = torch.empty(rows, dtype=torch.float32, device="cuda")
    ops.rmsnorm_rows_e4m3(x, dev(g), y8, ys, 1e-6, x_fmt=x_fmt)
    torch.cuda.synchronize()
    h = oracle.rmsnorm(xv, oracle.bf16_to_f64(g), 1e-6)
    _, s = oracle.quantize_rows_act(h)
    got_s = ys.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got_s - s) <= 2e-6 * s)  # fp32 amax of fp32 norm outputs vs fp64 (a few ulp)
    # The codes are a rounding decision the kernel takes in fp32 with its own scale: take it with the
    # same scale here; the two sides can then disagree only where h / s lies within fp32 rounding of
    # a tie between neighbouring codes.
    want = oracle.e4m3_round(h / got_s[:, None])
    got = oracle.e4m3_to_f64(y8.cpu().numpy())
    diff = got != want
    assert diff.mean() < 1e-3, diff.mean()
    step = np.exp2(np.floor(np.log2(np.maximum(np.abs(want), 2.0 ** -6))) - 3.0)
    assert np.all(np.abs(got - want)[diff] <= step[diff] * 1.0000001)
    assert np.array_equal(y8.cpu().numpy()[5], np.zeros(cols, np.uint8))


@pytest.mark.parametrize("shape,n_text,gh,gw,batch", [(synth.TINY, 16, 8, 8, 1), (synth.TINY, 5, 7, 9, 2),
                                                     (synth.C1024, 37, 9, 11, 1)], ids=["hd64", "hd64-b2", "hd128"])
@pytest.mark.parametrize("fmt", [ops.FMT_BF16, ops.FMT_F16], ids=["bf16", "f16"])
def test_qknorm_mrope_e4m3_codes_and_scales(shape, n_text, gh, gw, batch, fmt):
    """q and k codes of the e4m3 QK-norm against the oracle's normalised, rotated q and k divided by
    the static scale: the scales bit for bit, the codes equal except where the kernel's fp32 value
    and the fp64 one fall on opposite sides of a rounding tie (then one step apart); qkv untouched."""
    cfg = ops.make_config(shape)
    S, d, H, hd = n_text + gh * gw, shape.d_model, shape.n_heads, shape.head_dim
    r = np.random.default_rng(97)
    vals = (r.standard_normal((batch, S, 3 * d)) * np.exp(r.uniform(-2, 2, (batch, S, 1)))).astype(np.float32)
    if fmt == ops.FMT_BF16:
        qkv = dev(synth.to_bf16_bits(vals))
    else:
        qkv = torch.from_numpy(vals.astype(np.float16)).cuda()
    xv = (as_f64(qkv) if fmt == ops.FMT_BF16 else qkv.cpu().numpy().astype(np.float64)).reshape(batch, S, 3, H, hd)
    gq = synth.to_bf16_bits(1 + 0.05 * r.standard_normal(hd))
    gk = synth.to_bf16_bits(1 + 0.05 * r.standard_normal(hd))
    before = qkv.clone()
    q8 = torch.empty((batch, S, d), dtype=torch.uint8, device="cuda")
    k8 = torch.empty_like(q8)
    sc = torch.full((2,), float("nan"), dtype=torch.float32, device="cuda")
    ops.qknorm_mrope_e4m3(qkv, cfg, n_text, gh, gw, dev(gq), dev(gk), q8, k8, sc, fmt=fmt)
    torch.cuda.synchronize()
    assert torch.equal(qkv, before)
    got_sc = sc.cpu().numpy()
    want_sc = [oracle.qk_e4m3_scale(oracle.bf16_to_f64(g), hd) for g in (gq, gk)]
    assert got_sc.tolist() == want_sc
    pos = oracle.mrope_positions(n_text, gh, gw)
    for which, g, codes, s in ((0, gq, q8, want_sc[0]), (1, gk, k8, want_sc[1])):
        ref = oracle.mrope(oracle.rmsnorm(xv[:, :, which], oracle.bf16_to_f64(g), shape.eps), pos,
                           shape.rope_sections, shape.rope_theta)
        want = oracle.e4m3_round(ref / s)
        got = oracle.e4m3_to_f64(codes.cpu().numpy()).reshape(want.shape)
        diff = got != want
        assert diff.mean() < 1e-3, diff.mean()
        step = np.exp2(np.floor(np.log2(np.maximum(np.abs(want), 2.0 ** -6))) - 3.0)
        assert np.all(np.abs(got - want)[diff] <= step[diff] * 1.0000001)
        assert np.abs(got).max() <= 448.0


# (129, 160, 64, 1) and (200, 48, 128, 2): more work items than SM pairs (each pair walks several).
@pytest.mark.parametrize("S,H,hd,batch", [(80, 4, 64, 1), (300, 2, 128, 1), (1, 2, 128, 1), (129, 1, 64, 2),
                                          (640, 2, 128, 1), (129, 160, 64, 1), (200, 48, 128, 2)])
@pytest.mark.parametrize("fmt", [ops.FMT_BF16, ops.FMT_F16], ids=["bf16", "f16"])
def test_joint_attention_e4m3(S, H, hd, batch, fmt):
    """Attention with e4m3 q and k (seeded codes, static scales) and 16-bit v against the oracle's
    attention on the decoded q and k times their scales."""
    d = H * hd
    r = np.random.default_rng(S * 11 + H)
    vals = (r.standard_normal((batch, S, 3 * d)) * 1.5).astype(np.float32)
    if fmt == ops.FMT_BF16:
        qkv = dev(synth.to_bf16_bits(vals))
    else:
        qkv = torch.from_numpy(vals.astype(np.float16)).cuda()
    v = (as_f64(qkv) if fmt == ops.FMT_BF16 else qkv.cpu().numpy().astype(np.float64)).reshape(batch, S, 3, H, hd)[:, :, 2]
    # seeded e4m3 codes of N(0, 1) * 40 values (the range the static scale gives normalised q and k)
    q8 = torch.from_numpy(r.standard_normal((batch, S, d)).astype(np.float32) * 40).to(torch.float8_e4m3fn).view(torch.uint8)
    k8 = torch.from_numpy(r.standard_normal((batch, S, d)).astype(np.float32) * 40).to(torch.float8_e4m3fn).view(torch.uint8)
    scales = np.array([0.028, 0.031], dtype=np.float32)
    out = torch.empty((batch, S, d), dtype=torch.int16 if fmt == ops.FMT_BF16 else torch.float16, device="cuda")
    ops.joint_attention_e4m3(q8.cuda(), k8.cuda(), torch.from_numpy(scales).cuda(), qkv, out, H, hd, fmt=fmt)
    torch.cuda.synchronize()
    got = (as_f64(out) if fmt == ops.FMT_BF16 else out.cpu().numpy().astype(np.float64)).reshape(batch, S, H, hd)
    qd = oracle.e4m3_to_f64(q8.numpy()).reshape(batch, S, H, hd) * float(scales[0])
    kd = oracle.e4m3_to_f64(k8.numpy()).reshape(batch, S, H, hd) * float(scales[1])
    for b in range(batch):
        ref = oracle.attention(qd[b], kd[b], v[b])
        assert_close(got[b], ref, max_rel=2e-2, mean_rel=3e-3, what=f"e4m3 attention S={S} H={H} hd={hd}")


def _run_w8a8(shape, inp):
    cfg = ops.make_config(shape)
    w = ops.make_weights({k: dev(v) for k, v in inp.items() if k != "x"})
    x = dev(inp["x"])
    out = poisoned_like(x)
    ws = workspace(ops.block_workspace_bytes(cfg, x.shape[0], shape.n_text, shape.grid_h, shape.grid_w))
    ops.dit_block_forward_w8a8(cfg, w, x, out, shape.n_text, shape.grid_h, shape.grid_w, ws)
    torch.cuda.synchronize()
    return as_f64(out)


@pytest.mark.parametrize("n_text,gh,gw,batch", [(16, 8, 8, 1), (5, 7, 9, 2)])
def test_block_w8a8_against_oracle(n_text, gh, gw, batch):
    s = dataclasses.replace(synth.TINY, n_text=n_text, grid_h=gh, grid_w=gw, batch=batch)
    inp = synth.block_inputs(s)
    got = _run_w8a8(s, inp)
    ref8 = oracle.dit_block_forward(s, inp, inp["x"], n_text, gh, gw, w8a8=True)
    assert_close(got, ref8, what="w8a8 block vs w8a8 oracle")
    ref16 = oracle.dit_block_forward(s, inp, inp["x"], n_text, gh, gw)
    d = np.abs(got - ref16)
    print(f"w8a8 vs 16-bit oracle: max-rel {d.max() / np.abs(ref16).max():.3e}, "
          f"mean-rel {d.mean() / np.abs(ref16).mean():.3e}")


@pytest.mark.slow
def test_block_w8a8_1024px_sampled_rows():
    s = synth.C1024
    inp = synth.block_inputs(s)
    got = _run_w8a8(s, inp)
    rows = np.array([0, 100, s.n_text - 1, s.n_text, 2000, s.seq - 1])
    ref8 = oracle.dit_block_forward(s, inp, inp["x"], s.n_text, s.grid_h, s.grid_w, rows=rows, w8a8=True)
    # The variant's own tolerance at this size (mean 6e-3 instead of 3e-3): with bf16 inputs and
    # gains about 1.4e-4 of the per-token activation codes fall exactly on an e4m3 rounding tie,
    # where the last bit of the fp32 scale decides (the kernel and the fp64 oracle can round
    # either way; test_rmsnorm_e4m3_codes_and_scales allows it code by code).  Each such code moves
    # k by one e4m3 step of one product term, and rounding k to e4m3 again turns those moves into
    # whole-step differences in ~1.75 % of the k codes over 4608 tokens: 3.7e-3 mean-rel measured.
    assert_close(got[:, rows], ref8, max_rel=2e-2, mean_rel=6e-3, what="c1024 w8a8 sampled")
    ref16 = oracle.dit_block_forward(s, inp, inp["x"], s.n_text, s.grid_h, s.grid_w, rows=rows)
    d = np.abs(got[:, rows] - ref16)
    print(f"c1024 w8a8 vs 16-bit oracle: max-rel {d.max() / np.abs(ref16).max():.3e}, "
          f"mean-rel {d.mean() / np.abs(ref16).mean():.3e}")
