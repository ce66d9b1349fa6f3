"""Pins for the fp64 oracle: page facts, closed forms, invariants, library routines, brute force.

Each test ties the oracle to something other than itself, so that a dropped
term, a flipped sign, a wrong index or a transposed operand fails one of them.
"""
import json
import math
import os
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle
from joint_attention_block_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def facts():
    with open(GOLDEN) as f:
        return json.load(f)


# ---------------------------------------------------------------- e4m3 and dequant


def test_e4m3_all_codes_match_torch_float8():
    """All 256 codes against torch's own float8_e4m3fn decoder (a library routine)."""
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    fin = ~np.isnan(lib)
    assert np.array_equal(ours[fin], lib[fin])
    assert np.array_equal(np.signbit(ours[fin]), np.signbit(lib[fin]))


def test_e4m3_range_and_structure():
    v = oracle.e4m3_to_f64(np.arange(256, dtype=np.uint8))
    fin = v[~np.isnan(v)]
    assert np.isnan(v).sum() == 2 and np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    assert fin.max() == facts()["e4m3_max"]["value"] == -fin.min()
    assert v[1] == 2.0 ** -9 and v[8] == 2.0 ** -6 and v[0x38] == 1.0
    pos = v[:0x7F]
    assert np.all(np.diff(pos) > 0), "positive codes must be strictly increasing"
    assert np.array_equal(v[0x80:0xFF], -v[0:0x7F])


def test_dequant_scale_is_per_output_row():
    """weight_scale[:, None]: row i of the real weight is code row i times scale[i]."""
    r = np.random.default_rng(0)
    codes = r.integers(0, 256, size=(3, 5), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38
    scale = np.array([0.5, 2.0, 0.125], dtype=np.float32)
    w = oracle.dequant(codes, scale)
    for i in range(3):
        for j in range(5):
            assert w[i, j] == float(torch.tensor([int(codes[i, j])], dtype=torch.uint8).view(torch.float8_e4m3fn).float()) * float(scale[i])
    with pytest.raises(ValueError):
        oracle.dequant(codes, np.ones(5, dtype=np.float32))


def test_scale_in_epilogue_equals_scaled_weight():
    """scale[n] * sum_k x_k w8[n,k] == sum_k x_k (w8[n,k] scale[n]) exactly on small dyadic inputs."""
    r = np.random.default_rng(1)
    codes = r.integers(0, 0x70, size=(6, 8), dtype=np.uint8)
    scale = (2.0 ** r.integers(-6, 6, size=6)).astype(np.float32)
    x = r.integers(-8, 8, size=(4, 8)).astype(np.float64)
    lhs = (x @ oracle.e4m3_to_f64(codes).T) * scale.astype(np.float64)[None, :]
    rhs = x @ oracle.dequant(codes, scale).T
    assert np.array_equal(lhs, rhs)


def test_synthetic_quantiser_hits_448_per_row():
    codes, scale = synth.quantize_rows_e4m3(synth.normal(9, 0, (8, 64), std=0.02))
    w = oracle.e4m3_to_f64(codes)
    assert np.all(np.abs(w).max(axis=1) == 448.0)
    assert scale.dtype == np.float32 and np.all(scale > 0)


# ---------------------------------------------------------------- page arithmetic


def test_conditioning_width_and_cache_sizes():
    f = facts()
    k = f["cond_layers"]["value"] * f["cond_hidden"]["value"]
    assert k == f["cond_features_per_token"]["value"] == synth.COND.k
    per_tok = k * 4 / 2 ** 20
    assert round(per_tok, 3) == f["cond_raw_mib_per_token"]["value"]
    assert round(per_tok * 512) == f["cond_raw_mib_512_tokens"]["value"]
    # The projected size on the page is 512 tokens * 4608 bf16 values; the graded
    # projection width is 4096 (4.0 MiB).  Both readings are recorded.
    assert 512 * 4608 * 2 / 2 ** 20 == f["cond_projected_mib_512_tokens"]["value"]
    assert 512 * synth.COND.d_out * 2 / 2 ** 20 == 4.0


def test_shapes_follow_pages():
    f = facts()
    assert list(synth.C1024.rope_sections) == f["mrope_section"]["value"]
    assert sum(synth.C1024.rope_sections) == synth.C1024.head_dim // 2
    gh, gw, ch = f["latent_grid_1024"]["value"]
    assert (synth.C1024.grid_h, synth.C1024.grid_w, synth.LATENT_CHANNELS) == (gh, gw, ch)
    w = synth.block_inputs(synth.TINY)
    assert w["w_qkv"].shape == (f["qkv_rows_per_hidden"]["value"] * synth.TINY.d_model, synth.TINY.d_model)


# ---------------------------------------------------------------- RMSNorm


def test_rmsnorm_unit_rms_closed_form():
    r = np.random.default_rng(2)
    x = r.standard_normal((7, 33)) * 3.0
    eps = 1e-6
    y = oracle.rmsnorm(x, np.ones(33), eps)
    ms = np.mean(x * x, axis=1)
    assert np.allclose(np.mean(y * y, axis=1), ms / (ms + eps), rtol=1e-13, atol=0)


def test_rmsnorm_scale_invariance_and_gain():
    r = np.random.default_rng(3)
    x = r.standard_normal((5, 16))
    g = r.standard_normal(16)
    y1 = oracle.rmsnorm(x, g, 0.0)
    y2 = oracle.rmsnorm(7.5 * x, g, 0.0)
    assert np.allclose(y1, y2, rtol=1e-13, atol=1e-15)
    assert np.allclose(y1 / g, oracle.rmsnorm(x, np.ones(16), 0.0), rtol=1e-13)


# ---------------------------------------------------------------- M-RoPE


def test_positions_brute_force():
    pos = oracle.mrope_positions(3, 2, 3)
    want = [(0, 0, 0), (1, 1, 1), (2, 2, 2)]
    for r in range(2):
        for c in range(3):
            want.append((3, r, c))
    assert pos.tolist() == [list(p) for p in want]
    assert oracle.mrope_positions(3, 2, 3, t_img=9)[3:, 0].tolist() == [9] * 6
    assert oracle.mrope_positions(0, 1, 1).tolist() == [[0, 0, 0]]


def test_inv_freq_fp32_values():
    f = oracle.inv_freq(128, 10000.0)
    assert f[0] == 1.0
    assert f.dtype == np.float64 and np.all(f.astype(np.float32).astype(np.float64) == f)
    assert abs(f[32] - 0.01) < 1e-9  # theta^(-64/128) = 1e-2


def test_text_tokens_reduce_to_1d_rope_complex():
    """Text token j at (j, j, j): every pair turns by j * inv_freq_i, whatever the sections.

    Checked against the complex form z_i * exp(i j w_i), z_i = x_i + i x_{i+hd/2}.
    """
    hd, theta = 16, 10000.0
    r = np.random.default_rng(4)
    x = r.standard_normal((6, 2, hd))
    pos = oracle.mrope_positions(6, 0, 0)
    y = oracle.mrope(x, pos, (2, 3, 3), theta)
    w = np.array([theta ** (-2 * i / hd) for i in range(hd // 2)], dtype=np.float32).astype(np.float64)
    for j in range(6):
        for h in range(2):
            z = x[j, h, : hd // 2] + 1j * x[j, h, hd // 2 :]
            zr = z * np.exp(1j * j * w)
            assert np.allclose(y[j, h, : hd // 2], zr.real, atol=1e-12)
            assert np.allclose(y[j, h, hd // 2 :], zr.imag, atol=1e-12)


def test_mrope_sections_pick_their_axis():
    """A token at (0, 1, 0) turns only the h-section pairs, each by inv_freq_i; (0,0,0) is the identity."""
    hd, secs, theta = 16, (2, 3, 3), 100.0
    x = np.random.default_rng(5).standard_normal((3, 1, hd))
    pos = np.array([[0, 0, 0], [0, 1, 0], [0, 0, 2]])
    y = oracle.mrope(x, pos, secs, theta)
    assert np.array_equal(y[0], x[0])
    f = oracle.inv_freq(hd, theta)
    for tok, axis_pairs, p in ((1, range(2, 5), 1), (2, range(5, 8), 2)):
        for i in range(hd // 2):
            a, b = x[tok, 0, i], x[tok, 0, i + hd // 2]
            ang = p * f[i] if i in axis_pairs else 0.0
            assert math.isclose(y[tok, 0, i], a * math.cos(ang) - b * math.sin(ang), abs_tol=1e-13)
            assert math.isclose(y[tok, 0, i + hd // 2], b * math.cos(ang) + a * math.sin(ang), abs_tol=1e-13)


def test_mrope_norm_and_relative_invariance():
    hd, secs = 32, (4, 6, 6)
    r = np.random.default_rng(6)
    q = r.standard_normal((1, 1, hd))
    k = r.standard_normal((1, 1, hd))
    p1, p2 = np.array([[3, 5, 7]]), np.array([[1, 2, 9]])
    delta = np.array([[11, -4, 6]])
    yq = oracle.mrope(q, p1, secs, 10000.0)
    pairs = yq[0, 0, : hd // 2] ** 2 + yq[0, 0, hd // 2 :] ** 2
    assert np.allclose(pairs, q[0, 0, : hd // 2] ** 2 + q[0, 0, hd // 2 :] ** 2, rtol=1e-13)
    a = np.dot(oracle.mrope(q, p1, secs, 1e4).ravel(), oracle.mrope(k, p2, secs, 1e4).ravel())
    b = np.dot(oracle.mrope(q, p1 + delta, secs, 1e4).ravel(), oracle.mrope(k, p2 + delta, secs, 1e4).ravel())
    assert math.isclose(a, b, rel_tol=1e-10, abs_tol=1e-12)


# ---------------------------------------------------------------- attention


def _attention_loops(q, k, v):
    Sq, H, hd = q.shape
    out = np.zeros((Sq, H, v.shape[2]))
    for h in range(H):
        for i in range(Sq):
            logits = [sum(q[i, h, c] * k[j, h, c] for c in range(hd)) / math.sqrt(hd) for j in range(k.shape[0])]
            m = max(logits)
            ws = [math.exp(l - m) for l in logits]
            tot = sum(ws)
            for c in range(v.shape[2]):
                out[i, h, c] = sum(ws[j] * v[j, h, c] for j in range(k.shape[0])) / tot
    return out


def test_attention_brute_force():
    r = np.random.default_rng(7)
    q, k, v = (r.standard_normal((5, 2, 4)) for _ in range(3))
    assert np.allclose(oracle.attention(q, k, v), _attention_loops(q, k, v), rtol=1e-12, atol=1e-13)


def test_attention_special_cases():
    r = np.random.default_rng(8)
    v = r.standard_normal((6, 1, 4))
    q = r.standard_normal((3, 1, 4))
    k_same = np.repeat(r.standard_normal((1, 1, 4)), 6, axis=0)
    assert np.allclose(oracle.attention(q, k_same, v), v.mean(axis=0, keepdims=True).repeat(3, 0), atol=1e-13)
    assert np.allclose(oracle.attention(q[:1], k_same[:1], v[:1]), v[:1], atol=1e-15)
    k = np.zeros((6, 1, 4))
    k[4, 0, 0] = 1e3
    qd = np.zeros((1, 1, 4))
    qd[0, 0, 0] = 1.0
    assert np.allclose(oracle.attention(qd, k, v), v[4:5], atol=1e-12)


def test_attention_permutation_equivariance():
    """Bidirectional and unmasked: permuting the keys with their values changes nothing."""
    r = np.random.default_rng(9)
    q, k, v = (r.standard_normal((7, 2, 8)) for _ in range(3))
    perm = r.permutation(7)
    assert np.allclose(oracle.attention(q, k, v), oracle.attention(q, k[perm], v[perm]), atol=1e-13)
    assert np.allclose(oracle.attention(q[perm], k, v), oracle.attention(q, k, v)[perm], atol=1e-13)


# ---------------------------------------------------------------- GELU


def test_gelu_against_math_erf_and_identities():
    xs = np.linspace(-6, 6, 97)
    lib = np.array([0.5 * x * (1 + math.erf(x / math.sqrt(2))) for x in xs])
    assert np.allclose(oracle.gelu(xs), lib, rtol=1e-14, atol=1e-15)
    assert oracle.gelu(np.array([0.0]))[0] == 0.0
    assert np.allclose(oracle.gelu(xs) - oracle.gelu(-xs), xs, atol=1e-14)
    assert np.max(np.abs(oracle.gelu(xs) - oracle.gelu(xs, tanh=True))) < 1e-3
    t = torch.nn.functional.gelu(torch.from_numpy(xs), approximate="tanh").numpy()
    assert np.allclose(oracle.gelu(xs, tanh=True), t, rtol=1e-12, atol=1e-14)


# ---------------------------------------------------------------- Euler / CFG


def test_euler_cfg_closed_forms():
    e = synth.euler_inputs(64)
    x, vc, vu = e["x"], e["v_cond"], e["v_uncond"]
    fc, fu = oracle.bf16_to_f64(vc), oracle.bf16_to_f64(vu)
    dt = -1.0 / 50
    assert np.allclose(oracle.euler_cfg_step(x, vc, vu, 1.0, dt), x + dt * fc, rtol=0, atol=1e-15)
    assert np.allclose(oracle.euler_cfg_step(x, vc, vu, 0.0, dt), x + dt * fu, rtol=0, atol=1e-15)
    assert np.allclose(oracle.euler_cfg_step(x, vc, vc, 4.0, dt), oracle.euler_cfg_step(x, vc, vc, -3.0, dt), atol=1e-15)
    # The deep dive writes gw*v_c + (1-gw)*v_u; the same update as v_u + g*(v_c - v_u).
    assert np.allclose(oracle.euler_cfg_step(x, vc, vu, 4.0, dt), x + dt * (fu + 4.0 * (fc - fu)), atol=1e-13)
    assert np.allclose(oracle.euler_cfg_step(x, vc, vu, 4.0, 0.0), x, atol=0)


# ---------------------------------------------------------------- block and cond


def _tiny_cfg(**kw):
    base = dict(d_model=8, n_heads=2, head_dim=4, d_mlp=16, rope_sections=(1, 0, 1), rope_theta=10000.0, eps=1e-6, gelu_tanh=0)
    base.update(kw)
    return SimpleNamespace(**base)


def _tiny_weights(cfg, seed=10):
    r = np.random.default_rng(seed)
    d, f, hd = cfg.d_model, cfg.d_mlp, cfg.head_dim
    w = {}
    for name, shape in (("w_qkv", (3 * d, d)), ("w_o", (d, d)), ("w_up", (f, d)), ("w_down", (d, f))):
        codes, scale = synth.quantize_rows_e4m3(r.standard_normal(shape).astype(np.float32) * 0.3)
        w[name], w["s_" + name[2:]] = codes, scale
    for name, n in (("g_norm1", d), ("g_norm2", d), ("g_q", hd), ("g_k", hd)):
        w[name] = synth.to_bf16_bits(1.0 + 0.1 * r.standard_normal(n))
    return w


def _block_loops(cfg, w, x, n_text, gh, gw):
    """Whole block as explicit Python loops over tokens, heads and channels."""
    d, H, hd, F, eps = cfg.d_model, cfg.n_heads, cfg.head_dim, cfg.d_mlp, cfg.eps
    S = n_text + gh * gw
    dq = lambda name: oracle.dequant(w["w_" + name], w["s_" + name])  # noqa: E731
    Wqkv, Wo, Wup, Wdn = dq("qkv"), dq("o"), dq("up"), dq("down")
    g1, g2 = oracle.bf16_to_f64(w["g_norm1"]), oracle.bf16_to_f64(w["g_norm2"])
    gq, gk = oracle.bf16_to_f64(w["g_q"]), oracle.bf16_to_f64(w["g_k"])

    def norm(vec, g):
        ms = sum(t * t for t in vec) / len(vec)
        return [vec[i] / math.sqrt(ms + eps) * g[i] for i in range(len(vec))]

    def pos_of(s):
        if s < n_text:
            return (s, s, s)
        r, c = divmod(s - n_text, gw)
        return (n_text, r, c)

    secs = cfg.rope_sections

    def rot(vec, p):
        out = list(vec)
        for i in range(hd // 2):
            axis = 0 if i < secs[0] else (1 if i < secs[0] + secs[1] else 2)
            ang = p[axis] * float(np.float32(cfg.rope_theta ** (-2.0 * i / hd)))
            a, b = vec[i], vec[i + hd // 2]
            out[i] = a * math.cos(ang) - b * math.sin(ang)
            out[i + hd // 2] = b * math.cos(ang) + a * math.sin(ang)
        return out

    hs = [norm(list(x[s]), g1) for s in range(S)]
    qkv = [[sum(hs[s][c] * Wqkv[o, c] for c in range(d)) for o in range(3 * d)] for s in range(S)]
    Q = [[rot(norm(qkv[s][h * hd:(h + 1) * hd], gq), pos_of(s)) for h in range(H)] for s in range(S)]
    K = [[rot(norm(qkv[s][d + h * hd:d + (h + 1) * hd], gk), pos_of(s)) for h in range(H)] for s in range(S)]
    V = [[qkv[s][2 * d + h * hd:2 * d + (h + 1) * hd] for h in range(H)] for s in range(S)]
    y = np.zeros((S, d))
    for s in range(S):
        o = []
        for h in range(H):
            logits = [sum(Q[s][h][c] * K[t][h][c] for c in range(hd)) / math.sqrt(hd) for t in range(S)]
            m = max(logits)
            ws = [math.exp(l - m) for l in logits]
            o += [sum(ws[t] * V[t][h][c] for t in range(S)) / sum(ws) for c in range(hd)]
        x1 = [x[s][c] + sum(o[i] * Wo[c, i] for i in range(d)) for c in range(d)]
        h2 = norm(x1, g2)
        u = [0.5 * a * (1 + math.erf(a / math.sqrt(2))) for a in (sum(h2[c] * Wup[j, c] for c in range(d)) for j in range(F))]
        y[s] = [x1[c] + sum(u[j] * Wdn[c, j] for j in range(F)) for c in range(d)]
    return y


def test_block_brute_force_tiny():
    cfg = _tiny_cfg()
    w = _tiny_weights(cfg)
    r = np.random.default_rng(11)
    n_text, gh, gw = 2, 2, 2
    x_bits = synth.to_bf16_bits(r.standard_normal((1, n_text + gh * gw, cfg.d_model)))
    got = oracle.dit_block_forward(cfg, w, x_bits, n_text, gh, gw)[0]
    want = _block_loops(cfg, w, oracle.bf16_to_f64(x_bits)[0], n_text, gh, gw)
    assert np.allclose(got, want, rtol=1e-11, atol=1e-11)


def test_block_residual_special_cases():
    cfg = _tiny_cfg()
    w = _tiny_weights(cfg)
    r = np.random.default_rng(12)
    x_bits = synth.to_bf16_bits(r.standard_normal((1, 6, cfg.d_model)))
    x = oracle.bf16_to_f64(x_bits)
    z = dict(w)
    z["w_o"] = np.zeros_like(w["w_o"])
    z["w_down"] = np.zeros_like(w["w_down"])
    assert np.array_equal(oracle.dit_block_forward(cfg, z, x_bits, 2, 2, 2), x)
    z = dict(w)
    z["w_up"] = np.zeros_like(w["w_up"])
    full = oracle.dit_block_forward(cfg, w, x_bits, 2, 2, 2)
    attn_only = oracle.dit_block_forward(cfg, z, x_bits, 2, 2, 2)
    assert not np.allclose(full, attn_only)
    z2 = dict(z)
    z2["w_o"] = np.zeros_like(w["w_o"])
    assert np.array_equal(oracle.dit_block_forward(cfg, z2, x_bits, 2, 2, 2), x)


def test_block_sampled_rows_match_full():
    cfg = _tiny_cfg()
    w = _tiny_weights(cfg)
    x_bits = synth.to_bf16_bits(np.random.default_rng(13).standard_normal((2, 7, cfg.d_model)))
    full = oracle.dit_block_forward(cfg, w, x_bits, 3, 2, 2)
    rows = np.array([6, 0, 3])
    part = oracle.dit_block_forward(cfg, w, x_bits, 3, 2, 2, rows=rows)
    assert np.allclose(part, full[:, rows], rtol=1e-13, atol=1e-13)


def test_cond_proj_identity_weight():
    """Unit gain and an identity weight (code 0x38 = 1.0 on the diagonal): output = normalised features."""
    r = np.random.default_rng(14)
    feats = synth.to_bf16_bits(r.standard_normal((4, 12)))
    g = synth.to_bf16_bits(np.ones(12))
    codes = np.zeros((5, 12), dtype=np.uint8)
    codes[np.arange(5), np.arange(5)] = 0x38
    out = oracle.cond_proj_forward(feats, g, 1e-6, codes, np.full(5, 2.0, dtype=np.float32))
    f = oracle.bf16_to_f64(feats)
    norm = f / np.sqrt(np.mean(f * f, axis=1, keepdims=True) + 1e-6)
    assert np.allclose(out, 2.0 * norm[:, :5], rtol=1e-14)


def test_block_flop_count():
    s = synth.C1024
    assert s.seq == 4608
    assert abs(s.flops() - 2.203e12) / 2.203e12 < 1e-3
    assert abs(synth.UNCOND1024.flops() - 1.941e12) / 1.941e12 < 1e-3


# ---------------------------------------------------------------- stacks of blocks


def test_bf16_decode_all_patterns_match_torch():
    """Every one of the 65,536 bf16 bit patterns decoded by the oracle against torch's own
    bfloat16 -> float64 cast (a library routine): normals, subnormals, both zeros (sign kept),
    both infinities and every NaN pattern (NaN in, NaN out)."""
    pats = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):  # NaN patterns pass through the float32 -> float64 cast
        got = oracle.bf16_to_f64(pats)
    want = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(got), np.isnan(want))
    fin = ~np.isnan(want)
    assert np.array_equal(got[fin], want[fin])
    assert np.array_equal(np.signbit(got[fin]), np.signbit(want[fin]))
    # spot values fixed by the format: 0x3F80 = 1, 0xC000 = -2, 0x0001 = 2^-133, 0x7F80 = +inf
    assert oracle.bf16_to_f64(np.array([0x3F80, 0xC000, 0x0001, 0x7F80], dtype=np.uint16)).tolist() == \
        [1.0, -2.0, 2.0 ** -133, math.inf]


def test_bf16_rounding_matches_torch():
    """The oracle's fp64 -> bf16 rounding against torch's own bf16 cast (a library routine),
    on random values, exact ties, huge and tiny magnitudes."""
    r = np.random.default_rng(21)
    x = np.concatenate([r.standard_normal(4096) * 10.0 ** r.integers(-30, 30, 4096),
                        np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -1.0 - 2.0 ** -8, 3.0e38, -3.0e38, 0.0, -0.0,
                                  1e-40, 2.0 ** -133])])
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f64_to_bf16_bits(x), want)


def test_stack_of_blocks_with_zero_outputs_is_identity():
    """Blocks whose output projections are zero pass x through exactly, so a stack of them
    returns x; a single-block stack is the block itself."""
    cfg = _tiny_cfg()
    w = _tiny_weights(cfg)
    r = np.random.default_rng(22)
    x_bits = synth.to_bf16_bits(r.standard_normal((1, 6, cfg.d_model)))
    z = dict(w)
    z["w_o"] = np.zeros_like(w["w_o"])
    z["w_down"] = np.zeros_like(w["w_down"])
    assert np.array_equal(oracle.dit_stack_forward(cfg, [z, z, z], x_bits, 2, 2, 2), oracle.bf16_to_f64(x_bits))
    assert np.array_equal(oracle.dit_stack_forward(cfg, [w], x_bits, 2, 2, 2),
                          oracle.dit_block_forward(cfg, w, x_bits, 2, 2, 2))
    # a zero block after a real one returns the real block's output rounded to bf16
    two = oracle.dit_stack_forward(cfg, [w, z], x_bits, 2, 2, 2)
    one = oracle.dit_block_forward(cfg, w, x_bits, 2, 2, 2)
    assert np.array_equal(two, oracle.bf16_to_f64(oracle.f64_to_bf16_bits(one)))
    assert not np.array_equal(two, one)


# ---------------------------------------------------------------- padded batches of prompts


def test_padded_text_with_full_lengths_is_the_plain_block():
    cfg = _tiny_cfg()
    w = _tiny_weights(cfg)
    x_bits = synth.to_bf16_bits(np.random.default_rng(31).standard_normal((2, 5 + 4, cfg.d_model)))
    plain = oracle.dit_block_forward(cfg, w, x_bits, 5, 2, 2)
    assert np.array_equal(oracle.dit_block_forward(cfg, w, x_bits, 5, 2, 2, text_lens=[5, 5]), plain)


def test_padded_text_rows_equal_each_prompt_alone():
    """A batch of prompts with 3 and 5 text tokens, each followed by its 2x3 image tokens and padded
    at the end to 5 + 6 rows: every real row equals the block run on that prompt alone (its own
    positions, no padding); padding is invisible as a key."""
    cfg = _tiny_cfg()
    w = _tiny_weights(cfg)
    r = np.random.default_rng(32)
    n_text, gh, gw = 5, 2, 3
    x_bits = synth.to_bf16_bits(r.standard_normal((2, n_text + gh * gw, cfg.d_model)))
    lens = [3, 5]
    got = oracle.dit_block_forward(cfg, w, x_bits, n_text, gh, gw, text_lens=lens)
    for b, L in enumerate(lens):
        n = L + gh * gw
        alone = oracle.dit_block_forward(cfg, w, x_bits[b:b + 1, :n], L, gh, gw)[0]
        assert np.allclose(got[b, :n], alone, rtol=1e-12, atol=1e-12)
    # the padding rows' contents change nothing else
    x2 = x_bits.copy()
    x2[0, 3 + gh * gw:] = synth.to_bf16_bits(r.standard_normal((2, cfg.d_model)) * 7.0)
    got2 = oracle.dit_block_forward(cfg, w, x2, n_text, gh, gw, text_lens=lens)
    assert np.array_equal(got2[0, :3 + gh * gw], got[0, :3 + gh * gw])
    assert np.array_equal(got2[1], got[1])


def test_masked_attention_equals_attention_over_the_kept_keys():
    r = np.random.default_rng(33)
    q, k, v = (r.standard_normal((4, 2, 8)), r.standard_normal((7, 2, 8)), r.standard_normal((7, 2, 8)))
    keep = np.array([1, 0, 1, 1, 0, 0, 1], dtype=bool)
    assert np.allclose(oracle.attention(q, k, v, keep), oracle.attention(q, k[keep], v[keep]), rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- denoising steps and the guidance schedule


def test_guidance_schedule_and_depth_follow_the_pages():
    """V4_QUALITY_48 and the DiT depth as the pages print them (tests/golden/page_facts.json)."""
    from joint_attention_block_b200 import schedule

    f = facts()
    q = f["v4_quality_48"]["value"]
    gw = schedule.guidance("V4_QUALITY_48")
    assert len(gw) == q["steps"] == q["n_first"] + q["n_last"]
    assert gw[: q["n_first"]] == [float(q["gw_first"])] * q["n_first"]
    assert gw[q["n_first"]:] == [float(q["gw_last"])] * q["n_last"]
    assert schedule.DIT_LAYERS == f["dit_layers"]["value"]
    dts = schedule.uniform_dts(q["steps"])
    assert len(dts) == q["steps"] and abs(sum(dts) + 1.0) < 1e-6  # t runs from 1 to 0
    assert all(d == np.float32(-1.0 / q["steps"]) for d in dts)


def _zero_out(w):
    z = dict(w)
    z["w_o"] = np.zeros_like(w["w_o"])
    z["w_down"] = np.zeros_like(w["w_down"])
    return z


def test_denoise_with_identity_stacks_is_a_closed_form():
    """Stacks whose output projections are zero return their input, so each branch's velocity is
    bf16(z) and every step is z + dt * bf16(z), whatever the guidance."""
    cfg = _tiny_cfg()
    w = _zero_out(_tiny_weights(cfg))
    r = np.random.default_rng(40)
    z0 = r.standard_normal((1, 4, cfg.d_model))
    tc = synth.to_bf16_bits(r.standard_normal((1, 3, cfg.d_model)))
    tu = synth.to_bf16_bits(np.zeros((1, 2, cfg.d_model)))
    got = oracle.denoise_steps(cfg, [w, w], [w], tc, tu, z0, 2, 2, [7.0, 3.0], [-0.25, -0.5])
    want = z0.copy()
    for dt in (-0.25, -0.5):
        want = want + dt * oracle.bf16_to_f64(oracle.f64_to_bf16_bits(want))
    assert np.array_equal(got, want)


def test_denoise_guidance_one_and_zero_drop_a_branch():
    """gw = 1 uses only the conditional branch and gw = 0 only the unconditional one: changing the
    other branch's weights changes nothing."""
    cfg = _tiny_cfg()
    wa, wb, wc = _tiny_weights(cfg, 41), _tiny_weights(cfg, 42), _tiny_weights(cfg, 43)
    r = np.random.default_rng(44)
    z0 = r.standard_normal((1, 4, cfg.d_model))
    tc = synth.to_bf16_bits(r.standard_normal((1, 3, cfg.d_model)))
    tu = synth.to_bf16_bits(np.zeros((1, 1, cfg.d_model)))
    one = [oracle.denoise_steps(cfg, [wa], [u], tc, tu, z0, 2, 2, [1.0], [-0.1]) for u in (wb, wc)]
    assert np.array_equal(one[0], one[1])
    zero = [oracle.denoise_steps(cfg, [c], [wb], tc, tu, z0, 2, 2, [0.0], [-0.1]) for c in (wa, wc)]
    assert np.array_equal(zero[0], zero[1])
    assert not np.array_equal(one[0], zero[0])


# ---------------------------------------------------------------- FP8 activations (W8A8 variant)


def test_e4m3_round_matches_torch_float8_cast():
    """The oracle's e4m3 rounding against torch's float32 -> float8_e4m3fn cast (a library routine)
    on random in-range values, every exact tie between neighbouring codes, subnormals and zeros;
    values beyond 448 saturate."""
    r = np.random.default_rng(80)
    x = np.concatenate([r.standard_normal(20000) * 10.0 ** r.uniform(-3, 2.6, 20000),
                        r.uniform(-448, 448, 5000), [0.0, -0.0, 2.0 ** -9, 2.0 ** -10, 3 * 2.0 ** -10, 448.0, -448.0]])
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_to_f64(codes)
    fin = np.sort(np.unique(vals[np.isfinite(vals)]))
    ties = (fin[:-1] + fin[1:]) / 2.0  # halfway points: ties to even
    x = np.concatenate([x, ties]).astype(np.float32)
    x = x[np.abs(x) <= 448.0]
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(oracle.e4m3_round(x.astype(np.float64)), want)
    assert oracle.e4m3_round(np.array([500.0, -1e6, 449.0]))[:].tolist() == [448.0, -448.0, 448.0]
    assert np.array_equal(oracle.e4m3_round(fin), fin)  # every code is a fixed point


def test_activation_quantiser_scale_and_range():
    r = np.random.default_rng(81)
    h = r.standard_normal((5, 64)) * np.array([[1.0], [0.01], [100.0], [3.0], [0.5]])
    h[3] = 0.0
    q, s = oracle.quantize_rows_act(h)
    amax = np.abs(h).max(axis=1)
    assert np.array_equal(s, np.where(amax > 0, (amax / 448.0).astype(np.float32), 1.0))
    assert np.all(np.abs(q).max(axis=1)[amax > 0] <= 448.0 * s[amax > 0] * (1 + 1e-12))
    assert np.array_equal(q[3], np.zeros(64))
    # relative error of each element at most half an e4m3 step (2^-4 of its binade), or the subnormal step
    err = np.abs(q - h) / s[:, None]
    mag = np.abs(h) / s[:, None]
    bound = np.maximum(np.exp2(np.floor(np.log2(np.maximum(mag, 2.0 ** -6))) - 4.0), 2.0 ** -10)
    assert np.all(err <= bound * (1 + 1e-12))
    q2, s2 = oracle.quantize_rows_act(q)
    assert np.allclose(q2, q, rtol=0, atol=1e-12 * np.abs(q).max())  # quantised rows stay put


def test_qk_e4m3_scale_is_reached_by_a_one_hot_head_and_never_exceeded():
    """The static q/k scale against the closed-form bound it rests on: a head vector with all its
    energy in the component of the largest gain comes out of the per-head RMSNorm at sqrt(hd) times
    that gain (up to eps), i.e. at code 448 exactly; random head vectors, rotated by M-RoPE at
    random positions, never exceed it; and the rounding error is at most half an e4m3 step."""
    r = np.random.default_rng(83)
    for hd in (64, 128):
        g_bits = synth.to_bf16_bits(1.0 + 0.05 * r.standard_normal(hd))
        g = oracle.bf16_to_f64(g_bits)
        s = oracle.qk_e4m3_scale(g, hd)
        assert s == float(np.float32(np.float32(np.sqrt(np.float32(hd)) * np.float32(np.abs(g).max())) / np.float32(448)))
        i = int(np.argmax(np.abs(g)))
        x = np.zeros((1, 1, hd))
        x[0, 0, i] = 1000.0  # eps negligible against mean(x^2) = 1e6 / hd
        xn = oracle.rmsnorm(x, g, 1e-6)
        assert abs(abs(xn[0, 0, i]) - np.sqrt(hd) * np.abs(g).max()) < 1e-8
        assert abs(oracle.quantize_qk(xn, s)[0, 0, i]) / s == 448.0
        secs = (8, 12, 12) if hd == 64 else (24, 20, 20)
        xs = r.standard_normal((200, 3, hd)) * np.exp(r.uniform(-3, 3, (200, 3, 1)))
        xs[:, 0, :] = 0.0
        xs[:, 0, r.integers(0, hd, 200)] = 1.0  # some one-hot heads among them
        pos = r.integers(0, 4096, (200, 3))
        y = oracle.mrope(oracle.rmsnorm(xs, g, 1e-6), pos, secs, 1e4)
        assert np.abs(y).max() / s <= 448.0 * (1 + 1e-9)
        qy = oracle.quantize_qk(y, s)
        mag = np.abs(y) / s
        bound = np.maximum(np.exp2(np.floor(np.log2(np.maximum(mag, 2.0 ** -6))) - 4.0), 2.0 ** -10)
        assert np.all(np.abs(qy - y) / s <= bound * (1 + 1e-9))


def test_w8a8_block_is_the_block_with_quantised_norm_outputs():
    """The W8A8 block differs from the W8A16 block only through the two quantised inputs: with the
    attention and MLP output projections zeroed both reduce to the residual path exactly, and with
    real weights the difference is the few per cent that e4m3 activations cost."""
    cfg = _tiny_cfg()
    w = _zero_out(_tiny_weights(cfg))
    x_bits = synth.to_bf16_bits(np.random.default_rng(82).standard_normal((1, 6, cfg.d_model)))
    a = oracle.dit_block_forward(cfg, w, x_bits, 2, 2, 2, w8a8=True)
    assert np.array_equal(a, oracle.bf16_to_f64(x_bits))
    w2 = _tiny_weights(cfg)
    b16 = oracle.dit_block_forward(cfg, w2, x_bits, 2, 2, 2)
    b8 = oracle.dit_block_forward(cfg, w2, x_bits, 2, 2, 2, w8a8=True)
    assert not np.array_equal(b8, b16)
    assert np.abs(b8 - b16).max() / np.abs(b16).max() < 0.1  # a few per cent from e4m3 activations
