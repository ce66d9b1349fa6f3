"""The FP8 checkpoint reader against shards written by the safetensors package itself.

The layout facts tested here (unsloth diffusion_ideogram4.py commit log, fp8 loader commit and
its review follow-ups): the fp8 marker is a ``*.weight_scale`` key found in ANY shard header;
attention.qkv.weight is fused [3*hidden, hidden] and a different row count fails loudly; the
real weight is fp8 * weight_scale[:, None]; unmatched keys fail loudly.
"""
import dataclasses
import os
import struct

import numpy as np
import pytest
import torch
from safetensors import safe_open
from safetensors.torch import save_file

import oracle
from joint_attention_block_b200 import synth
from joint_attention_block_b200.fp8_checkpoint import (
    DEFAULT_NAMES, CheckpointError, ShardIndex, infer_block_dims, load_stack, read_block)

TINY = synth.TINY


def _block_tensors(inp, block, names=DEFAULT_NAMES, prefix="layers.{i}."):
    """The tiny block's synthetic weights as the checkpoint stores them (float8 codes, fp32
    scales, bf16 gains) under their checkpoint keys."""
    p = prefix.format(i=block)
    out = {}
    for f in ("w_qkv", "w_o", "w_up", "w_down"):
        out[p + names[f]] = torch.from_numpy(inp[f].copy()).view(torch.float8_e4m3fn)
        out[p + names["s" + f[1:]]] = torch.from_numpy(inp["s" + f[1:]].copy())
    for g in ("g_norm1", "g_norm2", "g_q", "g_k"):
        out[p + names[g]] = torch.from_numpy(inp[g].view(np.int16).copy()).view(torch.bfloat16)
    return out


def _inputs(block):
    return synth.block_inputs(dataclasses.replace(TINY, index=10 + block))


def _write(tmp_path, shards):
    paths = []
    for i, tensors in enumerate(shards):
        p = os.path.join(tmp_path, f"model-{i:05d}-of-{len(shards):05d}.safetensors")
        save_file({k: v.contiguous() for k, v in tensors.items()}, p, metadata={"format": "pt"})
        paths.append(p)
    return paths


def _two_block_shards(tmp_path):
    t0, t1 = _block_tensors(_inputs(0), 0), _block_tensors(_inputs(1), 1)
    allk = {**t0, **t1}
    keys = sorted(allk)
    # Interleave the keys over three shards so each block spans several files.
    shards = [{k: allk[k] for k in keys[j::3]} for j in range(3)]
    return _write(tmp_path, shards), allk


def test_header_entries_match_the_safetensors_reader(tmp_path):
    g = torch.Generator().manual_seed(3)
    tensors = {
        "a.f32": torch.randn(5, 7, generator=g),
        "b.bf16": torch.randn(3, generator=g).to(torch.bfloat16),
        "c.f16": torch.randn(2, 2, 2, generator=g).to(torch.float16),
        "d.e4m3": torch.randn(4, 9, generator=g).to(torch.float8_e4m3fn),
        "e.i32": torch.arange(11, dtype=torch.int32),
        "f.empty": torch.zeros(0, 4),
    }
    (path,) = _write(tmp_path, [tensors])
    idx = ShardIndex([path])
    assert idx.metadata[path] == {"format": "pt"}
    want_dtype = {"a.f32": "F32", "b.bf16": "BF16", "c.f16": "F16", "d.e4m3": "F8_E4M3", "e.i32": "I32", "f.empty": "F32"}
    with safe_open(path, framework="pt") as f:
        assert sorted(f.keys()) == idx.keys()
        for k in f.keys():
            ref = f.get_tensor(k)
            e = idx.entry(k)
            assert e.dtype == want_dtype[k] and e.shape == tuple(ref.shape)
            assert idx.read_bytes(k).tobytes() == ref.contiguous().view(torch.uint8).numpy().tobytes()


def test_round_trip_of_two_blocks_over_three_shards(tmp_path):
    paths, _ = _two_block_shards(tmp_path)
    st = load_stack(paths, device="cpu")
    assert st.dims.d_model == TINY.d_model and st.dims.head_dim == TINY.head_dim
    assert st.dims.n_heads == TINY.n_heads and st.dims.d_mlp == TINY.d_mlp
    assert len(st.blocks) == 2 and st.unclaimed == []
    for b in range(2):
        inp = _inputs(b)
        blk = st.blocks[b]
        for f in ("w_qkv", "w_o", "w_up", "w_down", "s_qkv", "s_o", "s_up", "s_down"):
            assert blk[f].numpy().tobytes() == np.ascontiguousarray(inp[f]).tobytes(), (b, f)
        for g in ("g_norm1", "g_norm2", "g_q", "g_k"):
            assert blk[g].dtype == torch.int16
            assert np.array_equal(blk[g].numpy().view(np.uint16), inp[g]), (b, g)


def test_scale_indexes_the_output_row(tmp_path):
    """The loaded codes and scales, dequantised by the oracle, equal the pages' formula
    fp8.float() * weight_scale[:, None] evaluated by torch on the stored tensors."""
    paths, allk = _two_block_shards(tmp_path)
    arrays = read_block(ShardIndex(paths), 1)
    for f in ("w_qkv", "w_o", "w_up", "w_down"):
        key = "layers.1." + DEFAULT_NAMES[f]
        ref = allk[key].to(torch.float64) * allk[key + "_scale"].to(torch.float64)[:, None]
        got = oracle.dequant(arrays[f], arrays["s" + f[1:]])
        assert np.array_equal(got, ref.numpy()), f
    # Q, K and V are the first, second and third thirds of the fused rows.
    d = TINY.d_model
    w = oracle.dequant(arrays["w_qkv"], arrays["s_qkv"])
    key = "layers.1.attention.qkv.weight"
    full = allk[key].to(torch.float64) * allk[key + "_scale"].to(torch.float64)[:, None]
    for j in range(3):
        assert np.array_equal(w[j * d:(j + 1) * d], full[j * d:(j + 1) * d].numpy())


def test_marker_found_in_any_shard(tmp_path):
    t = _block_tensors(_inputs(0), 0)
    gains = {k: v for k, v in t.items() if not k.endswith("_scale") and v.dtype == torch.bfloat16}
    rest = {k: v for k, v in t.items() if k not in gains}
    paths = _write(tmp_path, [gains, rest])
    assert ShardIndex(paths).fp8_layout()
    assert not ShardIndex(paths[:1]).fp8_layout()
    assert len(load_stack(paths, device="cpu").blocks) == 1


def test_dense_layout_is_refused(tmp_path):
    t = _block_tensors(_inputs(0), 0)
    dense = {k: (v.to(torch.bfloat16) if v.dtype == torch.float8_e4m3fn else v)
             for k, v in t.items() if not k.endswith("_scale")}
    paths = _write(tmp_path, [dense])
    assert not ShardIndex(paths).fp8_layout()
    with pytest.raises(CheckpointError, match="not the fp8 layout"):
        load_stack(paths, device="cpu")


def test_unscaled_bf16_projection_is_refused(tmp_path):
    t = _block_tensors(_inputs(0), 0)
    t["layers.0.feed_forward.up.weight"] = t["layers.0.feed_forward.up.weight"].to(torch.bfloat16)
    with pytest.raises(CheckpointError, match="e4m3 weights"):
        load_stack(_write(tmp_path, [t]), device="cpu")


def test_grouped_query_qkv_fails_loudly(tmp_path):
    t = _block_tensors(_inputs(0), 0)
    d = TINY.d_model
    k = "layers.0.attention.qkv.weight"
    t[k] = t[k][: d + 2 * (d // 4)].clone()
    t[k + "_scale"] = t[k + "_scale"][: d + 2 * (d // 4)].clone()
    with pytest.raises(CheckpointError, match="3 x hidden"):
        load_stack(_write(tmp_path, [t]), device="cpu")


def test_unmatched_keys_fail_loudly(tmp_path):
    t = _block_tensors(_inputs(0), 0)
    t["layers.0.attention.qkv.bias"] = torch.zeros(3 * TINY.d_model)
    with pytest.raises(CheckpointError, match="unmatched keys: layers.0.attention.qkv.bias"):
        load_stack(_write(tmp_path, [t]), device="cpu")


def test_keys_outside_the_blocks_need_an_allowed_prefix(tmp_path):
    t = _block_tensors(_inputs(0), 0)
    t["x_embedder.weight"] = torch.zeros(4, 4)
    t["layers.7.attention.o.weight"] = torch.zeros(2, 2)  # past the blocks asked for
    paths = _write(tmp_path, [t])
    with pytest.raises(CheckpointError, match="unmatched keys: layers.7.attention.o.weight, x_embedder.weight"):
        load_stack(paths, device="cpu", n_blocks=1)
    with pytest.raises(CheckpointError, match="layers.7"):
        load_stack(paths, device="cpu", n_blocks=1, allow_unclaimed=("x_embedder.",))
    del t["layers.7.attention.o.weight"]
    st = load_stack(_write(tmp_path, [t]), device="cpu", allow_unclaimed=("x_embedder.",))
    assert st.unclaimed == ["x_embedder.weight"] and len(st.blocks) == 1


def test_missing_field_fails_loudly(tmp_path):
    t = _block_tensors(_inputs(0), 0)
    del t["layers.0.attention.norm_k.weight"]
    with pytest.raises(CheckpointError, match="norm_k.weight' is in no shard"):
        load_stack(_write(tmp_path, [t]), device="cpu")


def test_scale_forms(tmp_path):
    t = _block_tensors(_inputs(0), 0)
    k = "layers.0.attention.o.weight_scale"
    s = t[k].clone()
    t[k] = s[:, None].clone()  # [out, 1] broadcasts by rank
    a = read_block(ShardIndex(_write(tmp_path, [t])), 0)
    assert np.array_equal(a["s_o"], s.numpy())
    t[k] = s.to(torch.bfloat16)  # widened exactly
    a = read_block(ShardIndex(_write(tmp_path, [t])), 0)
    assert np.array_equal(a["s_o"], s.to(torch.bfloat16).to(torch.float32).numpy())
    t[k] = torch.stack([s, s], dim=1)
    with pytest.raises(CheckpointError, match="one scale per output row"):
        read_block(ShardIndex(_write(tmp_path, [t])), 0)


def test_f32_gains_cast_to_bf16_nearest_even(tmp_path):
    t = _block_tensors(_inputs(0), 0)
    k = "layers.0.attention_norm.weight"
    # 1 + 2^-8 is a tie between two bf16 values and must go to the even one (1.0); 1 + 3*2^-9
    # rounds up to 1 + 2^-7.
    v = torch.full((TINY.d_model,), 1.0 + 2.0 ** -8)
    v[1] = 1.0 + 3 * 2.0 ** -9
    t[k] = v
    a = read_block(ShardIndex(_write(tmp_path, [t])), 0)
    assert a["g_norm1"][0] == 0x3F80 and a["g_norm1"][1] == 0x3F81


def test_nan_codes_are_refused(tmp_path):
    t = _block_tensors(_inputs(0), 0)
    k = "layers.0.feed_forward.down.weight"
    raw = t[k].view(torch.uint8).clone()
    raw[3, 5] = 0xFF
    t[k] = raw.view(torch.float8_e4m3fn)
    with pytest.raises(CheckpointError, match="NaN"):
        load_stack(_write(tmp_path, [t]), device="cpu")


def test_duplicate_key_across_shards(tmp_path):
    t = _block_tensors(_inputs(0), 0)
    k = "layers.0.attention.norm_q.weight"
    with pytest.raises(CheckpointError, match="in both"):
        ShardIndex(_write(tmp_path, [t, {k: t[k]}]))


def test_corrupt_headers(tmp_path):
    (path,) = _write(tmp_path, [{"a": torch.zeros(8)}])
    raw = open(path, "rb").read()
    bad = os.path.join(tmp_path, "bad.safetensors")
    open(bad, "wb").write(raw[:-4])  # data section shorter than the offsets
    with pytest.raises(CheckpointError, match="needs 32 bytes"):
        ShardIndex([bad])
    open(bad, "wb").write(struct.pack("<Q", 1 << 40) + raw[8:])
    with pytest.raises(CheckpointError, match="does not fit"):
        ShardIndex([bad])
    hdr = b'{"a": {"dtype": "F32", "shape": [8], "data_offsets": [0, 16]}}'
    open(bad, "wb").write(struct.pack("<Q", len(hdr)) + hdr + bytes(32))
    with pytest.raises(CheckpointError, match="needs 32 bytes"):
        ShardIndex([bad])
    hdr = b'{"a": {"dtype": "Q7", "shape": [8], "data_offsets": [0, 8]}}'
    open(bad, "wb").write(struct.pack("<Q", len(hdr)) + hdr + bytes(8))
    with pytest.raises(CheckpointError, match="unknown dtype"):
        ShardIndex([bad])


def test_infer_dims_of_the_d4608_variant(tmp_path):
    """Only shapes are read: a d = 4608 block (36 heads of 128) is recognised from its headers."""
    d, f, hd = 4608, 4 * 4608, 128
    t = {
        "layers.0.attention.o.weight": torch.zeros(d, d, dtype=torch.float8_e4m3fn),
        "layers.0.feed_forward.up.weight": torch.zeros(f, d, dtype=torch.float8_e4m3fn),
        "layers.0.attention.norm_q.weight": torch.ones(hd, dtype=torch.bfloat16),
        "layers.0.attention.o.weight_scale": torch.ones(d),
    }
    dims = infer_block_dims(ShardIndex(_write(tmp_path, [t])))
    assert (dims.d_model, dims.n_heads, dims.head_dim, dims.d_mlp) == (4608, 36, 128, 18432)


@pytest.mark.gpu
def test_loaded_block_runs_and_matches_the_oracle(tmp_path):
    from joint_attention_block_b200 import ops
    from gpu_util import as_f64, assert_close, dev, poisoned_like, workspace

    paths, _ = _two_block_shards(tmp_path)
    st = load_stack(paths, device="cuda")
    s = TINY
    cfg = ops.make_config(s)
    for b in range(2):
        inp = _inputs(b)
        weights = ops.make_weights(st.blocks[b])
        x = dev(inp["x"])
        out = poisoned_like(x)
        ws = workspace(ops.block_workspace_bytes(cfg, 1, s.n_text, s.grid_h, s.grid_w))
        ops.dit_block_forward(cfg, weights, x, out, s.n_text, s.grid_h, s.grid_w, ws)
        torch.cuda.synchronize()
        ref = oracle.dit_block_forward(s, inp, inp["x"], s.n_text, s.grid_h, s.grid_w)
        assert_close(as_f64(out), ref, what=f"block {b} loaded from shards")
    assert ops.poll_error() == 0
