"""Padded batches of prompts on the CUDA path against the oracle (needs a B200).

Prompts of different text lengths share one sequence length (SimpleTuner Ideogram 4
quickstart, "Text Embed Cache": embeddings are cached at each prompt's own length and padded
only when a batch is formed).  Element b holds its L_b text rows, its image rows, then
padding; dit_block_forward_padded must give every real row the value the oracle gives it
(oracle.dit_block_forward with text_lens), which equals that prompt run alone.
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


def run_padded(shape, inp, lens, t_img=-1):
    cfg = ops.make_config(shape)
    w = ops.make_weights({k: dev(v) for k, v in inp.items() if k != "x"})
    x = dev(inp["x"])
    out = poisoned_like(x)
    ws = workspace(ops.block_workspace_bytes(cfg, x.shape[0], shape.n_text, shape.grid_h, shape.grid_w))
    tl = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ops.dit_block_forward_padded(cfg, w, x, out, shape.n_text, shape.grid_h, shape.grid_w, tl, ws, t_img=t_img)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("n_text,gh,gw,lens", [
    (16, 8, 8, [16, 0, 1, 9]),                 # one key block: full, no text, one token, partial
    (140, 6, 6, [0, 1, 140, 70, 100]),        # two key blocks; counts 36, 37, 176, 106, 136
    (200, 1, 1, [200, 127, 128, 3]),          # counts 201, 128 (exactly one block), 129, 4
])
def test_padded_batch_real_rows_match_oracle(n_text, gh, gw, lens):
    s = dataclasses.replace(synth.TINY, index=9, n_text=n_text, grid_h=gh, grid_w=gw, batch=len(lens))
    inp = synth.block_inputs(s)
    got = as_f64(run_padded(s, inp, lens))
    ref = oracle.dit_block_forward(s, inp, inp["x"], n_text, gh, gw, text_lens=lens)
    for b, L in enumerate(lens):
        n = L + gh * gw
        assert_close(got[b, :n], ref[b, :n], what=f"element {b} (L={L})")


def test_padded_batch_with_t_img():
    s = dataclasses.replace(synth.TINY, index=10, n_text=24, grid_h=4, grid_w=5, batch=3)
    lens = [24, 5, 13]
    inp = synth.block_inputs(s)
    got = as_f64(run_padded(s, inp, lens, t_img=7))
    ref = oracle.dit_block_forward(s, inp, inp["x"], s.n_text, s.grid_h, s.grid_w, t_img=7, text_lens=lens)
    for b, L in enumerate(lens):
        n = L + s.n_img
        assert_close(got[b, :n], ref[b, :n], what=f"t_img=7 element {b}")


def test_full_lengths_equal_the_plain_block_bitwise():
    """Every element at the full text length: the padded call is the plain block, bit for bit."""
    s = dataclasses.replace(synth.TINY, index=11, n_text=40, grid_h=5, grid_w=7, batch=3)
    inp = synth.block_inputs(s)
    padded = run_padded(s, inp, [s.n_text] * 3)
    cfg = ops.make_config(s)
    w = ops.make_weights({k: dev(v) for k, v in inp.items() if k != "x"})
    x = dev(inp["x"])
    plain = poisoned_like(x)
    ws = workspace(ops.block_workspace_bytes(cfg, 3, s.n_text, s.grid_h, s.grid_w))
    ops.dit_block_forward(cfg, w, x, plain, s.n_text, s.grid_h, s.grid_w, ws)
    torch.cuda.synchronize()
    assert torch.equal(padded, plain)


def test_padded_element_equals_prompt_alone_on_gpu():
    """A short prompt inside a padded batch gives, on its real rows, what the GPU gives for that
    prompt run alone at its own length (same kernels, fewer rows): within one bf16 rounding."""
    s = dataclasses.replace(synth.TINY, index=12, n_text=30, grid_h=6, grid_w=6, batch=2)
    lens = [30, 11]
    inp = synth.block_inputs(s)
    got = as_f64(run_padded(s, inp, lens))
    alone_s = dataclasses.replace(s, n_text=11, batch=1)
    alone_inp = dict(inp)
    alone_inp["x"] = np.ascontiguousarray(inp["x"][1:2, : 11 + s.n_img])
    cfg = ops.make_config(alone_s)
    w = ops.make_weights({k: dev(v) for k, v in alone_inp.items() if k != "x"})
    x = dev(alone_inp["x"])
    out = poisoned_like(x)
    ws = workspace(ops.block_workspace_bytes(cfg, 1, 11, s.grid_h, s.grid_w))
    ops.dit_block_forward(cfg, w, x, out, 11, s.grid_h, s.grid_w, ws)
    torch.cuda.synchronize()
    assert_close(got[1, : 11 + s.n_img], as_f64(out)[0], max_rel=1e-2, mean_rel=1e-3, what="alone vs padded")


@pytest.mark.slow
def test_padded_1024px_batch_sampled_rows():
    """Two 1024 px prompts (512 and 300 text tokens) in one padded batch, sampled rows of each."""
    s = dataclasses.replace(synth.C1024, batch=2)
    lens = [512, 300]
    inp = synth.block_inputs(s)
    got = as_f64(run_padded(s, inp, lens))
    rng = np.random.default_rng(13)
    for b, L in enumerate(lens):
        n = L + s.n_img
        rows = np.unique(np.concatenate([rng.choice(n, size=10, replace=False), [0, L - 1, L, n - 1]]))
        one = dict(inp)
        one["x"] = np.ascontiguousarray(inp["x"][b:b + 1])
        ref = oracle.dit_block_forward(s, one, one["x"], s.n_text, s.grid_h, s.grid_w, rows=rows, text_lens=[L])
        assert_close(got[b:b + 1, rows], ref, what=f"c1024 padded element {b}")
