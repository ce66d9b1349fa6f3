"""The no-allocation block forward against the regular one (needs a B200).

dit_block_forward_noalloc serves callers that cannot allocate device memory at
call time (hosts that reserve all memory up front, plugin interfaces without an
allocator, latency-critical paths): it takes no workspace and keeps its
intermediates in a fixed array inside the library.  Its results must be those of
dit_block_forward with a caller-provided workspace, on two calls in a row (the
second call finds the first call's leftovers in the shared array).

This file sorts last so that a run stopping at the first failure has already run
every other test.
"""
import numpy as np
import pytest
import torch

from joint_attention_block_b200 import ops, synth
from gpu_util import as_f64, assert_close, dev, workspace

pytestmark = pytest.mark.gpu


def _inputs(shape):
    inp = synth.block_inputs(shape)
    weights = {k: dev(v) for k, v in inp.items() if k != "x"}
    return inp, weights


def test_noalloc_matches_workspace_forward_twice():
    s = synth.TINY
    inp, wd = _inputs(s)
    cfg = ops.make_config(s)
    w = ops.make_weights(wd)
    x = dev(inp["x"])
    ref = torch.empty_like(x)
    ws = workspace(ops.block_workspace_bytes(cfg, 1, s.n_text, s.grid_h, s.grid_w))
    ops.dit_block_forward(cfg, w, x, ref, s.n_text, s.grid_h, s.grid_w, ws)
    torch.cuda.synchronize()
    want = as_f64(ref)
    for call in range(2):
        out = torch.full_like(x, 0x7FC0)  # poison: a bf16 NaN pattern
        ops.dit_block_forward_noalloc(cfg, w, x, out, s.n_text, s.grid_h, s.grid_w)
        assert ops.poll_error() == 0
        assert_close(as_f64(out), want, what=f"no-alloc call {call}")


def test_noalloc_second_shape_after_first():
    """A different (smaller) shape on the same scratch right after a larger one."""
    import dataclasses

    s = dataclasses.replace(synth.TINY, n_text=5, grid_h=3, grid_w=7, batch=2)
    inp, wd = _inputs(s)
    cfg = ops.make_config(s)
    w = ops.make_weights(wd)
    x = dev(inp["x"])
    ref = torch.empty_like(x)
    ws = workspace(ops.block_workspace_bytes(cfg, 2, s.n_text, s.grid_h, s.grid_w))
    ops.dit_block_forward(cfg, w, x, ref, s.n_text, s.grid_h, s.grid_w, ws)
    out = torch.empty_like(x)
    ops.dit_block_forward_noalloc(cfg, w, x, out, s.n_text, s.grid_h, s.grid_w)
    assert ops.poll_error() == 0
    assert_close(as_f64(out), as_f64(ref), what="no-alloc second shape")
