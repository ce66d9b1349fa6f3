"""The no-allocation block forward against the regular one (needs a B200).

dit_block_forward_noalloc serves callers that cannot allocate device memory at
call time (hosts that reserve all memory up front, plugin interfaces without an
allocator, latency-critical paths): it takes no workspace and keeps its
intermediates in a fixed array inside the library.  Both entry points launch the
same deterministic kernels, so their results must be bit-identical, on two calls
in a row, after another shape has left unrelated data in the shared array, and
with the regular forward's workspace filled with NaN patterns.

This file sorts last so that a run stopping at the first failure has already run
every other test.
"""
import dataclasses

import numpy as np
import pytest
import torch

from joint_attention_block_b200 import ops, synth
from gpu_util import as_f64, dev, poisoned_like, workspace

pytestmark = pytest.mark.gpu


def _setup(shape):
    inp = synth.block_inputs(shape)
    cfg = ops.make_config(shape)
    w = ops.make_weights({k: dev(v) for k, v in inp.items() if k != "x"})
    x = dev(inp["x"])
    return cfg, w, x


def _reference(shape, cfg, w, x):
    ref = poisoned_like(x)
    ws = workspace(ops.block_workspace_bytes(cfg, x.shape[0], shape.n_text, shape.grid_h, shape.grid_w))  # NaN bytes
    ops.dit_block_forward(cfg, w, x, ref, shape.n_text, shape.grid_h, shape.grid_w, ws)
    assert ops.poll_error() == 0
    assert np.all(np.isfinite(as_f64(ref)))
    return ref


def test_noalloc_matches_workspace_forward_twice():
    # another shape first, so the shared array holds data unrelated to the call under test
    other = dataclasses.replace(synth.TINY, n_text=5, grid_h=3, grid_w=7, batch=2)
    ocfg, ow, ox = _setup(other)
    ops.dit_block_forward_noalloc(ocfg, ow, ox, torch.empty_like(ox), other.n_text, other.grid_h, other.grid_w)
    assert ops.poll_error() == 0

    s = synth.TINY
    cfg, w, x = _setup(s)
    ref = _reference(s, cfg, w, x)
    for call in range(2):
        out = poisoned_like(x)
        ops.dit_block_forward_noalloc(cfg, w, x, out, s.n_text, s.grid_h, s.grid_w)
        assert ops.poll_error() == 0
        assert torch.equal(out, ref), f"no-alloc call {call} differs from dit_block_forward"


def test_noalloc_second_shape_after_first():
    """A different (smaller, batched) shape on the same array right after the tiny one."""
    s = dataclasses.replace(synth.TINY, n_text=5, grid_h=3, grid_w=7, batch=2)
    cfg, w, x = _setup(s)
    ref = _reference(s, cfg, w, x)
    out = poisoned_like(x)
    ops.dit_block_forward_noalloc(cfg, w, x, out, s.n_text, s.grid_h, s.grid_w)
    assert ops.poll_error() == 0
    assert torch.equal(out, ref)
