"""The C-ABI library builds for sm_100a, loads without a GPU and exports every symbol the header declares."""
import ctypes
import os
import re

import pytest

from joint_attention_block_b200 import _abi, build

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "jab_dit.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*DIT_API\s+(?:const\s+)?\w+\s*\*?\s*(\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.lib()


def test_header_declares_the_three_calls():
    names = declared_functions()
    for n in ("dit_block_forward", "cond_proj_forward", "euler_cfg_step"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} declared in include/jab_dit.h but not exported"
        assert name in _abi.SIGNATURES, f"{name} has no Python binding"


def test_host_only_calls_without_gpu(lib):
    assert lib.dit_abi_version() == 2
    assert lib.dit_status_str(0) == b"ok"
    assert lib.dit_status_str(5).startswith(b"device-side bounded wait")
    cfg = _abi.BlockConfig()
    assert lib.dit_block_workspace_bytes(ctypes.byref(cfg), 1, 16, 8, 8) == 0  # invalid config -> 0
    from joint_attention_block_b200 import synth
    good = _abi.make_config(synth.TINY)
    assert lib.dit_block_workspace_bytes(ctypes.byref(good), 1, 16, 8, 8) > 0
    # normalised features (f16) + the fp32 split-K partials of the projection: 9 splits make 144
    # work units for 512 tokens (0.97 of 74 SM pairs busy), 4 splits 512 units for 4096 tokens
    assert lib.cond_proj_workspace_bytes(512, 13, 4096, 4096) == 512 * 53248 * 2 + 9 * 512 * 4096 * 4
    assert lib.cond_proj_workspace_bytes(4096, 13, 4096, 4096) == 4096 * 53248 * 2 + 4 * 4096 * 4096 * 4


def test_argument_validation_without_gpu(lib):
    from joint_attention_block_b200 import synth
    cfg = _abi.make_config(synth.TINY)
    bad = _abi.make_config(synth.TINY)
    bad.rope_sections[0] = 9  # sections no longer sum to head_dim / 2
    w = _abi.BlockWeights()
    assert lib.dit_block_forward(ctypes.byref(bad), ctypes.byref(w), 16, 32, 1, 16, 8, 8, -1, None, None, 0, None) == 1
    assert lib.dit_block_forward(ctypes.byref(cfg), ctypes.byref(w), 16, 32, 1, 16, 8, 8, -1, None, None, 0, None) == 1
    hd96 = _abi.make_config(synth.TINY)
    hd96.head_dim, hd96.n_heads, hd96.d_model = 96, 4, 384
    assert lib.dit_block_forward(ctypes.byref(hd96), ctypes.byref(w), 16, 32, 1, 16, 8, 8, -1, None, None, 0, None) == 2
    wide = _abi.make_config(synth.TINY)  # d_model 8448 > 8192: beyond the one-CTA-per-token QK-norm
    wide.head_dim, wide.n_heads, wide.d_model, wide.d_mlp = 128, 66, 8448, 8448
    wide.rope_sections[0], wide.rope_sections[1], wide.rope_sections[2] = 24, 20, 20
    assert lib.dit_block_workspace_bytes(ctypes.byref(wide), 1, 16, 8, 8) == 0
    assert lib.dit_block_forward(ctypes.byref(wide), ctypes.byref(w), 16, 32, 1, 16, 8, 8, -1, None, None, 0, None) == 2
    assert lib.euler_cfg_step(None, None, None, 8, 4.0, -0.02, None) == 1
    assert lib.euler_cfg_step(None, None, None, 0, 4.0, -0.02, None) == 0  # empty update: nothing to do
    assert lib.dit_gemm_w8a16(16, 0, 16, 16, 16, 0, None, 0, 128, 100, 64, 0, 0, None) == 2  # N % 32 != 0
    assert lib.dit_gemm_w8a16(16, 2, 16, 16, 16, 0, None, 0, 128, 128, 64, 0, 0, None) == 1  # A cannot be fp32
    assert lib.dit_gemm_w8a16(17, 0, 16, 16, 16, 0, None, 0, 128, 128, 64, 0, 0, None) == 1  # misaligned A
    assert lib.dit_gemm_w8a16(16, 0, 16, 16, 16, 0, 32, 7, 128, 128, 64, 0, 0, None) == 1  # bad residual format
    assert lib.cond_proj_forward(16, 4, 13, 4096, 16, 1e-6, 16, 16, 4096, 16, None, 0, None) == 3  # no workspace
    assert lib.dit_rmsnorm_rows(16, 0, 16, 16, 0, 4, 12, 1e-6, None) == 1  # cols % 8
    assert lib.dit_rmsnorm_rows(16, 0, 16, 16, 1, 4, 16, 1e-6, None) == 1  # in place with a format change
    assert lib.dit_joint_attention(16, 32, 2, 1, 8, 2, 64, None) == 1  # fp32 q/k/v
    assert lib.dit_joint_attention(16, 32, 1, 1, 8, 2, 96, None) == 2  # head_dim 96
    assert lib.dit_joint_attention_e4m3(16, 16, 16, 16, 32, 1, 1, 8, 2, 96, None) == 2  # head_dim 96
    assert lib.dit_joint_attention_e4m3(None, 16, 16, 16, 32, 1, 1, 8, 2, 64, None) == 1  # no q8
    assert lib.dit_joint_attention_e4m3(16, 16, 16, 16, 32, 2, 1, 8, 2, 64, None) == 1  # fp32 v
    assert lib.dit_qknorm_mrope_e4m3(16, 1, 1, 16, 8, 8, -1, None, ctypes.byref(cfg), 16, 16, None, 16, 16,
                                     None) == 1  # no q8


def test_noalloc_rejects_shapes_beyond_its_scratch(lib):
    """The 1024 px block needs more than the fixed scratch: rejected before any device work."""
    from joint_attention_block_b200 import synth
    s = synth.C1024
    cfg = _abi.make_config(s)
    assert lib.dit_block_workspace_bytes(ctypes.byref(cfg), 1, s.n_text, s.grid_h, s.grid_w) > _abi.NOALLOC_SCRATCH_BYTES
    w = _abi.BlockWeights()
    rc = lib.dit_block_forward_noalloc(ctypes.byref(cfg), ctypes.byref(w), None, None, 1, s.n_text, s.grid_h,
                                       s.grid_w, -1, None, None)
    assert rc == 2  # DIT_ERR_UNSUPPORTED


def test_stack_workspace_and_validation_without_gpu(lib):
    """The stack's workspace is one block's plus one [B, S, d] bf16 ping-pong buffer; bad calls
    are rejected on the host."""
    from joint_attention_block_b200 import synth
    s = synth.C1024
    cfg = _abi.make_config(s)
    blk = lib.dit_block_workspace_bytes(ctypes.byref(cfg), 1, s.n_text, s.grid_h, s.grid_w)
    assert lib.dit_stack_workspace_bytes(ctypes.byref(cfg), 1, s.n_text, s.grid_h, s.grid_w) == \
        blk + s.seq * s.d_model * 2
    w = (_abi.BlockWeights * 2)()
    # no blocks, null weights, aliasing input and output: INVALID_ARG before any device work
    assert lib.dit_stack_forward(ctypes.byref(cfg), w, 0, 16, 32, 1, s.n_text, s.grid_h, s.grid_w, -1, None,
                                 None, 0, None) == 1
    assert lib.dit_stack_forward(ctypes.byref(cfg), None, 2, 16, 32, 1, s.n_text, s.grid_h, s.grid_w, -1, None,
                                 None, 0, None) == 1
    assert lib.dit_stack_forward(ctypes.byref(cfg), w, 2, 16, 16, 1, s.n_text, s.grid_h, s.grid_w, -1, None,
                                 None, 0, None) == 1
    # no workspace
    assert lib.dit_stack_forward(ctypes.byref(cfg), w, 2, 16, 32, 1, s.n_text, s.grid_h, s.grid_w, -1, None,
                                 None, 0, None) == 3
