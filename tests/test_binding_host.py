"""The Python binding on the host: loud failure without the library, argument marshalling,
and errors surfaced as exceptions (no GPU needed)."""
import ctypes

import pytest
import torch

from joint_attention_block_b200 import _abi, synth


def test_missing_library_raises_instead_of_falling_back(monkeypatch):
    monkeypatch.setattr(_abi, "_LIB", None)
    monkeypatch.setattr(_abi, "LIB_PATH", "/nonexistent/libjab_b200.so")
    with pytest.raises(ImportError, match="no CPU fallback"):
        _abi.lib()


def test_non_contiguous_tensors_are_rejected():
    t = torch.zeros(8, 8)
    assert _abi._ptr(None) is None
    assert _abi._ptr(t) == t.data_ptr()
    with pytest.raises(ValueError):
        _abi._ptr(t.t())


def test_config_struct_carries_the_shape():
    s = synth.C1024
    c = _abi.make_config(s)
    assert (c.d_model, c.n_heads, c.head_dim, c.d_mlp) == (4096, 32, 128, 16384)
    assert list(c.rope_sections) == [24, 20, 20]
    assert c.rope_theta == 10000.0 and abs(c.eps - 1e-6) < 1e-12 and c.gelu_tanh == 0


def test_weights_struct_takes_every_named_pointer():
    names = [n for n, _ in _abi.BlockWeights._fields_]
    assert names == ["w_qkv", "w_o", "w_up", "w_down", "s_qkv", "s_o", "s_up", "s_down", "g_norm1", "g_norm2",
                     "g_q", "g_k"]
    tensors = {n: torch.zeros(16, dtype=torch.uint8) for n in names}
    w = _abi.make_weights(tensors)
    for n in names:
        assert getattr(w, n) == tensors[n].data_ptr()


def test_status_codes_become_exceptions_with_the_library_text():
    from joint_attention_block_b200 import build

    build.build()
    cfg = _abi.make_config(synth.TINY)
    w = _abi.BlockWeights()
    x = torch.zeros(1, synth.TINY.seq, synth.TINY.d_model, dtype=torch.int16)
    with pytest.raises(_abi.DitError) as e:  # null weight pointers: invalid argument, checked on the host
        _abi.dit_block_forward(cfg, w, x, torch.zeros_like(x), 16, 8, 8, torch.zeros(256, dtype=torch.uint8),
                               stream=0)
    assert e.value.status == 1 and "invalid" in str(e.value).lower()
