"""ctypes binding of the C ABI in ``include/jab_dit.h``.

Argument marshalling only: every step runs in the CUDA library.  Device tensors
are passed as raw pointers (``tensor.data_ptr()``) together with the current
torch CUDA stream.  There is no fallback: if the library is missing the import
fails loudly.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libjab_b200.so")

DIT_OK = 0
FMT_BF16, FMT_F16, FMT_F32 = 0, 1, 2
STATUS_NAMES = {
    0: "DIT_OK",
    1: "DIT_ERR_INVALID_ARG",
    2: "DIT_ERR_UNSUPPORTED",
    3: "DIT_ERR_WORKSPACE",
    4: "DIT_ERR_CUDA",
    5: "DIT_ERR_TIMEOUT",
    6: "DIT_ERR_DEVICE",
}


class DitError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = f"{fn} failed: {STATUS_NAMES.get(status, status)} ({lib().dit_status_str(status).decode()})"
        if status == 4:
            msg += f", cudaError {lib().dit_last_cuda_error()}"
        super().__init__(msg)


class BlockConfig(ctypes.Structure):
    _fields_ = [
        ("d_model", ctypes.c_int32),
        ("n_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("d_mlp", ctypes.c_int32),
        ("rope_sections", ctypes.c_int32 * 3),
        ("rope_theta", ctypes.c_float),
        ("eps", ctypes.c_float),
        ("gelu_tanh", ctypes.c_int32),
    ]


class BlockWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_qkv", "w_o", "w_up", "w_down", "s_qkv", "s_o", "s_up", "s_down",
                                                "g_norm1", "g_norm2", "g_q", "g_k")]


_LIB: Optional[ctypes.CDLL] = None

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t

SIGNATURES = {
    "dit_block_workspace_bytes": (_SZ, [ctypes.POINTER(BlockConfig), _I, _I, _I, _I]),
    "dit_block_forward": (_I, [ctypes.POINTER(BlockConfig), ctypes.POINTER(BlockWeights), _P, _P, _I, _I, _I, _I, _I,
                               _P, _P, _SZ, _P]),
    "dit_block_forward_padded": (_I, [ctypes.POINTER(BlockConfig), ctypes.POINTER(BlockWeights), _P, _P, _I, _I, _I,
                                      _I, _I, _P, _P, _SZ, _P]),
    "dit_block_forward_w8a8": (_I, [ctypes.POINTER(BlockConfig), ctypes.POINTER(BlockWeights), _P, _P, _I, _I, _I, _I,
                                    _I, _P, _P, _SZ, _P]),
    "dit_gemm_w8a8": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]),
    "dit_rmsnorm_rows_e4m3": (_I, [_P, _I, _P, _P, _P, _I64, _I64, _F, _P]),
    "dit_block_forward_noalloc": (_I, [ctypes.POINTER(BlockConfig), ctypes.POINTER(BlockWeights), _P, _P, _I, _I,
                                       _I, _I, _I, _P, _P]),
    "dit_stack_workspace_bytes": (_SZ, [ctypes.POINTER(BlockConfig), _I, _I, _I, _I]),
    "dit_stack_forward": (_I, [ctypes.POINTER(BlockConfig), ctypes.POINTER(BlockWeights), _I, _P, _P, _I, _I, _I, _I,
                               _I, _P, _P, _SZ, _P]),
    "dit_denoise_workspace_bytes": (_SZ, [ctypes.POINTER(BlockConfig), _I, _I, _I, _I, _I]),
    "dit_denoise_steps": (_I, [ctypes.POINTER(BlockConfig), ctypes.POINTER(BlockWeights), ctypes.POINTER(BlockWeights),
                               _I, _P, _I, _P, _I, _P, _I, _I, _I, _I, ctypes.POINTER(ctypes.c_float),
                               ctypes.POINTER(ctypes.c_float), _P, _SZ, _P]),
    "dit_tokens_from_latent": (_I, [_P, _P, _P, _I, _I, _I, _I, _P]),
    "cond_proj_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "cond_proj_forward": (_I, [_P, _I, _I, _I, _P, _F, _P, _P, _I, _P, _P, _SZ, _P]),
    "euler_cfg_step": (_I, [_P, _P, _P, _I64, _F, _F, _P]),
    "dit_e4m3_to_bf16": (_I, [_P, _P, _I64, _P]),
    "dit_rmsnorm_rows": (_I, [_P, _I, _P, _P, _I, _I64, _I64, _F, _P]),
    "dit_mrope_positions": (_I, [_I, _I, _I, _I, _P, _P]),
    "dit_gemm_w8a16": (_I, [_P, _I, _P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _P]),
    "dit_qknorm_mrope": (_I, [_P, _I, _I, _I, _I, _I, _I, _P, ctypes.POINTER(BlockConfig), _P, _P, _P, _SZ, _P]),
    "dit_joint_attention": (_I, [_P, _P, _I, _I, _I, _I, _I, _P]),
    "dit_qknorm_mrope_e4m3": (_I, [_P, _I, _I, _I, _I, _I, _I, _P, ctypes.POINTER(BlockConfig), _P, _P, _P, _P, _P,
                                   _P]),
    "dit_joint_attention_e4m3": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "dit_poll_error": (_I, [_P]),
    "dit_profile_enable": (_I, [_I]),
    "dit_profile_enable_tags": (_I, [_I, ctypes.c_uint32]),
    "dit_profile_disable": (_I, []),
    "dit_profile_read": (_I, [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_float), _I]),
    "dit_set_wait_timeout_ms": (_I, [ctypes.c_uint32]),
    "dit_last_device_error": (ctypes.c_uint32, []),
    "dit_wait_selftest": (_I, [_P]),
    "dit_status_str": (ctypes.c_char_p, [_I]),
    "dit_last_cuda_error": (_I, []),
    "dit_abi_version": (_I, []),
}


def lib() -> ctypes.CDLL:
    """Load the CUDA library (once).  Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m joint_attention_block_b200.build` "
                "(there is no CPU fallback)"
            )
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def _stream(stream=None) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the C ABI must be contiguous")
    return t.data_ptr()


def _check(name: str, status: int) -> None:
    if status != DIT_OK:
        raise DitError(name, status)


def make_config(shape) -> BlockConfig:
    c = BlockConfig()
    c.d_model, c.n_heads, c.head_dim, c.d_mlp = shape.d_model, shape.n_heads, shape.head_dim, shape.d_mlp
    for i in range(3):
        c.rope_sections[i] = int(shape.rope_sections[i])
    c.rope_theta, c.eps, c.gelu_tanh = float(shape.rope_theta), float(shape.eps), int(shape.gelu_tanh)
    return c


def make_weights(w) -> BlockWeights:
    """``w``: dict of device tensors named like the struct fields.

    The struct holds raw device addresses, so it also keeps a reference to every tensor it
    points into: the weights stay allocated for as long as the returned struct is alive, even
    when the caller's dict was a temporary.  Keep the struct alive until the kernels that read
    the weights have been queued (torch's caching allocator reuses freed memory in stream
    order, so work on the tensors' own stream is safe once the call has returned)."""
    bw = BlockWeights()
    keep = {}
    for name, _ in BlockWeights._fields_:
        t = w[name]
        setattr(bw, name, _ptr(t))
        keep[name] = t
    bw._keep = keep
    return bw


# ---------------------------------------------------------------- the three calls


def block_workspace_bytes(cfg: BlockConfig, batch: int, n_text: int, grid_h: int, grid_w: int) -> int:
    return int(lib().dit_block_workspace_bytes(ctypes.byref(cfg), batch, n_text, grid_h, grid_w))


def dit_block_forward(cfg: BlockConfig, weights: BlockWeights, x: torch.Tensor, out: torch.Tensor, n_text: int,
                      grid_h: int, grid_w: int, workspace: torch.Tensor, t_img: int = -1,
                      pos: Optional[torch.Tensor] = None, stream=None) -> None:
    _check("dit_block_forward", lib().dit_block_forward(
        ctypes.byref(cfg), ctypes.byref(weights), _ptr(x), _ptr(out), x.shape[0], n_text, grid_h, grid_w, t_img,
        _ptr(pos), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def dit_block_forward_padded(cfg: BlockConfig, weights: BlockWeights, x: torch.Tensor, out: torch.Tensor,
                             n_text: int, grid_h: int, grid_w: int, text_lens: torch.Tensor, workspace: torch.Tensor,
                             t_img: int = -1, stream=None) -> None:
    """Padded batch of prompts: element b has text_lens[b] text rows, then its image rows, then
    padding (``text_lens``: int32 device tensor [batch])."""
    if text_lens.dtype != torch.int32 or text_lens.numel() != x.shape[0]:
        raise ValueError("text_lens must be an int32 tensor with one entry per batch element")
    _check("dit_block_forward_padded", lib().dit_block_forward_padded(
        ctypes.byref(cfg), ctypes.byref(weights), _ptr(x), _ptr(out), x.shape[0], n_text, grid_h, grid_w, t_img,
        _ptr(text_lens), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def dit_block_forward_w8a8(cfg: BlockConfig, weights: BlockWeights, x: torch.Tensor, out: torch.Tensor, n_text: int,
                           grid_h: int, grid_w: int, workspace: torch.Tensor, t_img: int = -1,
                           pos: Optional[torch.Tensor] = None, stream=None) -> None:
    """The W8A8 variant: e4m3 per-token activations into the QKV and MLP-up projections."""
    _check("dit_block_forward_w8a8", lib().dit_block_forward_w8a8(
        ctypes.byref(cfg), ctypes.byref(weights), _ptr(x), _ptr(out), x.shape[0], n_text, grid_h, grid_w, t_img,
        _ptr(pos), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def gemm_w8a8(a8: torch.Tensor, sa: torch.Tensor, w8: torch.Tensor, sw: torch.Tensor, y: torch.Tensor, act: int = 0,
              gelu_tanh: int = 0, y_fmt: int = FMT_BF16, stream=None) -> None:
    M, K = a8.shape
    N = w8.shape[0]
    _check("dit_gemm_w8a8", lib().dit_gemm_w8a8(_ptr(a8), _ptr(sa), _ptr(w8), _ptr(sw), _ptr(y), y_fmt, M, N, K, act,
                                                gelu_tanh, _stream(stream)))


def rmsnorm_rows_e4m3(x: torch.Tensor, g: torch.Tensor, y8: torch.Tensor, y_scale: torch.Tensor, eps: float,
                      x_fmt: int = FMT_BF16, stream=None) -> None:
    cols = x.shape[-1]
    _check("dit_rmsnorm_rows_e4m3", lib().dit_rmsnorm_rows_e4m3(_ptr(x), x_fmt, _ptr(g), _ptr(y8), _ptr(y_scale),
                                                                x.numel() // cols, cols, eps, _stream(stream)))


def stack_workspace_bytes(cfg: BlockConfig, batch: int, n_text: int, grid_h: int, grid_w: int) -> int:
    return int(lib().dit_stack_workspace_bytes(ctypes.byref(cfg), batch, n_text, grid_h, grid_w))


def dit_stack_forward(cfg: BlockConfig, weights, x: torch.Tensor, out: torch.Tensor, n_text: int, grid_h: int,
                      grid_w: int, workspace: torch.Tensor, t_img: int = -1, pos: Optional[torch.Tensor] = None,
                      stream=None) -> None:
    """``weights``: sequence of BlockWeights, one per block, applied in order."""
    arr = (BlockWeights * len(weights))(*weights)
    _check("dit_stack_forward", lib().dit_stack_forward(
        ctypes.byref(cfg), arr, len(weights), _ptr(x), _ptr(out), x.shape[0], n_text, grid_h, grid_w, t_img,
        _ptr(pos), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def denoise_workspace_bytes(cfg: BlockConfig, batch: int, n_text_c: int, n_text_u: int, grid_h: int,
                            grid_w: int) -> int:
    return int(lib().dit_denoise_workspace_bytes(ctypes.byref(cfg), batch, n_text_c, n_text_u, grid_h, grid_w))


def dit_denoise_steps(cfg: BlockConfig, w_cond, w_uncond, text_cond: Optional[torch.Tensor],
                      text_uncond: Optional[torch.Tensor], z: torch.Tensor, grid_h: int, grid_w: int, guidance,
                      dt, workspace: torch.Tensor, stream=None) -> None:
    """len(guidance) denoising steps: ``w_cond``/``w_uncond`` are equal-length sequences of
    BlockWeights; text tensors are bf16 [batch, L, d] (or None for L = 0); z fp32 [batch, gh*gw, d]
    is updated in place; ``guidance`` and ``dt`` hold one value per step."""
    if len(w_cond) != len(w_uncond) or len(guidance) != len(dt):
        raise ValueError("w_cond/w_uncond and guidance/dt must have equal lengths")
    n = len(w_cond)
    wc = (BlockWeights * n)(*w_cond)
    wu = (BlockWeights * n)(*w_uncond)
    g = (ctypes.c_float * max(1, len(guidance)))(*[float(v) for v in guidance])
    t = (ctypes.c_float * max(1, len(dt)))(*[float(v) for v in dt])
    lc = 0 if text_cond is None else text_cond.shape[1]
    lu = 0 if text_uncond is None else text_uncond.shape[1]
    _check("dit_denoise_steps", lib().dit_denoise_steps(
        ctypes.byref(cfg), wc, wu, n, _ptr(text_cond), lc, _ptr(text_uncond), lu, _ptr(z), z.shape[0], grid_h,
        grid_w, len(guidance), g, t, _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def tokens_from_latent(z: torch.Tensor, text: Optional[torch.Tensor], x: torch.Tensor, stream=None) -> None:
    """x[b] = [text[b]; bf16(z[b])]: z fp32 [B, n_img, d], text bf16 [B, L, d] or None, x bf16 [B, L + n_img, d]."""
    n_text = 0 if text is None else text.shape[1]
    _check("dit_tokens_from_latent", lib().dit_tokens_from_latent(
        _ptr(z), _ptr(text), _ptr(x), z.shape[0], n_text, z.shape[1], z.shape[2], _stream(stream)))


NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024  # DIT_NOALLOC_SCRATCH_BYTES


def dit_block_forward_noalloc(cfg: BlockConfig, weights: BlockWeights, x: torch.Tensor, out: torch.Tensor,
                              n_text: int, grid_h: int, grid_w: int, t_img: int = -1,
                              pos: Optional[torch.Tensor] = None, stream=None) -> None:
    """dit_block_forward without a workspace: the library's fixed device scratch is used instead."""
    _check("dit_block_forward_noalloc", lib().dit_block_forward_noalloc(
        ctypes.byref(cfg), ctypes.byref(weights), _ptr(x), _ptr(out), x.shape[0], n_text, grid_h, grid_w, t_img,
        _ptr(pos), _stream(stream)))


def cond_proj_workspace_bytes(n_tok: int, n_layers: int, hidden: int, d_out: int) -> int:
    return int(lib().cond_proj_workspace_bytes(n_tok, n_layers, hidden, d_out))


def cond_proj_forward(feats: torch.Tensor, n_layers: int, hidden: int, g: torch.Tensor, eps: float, w: torch.Tensor,
                      scale: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    _check("cond_proj_forward", lib().cond_proj_forward(
        _ptr(feats), feats.shape[0], n_layers, hidden, _ptr(g), eps, _ptr(w), _ptr(scale), out.shape[1], _ptr(out),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def euler_cfg_step(x: torch.Tensor, v_cond: torch.Tensor, v_uncond: torch.Tensor, guidance: float, dt: float,
                   stream=None) -> None:
    _check("euler_cfg_step", lib().euler_cfg_step(_ptr(x), _ptr(v_cond), _ptr(v_uncond), x.numel(), guidance, dt,
                                                  _stream(stream)))


# ---------------------------------------------------------------- per-step kernels


def e4m3_to_bf16(codes: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    _check("dit_e4m3_to_bf16", lib().dit_e4m3_to_bf16(_ptr(codes), _ptr(out), codes.numel(), _stream(stream)))


def rmsnorm_rows(x: torch.Tensor, g: torch.Tensor, y: torch.Tensor, eps: float, x_fmt: int = FMT_BF16,
                 y_fmt: int = FMT_BF16, stream=None) -> None:
    cols = x.shape[-1]
    _check("dit_rmsnorm_rows", lib().dit_rmsnorm_rows(_ptr(x), x_fmt, _ptr(g), _ptr(y), y_fmt, x.numel() // cols, cols,
                                                      eps, _stream(stream)))


def mrope_positions(n_text: int, grid_h: int, grid_w: int, t_img: int, out: torch.Tensor, stream=None) -> None:
    _check("dit_mrope_positions", lib().dit_mrope_positions(n_text, grid_h, grid_w, t_img, _ptr(out),
                                                            _stream(stream)))


def gemm_w8a16(a: torch.Tensor, w8: torch.Tensor, scale: torch.Tensor, y: torch.Tensor,
               residual: Optional[torch.Tensor] = None, act: int = 0, gelu_tanh: int = 0, a_fmt: int = FMT_BF16,
               y_fmt: int = FMT_BF16, res_fmt: int = FMT_BF16, stream=None) -> None:
    M, K = a.shape
    N = w8.shape[0]
    _check("dit_gemm_w8a16", lib().dit_gemm_w8a16(_ptr(a), a_fmt, _ptr(w8), _ptr(scale), _ptr(y), y_fmt,
                                                  _ptr(residual), res_fmt, M, N, K, act, gelu_tanh, _stream(stream)))


def qknorm_mrope(qkv: torch.Tensor, cfg: BlockConfig, n_text: int, grid_h: int, grid_w: int, g_q: torch.Tensor,
                 g_k: torch.Tensor, workspace: torch.Tensor, t_img: int = -1, pos: Optional[torch.Tensor] = None,
                 fmt: int = FMT_BF16, stream=None) -> None:
    _check("dit_qknorm_mrope", lib().dit_qknorm_mrope(
        _ptr(qkv), fmt, qkv.shape[0], n_text, grid_h, grid_w, t_img, _ptr(pos), ctypes.byref(cfg), _ptr(g_q),
        _ptr(g_k), _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def joint_attention(qkv: torch.Tensor, out: torch.Tensor, n_heads: int, head_dim: int, fmt: int = FMT_BF16,
                    stream=None) -> None:
    _check("dit_joint_attention", lib().dit_joint_attention(_ptr(qkv), _ptr(out), fmt, qkv.shape[0], qkv.shape[1],
                                                            n_heads, head_dim, _stream(stream)))


def qknorm_mrope_e4m3(qkv: torch.Tensor, cfg: BlockConfig, n_text: int, grid_h: int, grid_w: int, g_q: torch.Tensor,
                      g_k: torch.Tensor, q8: torch.Tensor, k8: torch.Tensor, scale: torch.Tensor, t_img: int = -1,
                      pos: Optional[torch.Tensor] = None, fmt: int = FMT_BF16, stream=None) -> None:
    _check("dit_qknorm_mrope_e4m3", lib().dit_qknorm_mrope_e4m3(
        _ptr(qkv), fmt, qkv.shape[0], n_text, grid_h, grid_w, t_img, _ptr(pos), ctypes.byref(cfg), _ptr(g_q),
        _ptr(g_k), _ptr(q8), _ptr(k8), _ptr(scale), _stream(stream)))


def joint_attention_e4m3(q8: torch.Tensor, k8: torch.Tensor, scale: torch.Tensor, qkv: torch.Tensor, out: torch.Tensor,
                         n_heads: int, head_dim: int, fmt: int = FMT_BF16, stream=None) -> None:
    _check("dit_joint_attention_e4m3", lib().dit_joint_attention_e4m3(
        _ptr(q8), _ptr(k8), _ptr(scale), _ptr(qkv), _ptr(out), fmt, qkv.shape[0], qkv.shape[1], n_heads, head_dim,
        _stream(stream)))


KERNEL_TAGS = {1: "rope_table", 2: "rmsnorm", 3: "gemm_qkv", 4: "qknorm_mrope", 5: "attention", 6: "gemm_o",
               7: "gemm_up", 8: "gemm_down", 9: "cond_rmsnorm", 10: "cond_gemm", 11: "euler_cfg",
               12: "cond_reduce"}


def profile_enable(max_marks: int, kernels=None) -> None:
    """Bracket every launch (``kernels`` None) or only the launches of the named kernels
    (names as in KERNEL_TAGS) with CUDA events."""
    if kernels is None:
        _check("dit_profile_enable", lib().dit_profile_enable(max_marks))
        return
    ids = {v: k for k, v in KERNEL_TAGS.items()}
    mask = 0
    for name in kernels:
        mask |= 1 << ids[name]
    _check("dit_profile_enable_tags", lib().dit_profile_enable_tags(max_marks, mask))


def profile_disable() -> None:
    lib().dit_profile_disable()


def profile_read(max_records: int = 1 << 16):
    """[(kernel name, ms), ...] of every launch recorded since profile_enable / the last read."""
    tags = (ctypes.c_int * max_records)()
    ms = (ctypes.c_float * max_records)()
    n = lib().dit_profile_read(tags, ms, max_records)
    if n < 0:
        raise DitError("dit_profile_read", -n)
    return [(KERNEL_TAGS.get(tags[i], str(tags[i])), float(ms[i])) for i in range(n)]


def poll_error(stream=None) -> int:
    return int(lib().dit_poll_error(_stream(stream)))


def wait_selftest(stream=None) -> None:
    _check("dit_wait_selftest", lib().dit_wait_selftest(_stream(stream)))


def last_device_error() -> int:
    return int(lib().dit_last_device_error())


def set_wait_timeout_ms(ms: int) -> None:
    _check("dit_set_wait_timeout_ms", lib().dit_set_wait_timeout_ms(ms))
