"""Host-side reader for the Ideogram 4 FP8 checkpoint layout: safetensors shards whose
quantised weights are e4m3 bytes with a per-output-channel ``weight_scale`` (unsloth
diffusion_ideogram4.py commit log, fp8 loader commit and its review follow-ups).

What those commits fix, and what this module does with each fact:

- The fp8 layout is recognised from the shard HEADERS alone, by a key ending in
  ``.weight_scale``; every shard's header is scanned, not only the first, and no tensor
  data is read to decide it (``ShardIndex.fp8_layout``).
- Attention is stored fused: ``attention.qkv.weight`` of shape [3*hidden, hidden] with the
  Q, K and V rows stacked in that order, next to ``attention.o.weight``.  The row count of
  the fused weight is checked against 3*hidden, so a grouped-query export (fewer K/V rows)
  fails loudly instead of being split at the wrong rows.
- The real weight is ``fp8 * weight_scale[:, None]``: the scale indexes the output row.  A
  scale stored as [out] or [out, 1] is accepted (the scale broadcasts by rank, not by
  assuming a shape); anything else raises.
- Every key of a block that no field takes, and every field that no key supplies, raises:
  a partly loaded block never reaches the kernels.

What differs from the diffusers loader those commits describe: the block's GEMMs consume
the e4m3 bytes and the fp32 scale exactly as stored (the e4m3 -> f16 widening is exact and
the scale is applied in the GEMM epilogue), so this loader moves bytes and does not
dequantise, and it keeps the fused QKV weight fused (the fused QKV GEMM reads it as one
[3d, d] operand) instead of splitting it into to_q / to_k / to_v.  Gains not stored as
bf16 are cast to bf16 with round-to-nearest-even, as the diffusers loader casts the whole
model to its bf16 resident dtype at the end.

Key names the pages do not give (the two pre-norm gains, the QK-norm gains, the
FeedForward projections and the per-block prefix) are parameters; the defaults below are
this module's own.

The safetensors container: 8 bytes little-endian header length N, N bytes of JSON mapping
each key to ``{"dtype", "shape", "data_offsets": [begin, end]}`` (offsets relative to the
first byte after the header) plus an optional ``__metadata__`` object of strings.
"""
from __future__ import annotations

import dataclasses
import json
import os
import struct
from typing import Dict, Iterable, List, Mapping, Optional, Sequence, Tuple

import numpy as np
import torch

# Item size of each safetensors dtype string.
DTYPE_BYTES = {
    "BOOL": 1, "U8": 1, "I8": 1, "F8_E4M3": 1, "F8_E5M2": 1,
    "U16": 2, "I16": 2, "F16": 2, "BF16": 2,
    "U32": 4, "I32": 4, "F32": 4,
    "U64": 8, "I64": 8, "F64": 8,
}

# Block fields (the names of the C-ABI weight struct) -> key suffix within one block.  The
# two attention projections and their scales are the checkpoint's own names; the rest are
# this module's defaults for names the pages do not print.
DEFAULT_NAMES: Dict[str, str] = {
    "w_qkv": "attention.qkv.weight",
    "s_qkv": "attention.qkv.weight_scale",
    "w_o": "attention.o.weight",
    "s_o": "attention.o.weight_scale",
    "w_up": "feed_forward.up.weight",
    "s_up": "feed_forward.up.weight_scale",
    "w_down": "feed_forward.down.weight",
    "s_down": "feed_forward.down.weight_scale",
    "g_norm1": "attention_norm.weight",
    "g_norm2": "ffn_norm.weight",
    "g_q": "attention.norm_q.weight",
    "g_k": "attention.norm_k.weight",
}
DEFAULT_BLOCK_PREFIX = "layers.{i}."
_WEIGHTS = ("w_qkv", "w_o", "w_up", "w_down")
_GAINS = ("g_norm1", "g_norm2", "g_q", "g_k")
# Largest header this reader accepts (the format's own readers cap it at 100 MB).
MAX_HEADER_BYTES = 100 * 1024 * 1024


class CheckpointError(ValueError):
    """The shards do not hold a block in the FP8 layout the kernels consume."""


@dataclasses.dataclass(frozen=True)
class TensorEntry:
    """One tensor of one shard: absolute byte range [begin, end) in ``path``."""

    key: str
    path: str
    dtype: str
    shape: Tuple[int, ...]
    begin: int
    end: int

    @property
    def nbytes(self) -> int:
        return self.end - self.begin


def read_header(path: str) -> Tuple[Dict[str, TensorEntry], Dict[str, str]]:
    """Parse one shard's header (no tensor data is read) and check every entry's byte range
    against its dtype, its shape and the file's length."""
    size = os.path.getsize(path)
    with open(path, "rb") as f:
        head = f.read(8)
        if len(head) != 8:
            raise CheckpointError(f"{path}: shorter than the 8-byte header length")
        (n,) = struct.unpack("<Q", head)
        if n > MAX_HEADER_BYTES or 8 + n > size:
            raise CheckpointError(f"{path}: header length {n} does not fit the file ({size} bytes)")
        raw = f.read(n)
    try:
        hdr = json.loads(raw.decode("utf-8"))
    except (UnicodeDecodeError, json.JSONDecodeError) as e:
        raise CheckpointError(f"{path}: header is not JSON ({e})") from None
    if not isinstance(hdr, dict):
        raise CheckpointError(f"{path}: header is not a JSON object")
    meta = hdr.pop("__metadata__", None) or {}
    base = 8 + n
    entries: Dict[str, TensorEntry] = {}
    for key, e in hdr.items():
        try:
            dtype, shape, (b, t) = e["dtype"], tuple(int(s) for s in e["shape"]), e["data_offsets"]
        except (KeyError, TypeError, ValueError):
            raise CheckpointError(f"{path}: entry {key!r} lacks dtype / shape / data_offsets") from None
        if dtype not in DTYPE_BYTES:
            raise CheckpointError(f"{path}: entry {key!r} has unknown dtype {dtype!r}")
        if any(s < 0 for s in shape):
            raise CheckpointError(f"{path}: entry {key!r} has a negative dimension {shape}")
        want = int(np.prod(shape, dtype=np.int64)) * DTYPE_BYTES[dtype]
        if not (0 <= b <= t) or t - b != want or base + t > size:
            raise CheckpointError(
                f"{path}: entry {key!r} spans [{b}, {t}) but {dtype}{list(shape)} needs {want} bytes "
                f"inside a {size - base}-byte data section")
        entries[key] = TensorEntry(key, path, dtype, shape, base + b, base + t)
    return entries, {str(k): str(v) for k, v in meta.items()}


class ShardIndex:
    """The keys of every shard of one checkpoint, by name.  A key present in two shards
    raises: which copy would be loaded is not defined by the layout."""

    def __init__(self, paths: Sequence[str]):
        if not paths:
            raise CheckpointError("no shard paths given")
        self.paths = [os.fspath(p) for p in paths]
        self.entries: Dict[str, TensorEntry] = {}
        self.metadata: Dict[str, Dict[str, str]] = {}
        for p in self.paths:
            ents, meta = read_header(p)
            self.metadata[p] = meta
            for k, e in ents.items():
                if k in self.entries:
                    raise CheckpointError(f"key {k!r} is in both {self.entries[k].path} and {p}")
                self.entries[k] = e

    def fp8_layout(self) -> bool:
        """True when any shard's header holds a ``*.weight_scale`` key (the fp8 marker)."""
        return any(k.endswith(".weight_scale") for k in self.entries)

    def keys(self) -> List[str]:
        return sorted(self.entries)

    def entry(self, key: str) -> TensorEntry:
        try:
            return self.entries[key]
        except KeyError:
            raise CheckpointError(f"key {key!r} is in no shard") from None

    def read_bytes(self, key: str) -> np.ndarray:
        """The tensor's raw bytes (uint8, C order), read from its shard."""
        e = self.entry(key)
        with open(e.path, "rb") as f:
            f.seek(e.begin)
            buf = bytearray(e.nbytes)
            if f.readinto(buf) != e.nbytes:
                raise CheckpointError(f"{e.path}: short read of {key!r}")
        return np.frombuffer(buf, dtype=np.uint8)

    def count_blocks(self, prefix: str = DEFAULT_BLOCK_PREFIX) -> int:
        """Number of consecutive blocks 0, 1, ... that have at least one key under ``prefix``."""
        n = 0
        keys = self.keys()
        while any(k.startswith(prefix.format(i=n)) for k in keys):
            n += 1
        return n


@dataclasses.dataclass(frozen=True)
class BlockDims:
    """Sizes read from one block's shapes: d_model from attention.o, d_mlp from the up
    projection, head_dim from the QK-norm gain (one gain of head_dim shared by all heads)."""

    d_model: int
    n_heads: int
    head_dim: int
    d_mlp: int


def infer_block_dims(index: ShardIndex, block: int = 0, prefix: str = DEFAULT_BLOCK_PREFIX,
                     names: Mapping[str, str] = DEFAULT_NAMES) -> BlockDims:
    p = prefix.format(i=block)
    o = index.entry(p + names["w_o"]).shape
    up = index.entry(p + names["w_up"]).shape
    gq = index.entry(p + names["g_q"]).shape
    if len(o) != 2 or o[0] != o[1]:
        raise CheckpointError(f"{p + names['w_o']}: shape {o}, expected [hidden, hidden]")
    if len(up) != 2 or up[1] != o[0]:
        raise CheckpointError(f"{p + names['w_up']}: shape {up}, expected [d_mlp, {o[0]}]")
    if len(gq) != 1 or gq[0] <= 0 or o[0] % gq[0]:
        raise CheckpointError(f"{p + names['g_q']}: shape {gq} does not divide hidden {o[0]}")
    return BlockDims(o[0], o[0] // gq[0], gq[0], up[0])


def _expected_shapes(dims: BlockDims) -> Dict[str, Tuple[int, ...]]:
    d, f, hd = dims.d_model, dims.d_mlp, dims.head_dim
    return {"w_qkv": (3 * d, d), "w_o": (d, d), "w_up": (f, d), "w_down": (d, f),
            "g_norm1": (d,), "g_norm2": (d,), "g_q": (hd,), "g_k": (hd,)}


def _scale_f32(index: ShardIndex, key: str, rows: int) -> np.ndarray:
    e = index.entry(key)
    if e.shape not in ((rows,), (rows, 1)):
        raise CheckpointError(f"{key}: shape {list(e.shape)}, expected [{rows}] or [{rows}, 1] (one scale per output row)")
    raw = index.read_bytes(key)
    if e.dtype == "F32":
        s = raw.view(np.float32)
    elif e.dtype in ("BF16", "F16"):
        t = torch.from_numpy(raw.copy()).view(torch.bfloat16 if e.dtype == "BF16" else torch.float16)
        s = t.to(torch.float32).numpy()  # exact: every bf16 / f16 value is an fp32 value
    else:
        raise CheckpointError(f"{key}: scale dtype {e.dtype}, expected F32, BF16 or F16")
    s = np.ascontiguousarray(s.reshape(rows), dtype=np.float32)
    if not np.all(np.isfinite(s)):
        raise CheckpointError(f"{key}: non-finite scale")
    return s


def _gain_bf16_bits(index: ShardIndex, key: str, n: int) -> np.ndarray:
    e = index.entry(key)
    if e.shape != (n,):
        raise CheckpointError(f"{key}: shape {list(e.shape)}, expected [{n}]")
    raw = index.read_bytes(key)
    if e.dtype == "BF16":
        return raw.view(np.uint16).copy()
    if e.dtype in ("F32", "F16"):
        t = torch.from_numpy(raw.copy()).view(torch.float32 if e.dtype == "F32" else torch.float16)
        return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()
    raise CheckpointError(f"{key}: gain dtype {e.dtype}, expected BF16, F16 or F32")


def _e4m3_codes(index: ShardIndex, key: str, shape: Tuple[int, int]) -> np.ndarray:
    e = index.entry(key)
    if e.dtype != "F8_E4M3":
        raise CheckpointError(f"{key}: dtype {e.dtype}; the block's GEMMs take e4m3 weights with a weight_scale")
    if e.shape != shape:
        if key.endswith("qkv.weight") and len(e.shape) == 2 and e.shape[1] == shape[1]:
            raise CheckpointError(
                f"{key}: {e.shape[0]} rows, expected 3 x hidden = {shape[0]} (Q, K, V stacked); "
                "a grouped-query export is not this layout")
        raise CheckpointError(f"{key}: shape {list(e.shape)}, expected {list(shape)}")
    codes = index.read_bytes(key).reshape(shape)
    # 0x7F and 0xFF are e4m3's only NaN codes (the format has no infinities).
    if np.any((codes & 0x7F) == 0x7F):
        raise CheckpointError(f"{key}: holds e4m3 NaN codes")
    return codes


def read_block(index: ShardIndex, block: int, dims: Optional[BlockDims] = None,
               prefix: str = DEFAULT_BLOCK_PREFIX, names: Mapping[str, str] = DEFAULT_NAMES) -> Dict[str, np.ndarray]:
    """One block's host arrays named like the C-ABI weight struct: e4m3 codes uint8 [out, in],
    fp32 scales [out], bf16 gains as uint16 bit patterns.  Raises ``CheckpointError`` when the
    layout is not fp8, a field's key is missing, or a shape or dtype does not match."""
    if not index.fp8_layout():
        raise CheckpointError("no *.weight_scale key in any shard header: not the fp8 layout")
    dims = dims or infer_block_dims(index, block, prefix, names)
    shapes = _expected_shapes(dims)
    p = prefix.format(i=block)
    out: Dict[str, np.ndarray] = {}
    for w in _WEIGHTS:
        out[w] = _e4m3_codes(index, p + names[w], shapes[w])
        out["s" + w[1:]] = _scale_f32(index, p + names["s" + w[1:]], shapes[w][0])
    for g in _GAINS:
        out[g] = _gain_bf16_bits(index, p + names[g], shapes[g][0])
    return out


def block_keys(block: int, prefix: str = DEFAULT_BLOCK_PREFIX, names: Mapping[str, str] = DEFAULT_NAMES) -> List[str]:
    p = prefix.format(i=block)
    return [p + names[f] for f in DEFAULT_NAMES]


@dataclasses.dataclass
class LoadedStack:
    """The blocks of one checkpoint on a device, in block order, plus the keys outside every
    block that the caller allowed to stay unread."""

    dims: BlockDims
    blocks: List[Dict[str, torch.Tensor]]
    unclaimed: List[str]


def _to_device(a: np.ndarray, device) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a))
    if t.dtype == torch.uint16:
        t = t.view(torch.int16)
    dev = torch.device(device)
    if dev.type == "cuda":
        return t.pin_memory().to(dev, non_blocking=True)
    return t.clone()


def load_stack(paths: Sequence[str], device="cuda", n_blocks: Optional[int] = None,
               prefix: str = DEFAULT_BLOCK_PREFIX, names: Mapping[str, str] = DEFAULT_NAMES,
               allow_unclaimed: Iterable[str] = ()) -> LoadedStack:
    """Every block of a checkpoint onto ``device`` in the layout ``ops.make_weights`` takes.

    Every key under a block's prefix must be one of that block's fields, and every key outside
    the blocks must start with one of ``allow_unclaimed`` (the prefixes of modules this hot path
    does not run, such as embedders); any other key raises, so nothing in the shards is silently
    dropped.  All blocks must have the first block's sizes."""
    index = ShardIndex(paths)
    if not index.fp8_layout():
        raise CheckpointError("no *.weight_scale key in any shard header: not the fp8 layout")
    nb = index.count_blocks(prefix) if n_blocks is None else int(n_blocks)
    if nb <= 0:
        raise CheckpointError(f"no key starts with {prefix.format(i=0)!r}")
    dims = infer_block_dims(index, 0, prefix, names)
    claimed = set()
    blocks = []
    for i in range(nb):
        arrays = read_block(index, i, dims, prefix, names)
        blocks.append({k: _to_device(v, device) for k, v in arrays.items()})
        claimed.update(block_keys(i, prefix, names))
    allow = tuple(allow_unclaimed)
    unclaimed, bad = [], []
    block_prefixes = [prefix.format(i=i) for i in range(nb)]
    for k in index.keys():
        if k in claimed:
            continue
        in_block = any(k.startswith(bp) for bp in block_prefixes)
        if in_block or not (allow and k.startswith(allow)):
            bad.append(k)
        else:
            unclaimed.append(k)
    if bad:
        more = f" (+{len(bad) - 8} more)" if len(bad) > 8 else ""
        raise CheckpointError("unmatched keys: " + ", ".join(bad[:8]) + more)
    if torch.device(device).type == "cuda":
        torch.cuda.current_stream(torch.device(device)).synchronize()
    return LoadedStack(dims, blocks, unclaimed)
