"""The packed weights of one W4.4A8 linear on disk.

The global channel bit map and the pre-packed weight layout are what a
deployment keeps, and the pages leave their versioning open (the
awesome-system-papers summary of MixLLM, §系统性缺陷, on operations).  So the
packed layout gets a plain little-endian file whose magic carries a layout
version: no pickling, nothing executed on load.

  8 bytes   magic b"MIXLLMW1"
  5 int64   N, K, N4, N8, group
  7 times   int64 byte count, then the buffer's bytes in the device layout,
            for W4, z4, s_w4, idx4, W8, s_w8, idx8 in that order

A reader checks every count against mixllm_packed_sizes for the stated
shape, so a truncated file or one written for another layout is refused
instead of misread.
"""
from __future__ import annotations

import struct
import sys

import numpy as np
import torch

from . import _lib

MAGIC = b"MIXLLMW1"
FIELDS = ("W4", "z4", "s_w4", "idx4", "W8", "s_w8", "idx8")

def _little_endian_host():
    # the buffers are written and read in host order
    if sys.byteorder != "little":
        raise RuntimeError("the packed-weight file format needs a little-endian host")


def save_packed(p: _lib.PackedLinear, path: str) -> None:
    """Write `p` (device or host tensors) to `path`."""
    _little_endian_host()
    with open(path, "wb") as f:
        f.write(MAGIC)
        f.write(struct.pack("<5q", p.N, p.K, p.N4, p.N8, _lib.GROUP))
        for name in FIELDS:
            t = getattr(p, name).detach().contiguous().cpu()
            raw = t.reshape(-1).view(torch.uint8).numpy().tobytes() if t.numel() else b""
            f.write(struct.pack("<q", len(raw)))
            f.write(raw)


def load_packed(path: str, device="cuda") -> _lib.PackedLinear:
    """Read a file written by save_packed into tensors on `device`."""
    _little_endian_host()
    with open(path, "rb") as f:
        if f.read(len(MAGIC)) != MAGIC:
            raise ValueError(f"{path}: not a packed W4.4A8 weight file")
        head = f.read(40)
        if len(head) != 40:
            raise ValueError(f"{path}: truncated header")
        N, K, N4, N8, group = struct.unpack("<5q", head)
        if group != _lib.GROUP or N4 < 0 or N8 < 0 or N4 + N8 != N or K <= 0 or K % _lib.GROUP:
            raise ValueError(f"{path}: bad shape N={N} K={K} N4={N4} N8={N8} group={group}")
        p = _lib.empty_packed(N, K, N8, "cpu")
        sizes = _lib.packed_sizes(N, K, N8)
        for name, size in zip(FIELDS, sizes):
            t = getattr(p, name)
            count = f.read(8)
            if len(count) != 8:
                raise ValueError(f"{path}: truncated before {name}")
            (n,) = struct.unpack("<q", count)
            if n != size or n != t.numel() * t.element_size():
                raise ValueError(f"{path}: {name} holds {n} bytes, the layout has {size}")
            raw = f.read(n)
            if len(raw) != n:
                raise ValueError(f"{path}: truncated in {name}")
            if n:
                t.reshape(-1).view(torch.uint8).copy_(torch.from_numpy(np.frombuffer(raw, dtype=np.uint8).copy()))
        if f.read(1):
            raise ValueError(f"{path}: trailing bytes after idx8")
    if torch.device(device).type == "cpu":
        return p
    return _lib.PackedLinear(p.N, p.K, p.N4, p.N8, *(getattr(p, name).to(device) for name in FIELDS))
