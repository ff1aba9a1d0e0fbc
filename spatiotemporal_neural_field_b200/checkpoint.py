"""Checkpoint and resume of a decoder's training state (host side, outside
the hot path).

SPIN-4DGS stores a trained scene as its Gaussians' positions plus the
network (section 4, Table 1 reports the storage).  A checkpoint here holds
any named set of tensors -- the hash tables (fp16 working copy and fp32
master), the packed weights, Adam's m and v -- with the optimiser step and
free-form metadata (the grid and network descriptions, say).

File layout, little-endian throughout:

    bytes 0..7     magic  b"SPIN4DCK"
    bytes 8..15    uint64 length H of the JSON header
    bytes 16..     the JSON header (UTF-8), then zero padding to a multiple of 64
    then           each tensor's raw bytes, in header order, each starting on a
                   64-byte boundary

The header: {"version": 1, "step": int, "meta": {...}, "tensors": [{"name",
"dtype", "shape", "offset", "nbytes", "crc32"}, ...]}; offsets count from the
start of the file.  A save writes a temporary file and renames it over the
target, so a crash never leaves a half-written checkpoint under the name.
A load checks the magic, the version, every size and every CRC-32, and
raises ``CheckpointError`` on any mismatch.
"""
from __future__ import annotations

import json
import os
import struct
import zlib
from typing import Dict, Optional, Tuple

import numpy as np

MAGIC = b"SPIN4DCK"
VERSION = 1
ALIGN = 64
_DTYPES = {"float16": np.float16, "float32": np.float32, "float64": np.float64, "int32": np.int32,
           "int64": np.int64, "uint8": np.uint8, "uint32": np.uint32}


class CheckpointError(RuntimeError):
    pass


def _to_numpy(t) -> np.ndarray:
    """A tensor (torch, on any device) or array as a contiguous little-endian array."""
    if hasattr(t, "detach"):
        t = t.detach().cpu().numpy()
    a = np.ascontiguousarray(t)
    if a.dtype.name not in _DTYPES:
        raise CheckpointError("unsupported dtype %s" % a.dtype)
    return a.astype(a.dtype.newbyteorder("<"), copy=False)


def _pad(n: int) -> int:
    return (-n) % ALIGN


def save(path: str, tensors: Dict[str, object], step: int = 0, meta: Optional[dict] = None) -> None:
    """Writes ``tensors`` (name -> torch tensor or numpy array), the optimiser
    ``step`` and JSON-serialisable ``meta`` to ``path`` atomically."""
    arrays = [(name, _to_numpy(t)) for name, t in tensors.items()]
    entries = []
    for name, a in arrays:
        entries.append({"name": name, "dtype": a.dtype.name, "shape": list(a.shape), "nbytes": int(a.nbytes),
                        "crc32": zlib.crc32(a.tobytes()) & 0xFFFFFFFF, "offset": 0})
    # the header's length fixes the data offsets, which are part of the
    # header: lay it out again until its length stops changing
    header = b""
    for _ in range(8):
        start = 16 + len(header)
        off = start + _pad(start)
        for e in entries:
            e["offset"] = off
            off += e["nbytes"] + _pad(e["nbytes"])
        new = json.dumps({"version": VERSION, "step": int(step), "meta": meta or {}, "tensors": entries},
                         sort_keys=True).encode()
        if len(new) == len(header):
            header = new
            break
        header = new
    else:  # pragma: no cover - the length converges within a few passes
        raise CheckpointError("header layout did not converge")
    tmp = path + ".tmp"
    with open(tmp, "wb") as f:
        f.write(MAGIC)
        f.write(struct.pack("<Q", len(header)))
        f.write(header)
        f.write(b"\0" * _pad(16 + len(header)))
        for (name, a), e in zip(arrays, entries):
            assert f.tell() == e["offset"], (name, f.tell(), e["offset"])
            f.write(a.tobytes())
            f.write(b"\0" * _pad(e["nbytes"]))
        f.flush()
        os.fsync(f.fileno())
    os.replace(tmp, path)


def load(path: str, device=None) -> Tuple[Dict[str, object], int, dict]:
    """(tensors, step, meta) from ``path``.  Tensors come back as numpy
    arrays, or as torch tensors on ``device`` when one is given."""
    size = os.path.getsize(path)
    with open(path, "rb") as f:
        if f.read(8) != MAGIC:
            raise CheckpointError("%s: not a spin4d checkpoint" % path)
        (hlen,) = struct.unpack("<Q", f.read(8))
        if 16 + hlen > size:
            raise CheckpointError("%s: truncated header" % path)
        try:
            header = json.loads(f.read(hlen).decode())
        except (UnicodeDecodeError, json.JSONDecodeError) as e:
            raise CheckpointError("%s: unreadable header (%s)" % (path, e))
        if header.get("version") != VERSION:
            raise CheckpointError("%s: version %r, expected %d" % (path, header.get("version"), VERSION))
        out = {}
        for e in header["tensors"]:
            if e["dtype"] not in _DTYPES:
                raise CheckpointError("%s: tensor %s has unsupported dtype %s" % (path, e["name"], e["dtype"]))
            dt = np.dtype(_DTYPES[e["dtype"]]).newbyteorder("<")
            want = int(np.prod(e["shape"], dtype=np.int64)) * dt.itemsize
            if want != e["nbytes"] or e["offset"] + e["nbytes"] > size:
                raise CheckpointError("%s: tensor %s is truncated or mis-sized" % (path, e["name"]))
            f.seek(e["offset"])
            raw = f.read(e["nbytes"])
            if zlib.crc32(raw) & 0xFFFFFFFF != e["crc32"]:
                raise CheckpointError("%s: tensor %s fails its CRC-32" % (path, e["name"]))
            a = np.frombuffer(raw, dtype=dt).reshape(e["shape"]).astype(dt.newbyteorder("="))
            if device is not None:
                import torch
                a = torch.from_numpy(a.copy()).to(device)
            out[e["name"]] = a
    return out, int(header["step"]), header.get("meta", {})
