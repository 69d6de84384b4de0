"""Save and load NVFP4 tensors: packed E2M1 codes, E4M3 block scales and the
FP32 tensor scale, bit for bit.

Frozen-scale QAD carries exactly this state between the jobs of a training
run (the scales are calibrated once and held; Nemotron 3.5 Lightning NVFP4
article, "量化尺度处理策略"; the Qwen3.6-35B-A3B W4A4 tutorial's QAD saves
every 50 steps, section "3. QAD"), and the quantized checkpoint itself is
the pages' product (codes + block scales + tensor scale per tensor).

File layout (little-endian):
    8 bytes   magic b"NVFP4QAD"
    4 bytes   format version (1)
    8 bytes   length n of the JSON header
    n bytes   JSON: {"tensors": {name: {"codes": [off, rows, cols/2],
                     "block_scales": [off, nbytes], "layout": "rowmajor"|"mma",
                     "tensor_scale": [off], "cols": cols}}, "meta": {...}}
    payload   raw bytes of every array, each starting on a 64-byte boundary
Offsets are relative to the start of the payload.  Only host I/O happens
here; tensors are copied to the host to be written and to `device` when read.
"""
from __future__ import annotations

import json
import os
import struct

import torch

MAGIC = b"NVFP4QAD"
VERSION = 1
_ALIGN = 64


def _pad(n: int) -> int:
    return (n + _ALIGN - 1) // _ALIGN * _ALIGN


def save_nvfp4(path: str, tensors: dict, meta: dict | None = None) -> None:
    """tensors: name -> (codes uint8 [rows, cols/2], block_scales uint8 (row-major
    [rows, cols/16] or the MMA layout, flat), tensor_scale float32 [1], layout
    "rowmajor" or "mma").  Written atomically (temporary file, then rename)."""
    header = {"tensors": {}, "meta": meta or {}}
    blobs = []
    off = 0
    for name, (codes, sb, ts, layout) in tensors.items():
        if codes.dtype != torch.uint8 or codes.dim() != 2:
            raise ValueError(f"{name}: codes must be uint8 [rows, cols/2]")
        if sb.dtype != torch.uint8 or ts.dtype != torch.float32 or ts.numel() != 1:
            raise ValueError(f"{name}: block scales uint8, tensor scale one float32")
        if layout not in ("rowmajor", "mma"):
            raise ValueError(f"{name}: layout must be 'rowmajor' or 'mma'")
        c = codes.detach().contiguous().cpu()
        s = sb.detach().contiguous().cpu().reshape(-1)
        t = ts.detach().contiguous().cpu().reshape(-1)
        rows, half = c.shape
        if layout == "rowmajor" and s.numel() != rows * (2 * half // 16):
            raise ValueError(f"{name}: row-major block scales must hold rows * cols/16 bytes")
        entry = {"cols": 2 * half, "layout": layout}
        for key, arr in (("codes", c), ("block_scales", s), ("tensor_scale", t)):
            raw = arr.numpy().tobytes()
            blobs.append((off, raw))
            if key == "codes":
                entry[key] = [off, rows, half]
            elif key == "block_scales":
                entry[key] = [off, len(raw)]
            else:
                entry[key] = [off]
            off = _pad(off + len(raw))
        header["tensors"][name] = entry
    hdr = json.dumps(header, sort_keys=True).encode()
    tmp = f"{path}.tmp{os.getpid()}"
    with open(tmp, "wb") as f:
        f.write(MAGIC + struct.pack("<IQ", VERSION, len(hdr)) + hdr)
        base = f.tell()
        for o, raw in blobs:
            f.seek(base + o)
            f.write(raw)
        f.truncate(base + off)
    os.replace(tmp, path)


def load_nvfp4(path: str, device="cpu"):
    """Returns (tensors, meta): tensors[name] = (codes, block_scales, tensor_scale,
    layout) with the same bytes as were saved, on `device`."""
    with open(path, "rb") as f:
        data = f.read()
    if data[:8] != MAGIC:
        raise ValueError(f"{path}: not an NVFP4 checkpoint")
    version, n = struct.unpack("<IQ", data[8:20])
    if version != VERSION:
        raise ValueError(f"{path}: format version {version}, expected {VERSION}")
    header = json.loads(data[20:20 + n])
    base = 20 + n
    out = {}

    def view(o, nbytes, dtype):
        raw = bytearray(data[base + o: base + o + nbytes])
        if len(raw) != nbytes:
            raise ValueError(f"{path}: truncated")
        return torch.frombuffer(raw, dtype=dtype) if nbytes else torch.empty(0, dtype=dtype)

    for name, e in header["tensors"].items():
        o, rows, half = e["codes"]
        codes = view(o, rows * half, torch.uint8).reshape(rows, half)
        so, snb = e["block_scales"]
        sb = view(so, snb, torch.uint8)
        if e["layout"] == "rowmajor":
            sb = sb.reshape(rows, e["cols"] // 16)
        ts = view(e["tensor_scale"][0], 4, torch.float32)
        out[name] = (codes.to(device), sb.to(device), ts.to(device), e["layout"])
    return out, header["meta"]
