"""Storage of quantized weights: the Per-group(128) article's format (sec. 3.3, "storage
format"), one safetensors file holding, for every quantized tensor ``name``:

    name_packed   uint8  (N, K*b/8)   the packed codes (MSB-first bitstream per row)
    name_scales   float32 (N, K/128)  one step per 128-weight group
    name_bw       int8   ()           the bit width b
    name_nin      int32  ()           the input dimension K (padded to a multiple of 128)

Plain host-side file I/O (safetensors: an 8-byte little-endian header length, a JSON header
naming each tensor's dtype, shape and byte range, then the bytes); no computation. ``save``
takes the outputs of wq_quantize_pack (CUDA tensors or numpy arrays); ``load`` returns numpy
arrays, or CUDA tensors with ``device=``, ready for wq_linear / wq_dequantize.
"""
from __future__ import annotations

import json
import struct

import numpy as np

_DTYPES = {"U8": np.uint8, "F32": np.float32, "I8": np.int8, "I32": np.int32}
_NAMES = {np.dtype(v): k for k, v in _DTYPES.items()}


def _host(a):
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a)


def save(path: str, tensors: dict, metadata: dict | None = None) -> None:
    """tensors: name -> (packed, scales, bits) or (packed, scales, bits, nin)."""
    arrays = {}
    for name, entry in tensors.items():
        packed, scales, bits = entry[:3]
        packed, scales = _host(packed).astype(np.uint8, copy=False), _host(scales).astype(np.float32, copy=False)
        nin = int(entry[3]) if len(entry) > 3 else int(packed.shape[1] * 8 // int(bits))
        if packed.ndim != 2 or scales.ndim != 2 or packed.shape[0] != scales.shape[0]:
            raise ValueError(f"{name}: packed (N, K*b/8) and scales (N, K/128) expected")
        if nin % 128 or packed.shape[1] * 8 != nin * int(bits) or scales.shape[1] != nin // 128:
            raise ValueError(f"{name}: sizes disagree with bits={bits}, nin={nin}")
        arrays[f"{name}_packed"] = packed
        arrays[f"{name}_scales"] = scales
        arrays[f"{name}_bw"] = np.array(int(bits), np.int8)
        arrays[f"{name}_nin"] = np.array(nin, np.int32)
    header, offset = {}, 0
    for key, a in arrays.items():
        header[key] = {"dtype": _NAMES[a.dtype], "shape": list(a.shape), "data_offsets": [offset, offset + a.nbytes]}
        offset += a.nbytes
    if metadata:
        header["__metadata__"] = {str(k): str(v) for k, v in metadata.items()}
    blob = json.dumps(header, separators=(",", ":")).encode()
    blob += b" " * (-len(blob) % 8)
    with open(path, "wb") as f:
        f.write(struct.pack("<Q", len(blob)))
        f.write(blob)
        for a in arrays.values():
            f.write(a.tobytes())


def load(path: str, device=None) -> dict:
    """name -> dict(packed, scales, bits, nin); packed/scales as numpy arrays, or CUDA tensors
    on ``device``."""
    with open(path, "rb") as f:
        (n,) = struct.unpack("<Q", f.read(8))
        header = json.loads(f.read(n))
        data = f.read()
    header.pop("__metadata__", None)
    raw = {}
    for key, spec in header.items():
        a, b = spec["data_offsets"]
        raw[key] = np.frombuffer(data[a:b], dtype=_DTYPES[spec["dtype"]]).reshape(spec["shape"])
    out = {}
    for key in raw:
        if not key.endswith("_packed"):
            continue
        name = key[: -len("_packed")]
        packed, scales = raw[key], raw[f"{name}_scales"]
        if device is not None:
            import torch
            packed = torch.from_numpy(packed.copy()).to(device)
            scales = torch.from_numpy(scales.copy()).to(device)
        out[name] = {"packed": packed, "scales": scales, "bits": int(raw[f"{name}_bw"]),
                     "nin": int(raw[f"{name}_nin"])}
    return out
