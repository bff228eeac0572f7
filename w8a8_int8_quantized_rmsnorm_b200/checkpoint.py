"""ComfyUI ``comfy_quant`` checkpoints: read and write quantised linears.

The model cards describe the stored form of a ConvRot layer:

* "MOSS-Image Qwen3.5-9B text encoder, INT8 (W8A8, ConvRot)", file table:
  each quantised weight is int8 with one fp32 ``weight_scale`` per output
  row, and ComfyUI's mixed-precision loader reads ``comfy_quant`` per layer;
* "Qwen3-VL-8B-Heretic-1.3.0 - INT8 ConvRot (ComfyUI)", "Quantization
  metadata" and "Verification": one INT8 tensor, one F32 scale tensor and one
  U8 quantization-metadata tensor per quantised matrix, the metadata being
  {"format": "int8_tensorwise", "orig_dtype": "torch.bfloat16",
  "convrot": true, "convrot_groupsize": 256, "per_row": true};
* "MossInt4", "Format": the convrot_w4a4 layout keeps signed 4-bit codes two
  per byte in an I8 tensor with one F32 scale per row.

Readings of what the pages leave open: a layer ``<p>`` stores
``<p>.weight`` (I8, [N, K], or [N, K/2] packed for 4-bit codes),
``<p>.weight_scale`` (F32, [N] or [N, 1]) and ``<p>.comfy_quant`` (U8 bytes
of the metadata JSON); a 4-bit layer's metadata names the format
``convrot_w4a4``.  The file itself is the safetensors container: an 8-byte
little-endian header length, a JSON header mapping each tensor name to its
dtype, shape and byte range in the data section, then the data.

This module is host-side IO only (numpy and the standard library); moving
the arrays to a GPU and running layers is the caller's (see
``ConvRotLinear.from_checkpoint``).  Agreement of real checkpoints' Hadamard
ordering with this library's natural-order Sylvester matrix is not known:
no such file is available here.
"""
from __future__ import annotations

import json
import struct
from typing import Dict, Optional

import numpy as np

_DTYPES = {
    "BOOL": np.bool_, "U8": np.uint8, "I8": np.int8, "I16": np.int16, "U16": np.uint16,
    "I32": np.int32, "U32": np.uint32, "I64": np.int64, "U64": np.uint64,
    "F16": np.float16, "F32": np.float32, "F64": np.float64,
}
# bfloat16 has no numpy type: it is read as raw 16-bit words
_RAW16 = {"BF16"}

INT8_FORMAT = "int8_tensorwise"
INT4_FORMAT = "convrot_w4a4"

MAX_HEADER_BYTES = 100 * 1024 * 1024


class CheckpointError(ValueError):
    pass


def _parse_header(buf: bytes):
    if len(buf) < 8:
        raise CheckpointError("file shorter than the 8-byte header length")
    (n,) = struct.unpack("<Q", buf[:8])
    if n > MAX_HEADER_BYTES or 8 + n > len(buf):
        raise CheckpointError(f"header length {n} does not fit the file")
    try:
        header = json.loads(buf[8:8 + n].decode("utf-8"))
    except (UnicodeDecodeError, json.JSONDecodeError) as e:
        raise CheckpointError(f"header is not JSON: {e}") from None
    if not isinstance(header, dict):
        raise CheckpointError("header is not a JSON object")
    return header, 8 + n


def read_tensors(path: str) -> Dict[str, np.ndarray]:
    """Every tensor of a safetensors file as a numpy array (BF16 as uint16 words).

    The byte ranges are checked: inside the data section, consistent with
    dtype and shape, and not overlapping.  ``__metadata__`` is skipped.
    """
    with open(path, "rb") as f:
        buf = f.read()
    header, base = _parse_header(buf)
    data_len = len(buf) - base
    out, spans = {}, []
    for name, info in header.items():
        if name == "__metadata__":
            continue
        try:
            dtype, shape, (b, e) = info["dtype"], info["shape"], info["data_offsets"]
        except (KeyError, TypeError, ValueError):
            raise CheckpointError(f"{name}: malformed entry") from None
        if dtype in _RAW16:
            npt, item = np.uint16, 2
        elif dtype in _DTYPES:
            npt = _DTYPES[dtype]
            item = np.dtype(npt).itemsize
        else:
            raise CheckpointError(f"{name}: unsupported dtype {dtype}")
        count = int(np.prod(shape)) if shape else 1
        if not (0 <= b <= e <= data_len) or e - b != count * item:
            raise CheckpointError(f"{name}: byte range [{b}, {e}) does not match {dtype}{shape}")
        spans.append((b, e, name))
        out[name] = np.frombuffer(buf, dtype=npt, count=count, offset=base + b).reshape(shape).copy()
    spans.sort()
    for (b0, e0, n0), (b1, e1, n1) in zip(spans, spans[1:]):
        if b1 < e0:
            raise CheckpointError(f"{n0} and {n1} overlap")
    return out


def write_tensors(path: str, tensors: Dict[str, np.ndarray], dtypes: Optional[Dict[str, str]] = None,
                  metadata: Optional[Dict[str, str]] = None) -> None:
    """Writes numpy arrays as a safetensors file (``dtypes`` overrides, e.g. BF16
    for uint16 words).  Tensors are laid out in name order, 8-byte aligned."""
    rev = {np.dtype(v): k for k, v in _DTYPES.items()}
    header, chunks, off = {}, [], 0
    for name in sorted(tensors):
        a = np.ascontiguousarray(tensors[name])
        dt = (dtypes or {}).get(name) or rev.get(a.dtype)
        if dt is None:
            raise CheckpointError(f"{name}: no safetensors dtype for {a.dtype}")
        raw = a.tobytes()
        header[name] = {"dtype": dt, "shape": list(a.shape), "data_offsets": [off, off + len(raw)]}
        pad = (-len(raw)) % 8
        chunks.append(raw + b"\0" * pad)
        off += len(raw) + pad
    if metadata:
        header["__metadata__"] = {str(k): str(v) for k, v in metadata.items()}
    hj = json.dumps(header, separators=(",", ":")).encode("utf-8")
    hj += b" " * ((-len(hj)) % 8)
    with open(path, "wb") as f:
        f.write(struct.pack("<Q", len(hj)))
        f.write(hj)
        for c in chunks:
            f.write(c)


def quant_metadata(group: int = 256, bits: int = 8, orig_dtype: str = "torch.bfloat16") -> dict:
    """The per-layer metadata of a ConvRot linear (group 0: no rotation)."""
    return {"format": INT8_FORMAT if bits == 8 else INT4_FORMAT, "orig_dtype": orig_dtype,
            "convrot": group > 0, "convrot_groupsize": int(group) if group > 0 else 0, "per_row": True}


def load_quantized_layers(path: str) -> Dict[str, dict]:
    """The ConvRot linears of a comfy_quant checkpoint.

    Returns {layer prefix: {"Wq": int8 [N, K] or packed uint8 [N, K/2],
    "s_row": float32 [N], "group": 256 / 16 / 0, "bits": 8 or 4,
    "meta": the metadata dict}}.  Layers whose metadata is not per-row
    int8_tensorwise / convrot_w4a4 raise CheckpointError.
    """
    t = read_tensors(path)
    layers = {}
    for name in t:
        if not name.endswith(".comfy_quant"):
            continue
        p = name[: -len(".comfy_quant")]
        try:
            meta = json.loads(bytes(t[name].astype(np.uint8)).decode("utf-8"))
        except (UnicodeDecodeError, json.JSONDecodeError) as e:
            raise CheckpointError(f"{name}: metadata is not JSON: {e}") from None
        fmt = meta.get("format")
        if fmt not in (INT8_FORMAT, INT4_FORMAT):
            raise CheckpointError(f"{p}: unsupported format {fmt!r}")
        if not meta.get("per_row", False):
            raise CheckpointError(f"{p}: only row-wise scales are supported")
        group = int(meta.get("convrot_groupsize", 0)) if meta.get("convrot", False) else 0
        if group not in (0, 16, 256):
            raise CheckpointError(f"{p}: unsupported ConvRot group size {group}")
        if p + ".weight" not in t or p + ".weight_scale" not in t:
            raise CheckpointError(f"{p}: weight or weight_scale missing")
        W, s = t[p + ".weight"], t[p + ".weight_scale"]
        if W.ndim != 2 or W.dtype not in (np.int8, np.uint8):
            raise CheckpointError(f"{p}: weight must be a 2-D int8 tensor")
        s = s.reshape(-1)
        if s.dtype != np.float32 or s.shape[0] != W.shape[0]:
            raise CheckpointError(f"{p}: weight_scale must be fp32 with one value per row")
        bits = 8 if fmt == INT8_FORMAT else 4
        layers[p] = {"Wq": W.view(np.int8) if bits == 8 else W.view(np.uint8), "s_row": s,
                     "group": group, "bits": bits, "meta": meta}
    return layers


def save_quantized_layers(path: str, layers: Dict[str, dict], extra: Optional[Dict[str, np.ndarray]] = None,
                          extra_dtypes: Optional[Dict[str, str]] = None) -> None:
    """Writes ConvRot linears ({prefix: {"Wq", "s_row", "group", "bits"}}) in the
    comfy_quant form read by load_quantized_layers; ``extra`` holds other tensors."""
    tensors = dict(extra or {})
    for p, L in layers.items():
        bits = int(L.get("bits", 8))
        meta = L.get("meta") or quant_metadata(int(L.get("group", 256)), bits)
        tensors[p + ".weight"] = np.asarray(L["Wq"]).view(np.int8)
        tensors[p + ".weight_scale"] = np.asarray(L["s_row"], dtype=np.float32).reshape(-1)
        tensors[p + ".comfy_quant"] = np.frombuffer(json.dumps(meta).encode("utf-8"), dtype=np.uint8)
    write_tensors(path, tensors, extra_dtypes)
