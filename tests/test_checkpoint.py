"""The comfy_quant checkpoint reader and writer: the safetensors container
(checked against a file assembled by hand from the format's definition), the
per-layer metadata the cards print, round trips and malformed inputs."""
import json
import os
import struct

import numpy as np
import pytest

from w8a8_int8_quantized_rmsnorm_b200 import checkpoint as ck

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _hand_file(path, entries, data, header_extra=None):
    header = dict(entries)
    if header_extra:
        header.update(header_extra)
    hj = json.dumps(header).encode()
    with open(path, "wb") as f:
        f.write(struct.pack("<Q", len(hj)) + hj + data)


def test_reader_against_a_hand_assembled_file(tmp_path):
    # two tensors written byte by byte: I8 [2, 3] then F32 [2], little endian
    w = bytes([1, 2, 3, 0xFF, 0x80, 0x7F])
    s = struct.pack("<2f", 0.5, -2.25)
    p = str(tmp_path / "hand.safetensors")
    _hand_file(p, {"a.weight": {"dtype": "I8", "shape": [2, 3], "data_offsets": [0, 6]},
                   "a.weight_scale": {"dtype": "F32", "shape": [2], "data_offsets": [6, 14]}},
               w + s, {"__metadata__": {"format": "pt"}})
    t = ck.read_tensors(p)
    assert t["a.weight"].tolist() == [[1, 2, 3], [-1, -128, 127]]
    assert t["a.weight_scale"].tolist() == [0.5, -2.25]


def test_metadata_matches_the_card():
    assert ck.quant_metadata(256, 8) == _golden("comfy_quant_metadata.json")["metadata"]


def test_writer_layout_and_round_trip(tmp_path):
    rng = np.random.default_rng(0)
    layers = {
        "model.layers.1.mlp.down_proj": {"Wq": rng.integers(-127, 128, (16, 512), dtype=np.int8),
                                         "s_row": rng.random(16, dtype=np.float32), "group": 256, "bits": 8},
        "model.visual.blocks.1.mlp.linear_fc1": {"Wq": rng.integers(-127, 128, (8, 1152), dtype=np.int8),
                                                 "s_row": rng.random(8, dtype=np.float32), "group": 16,
                                                 "bits": 8},
        "model.layers.2.self_attn.q_proj": {"Wq": rng.integers(0, 256, (8, 128), dtype=np.uint8),
                                            "s_row": rng.random(8, dtype=np.float32), "group": 256, "bits": 4},
    }
    norm = rng.integers(0, 1 << 16, 64, dtype=np.uint16)  # bf16 words
    p = str(tmp_path / "q.safetensors")
    ck.save_quantized_layers(p, layers, extra={"model.norm.weight": norm},
                             extra_dtypes={"model.norm.weight": "BF16"})
    # container: header length, JSON, contiguous 8-byte aligned ranges
    raw = open(p, "rb").read()
    (n,) = struct.unpack("<Q", raw[:8])
    header = json.loads(raw[8:8 + n])
    spans = sorted(v["data_offsets"] for k, v in header.items() if k != "__metadata__")
    assert spans[0][0] == 0 and all(b % 8 == 0 for b, _ in spans)
    assert all(e0 <= b1 for (_, e0), (b1, _) in zip(spans, spans[1:]))
    assert header["model.norm.weight"]["dtype"] == "BF16"
    assert header["model.layers.1.mlp.down_proj.comfy_quant"]["dtype"] == "U8"
    assert header["model.layers.1.mlp.down_proj.weight_scale"]["dtype"] == "F32"
    # counts by dtype follow the card's "Verification" pattern: one I8, one F32
    # and one U8 tensor per quantised matrix
    kinds = [v["dtype"] for k, v in header.items() if k != "__metadata__"]
    assert kinds.count("I8") == kinds.count("F32") == kinds.count("U8") == 3
    got = ck.load_quantized_layers(p)
    assert set(got) == set(layers)
    for k, L in layers.items():
        g = got[k]
        assert g["group"] == L["group"] and g["bits"] == L["bits"]
        assert np.array_equal(g["Wq"].view(np.uint8), L["Wq"].view(np.uint8))
        assert np.array_equal(g["s_row"], L["s_row"])
    assert got["model.visual.blocks.1.mlp.linear_fc1"]["meta"]["convrot_groupsize"] == 16
    assert got["model.layers.2.self_attn.q_proj"]["meta"]["format"] == "convrot_w4a4"
    assert np.array_equal(ck.read_tensors(p)["model.norm.weight"], norm)


@pytest.mark.parametrize("case", ["short", "length", "json", "range", "overlap", "dtype"])
def test_malformed_files_are_rejected(tmp_path, case):
    p = str(tmp_path / "bad.safetensors")
    good = {"x": {"dtype": "I8", "shape": [4], "data_offsets": [0, 4]}}
    if case == "short":
        open(p, "wb").write(b"\1\2\3")
    elif case == "length":
        open(p, "wb").write(struct.pack("<Q", 1 << 40) + b"{}")
    elif case == "json":
        open(p, "wb").write(struct.pack("<Q", 3) + b"{x}")
    elif case == "range":
        _hand_file(p, {"x": {"dtype": "I8", "shape": [4], "data_offsets": [0, 8]}}, bytes(4))
    elif case == "overlap":
        _hand_file(p, {**good, "y": {"dtype": "I8", "shape": [4], "data_offsets": [2, 6]}}, bytes(8))
    else:
        _hand_file(p, {"x": {"dtype": "Q4", "shape": [4], "data_offsets": [0, 4]}}, bytes(4))
    with pytest.raises(ck.CheckpointError):
        ck.read_tensors(p)


@pytest.mark.parametrize("bad", ["no_scale", "per_tensor", "group", "format", "scale_len"])
def test_layer_validation(tmp_path, bad):
    meta = ck.quant_metadata(256, 8)
    t = {"l.weight": np.zeros((4, 256), np.int8), "l.weight_scale": np.ones(4, np.float32)}
    if bad == "no_scale":
        del t["l.weight_scale"]
    elif bad == "per_tensor":
        meta["per_row"] = False
    elif bad == "group":
        meta["convrot_groupsize"] = 64
    elif bad == "format":
        meta["format"] = "float8_e4m3fn"
    else:
        t["l.weight_scale"] = np.ones(3, np.float32)
    t["l.comfy_quant"] = np.frombuffer(json.dumps(meta).encode(), np.uint8)
    p = str(tmp_path / "l.safetensors")
    ck.write_tensors(p, t)
    with pytest.raises(ck.CheckpointError):
        ck.load_quantized_layers(p)
