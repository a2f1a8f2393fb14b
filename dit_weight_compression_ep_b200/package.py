"""Compressed-model packages: a safetensors file of compressed tensors and a same-named JSON sidecar
(the pages ship their pre-quantised models this way: each `*.safetensors` with a `*.json`).

Layout (all little-endian, the library's stored representation unchanged):
  `<layer>.payload`      U16  the payload words, padded with zeros to a multiple of 8
  `<layer>.tile_index`   U32  33 T + 1 words: per tile [offset, 32 states], then the end offset
  `<layer>.freq_tables`  U8   the table header and frequencies
  `<layer>.row_scales`   F32  one per row
The safetensors metadata holds the format name and, per layer, its shape and geometry (rows,
cols, b, V, tiles, payload words, the search's scale, stored bytes and bpp).  The sidecar repeats
that and adds the package totals: numel, stored bytes, bpp = 8 * sum(stored bytes) / sum(numel)
and the linear-weight compression ratio against bf16, bpp / 16 (the pages' two package metrics).
"""
from __future__ import annotations

import json
import os

import numpy as np

from ._lib import Blob, DeviceBlob

FORMAT = "entropack-b200/1"
ARRAYS = ("payload", "tile_index", "freq_tables", "row_scales")


def _sidecar_path(path: str) -> str:
    root, _ = os.path.splitext(path)
    return root + ".json"


def save_package(path: str, blobs: dict, extra: dict | None = None) -> dict:
    """Write `blobs` ({layer name: Blob}) to `path` (.safetensors) and its .json sidecar; returns the
    sidecar's contents.  `extra` (JSON-serialisable) is stored in the sidecar as given."""
    from safetensors.numpy import save_file

    tensors, layers = {}, {}
    for name, b in blobs.items():
        if "." in name or not name:
            raise ValueError(f"layer names may not be empty or contain '.': {name!r}")
        alloc = max(8, (int(b.payload_words) + 7) // 8 * 8)
        pay = np.zeros(alloc, np.uint16)
        pay[: int(b.payload_words)] = np.asarray(b.payload, np.uint16)[: int(b.payload_words)]
        tensors[f"{name}.payload"] = pay
        tensors[f"{name}.tile_index"] = np.ascontiguousarray(b.tile_index, np.uint32)
        tensors[f"{name}.freq_tables"] = np.ascontiguousarray(b.freq_tables, np.uint8)
        tensors[f"{name}.row_scales"] = np.ascontiguousarray(b.row_scales, np.float32)
        layers[name] = {"rows": int(b.rows), "cols": int(b.cols), "b": int(b.b), "V": int(b.V),
                        "ntiles": int(b.ntiles), "payload_words": int(b.payload_words), "s": float(b.s),
                        "stored_bytes": int(b.stored_bytes), "stored_bpp": float(b.stored_bpp)}
    numel = sum(v["rows"] * v["cols"] for v in layers.values())
    stored = sum(v["stored_bytes"] for v in layers.values())
    save_file(tensors, path, metadata={"format": FORMAT, "layers": json.dumps(layers, sort_keys=True)})
    bpp = 8.0 * stored / numel if numel else 0.0
    side = {"format": FORMAT, "package": os.path.basename(path), "layers": layers, "numel": numel,
            "stored_bytes": stored, "bpp": bpp, "ratio_vs_bf16": bpp / 16.0}
    if extra is not None:
        side["extra"] = extra
    with open(_sidecar_path(path), "w") as f:
        json.dump(side, f, indent=1, sort_keys=True)
    return side


def _layers_of(path: str) -> dict:
    from safetensors import safe_open

    with safe_open(path, framework="np") as f:
        meta = f.metadata() or {}
    if meta.get("format") != FORMAT:
        raise ValueError(f"{path}: not an {FORMAT} package")
    return json.loads(meta["layers"])


def load_package(path: str) -> dict:
    """{layer name: Blob} from a package written by save_package (host memory)."""
    from safetensors.numpy import load_file

    layers = _layers_of(path)
    t = load_file(path)
    out = {}
    for name, v in layers.items():
        arr = {a: t[f"{name}.{a}"] for a in ARRAYS}
        if arr["tile_index"].size != 33 * v["ntiles"] + 1 or arr["row_scales"].size != v["rows"]:
            raise ValueError(f"{path}: layer {name!r} does not match its metadata")
        out[name] = Blob(v["rows"], v["cols"], v["b"], v["V"], v["ntiles"], arr["payload"], v["payload_words"],
                         arr["tile_index"], arr["freq_tables"], arr["row_scales"], v["s"], v["stored_bpp"],
                         v["stored_bytes"])
    return out


def load_package_to_device(path: str, device="cuda") -> dict:
    """{layer name: DeviceBlob} from a package: each layer's arrays copied to `device`."""
    return {name: DeviceBlob(b, device) for name, b in load_package(path).items()}
