"""The on-disk format of quantized weights, as the "量化推理：INT8/INT4 ..." page writes it.

A folder holds, for every quantized tensor `name`:

    name.bin      the payload bytes of qpack (int4: code + 8, two per byte, the even element in
                  the low nibble; int8: two's complement), flattened row-major
    name.scale    its scales, little-endian fp32, one per `group` consecutive weights

for every tensor kept unquantized, `name.f32` (little-endian fp32, row-major), and
`manifest.json`, which maps each quantized name to {"bits", "group", "shape"} (the page
writes it with an indent of 2; unquantized tensors are not listed, so their shape is not
stored and they load flat unless the caller gives shapes).

Writing and reading are plain file IO on the host. `quantize_and_save` packs CUDA tensors
with qpack on the GPU; `load(..., device="cuda")` returns tensors ready for qdequant and
qgemm. Loading checks every file's size against its manifest entry and raises ValueError
on any mismatch.
"""
from __future__ import annotations

import json
import os
from dataclasses import dataclass
from typing import Dict, Iterable, Mapping, Optional, Sequence, Tuple

import numpy as np
import torch

from . import payload_bytes, qpack

MANIFEST = "manifest.json"


@dataclass
class QTensor:
    payload: torch.Tensor   # uint8, flat
    scales: torch.Tensor    # float32, flat
    bits: int
    group: int
    shape: Tuple[int, ...]

    @property
    def numel(self) -> int:
        return int(np.prod(self.shape)) if self.shape else 1


def _as_bytes(t) -> bytes:
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().numpy()
    return np.ascontiguousarray(t).tobytes()


def save(folder: str, quantized: Mapping[str, QTensor], plain: Optional[Mapping[str, object]] = None) -> None:
    """Write `quantized` (payload + scales + manifest entries) and `plain` fp32 tensors."""
    os.makedirs(folder, exist_ok=True)
    manifest = {}
    for name, q in quantized.items():
        if q.payload.numel() != payload_bytes(q.numel, 1, q.bits) or q.scales.numel() * q.group != q.numel:
            raise ValueError(f"{name}: payload or scales do not match bits={q.bits}, group={q.group}, shape={q.shape}")
        with open(os.path.join(folder, f"{name}.bin"), "wb") as f:
            f.write(_as_bytes(q.payload))
        scales = q.scales.detach().cpu().numpy() if isinstance(q.scales, torch.Tensor) else np.asarray(q.scales)
        with open(os.path.join(folder, f"{name}.scale"), "wb") as f:
            f.write(np.ascontiguousarray(scales, dtype="<f4").tobytes())
        manifest[name] = {"bits": int(q.bits), "group": int(q.group), "shape": [int(s) for s in q.shape]}
    for name, t in (plain or {}).items():
        a = t.detach().cpu().numpy() if isinstance(t, torch.Tensor) else np.asarray(t)
        with open(os.path.join(folder, f"{name}.f32"), "wb") as f:
            f.write(np.ascontiguousarray(a, dtype="<f4").tobytes())
    with open(os.path.join(folder, MANIFEST), "w") as f:
        f.write(json.dumps(manifest, indent=2))


def load(folder: str, device=None, shapes: Optional[Mapping[str, Sequence[int]]] = None
         ) -> Tuple[Dict[str, QTensor], Dict[str, torch.Tensor]]:
    """Read a folder back: ({name: QTensor}, {name: fp32 tensor}) on `device` (CPU if None)."""
    with open(os.path.join(folder, MANIFEST)) as f:
        manifest = json.load(f)
    dev = torch.device("cpu") if device is None else torch.device(device)
    quantized = {}
    for name, meta in manifest.items():
        bits, group, shape = int(meta["bits"]), int(meta["group"]), tuple(int(s) for s in meta["shape"])
        n = int(np.prod(shape)) if shape else 1
        if bits not in (4, 8) or group < 1 or n % group or (bits == 4 and n % 2):
            raise ValueError(f"{name}: invalid manifest entry {meta}")
        with open(os.path.join(folder, f"{name}.bin"), "rb") as f:
            pb = f.read()
        with open(os.path.join(folder, f"{name}.scale"), "rb") as f:
            sb = f.read()
        if len(pb) != n * bits // 8 or len(sb) != 4 * (n // group):
            raise ValueError(f"{name}: {len(pb)} payload / {len(sb)} scale bytes do not match {meta}")
        payload = torch.from_numpy(np.frombuffer(pb, dtype=np.uint8).copy()).to(dev)
        scales = torch.from_numpy(np.frombuffer(sb, dtype="<f4").astype(np.float32)).to(dev)
        quantized[name] = QTensor(payload, scales, bits, group, shape)
    plain = {}
    for fn in sorted(os.listdir(folder)):
        if fn.endswith(".f32"):
            name = fn[:-4]
            with open(os.path.join(folder, fn), "rb") as f:
                a = np.frombuffer(f.read(), dtype="<f4").astype(np.float32)
            if shapes and name in shapes:
                a = a.reshape(tuple(shapes[name]))
            plain[name] = torch.from_numpy(a).to(dev)
    return quantized, plain


def quantize_and_save(folder: str, weights: Mapping[str, torch.Tensor], bits: int, group: Optional[int],
                      keep: Iterable[str] = ()) -> Dict[str, QTensor]:
    """qpack every CUDA fp32 tensor of `weights` (group None: the whole tensor, one scale)
    except the names in `keep`, which are written as fp32; then save the folder."""
    keep = set(keep)
    quantized, plain = {}, {}
    for name, w in weights.items():
        if name in keep:
            plain[name] = w
            continue
        g = w.numel() if group is None else group
        payload, scales = qpack(w.contiguous(), bits, g)
        quantized[name] = QTensor(payload, scales, bits, g, tuple(w.shape))
    save(folder, quantized, plain)
    return quantized
