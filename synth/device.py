"""Put a synthetic workload's tensors on a CUDA device (torch tensors, bf16).

Generation happens on the host in row chunks (so a full-size workload never needs
its whole input in host memory at once) and each chunk is copied into the device
tensor. Shapes follow the operand layouts:
    x, residual            (B, L, D)
    bcast operand          (1, 1, D)
    row operand            (B, L, D)
    frame operand          (B, F, 1, D)
    batch operand          (B, 1, D)
    weight, bias           (D,)
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import Spec, Workload


def operand_view_shape(w: Workload, op: str):
    if op in ("weight", "bias"):
        return (w.D,)
    lay = w.layout(op)
    return {"bcast": (1, 1, w.D), "row": (w.B, w.L, w.D), "frame": (w.B, w.F, 1, w.D),
            "batch": (w.B, 1, w.D)}[lay]


def upload_tensor(w: Workload, tensor: str, device, chunk_rows: int = 16384,
                  out: Optional[torch.Tensor] = None) -> torch.Tensor:
    n = 1 if tensor in ("weight", "bias") else w.stored_rows(tensor)
    dev = out if out is not None else torch.empty((n, w.D), dtype=torch.bfloat16, device=device)
    flat = dev.view(n, w.D)
    host = torch.empty((min(chunk_rows, n), w.D), dtype=torch.int16, pin_memory=True)
    host_np = host.numpy().view(np.uint16)
    for r0 in range(0, n, chunk_rows):
        r1 = min(n, r0 + chunk_rows)
        w.generate(tensor, np.arange(r0, r1, dtype=np.int64), out=host_np[: r1 - r0])
        flat[r0:r1].copy_(host[: r1 - r0].view(torch.bfloat16), non_blocking=False)
    return dev.view(operand_view_shape(w, tensor))


def upload(w: Workload, spec: Spec, device, chunk_rows: int = 16384) -> Dict[str, Optional[torch.Tensor]]:
    """Device tensors for every operand the specialisation reads (others are None)."""
    t = {"x": upload_tensor(w, "x", device, chunk_rows)}
    t["residual"] = None if spec.norm_only else upload_tensor(w, "residual", device, chunk_rows)
    t["gate"] = upload_tensor(w, "gate", device, chunk_rows) if (spec.has_gate and not spec.norm_only) else None
    t["weight"] = upload_tensor(w, "weight", device) if spec.has_weight else None
    t["bias"] = upload_tensor(w, "bias", device) if spec.has_bias else None
    t["scale"] = upload_tensor(w, "scale", device, chunk_rows)
    t["shift"] = upload_tensor(w, "shift", device, chunk_rows)
    return t


def to_bits(t: torch.Tensor) -> np.ndarray:
    """A bf16 tensor's bit patterns as a host numpy uint16 array."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def from_bits(a: np.ndarray, device) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
