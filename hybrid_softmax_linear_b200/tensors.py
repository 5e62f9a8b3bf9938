"""Host <-> device plumbing for the binding's callers (tests, benchmark, smoke check):
numpy arrays from ``synth`` become torch device tensors of the library's element types,
and device results come back as float64 numpy arrays."""
from __future__ import annotations

import numpy as np
import torch


def to_torch(x: np.ndarray) -> torch.Tensor:
    """float32 stays float32; uint16 holds bf16 bit patterns and becomes bfloat16."""
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x))


def to_device(x: np.ndarray, device="cuda", pin: bool = False) -> torch.Tensor:
    t = to_torch(x)
    if pin:
        return t.pin_memory()
    return t.to(device, non_blocking=False)


def to_numpy(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def empty(shape, dtype: str, device="cuda") -> torch.Tensor:
    return torch.empty(shape, dtype={"f32": torch.float32, "bf16": torch.bfloat16}[dtype], device=device)


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A 256-byte aligned device workspace (torch's caching allocator aligns to 512)."""
    t = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    assert t.data_ptr() % 256 == 0
    return t
