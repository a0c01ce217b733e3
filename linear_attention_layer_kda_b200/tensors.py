"""Host <-> device plumbing for workloads made by ``inputs`` (torch tensors only)."""
from __future__ import annotations

import numpy as np
import torch

from .binding import WEIGHT_FIELDS, kda_weights, weights_from_tensors


def to_device_weights(inp, device="cuda") -> dict:
    """Dict of contiguous CUDA tensors holding the raw weight bytes (FP8 codes as uint8, bf16 bits as int16)."""
    out = {}
    for n in WEIGHT_FIELDS:
        a = np.ascontiguousarray(getattr(inp, n))
        if a.dtype == np.uint16:
            a = a.view(np.int16)
        out[n] = torch.from_numpy(a).to(device)
    return out


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def state_tensor(state: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(state, dtype=np.float32)).to(device)


def weights_struct(wt: dict) -> kda_weights:
    return weights_from_tensors(wt)
