"""Host -> device marshalling of the generator's arrays (no arithmetic of the method).

The input generator stores bf16 values as their 16-bit patterns in numpy uint16 arrays (numpy has no
bfloat16); they are reinterpreted, not converted, on the way to the device."""
from __future__ import annotations

import numpy as np
import torch

__all__ = ["to_device"]


def to_device(a: np.ndarray, device: str = "cuda") -> torch.Tensor:
    """Copy a numpy array to `device`; uint16 arrays become bfloat16 tensors with the same bits."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(a).to(device)
