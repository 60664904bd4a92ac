"""Helpers shared by the GPU parity tests (marshalling only, no arithmetic)."""
from __future__ import annotations

import numpy as np
import torch


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 bit patterns on the host."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def host_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().contiguous().numpy()
