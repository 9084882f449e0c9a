"""Comparison helpers shared by the tests (no arithmetic of the operators)."""
from __future__ import annotations

import numpy as np
import torch


def bits16(t) -> np.ndarray:
    """uint16 bit patterns of a 16-bit torch tensor (any device) or array."""
    if isinstance(t, torch.Tensor):
        return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(t)
    assert a.dtype.itemsize == 2
    return a.view(np.uint16)


def codes8(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().cpu().contiguous().view(torch.uint8).numpy()
    return np.ascontiguousarray(t, dtype=np.uint8)


def ordered16(b: np.ndarray) -> np.ndarray:
    """Maps sign-magnitude 16-bit floats onto integers ordered like their values
    (+0 and -0 both map to 0), so |a - b| counts ulps."""
    b = b.astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def ordered8(c: np.ndarray) -> np.ndarray:
    c = c.astype(np.int64)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def ulp16(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    return np.abs(ordered16(a) - ordered16(b))


def code_dist8(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    return np.abs(ordered8(a) - ordered8(b))


def from_bits(bits: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).view(dtype)
