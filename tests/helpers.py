"""Test helpers: bit views and dense (un-paged) copies built with numpy indexing."""
from __future__ import annotations

import numpy as np
import torch


def bits16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def bf16_values(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bits -> fp64 via numpy (independent of the oracle's C)."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def dense_kv(cache_vals: np.ndarray, page_table: np.ndarray, b: int, L: int, page_size: int = 64):
    """Contiguous [L][Hkv][D] copy of sequence b's cache, via numpy fancy indexing."""
    j = np.arange(L)
    pages = page_table[b, j // page_size]
    return cache_vals[pages, :, j % page_size, :]


def dense_attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """softmax(Q K^T * scale) V for one sequence, dense fp64 matrices.

    q: [Hq][D]; K, V: [L][Hkv][D]; head h reads kv head h // (Hq // Hkv)."""
    Hq, D = q.shape
    Hkv = K.shape[1]
    G = Hq // Hkv
    out = np.empty((Hq, D))
    for g in range(Hkv):
        Q = q[g * G:(g + 1) * G]                    # [G][D]
        S = (Q @ K[:, g, :].T) * scale              # [G][L]
        S = S - S.max(axis=1, keepdims=True)
        P = np.exp(S)
        P = P / P.sum(axis=1, keepdims=True)
        out[g * G:(g + 1) * G] = P @ V[:, g, :]
    return out
