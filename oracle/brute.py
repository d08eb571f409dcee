"""Independent numpy fp64 brute force over CONTIGUOUS arrays (test infrastructure).

Used only to pin the C oracle: it never sees a block table or a pool.  It is
the textbook scaled-dot-product attention for one query row,
softmax(scale * q K^T) V, computed with numpy's own exp / max / matmul.
"""
from __future__ import annotations

import numpy as np


def attention_contiguous(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """q: [D]; K, V: [L][D] (any float dtype, widened to fp64).  Returns [D]."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    if K.shape[0] == 0:
        return np.zeros(q.shape[-1])
    logits = scale * (K @ q)
    w = np.exp(logits - logits.max())
    w = w / w.sum()
    return w @ V


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns, via the float32 they are the top half of."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)
