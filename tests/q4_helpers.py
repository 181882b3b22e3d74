"""Test-side helpers that build Q4_0 inputs from chosen codes (the encoding
direction), so the oracle's decoding can be checked against values fixed by
construction rather than against a retyped decoder."""
from __future__ import annotations

import numpy as np


def encode_q4_0(q: np.ndarray, d_bits: np.ndarray) -> np.ndarray:
    """GGUF Q4_0 bytes from codes q[N][K] (0..15) and f16 scale bit patterns
    d_bits[N][K/32].  Byte j of block b holds code 32b+j in its low nibble
    and code 32b+16+j in its high nibble; the scale precedes the 16 bytes."""
    q = np.asarray(q, dtype=np.int64)
    N, K = q.shape
    assert K % 32 == 0 and q.min() >= 0 and q.max() <= 15
    d_bits = np.asarray(d_bits, dtype=np.uint16).reshape(N, K // 32)
    out = np.zeros((N, K // 32, 18), dtype=np.uint8)
    qb = q.reshape(N, K // 32, 32)
    out[:, :, 0] = (d_bits & 0xFF).astype(np.uint8)
    out[:, :, 1] = (d_bits >> 8).astype(np.uint8)
    out[:, :, 2:] = (qb[:, :, :16] | (qb[:, :, 16:] << 4)).astype(np.uint8)
    return out.reshape(N, (K // 32) * 18)


def f16_bits(values) -> np.ndarray:
    return np.asarray(values, dtype=np.float16).view(np.uint16)


def f16_values(bits) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def unrepack(packed: np.ndarray, N: int, K: int):
    """Inverse of the packed tile layout written with reshapes: returns GGUF
    bytes (N, K/32*18) and the padding rows.  Segment (t, b) is 576 bytes:
    codes [g=8][c=4][i=4][e=4] (row 32t+8i+g, qs byte 4c+e), then scales
    [g=8][i=4][2]."""
    KB = K // 32
    Np = (N + 31) // 32 * 32
    T = Np // 32
    seg = packed.reshape(T, KB, 576)
    nib = seg[:, :, :512].reshape(T, KB, 8, 4, 4, 4)
    nib = nib.transpose(0, 4, 2, 1, 3, 5).reshape(Np, KB, 16)   # (t,i,g,b,c,e)
    scl = seg[:, :, 512:].reshape(T, KB, 8, 4, 2)
    scl = scl.transpose(0, 3, 2, 1, 4).reshape(Np, KB, 2)        # (t,i,g,b,h)
    out = np.concatenate([scl, nib], axis=2)
    return out[:N].reshape(N, KB * 18), out[N:].reshape(Np - N, KB * 18)
