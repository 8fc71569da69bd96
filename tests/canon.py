"""Hand-made canonical expert blobs for tests.

Packs explicit code / scale / bias matrices into the canonical blob format the
library and the oracle both consume: for each matrix in order gate [I][H],
up [I][H], down [H][I]: codes row-major, 32/bits codes per little-endian
uint32 with element c at bit bits*(c % (32/bits)) of word c/(32/bits) of its
row; then bf16 scales [R][C/64]; then bf16 biases [R][C/64].
"""
from __future__ import annotations

import numpy as np

GROUP = 64


def f32_to_bf16_exact(v) -> np.ndarray:
    """bf16 bits of values that are exactly representable in bf16."""
    a = np.asarray(v, dtype=np.float32)
    u = a.view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("value not exact in bf16")
    return (u >> 16).astype(np.uint16)


def pack_codes(q: np.ndarray, bits: int) -> bytes:
    q = np.asarray(q, dtype=np.uint32)
    R, C = q.shape
    per = 32 // bits
    assert C % per == 0 and q.max(initial=0) < (1 << bits)
    words = np.zeros((R, C // per), dtype=np.uint32)
    for j in range(per):
        words |= q[:, j::per] << np.uint32(bits * j)
    return words.astype("<u4").tobytes()


def pack_matrix(q, scale, bias, bits) -> bytes:
    q = np.asarray(q)
    R, C = q.shape
    s = np.broadcast_to(np.asarray(scale, dtype=np.float32), (R, C // GROUP))
    b = np.broadcast_to(np.asarray(bias, dtype=np.float32), (R, C // GROUP))
    return pack_codes(q, bits) + f32_to_bf16_exact(s).astype("<u2").tobytes() + \
        f32_to_bf16_exact(b).astype("<u2").tobytes()


def make_blob(hidden, inter, bits, gate, up, down) -> np.ndarray:
    """gate/up/down are (q, scale, bias) with q broadcastable to the matrix shape
    ([I][H] for gate and up, [H][I] for down) and scale/bias broadcastable to
    [R][C/64]."""
    parts = []
    for (q, s, b), (R, C) in zip((gate, up, down), ((inter, hidden), (inter, hidden), (hidden, inter))):
        qq = np.broadcast_to(np.asarray(q, dtype=np.uint32), (R, C))
        parts.append(pack_matrix(qq, s, b, bits))
    return np.frombuffer(b"".join(parts), dtype=np.uint8).copy()


def bf16_bits(values) -> np.ndarray:
    return f32_to_bf16_exact(values)
