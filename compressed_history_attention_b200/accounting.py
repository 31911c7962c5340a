"""Algorithmic work and storage of the path, counted once per call.

Attention multiply-adds are counted as in the pages' Table 11 accounting of
visual-attention MACs: each score and each value product once, the decode of
a history token once (not once per query tile that re-decodes it), and the
low-dim query prep and output restore once per query row and head.
"""
from __future__ import annotations


def attend_flops(Tq: int, H: int, d: int, r: int, C: int, T_full: int, T_low: int, T_cur: int) -> dict:
    J = H * d
    full = 4 * Tq * T_full * J + (4 * T_full * J * r if Tq else 0)
    low = 0
    if T_low and Tq:
        low = 4 * Tq * T_low * H * r + 2 * Tq * J * (r + C) + 2 * Tq * H * (r + C) * d
    cur = 4 * Tq * T_cur * J
    return {"full": full, "low": low, "current": cur, "total": full + low + cur}


def encode_flops(T: int, J: int, r: int, C: int) -> int:
    """One branch: distances to C centers and the projection, 2 flops per MAC."""
    return 2 * T * J * (C + r)


def encode_bytes(T: int, J: int, r: int, x_bytes: int = 2, scale_bytes: int = 2) -> int:
    """One branch: read the tokens, write ids, packed codes and scales."""
    return T * J * x_bytes + T * (1 + r // 2 + scale_bytes)


def token_bytes(r: int, scale_bytes: int = 2) -> int:
    """Compressed bytes of one token in one branch: id + codes + scale."""
    return 1 + r // 2 + scale_bytes
