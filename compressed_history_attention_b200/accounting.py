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


def reduced_flops(Tq: int, T_low: int, d: int, r: int, dims) -> int:
    """Low-dim tokens of heads at reduced attention dimensions `dims` (one
    d_h per reduced head): scores and value products of width d_h, the decode
    of each token's key and value into d_h (once per token), the query
    reduction and the output restore (once per query row)."""
    if not (Tq and T_low):
        return 0
    return sum(4 * Tq * T_low * n + 4 * T_low * n * r + 2 * Tq * d * n + 2 * Tq * n * d for n in dims)


def routed_flops(Tq: int, H: int, d: int, r: int, C: int, T_full: int, T_low: int, T_cur: int,
                 kept: int = 0, dims=(), low_full: bool = False) -> dict:
    """A routed call: T_full tokens full-dim for every head; the T_low others
    full-dim for the `kept` heads (and for the ordinary heads too when
    `low_full`: codecs whose low-dim tokens run on the full-dim kernel), at
    reduced widths `dims` for the reduced heads, in the coefficient space for
    the rest; the current chunk and merge as in attend_flops."""
    nred = len(dims)
    nlow = H - kept - nred
    base = attend_flops(Tq, H, d, r, C, T_full, 0, T_cur)
    per_head = attend_flops(Tq, 1, d, r, C, T_low, 0, 0)["full"]     # one head, full-dim over T_low
    low_one = attend_flops(Tq, 1, d, r, C, 0, T_low, 0)["low"]       # one head, coefficient space
    full_low = (kept + (nlow if low_full else 0)) * per_head
    low = (0 if low_full else nlow) * low_one
    red = reduced_flops(Tq, T_low, d, r, dims)
    out = {"full": base["full"] + full_low, "low": low, "reduced": red, "current": base["current"]}
    out["total"] = out["full"] + out["low"] + out["reduced"] + out["current"]
    return out


def storage(T: int, H: int, d: int, r: int, C: int, x_bytes: int = 2, param_bytes: int = 2,
            scale_bytes: int = 2) -> dict:
    """Storage of a compressed history of T tokens (K and V), against the
    uncompressed cache (the pages' KV compression ratio, counted here for
    this layout): per token, J values of x_bytes against an id, r/2 bytes
    of codes and a scale; for the whole history, the two branches' codec
    parameters added (centers [C, J] and decoder D [J, r]; the encoder E,
    which attention never reads, in the second figure)."""
    J = H * d
    raw = 2 * T * J * x_bytes
    coded = 2 * T * token_bytes(r, scale_bytes)
    centers_d = 2 * (C * J + J * r) * param_bytes
    enc = 2 * r * J * param_bytes
    return {
        "raw_bytes": raw,
        "compressed_bytes": coded,
        "codec_bytes": centers_d,
        "encoder_bytes": enc,
        "per_token_ratio": (J * x_bytes) / token_bytes(r, scale_bytes),
        "effective_ratio": raw / (coded + centers_d) if T else 0.0,
        "effective_ratio_with_encoder": raw / (coded + centers_d + enc) if T else 0.0,
    }
