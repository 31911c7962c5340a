"""Plant plausible mistakes in the oracle (on the CPU, one at a time) and check
that at least one pin catches each of them."""
import numpy as np
import pytest

from oracle import nanokv_oracle as orc
from tests import test_oracle_pins as pins

PINS = [getattr(pins, n) for n in dir(pins) if n.startswith("test_")]


def _run_pins():
    failed = []
    for fn in PINS:
        kwargs = {"tau": 1.0} if "tau" in fn.__code__.co_varnames[:fn.__code__.co_argcount] else {}
        try:
            fn(**kwargs)
        except Exception:
            failed.append(fn.__name__)
    return failed


def _decode_no_center(ids, codes, scales, centers, D):
    return scales[:, None] * (np.asarray(codes, np.float64) @ D.T)


def _decode_no_scale(ids, codes, scales, centers, D):
    return centers[ids] + (np.asarray(codes, np.float64) @ D.T)


def _quantise_floor(y, s):
    codes = np.zeros(y.shape, dtype=np.int64)
    nz = s > 0
    codes[nz] = np.clip(np.floor(y[nz] / s[nz, None] + 0.5), -7, 7).astype(np.int64)
    return codes


def _scale_unrounded(y, scale_dtype):
    return np.max(np.abs(y), axis=1) / 7


def _assign_argmax(x, centers):
    return np.argmax(orc.squared_distances(x, centers), axis=1)


def _project_no_center(x, centers, ids, E):
    return x @ E.T


def _merge_max(parts):
    lses = np.stack([p[1] for p in parts])
    idx = np.argmax(lses, axis=0)
    O = np.zeros_like(parts[0][0])
    for i, (o, _) in enumerate(parts):
        O += (idx == i).T[:, :, None] * o
    return O, lses.max(axis=0)


def _pack_swapped(codes):
    c = (np.asarray(codes, dtype=np.int64) & 0xF).astype(np.uint8)
    return (c[:, 1::2] | (c[:, 0::2] << 4)).astype(np.uint8)


_orig_low = orc.attend_low


def _low_wrong_value_scale(q, ck, cv, hk, hv, tau):
    hv2 = dict(hv, scales=hk["scales"])
    return _orig_low(q, ck, cv, hk, hv2, tau)


def _low_no_key_center(q, ck, cv, hk, hv, tau):
    ck2 = dict(ck, centers=np.zeros_like(ck["centers"]))
    return _orig_low(q, ck2, cv, hk, hv, tau)


_orig_sm = orc.softmax_attention


def _softmax_no_tau(q, k, v, tau):
    return _orig_sm(q, k, v, 1.0 if tau != 1.0 else 0.5)


_orig_encode = orc.encode


def _encode_projects_from_first_center(x, centers, E, scale_dtype):
    r = _orig_encode(x, centers, E, scale_dtype)
    y = orc.project(x, centers, np.zeros_like(r["ids"]), E)
    s = orc.scale_of(y, scale_dtype)
    return dict(r, y=y, scales=s, codes=orc.quantise(y, s))


def _encode_codes_from_unrounded_scale(x, centers, E, scale_dtype):
    r = _orig_encode(x, centers, E, scale_dtype)
    m = np.max(np.abs(r["y"]), axis=1) / 7
    return dict(r, codes=orc.quantise(r["y"], m))


def _encode_returns_unquantised(x, centers, E, scale_dtype):
    r = _orig_encode(x, centers, E, scale_dtype)
    return dict(r, codes=r["y"])


def _encode_scale_from_residual(x, centers, E, scale_dtype):
    r = _orig_encode(x, centers, E, scale_dtype)
    s = orc.scale_of(x - centers[r["ids"]], scale_dtype)
    return dict(r, scales=s, codes=orc.quantise(r["y"], s))


_orig_routed = orc.attend_routed


def _routed_drops_low_tokens(q, ck, cv, hk, hv, full_mask, full_heads=None, k_cur=None, v_cur=None, tau=None,
                             lowdim=None):
    m = np.asarray(full_mask, dtype=bool)
    keep = np.nonzero(m)[0]
    return _orig_routed(q, ck, cv, orc.take_history(hk, keep), orc.take_history(hv, keep), m[keep],
                        full_heads, k_cur, v_cur, tau, lowdim)


def _routed_kept_heads_skip_current(q, ck, cv, hk, hv, full_mask, full_heads=None, k_cur=None, v_cur=None, tau=None,
                                    lowdim=None):
    O, L = _orig_routed(q, ck, cv, hk, hv, full_mask, full_heads, k_cur, v_cur, tau, lowdim)
    if full_heads is None:
        return O, L
    O2, L2 = _orig_routed(q, ck, cv, hk, hv, np.ones_like(np.asarray(full_mask, bool)), None, None, None, tau)
    sel = np.asarray(full_heads, dtype=bool)
    return np.where(sel[None, :, None], O2, O), np.where(sel[:, None], L2, L)


_orig_reduced = orc.attend_reduced


def _reduced_swaps_maps(q, ck, cv, hk, hv, maps, tau):
    return _orig_reduced(q, ck, cv, hk, hv, dict(maps, U=maps["W"], W=maps["U"]), tau)


def _reduced_trailing_columns(q, ck, cv, hk, hv, maps, tau):
    U, W = np.asarray(maps["U"]), np.asarray(maps["W"])
    return _orig_reduced(q, ck, cv, hk, hv, dict(maps, U=U[:, :, ::-1], W=W[:, :, ::-1]), tau)


def _reduced_rescales_tau(q, ck, cv, hk, hv, maps, tau):
    d = q.shape[2]
    O = np.zeros(q.shape)
    L = np.zeros((q.shape[1], q.shape[0]))
    for h in range(q.shape[1]):
        n = int(maps["d_h"][h])
        o, lse = _orig_reduced(q, ck, cv, hk, hv, maps, tau * np.sqrt(d / n))
        O[:, h], L[h] = o[:, h], lse[h]
    return O, L


def _reduced_restores_with_key_map(q, ck, cv, hk, hv, maps, tau):
    Tq, H, d = q.shape
    O, L = _orig_reduced(q, ck, cv, hk, hv, maps, tau)
    for h in range(H):
        n = int(maps["d_h"][h])
        U, W = np.asarray(maps["U"][h])[:, :n], np.asarray(maps["W"][h])[:, :n]
        O[:, h] = O[:, h] @ W @ U.T
    return O, L


_orig_maps = orc.lowdim_maps


def _maps_ascending(D, H, d):
    return _orig_maps(D, H, d)[:, :, ::-1]


def _routed_reduces_full_set(q, ck, cv, hk, hv, full_mask, full_heads=None, k_cur=None, v_cur=None, tau=None,
                             lowdim=None):
    if lowdim is None:
        return _orig_routed(q, ck, cv, hk, hv, full_mask, full_heads, k_cur, v_cur, tau)
    return _orig_routed(q, ck, cv, hk, hv, np.zeros_like(np.asarray(full_mask, bool)), full_heads, k_cur, v_cur,
                        tau, lowdim)


_orig_kmeans = orc.kmeans
_orig_pca = orc.joint_pca


def _kmeans_sums(x, init_centers, rounds):
    c = np.array(init_centers, dtype=np.float64, copy=True)
    for _ in range(rounds):
        ids = orc.assign(x, c)
        for j in range(c.shape[0]):
            if (ids == j).any():
                c[j] = x[ids == j].sum(axis=0)
    return c, orc.assign(x, c)


def _kmeans_assigns_once(x, init_centers, rounds):
    c = np.array(init_centers, dtype=np.float64, copy=True)
    ids = orc.assign(x, c)
    for _ in range(rounds):
        for j in range(c.shape[0]):
            if (ids == j).any():
                c[j] = x[ids == j].mean(axis=0)
    return c, orc.assign(x, c)


def _kmeans_empty_to_zero(x, init_centers, rounds):
    c = np.array(init_centers, dtype=np.float64, copy=True)
    for _ in range(rounds):
        ids = orc.assign(x, c)
        for j in range(c.shape[0]):
            c[j] = x[ids == j].mean(axis=0) if (ids == j).any() else 0.0
    return c, orc.assign(x, c)


def _pca_ascending(x, centers, ids, r):
    rho = x - centers[ids]
    w, v = np.linalg.eigh(rho.T @ rho / x.shape[0])
    return orc.sign_fixed(v[:, :r]), w[:r]


def _pca_of_raw_tokens(x, centers, ids, r):
    return _orig_pca(x, np.zeros_like(centers), ids, r)


def _pca_no_sign_rule(x, centers, ids, r):
    rho = x - centers[ids]
    w, v = np.linalg.eigh(rho.T @ rho / x.shape[0])
    order = np.argsort(-w)[:r]
    return -orc.sign_fixed(v[:, order]), w[order]


MUTANTS = {
    "kmeans_sums": ("kmeans", _kmeans_sums),
    "kmeans_assigns_once": ("kmeans", _kmeans_assigns_once),
    "kmeans_empty_to_zero": ("kmeans", _kmeans_empty_to_zero),
    "pca_ascending": ("joint_pca", _pca_ascending),
    "pca_of_raw_tokens": ("joint_pca", _pca_of_raw_tokens),
    "pca_no_sign_rule": ("joint_pca", _pca_no_sign_rule),
    "reduced_swaps_maps": ("attend_reduced", _reduced_swaps_maps),
    "reduced_trailing_columns": ("attend_reduced", _reduced_trailing_columns),
    "reduced_rescales_tau": ("attend_reduced", _reduced_rescales_tau),
    "reduced_restores_with_key_map": ("attend_reduced", _reduced_restores_with_key_map),
    "maps_ascending": ("lowdim_maps", _maps_ascending),
    "routed_reduces_full_set": ("attend_routed", _routed_reduces_full_set),
    "routed_drops_low_tokens": ("attend_routed", _routed_drops_low_tokens),
    "routed_kept_heads_skip_current": ("attend_routed", _routed_kept_heads_skip_current),
    "encode_projects_from_first_center": ("encode", _encode_projects_from_first_center),
    "encode_codes_from_unrounded_scale": ("encode", _encode_codes_from_unrounded_scale),
    "encode_returns_unquantised": ("encode", _encode_returns_unquantised),
    "encode_scale_from_residual": ("encode", _encode_scale_from_residual),
    "decode_no_center": ("decode", _decode_no_center),
    "decode_no_scale": ("decode", _decode_no_scale),
    "quantise_half_up": ("quantise", _quantise_floor),
    "scale_unrounded": ("scale_of", _scale_unrounded),
    "assign_argmax": ("assign", _assign_argmax),
    "project_no_center": ("project", _project_no_center),
    "merge_hard_max": ("lse_merge", _merge_max),
    "pack_nibbles_swapped": ("pack_codes", _pack_swapped),
    "low_value_uses_key_scale": ("attend_low", _low_wrong_value_scale),
    "low_drops_key_center": ("attend_low", _low_no_key_center),
    "softmax_wrong_tau": ("softmax_attention", _softmax_no_tau),
}


def test_pins_pass_unmutated():
    assert _run_pins() == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(orc, attr, fn)
    assert _run_pins(), f"no pin catches mutant {name}"
