"""Pins of the fp64 oracle to things other than itself: hand-worked cases, pure
Python brute force, library routines, closed forms, algebraic invariants and
the pages' printed tables.  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import nanokv_oracle as orc

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _rand_codec(rng, H, d, r, C, T):
    J = H * d
    ck = {"centers": rng.standard_normal((C, J)), "D": rng.standard_normal((J, r)) / math.sqrt(r)}
    cv = {"centers": rng.standard_normal((C, J)), "D": rng.standard_normal((J, r)) / math.sqrt(r)}

    def hist():
        return {"ids": rng.integers(0, C, T), "codes": rng.integers(-7, 8, (T, r)),
                "scales": rng.uniform(0.05, 0.6, T)}
    return ck, cv, hist(), hist()


# --------------------------------------------------------------------------
# assignment
# --------------------------------------------------------------------------

def test_assign_matches_python_loop():
    rng = np.random.default_rng(11)
    x = rng.standard_normal((9, 5))
    cen = rng.standard_normal((4, 5))
    cen[3] = cen[1]                      # duplicate center: tie -> lowest index
    x[0] = cen[1] + 1e-3
    want = []
    for t in range(9):
        best, bj = None, None
        for j in range(4):
            dd = sum((float(x[t, i]) - float(cen[j, i])) ** 2 for i in range(5))
            if best is None or dd < best:
                best, bj = dd, j
        want.append(bj)
    assert list(orc.assign(x, cen)) == want
    assert orc.assign(x, cen)[0] == 1


def test_assign_recovers_generator_labels():
    from synth.gen import WORKLOADS, make_codec, make_tokens, scaled, _gen
    w = scaled(WORKLOADS["full"], T=300, Tq=8)
    g = _gen(123, "cpu")
    codec = make_codec(w, g, "cpu")
    x, labels = make_tokens(w, codec, 300, g, "cpu")
    cen = orc.f64(codec["centers"])
    xx = orc.f64(x)
    assert np.array_equal(orc.assign(xx, cen), labels.numpy())
    assert not orc.argmin_ties(xx, cen).any()


# --------------------------------------------------------------------------
# INT4 coefficients
# --------------------------------------------------------------------------

def test_int4_hand_picked_cases():
    g = _load("int4_cases.json")
    for c in g["cases"]:
        y = np.array([c["y"]], dtype=np.float64)
        s = orc.scale_of(y, c["scale_dtype"])
        assert s[0] == c["scale"], c
        assert list(orc.quantise(y, s)[0]) == c["codes"], c
    codes = np.array([g["pack"]["codes"]])
    packed = orc.pack_codes(codes)
    assert list(packed[0]) == g["pack"]["bytes"]
    assert np.array_equal(orc.unpack_codes(packed), codes)


def test_encode_worked_example():
    """The whole encode (assign, project, scale, quantise, pack) on five tokens
    worked by hand: an argmin tie, half-steps on both sides of zero, a zero
    residual, and a token whose fp16-rounded scale moves a code."""
    g = _load("encode_worked.json")
    x, cen, E = (np.array(g[k], dtype=np.float64) for k in ("x", "centers", "E"))
    r = orc.encode(x, cen, E, g["scale_dtype"])
    assert r["ids"].tolist() == g["ids"]
    assert np.array_equal(r["y"], np.array(g["y"], dtype=np.float64))
    assert r["scales"].tolist() == g["scales"]
    assert r["codes"].tolist() == g["codes"]
    assert orc.pack_codes(r["codes"]).tolist() == g["packed"]
    assert orc.argmin_ties(x, cen).tolist() == g["argmin_tie"]
    s = r["scales"]
    assert orc.rounding_ties(x, cen, r["ids"], E, r["y"], s).tolist() == g["rounding_tie"]
    assert orc.scale_ties(r["y"], g["scale_dtype"]).tolist() == g["scale_tie"]


def test_int4_clamp_and_zero_scale():
    y = np.array([[10.0, -10.0, 0.2]])
    assert list(orc.quantise(y, np.array([1.0]))[0]) == [7, -7, 0]
    assert list(orc.quantise(y, np.array([0.0]))[0]) == [0, 0, 0]


def test_pack_roundtrip_all_nibbles():
    vals = np.arange(-8, 8)
    codes = np.array(np.meshgrid(vals, vals)).reshape(2, -1).T.reshape(-1, 2)
    assert np.array_equal(orc.unpack_codes(orc.pack_codes(codes)), codes)


# --------------------------------------------------------------------------
# codec round trip (invariant: unquantised full-rank orthonormal D is exact)
# --------------------------------------------------------------------------

def test_orthonormal_full_rank_roundtrip():
    rng = np.random.default_rng(5)
    J, C, T = 24, 3, 40
    D = np.linalg.qr(rng.standard_normal((J, J)))[0]
    E = D.T
    cen = rng.standard_normal((C, J))
    x = cen[rng.integers(0, C, T)] + 0.3 * rng.standard_normal((T, J))
    ids = orc.assign(x, cen)
    y = orc.project(x, cen, ids, E)
    xhat = orc.decode(ids, y, np.ones(T), cen, D)
    assert np.max(np.abs(xhat - x)) < 1e-12


def test_decode_adds_center_and_scales_codes():
    cen = np.array([[1.0, 2.0], [-3.0, 0.5]])
    D = np.array([[1.0, 0.0, 2.0], [0.0, -1.0, 1.0]])     # J=2, r=3
    ids = np.array([1, 0])
    codes = np.array([[1, 2, -1], [0, 7, 3]])
    s = np.array([0.5, 0.25])
    want = np.array([[-3.0 + 0.5 * (1 - 2), 0.5 + 0.5 * (-2 - 1)],
                     [1.0 + 0.25 * (0 + 6), 2.0 + 0.25 * (-7 + 3)]])
    assert np.allclose(orc.decode(ids, codes, s, cen, D), want, rtol=0, atol=1e-15)


# --------------------------------------------------------------------------
# attention branches
# --------------------------------------------------------------------------

def _brute_full(q, ck, cv, hk, hv, tau):
    """Pure-Python loops: decode every key/value element, then softmax."""
    Tq, H, d = q.shape
    T = len(hk["ids"])
    r = ck["D"].shape[1]

    def dec(c, h, t, i):
        col = h * d + i
        acc = 0.0
        for j in range(r):
            acc += float(c["D"][col, j]) * float(h_["codes"][t][j])
        return float(c["centers"][h_["ids"][t], col]) + float(h_["scales"][t]) * acc

    O = np.zeros((Tq, H, d))
    L = np.zeros((H, Tq))
    for h in range(H):
        h_ = hk
        K = [[dec(ck, h, t, i) for i in range(d)] for t in range(T)]
        h_ = hv
        V = [[dec(cv, h, t, i) for i in range(d)] for t in range(T)]
        for a in range(Tq):
            z = [tau * sum(float(q[a, h, i]) * K[t][i] for i in range(d)) for t in range(T)]
            m = max(z)
            p = [math.exp(zz - m) for zz in z]
            l = sum(p)
            for i in range(d):
                O[a, h, i] = sum(p[t] * V[t][i] for t in range(T)) / l
            L[h, a] = m + math.log(l)
    return O, L


def test_full_branch_matches_python_loops():
    rng = np.random.default_rng(7)
    H, d, r, C, T, Tq = 2, 4, 3, 3, 7, 3
    ck, cv, hk, hv = _rand_codec(rng, H, d, r, C, T)
    q = rng.standard_normal((Tq, H, d))
    O, L = orc.attend_full(q, ck, cv, hk, hv, 0.7)
    Ob, Lb = _brute_full(q, ck, cv, hk, hv, 0.7)
    assert np.max(np.abs(O - Ob)) < 1e-12
    assert np.max(np.abs(L - Lb)) < 1e-12


def test_textbook_special_case_against_torch_sdpa():
    """C = 1 zero center, D = I (r = J): K_hat = s * code, so decode-attention
    is plain softmax attention; torch's SDPA (fp64, CPU) is the reference."""
    rng = np.random.default_rng(3)
    H, d, T, Tq = 3, 4, 11, 5
    J = H * d
    ck = {"centers": np.zeros((1, J)), "D": np.eye(J)}
    cv = {"centers": np.zeros((1, J)), "D": np.eye(J)}
    hk = {"ids": np.zeros(T, int), "codes": rng.integers(-7, 8, (T, J)), "scales": rng.uniform(0.1, 0.5, T)}
    hv = {"ids": np.zeros(T, int), "codes": rng.integers(-7, 8, (T, J)), "scales": rng.uniform(0.1, 0.5, T)}
    q = rng.standard_normal((Tq, H, d))
    tau = 1 / math.sqrt(d)
    O, L = orc.attend_full(q, ck, cv, hk, hv, tau)
    K = (hk["scales"][:, None] * hk["codes"]).reshape(T, H, d)
    V = (hv["scales"][:, None] * hv["codes"]).reshape(T, H, d)
    qt = torch.tensor(q).permute(1, 0, 2)[None]
    kt = torch.tensor(K).permute(1, 0, 2)[None]
    vt = torch.tensor(V).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=tau)[0].permute(1, 0, 2).numpy()
    assert np.max(np.abs(O - ref)) < 1e-12
    z = tau * torch.einsum("hqd,hkd->hqk", qt[0], kt[0])
    assert np.max(np.abs(L - torch.logsumexp(z, dim=-1).numpy())) < 1e-12


def test_all_keys_equal_gives_value_mean():
    rng = np.random.default_rng(4)
    H, d, r, C, T, Tq = 2, 3, 4, 5, 6, 2
    ck, cv, hk, hv = _rand_codec(rng, H, d, r, C, T)
    hk["ids"][:] = 2
    hk["codes"][:] = hk["codes"][0]
    hk["scales"][:] = 0.3
    q = rng.standard_normal((Tq, H, d))
    O, L = orc.attend_full(q, ck, cv, hk, hv, 1.0)
    vh = orc.decode(hv["ids"], hv["codes"], hv["scales"], cv["centers"], cv["D"]).reshape(T, H, d)
    assert np.max(np.abs(O - vh.mean(axis=0)[None])) < 1e-12
    kh = orc.decode(hk["ids"][:1], hk["codes"][:1], hk["scales"][:1], ck["centers"], ck["D"]).reshape(H, d)
    z = np.einsum("qhd,hd->hq", q, kh)
    assert np.max(np.abs(L - (z + math.log(T)))) < 1e-12


@pytest.mark.parametrize("tau", [1.0, 0.125])
def test_low_dim_equals_full_decode(tau):
    """Invariant: the mixed-dimensional branch is algebraically the
    full-decode branch on the same compressed data."""
    rng = np.random.default_rng(8)
    H, d, r, C, T, Tq = 3, 8, 6, 5, 50, 7
    ck, cv, hk, hv = _rand_codec(rng, H, d, r, C, T)
    q = rng.standard_normal((Tq, H, d))
    Of, Lf = orc.attend_full(q, ck, cv, hk, hv, tau)
    Ol, Ll = orc.attend_low(q, ck, cv, hk, hv, tau)
    assert np.max(np.abs(Of - Ol)) < 1e-12 * max(1.0, np.max(np.abs(Of)))
    assert np.max(np.abs(Lf - Ll)) < 1e-11


def test_lse_merge_of_split_history_equals_concatenation():
    rng = np.random.default_rng(9)
    H, d, T, Tq = 2, 5, 30, 6
    q = rng.standard_normal((Tq, H, d))
    k = rng.standard_normal((T, H, d))
    v = rng.standard_normal((T, H, d))
    full = orc.softmax_attention(q, k, v, 0.9)
    for cuts in ([12], [0, 12], [7, 19, 30]):
        bounds = [0] + cuts + [T]
        parts = [orc.softmax_attention(q, k[a:b], v[a:b], 0.9) for a, b in zip(bounds[:-1], bounds[1:])]
        O, L = orc.lse_merge(parts)
        assert np.max(np.abs(O - full[0])) < 1e-12
        assert np.max(np.abs(L - full[1])) < 1e-12


def test_lse_merge_closed_forms():
    rng = np.random.default_rng(10)
    O1 = rng.standard_normal((4, 2, 3))
    L1 = rng.standard_normal((2, 4))
    O, L = orc.lse_merge([(O1, L1)])
    assert np.array_equal(O, O1) or np.max(np.abs(O - O1)) < 1e-15
    assert np.max(np.abs(L - L1)) < 1e-15
    O2 = rng.standard_normal((4, 2, 3))
    O, L = orc.lse_merge([(O1, L1), (O2, L1.copy())])
    assert np.max(np.abs(O - (O1 + O2) / 2)) < 1e-15
    assert np.max(np.abs(L - (L1 + math.log(2)))) < 1e-14
    empty = (np.zeros_like(O1), np.full_like(L1, -np.inf))
    O, L = orc.lse_merge([empty, (O1, L1), empty])
    assert np.max(np.abs(O - O1)) < 1e-15 and np.max(np.abs(L - L1)) < 1e-15
    O, L = orc.lse_merge([empty, empty])
    assert np.all(O == 0) and np.all(np.isneginf(L))


def test_attend_routing_equals_one_big_attention():
    """attend() with any split point equals plain attention over the
    explicitly decoded history concatenated with the current chunk."""
    rng = np.random.default_rng(12)
    H, d, r, C, T, Tq = 2, 8, 6, 4, 40, 9
    ck, cv, hk, hv = _rand_codec(rng, H, d, r, C, T)
    q = rng.standard_normal((Tq, H, d))
    kc = rng.standard_normal((Tq, H, d))
    vc = rng.standard_normal((Tq, H, d))
    K = orc.decode(hk["ids"], hk["codes"], hk["scales"], ck["centers"], ck["D"]).reshape(T, H, d)
    V = orc.decode(hv["ids"], hv["codes"], hv["scales"], cv["centers"], cv["D"]).reshape(T, H, d)
    ref = orc.softmax_attention(q, np.concatenate([K, kc]), np.concatenate([V, vc]), 1 / math.sqrt(d))
    for T_full in (0, 1, 17, T):
        O, L = orc.attend(q, ck, cv, hk, hv, T_full, kc, vc)
        assert np.max(np.abs(O - ref[0])) < 1e-12, T_full
        assert np.max(np.abs(L - ref[1])) < 1e-12, T_full
    # no current chunk, empty history -> O = 0, LSE = -inf
    e = {"ids": hk["ids"][:0], "codes": hk["codes"][:0], "scales": hk["scales"][:0]}
    O, L = orc.attend(q, ck, cv, e, e, 0)
    assert np.all(O == 0) and np.all(np.isneginf(L))


# --------------------------------------------------------------------------
# tie accounting
# --------------------------------------------------------------------------

def test_tie_detectors():
    # fp16 midpoint: 7 * (1 + 2^-11) lies halfway between 1 and 1 + 2^-10
    y = np.array([[7 * (1 + 2 ** -11), 1.0], [7.0, 1.0]])
    assert list(orc.scale_ties(y, "f16")) == [True, False]
    x = np.array([[1.0, 0.0]])
    cen = np.array([[0.0, 0.0], [2.0, 0.0], [5.0, 5.0]])
    assert orc.argmin_ties(x, cen)[0]
    assert not orc.argmin_ties(np.array([[0.2, 0.0]]), cen)[0]
    E = np.eye(2)
    ids = np.array([0])
    yy = np.array([[2.5, 1.2]])
    t = orc.rounding_ties(np.array([[2.5, 1.2]]), np.zeros((1, 2)), ids, E, yy, np.array([1.0]))
    assert list(t[0]) == [True, False]


# --------------------------------------------------------------------------
# the pages' printed numbers: representation and arithmetic accounting
# --------------------------------------------------------------------------

def test_nominal_cr_matches_table5_table9():
    g = _load("codec_ranks.json")
    for row in g["rows"]:
        cr = orc.nominal_coefficient_cr(row["heads"], row["head_dim"], row["rank"])
        assert cr == row["budget"], row


def test_table11_product_rule():
    g = _load("fast_macs.json")
    for row in g["rows"]:
        prod = orc.overall_saving(row["historical_share"] / 100, row["history_saved"] / 100) * 100
        assert abs(prod - row["all_saved"]) < 0.006, row


def test_table6_head_layer_counts():
    g = _load("head_dims.json")
    for row in g["rows"]:
        assert sum(row["counts"]) == row["layers"] * row["heads"], row


# --------------------------------------------------------------------------
# routed attention (Table 7 policies) and the policy builder
# --------------------------------------------------------------------------

def _decoded_softmax(q, ck, cv, hk, hv, kc, vc, tau):
    """One textbook softmax over every decoded history key plus the current chunk."""
    Tq, H, d = q.shape
    kh = orc.decode(hk["ids"], hk["codes"], hk["scales"], ck["centers"], ck["D"]).reshape(-1, H, d)
    vh = orc.decode(hv["ids"], hv["codes"], hv["scales"], cv["centers"], cv["D"]).reshape(-1, H, d)
    return orc.softmax_attention(q, np.concatenate([kh, kc]), np.concatenate([vh, vc]), tau)


def test_routed_attention_equals_one_softmax():
    """Any token routing and any set of heads kept full-dim gives the attention
    over the concatenation of all keys (the low-dim branch only reorders the
    contraction; LSE merging recombines the branches)."""
    for seed in (0, 1, 2):
        rng = np.random.default_rng(seed)
        H, d, r, C, T, Tq, Tc = 3, 8, 6, 5, 40, 7, 6
        ck, cv, hk, hv = _rand_codec(rng, H, d, r, C, T)
        q = rng.standard_normal((Tq, H, d))
        kc, vc = rng.standard_normal((Tc, H, d)), rng.standard_normal((Tc, H, d))
        mask = rng.random(T) < 0.4
        heads = np.array([False, True, False]) if seed else None
        O, L = orc.attend_routed(q, ck, cv, hk, hv, mask, heads, kc, vc, tau=0.7)
        Or, Lr = _decoded_softmax(q, ck, cv, hk, hv, kc, vc, 0.7)
        assert np.allclose(O, Or, rtol=0, atol=1e-12) and np.allclose(L, Lr, rtol=0, atol=1e-12)


def test_routed_attention_recent_range_is_attend():
    """The fixed policy of the configs (the most recent T_full tokens) as a
    routing mask gives attend() with that T_full."""
    rng = np.random.default_rng(5)
    H, d, r, C, T, Tq = 2, 8, 6, 4, 30, 5
    ck, cv, hk, hv = _rand_codec(rng, H, d, r, C, T)
    q = rng.standard_normal((Tq, H, d))
    mask = np.zeros(T, dtype=bool)
    mask[T - 12:] = True
    O, L = orc.attend_routed(q, ck, cv, hk, hv, mask, tau=0.5)
    Or, Lr = orc.attend(q, ck, cv, hk, hv, 12, tau=0.5)
    assert np.allclose(O, Or, rtol=0, atol=1e-13) and np.allclose(L, Lr, rtol=0, atol=1e-13)


def test_frame_policy_ranges():
    """Hand-worked policies: 10 frames of 100 tokens, 4 recent, 1 sink, an
    anchor every 4 older frames -> frames {0, 4, 6, 7, 8, 9}; a partial last
    frame is clipped; the per-layer fallback reads everything full-dim."""
    from compressed_history_attention_b200.routing import frame_policy, full_mask
    assert frame_policy(1000, 100, recent=4, sinks=1, anchor_every=4) == [(0, 100), (400, 100), (600, 400)]
    assert frame_policy(950, 100, recent=4, sinks=1, anchor_every=4) == [(0, 100), (400, 100), (600, 350)]
    assert frame_policy(1000, 100, recent=2) == [(800, 200)]
    assert frame_policy(1000, 100, sinks=3, recent=2) == [(0, 300), (800, 200)]
    assert frame_policy(1000, 100, full_layer=True) == [(0, 1000)]
    assert frame_policy(0, 100, recent=2) == []
    m = full_mask([(0, 100), (400, 100), (600, 350)], 950)
    assert m.sum() == 550 and m[0] and not m[100] and m[949]


# --------------------------------------------------------------------------
# reduced attention dimension per head (Table 6; Fig. 4(d) reduce / restore;
# Table 8 analytical maps)
# --------------------------------------------------------------------------

def _orthonormal(rng, H, d):
    return np.stack([np.linalg.qr(rng.standard_normal((d, d)))[0] for _ in range(H)])


def _subspace_codec(rng, maps, n, d, r, C, T, key):
    """A codec whose decoder columns and centers lie, per head, in the span
    of the first n columns of that head's map (U for keys, W for values)."""
    H = maps.shape[0]
    D = np.concatenate([maps[h][:, :n] @ rng.standard_normal((n, r)) for h in range(H)])
    cen = np.concatenate([(maps[h][:, :n] @ rng.standard_normal((n, C))).T for h in range(H)], axis=1)
    hist = {"ids": rng.integers(0, C, T), "codes": rng.integers(-7, 8, (T, r)), "scales": rng.uniform(0.05, 0.6, T)}
    return {"centers": cen, "D": D}, hist


def test_reduced_at_full_dimension_is_full_attention():
    """d_h = d with any orthonormal maps: U^T q . U^T k = q . k and W W^T = I,
    so the reduced branch is the full-dim branch."""
    rng = np.random.default_rng(21)
    H, d, r, C, T, Tq = 3, 8, 6, 5, 30, 7
    ck, cv, hk, hv = _rand_codec(rng, H, d, r, C, T)
    q = rng.standard_normal((Tq, H, d))
    maps = {"U": _orthonormal(rng, H, d), "W": _orthonormal(rng, H, d), "d_h": [d] * H}
    O, L = orc.attend_reduced(q, ck, cv, hk, hv, maps, 0.6)
    Of, Lf = orc.attend_full(q, ck, cv, hk, hv, 0.6)
    assert np.allclose(O, Of, rtol=0, atol=1e-12) and np.allclose(L, Lf, rtol=0, atol=1e-12)


def test_reduced_is_exact_when_keys_and_values_live_in_the_maps():
    """Keys confined to span(U_h[:, :d_h]) and values to span(W_h[:, :d_h])
    (different subspaces, d_h < d, queries arbitrary): the reduction loses
    nothing, so attention at d_h equals full-dim attention."""
    rng = np.random.default_rng(22)
    H, d, r, C, T, Tq = 2, 12, 7, 4, 25, 6
    for n in (3, 5):
        U, W = _orthonormal(rng, H, d), _orthonormal(rng, H, d)
        ck, hk = _subspace_codec(rng, U, n, d, r, C, T, "k")
        cv, hv = _subspace_codec(rng, W, n, d, r, C, T, "v")
        q = rng.standard_normal((Tq, H, d))
        O, L = orc.attend_reduced(q, ck, cv, hk, hv, {"U": U, "W": W, "d_h": [n] * H}, 0.8)
        Of, Lf = orc.attend_full(q, ck, cv, hk, hv, 0.8)
        assert np.allclose(O, Of, rtol=0, atol=1e-11) and np.allclose(L, Lf, rtol=0, atol=1e-11)
        # and it is a real reduction: the same maps on an unconfined codec differ
        ck2, cv2, hk2, hv2 = _rand_codec(rng, H, d, r, C, T)
        O2, _ = orc.attend_reduced(q, ck2, cv2, hk2, hv2, {"U": U, "W": W, "d_h": [n] * H}, 0.8)
        Of2, _ = orc.attend_full(q, ck2, cv2, hk2, hv2, 0.8)
        assert np.abs(O2 - Of2).max() > 1e-3


def test_analytic_maps_are_the_decoder_principal_subspace():
    """The leading n columns of lowdim_maps span the top-n eigenvectors of
    D_h D_h^T (the symmetric eigensolver, another routine) for every n up to
    the rank, and each head's map is orthonormal."""
    rng = np.random.default_rng(23)
    H, d, r = 2, 10, 7
    D = rng.standard_normal((H * d, r)) * np.linspace(2.0, 0.3, r)[None, :]
    maps = orc.lowdim_maps(D, H, d)
    for h in range(H):
        Dh = D[h * d:(h + 1) * d]
        w, v = np.linalg.eigh(Dh @ Dh.T)
        v = v[:, np.argsort(w)[::-1]]
        assert np.allclose(maps[h].T @ maps[h], np.eye(d), atol=1e-12)
        for n in range(1, r + 1):
            P1 = maps[h][:, :n] @ maps[h][:, :n].T
            P2 = v[:, :n] @ v[:, :n].T
            assert np.allclose(P1, P2, atol=1e-9), (h, n)


def test_analytic_maps_are_exact_for_low_rank_decoders():
    """Decoders of rank n with centers in their column space: the analytical
    maps at d_h = n reproduce full-dim attention (Eckart-Young: the rank-n
    truncation of a rank-n decoder is the decoder)."""
    rng = np.random.default_rng(24)
    H, d, r, C, T, Tq, n = 2, 12, 8, 4, 20, 5, 4
    ck, hk = _subspace_codec(rng, _orthonormal(rng, H, d), n, d, r, C, T, "k")
    cv, hv = _subspace_codec(rng, _orthonormal(rng, H, d), n, d, r, C, T, "v")
    maps = {"U": orc.lowdim_maps(ck["D"], H, d), "W": orc.lowdim_maps(cv["D"], H, d), "d_h": [n] * H}
    q = rng.standard_normal((Tq, H, d))
    O, L = orc.attend_reduced(q, ck, cv, hk, hv, maps, 0.5)
    Of, Lf = orc.attend_full(q, ck, cv, hk, hv, 0.5)
    assert np.allclose(O, Of, rtol=0, atol=1e-11) and np.allclose(L, Lf, rtol=0, atol=1e-11)


def test_routed_with_reduced_heads():
    """Reduced heads read their low-dim tokens at d_h and their full-dim
    tokens full-dim: with keys/values confined to the maps' subspaces the
    whole call equals one softmax over every key; on an unconfined codec the
    reduced heads equal the LSE merge of full-dim attention over the routed
    tokens, reduced attention over the others and the current chunk, and the
    other heads are untouched."""
    rng = np.random.default_rng(25)
    H, d, r, C, T, Tq, Tc, n = 3, 12, 7, 4, 30, 5, 4, 5
    U, W = _orthonormal(rng, H, d), _orthonormal(rng, H, d)
    ck, hk = _subspace_codec(rng, U, n, d, r, C, T, "k")
    cv, hv = _subspace_codec(rng, W, n, d, r, C, T, "v")
    q = rng.standard_normal((Tq, H, d))
    kc, vc = rng.standard_normal((Tc, H, d)), rng.standard_normal((Tc, H, d))
    mask = rng.random(T) < 0.3
    lowdim = {"U": U, "W": W, "d_h": np.array([n, 0, n])}
    O, L = orc.attend_routed(q, ck, cv, hk, hv, mask, None, kc, vc, tau=0.7, lowdim=lowdim)
    Or, Lr = _decoded_softmax(q, ck, cv, hk, hv, kc, vc, 0.7)
    assert np.allclose(O, Or, rtol=0, atol=1e-11) and np.allclose(L, Lr, rtol=0, atol=1e-11)

    ck, cv, hk, hv = _rand_codec(rng, H, d, r, C, T)
    O, L = orc.attend_routed(q, ck, cv, hk, hv, mask, None, kc, vc, tau=0.7, lowdim=lowdim)
    O0, L0 = orc.attend_routed(q, ck, cv, hk, hv, mask, None, kc, vc, tau=0.7)
    f, l = np.nonzero(mask)[0], np.nonzero(~mask)[0]
    maps = {"U": U, "W": W, "d_h": [n] * H}
    Oe, Le = orc.lse_merge([orc.attend_full(q, ck, cv, orc.take_history(hk, f), orc.take_history(hv, f), 0.7),
                            orc.attend_reduced(q, ck, cv, orc.take_history(hk, l), orc.take_history(hv, l), maps, 0.7),
                            orc.softmax_attention(q, kc, vc, 0.7)])
    for h in (0, 2):
        assert np.allclose(O[:, h], Oe[:, h], rtol=0, atol=1e-12) and np.allclose(L[h], Le[h], rtol=0, atol=1e-12)
    assert np.array_equal(O[:, 1], O0[:, 1]) and np.array_equal(L[1], L0[1])
    assert np.abs(O[:, 0] - O0[:, 0]).max() > 1e-3


# --------------------------------------------------------------------------
# calibration: k-means centers and joint PCA (Tables 2, 5; Fig. 3(a))
# --------------------------------------------------------------------------

def test_kmeans_worked_example():
    g = _load("kmeans_worked.json")
    x, init = np.array(g["x"]), np.array(g["init"])
    for n in range(1, len(g["rounds"]) + 1):
        c, ids = orc.kmeans(x, init, n)
        assert np.allclose(c, np.array(g["rounds"][n - 1]["centers"]), rtol=0, atol=1e-12), n
        nxt = g["rounds"][min(n, len(g["rounds"]) - 1)]["ids"]
        assert ids.tolist() == nxt, n


def test_kmeans_single_center_is_the_mean():
    rng = np.random.default_rng(31)
    x = rng.standard_normal((50, 7))
    c, ids = orc.kmeans(x, rng.standard_normal((1, 7)), 1)
    assert np.allclose(c[0], x.mean(axis=0), rtol=0, atol=1e-14) and (ids == 0).all()


def test_kmeans_center_without_tokens_stays():
    rng = np.random.default_rng(32)
    x = rng.standard_normal((40, 5))
    init = np.stack([x[0], x[1], np.full(5, 1e3)])
    c, ids = orc.kmeans(x, init, 3)
    assert np.array_equal(c[2], init[2]) and not (ids == 2).any()


def test_kmeans_objective_never_increases_and_is_permutation_equivariant():
    rng = np.random.default_rng(33)
    x = np.concatenate([rng.standard_normal((60, 6)) + 4 * rng.standard_normal(6) for _ in range(4)])
    init = x[rng.choice(len(x), 5, replace=False)]
    prev = np.inf
    for n in range(6):
        c, ids = orc.kmeans(x, init, n)
        obj = ((x - c[ids]) ** 2).sum()
        assert obj <= prev + 1e-9
        prev = obj
    perm = np.array([3, 0, 4, 1, 2])
    c1, ids1 = orc.kmeans(x, init, 4)
    c2, ids2 = orc.kmeans(x, init[perm], 4)
    assert np.allclose(c2, c1[perm], rtol=0, atol=1e-12)
    assert np.array_equal(perm[ids2], ids1)


def test_joint_pca_eigenpairs_match_the_svd_of_the_residuals():
    """D's columns are orthonormal eigenvectors of the residual second moment,
    eigenvalues decreasing, equal to the squared singular values of
    rho / sqrt(N) (np.linalg.svd, another routine), and their span is the
    leading right-singular subspace; each column's largest entry is
    positive."""
    rng = np.random.default_rng(34)
    N, J, C, r = 200, 12, 3, 5
    x = rng.standard_normal((N, J)) * np.linspace(3.0, 0.2, J)[None, :]
    centers, ids = orc.kmeans(x, x[:C], 2)
    D, w = orc.joint_pca(x, centers, ids, r)
    rho = x - centers[ids]
    S = rho.T @ rho / N
    assert np.allclose(D.T @ D, np.eye(r), atol=1e-12)
    assert np.allclose(S @ D, D * w[None, :], atol=1e-10)
    assert (np.diff(w) <= 0).all()
    _, sv, vt = np.linalg.svd(rho / np.sqrt(N), full_matrices=False)
    assert np.allclose(w, sv[:r] ** 2, rtol=1e-10, atol=1e-12)
    assert np.allclose(D @ D.T, vt[:r].T @ vt[:r], atol=1e-9)
    for i in range(r):
        assert D[np.argmax(np.abs(D[:, i])), i] > 0


def test_calibrated_codec_is_exact_on_low_rank_residuals():
    """Tokens = a center + a residual in a rank-r subspace: k-means from the
    true centers keeps them, and the calibrated D reconstructs every residual
    exactly (x = c_a + D D^T (x - c_a))."""
    rng = np.random.default_rng(35)
    N, J, C, r = 120, 16, 3, 4
    true_c = 30 * rng.standard_normal((C, J))
    B = np.linalg.qr(rng.standard_normal((J, r)))[0]
    z = rng.integers(0, C, N)
    g = rng.standard_normal((N, r))
    g -= np.stack([g[z == j].mean(axis=0) for j in range(C)])[z]   # residuals of zero mean per cluster
    x = true_c[z] + g @ B.T
    cal = orc.calibrate(x, true_c, 2, r)
    assert np.array_equal(cal["ids"], z)
    rho = x - cal["centers"][cal["ids"]]
    assert np.allclose(rho @ cal["D"] @ cal["E"], rho, atol=1e-10)
    assert np.allclose(cal["E"], cal["D"].T)


def test_zero_residual_tie_rule_of_the_encode_comparison():
    """The encode comparison's rule for residuals within rounding of zero,
    checked on the CPU with encodes made by the oracle: tokens on a center
    are counted and may carry any codes under a scale at the rounding floor;
    a larger scale fails, and ordinary tokens are never counted."""
    import torch
    from compressed_history_attention_b200._lib import Hist
    from tests import _parity as P

    rng = np.random.default_rng(3)
    C, J, r = 8, 64, 8
    cen = orc.f64(torch.tensor(rng.standard_normal((C, J)), dtype=torch.bfloat16))
    E = orc.f64(torch.tensor(rng.standard_normal((r, J)) / np.sqrt(J), dtype=torch.bfloat16))
    x = np.concatenate([cen, cen[:2] + rng.standard_normal((2, J))])
    codec = {"centers": torch.tensor(cen), "E": torch.tensor(E)}
    xt = torch.tensor(x)
    ref = orc.encode(x, cen, E, "f16")

    def hist(scales, codes):
        return Hist(torch.tensor(ref["ids"].astype(np.uint8)), torch.tensor(orc.pack_codes(codes)),
                    torch.tensor(scales.astype(np.float16)))

    ties = P.check_encode(xt, codec, hist(ref["scales"], ref["codes"]), "f16")
    assert ties["zero_residual_ties"] == C  # the on-center tokens, not the others
    # on-center tokens with a scale at the fp16 floor and arbitrary codes pass
    s = ref["scales"].copy()
    s[:C] = 2.0 ** -24
    codes = ref["codes"].copy()
    codes[:C] = rng.integers(-7, 8, (C, r))
    P.check_encode(xt, codec, hist(s, codes), "f16")
    # a scale well above the rounding bound fails
    s[0] = 1e-2
    with pytest.raises(AssertionError):
        P.check_encode(xt, codec, hist(s, codes), "f16")
