"""Routed compressed-history attention (NanoKV-Fast, Table 7: sink, anchor and
recent frames read at full dimension, per-layer full fallback, heads kept at
full dimension) through the C ABI, against the oracle's routed attention on
the same compressed history."""
import math

import numpy as np
import pytest
import torch

import compressed_history_attention_b200 as nk
from compressed_history_attention_b200 import _lib
from compressed_history_attention_b200.routing import frame_policy, full_mask
from synth.gen import WORKLOADS, scaled
from tests import _parity as P

pytestmark = pytest.mark.gpu

CASES = {
    "mixed_small": scaled(WORKLOADS["mixed"], T=900, T_full=300, Tq=300),
    "long_small": scaled(WORKLOADS["long"], H=4, T=900, T_full=200, Tq=200),
    "tiny": WORKLOADS["tiny"],
}


def _case(name, heads_every):
    w = CASES[name]
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    ft = 64 if not w.fp32 else 16
    full = frame_policy(w.T, ft, recent=3, sinks=1, anchor_every=4)
    heads = [h % heads_every == 0 for h in range(w.H)] if heads_every else None
    return w, prob, ck, cv, hk, hv, full, heads


def _oracle(w, prob, hk, hv, full, heads):
    orc = P.orc
    return orc.attend_routed(orc.f64(prob["q"]), P.oracle_codec(prob["codec_k"]), P.oracle_codec(prob["codec_v"]),
                             P.oracle_hist(hk), P.oracle_hist(hv), full_mask(full, w.T), heads,
                             orc.f64(prob["k_cur"]), orc.f64(prob["v_cur"]), 1.0 / math.sqrt(w.d))


@pytest.mark.parametrize("name,heads_every", [("mixed_small", 0), ("mixed_small", 3), ("long_small", 0),
                                              ("long_small", 2), ("tiny", 0), ("tiny", 1)])
def test_routed_policy_matches_oracle(name, heads_every):
    """Sink + periodic anchors + recent frames full-dim, the rest low-dim; with
    some (or all) heads kept full-dim."""
    w, prob, ck, cv, hk, hv, full, heads = _case(name, heads_every)
    O, L = nk.nanokv_attend_routed(prob["q"], ck, cv, hk, hv, full, heads, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    nk.nanokv_check()
    Or, Lr = _oracle(w, prob, hk, hv, full, heads)
    P.compare_attn(O, L, Or, Lr, w.fp32)


def test_routed_runs_each_head_set_on_its_kernel():
    """With heads of both kinds: the routed tokens once on the full-dim kernel
    (all heads), the other tokens on the full-dim kernel for the kept heads and
    on the low-dim kernel for the others."""
    w, prob, ck, cv, hk, hv, full, heads = _case("mixed_small", 3)
    nk.nanokv_timing_read()
    nk.nanokv_attend_routed(prob["q"], ck, cv, hk, hv, full, heads, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    n = {k: v[1] for k, v in nk.nanokv_timing_read().items()}
    assert n["attend_full"] == 2 and n["attend_low"] == 1 and n["attend_dense"] == 1 and n["lse_merge"] == 1


@pytest.mark.parametrize("name", ["mixed_small", "long_small"])
def test_routed_recent_range_equals_attend(name):
    """The configs' fixed policy (the most recent T_full tokens) as one range,
    and the per-layer full fallback as [0, T): the same kernels on the same
    tokens in the same order as nanokv_attend, so equal bit for bit."""
    w = CASES[name]
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    for T_full in (w.T_full, w.T):
        ref = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, T_full, prob["k_cur"], prob["v_cur"])
        got = nk.nanokv_attend_routed(prob["q"], ck, cv, hk, hv, [(w.T - T_full, T_full)], None,
                                      prob["k_cur"], prob["v_cur"])
        torch.cuda.synchronize()
        assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])


def test_routed_mixed_heads_need_tensor_cores():
    """On the CUDA-core path, heads of both kinds in one call are refused
    (nothing launched); a policy without kept heads runs there."""
    w, prob, ck, cv, hk, hv, full, heads = _case("mixed_small", 3)
    prev = nk.nanokv_set_kernel_path(1)
    try:
        with pytest.raises(nk.NanoKVError) as e:
            nk.nanokv_attend_routed(prob["q"], ck, cv, hk, hv, full, heads, prob["k_cur"], prob["v_cur"])
        assert e.value.status == _lib.ERR_UNSUPPORTED
        O, L = nk.nanokv_attend_routed(prob["q"], ck, cv, hk, hv, full, None, prob["k_cur"], prob["v_cur"])
        torch.cuda.synchronize()
    finally:
        nk.nanokv_set_kernel_path(prev)
    Or, Lr = _oracle(w, prob, hk, hv, full, None)
    P.compare_attn(O, L, Or, Lr, False)


# --------------------------------------------------------------------------
# heads at a reduced attention dimension (Table 6; Fig. 4(d))
# --------------------------------------------------------------------------

def _maps(w, seed):
    from synth.gen import make_lowdim_maps
    m = make_lowdim_maps(w, seed, device="cuda")
    return m["U"], m["W"]


def _oracle_lowdim(U, W, d_h):
    return {"U": P.orc.f64(U), "W": P.orc.f64(W), "d_h": np.asarray(d_h)}


@pytest.mark.parametrize("name,dims,kept", [
    ("mixed_small", [32, 64, 96, 0], None),
    ("mixed_small", [96, 0, 32, 64], [1, 0, 0, 0]),
    ("long_small", [64, 32, 96, 64], None),
    ("long_small", [0, 96, 0, 32], [0, 0, 1, 0]),
])
def test_routed_reduced_heads_match_oracle(name, dims, kept):
    """Heads at d_h = 32, 64, 96 read their low-dim tokens through the maps,
    the others as usual (coefficient space, or kept full-dim), all merged
    with the routed full-dim tokens and the current chunk."""
    w, prob, ck, cv, hk, hv, full, _ = _case(name, 0)
    d_h = [dims[h % len(dims)] for h in range(w.H)]
    heads = None if kept is None else [bool(kept[h % len(kept)]) for h in range(w.H)]
    U, W = _maps(w, 7)
    ld = nk.nanokv_lowdim_prepare(ck, cv, U, W)
    O, L = nk.nanokv_attend_routed(prob["q"], ck, cv, hk, hv, full, heads, prob["k_cur"], prob["v_cur"],
                                   lowdim=ld, d_h=d_h)
    torch.cuda.synchronize()
    nk.nanokv_check()
    orc = P.orc
    Or, Lr = orc.attend_routed(orc.f64(prob["q"]), P.oracle_codec(prob["codec_k"]), P.oracle_codec(prob["codec_v"]),
                               P.oracle_hist(hk), P.oracle_hist(hv), full_mask(full, w.T), heads,
                               orc.f64(prob["k_cur"]), orc.f64(prob["v_cur"]), 1.0 / math.sqrt(w.d),
                               lowdim=_oracle_lowdim(U, W, d_h))
    P.compare_attn(O, L, Or, Lr, False)


def test_routed_reduced_launches():
    """One query reduction and one launch per width in use, on the low-dim
    tokens; the heads not reduced keep their low-dim kernel."""
    w, prob, ck, cv, hk, hv, full, _ = _case("mixed_small", 0)
    U, W = _maps(w, 8)
    ld = nk.nanokv_lowdim_prepare(ck, cv, U, W)
    d_h = [32, 32, 96, 0] * (w.H // 4)
    nk.nanokv_timing_read()
    nk.nanokv_attend_routed(prob["q"], ck, cv, hk, hv, full, None, prob["k_cur"], prob["v_cur"], lowdim=ld, d_h=d_h)
    torch.cuda.synchronize()
    n = {k: v[1] for k, v in nk.nanokv_timing_read().items()}
    assert n["attend_full"] == 1 and n["attend_low"] == 1 + 1 + 2 and n["attend_dense"] == 1


def test_lowdim_tables():
    """The mapped decoder rows U_h^T D_h and centers c_h U_h that the reduced
    heads decode through, against fp64 on the stored inputs (one bf16
    rounding of an fp32 sum)."""
    w = CASES["long_small"]
    prob = P.problem(w)
    ck, cv = P.gpu_codecs(w, prob)
    U, W = _maps(w, 9)
    ld = nk.nanokv_lowdim_prepare(ck, cv, U, W)
    torch.cuda.synchronize()
    H, d, r, C = w.H, w.d, w.r, w.C
    J = H * d
    aux = ld.aux
    nD = J * r * 2
    got = [aux[:nD].view(torch.bfloat16).view(J, r), aux[nD:2 * nD].view(torch.bfloat16).view(J, r),
           aux[2 * nD:2 * nD + C * J * 2].view(torch.bfloat16).view(C, J),
           aux[2 * nD + C * J * 2:2 * nD + 2 * C * J * 2].view(torch.bfloat16).view(C, J)]
    for br, (codec, M) in enumerate(((prob["codec_k"], U), (prob["codec_v"], W))):
        D = codec["D"].double().cpu().view(H, d, r)
        Mh = M.double().cpu()
        want_D = torch.einsum("hij,hik->hjk", Mh, D).reshape(J, r)
        cen = codec["centers"].double().cpu().view(C, H, d)
        want_c = torch.einsum("ahi,hij->ahj", cen, Mh).reshape(C, J)
        for g, want in ((got[br], want_D), (got[2 + br], want_c)):
            g = g.double().cpu()
            err = (g - want).abs()
            # one bf16 rounding (2^-9 relative) plus fp32 accumulation
            assert (err <= want.abs() * 2.0 ** -8 + 1e-4).all(), float(err.max())


@pytest.mark.parametrize("name", ["mixed_small", "long_small"])
def test_analytic_maps(name):
    """The GPU's analytical maps against the oracle's (fp64 SVD of the same
    stored decoder): the leading d_h columns span the same subspace, for
    d_h = 32, 64, 96, within the bf16 rounding of the maps plus the
    eigenvector error of an fp32 solver, which grows as the singular-value
    gap at d_h shrinks; every map is orthonormal to bf16 accuracy."""
    w = CASES[name]
    prob = P.problem(w)
    ck, cv = P.gpu_codecs(w, prob)
    orc = P.orc
    for c, codec in ((ck, prob["codec_k"]), (cv, prob["codec_v"])):
        maps = nk.nanokv_lowdim_analytic(c).double().cpu().numpy()
        torch.cuda.synchronize()
        D = orc.f64(codec["D"])
        ref = orc.lowdim_maps(D, w.H, w.d)
        for h in range(w.H):
            assert np.abs(maps[h].T @ maps[h] - np.eye(w.d)).max() < 1e-2
            sv = np.linalg.svd(D[h * w.d:(h + 1) * w.d], compute_uv=False)
            sv = np.concatenate([sv, np.zeros(w.d - len(sv))])
            for n in (32, 64, 96):
                gap = (sv[n - 1] ** 2 - sv[n] ** 2) / max(sv[0] ** 2, 1e-30)
                P1 = maps[h][:, :n] @ maps[h][:, :n].T
                P2 = ref[h][:, :n] @ ref[h][:, :n].T
                tol = 5e-3 + 1e-5 / max(gap, 1e-12)
                assert np.abs(P1 - P2).max() < tol, (h, n, gap, np.abs(P1 - P2).max())


def test_routed_many_ranges_and_empty_ones():
    """The largest policy the ABI takes: 64 ranges (single tokens spread over
    the history, some of count 0), against the oracle."""
    w, prob, ck, cv, hk, hv, _, _ = _case("mixed_small", 0)
    starts = np.linspace(0, w.T - 1, _lib.MAX_RANGES).astype(int)
    full = [(int(s), 0 if i % 7 == 3 else 1) for i, s in enumerate(starts)]
    O, L = nk.nanokv_attend_routed(prob["q"], ck, cv, hk, hv, full, None, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    Or, Lr = _oracle(w, prob, hk, hv, full, None)
    P.compare_attn(O, L, Or, Lr, False)


def test_routed_reduced_heads_without_low_tokens():
    """With every history token routed full-dim, heads at reduced dimensions
    have nothing to reduce: the call equals nanokv_attend with T_full = T
    bit for bit."""
    w, prob, ck, cv, hk, hv, _, _ = _case("mixed_small", 0)
    U, W = _maps(w, 12)
    ld = nk.nanokv_lowdim_prepare(ck, cv, U, W)
    d_h = [32, 64, 96, 0] * (w.H // 4)
    got = nk.nanokv_attend_routed(prob["q"], ck, cv, hk, hv, [(0, w.T)], None, prob["k_cur"], prob["v_cur"],
                                  lowdim=ld, d_h=d_h)
    ref = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, w.T, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
