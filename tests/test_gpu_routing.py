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
