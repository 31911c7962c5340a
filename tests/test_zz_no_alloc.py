"""The allocation-free attend entry point (for callers that cannot allocate
device memory) against the ordinary one, through the C ABI.  Collected last."""
import pytest
import torch

import compressed_history_attention_b200 as nk
from compressed_history_attention_b200 import _lib
from synth.gen import WORKLOADS, scaled
from tests import _parity as P

pytestmark = pytest.mark.gpu


def test_attend_static_matches_attend_on_two_calls():
    w = scaled(WORKLOADS["mixed"], T=700, T_full=300, Tq=300)
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    ref_O, ref_L = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    for _ in range(2):
        O = torch.full_like(prob["q"], float("nan"))
        L = torch.full((w.H, w.Tq), float("nan"), dtype=torch.float32, device="cuda")
        nk.nanokv_attend_static(prob["q"], ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"],
                                out=O, lse=L)
        torch.cuda.synchronize()
        # same kernels on the same inputs: compared with the attention tolerance
        P.compare_attn(O, L, P.orc.f64(ref_O), P.orc.f64(ref_L), False)


def test_attend_static_refuses_oversized_calls():
    # two branches of 4680 x 12 x 128 fp32 partials need ~58 MB of scratch
    w = scaled(WORKLOADS["full"], T=256, T_full=256, Tq=4680)
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    out = torch.empty_like(prob["q"])
    with pytest.raises(nk.NanoKVError) as e:
        nk.nanokv_attend_static(prob["q"], ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"], out=out)
    assert e.value.status == _lib.ERR_INVALID
    assert "32 MiB" in str(e.value)
