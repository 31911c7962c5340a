"""The allocation-free attend entry point against the ordinary one, through
the C ABI.  Some callers cannot allocate device memory: code that must not
enter the CUDA allocator (it can synchronise the device and takes process-wide
locks), or a plug-in that its host hands only input and output buffers.
nanokv_attend_static serves them from a fixed array inside the library.
Collected last, so that a failure here comes after every other test has run."""
import pytest
import torch

import compressed_history_attention_b200 as nk
from compressed_history_attention_b200 import _lib
from synth.gen import WORKLOADS, scaled
from tests import _parity as P

pytestmark = pytest.mark.gpu


def _case(w):
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    ref_O, ref_L = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"])
    O = torch.full_like(prob["q"], float("nan"))
    L = torch.full((w.H, w.Tq), float("nan"), dtype=torch.float32, device="cuda")
    return prob, ck, cv, hk, hv, ref_O, ref_L, O, L


def _static(w, case):
    prob, ck, cv, hk, hv, _, _, O, L = case
    nk.nanokv_attend_static(prob["q"], ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"], out=O, lse=L)


def test_attend_static_matches_attend_on_two_calls():
    # two different problems in a row: the second call reuses the array the
    # first one filled, so a read of its stale contents would show
    ws = [scaled(WORKLOADS["mixed"], T=700, T_full=300, Tq=300),
          scaled(WORKLOADS["mixed"], T=540, T_full=200, Tq=257)]
    cases = [_case(w) for w in ws]
    torch.cuda.synchronize()
    _static(ws[0], cases[0])  # warm-up: the first call looks up the array's address
    torch.cuda.synchronize()
    for w, c in zip(ws, cases):
        alloc0, free0 = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
        _static(w, c)
        torch.cuda.synchronize()
        assert torch.cuda.memory_allocated() == alloc0
        assert torch.cuda.mem_get_info()[0] == free0
        _, _, _, _, _, ref_O, ref_L, O, L = c
        # the same kernels on the same inputs, deterministic: equal bit for bit
        assert torch.equal(O, ref_O)
        assert torch.equal(L, ref_L)


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
