"""Failure detection on the GPU without a fault: a kernel waits on a barrier
that nothing arrives on, gives up after a short bounded wait exactly as the
attention and encode pipelines do, and the host reads the timeout from the
device error word.  The context stays usable afterwards."""
import pytest
import torch

import compressed_history_attention_b200 as nk
from compressed_history_attention_b200 import _lib
from synth.gen import WORKLOADS
from tests import _parity as P

pytestmark = pytest.mark.gpu


def test_bounded_wait_timeout_is_reported_and_cleared():
    nk.nanokv_check()  # start from a clean error word
    nk.nanokv_selftest_wait(limit_ms=20)
    with pytest.raises(_lib.NanoKVError) as ei:
        nk.nanokv_check()
    assert f"status {_lib.ERR_TIMEOUT}" in str(ei.value)
    nk.nanokv_check()  # the word was cleared by the read


def test_context_usable_after_timeout():
    nk.nanokv_selftest_wait(limit_ms=5)
    with pytest.raises(_lib.NanoKVError):
        nk.nanokv_check()
    w = WORKLOADS["tiny"]
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    O, L = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    nk.nanokv_check()
    Or, Lr = P.oracle_attend(w, prob, hk, hv, w.T_full)
    P.compare_attn(O, L, Or, Lr, w.fp32)
