"""The library calls behind the sharded attention, on one GPU: the fp32
partial of nanokv_attend_partial against the oracle, and the history and
head shards of several ranks computed one after another (the ranks' kernels
do not wait on one another) and combined as the sharded path combines
them, against the oracle's attention over the whole history."""
import math

import numpy as np
import pytest
import torch

import compressed_history_attention_b200 as nk
from compressed_history_attention_b200 import sharded
from synth.gen import WORKLOADS, scaled
from tests import _parity as P

pytestmark = pytest.mark.gpu

W = {"mixed_small": scaled(WORKLOADS["mixed"], T=900, T_full=300, Tq=300),
     "long_small": scaled(WORKLOADS["long"], H=4, T=900, T_full=200, Tq=200)}


def _setup(name):
    w = W[name]
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    return w, prob, ck, cv, hk, hv


@pytest.mark.parametrize("name", sorted(W))
def test_attend_partial_matches_oracle(name):
    w, prob, ck, cv, hk, hv = _setup(name)
    O, L = nk.nanokv_attend_partial(prob["q"], ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    assert O.dtype == torch.float32
    Or, Lr = P.oracle_attend(w, prob, hk, hv, w.T_full)
    P.compare_attn(O, L, Or, Lr, False)


@pytest.mark.parametrize("name,world", [("mixed_small", 2), ("mixed_small", 3), ("long_small", 2)])
def test_history_shards_merged(name, world):
    """Each rank's range (routed by the global T_full, the current chunk on
    rank 0) as an fp32 partial, then the LSE merge of the partials."""
    w, prob, ck, cv, hk, hv = _setup(name)
    parts = [sharded.history_partial(prob["q"], ck, cv, hk, hv, w.T, w.T_full, prob["k_cur"], prob["v_cur"],
                                     world, r) for r in range(world)]
    O, L = nk.nanokv_lse_merge([p[0] for p in parts], [p[1] for p in parts], out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    nk.nanokv_check()
    Or, Lr = P.oracle_attend(w, prob, hk, hv, w.T_full)
    P.compare_attn(O, L, Or, Lr, False)


def test_head_shards_gathered():
    """Each rank's heads through sub-codecs (the heads' decoder rows and
    center columns), concatenated along the head axis."""
    w, prob, ck, cv, hk, hv = _setup("mixed_small")
    ops = sharded.LibraryOps()
    tau = 1.0 / math.sqrt(w.d)
    outs, lses = [], []
    for r in range(3):
        h0, h1 = sharded.head_shard(w.H, 3, r)
        sub = lambda x: x[:, h0:h1].contiguous()  # noqa: E731
        O, L = ops.attend(sub(prob["q"]), ops.head_codec(ck, h0, h1), ops.head_codec(cv, h0, h1), hk, hv,
                          w.T_full, sub(prob["k_cur"]), sub(prob["v_cur"]), tau)
        outs.append(O)
        lses.append(L)
    torch.cuda.synchronize()
    Or, Lr = P.oracle_attend(w, prob, hk, hv, w.T_full)
    P.compare_attn(torch.cat(outs, dim=1), torch.cat(lses, dim=0), Or, Lr, False)
