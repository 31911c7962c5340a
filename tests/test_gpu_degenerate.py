"""Degenerate inputs of the method through the C ABI, against the fp64 oracle:
tokens that sit exactly on a cluster center (a zero residual: scale 0, codes
0), the zero token, a scaled center, and a history whose every token is one
center (every decoded key and value is that center, so the attention over
the history is the mean of identical values)."""
import numpy as np
import pytest
import torch

import compressed_history_attention_b200 as nk
from synth.gen import WORKLOADS, scaled
from tests import _parity as P

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": WORKLOADS["tiny"],
    "full_small": scaled(WORKLOADS["full"], T=700, T_full=700, Tq=300),
    "mixed_small": scaled(WORKLOADS["mixed"], T=700, T_full=300, Tq=300),
    "long_small": scaled(WORKLOADS["long"], H=4, T=900, T_full=200, Tq=200),
}
PATHS = {"auto": 0, "simt": 1}


@pytest.fixture(params=sorted(PATHS))
def path(request):
    prev = nk.nanokv_set_kernel_path(PATHS[request.param])
    yield request.param
    nk.nanokv_set_kernel_path(prev)


def _sd(w):
    return "f32" if w.fp32 else "f16"


def _degenerate_tokens(cen: torch.Tensor) -> torch.Tensor:
    """Every center, the zero token, and center 0 scaled by 8 (powers of two
    keep the stored values exact)."""
    rows = [cen, torch.zeros_like(cen[:1]), cen[:1] * 8]
    return torch.cat(rows).contiguous()


@pytest.mark.parametrize("name", sorted(CASES))
def test_encode_tokens_on_centers(name, path):
    w = CASES[name]
    prob = P.problem(w)
    ck, cv = P.gpu_codecs(w, prob)
    xk = _degenerate_tokens(prob["codec_k"]["centers"])
    xv = _degenerate_tokens(prob["codec_v"]["centers"])
    hk, hv = nk.nanokv_encode(ck, cv, xk, xv)
    torch.cuda.synchronize()
    for x, c, h in ((xk, prob["codec_k"], hk), (xv, prob["codec_v"], hv)):
        ties = P.check_encode(x, c, h, _sd(w))
        C = c["centers"].shape[0]
        ids = h.ids.cpu().numpy().astype(np.int64)
        # a token on center j is nearest to it (the generator's centers are distinct)
        assert np.array_equal(ids[:C], np.arange(C)), ids[:C]
        # the oracle's residual is exactly zero for them: counted as
        # residuals within rounding of zero, whose scales check_encode has
        # held within the rounding bound
        assert ties["zero_residual_ties"] >= C, ties
        if path == "simt":
            # the CUDA-core encode forms E (x - c_a) itself: exactly zero,
            # so scale 0 and codes 0 as the oracle gives
            assert np.all(P.orc.f64(h.scales)[:C] == 0)
            assert np.all(P.orc.unpack_codes(h.codes.cpu().numpy())[:C] == 0)


@pytest.mark.parametrize("name", ["full_small", "mixed_small", "long_small"])
def test_attend_history_of_one_center(name, path):
    """Every history token is center 0 of its branch: K_hat = c_K[0] and
    V_hat = c_V[0] for every key, so the history's part of the attention
    output is c_V[0] and the whole matches the oracle."""
    w = CASES[name]
    prob = P.problem(w)
    ck, cv = P.gpu_codecs(w, prob)
    T = w.T
    prob["hist_k"] = prob["codec_k"]["centers"][:1].expand(T, -1).contiguous()
    prob["hist_v"] = prob["codec_v"]["centers"][:1].expand(T, -1).contiguous()
    hk, hv = nk.nanokv_encode(ck, cv, prob["hist_k"], prob["hist_v"])
    O, L = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    Or, Lr = P.oracle_attend(w, prob, hk, hv, w.T_full)
    P.compare_attn(O, L, Or, Lr, w.fp32)
    # the history alone (no current chunk): every output row is c_V[0]
    Oh, Lh = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, w.T_full, None, None)
    torch.cuda.synchronize()
    cv0 = P.orc.f64(prob["codec_v"]["centers"][0]).reshape(w.H, w.d)
    err = np.abs(P.orc.f64(Oh) - cv0[None])
    assert err.max() <= 2e-2 * max(1.0, np.abs(cv0).max()), err.max()


@pytest.mark.parametrize("name", ["tiny", "full_small", "mixed_small", "long_small"])
def test_attend_zero_queries(name, path):
    """q = 0 scores every key 0: the weights are uniform over the T history
    keys and the current chunk's keys, so LSE = ln(T + T_cur) exactly and O
    is the oracle's mean of the values."""
    w = CASES[name]
    prob = P.problem(w)
    prob["q"] = torch.zeros_like(prob["q"])
    ck, cv, hk, hv = P.encode_history(w, prob)
    O, L = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    n = w.T + prob["k_cur"].shape[0]
    lse = P.orc.f64(L)
    assert np.abs(lse - np.log(n)).max() <= (1e-5 if w.fp32 else 2e-3) * max(1.0, np.log(n))
    Or, Lr = P.oracle_attend(w, prob, hk, hv, w.T_full)
    P.compare_attn(O, L, Or, Lr, w.fp32)


# The widest codec the ABI takes (H = 256 heads of d = 128: J = 32768) and
# the largest rank with the most centers (r = 512, C = 256), which no
# tensor-core kernel covers: both kernel families, encode and attend.
EXTREMES = {
    "widest": scaled(WORKLOADS["mixed"], H=256, C=16, r=64, rank=48, T=256, T_full=128, Tq=64),
    "max_rank": scaled(WORKLOADS["mixed"], H=8, C=256, r=512, rank=160, T=300, T_full=100, Tq=64),
}


@pytest.mark.parametrize("name", sorted(EXTREMES))
def test_extreme_codec_shapes(name, path):
    w = EXTREMES[name]
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    torch.cuda.synchronize()
    for x, c, h in ((prob["hist_k"], prob["codec_k"], hk), (prob["hist_v"], prob["codec_v"], hv)):
        P.check_encode(x, c, h, _sd(w))
    O, L = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    Or, Lr = P.oracle_attend(w, prob, hk, hv, w.T_full)
    P.compare_attn(O, L, Or, Lr, w.fp32)
