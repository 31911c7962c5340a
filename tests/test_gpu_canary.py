"""Out-of-bounds write checks for the CUDA path, standing in for a memory
sanitizer (not available on these GPUs): every output, and the attend
workspace, is a view into a larger buffer whose tail holds a known byte
pattern; after a call on ragged sizes the tails must be unchanged."""
import pytest
import torch

import compressed_history_attention_b200 as nk
from synth.gen import WORKLOADS, scaled
from tests import _parity as P

pytestmark = pytest.mark.gpu

PAD = 4096        # canary bytes after each buffer
PATTERN = 0xA5

CASES = {
    # 2-CTA encode / low-dim + full-dim + current chunk
    "mixed": scaled(WORKLOADS["mixed"], T=333, T_full=201, Tq=129),
    # full-dim only
    "full": scaled(WORKLOADS["full"], T=333, T_full=333, Tq=129),
    # multi-pass encode; low-dim tokens routed to the full-dim kernel
    "long": scaled(WORKLOADS["long"], H=4, T=333, T_full=77, Tq=129),
}


def _padded(nbytes, device):
    return torch.full((nbytes + PAD,), PATTERN, dtype=torch.uint8, device=device)


def _tail_intact(buf, nbytes):
    return bool((buf[nbytes:] == PATTERN).all())


@pytest.mark.parametrize("name", sorted(CASES))
def test_encode_writes_stay_in_bounds(name):
    w = CASES[name]
    prob = P.problem(w)
    ck, cv = P.gpu_codecs(w, prob)
    T = 300  # 2 tiles of 128 tokens + 44
    xk, xv = prob["hist_k"][:T], prob["hist_v"][:T]
    dev = xk.device
    outs, bufs = [], []
    for c in (ck, cv):
        sb = torch.empty(0, dtype=c.scale_dtype).element_size()
        n_ids, n_codes, n_sc = T, T * (c.r // 2), T * sb
        b_ids, b_codes, b_sc = _padded(n_ids, dev), _padded(n_codes, dev), _padded(n_sc, dev)
        outs.append(nk.Hist(b_ids[:n_ids], b_codes[:n_codes].view(T, c.r // 2), b_sc[:n_sc].view(c.scale_dtype)))
        bufs += [(b_ids, n_ids), (b_codes, n_codes), (b_sc, n_sc)]
    nk.nanokv_encode(ck, cv, xk, xv, out_k=outs[0], out_v=outs[1])
    torch.cuda.synchronize()
    nk.nanokv_check()
    for b, n in bufs:
        assert _tail_intact(b, n)
    # the views were written: same result as an encode into fresh buffers
    hk, hv = nk.nanokv_encode(ck, cv, xk, xv)
    torch.cuda.synchronize()
    for a, b in ((outs[0], hk), (outs[1], hv)):
        assert torch.equal(a.ids, b.ids) and torch.equal(a.codes, b.codes)
        assert torch.equal(a.scales.view(torch.uint8), b.scales.view(torch.uint8))


@pytest.mark.parametrize("name", sorted(CASES))
def test_attend_writes_stay_in_bounds(name):
    w = CASES[name]
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    q = prob["q"]
    Tq, H, d = q.shape
    dev = q.device
    need = nk.nanokv_attend_workspace(Tq, ck, cv, w.T, w.T_full, Tq)
    n_out, n_lse = Tq * H * d * q.element_size(), H * Tq * 4
    b_out, b_lse, b_ws = _padded(n_out, dev), _padded(n_lse, dev), _padded(need, dev)
    out = b_out[:n_out].view(q.dtype).view(Tq, H, d)
    lse = b_lse[:n_lse].view(torch.float32).view(H, Tq)
    O, L = nk.nanokv_attend(q, ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"],
                            out=out, lse=lse, workspace=b_ws[:need])
    torch.cuda.synchronize()
    nk.nanokv_check()
    assert _tail_intact(b_out, n_out)
    assert _tail_intact(b_lse, n_lse)
    assert _tail_intact(b_ws, need)
    O2, L2 = nk.nanokv_attend(q, ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    assert torch.equal(out, O2) and torch.equal(lse, L2)
