"""Checkpoint and resume of the compressed history.  The history (ids,
codes, scales) and the codec parameters are the whole persistent state and
live in caller-owned buffers; they are saved to disk, loaded back, and must
be bit-identical, and (on the GPU) attention over the reloaded state must
equal attention over the original bit for bit."""
import numpy as np
import pytest
import torch

import compressed_history_attention_b200 as nk
from oracle import nanokv_oracle as orc
from synth.gen import WORKLOADS, make_problem, scaled


def _state_of(codecs, hists):
    st = {}
    for name, c in codecs.items():
        st[name] = {"H": c.H, "d": c.d, "centers": c.centers.cpu(), "D": c.D.cpu(), "E": c.E.cpu()}
    for name, h in hists.items():
        st[name] = {"ids": h.ids.cpu(), "codes": h.codes.cpu(), "scales": h.scales.cpu()}
    return st


def test_oracle_history_roundtrip(tmp_path):
    """The history the oracle encodes survives a save / load unchanged."""
    w = WORKLOADS["tiny"]
    prob = make_problem(w, device="cpu")
    codec = prob["codec_k"]
    ref = orc.encode(orc.f64(prob["hist_k"]), orc.f64(codec["centers"]), orc.f64(codec["E"]), "f32")
    path = tmp_path / "hist.npz"
    np.savez(path, ids=ref["ids"], codes=ref["codes"], scales=ref["scales"],
             centers=codec["centers"].numpy(), D=codec["D"].numpy(), E=codec["E"].numpy())
    back = np.load(path)
    for k in ("ids", "codes", "scales"):
        assert back[k].dtype == np.asarray(ref[k]).dtype
        assert np.array_equal(back[k], ref[k])
    for k in ("centers", "D", "E"):
        assert np.array_equal(back[k].view(np.uint8), codec[k].numpy().view(np.uint8))


@pytest.mark.gpu
def test_gpu_history_checkpoint_resume(tmp_path):
    w = scaled(WORKLOADS["mixed"], T=700, T_full=300, Tq=300)
    prob = make_problem(w, device="cuda")
    ck = nk.Codec(w.H, w.d, prob["codec_k"]["centers"], prob["codec_k"]["D"], prob["codec_k"]["E"])
    cv = nk.Codec(w.H, w.d, prob["codec_v"]["centers"], prob["codec_v"]["D"], prob["codec_v"]["E"])
    hk, hv = nk.nanokv_encode(ck, cv, prob["hist_k"], prob["hist_v"])
    args = (prob["q"],)
    O1, L1 = nk.nanokv_attend(*args, ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()

    path = tmp_path / "kv_state.pt"
    torch.save(_state_of({"ck": ck, "cv": cv}, {"hk": hk, "hv": hv}), path)
    st = torch.load(path)
    dev = prob["q"].device
    ck2, cv2 = (nk.Codec(st[n]["H"], st[n]["d"], st[n]["centers"].to(dev), st[n]["D"].to(dev), st[n]["E"].to(dev))
                for n in ("ck", "cv"))
    hk2, hv2 = (nk.Hist(st[n]["ids"].to(dev), st[n]["codes"].to(dev), st[n]["scales"].to(dev)) for n in ("hk", "hv"))
    for a, b in ((hk, hk2), (hv, hv2)):
        assert torch.equal(a.ids, b.ids) and torch.equal(a.codes, b.codes)
        assert torch.equal(a.scales.view(torch.uint8), b.scales.view(torch.uint8))
    O2, L2 = nk.nanokv_attend(*args, ck2, cv2, hk2, hv2, w.T_full, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    nk.nanokv_check()
    assert torch.equal(O1, O2) and torch.equal(L1, L2)
