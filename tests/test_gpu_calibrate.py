"""Codec calibration on the GPU (k-means centers, joint PCA; Tables 2, 5;
Fig. 3(a)) through the C ABI, against the oracle's calibrate on the same
tokens and initial centers."""
import numpy as np
import pytest
import torch

import compressed_history_attention_b200 as nk
from synth.gen import WORKLOADS, make_problem, scaled
from tests import _parity as P

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": (WORKLOADS["tiny"], 3, 8),
    "small": (scaled(WORKLOADS["full"], H=4, T=1000, T_full=1000, Tq=64, C=16, rank=48), 3, 64),
    "full": (WORKLOADS["full"], 2, 192),
}


def _tokens(w):
    prob = make_problem(w, device="cuda")
    x, labels = prob["hist_k"][:min(w.T, 4680)], prob["labels_k"][:min(w.T, 4680)]
    # initial centers: the first token of each generating label (the
    # caller's choice; any C tokens would do)
    lab = labels.cpu().numpy()
    first = [int(np.nonzero(lab == j)[0][0]) for j in range(w.C)]
    return x.contiguous(), x[first].float().contiguous()


@pytest.mark.parametrize("name", sorted(CASES))
def test_calibrate_matches_oracle(name):
    w, rounds, r = CASES[name]
    x, init = _tokens(w)
    got = nk.nanokv_calibrate(x, init, rounds, r)
    torch.cuda.synchronize()
    orc = P.orc
    x64 = orc.f64(x)
    ref = orc.calibrate(x64, orc.f64(init), rounds, r)
    # the final assignment: equal except argmin ties at the oracle's centers
    ids = got["ids"].cpu().numpy().astype(np.int64)
    ties = orc.argmin_ties(x64, ref["centers"])
    assert ((ids == ref["ids"]) | ties).all(), int((ids != ref["ids"]).sum())
    # centers: fp32 means rounded to the storage dtype
    c = orc.f64(got["centers"])
    rel = 2.0 ** -24 if w.fp32 else 2.0 ** -8
    assert (np.abs(c - ref["centers"]) <= rel * np.abs(ref["centers"]) + 1e-5).all()
    # eigenvalues: fp32 second moment and fp32 rotations (each entry is
    # rotated ~2 J times per sweep; ~sqrt(that) roundings of 2^-24 |S|)
    lam = got["eigenvalues"].cpu().numpy().astype(np.float64)
    lam1 = ref["eigenvalues"][0]
    assert np.abs(lam - ref["eigenvalues"]).max() <= 5e-5 * lam1
    # eigenvectors: E = D^T exactly; a column whose eigenvalue is separated
    # from its neighbours matches the oracle's within the storage rounding
    # plus the solver's eigenvector error (~1e-6 lam1 / gap); every column is
    # an eigenvector of the oracle's second moment to the storage rounding;
    # each column's largest entry is positive
    D, E = orc.f64(got["D"]), orc.f64(got["E"])
    assert np.array_equal(D.T, E)
    rho = x64 - ref["centers"][ref["ids"]]
    S = rho.T @ rho / x64.shape[0]
    w_all = np.sort(np.linalg.eigvalsh(S))[::-1]
    eps = 2.0 ** -24 if w.fp32 else 2.0 ** -8
    for i in range(r):
        v = D[:, i]
        res = np.linalg.norm(S @ v - ref["eigenvalues"][i] * v)
        assert res <= (4 * eps + 1e-4) * lam1, (i, res)
        assert v.max() >= -v.min()          # the sign rule (decided in fp32, before rounding)
        gap = min(abs(w_all[i] - w_all[i + 1]) if i + 1 < len(w_all) else np.inf,
                  abs(w_all[i - 1] - w_all[i]) if i > 0 else np.inf) / lam1
        if gap > 1e-3:
            u = ref["D"][:, i]
            top = np.sort(np.abs(u))[::-1]
            # the sign follows the largest entry; where the two largest are
            # within rounding of each other either sign is correct
            err = np.abs(v - u).max() if top[1] < 0.98 * top[0] else min(np.abs(v - u).max(), np.abs(v + u).max())
            assert err <= 2 * eps * top[0] + 1e-6 / gap + 1e-5, (i, gap, err)


def test_calibrate_center_without_tokens_stays():
    """An initial center far from every token keeps its place (and no token
    is assigned to it), as in the oracle."""
    w, rounds, r = CASES["small"]
    x, init = _tokens(w)
    init[3] = 1e3
    got = nk.nanokv_calibrate(x, init, rounds, r)
    torch.cuda.synchronize()
    ids = got["ids"].cpu().numpy()
    assert not (ids == 3).any()
    assert torch.equal(got["centers"][3].float().cpu(), init[3].to(got["centers"].dtype).float().cpu())
    orc = P.orc
    ref = orc.calibrate(orc.f64(x), orc.f64(init), rounds, r)
    ties = orc.argmin_ties(orc.f64(x), ref["centers"])
    assert ((ids.astype(np.int64) == ref["ids"]) | ties).all()
