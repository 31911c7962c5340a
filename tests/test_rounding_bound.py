"""The per-element error bound that the tensor-core parity checks use for the
tau = 1 stress case (tests/_parity.rounding_bound) covers a numpy simulation
of that path's bf16 rounding points, on a small problem with unit-variance
queries.  CPU only; the oracle gives the exact result."""
import math

import numpy as np
import torch

from oracle import nanokv_oracle as orc
from tests import _parity as P

LOG2E = 1.0 / math.log(2.0)


def _bf16(x):
    return torch.from_numpy(np.asarray(x, np.float64)).to(torch.float32).to(torch.bfloat16).double().numpy()


def _problem(seed=0, H=2, d=32, r=32, C=8, T=240, T_full=112, Tc=64, R=24):
    rng = np.random.default_rng(seed)
    J = H * d

    def codec():
        D = _bf16(np.linalg.qr(rng.standard_normal((J, r)))[0])
        return {"centers": _bf16(rng.standard_normal((C, J))), "D": D, "E": D.T.copy()}

    ck, cv = codec(), codec()

    def hist(c):
        x = c["centers"][rng.integers(0, C, T)] + rng.standard_normal((T, J)) * 0.7
        e = orc.encode(_bf16(x), c["centers"], c["E"], "f16")
        return {"ids": e["ids"], "codes": e["codes"], "scales": e["scales"]}

    hk, hv = hist(ck), hist(cv)
    q = _bf16(rng.standard_normal((R, H, d)))
    kc, vc = _bf16(rng.standard_normal((Tc, H, d))), _bf16(rng.standard_normal((Tc, H, d)))
    return q, ck, cv, hk, hv, kc, vc, T_full


def _simulated(q, ck, cv, hk, hv, kc, vc, T_full, tau):
    """The tensor-core path's arithmetic with its bf16 roundings (fp64 elsewhere)."""
    R, H, d = q.shape
    T = len(hk["ids"])
    T_low = T - T_full
    zs = tau * LOG2E

    def full_dec(h, c):
        x = np.asarray(h["codes"][T_low:], np.float64) @ c["D"].T
        s = _bf16(h["scales"][T_low:])[:, None]
        return _bf16(s * _bf16(x) + c["centers"][h["ids"][T_low:]])

    kf, vf = full_dec(hk, ck), full_dec(hv, cv)
    ckl = np.asarray(hk["codes"][:T_low], np.float64)
    cvl = np.asarray(hv["codes"][:T_low], np.float64)
    O = np.zeros((R, H, d))
    L = np.zeros((H, R))
    for h in range(H):
        cols = slice(h * d, (h + 1) * d)
        qh = q[:, h, :]
        qred = _bf16(qh @ ck["D"][cols, :] * zs) / zs
        z_low = tau * (hk["scales"][:T_low][None, :] * (qred @ ckl.T) + qh @ ck["centers"][hk["ids"][:T_low], cols].T)
        z_full = tau * qh @ kf[:, cols].T
        z_cur = tau * qh @ kc[:, h, :].T
        parts = []
        for z in (z_low, z_full, z_cur):
            m = z.max(axis=1, keepdims=True)
            p = np.exp(z - m)
            parts.append((m, p, p.sum(axis=1, keepdims=True)))
        (m0, p0, l0), (m1, p1, l1), (m2, p2, l2) = parts
        o_low = (_bf16((_bf16(p0 * hv["scales"][:T_low][None, :]) @ cvl) / l0) @ cv["D"][cols, :].T
                 + _bf16(_bf16(p0) @ np.eye(cv["centers"].shape[0])[hv["ids"][:T_low]] / l0) @ cv["centers"][:, cols])
        o_full = _bf16(p1) @ vf[:, cols] / l1
        o_cur = _bf16(p2) @ vc[:, h, :] / l2
        lse = np.concatenate([m0 + np.log(l0), m1 + np.log(l1), m2 + np.log(l2)], axis=1)
        wts = np.exp(lse - lse.max(axis=1, keepdims=True))
        L[h] = lse.max(axis=1) + np.log(wts.sum(axis=1))
        wts /= wts.sum(axis=1, keepdims=True)
        O[:, h, :] = wts[:, :1] * o_low + wts[:, 1:2] * o_full + wts[:, 2:] * o_cur
    return _bf16(O), L


def test_rounding_bound_covers_simulated_bf16_path():
    q, ck, cv, hk, hv, kc, vc, T_full = _problem()
    tau = 1.0
    O_ref, L_ref = orc.attend(q, ck, cv, hk, hv, T_full, kc, vc, tau)
    O_sim, L_sim = _simulated(q, ck, cv, hk, hv, kc, vc, T_full, tau)
    bound, lse_bound = P.rounding_bound(q, ck, cv, hk, hv, kc, vc, T_full, tau)
    err = np.abs(O_sim - O_ref)
    assert np.all(err <= bound), f"max err/bound {np.max(err / bound):.3f}"
    assert np.all(np.abs(L_sim - L_ref) <= lse_bound)
    # a worst case over rounding signs, yet the worst element reaches a
    # sizeable part of it: the bound is not vacuous
    assert np.max(err / bound) > 0.2
    assert np.median(bound) < 0.1
