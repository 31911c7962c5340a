"""Helpers shared by the GPU parity tests: build GPU inputs from the seeded
generator, run the CUDA path through the C ABI, and compare with the oracle."""
from __future__ import annotations

import math

import numpy as np
import torch

import compressed_history_attention_b200 as nk
from oracle import nanokv_oracle as orc
from synth.gen import make_problem

# tolerances (attention outputs): bf16 I/O and the fp32 mode
TOL_BF16_MAXABS, TOL_BF16_RELL2, TOL_BF16_LSE = 2e-2, 5e-3, 2e-3
TOL_F32_MAXABS, TOL_F32_LSE = 1e-5, 1e-5


def gpu_codecs(w, prob):
    ck = nk.Codec(w.H, w.d, prob["codec_k"]["centers"], prob["codec_k"]["D"], prob["codec_k"]["E"])
    cv = nk.Codec(w.H, w.d, prob["codec_v"]["centers"], prob["codec_v"]["D"], prob["codec_v"]["E"])
    return ck, cv


def oracle_codec(c):
    return {"centers": orc.f64(c["centers"]), "D": orc.f64(c["D"]), "E": orc.f64(c["E"])}


def oracle_hist(h: nk.Hist, rows=None):
    ids = h.ids.cpu().numpy().astype(np.int64)
    codes = orc.unpack_codes(h.codes.cpu().numpy())
    scales = orc.f64(h.scales)
    return {"ids": ids, "codes": codes, "scales": scales}


def problem(w, device="cuda", layer=0):
    return make_problem(w, layer=layer, device=device)


def encode_history(w, prob):
    ck, cv = gpu_codecs(w, prob)
    hk, hv = nk.nanokv_encode(ck, cv, prob["hist_k"], prob["hist_v"])
    return ck, cv, hk, hv


def check_encode(x_gpu, codec, hist: nk.Hist, scale_dtype: str, sample=None):
    """Compares GPU encode outputs with the oracle: ids bit-exact except
    argmin ties; scales equal (fp16: except scale ties, where the neighbouring
    value is allowed; fp32: within 1e-6 relative); codes bit-exact under the
    stored scale except rounding ties.  Returns the tie counts."""
    idx = np.arange(x_gpu.shape[0]) if sample is None else np.asarray(sample)
    ti = torch.as_tensor(idx, device=x_gpu.device)
    x = orc.f64(x_gpu[ti])
    cen, E = orc.f64(codec["centers"]), orc.f64(codec["E"])
    ref = orc.encode(x, cen, E, scale_dtype)
    ids = hist.ids[ti].cpu().numpy().astype(np.int64)
    codes = orc.unpack_codes(hist.codes[ti].cpu().numpy())
    s = orc.f64(hist.scales[ti])

    tie_a = orc.argmin_ties(x, cen)
    bad_ids = (ids != ref["ids"]) & ~tie_a
    assert bad_ids.sum() == 0, f"{bad_ids.sum()} center ids differ outside ties (first {np.nonzero(bad_ids)[0][:5]})"
    same = ids == ref["ids"]

    # A residual within rounding of zero.  The tensor-core encode forms
    # y = E x - (E c)[a], algebraically E (x - c_a), from two fp32 sums of J
    # exact products each, which err by at most J 2^-23 (|E| |x| + |E| |c_a|)
    # per element.  Where every element of the exact y lies within that
    # bound (a token on its center, say), the arithmetic does not decide the
    # scale: it must stay within the bound's fp16 scale, and the codes (whose
    # contribution s * code is at the same noise level) are not compared.
    bnd = x.shape[1] * 2.0 ** -23 * ((np.abs(x) + np.abs(cen[ref["ids"]])) @ np.abs(E).T)
    zero_tie = np.all(np.abs(ref["y"]) <= bnd, axis=1)
    if zero_tie.any():
        cap = orc.round_to_storage(np.max(bnd, axis=1) / orc.QMAX, scale_dtype)
        cap = np.nextafter(cap.astype(np.float16 if scale_dtype == "f16" else np.float32), np.inf).astype(np.float64)
        big = zero_tie & same & (s > cap)
        assert big.sum() == 0, f"{big.sum()} near-zero residuals got a scale above the rounding bound"

    tie_s = orc.scale_ties(ref["y"], scale_dtype)
    if scale_dtype == "f16":
        eq = s == ref["scales"]
        lo = np.nextafter(ref["scales"].astype(np.float16), np.float16(-np.inf)).astype(np.float64)
        hi = np.nextafter(ref["scales"].astype(np.float16), np.float16(np.inf)).astype(np.float64)
        ok_s = eq | (tie_s & ((s == lo) | (s == hi)))
    else:
        ok_s = np.abs(s - ref["scales"]) <= 1e-6 * np.abs(ref["scales"])
    bad_s = ~ok_s & same & ~zero_tie
    assert bad_s.sum() == 0, f"{bad_s.sum()} scales differ (first {np.nonzero(bad_s)[0][:5]}: gpu {s[bad_s][:3]} oracle {ref['scales'][bad_s][:3]})"

    want = orc.codes_given_scale(ref["y"], s)
    tie_r = orc.rounding_ties(x, cen, ref["ids"], E, ref["y"], s)
    bad_c = (codes != want) & ~tie_r & same[:, None] & ~zero_tie[:, None]
    assert bad_c.sum() == 0, f"{bad_c.sum()} codes differ outside ties"
    return {"argmin_ties": int(tie_a.sum()), "scale_ties_f16": int(tie_s.sum()) if scale_dtype == "f16" else 0,
            "rounding_ties": int(tie_r.sum()), "code_flips_at_ties": int(((codes != want) & same[:, None]).sum()),
            "zero_residual_ties": int(zero_tie.sum()), "tokens": len(idx)}


def sample_rows(Tq: int, n: int, seed: int = 0):
    """A seeded subset of query rows that always contains the last rows (the
    ragged tail tile)."""
    if Tq <= n:
        return np.arange(Tq)
    rng = np.random.default_rng(seed)
    tail = np.arange(max(0, Tq - 40), Tq)
    rest = rng.choice(Tq - len(tail), n - len(tail), replace=False)
    return np.sort(np.concatenate([rest, tail]))


def oracle_attend(w, prob, hk, hv, T_full, rows=None, tau=None, with_cur=True):
    q = orc.f64(prob["q"])
    if rows is not None:
        q = q[rows]
    ck, cv = oracle_codec(prob["codec_k"]), oracle_codec(prob["codec_v"])
    kc = orc.f64(prob["k_cur"]) if with_cur else None
    vc = orc.f64(prob["v_cur"]) if with_cur else None
    return orc.attend(q, ck, cv, oracle_hist(hk), oracle_hist(hv), T_full, kc, vc, tau)


def compare_attn(O_gpu, L_gpu, O_ref, L_ref, fp32: bool, rows=None, tol=None):
    O = orc.f64(O_gpu)
    L = orc.f64(L_gpu)
    if rows is not None:
        O, L = O[rows], L[:, rows]
    err = np.abs(O - O_ref)
    fin = np.isfinite(L_ref)
    assert np.array_equal(np.isfinite(L), fin), "LSE finiteness differs"
    lerr = np.abs(L[fin] - L_ref[fin]).max() if fin.any() else 0.0
    nrm = np.linalg.norm(O_ref)
    rel = np.linalg.norm(O - O_ref) / nrm if nrm > 0 else np.linalg.norm(O - O_ref)
    stats = {"max_abs": float(err.max()) if err.size else 0.0, "rel_l2": float(rel), "lse_max_abs": float(lerr)}
    if fp32:
        assert stats["max_abs"] <= TOL_F32_MAXABS, stats
        assert stats["lse_max_abs"] <= TOL_F32_LSE, stats
    else:
        mx, rl, ls = tol if tol is not None else (TOL_BF16_MAXABS, TOL_BF16_RELL2, TOL_BF16_LSE)
        assert stats["max_abs"] <= mx, stats
        assert stats["rel_l2"] <= rl, stats
        assert stats["lse_max_abs"] <= ls, stats
    return stats


def tau_of(w):
    return 1.0 / math.sqrt(w.d)


U_BF16 = 2.0 ** -8  # unit roundoff of bf16 (8 significant bits, round to nearest)


def rounding_bound(q, ck, cv, ohk, ohv, kc, vc, T_full, tau):
    """Per-element bound on |O_gpu - O_exact| for the tensor-core path, for
    queries q [R, H, d] over the compressed history (oracle dicts) plus the
    current chunk kc, vc [Tc, H, d], all in fp64.

    Rounding points of that path (everything else is fp32 with errors ~2^-24):
      * full-dim history: K_hat = bf16(c + bf16(s) bf16(x)) with x = D code,
        so each element errs by at most u (2 |s x| + |k_hat|); V_hat alike;
      * low-dim history: the reduced query D_K^T q (scaled) is rounded to bf16,
        so a score errs by at most u s sum_r |q~_r| |code_r|; the value side
        rounds P s_V, P and the restore operands O~ / l, P_C / l to bf16;
      * every branch rounds P to bf16 for the value MMA; the output is bf16.
    With score errors dz_t, the weights become w_t e^{dz_t} / A with
    A = sum_s w_s e^{dz_s}, so O moves by (1/A) sum_t w_t (e^{dz_t} - 1)(v_t - O)
    exactly, and 1/A <= exp(sum_s w_s |dz_s|) (Jensen); the LSE moves by
    log A, at most log(1 + sum_t w_t (e^{|dz_t|} - 1)) in magnitude.  Returns
    (bound on O [R, H, d], bound on LSE [H, R])."""
    u = U_BF16
    R, H, d = q.shape
    T = len(ohk["ids"])
    T_low = T - T_full

    def decode(h, c, lo, hi):
        sx = h["scales"][lo:hi, None] * (np.asarray(h["codes"][lo:hi], np.float64) @ c["D"].T)  # s D code
        return sx, c["centers"][h["ids"][lo:hi]] + sx

    sxk, kf = decode(ohk, ck, T_low, T)
    sxv, vf = decode(ohv, cv, T_low, T)
    _, kl = decode(ohk, ck, 0, T_low)
    _, vl = decode(ohv, cv, 0, T_low)
    ek = u * (2 * np.abs(sxk) + np.abs(kf))
    ev = u * (2 * np.abs(sxv) + np.abs(vf))
    ck_low, sk_low = np.abs(np.asarray(ohk["codes"][:T_low], np.float64)), ohk["scales"][:T_low]
    cv_low, sv_low = np.abs(np.asarray(ohv["codes"][:T_low], np.float64)), ohv["scales"][:T_low]
    bound = np.zeros((R, H, d))
    lse_bound = np.zeros((H, R))
    for h in range(H):
        cols = slice(h * d, (h + 1) * d)
        qh = q[:, h, :]
        keys = np.concatenate([kl[:, cols], kf[:, cols], kc[:, h, :]])          # [T + Tc, d]
        vals = np.concatenate([vl[:, cols], vf[:, cols], vc[:, h, :]])
        z = tau * qh @ keys.T
        z -= z.max(axis=1, keepdims=True)
        wgt = np.exp(z)
        wgt /= wgt.sum(axis=1, keepdims=True)                                    # [R, T + Tc]
        O = wgt @ vals
        qred = qh @ ck["D"][cols, :]                                             # [R, r]
        dz = np.zeros_like(wgt)
        dz[:, :T_low] = tau * u * (np.abs(qred) @ ck_low.T) * sk_low[None, :]
        dz[:, T_low:T] = tau * (np.abs(qh) @ ek[:, cols].T)
        lse_bound[h] = np.log1p((wgt * np.expm1(dz)).sum(axis=1))
        a = wgt * np.expm1(dz) * np.exp((wgt * dz).sum(axis=1, keepdims=True))
        b = np.empty((R, d))
        for r0 in range(0, R, 16):                                               # softmax weights
            rs = slice(r0, r0 + 16)
            b[rs] = np.einsum("rt,rtk->rk", a[rs], np.abs(vals[None, :, :] - O[rs, None, :]))
        b += wgt[:, T_low:T] @ ev[:, cols]                                       # V_hat rounding
        b += u * (wgt @ np.abs(vals))                                            # P rounding
        low_coef = (cv_low * sv_low[:, None]) @ np.abs(cv["D"][cols, :]).T       # [T_low, d]
        b += 2 * u * (wgt[:, :T_low] @ low_coef)                                 # P s_V and O~ / l
        b += u * (wgt[:, :T_low] @ np.abs(cv["centers"][ohv["ids"][:T_low], cols]))  # P_C / l
        b += u * np.abs(O)                                                       # bf16 output
        bound[:, h, :] = b
    return bound, lse_bound


def gpu_rounding_bound(w, prob, hk, hv, T_full, rows, tau):
    """rounding_bound for rows of a GPU problem and its GPU-encoded history."""
    return rounding_bound(orc.f64(prob["q"])[rows], oracle_codec(prob["codec_k"]), oracle_codec(prob["codec_v"]),
                          oracle_hist(hk), oracle_hist(hv), orc.f64(prob["k_cur"]), orc.f64(prob["v_cur"]),
                          T_full, tau)
