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

    tie_s = orc.scale_ties(ref["y"], scale_dtype)
    if scale_dtype == "f16":
        eq = s == ref["scales"]
        lo = np.nextafter(ref["scales"].astype(np.float16), np.float16(-np.inf)).astype(np.float64)
        hi = np.nextafter(ref["scales"].astype(np.float16), np.float16(np.inf)).astype(np.float64)
        ok_s = eq | (tie_s & ((s == lo) | (s == hi)))
    else:
        ok_s = np.abs(s - ref["scales"]) <= 1e-6 * np.abs(ref["scales"])
    bad_s = ~ok_s & same
    assert bad_s.sum() == 0, f"{bad_s.sum()} scales differ (first {np.nonzero(bad_s)[0][:5]}: gpu {s[bad_s][:3]} oracle {ref['scales'][bad_s][:3]})"

    want = orc.codes_given_scale(ref["y"], s)
    tie_r = orc.rounding_ties(x, cen, ref["ids"], E, ref["y"], s)
    bad_c = (codes != want) & ~tie_r & same[:, None]
    assert bad_c.sum() == 0, f"{bad_c.sum()} codes differ outside ties"
    return {"argmin_ties": int(tie_a.sum()), "scale_ties_f16": int(tie_s.sum()) if scale_dtype == "f16" else 0,
            "rounding_ties": int(tie_r.sum()), "code_flips_at_ties": int(((codes != want) & same[:, None]).sum()),
            "tokens": len(idx)}


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
