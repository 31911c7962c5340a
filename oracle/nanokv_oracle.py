"""Plain, slow fp64 CPU oracle for NanoKV compressed-history attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke entry point and the
benchmark's CPU-baseline leg may import this module.  The CUDA path never
calls it, and it shares no code with the CUDA path.

Source: "NanoKV: High-Ratio KV Cache Compression for Autoregressive Video
Generation" (arXiv 2611.06377): abstract; Fig. 2(b,c); Fig. 4(a) joint
head-channel encoding read through full- or mixed-dimensional attention;
Fig. 4(b) encoder to INT4 coefficients, decoder adds back centers; Fig. 4(d)
fixed routing, reduced queries, output restore, LSE merging; Table 5 (rank per
layer per K/V branch, centers fitted separately for K and V).

The pages print no formulas.  Where they are silent this module takes the
plain readings below (each also listed in the design notes):
  * nearest center = smallest squared Euclidean distance in the joint H*d
    space, ties to the lowest index;
  * per-token symmetric scale s = stored_dtype(max_i |y_i| / 7), INT4 codes in
    [-7, 7] (-8 unused), round-half-to-even, s = 0 gives all-zero codes;
  * softmax scale tau (1/sqrt(d) by default), no mask, natural-log LSE;
  * head h owns joint columns [h*d, (h+1)*d) of K/V and rows of D;
  * the current chunk is a third, uncompressed attention branch merged by LSE;
  * routing: the most recent T_full history tokens are full-dim, the older
    T - T_full tokens low-dim;
  * calibration (Tables 2, 5; Fig. 3(a)): Lloyd k-means from given initial
    centers, then the leading eigenvectors of the residual second moment
    (see the calibration section below);
  * reduced attention dimension (Table 6): head h attends in R^{d_h} through
    orthonormal maps U_h (queries, keys) and W_h (values, output restore);
    the analytical maps are the leading left singular vectors of the head's
    decoder rows (see the section on reduced dimensions below).

Every stored value (bf16 / fp16 / fp32) converts exactly to fp64, and all
arithmetic here is fp64 numpy.  Parity of every function is pinned by the
"not gpu" tests (brute force, closed forms, invariants, the pages' tables).
"""
from __future__ import annotations

import numpy as np

QMAX = 7  # symmetric INT4 range [-7, 7]


def f64(a) -> np.ndarray:
    """Exact conversion of a stored array (numpy or torch CPU) to fp64."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu")
        if a.dtype.is_floating_point:
            a = a.double()
        a = a.numpy()
    return np.asarray(a, dtype=np.float64)


def round_to_storage(v: np.ndarray, scale_dtype: str) -> np.ndarray:
    """Round fp64 values to the scale's storage dtype (RNE), back in fp64."""
    if scale_dtype == "f16":
        return np.asarray(v, dtype=np.float64).astype(np.float16).astype(np.float64)
    if scale_dtype == "f32":
        return np.asarray(v, dtype=np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(scale_dtype)


# ----------------------------------------------------------------------------
# Encode (Fig. 4(a,b); abstract: shared content in cluster centers, joint
# head-channel residuals encoded into low-bit coefficients)
# ----------------------------------------------------------------------------

def squared_distances(x: np.ndarray, centers: np.ndarray) -> np.ndarray:
    """dist[t, j] = sum_i (x[t, i] - centers[j, i])^2, one center at a time."""
    T, C = x.shape[0], centers.shape[0]
    dist = np.empty((T, C), dtype=np.float64)
    for j in range(C):
        diff = x - centers[j][None, :]
        dist[:, j] = np.einsum("ti,ti->t", diff, diff)
    return dist


def assign(x: np.ndarray, centers: np.ndarray) -> np.ndarray:
    """Nearest center of each token (lowest index on exact ties)."""
    return np.argmin(squared_distances(x, centers), axis=1)


def project(x: np.ndarray, centers: np.ndarray, ids: np.ndarray, E: np.ndarray) -> np.ndarray:
    """Residual coefficients y_t = E (x_t - c_{a_t}),  E is [r, J]."""
    rho = x - centers[ids]
    return rho @ E.T


def scale_of(y: np.ndarray, scale_dtype: str) -> np.ndarray:
    """Per-token symmetric scale s_t = stored(max_i |y_ti| / 7)."""
    m = np.max(np.abs(y), axis=1) if y.shape[1] else np.zeros(y.shape[0])
    return round_to_storage(m / QMAX, scale_dtype)


def quantise(y: np.ndarray, s: np.ndarray) -> np.ndarray:
    """INT4 codes clamp(round_half_even(y / s), -7, 7); s = 0 gives zeros."""
    codes = np.zeros(y.shape, dtype=np.int64)
    nz = s > 0
    codes[nz] = np.clip(np.rint(y[nz] / s[nz, None]), -QMAX, QMAX).astype(np.int64)
    return codes


def encode(x: np.ndarray, centers: np.ndarray, E: np.ndarray, scale_dtype: str) -> dict:
    """Full encode of tokens x [T, J]: ids, unpacked codes [T, r], scales [T],
    plus the fp64 intermediates used by the tie accounting."""
    ids = assign(x, centers)
    y = project(x, centers, ids, E)
    s = scale_of(y, scale_dtype)
    return {"ids": ids, "codes": quantise(y, s), "scales": s, "y": y}


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """[T, r] ints in [-8, 7] -> [T, r/2] bytes; code 2i in the low nibble of
    byte i, two's complement."""
    c = (np.asarray(codes, dtype=np.int64) & 0xF).astype(np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """Inverse of pack_codes: [T, r/2] bytes -> [T, r] int64 in [-8, 7]."""
    p = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    lo, hi = p & 0xF, (p >> 4) & 0xF
    out = np.empty((p.shape[0], 2 * p.shape[1]), dtype=np.int64)
    out[:, 0::2] = np.where(lo >= 8, lo - 16, lo)
    out[:, 1::2] = np.where(hi >= 8, hi - 16, hi)
    return out


def decode(ids, codes, scales, centers, D) -> np.ndarray:
    """x_hat_t = c_{a_t} + s_t * D q_t   (Fig. 4(b): decoder reconstructs the
    residual and adds back the center).  D is [J, r]."""
    return centers[ids] + scales[:, None] * (np.asarray(codes, np.float64) @ D.T)


# ----------------------------------------------------------------------------
# Attention branches.  Layout: q [Tq, H, d]; history K/V joint vectors [T, J]
# with head h in columns [h*d, (h+1)*d); outputs O [Tq, H, d], LSE [H, Tq].
# ----------------------------------------------------------------------------

def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, tau: float):
    """Textbook softmax attention per head over keys k, v [T, H, d]."""
    Tq, H, d = q.shape
    T = k.shape[0]
    O = np.zeros((Tq, H, d))
    lse = np.full((H, Tq), -np.inf)
    if T == 0:
        return O, lse
    for h in range(H):
        z = tau * (q[:, h, :] @ k[:, h, :].T)
        m = z.max(axis=1, keepdims=True)
        p = np.exp(z - m)
        l = p.sum(axis=1, keepdims=True)
        O[:, h, :] = (p @ v[:, h, :]) / l
        lse[h] = (m + np.log(l))[:, 0]
    return O, lse


def attend_full(q, ck: dict, cv: dict, hk: dict, hv: dict, tau: float):
    """Full-dimensional branch (Fig. 4(a), NanoKV): decode K_hat, V_hat to the
    full joint dimension, then ordinary attention over them."""
    Tq, H, d = q.shape
    kh = decode(hk["ids"], hk["codes"], hk["scales"], ck["centers"], ck["D"])
    vh = decode(hv["ids"], hv["codes"], hv["scales"], cv["centers"], cv["D"])
    T = kh.shape[0]
    return softmax_attention(q, kh.reshape(T, H, d), vh.reshape(T, H, d), tau)


def attend_low(q, ck: dict, cv: dict, hk: dict, hv: dict, tau: float):
    """Mixed-dimensional branch (abstract: NanoKV-Fast reuses the stored
    coefficients; Fig. 4(d): reduce the queries, restore the output dimension).

    Per head h with D_h = rows [h*d, (h+1)*d) of D and c_{j,h} the head's slice
    of center j:
        q~   = D_{K,h}^T q                  (reduced query, length r)
        qc_j = c_{K,j,h} . q                (query against each K center)
        z_t  = tau * (s_t * q~ . code_t + qc_{a_t})
        O    = (sum_t p_t c_{V,a_t,h} + D_{V,h} sum_t p_t s_t code^V_t) / sum_t p_t
    """
    Tq, H, d = q.shape
    T = len(hk["ids"])
    O = np.zeros((Tq, H, d))
    lse = np.full((H, Tq), -np.inf)
    if T == 0:
        return O, lse
    codes_k = np.asarray(hk["codes"], np.float64)
    codes_v = np.asarray(hv["codes"], np.float64)
    sk, sv = hk["scales"], hv["scales"]
    C_v = cv["centers"].shape[0]
    onehot_v = np.zeros((T, C_v))
    onehot_v[np.arange(T), hv["ids"]] = 1.0
    for h in range(H):
        cols = slice(h * d, (h + 1) * d)
        qh = q[:, h, :]
        q_red = qh @ ck["D"][cols, :]                 # [Tq, r]
        qc = qh @ ck["centers"][:, cols].T           # [Tq, C]
        z = tau * (sk[None, :] * (q_red @ codes_k.T) + qc[:, hk["ids"]])
        m = z.max(axis=1, keepdims=True)
        p = np.exp(z - m)
        l = p.sum(axis=1, keepdims=True)
        o_red = p @ (sv[:, None] * codes_v)          # [Tq, r]
        p_c = p @ onehot_v                           # [Tq, C]
        O[:, h, :] = (p_c @ cv["centers"][:, cols] + o_red @ cv["D"][cols, :].T) / l
        lse[h] = (m + np.log(l))[:, 0]
    return O, lse


def lse_merge(parts):
    """Combine branch partials (O_i, LSE_i) by log-sum-exp weights (Fig. 4(d)):
    LSE = log sum_i exp(LSE_i),  O = sum_i exp(LSE_i - LSE) O_i.  Branches with
    LSE = -inf contribute nothing; if all are empty, O = 0 and LSE = -inf."""
    lses = np.stack([p[1] for p in parts])           # [n, H, Tq]
    m = lses.max(axis=0)
    safe_m = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(lses - safe_m[None])                  # exp(-inf) = 0
    tot = w.sum(axis=0)
    lse = np.where(tot > 0, safe_m + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    O = np.zeros_like(parts[0][0])
    for (o_i, _), w_i in zip(parts, w):
        coef = np.where(tot > 0, w_i / np.where(tot > 0, tot, 1.0), 0.0)   # [H, Tq]
        O += coef.T[:, :, None] * o_i
    return O, lse


def split_history(h: dict, lo: int, hi: int) -> dict:
    return {"ids": h["ids"][lo:hi], "codes": h["codes"][lo:hi], "scales": h["scales"][lo:hi]}


def attend(q, ck, cv, hk, hv, T_full: int, k_cur=None, v_cur=None, tau=None):
    """Compressed-history attention of a query chunk (Fig. 4(d) with Fig. 4(a)):
    the oldest T - T_full history tokens go through the low-dim branch, the most
    recent T_full through full-dim decode-attention, the current chunk's
    uncompressed K/V through plain attention; the three are LSE-merged."""
    Tq, H, d = q.shape
    if tau is None:
        tau = 1.0 / np.sqrt(d)
    T = len(hk["ids"])
    T_low = T - T_full
    parts = [
        attend_low(q, ck, cv, split_history(hk, 0, T_low), split_history(hv, 0, T_low), tau),
        attend_full(q, ck, cv, split_history(hk, T_low, T), split_history(hv, T_low, T), tau),
    ]
    if k_cur is not None and len(k_cur):
        parts.append(softmax_attention(q, k_cur, v_cur, tau))
    return lse_merge(parts)


def take_history(h: dict, idx) -> dict:
    return {"ids": h["ids"][idx], "codes": h["codes"][idx], "scales": h["scales"][idx]}


def attend_routed(q, ck, cv, hk, hv, full_mask, full_heads=None, k_cur=None, v_cur=None, tau=None,
                  lowdim=None):
    """Compressed-history attention under a general full-dim routing policy
    (NanoKV-Fast Table 7: recent, anchor and sink frames read at full
    dimension, per-layer full fallback, sensitive heads kept at full
    dimension; Fig. 4(d): LSE merging of the branches).  History tokens with
    full_mask[t] go through full-dim decode-attention and the others through
    the low-dim branch; a head with full_heads[h] reads every history token
    full-dim.  With lowdim (maps as in attend_reduced, d_h[h] = 0 for heads
    not reduced), the low-dim tokens of a reduced head go through attention
    at its reduced dimension (Table 6) instead.  The current chunk is the
    third branch, as in attend()."""
    Tq, H, d = q.shape
    if tau is None:
        tau = 1.0 / np.sqrt(d)
    full_mask = np.asarray(full_mask, dtype=bool)
    f_idx, l_idx = np.nonzero(full_mask)[0], np.nonzero(~full_mask)[0]
    cur = [softmax_attention(q, k_cur, v_cur, tau)] if k_cur is not None and len(k_cur) else []
    hk_f, hv_f = take_history(hk, f_idx), take_history(hv, f_idx)
    hk_l, hv_l = take_history(hk, l_idx), take_history(hv, l_idx)
    full_part = attend_full(q, ck, cv, hk_f, hv_f, tau)
    routed = lse_merge([full_part, attend_low(q, ck, cv, hk_l, hv_l, tau)] + cur)
    if lowdim is not None and np.any(np.asarray(lowdim["d_h"]) > 0):
        red = np.asarray(lowdim["d_h"]) > 0
        dims = {"U": lowdim["U"], "W": lowdim["W"], "d_h": np.where(red, lowdim["d_h"], d)}
        reduced = lse_merge([full_part, attend_reduced(q, ck, cv, hk_l, hv_l, dims, tau)] + cur)
        routed = (np.where(red[None, :, None], reduced[0], routed[0]), np.where(red[:, None], reduced[1], routed[1]))
    if full_heads is None or not np.any(full_heads):
        return routed
    all_idx = np.arange(len(full_mask))
    kept = lse_merge([attend_full(q, ck, cv, take_history(hk, all_idx), take_history(hv, all_idx), tau)] + cur)
    sel = np.asarray(full_heads, dtype=bool)
    O = np.where(sel[None, :, None], kept[0], routed[0])
    lse = np.where(sel[:, None], kept[1], routed[1])
    return O, lse


# ----------------------------------------------------------------------------
# Calibration of a codec on a chunk of tokens (Table 5: centers fitted
# separately for K and V; Table 2: joint PCA with INT4 coefficients, then
# shared centers; Fig. 3(a): joint head-channel PCA retains the most KV
# variance at matched dimensional compression).
#
# Readings (the pages give no algorithm):
#   * centers: Lloyd's k-means from caller-given initial centers, a fixed
#     number of rounds; each round assigns every token to its nearest center
#     (assign(): ties to the lowest index), then moves every center to the
#     mean of its tokens; a center with no tokens stays where it is;
#   * decoder: the r leading eigenvectors (decreasing eigenvalue) of the
#     residual second-moment matrix (1/N) sum_t rho_t rho_t^T over the joint
#     H*d channels, rho_t = x_t - c_{a_t} with the final centers and their
#     assignment; E = D^T;
#   * each eigenvector's sign: its entry of largest magnitude is positive
#     (the first such entry on a tie).
# ----------------------------------------------------------------------------

def kmeans(x: np.ndarray, init_centers: np.ndarray, rounds: int):
    """Lloyd rounds from init_centers [C, J]; returns (centers, ids), ids the
    assignment to the returned centers."""
    c = np.array(init_centers, dtype=np.float64, copy=True)
    for _ in range(rounds):
        ids = assign(x, c)
        for j in range(c.shape[0]):
            members = ids == j
            if members.any():
                c[j] = x[members].mean(axis=0)
    return c, assign(x, c)


def sign_fixed(v: np.ndarray) -> np.ndarray:
    """Columns of v with the sign that makes each column's entry of largest
    magnitude positive (first such entry on a tie)."""
    v = np.array(v, dtype=np.float64, copy=True)
    for i in range(v.shape[1]):
        k = int(np.argmax(np.abs(v[:, i])))
        if v[k, i] < 0:
            v[:, i] = -v[:, i]
    return v


def joint_pca(x: np.ndarray, centers: np.ndarray, ids: np.ndarray, r: int):
    """Decoder D [J, r] and the eigenvalues [r] of the residual second-moment
    matrix (leading r, decreasing)."""
    rho = x - centers[ids]
    S = rho.T @ rho / x.shape[0]
    w, v = np.linalg.eigh(S)
    order = np.argsort(-w, kind="stable")[:r]
    return sign_fixed(v[:, order]), w[order]


def calibrate(x: np.ndarray, init_centers: np.ndarray, rounds: int, r: int) -> dict:
    """Codec of one branch from a calibration chunk x [N, J]: centers [C, J],
    D [J, r], E = D^T, plus the final assignment and the eigenvalues."""
    centers, ids = kmeans(x, init_centers, rounds)
    D, w = joint_pca(x, centers, ids, r)
    return {"centers": centers, "D": D, "E": D.T.copy(), "ids": ids, "eigenvalues": w}


# ----------------------------------------------------------------------------
# Reduced attention dimension per head (NanoKV-Fast: Table 6, head-layer
# pairs deployed at d_h in {32, 64, 96, 128}; Fig. 4(d), the low-dimensional
# branch reduces the queries and restores the output dimension; Table 8,
# low-dimensional maps with an analytical initialization).
#
# Readings (the pages print no formulas for the maps):
#   * head h has a key/query map U_h and a value map W_h, each [d, d_h] with
#     orthonormal columns; the attention of that head runs in R^{d_h}:
#         q~ = U_h^T q,  k~_t = U_h^T K_hat_t,  v~_t = W_h^T V_hat_t,
#         o~ = softmax(tau q~ k~^T) v~,        O_h = W_h o~;
#     tau stays the model's softmax scale;
#   * the stored coefficients are reused: k~_t = U_h^T c_K[a_t] +
#     s_t (U_h^T D_K,h) code_t, i.e. the decoder and centers are mapped once
#     and the coefficients decode straight into d_h dimensions;
#   * the analytical initialization takes U_h (W_h) as the leading d_h left
#     singular vectors of the head's decoder rows D_K,h (D_V,h), [d, r];
#   * maps are stored padded as [H, d, d]: head h uses columns [0, d_h).
# ----------------------------------------------------------------------------

def lowdim_maps(D: np.ndarray, H: int, d: int) -> np.ndarray:
    """Analytical low-dimensional maps [H, d, d]: head h's left singular
    vectors of its decoder rows D[h*d:(h+1)*d, :], by decreasing singular
    value (a complete orthonormal basis of R^d, so any leading d_h columns
    form the rank-d_h truncation's column space)."""
    out = np.zeros((H, d, d))
    for h in range(H):
        u, _, _ = np.linalg.svd(D[h * d:(h + 1) * d, :], full_matrices=True)
        out[h] = u
    return out


def attend_reduced(q, ck: dict, cv: dict, hk: dict, hv: dict, maps: dict, tau: float):
    """History attention of every head at its reduced dimension.  maps:
    {"U": [H, d, d], "W": [H, d, d], "d_h": [H]} with 0 < d_h[h] <= d."""
    Tq, H, d = q.shape
    T = len(hk["ids"])
    O = np.zeros((Tq, H, d))
    lse = np.full((H, Tq), -np.inf)
    if T == 0:
        return O, lse
    codes_k = np.asarray(hk["codes"], np.float64)
    codes_v = np.asarray(hv["codes"], np.float64)
    for h in range(H):
        n = int(maps["d_h"][h])
        U = np.asarray(maps["U"][h], np.float64)[:, :n]          # [d, d_h]
        W = np.asarray(maps["W"][h], np.float64)[:, :n]
        cols = slice(h * d, (h + 1) * d)
        q_red = q[:, h, :] @ U                                    # reduce the queries
        Dk, Dv = U.T @ ck["D"][cols, :], W.T @ cv["D"][cols, :]   # decoders into d_h
        ck_red, cv_red = ck["centers"][:, cols] @ U, cv["centers"][:, cols] @ W
        k_red = ck_red[hk["ids"]] + hk["scales"][:, None] * (codes_k @ Dk.T)
        v_red = cv_red[hv["ids"]] + hv["scales"][:, None] * (codes_v @ Dv.T)
        z = tau * (q_red @ k_red.T)
        m = z.max(axis=1, keepdims=True)
        p = np.exp(z - m)
        l = p.sum(axis=1, keepdims=True)
        O[:, h, :] = ((p @ v_red) / l) @ W.T                      # restore to d
        lse[h] = (m + np.log(l))[:, 0]
    return O, lse


# ----------------------------------------------------------------------------
# Tie accounting: an integer decided by floating point (argmin, rounding, the
# fp16 scale) may legitimately differ between two correct implementations only
# when the real-valued quantity sits within rounding error of the boundary.
# ----------------------------------------------------------------------------

TIE_REL = 1e-6


def argmin_ties(x: np.ndarray, centers: np.ndarray) -> np.ndarray:
    """Tokens whose best and second-best center distances are within
    1e-6 * (|x|^2 + |c_best|^2)."""
    dist = squared_distances(x, centers)
    if dist.shape[1] < 2:
        return np.zeros(dist.shape[0], dtype=bool)
    srt = np.sort(dist, axis=1)
    best = np.argmin(dist, axis=1)
    scale = np.einsum("ti,ti->t", x, x) + np.einsum("ti,ti->t", centers[best], centers[best])
    return (srt[:, 1] - srt[:, 0]) <= TIE_REL * scale


def codes_given_scale(y: np.ndarray, s: np.ndarray) -> np.ndarray:
    """The oracle's code decision under a given stored scale."""
    return quantise(y, s)


def rounding_ties(x, centers, ids, E, y, s) -> np.ndarray:
    """Code entries whose y/s lies within 1e-6 * max(1, sum_j |E_ij||rho_j| / s)
    of a half-integer (the forward-error scale of the dot product)."""
    rho = x - centers[ids]
    mag = np.abs(rho) @ np.abs(E).T                  # [T, r]
    ss = np.where(s > 0, s, 1.0)[:, None]
    u = y / ss
    dist = np.abs(u - (np.floor(u) + 0.5))
    band = TIE_REL * np.maximum(1.0, mag / ss)
    return (dist <= band) & (s[:, None] > 0)


def scale_ties(y: np.ndarray, scale_dtype: str) -> np.ndarray:
    """Tokens whose max|y|/7 lies within 1e-6 relative of a rounding midpoint of
    the scale's storage dtype (fp16).  For fp32 scales every value is that close
    to a midpoint; those are compared with a relative tolerance instead."""
    v = np.max(np.abs(y), axis=1) / QMAX if y.shape[1] else np.zeros(y.shape[0])
    if scale_dtype == "f32":
        return np.ones(v.shape, dtype=bool)
    f = v.astype(np.float16)
    up = np.nextafter(f, np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(f, np.float16(-np.inf)).astype(np.float64)
    ff = f.astype(np.float64)
    mid = np.where(v >= ff, (ff + up) / 2, (ff + dn) / 2)
    return np.abs(v - mid) <= TIE_REL * np.abs(v)


# ----------------------------------------------------------------------------
# Accounting (Table 5 x Table 9; Table 11)
# ----------------------------------------------------------------------------

def nominal_coefficient_cr(H: int, d: int, r: int, src_bits: int = 16, code_bits: int = 4) -> float:
    """Coefficient compression of one token: H*d values of src_bits against r
    coefficients of code_bits."""
    return (src_bits * H * d) / (code_bits * r)


def overall_saving(historical_share: float, saving_within_history: float) -> float:
    """Table 11: overall visual-attention MAC saving = historical share x saving
    within history."""
    return historical_share * saving_within_history

