"""Parity of the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs: encode codes bit-exact up to counted ties, attention
outputs within the stated tolerances."""
import math

import numpy as np
import pytest
import torch

import compressed_history_attention_b200 as nk
from synth.gen import WORKLOADS, scaled
from tests import _parity as P

pytestmark = pytest.mark.gpu

SMALL = {
    "tiny": WORKLOADS["tiny"],
    "full_small": scaled(WORKLOADS["full"], T=700, T_full=700, Tq=300),
    "mixed_small": scaled(WORKLOADS["mixed"], T=700, T_full=300, Tq=300),
    "long_small": scaled(WORKLOADS["long"], H=4, T=900, T_full=200, Tq=200),
}
FULL = ["full", "mixed", "long", "step30"]

PATHS = {"auto": 0, "simt": 1}


@pytest.fixture(params=sorted(PATHS))
def path(request):
    prev = nk.nanokv_set_kernel_path(PATHS[request.param])
    yield request.param
    nk.nanokv_set_kernel_path(prev)


def _sd(w):
    return "f32" if w.fp32 else "f16"


@pytest.mark.parametrize("name", sorted(SMALL))
def test_encode_small(name, path):
    w = SMALL[name]
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    torch.cuda.synchronize()
    for x, c, h in ((prob["hist_k"], prob["codec_k"], hk), (prob["hist_v"], prob["codec_v"], hv)):
        P.check_encode(x, c, h, _sd(w))


@pytest.mark.parametrize("name", FULL)
def test_encode_full_size_chunk(name, path):
    """One appended chunk (4680 tokens) at the full workload's shapes."""
    w = WORKLOADS[name]
    prob = P.problem(w)
    ck, cv = P.gpu_codecs(w, prob)
    n = w.chunk
    xk, xv = prob["hist_k"][-n:], prob["hist_v"][-n:]
    hk, hv = nk.nanokv_encode(ck, cv, xk, xv)
    torch.cuda.synchronize()
    sample = P.sample_rows(n, 1024, seed=1)
    for x, c, h in ((xk, prob["codec_k"], hk), (xv, prob["codec_v"], hv)):
        P.check_encode(x, c, h, _sd(w), sample=sample)


@pytest.mark.parametrize("H,C,r", [(2, 16, 64), (4, 48, 128), (8, 32, 192), (2, 128, 64), (3, 96, 192),
                                   (4, 80, 320), (8, 256, 256), (24, 256, 384)])
def test_encode_codec_shapes(H, C, r, path):
    """Every column split of the 2-CTA encode (r = 64, 128, 192 with fewer than
    64 centers, whose padded center rows read as zero), and codecs past it
    (more than 64 centers or r > 192): E shorter than one 128-row projection
    slice (r = 64), a 64-wide last slice (r = 320), the long workload's codec.
    A ragged token count (300 = 2 tiles + 44)."""
    w = scaled(WORKLOADS["long"], H=H, C=C, r=r, rank=min(r, 48), T=300, T_full=300, Tq=64)
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    torch.cuda.synchronize()
    for x, c, h in ((prob["hist_k"], prob["codec_k"], hk), (prob["hist_v"], prob["codec_v"], hv)):
        P.check_encode(x, c, h, _sd(w))


@pytest.mark.parametrize("name", sorted(SMALL))
def test_attend_small(name, path):
    w = SMALL[name]
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    O, L = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    Or, Lr = P.oracle_attend(w, prob, hk, hv, w.T_full)
    P.compare_attn(O, L, Or, Lr, w.fp32)


@pytest.mark.parametrize("name", FULL)
def test_attend_full_size_sampled_rows(name):
    """The full workload in the benchmark's launch configuration, checked on a
    seeded sample of query rows (always including the ragged last tile)."""
    w = WORKLOADS[name]
    prob = P.problem(w, layer=w.layers - 1)
    ck, cv, hk, hv = P.encode_history(w, prob)
    O, L = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    rows = P.sample_rows(w.Tq, 96 if name == "long" else 256, seed=2)
    Or, Lr = P.oracle_attend(w, prob, hk, hv, w.T_full, rows=rows)
    P.compare_attn(O, L, Or, Lr, w.fp32, rows=rows)


@pytest.mark.parametrize("T_full_frac", [0.0, 1.0])
def test_attend_single_branch(T_full_frac, path):
    w = SMALL["mixed_small"]
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    T_full = int(T_full_frac * w.T)
    O, L = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, T_full, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    Or, Lr = P.oracle_attend(w, prob, hk, hv, T_full)
    P.compare_attn(O, L, Or, Lr, False)


def test_attend_history_only_and_current_only(path):
    w = scaled(SMALL["mixed_small"], Tq=129)
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    # no current chunk
    O, L = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, w.T_full)
    torch.cuda.synchronize()
    Or, Lr = P.oracle_attend(w, prob, hk, hv, w.T_full, with_cur=False)
    P.compare_attn(O, L, Or, Lr, False)
    # no history
    e = hk.slice(0, 0)
    O, L = nk.nanokv_attend(prob["q"], ck, cv, e, e, 0, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    Or, Lr = P.oracle_attend(w, prob, e, e, 0)
    P.compare_attn(O, L, Or, Lr, False)
    # nothing at all: zeros and -inf
    O, L = nk.nanokv_attend(prob["q"], ck, cv, e, e, 0)
    torch.cuda.synchronize()
    assert torch.all(O == 0) and torch.all(torch.isneginf(L))


@pytest.mark.parametrize("Tq", [1, 127, 129])
def test_attend_ragged_query_counts(Tq, path):
    w = scaled(SMALL["mixed_small"], Tq=Tq, T=333, T_full=201)
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    O, L = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    Or, Lr = P.oracle_attend(w, prob, hk, hv, w.T_full)
    P.compare_attn(O, L, Or, Lr, False)


def test_attend_peaked_softmax(path):
    """tau = 1 with unit-variance queries: large scores exercise the running max."""
    w = SMALL["mixed_small"]
    prob = P.problem(w)
    prob["q"] = (prob["q"].float() * math.sqrt(w.d)).to(prob["q"].dtype)
    ck, cv, hk, hv = P.encode_history(w, prob)
    O, L = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"],
                            softmax_scale=1.0)
    torch.cuda.synchronize()
    Or, Lr = P.oracle_attend(w, prob, hk, hv, w.T_full, tau=1.0)
    if path == "simt":
        P.compare_attn(O, L, Or, Lr, False)
    else:
        # The tensor-core kernels round decoded K_hat / V_hat, the reduced
        # query and P to bf16.  With unit-variance queries and tau = 1 the
        # scores reach ~10, so those roundings move scores by up to ~0.1: the
        # check is the per-element bound derived from the oracle's quantities
        # (rounding_bound), plus 1e-4 for the fp32 accumulations.
        rows = np.arange(w.Tq)
        bound, lse_bound = P.gpu_rounding_bound(w, prob, hk, hv, w.T_full, rows, 1.0)
        err = np.abs(P.orc.f64(O) - Or)
        assert np.all(err <= bound + 1e-4), f"max err/bound {np.max(err / (bound + 1e-4)):.3f}"
        lerr = np.abs(P.orc.f64(L) - Lr)
        assert np.all(lerr <= lse_bound + 1e-4), f"max LSE err/bound {np.max(lerr / (lse_bound + 1e-4)):.3f}"


@pytest.mark.parametrize("H,C,r", [(12, 64, 192), (24, 256, 384), (2, 8, 8)])
def test_codec_prepare_tables(H, C, r):
    """The derived encode tables E c_j and |c_j|^2 against fp64: bf16 (or
    fp32) products summed in fp32, so within J * 2^-24 of the sum of |terms|."""
    g = torch.Generator(device="cpu").manual_seed(7)
    J = H * (16 if C == 8 else 128)
    dt = torch.float32 if C == 8 else torch.bfloat16
    cen = torch.randn(C, J, generator=g).to(dt).cuda()
    E = (torch.randn(r, J, generator=g) / math.sqrt(J)).to(dt).cuda()
    c = nk.Codec(H, J // H, cen, torch.zeros(J, r, dtype=dt, device="cuda"), E).prepare()
    torch.cuda.synchronize()
    aux = c.aux.view(torch.float32)[: C * r + C].double().cpu().numpy()
    cd, ed = P.orc.f64(cen), P.orc.f64(E)
    ec, mag = cd @ ed.T, np.abs(cd) @ np.abs(ed).T
    assert np.all(np.abs(aux[: C * r].reshape(C, r) - ec) <= J * 2.0 ** -24 * mag + 1e-30)
    nrm = (cd * cd).sum(axis=1)
    assert np.all(np.abs(aux[C * r:] - nrm) <= J * 2.0 ** -24 * nrm)


def test_lse_merge_parity():
    from oracle import nanokv_oracle as orc
    g = torch.Generator(device="cuda").manual_seed(5)
    Tq, H, d = 77, 3, 128
    parts = []
    for i in range(3):
        o = torch.randn(Tq, H, d, device="cuda", generator=g)
        l = torch.randn(H, Tq, device="cuda", generator=g) * 3
        if i == 1:
            l[:, :10] = -math.inf
        parts.append((o, l))
    parts[0][1][:, :5] = -math.inf
    parts[2][1][:, :5] = -math.inf
    # fp32 output within 1e-5; bf16 output within one bf16 rounding (2^-8 relative)
    for dt, rel in ((torch.float32, 0.0), (torch.bfloat16, 2.0 ** -8)):
        out, lse = nk.nanokv_lse_merge([p[0] for p in parts], [p[1] for p in parts], out_dtype=dt)
        torch.cuda.synchronize()
        Or, Lr = orc.lse_merge([(orc.f64(o), orc.f64(l)) for o, l in parts])
        assert np.all(np.abs(orc.f64(out) - Or) <= 1e-5 + rel * np.abs(Or))
        fin = np.isfinite(Lr)
        assert np.array_equal(np.isfinite(orc.f64(lse)), fin)
        assert np.abs(orc.f64(lse)[fin] - Lr[fin]).max() <= 1e-5


@pytest.mark.parametrize("name", ["mixed_small", "full_small"])
def test_attend_graph_capture_matches_eager(name):
    """With several branches the call forks onto helper streams and joins
    before the merge; captured in a CUDA graph and replayed (after the inputs
    changed) it must give the eager result for the new inputs, bit for bit."""
    w = SMALL[name]
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    q = prob["q"].clone()
    out = torch.empty_like(q)
    lse = torch.empty(w.H, w.Tq, dtype=torch.float32, device=q.device)
    ws = torch.empty(nk.nanokv_attend_workspace(w.Tq, ck, cv, w.T, w.T_full, w.Tq), dtype=torch.uint8,
                     device=q.device)
    nk.nanokv_attend(q, ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"], out=out, lse=lse, workspace=ws)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            nk.nanokv_attend(q, ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"], out=out, lse=lse,
                             workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    gen = torch.Generator(device=q.device).manual_seed(11)
    q.copy_((torch.randn(q.shape, device=q.device, generator=gen) / math.sqrt(w.d)).to(q.dtype))
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    Og, Lg = out.clone(), lse.clone()
    Oe, Le = nk.nanokv_attend(q, ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"])
    torch.cuda.synchronize()
    assert torch.equal(Og, Oe)
    assert torch.equal(Lg, Le)
    del g


@pytest.mark.parametrize("name", ["full", "mixed"])
def test_attend_is_deterministic(name):
    """Every output is a fixed function of the inputs: repeated calls at the
    full workload agree bit for bit.  (Rounding-level differences between runs
    would mean some key was decoded or scored from data a producer had not
    finished writing, or had already replaced, which a tolerance check on a
    near-uniform softmax cannot see.)"""
    w = WORKLOADS[name]
    prob = P.problem(w)
    ck, cv, hk, hv = P.encode_history(w, prob)
    runs = []
    for _ in range(4):
        O, L = nk.nanokv_attend(prob["q"], ck, cv, hk, hv, w.T_full, prob["k_cur"], prob["v_cur"])
        torch.cuda.synchronize()
        runs.append((O.clone(), L.clone()))
    for O, L in runs[1:]:
        assert torch.equal(O, runs[0][0])
        assert torch.equal(L, runs[0][1])
