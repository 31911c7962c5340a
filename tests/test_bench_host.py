"""Host-side checks of the benchmark's work accounting (no GPU): the
algorithmic totals of each workload against the values derived independently
for the hot-path scope table, and the split of the history between the
kernels when low-dim tokens run through the full-dim kernel."""
import pytest
import torch

import bench
import compressed_history_attention_b200 as nk
from synth.gen import WORKLOADS


def _codec(w):
    # shapes only: the routing query reads sizes and dtypes, never the data
    J, dt = w.J, torch.bfloat16
    return nk.Codec(w.H, w.d, torch.zeros(w.C, J, dtype=dt), torch.zeros(J, w.r, dtype=dt),
                    torch.zeros(w.r, J, dtype=dt))


def _work(name):
    w = WORKLOADS[name]
    s = {"ck": _codec(w), "cv": _codec(w)}
    return w, bench.work_of(w, w.chunk, s)


# totals in TFLOP: attention as the workload names its split, and the encode
# of one chunk (K and V)
@pytest.mark.parametrize("name,attend,with_encode", [
    ("full", 0.5548, 0.562),
    ("mixed", 0.686, None),
    ("long", 15.42, None),
    ("step30", 2.10, None),
])
def test_named_work_totals(name, attend, with_encode):
    w, (af, ak, ef, eb) = _work(name)
    assert af["total"] / 1e12 == pytest.approx(attend, rel=2e-3)
    if with_encode is not None:
        assert (af["total"] + ef) / 1e12 == pytest.approx(with_encode, rel=2e-3)
    # encode bytes: x read once, ids + codes + scales written, per branch
    assert eb == 2 * (w.chunk * w.J * 2 + w.chunk * (1 + w.r // 2 + 2))


def test_long_low_dim_main_term():
    """The long workload's low-dim scores and values: 4 Tq T_l H r."""
    w, (af, _, _, _) = _work("long")
    main = 4 * w.Tq * w.T_low * w.H * w.r
    assert main / 1e12 == pytest.approx(14.53, rel=1e-3)
    assert af["low"] > main  # plus the query prep and the output restore


@pytest.mark.parametrize("name", ["full", "mixed", "long", "step30"])
def test_work_as_run_equals_named(name):
    """Every workload's codecs have a low-dim tensor-core kernel (the long
    rollout's C = 256, r = 384 included), so the history runs split as named."""
    _, (af, ak, _, _) = _work(name)
    assert ak == af


def test_encode_parity_counts_mismatches_outside_ties():
    """The bench's parity block: identical outputs give zero mismatches; a
    changed id and a changed code outside any tie are counted."""
    import numpy as np
    from oracle import nanokv_oracle as orc
    rng = np.random.default_rng(0)
    cen = rng.standard_normal((8, 32))
    E = np.linalg.qr(rng.standard_normal((32, 8)))[0].T
    x = cen[rng.integers(0, 8, 40)] + 0.3 * rng.standard_normal((40, 32))
    ref = orc.encode(x, cen, E, "f16")
    codec = {"centers": cen, "E": E}
    same = bench.encode_parity(x, codec, ref["ids"].copy(), ref["codes"].copy(), ref["scales"].copy(), ref, "f16")
    assert same["ids_differ_outside_ties"] == 0 and same["codes_differ_outside_ties"] == 0
    assert same["scales_differ_outside_ties"] == 0 and same["tokens"] == 40
    ids, codes = ref["ids"].copy(), ref["codes"].copy()
    ids[3] = (ids[3] + 1) % 8
    codes[5, 2] += 1 if codes[5, 2] < 7 else -1
    bad = bench.encode_parity(x, codec, ids, codes, ref["scales"].copy(), ref, "f16")
    assert bad["ids_differ_outside_ties"] == 1
    assert bad["codes_differ_outside_ties"] == 1


def test_routed_work_accounting():
    """routed_flops reduces to attend_flops for the fixed policy, counts a
    kept head's low-dim tokens full-dim, and a reduced head's at its width:
    scores and values of width d_h, a decode into d_h per token, the query
    reduction and the restore per query row."""
    from compressed_history_attention_b200.accounting import attend_flops, routed_flops
    Tq, H, d, r, C, Tf, Tl, Tc = 100, 4, 128, 192, 64, 300, 500, 100
    base = attend_flops(Tq, H, d, r, C, Tf, Tl, Tc)
    assert routed_flops(Tq, H, d, r, C, Tf, Tl, Tc)["total"] == base["total"]
    assert routed_flops(Tq, H, d, r, C, Tf, Tl, Tc, kept=H)["total"] == attend_flops(Tq, H, d, r, C, Tf + Tl, 0, Tc)["total"]
    assert routed_flops(Tq, H, d, r, C, Tf, Tl, Tc, low_full=True)["total"] == \
        attend_flops(Tq, H, d, r, C, Tf + Tl, 0, Tc)["total"]
    one = routed_flops(Tq, H, d, r, C, Tf, Tl, Tc, dims=[32])
    assert one["reduced"] == 4 * Tq * Tl * 32 + 4 * Tl * 32 * r + 4 * Tq * d * 32
    assert one["low"] == base["low"] * (H - 1) // H
    assert one["total"] < base["total"]


@pytest.mark.parametrize("name,per_token,effective,with_encoder", [
    # bf16 K/V of J values per token against 1 id byte + r/2 code bytes + a
    # 2-byte scale; the effective figures add the two branches' centers and
    # decoders (and encoders): e.g. full, T = 14040, J = 1536, C = 64, r = 192:
    # 2*14040*3072 / (2*14040*99 + 2*(64*1536 + 1536*192)*2) = 19.82
    ("full", 3072 / 99, 86261760 / (2779920 + 1572864), 86261760 / (2779920 + 1572864 + 1179648)),
    ("long", 6144 / 195, 2 * 93600 * 6144 / (2 * 93600 * 195 + 2 * (256 * 3072 + 3072 * 384) * 2),
     2 * 93600 * 6144 / (2 * 93600 * 195 + 2 * (256 * 3072 + 3072 * 384) * 2 + 2 * 384 * 3072 * 2)),
    ("step30", 3072 / 99, 2 * 46800 * 3072 / (2 * 46800 * 99 + 1572864),
     2 * 46800 * 3072 / (2 * 46800 * 99 + 1572864 + 1179648)),
])
def test_storage_accounting(name, per_token, effective, with_encoder):
    st = bench.storage_block(WORKLOADS[name])
    assert st["per_token_ratio"] == pytest.approx(per_token, abs=0.01)
    assert st["effective_ratio"] == pytest.approx(effective, abs=0.01)
    assert st["effective_ratio_with_encoder"] == pytest.approx(with_encoder, abs=0.01)
    assert st["history_tokens"] == WORKLOADS[name].T
