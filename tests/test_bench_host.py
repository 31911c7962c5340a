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


@pytest.mark.parametrize("name", ["full", "mixed", "step30"])
def test_work_as_run_equals_named_where_low_dim_kernel_exists(name):
    _, (af, ak, _, _) = _work(name)
    assert ak == af


def test_long_work_as_run_is_full_dim():
    """r = 384 > d = 128 and 256 centers: no low-dim tensor-core kernel, so
    every history token is attended full-dim; that is less arithmetic than
    the named low-dim split, and the throughput numerator counts it."""
    w, (af, ak, _, _) = _work("long")
    assert ak["low"] == 0
    assert ak["full"] == 4 * w.Tq * w.T * w.J + 4 * w.T * w.J * w.r
    assert ak["total"] / 1e12 == pytest.approx(6.093, rel=1e-3)
    assert ak["total"] < af["total"]
