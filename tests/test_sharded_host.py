"""Host logic of the sharded attention (compressed_history_attention_b200.sharded)
on CPU with two gloo ranks: the shard ranges, the per-range routing of the
most recent T_full tokens, the current chunk on rank 0 only, the all-gather
of the partials and their merge, and head sharding with its gather.  The
attend / merge calls are the oracle's (the library's need a GPU); the
result must equal the oracle's attention over the whole history."""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(seed=7, H=4, d=8, r=6, C=5, T=53, Tq=6, Tc=5):
    rng = np.random.default_rng(seed)
    J = H * d
    ck = {"centers": rng.standard_normal((C, J)), "D": rng.standard_normal((J, r)) / np.sqrt(r)}
    cv = {"centers": rng.standard_normal((C, J)), "D": rng.standard_normal((J, r)) / np.sqrt(r)}

    def hist():
        return {"ids": rng.integers(0, C, T), "codes": rng.integers(-7, 8, (T, r)), "scales": rng.uniform(0.05, 0.6, T)}
    return {"ck": ck, "cv": cv, "hk": hist(), "hv": hist(), "q": rng.standard_normal((Tq, H, d)),
            "kc": rng.standard_normal((Tc, H, d)), "vc": rng.standard_normal((Tc, H, d)), "T": T, "d": d}


def _ops(d):
    import torch
    from oracle import nanokv_oracle as orc
    np_ = lambda t: None if t is None else (t.numpy() if hasattr(t, "numpy") else t)  # noqa: E731

    class OracleOps:
        def attend_partial(self, q, ck, cv, hk, hv, T_full, k_cur, v_cur, tau):
            if hk is None:
                hk = hv = {"ids": np.zeros(0, np.int64), "codes": np.zeros((0, ck["D"].shape[1])),
                           "scales": np.zeros(0)}
            O, L = orc.attend(np_(q), ck, cv, hk, hv, T_full, np_(k_cur), np_(v_cur), tau)
            return torch.from_numpy(O), torch.from_numpy(L)

        attend = attend_partial

        def merge(self, Os, Ls, out_dtype):
            O, L = orc.lse_merge([(o.numpy(), l.numpy()) for o, l in zip(Os, Ls)])
            return torch.from_numpy(O), torch.from_numpy(L)

        def slice_hist(self, h, lo, hi):
            return orc.split_history(h, lo, hi) if hi > lo else None

        def head_codec(self, c, h0, h1):
            return {"centers": c["centers"][:, h0 * d:h1 * d], "D": c["D"][h0 * d:h1 * d]}
    return OracleOps()


def _worker(rank, world, port, q, T_full):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch
    import torch.distributed as dist
    from compressed_history_attention_b200 import sharded
    from oracle import nanokv_oracle as orc
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        p = _problem()
        ops = _ops(p["d"])
        tau = 0.4
        qt, kc, vc = (torch.from_numpy(p[k]) for k in ("q", "kc", "vc"))
        lo, hi, _ = sharded.history_shard(p["T"], T_full, world, rank)
        O1, L1 = sharded.attend_history_sharded(qt, p["ck"], p["cv"], ops.slice_hist(p["hk"], lo, hi),
                                                ops.slice_hist(p["hv"], lo, hi), p["T"], T_full, kc, vc, tau=tau,
                                                ops=ops)
        O2, L2 = sharded.attend_head_sharded(qt, p["ck"], p["cv"], p["hk"], p["hv"], T_full, kc, vc, tau=tau, ops=ops)
        Or, Lr = orc.attend(p["q"], p["ck"], p["cv"], p["hk"], p["hv"], T_full, p["kc"], p["vc"], tau)
        err = (float(np.abs(O1.numpy() - Or).max()), float(np.abs(L1.numpy() - Lr).max()),
               float(np.abs(O2.numpy() - Or).max()), float(np.abs(L2.numpy() - Lr).max()))
        dist.barrier()
    finally:
        dist.destroy_process_group()
    q.put((rank, err))


@pytest.mark.parametrize("T_full", [0, 10, 40, 53])
def test_sharded_attention_gloo_world2(T_full):
    """History split 26 / 27 tokens; T_full = 10 lies in rank 1's range, 40
    crosses the boundary, 0 and 53 are the all-low and all-full cases."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, T_full)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = dict(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    for r in (0, 1):
        assert max(res[r]) < 1e-12, res[r]


def test_shard_ranges():
    from compressed_history_attention_b200.sharded import head_shard, history_shard
    assert [history_shard(53, 40, 2, r) for r in (0, 1)] == [(0, 26, 13), (26, 53, 27)]
    assert [history_shard(53, 10, 2, r) for r in (0, 1)] == [(0, 26, 0), (26, 53, 10)]
    assert [history_shard(10, 10, 4, r)[:2] for r in range(4)] == [(0, 2), (2, 5), (5, 7), (7, 10)]
    assert sum(history_shard(93600, 9360, 8, r)[2] for r in range(8)) == 9360
    assert [head_shard(12, 4, r) for r in range(4)] == [(0, 3), (3, 6), (6, 9), (9, 12)]
