"""Compressed-history attention sharded over several GPUs, one process per
GPU (torch.distributed for the exchange, NCCL on GPUs).

The method's pages describe a single device; the attention shards two
natural ways, both exact up to rounding:

* by history: rank r holds a contiguous range of the history tokens and
  attends it (and rank 0 the current chunk) into an fp32 partial (O, LSE);
  one all-gather of the partials, then the LSE merge of Fig. 4(d) -- the
  identity that merging a split history equals attending the concatenation.
  The fixed routing (the most recent T_full tokens full-dim) is applied per
  range: a range's full-dim tokens are its overlap with the last T_full.
* by head: rank r attends heads [h0, h1) with the heads' slices of the
  codecs and queries; the compressed history is joint over the heads, so
  every rank holds all of it.  One all-gather of the outputs.

Every attention and merge runs in the library's kernels (`LibraryOps`); the
orchestration takes its attend / merge calls from an `ops` object so that
the same code runs with other implementations of those two calls.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


def history_shard(T: int, T_full: int, world: int, rank: int) -> tuple[int, int, int]:
    """(lo, hi, local_T_full): rank's contiguous history tokens [lo, hi) --
    near-equal ranges in token order -- and how many of them are among the
    most recent T_full of the whole history (a suffix of the range)."""
    lo = (T * rank) // world
    hi = (T * (rank + 1)) // world
    local_full = max(0, hi - max(lo, T - T_full))
    return lo, hi, local_full


def head_shard(H: int, world: int, rank: int) -> tuple[int, int]:
    """Rank's heads [h0, h1): near-equal ranges in head order."""
    return (H * rank) // world, (H * (rank + 1)) // world


@dataclass
class LibraryOps:
    """The library's calls: attend_partial -> fp32 (O, LSE) over the given
    keys; merge -> nanokv_lse_merge of the partials; attend -> nanokv_attend."""

    def attend_partial(self, q, ck, cv, hk, hv, T_full, k_cur, v_cur, tau):
        from . import _lib
        return _lib.nanokv_attend_partial(q, ck, cv, hk, hv, T_full, k_cur, v_cur, softmax_scale=tau)

    def merge(self, Os, Ls, out_dtype):
        from . import _lib
        return _lib.nanokv_lse_merge(Os, Ls, out_dtype=out_dtype)

    def attend(self, q, ck, cv, hk, hv, T_full, k_cur, v_cur, tau):
        from . import _lib
        return _lib.nanokv_attend(q, ck, cv, hk, hv, T_full, k_cur, v_cur, softmax_scale=tau)

    def slice_hist(self, h, lo, hi):
        return h.slice(lo, hi) if h is not None and hi > lo else None

    def head_codec(self, c, h0, h1):
        from . import _lib
        d = c.d
        return _lib.Codec(h1 - h0, d, c.centers[:, h0 * d:h1 * d].contiguous(), c.D[h0 * d:h1 * d].contiguous())


def _gather(t: torch.Tensor, group) -> list[torch.Tensor]:
    import torch.distributed as dist
    world = dist.get_world_size(group)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return parts


def history_partial(q, ck, cv, hk, hv, T: int, T_full: int, k_cur, v_cur, world: int, rank: int,
                    tau: float | None = None, ops=None):
    """This rank's fp32 partial (O, LSE): its history range (routed by the
    global T_full) and, on rank 0, the current chunk."""
    ops = ops or LibraryOps()
    if tau is None:
        tau = 1.0 / math.sqrt(q.shape[-1])
    lo, hi, local_full = history_shard(T, T_full, world, rank)
    cur_k, cur_v = (k_cur, v_cur) if rank == 0 else (None, None)
    return ops.attend_partial(q, ck, cv, ops.slice_hist(hk, lo, hi), ops.slice_hist(hv, lo, hi), local_full,
                              cur_k, cur_v, tau)


def attend_history_sharded(q, ck, cv, hk, hv, T: int, T_full: int, k_cur=None, v_cur=None, group=None,
                           tau: float | None = None, ops=None):
    """Attention of q over a history sharded by token range across the ranks
    of `group` (every rank passes its own range's compressed history hk, hv,
    i.e. tokens history_shard(T, T_full, world, rank)[:2], and the same q and
    current chunk).  Returns (out, lse) on every rank."""
    import torch.distributed as dist
    ops = ops or LibraryOps()
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    if tau is None:
        tau = 1.0 / math.sqrt(q.shape[-1])
    lo, hi, local_full = history_shard(T, T_full, world, rank)
    cur_k, cur_v = (k_cur, v_cur) if rank == 0 else (None, None)
    O, L = ops.attend_partial(q, ck, cv, hk, hv, local_full, cur_k, cur_v, tau)
    return ops.merge(_gather(O, group), _gather(L, group), q.dtype)


def attend_head_sharded(q, ck, cv, hk, hv, T_full: int, k_cur=None, v_cur=None, group=None,
                        tau: float | None = None, ops=None):
    """Attention sharded by head across the ranks of `group`: every rank
    passes the full q, codecs, compressed history and current chunk, attends
    its heads head_shard(H, world, rank) and receives every head's output.
    Returns (out [Tq, H, d], lse [H, Tq]) on every rank."""
    import torch.distributed as dist
    ops = ops or LibraryOps()
    world, rank = dist.get_world_size(group), dist.get_rank(group)
    Tq, H, d = q.shape
    if tau is None:
        tau = 1.0 / math.sqrt(d)
    h0, h1 = head_shard(H, world, rank)
    if H % world:
        raise ValueError(f"head sharding needs H ({H}) divisible by the world size ({world})")
    sub = lambda x: x[:, h0:h1].contiguous() if x is not None else None  # noqa: E731
    O, L = ops.attend(sub(q), ops.head_codec(ck, h0, h1), ops.head_codec(cv, h0, h1), hk, hv, T_full, sub(k_cur),
                      sub(v_cur), tau)
    Os, Ls = _gather(O, group), _gather(L, group)
    return torch.cat(Os, dim=1), torch.cat(Ls, dim=0)
