"""Decode attention and nearest-neighbour search over a cache split across
GPUs: one process per GPU, the library's per-slice calls, one all-gather over
``torch.distributed`` (NCCL between GPUs), and the library's merges.

Decode: every rank holds a contiguous slice of the context of every (batch,
kv-head) and runs ``tq_attn_decode_partial`` on it; the [B*Hq][d + 2] softmax
records (about 133 KB per rank at batch 8, 32 heads, d = 128) are all-gathered
and ``tq_attn_merge`` combines them and rotates back once, on every rank.

Search: every rank holds a contiguous slice of the database keys, scores it
with its own top-k (``tq_ip_scores``), and the [nq][k] candidate lists are
all-gathered and merged by ``tq_topk_merge`` into the global top-k.

Every rank takes the same collective steps in the same order.  The
exchange is small next to the slice's own work, so it is a plain NCCL
collective on the caller's stream.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import api


def shard_range(n: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous slice [lo, hi) of n items held by `rank` of `world` (sizes
    differ by at most one)."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError(f"shard_range(n={n}, world={world}, rank={rank})")
    return n * rank // world, n * (rank + 1) // world


def all_gather_stacked(t: torch.Tensor, group=None) -> torch.Tensor:
    """[world, *t.shape]: every rank's tensor, in rank order."""
    world = dist.get_world_size(group)
    t = t.contiguous()
    out = torch.empty((world, *t.shape), dtype=t.dtype, device=t.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, t, group=group)
    else:
        dist.all_gather(list(out.unbind(0)), t, group=group)
    return out


def gather_offsets(first: int, device, group=None) -> list[int]:
    """The first global index of every rank's slice, in rank order."""
    t = torch.tensor([int(first)], dtype=torch.int64, device=device)
    return [int(v) for v in all_gather_stacked(t, group).reshape(-1).cpu().tolist()]


def sharded_attn_decode(hk, hv, q: torch.Tensor, Hkv: int, T_local: int, kv_stride: int, kcodes, ksigns, knorms,
                        krnorms, vcodes, vnorms, scale: float, out: torch.Tensor, group=None, workspace=None,
                        stream=None) -> None:
    """One decode step whose context is split across the ranks of `group`:
    this rank's cache arrays hold T_local tokens of every (batch, kv-head)
    (layout of tq_attn_decode, T_local may be 0).  `out` [B][Hq][d] receives the
    attention over the whole context on every rank."""
    B, Hq, _ = q.shape
    d = out.shape[-1]
    partial = torch.empty((B * Hq, d + 2), dtype=torch.float32, device=q.device)
    api.tq_attn_decode_partial(hk, hv, q, Hkv, T_local, kv_stride, kcodes, ksigns, knorms, krnorms, vcodes, vnorms,
                               scale, partial, workspace=workspace, stream=stream)
    gathered = all_gather_stacked(partial, group)
    api.tq_attn_merge(hv, gathered, out.view(B * Hq, d), stream=stream)


def sharded_search(h, q: torch.Tensor, codes, signs, norms, rnorms, k: int, first: int, out_idx: torch.Tensor,
                   out_val: torch.Tensor, group=None, workspace=None, stream=None) -> None:
    """Top-k of every query over a database split across the ranks of `group`:
    this rank holds keys first .. first + len(norms) - 1 of the global
    numbering.  out_idx / out_val [nq][k] receive the global top-k (global
    indices, ties to the lower index) on every rank."""
    nq = q.shape[0]
    n_local = int(norms.shape[0])
    kk = min(k, n_local)
    ti = torch.full((nq, k), 2 ** 31 - 1, dtype=torch.int32, device=q.device)
    tv = torch.full((nq, k), -torch.finfo(torch.float32).max, dtype=torch.float32, device=q.device)
    if kk > 0:
        li = torch.empty((nq, kk), dtype=torch.int32, device=q.device)
        lv = torch.empty((nq, kk), dtype=torch.float32, device=q.device)
        api.tq_ip_scores(h, q, codes, signs, norms, rnorms, topk=kk, top_idx=li, top_val=lv, workspace=workspace,
                         stream=stream)
        ti[:, :kk] = li
        tv[:, :kk] = lv
    offsets = gather_offsets(first, q.device, group)
    vals = all_gather_stacked(tv, group)
    idxs = all_gather_stacked(ti, group)
    api.tq_topk_merge(vals, idxs, offsets, out_idx, out_val, stream=stream)
