"""A cache split across devices, on CPU: two gloo ranks.

Each rank holds a contiguous slice of the context (decode) or of the database
(search).  The rank plumbing of ``compressed_kv_cache_turboquant_b200.sharded``
-- the slice ranges, the all-gather of the per-slice records and of the slice
offsets, in rank order on every rank -- is exercised here with the oracle
computing each slice's record (the library's kernels need a GPU; their merge is
compared with the oracle in tests/test_gpu_sharded.py).  The merged result
must equal the oracle's answer over the whole context or database.
"""
import math
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_ranges_cover_everything_once():
    sys.path.insert(0, ROOT)
    from compressed_kv_cache_turboquant_b200.sharded import shard_range
    for n in (0, 1, 7, 1000, 131072):
        for world in (1, 2, 3, 8):
            parts = [shard_range(n, world, r) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            assert all(parts[r][1] == parts[r + 1][0] for r in range(world - 1))
            sizes = [hi - lo for lo, hi in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_range(10, 2, 2)


def _rank_main(rank: int, world: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import datetime

    import torch
    import torch.distributed as dist

    import synth
    from oracle import turboquant as oq
    from compressed_kv_cache_turboquant_b200 import sharded

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # ---- decode: context T split across the ranks; oracle records per slice
        B, Hq, Hkv, T, d = 2, 8, 2, 301, 16
        r = synth.rng(11, 0)
        k = r.standard_normal((B, Hkv, T, d))
        v = r.standard_normal((B, Hkv, T, d))
        q = r.standard_normal((B, Hq, d)) * 2
        lo, hi = sharded.shard_range(T, world, rank)
        m, l, acc = oq.attention_partial(q, lambda b, h, qs: qs @ k[b, h, lo:hi].T, lambda b, h: v[b, h, lo:hi], Hkv)
        rec = torch.from_numpy(np.concatenate([acc.reshape(B * Hq, d), m.reshape(-1, 1), l.reshape(-1, 1)], axis=1))
        allrec = sharded.all_gather_stacked(rec).numpy()          # [world][B*Hq][d + 2]
        merged = oq.merge_attention_partials(allrec[:, :, d], allrec[:, :, d + 1], allrec[:, :, :d])
        full, _ = oq.attention_decode(q, lambda b, h, qs: qs @ k[b, h].T, lambda b, h: v[b, h], Hkv)
        dec_err = float(np.max(np.abs(merged.reshape(B, Hq, d) - full)))

        # ---- search: N keys split across the ranks; local top-k, global merge
        N, nq, kk = 523, 6, 10
        keys = r.standard_normal((N, d))
        qs = r.standard_normal((nq, d))
        a, e = sharded.shard_range(N, world, rank)
        li, lv = oq.topk(qs @ keys[a:e].T, kk)
        offs = sharded.gather_offsets(a, "cpu")
        vals = sharded.all_gather_stacked(torch.from_numpy(lv)).numpy()
        idxs = sharded.all_gather_stacked(torch.from_numpy(li.astype(np.int64))).numpy()
        cand_v = np.concatenate([vals[s] for s in range(world)], axis=1)
        cand_i = np.concatenate([idxs[s] + offs[s] for s in range(world)], axis=1)
        order = np.lexsort((cand_i, -cand_v), axis=1)[:, :kk]
        gi = np.take_along_axis(cand_i, order, axis=1)
        ei, _ = oq.topk(qs @ keys.T, kk)
        out.put((rank, dec_err, offs, bool(np.array_equal(gi, ei))))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_merge_slices_to_the_whole():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(i, world, port, q)) for i in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, dec_err, offs, same in got:
        assert dec_err < 1e-12, dec_err
        assert offs == [0, 523 // 2]
        assert same
