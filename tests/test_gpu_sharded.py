"""The library's calls for a cache split across devices, on one GPU: the
ranks' slices are run one after another (their kernels never wait on each
other) and their records combined by the library's merges, through the C ABI.

Decode: the context of every (batch, kv-head) is cut into slices (one of them
empty); tq_attn_decode_partial on each slice, tq_attn_merge over the stacked
records, compared with the oracle's attention over the whole context.
Search: the database is cut into slices; tq_ip_scores keeps each slice's
top-k, tq_topk_merge makes the global list, checked against the oracle's
estimator over the whole database.
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import turboquant as oq

from cases import DEV, Instance, assert_status_clean, decode_cache, decode_tolerance, to_device, upload_words

import compressed_kv_cache_turboquant_b200 as tq
from compressed_kv_cache_turboquant_b200.sharded import shard_range

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


def _slice(c, B, Hkv, T, lo, hi):
    """Tokens [lo, hi) of every (batch, kv-head) as a cache of its own."""
    out = {}
    for k, t in c.items():
        v = t.view(B * Hkv, T, *t.shape[1:])[:, lo:hi]
        out[k] = v.reshape(B * Hkv * (hi - lo), *t.shape[1:]).contiguous()
    return out


@pytest.mark.parametrize("Hq,cuts", [(32, [0, 4000, 4000, 9001, 20011]), (16, [0, 7000, 20011])])
def test_context_split_decode_merges_to_the_whole(Hq, cuts):
    # Hq = 32 (4 q-heads per kv-head) runs the tensor-core decode; Hq = 16 the general kernel
    B, Hkv, T, d = 2, 8, 20011, 128
    sample = [(0, 3), (1, 7)]
    hk, hv, c, q64, refs = decode_cache(B, Hq, Hkv, T, d, sample, seed=7)
    q = to_device(q64, torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    recs = []
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        s = _slice(c, B, Hkv, T, lo, hi)
        part = torch.full((B * Hq, d + 2), float("nan"), dtype=torch.float32, device=DEV)
        tq.tq_attn_decode_partial(hk.h, hv.h, q, Hkv, hi - lo, hi - lo, s["kcodes"], s["ksigns"], s["knorms"],
                                  s["krnorms"], s["vcodes"], s["vnorms"], scale, part)
        recs.append(part)
    stacked = torch.stack(recs)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=DEV)
    tq.tq_attn_merge(hv.h, stacked, out.view(B * Hq, d))
    # the same context in one piece through the single-device call
    whole = torch.empty_like(out)
    tq.tq_attn_decode(hk.h, hv.h, q, Hkv, T, T, c["kcodes"], c["ksigns"], c["knorms"], c["krnorms"], c["vcodes"],
                      c["vnorms"], scale, whole)
    torch.cuda.synchronize()
    st = stacked.cpu().numpy()
    empty = [i for i, (a, e) in enumerate(zip(cuts[:-1], cuts[1:])) if a == e]
    for i in empty:
        assert np.all(st[i, :, d + 1] == 0) and np.all(st[i, :, :d] == 0)
    got = out.cpu().numpy()
    gsz = Hq // Hkv
    for (b, h), (kst, vhat) in refs.items():
        qs = q64[b, h * gsz:(h + 1) * gsz]
        est = lambda _b, _h, rows: oq.prod_estimate(rows, kst["idx"], kst["norms"], kst["signs"], kst["rnorms"],
                                                    hk.Pi_o, hk.S, hk.c_o, 4)
        ref_out, ref_logits = oq.attention_decode(qs[None], est, lambda _b, _h: vhat, 1, scale=scale)
        ref = ref_out[0]
        tol = decode_tolerance(ref, ref_logits[(0, 0)], qs, kst, vhat, scale)
        err = np.linalg.norm(got[b, h * gsz:(h + 1) * gsz] - ref, axis=1)
        assert np.all(err <= tol), (b, h, err, tol)
    rel = np.linalg.norm(got - whole.cpu().numpy(), axis=2) / np.linalg.norm(whole.cpu().numpy(), axis=2)
    assert np.max(rel) < 2e-3
    assert_status_clean(hk, hv)


def test_database_split_search_merges_to_the_global_top_k():
    d, N, nq, k, world = 200, 30011, 64, 10, 3
    inst = Instance(d, 4, tq.TQ_PROD, seed=5)
    x64 = synth.unit_rows(N, d, 5)
    q64 = synth.unit_rows(nq, d, 5, stream=synth.QUERY)
    st = inst.oracle_quant(x64)
    codes = upload_words(oq.pack_codes_vec(st["idx"], inst.bm))
    signs = upload_words(oq.pack_signs(st["signs"]))
    norms = torch.tensor(st["norms"], device=DEV)
    rnorms = torch.tensor(st["rnorms"], device=DEV)
    q = to_device(q64, torch.float32)
    vals, idxs, offs = [], [], []
    for r in range(world):
        lo, hi = shard_range(N, world, r)
        ti = torch.empty((nq, k), dtype=torch.int32, device=DEV)
        tv = torch.empty((nq, k), dtype=torch.float32, device=DEV)
        # each rank holds its slice in arrays of its own
        tq.tq_ip_scores(inst.h, q, codes[lo:hi].clone(), signs[lo:hi].clone(), norms[lo:hi].clone(),
                        rnorms[lo:hi].clone(), topk=k, top_idx=ti, top_val=tv)
        vals.append(tv)
        idxs.append(ti)
        offs.append(lo)
    gi = torch.empty((nq, k), dtype=torch.int32, device=DEV)
    gv = torch.empty((nq, k), dtype=torch.float32, device=DEV)
    tq.tq_topk_merge(torch.stack(vals), torch.stack(idxs), offs, gi, gv)
    torch.cuda.synchronize()
    gi, gv = gi.cpu().numpy(), gv.cpu().numpy()
    ref = oq.prod_estimate(q64, st["idx"], st["norms"], st["signs"], st["rnorms"], inst.Pi_o, inst.S, inst.c_o, 4)
    for r in range(nq):
        tol = 1e-4 * np.linalg.norm(q64[r]) * np.linalg.norm(x64, axis=1)
        assert len(set(gi[r].tolist())) == k and np.all(np.diff(gv[r]) <= 0)
        assert np.all(np.abs(gv[r] - ref[r, gi[r]]) <= tol[gi[r]]), r
        rest = np.ones(N, bool)
        rest[gi[r]] = False
        assert np.max(ref[r, rest]) <= gv[r, -1] + 2 * np.max(tol), r
    assert_status_clean(inst)
