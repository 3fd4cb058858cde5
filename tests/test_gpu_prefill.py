"""Prefill (multi-query) attention over a TurboQuant K/V cache through the C
ABI, against the oracle's causal attention: a block of nq new tokens at the
end of a context of T tokens, token i attending keys t <= T - nq + i.  The
bound per output row is the decode bound (the score bound 1e-4 ||q|| ||k||
propagated through the softmax, plus 1e-3 relative for the fp16 operands)."""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import turboquant as oq

from cases import DEV, assert_status_clean, bf16_exact, decode_cache, to_device

import compressed_kv_cache_turboquant_b200 as tq

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


def _prefill_case(B, nq, Hq, Hkv, T, sample, seed, stride_extra=0):
    d = 128
    hk, hv, c, _, refs = decode_cache(B, Hq, Hkv, T, d, sample, seed=seed, stride_extra=stride_extra)
    S = T + stride_extra
    q64 = bf16_exact(synth.rng(seed, synth.QUERY, 77).standard_normal((B, nq, Hq, d)) *
                     synth.lognormal_channel_scales(d, 1.0, seed, 20)[None, None, None, :])
    q = to_device(q64, torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    out = torch.full((B, nq, Hq, d), float("nan"), dtype=torch.float32, device=DEV)
    tq.tq_attn_prefill(hk.h, hv.h, q, Hkv, T, S, c["kcodes"], c["ksigns"], c["knorms"], c["krnorms"], c["vcodes"],
                       c["vnorms"], scale, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    g = Hq // Hkv
    for (b, h), (kst, vhat) in refs.items():
        qs = q64[b, :, h * g:(h + 1) * g]                          # [nq, g, d]
        est = lambda _b, _h, rows: oq.prod_estimate(rows, kst["idx"], kst["norms"], kst["signs"], kst["rnorms"],
                                                    hk.Pi_o, hk.S, hk.c_o, 4)
        ref = oq.attention_prefill(qs[None], est, lambda _b, _h: vhat, 1, T, scale=scale)[0]   # [nq, g, d]
        rows = qs.reshape(nq * g, d)
        logits = est(0, 0, rows) * scale
        kn = np.asarray(kst["norms"], dtype=np.float64)
        for i in range(nq):
            vis = T - nq + i + 1
            for j in range(g):
                lg = logits[i * g + j, :vis]
                p = np.exp(lg - lg.max())
                p /= p.sum()
                r = ref[i, j]
                eps = scale * 1e-4 * np.linalg.norm(qs[i, j]) * kn[:vis]
                spread = np.linalg.norm(vhat[:vis] - r[None, :], axis=1)
                tol = 2 * np.sum(p * eps * spread) + 1e-3 * np.linalg.norm(r)
                err = np.linalg.norm(got[b, i, h * g + j] - r)
                assert err <= tol, (b, h, i, j, err, tol)
    assert np.all(np.isfinite(got))
    assert_status_clean(hk, hv)


def test_prefill_ragged_query_tiles():
    # g = 4: 32 tokens per 128-row tile; 300 tokens = nine full tiles and a ragged one
    _prefill_case(B=2, nq=300, Hq=8, Hkv=2, T=3000, sample=[(0, 1), (1, 0)], seed=1, stride_extra=4)


@pytest.mark.parametrize("Hq,Hkv,nq", [(2, 2, 129), (16, 2, 40)])
def test_prefill_group_sizes(Hq, Hkv, nq):
    # one query head per kv-head (128 tokens per tile) and eight (16 tokens per tile)
    _prefill_case(B=1, nq=nq, Hq=Hq, Hkv=Hkv, T=1500, sample=[(0, 1)], seed=2)


def test_prefill_whole_prompt():
    # no earlier context: the block is the whole cache, token 0 sees only itself
    _prefill_case(B=1, nq=700, Hq=8, Hkv=2, T=700, sample=[(0, 0)], seed=3)


def test_prefill_empty_context_slices_and_ragged_tail():
    """nq = 600 of T = 1203 in rows of 1204 (the row stride stays a multiple of
    four; the 3-token tail past the last whole group of four has its norms read
    from global memory): with two context slices per query tile, the early
    tokens' tiles see no key of the second slice, so those CTAs write empty
    softmax records (m = -inf, l = 0) that the merge must ignore, and tiles of
    several keys run through both logit buffers."""
    _prefill_case(B=1, nq=600, Hq=4, Hkv=1, T=1203, sample=[(0, 0)], seed=4, stride_extra=1)


def test_prefill_config4_cache_sampled():
    """A block of 128 tokens at the end of the decode configuration's cache
    (B = 8, Hq = 32, Hkv = 8, d = 128, T = 131072): the full launch, one
    (batch, kv-head) slice checked against the oracle."""
    _prefill_case(B=8, nq=128, Hq=32, Hkv=8, T=131072, sample=[(3, 5)], seed=0)
