"""A paged TurboQuant cache through the C ABI: quantize-on-write into slots of
a paged cache, decode attention through a block table, and the residual norm
stored as one FP16 scalar, each against the float64 oracle."""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import turboquant as oq

from cases import (DEV, Instance, assert_status_clean, bf16_exact, compare_codes, compare_signs, decode_cache,
                   decode_tolerance, rel_err, to_device, words_u32)

import compressed_kv_cache_turboquant_b200 as tq

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


@pytest.mark.parametrize("variant,b,rn16", [(tq.TQ_PROD, 4, False), (tq.TQ_PROD, 4, True), (tq.TQ_MSE, 4, False),
                                            (tq.TQ_PROD, 3, True)])
def test_quantize_on_write_into_slots(variant, b, rn16):
    """1000 bf16 vectors (d = 128) written to scattered rows of a 5000-row cache;
    untouched rows keep their contents."""
    d, N, rows = 128, 1000, 5000
    inst = Instance(d, b, variant, seed=3)
    x64 = bf16_exact(synth.scaled_gaussian_rows(N, d, 1.0, seed=3))
    slots = torch.tensor(synth.rng(3, 7).choice(rows, N, replace=False).astype(np.int64), device=DEV)
    out = inst.alloc_outputs(rows)
    if inst.prod and rn16:
        out["rnorms"] = torch.zeros(rows, dtype=torch.float16, device=DEV)
    tq.tq_quant_paged(inst.h, to_device(x64, torch.bfloat16), slots, out["codes"], out["norms"],
                      signs=out.get("signs"), rnorms=out.get("rnorms"))
    torch.cuda.synchronize()
    s = slots.cpu().numpy()
    ref = inst.oracle_quant(x64)
    exact, _ = compare_codes(words_u32(out["codes"])[s], ref["idx"], ref["y"], inst.t_o, d, inst.bm)
    assert np.max(rel_err(out["norms"].cpu().numpy()[s], ref["norms"])) <= 1e-5
    if inst.prod:
        compare_signs(words_u32(out["signs"])[s], ref["signs"], ref["Sr"], ref["norms"], exact)
        rn = out["rnorms"].float().cpu().numpy()[s]
        if rn16:
            # fp16 of the float32 result against fp16 of the float64 norm: at most one fp16 step apart
            want = ref["rnorms"].astype(np.float16).astype(np.float64)
            assert np.max(rel_err(rn[exact], want[exact])) <= 2.0 ** -10
        else:
            assert np.max(rel_err(rn[exact], ref["rnorms"][exact])) <= 1e-5
    untouched = np.setdiff1d(np.arange(rows), s)
    assert int(out["codes"][torch.tensor(untouched, device=DEV)].abs().sum()) == 0
    assert_status_clean(inst)


def test_quantize_on_write_gathers_a_channel_group():
    """One channel group (64 of 128 channels) of 600 arriving tokens, fp32 input."""
    d_in, N, rows = 128, 600, 2048
    inst = Instance(64, 3, tq.TQ_PROD, seed=5, sub=(1,))
    ch = np.sort(synth.rng(5, 2).choice(d_in, 64, replace=False)).astype(np.int32)
    x64 = synth.scaled_gaussian_rows(N, d_in, 1.0, seed=5)
    slots = torch.tensor(synth.rng(5, 3).choice(rows, N, replace=False).astype(np.int64), device=DEV)
    out = inst.alloc_outputs(rows)
    tq.tq_quant_paged(inst.h, to_device(x64, torch.float32), slots, out["codes"], out["norms"],
                      signs=out["signs"], rnorms=out["rnorms"], channels=torch.tensor(ch, device=DEV))
    torch.cuda.synchronize()
    s = slots.cpu().numpy()
    ref = inst.oracle_quant(x64[:, ch])
    exact, _ = compare_codes(words_u32(out["codes"])[s], ref["idx"], ref["y"], inst.t_o, 64, inst.bm)
    compare_signs(words_u32(out["signs"])[s], ref["signs"], ref["Sr"], ref["norms"], exact)
    assert np.max(rel_err(out["norms"].cpu().numpy()[s], ref["norms"])) <= 1e-5
    assert_status_clean(inst)


def _paginate(c, B, Hkv, T, page, seed, spare=3):
    """Scatter a dense [B*Hkv][T] cache into pages of `page` rows in a shuffled
    pool (with spare pages never referenced); returns (paged arrays, block table)."""
    per = (T + page - 1) // page
    pool = B * Hkv * per + spare
    perm = synth.rng(seed, 50).permutation(pool)[: B * Hkv * per].reshape(B * Hkv, per)
    table = torch.tensor(perm.astype(np.int32), device=DEV)
    t = np.arange(T)
    rows = (perm[:, t // page] * page + t % page).reshape(-1)      # [B*Hkv*T] paged row of each dense row
    idx = torch.tensor(rows, device=DEV)
    paged = {}
    for k, v in c.items():
        p = torch.zeros((pool * page, *v.shape[1:]), dtype=v.dtype, device=DEV)
        p[idx] = v
        paged[k] = p
    return paged, table


@pytest.mark.parametrize("page,rn16,Hq", [(16, False, 32), (64, True, 32), (256, False, 32), (64, True, 16)])
def test_paged_decode_matches_oracle(monkeypatch, page, rn16, Hq):
    # Hq = 32 takes the mma.sync decode (the paged kernel), Hq = 16 (2 q-heads
    # per kv-head) the general kernel.  The handles take the mma.sync kernel
    # for dense caches as well, so the paged result can be compared with the
    # dense one of the same arithmetic (only the addressing differs).
    monkeypatch.delenv("TQ_TCGEN05_ATTN", raising=False)
    B, Hkv, T, d = 2, 8, 9000, 128
    sample = [(0, 2), (1, 5)]
    hk, hv, c, q64, refs = decode_cache(B, Hq, Hkv, T, d, sample, seed=9)
    if rn16:
        c["krnorms"] = c["krnorms"].to(torch.float16)
        refs = {k: (dict(kst, rnorms=kst["rnorms"].astype(np.float16)), vh) for k, (kst, vh) in refs.items()}
    paged, table = _paginate(c, B, Hkv, T, page, seed=page)
    q = to_device(q64, torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=DEV)
    tq.tq_attn_decode_paged(hk.h, hv.h, q, Hkv, T, table, page, paged["kcodes"], paged["ksigns"], paged["knorms"],
                            paged["krnorms"], paged["vcodes"], paged["vnorms"], scale, out)
    torch.cuda.synchronize()
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
    if not rn16:
        dense = torch.empty_like(out)
        tq.tq_attn_decode(hk.h, hv.h, q, Hkv, T, T, c["kcodes"], c["ksigns"], c["knorms"], c["krnorms"], c["vcodes"],
                          c["vnorms"], scale, dense)
        torch.cuda.synchronize()
        assert torch.allclose(out, dense, rtol=1e-5, atol=1e-6)
    assert_status_clean(hk, hv)
