"""GPU parity of every hot-path call against the float64 oracle.

Codes: bit-exact except coordinates whose oracle rotated value lies within
1e-5/sqrt(d) of a decision threshold (at most 1e-4 of all coordinates).
QJL signs: bit-exact on vectors whose mse codes match, except |(S r)_j| <=
1e-5 ||x|| (the same 1e-5/sqrt(d) band in the unit frame of x, with S's rows
normalised to unit length).  Reconstructions: relative L2 <= 1e-5.  Scores: |delta| <=
1e-4 ||q|| ||k|| against the oracle estimator on the same (oracle) codes.
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import turboquant as oq

from cases import (DEV, Instance, assert_status_clean, bf16_exact, compare_codes, compare_signs, decode_cache,
                   decode_tolerance, rel_err, rel_l2_rows, to_device, upload_words, words_u32)

import compressed_kv_cache_turboquant_b200 as tq

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

NORM_RTOL = 1e-5


def _check_quant(inst: Instance, x64: np.ndarray, out: dict, rows=None):
    rows = np.arange(x64.shape[0]) if rows is None else rows
    ref = inst.oracle_quant(x64[rows])
    codes = words_u32(out["codes"])[rows]
    exact, _ = compare_codes(codes, ref["idx"], ref["y"], inst.t_o, inst.d, inst.bm)
    norms = out["norms"].cpu().numpy()[rows]
    assert np.max(rel_err(norms, ref["norms"])) <= NORM_RTOL
    if inst.prod:
        compare_signs(words_u32(out["signs"])[rows], ref["signs"], ref["Sr"], ref["norms"], exact)
        rn = out["rnorms"].cpu().numpy()[rows]
        assert np.max(rel_err(rn[exact], ref["rnorms"][exact])) <= NORM_RTOL
    assert_status_clean(inst)
    return ref, exact


# ------------------------------------------------------------------ quantize

@pytest.mark.parametrize("variant,b", [(tq.TQ_MSE, 2), (tq.TQ_PROD, 3), (tq.TQ_MSE, 1), (tq.TQ_MSE, 4)])
def test_pr1_fp32_quantize(variant, b):
    """N = 4096 fp32, d = 128, N(0,1) x lognormal(0, 0.5) channel scales, seed 0."""
    inst = Instance(128, b, variant)
    x64 = synth.scaled_gaussian_rows(4096, 128, 0.5, seed=0)
    out = inst.alloc_outputs(4096)
    inst.gpu_quant(to_device(x64, torch.float32), out)
    torch.cuda.synchronize()
    _check_quant(inst, x64, out)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_sweep_bf16_full_size_sampled(b):
    """N = 2^20 bf16, d = 128, lognormal(0, 1) scales, 4 channels x20 outliers;
    the whole batch on the GPU, the oracle on sampled rows and the tail."""
    N, d = 1 << 20, 128
    inst = Instance(d, b, tq.TQ_MSE)
    x64 = bf16_exact(synth.scaled_gaussian_rows(N, d, 1.0, seed=0, outliers=4))
    out = inst.alloc_outputs(N)
    inst.gpu_quant(to_device(x64, torch.bfloat16), out)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([synth.rng(9, b).choice(N, 3000, replace=False), np.arange(N - 40, N)]))
    _check_quant(inst, x64, out, rows)
    # dequantized batch on the GPU: mean relative MSE close to the closed-form D(b, d)
    xh = torch.empty((N, d), dtype=torch.float32, device=DEV)
    tq.tq_dequant_mse(inst.h, out["codes"], out["norms"], xh)
    xt = to_device(x64, torch.float32)
    rel = ((xt - xh).square().sum(1) / xt.square().sum(1)).mean().item()
    from oracle import codebook as ocb
    D = ocb.distortion(inst.c_o, d)
    assert abs(rel / D - 1) < 0.05, (rel, D)


@pytest.mark.parametrize("d", [64, 128, 200])
@pytest.mark.parametrize("N", [1, 33, 1000])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_quantize_shapes(d, N, dtype):
    for variant, b in [(tq.TQ_MSE, 3), (tq.TQ_PROD, 4), (tq.TQ_PROD, 2)]:
        inst = Instance(d, b, variant, seed=d + N)
        x64 = synth.scaled_gaussian_rows(N, d, 1.0, seed=N)
        if dtype == torch.bfloat16:
            x64 = bf16_exact(x64)
        out = inst.alloc_outputs(N)
        inst.gpu_quant(to_device(x64, dtype), out)
        torch.cuda.synchronize()
        _check_quant(inst, x64, out)


def test_zero_vectors_strides_and_slots():
    d, N, stride, slots = 128, 50, 136, 3
    inst = Instance(d, 4, tq.TQ_PROD, seed=5)
    x64 = synth.scaled_gaussian_rows(N, d, 1.0, seed=5)
    x64[[0, 17, 49]] = 0.0
    xp = np.zeros((N, stride))
    xp[:, :d] = x64
    out = inst.alloc_outputs(N, slots=N * slots)
    inst.gpu_quant(to_device(xp, torch.float32), out, out_stride=slots)
    torch.cuda.synchronize()
    sub = {k: v[::slots] for k, v in out.items()}
    ref, _ = _check_quant(inst, x64, sub)
    assert np.all(sub["norms"].cpu().numpy()[[0, 17, 49]] == 0)
    assert np.all(sub["rnorms"].cpu().numpy()[[0, 17, 49]] == 0)
    # untouched slots stay zero
    other = out["codes"].view(N, slots, -1)[:, 1:]
    assert int(other.abs().sum()) == 0


@pytest.mark.parametrize("d", [64, 128, 200])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("variant,b", [(tq.TQ_MSE, 3), (tq.TQ_PROD, 4)])
def test_zero_vectors_every_path(d, dtype, variant, b):
    """Zero rows among ordinary ones: y := 0 takes the cell above the middle
    threshold, x_hat = 0, every QJL bit set, rn = 0 (every quantizer path)."""
    N = 300
    inst = Instance(d, b, variant, seed=11)
    x64 = synth.scaled_gaussian_rows(N, d, 1.0, seed=11)
    zero = [0, 1, 150, 299]
    x64[zero] = 0.0
    if dtype == torch.bfloat16:
        x64 = bf16_exact(x64)
    out = inst.alloc_outputs(N)
    inst.gpu_quant(to_device(x64, dtype), out)
    torch.cuda.synchronize()
    _check_quant(inst, x64, out)
    assert np.all(out["norms"].cpu().numpy()[zero] == 0)


@pytest.mark.parametrize("d", [8, 200, 240, 256])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("register_loads", [False, True])
def test_quantize_tile_shape_edges(d, dtype, register_loads, monkeypatch):
    """Dimensions at the edges of the fused tile shapes: one 16-wide K step (d = 8),
    a half-filled last 32-group (d = 200, 240) and the widest tile, whose rings
    are shallower (d = 256); 700 rows = five tiles and a ragged tail.  Both fused
    kernels: the TMA-staged one and (register_loads) the one whose producer
    threads load x themselves."""
    N = 700
    if register_loads:
        monkeypatch.setenv("TQ_FUSED_REGISTER_LOADS", "1")
    for variant, b in [(tq.TQ_MSE, 2), (tq.TQ_PROD, 4), (tq.TQ_PROD, 3)]:
        inst = Instance(d, b, variant, seed=d + 1)
        x64 = synth.scaled_gaussian_rows(N, d, 1.0, seed=d)
        if dtype == torch.bfloat16:
            x64 = bf16_exact(x64)
        out = inst.alloc_outputs(N)
        inst.gpu_quant(to_device(x64, dtype), out)
        torch.cuda.synchronize()
        _check_quant(inst, x64, out)


def test_search_quantize_d200_full_size_sampled():
    """The search workload's quantize in the launch the bench times: 10^6 unit
    fp32 vectors at d = 200, prod 4 bits; sampled rows, the first and the last
    tiles checked against the oracle."""
    d, N = 200, 1_000_000
    inst = Instance(d, 4, tq.TQ_PROD, seed=0)
    x64 = synth.unit_rows(N, d, 0)
    out = inst.alloc_outputs(N)
    inst.gpu_quant(to_device(x64, torch.float32), out)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([synth.rng(31, 1).choice(N, 4000, replace=False), np.arange(128),
                                     np.arange(N - 300, N)]))
    _check_quant(inst, x64, out, rows)


def test_prod_many_row_tiles_per_cta():
    """40000 fp32 vectors at d = 200: several 128-vector tiles per persistent CTA."""
    d, N = 200, 40000
    inst = Instance(d, 3, tq.TQ_PROD, seed=21)
    x64 = synth.scaled_gaussian_rows(N, d, 0.5, seed=21)
    out = inst.alloc_outputs(N)
    inst.gpu_quant(to_device(x64, torch.float32), out)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([synth.rng(21, 1).choice(N, 2000, replace=False), np.arange(N - 130, N)]))
    _check_quant(inst, x64, out, rows)


def test_prod_d1536_workspace_chunks_and_no_workspace():
    """d = 1536: a workspace of exactly 128 rows walks 300 vectors in three
    chunks and gives the same words as one launch; without a workspace the C
    call runs the CUDA-core path; both match the oracle."""
    from compressed_kv_cache_turboquant_b200._lib import lib
    from compressed_kv_cache_turboquant_b200.api import _ptr
    d, N = 1536, 300
    inst = Instance(d, 3, tq.TQ_PROD, seed=4)
    x64 = synth.unit_rows(N, d, 4)
    x = to_device(x64, torch.float32)
    full, small, none = inst.alloc_outputs(N), inst.alloc_outputs(N), inst.alloc_outputs(N)
    inst.gpu_quant(x, full)
    row_bytes = tq.tq_quant_prod_workspace(inst.h, 1) // 128
    ws = torch.empty(128 * row_bytes, dtype=torch.uint8, device=DEV)
    tq.tq_quant_prod(inst.h, x, small["codes"], small["signs"], small["norms"], small["rnorms"], workspace=ws)
    rc = lib.tq_quant_prod(inst.h.ptr, _ptr(x), tq.TQ_F32, N, d, _ptr(none["codes"]), _ptr(none["signs"]),
                           _ptr(none["norms"]), _ptr(none["rnorms"]), 1, None)
    assert rc == 0
    torch.cuda.synchronize()
    for k in full:
        assert torch.equal(full[k], small[k]), k
    _check_quant(inst, x64, full)
    _check_quant(inst, x64, none)
    # a workspace below one 128-row tile is refused
    with pytest.raises(tq.TQError):
        tq.tq_quant_prod(inst.h, x, small["codes"], small["signs"], small["norms"], small["rnorms"],
                         workspace=ws[: 127 * row_bytes])


def test_fp32_d1536_prod_sampled():
    d, N = 1536, 300
    inst = Instance(d, 4, tq.TQ_PROD, seed=3)
    x64 = synth.unit_rows(N, d, 3)
    out = inst.alloc_outputs(N)
    inst.gpu_quant(to_device(x64, torch.float32), out)
    torch.cuda.synchronize()
    _check_quant(inst, x64, out)


# ------------------------------------------------------------------ dequant

@pytest.mark.parametrize("b", [1, 2, 3, 4])
@pytest.mark.parametrize("d", [64, 128, 200])
def test_dequant_matches_oracle(b, d):
    N = 777
    inst = Instance(d, b, tq.TQ_MSE, seed=b)
    x64 = synth.scaled_gaussian_rows(N, d, 1.0, seed=b)
    idx, n, _ = oq.quant_mse(x64, inst.Pi_o, inst.t_o)
    ref = oq.dequant_mse(idx, n, inst.Pi_o, inst.c_o)
    codes = upload_words(oq.pack_codes_vec(idx, b))
    norms = torch.tensor(n, device=DEV)
    out = torch.empty((N, d), dtype=torch.float32, device=DEV)
    tq.tq_dequant_mse(inst.h, codes, norms, out)
    outb = torch.empty((N, d), dtype=torch.bfloat16, device=DEV)
    tq.tq_dequant_mse(inst.h, codes, norms, outb)
    torch.cuda.synchronize()
    assert np.max(rel_l2_rows(out.cpu().numpy(), ref)) <= 1e-5
    assert np.max(rel_l2_rows(outb.float().cpu().numpy(), ref)) <= 2 ** -8
    assert_status_clean(inst)


@pytest.mark.parametrize("b", [1, 2, 3, 4])
def test_sweep_dequant_full_size_every_row(b):
    """The sweep batch (N = 2^20 bf16 rows, d = 128, lognormal(0, 1) scales, 4
    outlier channels x20) quantized by the oracle, dequantized on the GPU in the
    launch the bench times, and every row compared with the oracle's
    reconstruction (relative L2 <= 1e-5).  At this size each persistent CTA
    walks dozens of 128-row tiles, so the code prefetch of the next tile and
    the reuse of every output staging box are compared, not only the first
    tile of each CTA."""
    N, d, chunk = 1 << 20, 128, 1 << 16
    inst = Instance(d, b, tq.TQ_MSE)
    x64 = bf16_exact(synth.scaled_gaussian_rows(N, d, 1.0, seed=0, outliers=4))
    codes = torch.empty((N, inst.h.words), dtype=torch.int32, device=DEV)
    norms = torch.empty(N, dtype=torch.float32, device=DEV)
    parts = []
    for r0 in range(0, N, chunk):
        idx, n, _ = oq.quant_mse(x64[r0:r0 + chunk], inst.Pi_o, inst.t_o)
        codes[r0:r0 + chunk] = upload_words(oq.pack_codes_vec(idx, b))
        norms[r0:r0 + chunk] = torch.tensor(n, device=DEV)
        parts.append((idx, n))
    out = torch.empty((N, d), dtype=torch.float32, device=DEV)
    tq.tq_dequant_mse(inst.h, codes, norms, out)
    torch.cuda.synchronize()
    worst = 0.0
    for k, r0 in enumerate(range(0, N, chunk)):
        idx, n = parts[k]
        ref = oq.dequant_mse(idx, n, inst.Pi_o, inst.c_o)
        worst = max(worst, float(np.max(rel_l2_rows(out[r0:r0 + chunk].cpu().numpy(), ref))))
    assert worst <= 1e-5, worst
    assert_status_clean(inst)


# ------------------------------------------------------------------ scores

def _score_case(inst, N, nq, seed, topk=0):
    d = inst.d
    x64 = synth.scaled_gaussian_rows(N, d, 0.5, seed=seed)
    q64 = synth.gaussian_queries(nq, d, seed=seed)
    st = inst.oracle_quant(x64)
    if inst.prod:
        ref = oq.prod_estimate(q64, st["idx"], st["norms"], st["signs"], st["rnorms"], inst.Pi_o, inst.S,
                               inst.c_o, inst.b)
    else:
        ref = oq.mse_estimate(q64, st["idx"], st["norms"], inst.Pi_o, inst.c_o)
    codes = upload_words(oq.pack_codes_vec(st["idx"], inst.bm))
    norms = torch.tensor(st["norms"], device=DEV)
    signs = upload_words(oq.pack_signs(st["signs"])) if inst.prod else None
    rnorms = torch.tensor(st["rnorms"], device=DEV) if inst.prod else None
    q = to_device(q64, torch.float32)
    scores = torch.empty((nq, N), dtype=torch.float32, device=DEV)
    kw = {}
    if topk:
        kw = dict(topk=topk, top_idx=torch.empty((nq, topk), dtype=torch.int32, device=DEV),
                  top_val=torch.empty((nq, topk), dtype=torch.float32, device=DEV))
    tq.tq_ip_scores(inst.h, q, codes, signs, norms, rnorms, scores=scores, **kw)
    torch.cuda.synchronize()
    tol = 1e-4 * np.linalg.norm(q64, axis=1)[:, None] * np.linalg.norm(x64, axis=1)[None, :]
    err = np.abs(scores.cpu().numpy() - ref)
    assert np.all(err <= tol), float(np.max(err / tol))
    assert_status_clean(inst)
    return ref, tol, kw


@pytest.mark.parametrize("variant,b", [(tq.TQ_MSE, 2), (tq.TQ_PROD, 3)])
def test_pr1_scores(variant, b):
    """64 seeded Gaussian queries against all 4096 PR1 vectors."""
    _score_case(Instance(128, b, variant), 4096, 64, 0)


@pytest.mark.parametrize("d,b", [(64, 4), (200, 2), (200, 4), (128, 4)])
def test_scores_shapes_and_topk(d, b):
    ref, tol, kw = _score_case(Instance(d, b, tq.TQ_PROD, seed=d), 2500, 9, d, topk=10)
    ti = kw["top_idx"].cpu().numpy()
    tv = kw["top_val"].cpu().numpy()
    oi, ov = oq.topk(ref, 10)
    for r in range(ref.shape[0]):
        # returned values are the oracle's scores of the returned keys (within tolerance),
        # sorted, and no excluded key beats the k-th by more than the tolerance
        assert np.all(np.abs(tv[r] - ref[r, ti[r]]) <= tol[r, ti[r]])
        assert np.all(np.diff(tv[r]) <= 0)
        assert len(set(ti[r].tolist())) == 10
        rest = np.setdiff1d(np.arange(ref.shape[1]), ti[r])
        assert np.max(ref[r, rest]) <= tv[r, -1] + 2 * np.max(tol[r])
        assert np.allclose(np.sort(tv[r]), np.sort(ov[r]), atol=2 * np.max(tol[r]))


# ------------------------------------------------------------------ decode

def _decode_case(B, Hq, Hkv, T, d, sample, seed=0, stride_extra=0):
    """Quantize K (prod 4b) and V (mse 4b) with the oracle for the sampled
    (batch, kv-head) slices, random valid codes elsewhere; decode on the GPU
    and compare the sampled outputs with the oracle's attention."""
    hk, hv, c, q64, refs = decode_cache(B, Hq, Hkv, T, d, sample, seed, stride_extra)
    S = T + stride_extra
    q = to_device(q64, torch.bfloat16)
    out = torch.empty((B, Hq, d), dtype=torch.float32, device=DEV)
    scale = 1.0 / math.sqrt(d)
    tq.tq_attn_decode(hk.h, hv.h, q, Hkv, T, S, c["kcodes"], c["ksigns"], c["knorms"], c["krnorms"], c["vcodes"],
                      c["vnorms"], scale, out)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    gsz = Hq // Hkv
    for (b, h), (kst, vhat) in refs.items():
        qs = q64[b, h * gsz:(h + 1) * gsz]
        # the oracle's attention step on this (batch, kv-head) as a one-head problem
        est = lambda _b, _h, rows: oq.prod_estimate(rows, kst["idx"], kst["norms"], kst["signs"], kst["rnorms"],
                                                    hk.Pi_o, hk.S, hk.c_o, 4)
        ref_out, ref_logits = oq.attention_decode(qs[None], est, lambda _b, _h: vhat, 1, scale=scale)
        ref = ref_out[0]
        tol = decode_tolerance(ref, ref_logits[(0, 0)], qs, kst, vhat, scale)
        err = np.linalg.norm(got[b, h * gsz:(h + 1) * gsz] - ref, axis=1)
        assert np.all(err <= tol), (b, h, err, tol)
    assert_status_clean(hk, hv)


# The dense 4-heads-per-kv-head decode and the two-group logits run on the
# mma.sync kernels; handles created with TQ_TCGEN05_ATTN=1 take the tcgen05
# kernels instead.
DECODE_KERNELS = ["tcgen05", "mma_sync"]


def _pick_decode_kernel(monkeypatch, kernel):
    if kernel == "tcgen05":
        monkeypatch.setenv("TQ_TCGEN05_ATTN", "1")
    else:
        monkeypatch.delenv("TQ_TCGEN05_ATTN", raising=False)


@pytest.mark.parametrize("kernel", DECODE_KERNELS)
def test_decode_small_ragged(monkeypatch, kernel):
    _pick_decode_kernel(monkeypatch, kernel)
    _decode_case(B=2, Hq=8, Hkv=2, T=1531, d=128, sample=[(0, 0), (0, 1), (1, 0), (1, 1)], seed=1,
                 stride_extra=5)


@pytest.mark.parametrize("kernel", DECODE_KERNELS)
def test_decode_cfg4_full_size_sampled(monkeypatch, kernel):
    """B = 8, Hq = 32, Hkv = 8, d = 128, T = 131072: full launch, sampled slices."""
    _pick_decode_kernel(monkeypatch, kernel)
    _decode_case(B=8, Hq=32, Hkv=8, T=131072, d=128, sample=[(0, 0), (7, 7), (3, 5)], seed=0)


@pytest.mark.parametrize("kernel", DECODE_KERNELS)
def test_decode_one_kv_head_long_context(monkeypatch, kernel):
    """A single (batch, kv-head): every CTA of the persistent grid works on it and the
    merge combines hundreds of partials."""
    _pick_decode_kernel(monkeypatch, kernel)
    _decode_case(B=1, Hq=4, Hkv=1, T=70001, d=128, sample=[(0, 0)], seed=2)


def test_decode_tc_short_contexts(monkeypatch):
    """Contexts of one partial block, of a block and one token, and of many
    (batch, kv-head) pairs per CTA: segment starts and ends inside the
    tcgen05 kernel's pipeline, records of single-block segments."""
    _pick_decode_kernel(monkeypatch, "tcgen05")
    _decode_case(B=3, Hq=8, Hkv=2, T=37, d=128, sample=[(0, 0), (2, 1)], seed=6, stride_extra=3)
    _decode_case(B=2, Hq=4, Hkv=1, T=129, d=128, sample=[(1, 0)], seed=7, stride_extra=3)
    _decode_case(B=64, Hq=16, Hkv=4, T=300, d=128, sample=[(0, 0), (31, 2), (63, 3)], seed=8)


def test_decode_fallback_shapes():
    """Shapes the register-decode kernel does not take (odd cache stride, 2 q-heads per
    kv-head) go through the general kernel and must agree just the same."""
    _decode_case(B=1, Hq=4, Hkv=1, T=777, d=128, sample=[(0, 0)], seed=3, stride_extra=3)
    _decode_case(B=2, Hq=4, Hkv=2, T=500, d=128, sample=[(0, 1), (1, 0)], seed=4)


def test_decode_runtime_table_addresses(monkeypatch):
    """The decode kernel instance that adds its table addresses at run time (taken when the
    dynamic shared window is not where the library expects it) agrees just the same."""
    monkeypatch.setenv("TQ_RUNTIME_TABLE_ADDRESSES", "1")
    _decode_case(B=2, Hq=8, Hkv=2, T=1531, d=128, sample=[(0, 1), (1, 0)], seed=5, stride_extra=5)


# ------------------------------------------------------------------ channel groups (3.5-bit streaming cache)

def _split_instances(d=128, n_hi=64, seed=0):
    scales = synth.lognormal_channel_scales(d, 1.0, seed, 30)
    hi, lo = oq.channel_split(scales, n_hi)
    ia = Instance(64, 4, tq.TQ_PROD, seed=seed, sub=(0,))
    ib = Instance(64, 3, tq.TQ_PROD, seed=seed, sub=(1,))
    channels = torch.tensor(np.concatenate([hi, lo]).astype(np.int32), device=DEV)
    return scales, hi, lo, ia, ib, channels


def _split_keys(T, h, scales, seed):
    z = synth.rng(seed, synth.DATA, 40, h).standard_normal((T, len(scales)))
    return bf16_exact(z * scales[None, :])


def test_streaming_append_gathers_channel_groups():
    """Tokens arrive one at a time for 8 kv-heads; each group of channels is
    quantized into its own cache slot t (out_stride = cache capacity)."""
    Hkv, cap, steps = 8, 40, 5
    scales, hi, lo, ia, ib, channels = _split_instances()
    keys = [_split_keys(steps, h, scales, 7) for h in range(Hkv)]
    caches = {}
    for inst, name, off in ((ia, "a", 0), (ib, "b", 64)):
        caches[name] = inst.alloc_outputs(Hkv * cap)
    for t in range(steps):
        x = to_device(np.stack([keys[h][t] for h in range(Hkv)]), torch.bfloat16)  # [Hkv][128]
        for inst, name, off in ((ia, "a", 0), (ib, "b", 64)):
            c = caches[name]
            sl = slice(t, None)
            tq.tq_quant_gather(inst.h, x, channels[off:off + 64], c["codes"][sl], c["norms"][sl],
                               signs=c["signs"][sl], rnorms=c["rnorms"][sl], out_stride=cap)
    torch.cuda.synchronize()
    for inst, name, chans in ((ia, "a", hi), (ib, "b", lo)):
        c = caches[name]
        rows = np.array([h * cap + t for h in range(Hkv) for t in range(steps)])
        x64 = np.stack([keys[h][t][chans] for h in range(Hkv) for t in range(steps)])
        sub = {k: v[torch.tensor(rows, device=DEV)] for k, v in c.items()}
        _check_quant(inst, x64, sub)


def test_streaming_append_both_groups_in_one_launch():
    """The same append as above through tq_quant_gather_groups: one launch per
    arriving token covers both channel groups of all 8 kv-heads; the words
    equal those of the per-group calls, and both match the oracle."""
    Hkv, cap, steps = 8, 40, 5
    scales, hi, lo, ia, ib, channels = _split_instances()
    keys = [_split_keys(steps, h, scales, 8) for h in range(Hkv)]
    one = {n: inst.alloc_outputs(Hkv * cap) for inst, n in ((ia, "a"), (ib, "b"))}
    per = {n: inst.alloc_outputs(Hkv * cap) for inst, n in ((ia, "a"), (ib, "b"))}
    for t in range(steps):
        x = to_device(np.stack([keys[h][t] for h in range(Hkv)]), torch.bfloat16)
        tq.tq_quant_gather_groups([ia.h, ib.h], x, channels, [one[n]["codes"][t:] for n in "ab"],
                                  [one[n]["norms"][t:] for n in "ab"], signs=[one[n]["signs"][t:] for n in "ab"],
                                  rnorms=[one[n]["rnorms"][t:] for n in "ab"], out_stride=cap)
        for inst, n, off in ((ia, "a", 0), (ib, "b", 64)):
            c = per[n]
            tq.tq_quant_gather(inst.h, x, channels[off:off + 64], c["codes"][t:], c["norms"][t:],
                               signs=c["signs"][t:], rnorms=c["rnorms"][t:], out_stride=cap)
    torch.cuda.synchronize()
    for inst, n, chans in ((ia, "a", hi), (ib, "b", lo)):
        for k in one[n]:
            assert torch.equal(one[n][k], per[n][k]), (n, k)
        rows = np.array([h * cap + t for h in range(Hkv) for t in range(steps)])
        x64 = np.stack([keys[h][t][chans] for h in range(Hkv) for t in range(steps)])
        sub = {k: v[torch.tensor(rows, device=DEV)] for k, v in one[n].items()}
        _check_quant(inst, x64, sub)


def test_bulk_gather_on_the_tensor_cores():
    """A cache fill through tq_quant_gather (N >= 256 takes the tensor-core
    quantizer with the channel gather in its producers): 3000 tokens, both groups."""
    N = 3000
    scales, hi, lo, ia, ib, channels = _split_instances(seed=4)
    k64 = _split_keys(N, 0, scales, 4)
    x = to_device(k64, torch.bfloat16)
    for inst, chans, off in ((ia, hi, 0), (ib, lo, 64)):
        out = inst.alloc_outputs(N)
        tq.tq_quant_gather(inst.h, x, channels[off:off + 64], out["codes"], out["norms"], signs=out["signs"],
                           rnorms=out["rnorms"])
        torch.cuda.synchronize()
        _check_quant(inst, k64[:, chans], out)


def _logits_case(B, Hq, Hkv, T, sample, seed=0, stride_extra=0):
    scales, hi, lo, ia, ib, channels = _split_instances(seed=seed)
    S = T + stride_extra
    rows = B * Hkv * S
    g = torch.Generator(device=DEV).manual_seed(seed)
    cache = {}
    for inst, name in ((ia, "a"), (ib, "b")):
        cache[name] = dict(
            codes=torch.randint(-2 ** 31, 2 ** 31 - 1, (rows, inst.h.words), dtype=torch.int32, device=DEV, generator=g),
            signs=torch.randint(-2 ** 31, 2 ** 31 - 1, (rows, 2), dtype=torch.int32, device=DEV, generator=g),
            norms=torch.rand(rows, device=DEV, generator=g) + 1,
            rnorms=torch.rand(rows, device=DEV, generator=g) * 0.3)
    q64 = bf16_exact(synth.decode_queries(B, Hq, 128, seed=seed))
    refs = {}
    for (b, h) in sample:
        k64 = _split_keys(T, b * Hkv + h, scales, seed)
        r0 = (b * Hkv + h) * S
        st = {}
        for inst, name, chans in ((ia, "a", hi), (ib, "b", lo)):
            s_ = inst.oracle_quant(k64[:, chans])
            c = cache[name]
            c["codes"][r0:r0 + T] = upload_words(oq.pack_codes_vec(s_["idx"], inst.bm))
            c["signs"][r0:r0 + T] = upload_words(oq.pack_signs(s_["signs"]))
            c["norms"][r0:r0 + T] = torch.tensor(s_["norms"], device=DEV)
            c["rnorms"][r0:r0 + T] = torch.tensor(s_["rnorms"], device=DEV)
            st[name] = s_
        refs[(b, h)] = (st, k64)
    q = to_device(q64, torch.bfloat16)
    logits = torch.empty((B, Hq, T), dtype=torch.float32, device=DEV)
    scale = 1.0 / math.sqrt(128)
    tq.tq_attn_logits([ia.h, ib.h], channels, q, Hkv, T, S, [cache["a"]["codes"], cache["b"]["codes"]],
                      [cache["a"]["signs"], cache["b"]["signs"]], [cache["a"]["norms"], cache["b"]["norms"]],
                      [cache["a"]["rnorms"], cache["b"]["rnorms"]], scale, logits)
    torch.cuda.synchronize()
    got = logits.cpu().numpy()
    for (b, h), (st, k64) in refs.items():
        for j in range(4):
            qv = q64[b, 4 * h + j]
            ref = np.zeros(T)
            for inst, name, chans in ((ia, "a", hi), (ib, "b", lo)):
                s_ = st[name]
                ref += oq.prod_estimate(qv[chans], s_["idx"], s_["norms"], s_["signs"], s_["rnorms"], inst.Pi_o,
                                        inst.S, inst.c_o, inst.b)[0]
            ref *= scale
            tol = scale * 1e-4 * np.linalg.norm(qv) * np.linalg.norm(k64, axis=1)
            err = np.abs(got[b, 4 * h + j] - ref)
            assert np.all(err <= tol), (b, h, j, float(np.max(err / tol)))
    assert_status_clean(ia, ib)


def test_split_group_logits_small_ragged():
    """Context 1001 with a cache stride of 1001: the general kernel."""
    _logits_case(B=2, Hq=8, Hkv=2, T=1001, sample=[(0, 0), (1, 1)], seed=1)


@pytest.mark.parametrize("kernel", DECODE_KERNELS)
def test_split_group_logits_ragged_tensor_core(monkeypatch, kernel):
    """Context 1001 (a 3-token tail past the last whole group of 4) with a cache
    stride of 1004, and a context shorter than one block: the tensor-core kernels."""
    _pick_decode_kernel(monkeypatch, kernel)
    _logits_case(B=2, Hq=8, Hkv=2, T=1001, sample=[(0, 0), (1, 1)], seed=1, stride_extra=3)
    _logits_case(B=3, Hq=4, Hkv=1, T=70, sample=[(2, 0)], seed=3, stride_extra=2)


def test_split_group_logits_runtime_table_addresses(monkeypatch):
    monkeypatch.setenv("TQ_RUNTIME_TABLE_ADDRESSES", "1")
    _logits_case(B=2, Hq=8, Hkv=2, T=1001, sample=[(0, 1), (1, 0)], seed=2, stride_extra=3)


@pytest.mark.parametrize("kernel", DECODE_KERNELS)
def test_split_group_logits_full_context_sampled(monkeypatch, kernel):
    """Batch 1, 32 q-heads / 8 kv-heads, context 2^20: the full launch, one kv-head checked."""
    _pick_decode_kernel(monkeypatch, kernel)
    _logits_case(B=1, Hq=32, Hkv=8, T=1 << 20, sample=[(0, 5)], seed=0)


# ------------------------------------------------------------------ nearest-neighbour search (scores + top-k)

def _search_case(d, b, N, nq, sample, seed=0, with_scores=False, k=10):
    inst = Instance(d, b, tq.TQ_PROD, seed=seed)
    x64 = synth.unit_rows(N, d, seed)
    q64 = synth.unit_rows(nq, d, seed, stream=synth.QUERY)
    st = inst.oracle_quant(x64)
    codes = upload_words(oq.pack_codes_vec(st["idx"], inst.bm))
    signs = upload_words(oq.pack_signs(st["signs"]))
    norms = torch.tensor(st["norms"], device=DEV)
    rnorms = torch.tensor(st["rnorms"], device=DEV)
    q = to_device(q64, torch.float32)
    ti = torch.empty((nq, k), dtype=torch.int32, device=DEV)
    tv = torch.empty((nq, k), dtype=torch.float32, device=DEV)
    scores = torch.empty((nq, N), dtype=torch.float32, device=DEV) if with_scores else None
    tq.tq_ip_scores(inst.h, q, codes, signs, norms, rnorms, scores=scores, topk=k, top_idx=ti, top_val=tv)
    torch.cuda.synchronize()
    ti, tv = ti.cpu().numpy(), tv.cpu().numpy()
    refs = oq.prod_estimate(q64[sample], st["idx"], st["norms"], st["signs"], st["rnorms"], inst.Pi_o, inst.S,
                            inst.c_o, b)
    for ref, r in zip(refs, sample):
        tol = 1e-4 * np.linalg.norm(q64[r]) * np.linalg.norm(x64, axis=1)
        assert np.all(np.abs(tv[r] - ref[ti[r]]) <= tol[ti[r]]), r
        assert np.all(np.diff(tv[r]) <= 0) and len(set(ti[r].tolist())) == k
        rest = np.ones(N, bool)
        rest[ti[r]] = False
        assert np.max(ref[rest]) <= tv[r, -1] + 2 * np.max(tol), r
        if with_scores:
            err = np.abs(scores[r].cpu().numpy() - ref)
            assert np.all(err <= tol), (r, float(np.max(err / tol)))
    assert_status_clean(inst)
    return inst


def test_search_d200_full_size_sampled():
    """10^6 unit database vectors (the GloVe shape, d = 200), 10^4 queries, prod 4 bits,
    top-10 for all queries in one call; 8 queries checked against the exact estimator."""
    _search_case(200, 4, 1_000_000, 10_000, sample=[0, 1, 777, 4095, 5000, 8191, 9998, 9999])


@pytest.mark.parametrize("b", [2, 3, 4])
def test_search_d1536_scores_and_topk(b):
    _search_case(1536, b, 3000, 200, sample=list(range(0, 200, 17)), seed=b, with_scores=True)
