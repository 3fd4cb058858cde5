"""Shared builders for the GPU parity tests.

Both sides start from the same seeded Gaussian draws (``synth``).  The oracle
builds its rotation (numpy QR) and codebook (scipy closed forms) itself; the
product builds its own with ``tq_make_rotation`` / ``tq_create`` (C++).  No
value computed by the CUDA path is ever handed to the oracle: comparisons of
packed codes are done word by word against the oracle's own packing, with the
excused threshold-band coordinates masked out.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import synth
from oracle import codebook as ocb
from oracle import turboquant as oq

import compressed_kv_cache_turboquant_b200 as tq

DEV = "cuda"


class Instance:
    """One quantizer instance on both sides (oracle and product)."""

    def __init__(self, d: int, b: int, variant: int, seed: int = 0, rot_stream: int = synth.ROT_K,
                 qjl_stream: int = synth.QJL_K, sub: tuple = ()):
        self.d, self.b, self.variant = d, b, variant
        self.prod = variant == tq.TQ_PROD
        self.bm = b - 1 if self.prod else b
        G = synth.gaussian_matrix(d, d, seed, rot_stream, *sub)
        self.S = synth.gaussian_matrix(d, d, seed, qjl_stream, *sub) if self.prod else None
        self.Pi_o = oq.haar_rotation(G)
        self.c_o, self.t_o = ocb.lloyd_max(self.bm, d)
        self.h = tq.tq_create(d, b, variant, tq.tq_make_rotation(G), self.S)

    # ----- oracle side
    def oracle_quant(self, x64: np.ndarray):
        if self.prod:
            return oq.quant_prod(x64, self.b, self.Pi_o, self.S, self.t_o, self.c_o)
        idx, n, y = oq.quant_mse(x64, self.Pi_o, self.t_o)
        return dict(idx=idx, norms=n, y=y)

    # ----- product side
    def alloc_outputs(self, N: int, slots: int | None = None):
        slots = N if slots is None else slots
        out = dict(codes=torch.zeros((slots, self.h.words), dtype=torch.int32, device=DEV),
                   norms=torch.zeros(slots, dtype=torch.float32, device=DEV))
        if self.prod:
            out["signs"] = torch.zeros((slots, tq.sign_words(self.d)), dtype=torch.int32, device=DEV)
            out["rnorms"] = torch.zeros(slots, dtype=torch.float32, device=DEV)
        return out

    def gpu_quant(self, x: torch.Tensor, out: dict, out_stride: int = 1):
        if self.prod:
            tq.tq_quant_prod(self.h, x, out["codes"], out["signs"], out["norms"], out["rnorms"], out_stride)
        else:
            tq.tq_quant_mse(self.h, x, out["codes"], out["norms"], out_stride)


def to_device(x64: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.tensor(np.ascontiguousarray(x64, dtype=np.float32)).to(DEV).to(dtype)


def bf16_exact(x: np.ndarray) -> np.ndarray:
    return synth.to_bf16_exact(x).astype(np.float64)


def words_u32(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


def compare_codes(gpu_words: np.ndarray, idx: np.ndarray, y_unit: np.ndarray, thresholds: np.ndarray,
                  d: int, bm: int, check_fraction: bool = True):
    """Codes bit-exact except coordinates within 1e-5/sqrt(d) of a threshold.
    Returns (rows whose codes all match, excused count)."""
    excused = oq.near_threshold_mask(y_unit, thresholds, d)
    total = excused.size
    if check_fraction and total >= 200000:
        assert excused.sum() <= 1e-4 * total, f"{excused.sum()} excused of {total}"
    mask = oq.pack_codes_vec(np.where(excused, 2 ** bm - 1, 0), bm)
    expect = oq.pack_codes_vec(idx, bm)
    diff = (gpu_words ^ expect) & ~mask
    bad = np.argwhere(diff != 0)
    assert len(bad) == 0, f"{len(bad)} code words differ outside the threshold band, first at {bad[:5]}"
    rows_exact = np.all(gpu_words == expect, axis=1)
    return rows_exact, int(excused.sum())


def compare_signs(gpu_words: np.ndarray, bits: np.ndarray, Sr: np.ndarray, n: np.ndarray, rows: np.ndarray,
                  check_fraction: bool = True):
    """QJL sign bits on rows whose mse codes match, bit-exact except where the
    projected residual lies within 1e-5 of zero in the unit frame of x:
    |(S r)_j| <= 1e-5 ||x||.  (The code band is 1e-5/sqrt(d) on y = Pi x/||x||;
    with S's rows normalised to unit length, (S r)_j / (sqrt(d) ||x||) is the
    same kind of coordinate, so its band is 1e-5/sqrt(d) on that value.)  At
    most 1e-4 of the compared bits may fall in the band."""
    excused = np.abs(Sr) <= 1e-5 * np.asarray(n, dtype=np.float64)[:, None]
    if check_fraction and excused[rows].size >= 200000:
        assert excused[rows].sum() <= 1e-4 * excused[rows].size, f"{excused[rows].sum()} excused sign bits"
    mask = oq.pack_codes_vec(excused.astype(np.int64), 1)
    expect = oq.pack_codes_vec(bits.astype(np.int64), 1)
    diff = (gpu_words ^ expect) & ~mask
    diff[~np.asarray(rows)] = 0
    bad = np.argwhere(diff != 0)  # (row, word) in the caller's numbering
    assert len(bad) == 0, f"{len(bad)} sign words differ, first at {bad[:5]}"


def rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return np.abs(a - b) / np.maximum(np.abs(b), 1e-30)


def rel_l2_rows(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return np.linalg.norm(a - b, axis=1) / np.maximum(np.linalg.norm(b, axis=1), 1e-30)


def upload_words(w: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(w).view(np.int32)).to(DEV)


def sqrt_half_pi_over(d: int) -> float:
    return math.sqrt(math.pi / 2) / d


def decode_cache(B, Hq, Hkv, T, d, sample, seed=0, stride_extra=0):
    """A K (prod 4 bits) / V (mse 4 bits) cache [B*Hkv][T + stride_extra] on the
    GPU: the sampled (batch, kv-head) slices hold the oracle's codes of seeded
    synthetic keys and values, every other slot random valid words.  Returns
    (key Instance, value Instance, cache dict, bf16-exact queries [B][Hq][d] as
    float64, {(b, h): (oracle key record, oracle x_hat of the values)})."""
    hk = Instance(d, 4, tq.TQ_PROD, seed=seed)
    hv = Instance(d, 4, tq.TQ_MSE, seed=seed, rot_stream=synth.ROT_V)
    S = T + stride_extra
    rows = B * Hkv * S
    g = torch.Generator(device=DEV).manual_seed(seed)
    rnd = lambda cols: torch.randint(-2 ** 31, 2 ** 31 - 1, (rows, cols), dtype=torch.int32, device=DEV, generator=g)
    c = dict(kcodes=rnd(hk.h.words), ksigns=rnd(tq.sign_words(d)), vcodes=rnd(hv.h.words))
    c["knorms"] = torch.rand(rows, device=DEV, generator=g) * 10 + 1
    c["krnorms"] = c["knorms"] * 0.2
    c["vnorms"] = torch.rand(rows, device=DEV, generator=g) * 10 + 1
    q64 = bf16_exact(synth.decode_queries(B, Hq, d, seed=seed))
    refs = {}
    for (b, h) in sample:
        k64 = synth.kv_head_rows(T, d, 0, b, h, seed=seed)
        v64 = synth.kv_head_rows(T, d, 1, b, h, seed=seed)
        kst = hk.oracle_quant(k64)
        vidx, vn, _ = oq.quant_mse(v64, hv.Pi_o, hv.t_o)
        r0 = (b * Hkv + h) * S
        c["kcodes"][r0:r0 + T] = upload_words(oq.pack_codes_vec(kst["idx"], 3))
        c["ksigns"][r0:r0 + T] = upload_words(oq.pack_signs(kst["signs"]))
        c["knorms"][r0:r0 + T] = torch.tensor(kst["norms"], device=DEV)
        c["krnorms"][r0:r0 + T] = torch.tensor(kst["rnorms"], device=DEV)
        c["vcodes"][r0:r0 + T] = upload_words(oq.pack_codes_vec(vidx, 4))
        c["vnorms"][r0:r0 + T] = torch.tensor(vn, device=DEV)
        refs[(b, h)] = (kst, oq.dequant_mse(vidx, vn, hv.Pi_o, hv.c_o))
    return hk, hv, c, q64, refs


def decode_tolerance(ref, logits, qs, kst, vhat, scale):
    """Per-head bound on |out - ref| of a decode step: the score bound
    1e-4 ||q|| ||k|| (scaled) propagated through the softmax, plus 1e-3
    relative for the fp16 value table."""
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    eps = scale * 1e-4 * np.linalg.norm(qs, axis=1)[:, None] * (np.asarray(kst["norms"], dtype=np.float64)[None, :])
    spread = np.linalg.norm(vhat[None, :, :] - ref[:, None, :], axis=2)
    return 2 * np.sum(p * eps * spread, axis=1) + 1e-3 * np.linalg.norm(ref, axis=1)


def assert_status_clean(*handles):
    """Every bounded wait of the calls made so far completed and every kernel
    found its shared-memory window where it was built to (reads and clears the
    handles' device status words)."""
    for h in handles:
        h = h.h if isinstance(h, Instance) else h
        st = tq.tq_device_status(h)
        assert st == 0, f"device status {st:#x} (1 = a wait gave up, 2 = shared-memory layout mismatch)"
