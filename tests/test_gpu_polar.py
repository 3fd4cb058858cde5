"""PolarQuant (the polar stage-one variant) through the C ABI against the
oracle: the angle codes of every level bit-exact except angles inside the
parity band (at most 1e-4 of them), norms to 1e-5, and reconstructions from
the oracle's codes to relative L2 1e-5."""
import numpy as np
import pytest
import torch

import synth
from oracle import polar as opq
from oracle import turboquant as oq

from cases import DEV, assert_status_clean, bf16_exact, rel_err, rel_l2_rows, to_device, upload_words, words_u32

import compressed_kv_cache_turboquant_b200 as tq

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


class Polar:
    def __init__(self, d, b1, bh, seed=0):
        self.d, self.b1, self.bh = d, b1, bh
        G = synth.gaussian_matrix(d, d, seed, synth.ROT_K)
        self.Pi_o = oq.haar_rotation(G)
        self.books = opq.make_books(d, b1, bh)
        self.h = tq.tq_create_polar(d, b1, bh, tq.tq_make_rotation(G))


def _check(p: Polar, x64, codes, norms, rows=None):
    rows = np.arange(x64.shape[0]) if rows is None else rows
    st = opq.quant_polar(x64[rows], p.Pi_o, p.books)
    got = opq.unpack_polar(words_u32(codes)[rows], p.d, p.b1, p.bh)
    band = opq.polar_band(st["y"], p.books, p.d)
    excused = sum(int(m.sum()) for m in band)
    total = sum(m.size for m in band)
    if total >= 200000:
        assert excused <= 1e-4 * total, (excused, total)
    for lev, (g, e, m) in enumerate(zip(got, st["codes"], band), start=1):
        bad = (g != e) & ~m
        assert not np.any(bad), (lev, int(bad.sum()), np.argwhere(bad)[:5])
    assert np.max(rel_err(norms.cpu().numpy()[rows], st["norms"])) <= 1e-5
    assert_status_clean(p.h)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("b1,bh", [(4, 2), (2, 1), (4, 1)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_polar_quantize_matches_oracle(d, b1, bh, dtype):
    N = 1500
    p = Polar(d, b1, bh, seed=d + b1)
    x64 = synth.scaled_gaussian_rows(N, d, 1.0, seed=b1 + bh)
    x64[[0, 700]] = 0.0                      # zero vectors: every angle 0, every code 0
    if dtype == torch.bfloat16:
        x64 = bf16_exact(x64)
    codes = torch.zeros((N, p.h.words), dtype=torch.int32, device=DEV)
    norms = torch.zeros(N, dtype=torch.float32, device=DEV)
    tq.tq_quant_polar(p.h, to_device(x64, dtype), codes, norms)
    torch.cuda.synchronize()
    _check(p, x64, codes, norms)
    assert int(codes[0].abs().sum()) == 0


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("b1,bh", [(4, 2), (2, 1)])
def test_polar_dequant_matches_oracle(d, b1, bh):
    N = 1000
    p = Polar(d, b1, bh, seed=3)
    x64 = synth.scaled_gaussian_rows(N, d, 1.0, seed=3)
    st = opq.quant_polar(x64, p.Pi_o, p.books)
    ref = opq.dequant_polar(st["codes"], st["norms"], p.Pi_o, p.books)
    codes = upload_words(opq.pack_polar(st["codes"], b1, bh))
    norms = torch.tensor(st["norms"], device=DEV)
    out = torch.empty((N, d), dtype=torch.float32, device=DEV)
    tq.tq_dequant_polar(p.h, codes, norms, out)
    outb = torch.empty((N, d), dtype=torch.bfloat16, device=DEV)
    tq.tq_dequant_polar(p.h, codes, norms, outb)
    torch.cuda.synchronize()
    assert np.max(rel_l2_rows(out.cpu().numpy(), ref)) <= 1e-5
    assert np.max(rel_l2_rows(outb.float().cpu().numpy(), ref)) <= 2 ** -8
    assert_status_clean(p.h)


def test_polar_full_size_sampled_and_distortion():
    """2^20 bf16 vectors at d = 128 (the sweep's shape) at about 3 bits per
    coordinate: sampled rows and the tail against the oracle; the batch's
    distortion after a GPU round trip close to the oracle's on the sample."""
    N, d = 1 << 20, 128
    p = Polar(d, 4, 2, seed=0)
    x64 = bf16_exact(synth.scaled_gaussian_rows(N, d, 1.0, seed=0, outliers=4))
    x = to_device(x64, torch.bfloat16)
    codes = torch.zeros((N, p.h.words), dtype=torch.int32, device=DEV)
    norms = torch.zeros(N, dtype=torch.float32, device=DEV)
    tq.tq_quant_polar(p.h, x, codes, norms)
    xh = torch.empty((N, d), dtype=torch.float32, device=DEV)
    tq.tq_dequant_polar(p.h, codes, norms, xh)
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([synth.rng(9, 9).choice(N, 3000, replace=False), np.arange(N - 40, N)]))
    _check(p, x64, codes, norms, rows)
    xt = x.float()
    rel = ((xt - xh).square().sum(1) / xt.square().sum(1)).mean().item()
    st = opq.quant_polar(x64[rows], p.Pi_o, p.books)
    xo = opq.dequant_polar(st["codes"], st["norms"], p.Pi_o, p.books)
    ref = np.mean(np.sum((x64[rows] - xo) ** 2, axis=1) / np.sum(x64[rows] ** 2, axis=1))
    assert abs(rel / ref - 1) < 0.05, (rel, ref)
