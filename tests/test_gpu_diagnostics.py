"""The device status word reports a wait that ran out and a kernel that found
its shared-memory window elsewhere, and the call returns with the context
still usable.

Both failures are made without faulting or hanging the GPU, through
diagnostic settings read when a handle is created:

* ``TQ_DEBUG_STALL_MS=m``: the decode kernel's consumer warps first wait (m ms
  at most) on a barrier that nothing completes, and every other wait of that
  kernel gives up after m ms.  The consumers abandon the call, the producer
  gives up waiting for free stages, waits for the copies it already issued to
  land, and the CTA exits; the handle's status word has TQ_STATUS_TIMEOUT.
* ``TQ_DEBUG_DYN_BASE=a``: the handle records ``a`` as the measured start of a
  kernel's dynamic shared-memory window, so the decode and logits kernels
  built for the usual address start, see the mismatch, write nothing and
  report TQ_STATUS_LAYOUT.
"""
import math

import numpy as np
import pytest
import torch

import synth

import compressed_kv_cache_turboquant_b200 as tq

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]

DEV = "cuda"


def _kv_handles(seed=0):
    d = 128
    Pk = tq.tq_make_rotation(synth.gaussian_matrix(d, d, seed, synth.ROT_K))
    Sk = synth.gaussian_matrix(d, d, seed, synth.QJL_K)
    Pv = tq.tq_make_rotation(synth.gaussian_matrix(d, d, seed, synth.ROT_V))
    return tq.tq_create(d, 4, tq.TQ_PROD, Pk, Sk), tq.tq_create(d, 4, tq.TQ_MSE, Pv)


def _cache(hk, hv, rows, seed=0):
    g = torch.Generator(device=DEV).manual_seed(seed)
    kx = torch.randn((rows, 128), generator=g, device=DEV).to(torch.bfloat16)
    vx = torch.randn((rows, 128), generator=g, device=DEV).to(torch.bfloat16)
    c = dict(kcodes=torch.empty((rows, hk.words), dtype=torch.int32, device=DEV),
             ksigns=torch.empty((rows, 4), dtype=torch.int32, device=DEV),
             knorms=torch.empty(rows, dtype=torch.float32, device=DEV),
             krnorms=torch.empty(rows, dtype=torch.float32, device=DEV),
             vcodes=torch.empty((rows, hv.words), dtype=torch.int32, device=DEV),
             vnorms=torch.empty(rows, dtype=torch.float32, device=DEV))
    tq.tq_quant_prod(hk, kx, c["kcodes"], c["ksigns"], c["knorms"], c["krnorms"])
    tq.tq_quant_mse(hv, vx, c["vcodes"], c["vnorms"])
    return c


def _decode(hk, hv, c, B, Hq, Hkv, T, q):
    out = torch.full((B, Hq, 128), float("nan"), dtype=torch.float32, device=DEV)
    tq.tq_attn_decode(hk, hv, q, Hkv, T, T, c["kcodes"], c["ksigns"], c["knorms"], c["krnorms"], c["vcodes"],
                      c["vnorms"], 1 / math.sqrt(128), out)
    return out


def test_decode_wait_that_runs_out_is_reported(monkeypatch):
    # six 192-token blocks per CTA: the producer fills its four stages, then
    # waits for a free one that the stalled consumers never release
    B, Hq, Hkv = 1, 4, 1
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    T = sms * 192 * 6
    hk0, hv0 = _kv_handles()
    c = _cache(hk0, hv0, B * Hkv * T)
    q = torch.randn((B, Hq, 128), device=DEV).to(torch.bfloat16)
    ref = _decode(hk0, hv0, c, B, Hq, Hkv, T, q)
    torch.cuda.synchronize()
    assert tq.tq_device_status(hk0) == 0 and tq.tq_device_status(hv0) == 0

    monkeypatch.setenv("TQ_DEBUG_STALL_MS", "20")
    hk, hv = _kv_handles()
    monkeypatch.delenv("TQ_DEBUG_STALL_MS")
    _decode(hk, hv, c, B, Hq, Hkv, T, q)  # returns TQ_OK: the launch itself succeeded
    torch.cuda.synchronize()
    assert tq.tq_device_status(hk) & tq.TQ_STATUS_TIMEOUT
    assert tq.tq_device_status(hk) == 0  # reading clears the word

    # the context is intact: the ordinary handles give the same result as before
    again = _decode(hk0, hv0, c, B, Hq, Hkv, T, q)
    torch.cuda.synchronize()
    assert torch.equal(again, ref)
    assert tq.tq_device_status(hk0) == 0


def test_shared_window_mismatch_is_reported(monkeypatch):
    B, Hq, Hkv, T = 1, 8, 2, 3000
    hk0, hv0 = _kv_handles(seed=1)
    c = _cache(hk0, hv0, B * Hkv * T, seed=1)
    q = torch.randn((B, Hq, 128), device=DEV).to(torch.bfloat16)
    monkeypatch.setenv("TQ_DEBUG_DYN_BASE", "2048")
    hk, hv = _kv_handles(seed=1)
    d64 = [tq.tq_create(64, b, tq.TQ_PROD, tq.tq_make_rotation(synth.gaussian_matrix(64, 64, 1, synth.ROT_K, g)),
                        synth.gaussian_matrix(64, 64, 1, synth.QJL_K, g)) for g, b in ((0, 4), (1, 3))]
    monkeypatch.delenv("TQ_DEBUG_DYN_BASE")
    _decode(hk, hv, c, B, Hq, Hkv, T, q)
    torch.cuda.synchronize()
    assert tq.tq_device_status(hk) & tq.TQ_STATUS_LAYOUT

    # split-cache logits over two d = 64 groups (random valid words are enough here)
    rows = B * Hkv * T
    g = torch.Generator(device=DEV).manual_seed(3)
    caches = [dict(codes=torch.randint(-2 ** 31, 2 ** 31 - 1, (rows, h.words), dtype=torch.int32, device=DEV,
                                       generator=g),
                   signs=torch.randint(-2 ** 31, 2 ** 31 - 1, (rows, 2), dtype=torch.int32, device=DEV, generator=g),
                   norms=torch.rand(rows, device=DEV, generator=g) + 1,
                   rnorms=torch.rand(rows, device=DEV, generator=g)) for h in d64]
    channels = torch.arange(128, dtype=torch.int32, device=DEV)
    logits = torch.empty((B, Hq, T), dtype=torch.float32, device=DEV)
    tq.tq_attn_logits(d64, channels, q, Hkv, T, T, [c_["codes"] for c_ in caches], [c_["signs"] for c_ in caches],
                      [c_["norms"] for c_ in caches], [c_["rnorms"] for c_ in caches], 0.1, logits)
    torch.cuda.synchronize()
    assert tq.tq_device_status(d64[0]) & tq.TQ_STATUS_LAYOUT

    # handles created without the setting still decode normally
    out = _decode(hk0, hv0, c, B, Hq, Hkv, T, q)
    torch.cuda.synchronize()
    assert torch.all(torch.isfinite(out))
    assert tq.tq_device_status(hk0) == 0
