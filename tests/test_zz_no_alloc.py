"""tq_attn_decode_static against tq_attn_decode.

tq_attn_decode_static serves callers that may not allocate device memory (a
plugin whose host application owns the device memory pool, a service with a
fixed device footprint): it keeps its scratch in an array compiled into the
library instead of a caller-provided workspace.  Here it is called twice in a
row through the C ABI, with different queries, and each output must agree
with tq_attn_decode on the same inputs within the decode tolerance the other
tests use (relative L2 1e-3; the two run the same kernels, so in practice they
agree exactly).  The file is named so that pytest collects it last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import synth

tq = pytest.importorskip("compressed_kv_cache_turboquant_b200")
from compressed_kv_cache_turboquant_b200 import _lib  # noqa: E402

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")]


def _static_vs_workspace_twice(B, Hq, Hkv, T, seed):
    dev = "cuda"
    d = 128
    Pk = tq.tq_make_rotation(synth.gaussian_matrix(d, d, seed, synth.ROT_K))
    Sk = synth.gaussian_matrix(d, d, seed, synth.QJL_K)
    Pv = tq.tq_make_rotation(synth.gaussian_matrix(d, d, seed, synth.ROT_V))
    hk = tq.tq_create(d, 4, tq.TQ_PROD, Pk, Sk)
    hv = tq.tq_create(d, 4, tq.TQ_MSE, Pv)
    rows = B * Hkv * T
    g = torch.Generator(device=dev).manual_seed(7 + seed)
    # quantize synthetic keys and values into the cache with the library itself
    kx = torch.randn((rows, d), generator=g, device=dev).to(torch.bfloat16)
    vx = torch.randn((rows, d), generator=g, device=dev).to(torch.bfloat16)
    kcodes = torch.empty((rows, hk.words), dtype=torch.int32, device=dev)
    ksigns = torch.empty((rows, tq.sign_words(d)), dtype=torch.int32, device=dev)
    knorms = torch.empty(rows, dtype=torch.float32, device=dev)
    krnorms = torch.empty(rows, dtype=torch.float32, device=dev)
    vcodes = torch.empty((rows, hv.words), dtype=torch.int32, device=dev)
    vnorms = torch.empty(rows, dtype=torch.float32, device=dev)
    tq.tq_quant_prod(hk, kx, kcodes, ksigns, knorms, krnorms)
    tq.tq_quant_mse(hv, vx, vcodes, vnorms)
    scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream().cuda_stream

    for call in range(2):
        q = (torch.randn((B, Hq, d), generator=g, device=dev) * (1.0 + call)).to(torch.bfloat16)
        ref = torch.empty((B, Hq, d), dtype=torch.float32, device=dev)
        tq.tq_attn_decode(hk, hv, q, Hkv, T, T, kcodes, ksigns, knorms, krnorms, vcodes, vnorms, scale, ref)
        out = torch.full((B, Hq, d), float("nan"), dtype=torch.float32, device=dev)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        rc = _lib.lib.tq_attn_decode_static(
            hk.ptr, hv.ptr, q.data_ptr(), _lib.TQ_BF16, B, Hq, Hkv, T, T, kcodes.data_ptr(),
            ksigns.data_ptr(), knorms.data_ptr(), krnorms.data_ptr(), vcodes.data_ptr(), vnorms.data_ptr(),
            ctypes.c_float(scale), out.data_ptr(), stream)
        assert rc == _lib.TQ_OK, _lib.lib.tq_last_error()
        torch.cuda.synchronize()
        if call == 1:
            # the first call on a device may load the library's device code and
            # its scratch array; from then on a call takes no device memory
            assert torch.cuda.mem_get_info()[0] == free_before
        a = out.reshape(-1, d).cpu().numpy().astype(np.float64)
        r = ref.reshape(-1, d).cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(a))
        rel = np.linalg.norm(a - r, axis=1) / np.linalg.norm(r, axis=1)
        assert np.max(rel) <= 1e-3, (call, float(np.max(rel)))
    assert tq.tq_device_status(hk) == 0


def test_static_scratch_decode_matches_workspace_decode_twice():
    # 4 query heads per kv-head: the tensor-core decode kernel and its merge
    _static_vs_workspace_twice(B=2, Hq=8, Hkv=2, T=3000, seed=0)


def test_static_scratch_decode_fallback_kernel_twice():
    # 2 query heads per kv-head: the general split kernel and its merge, with
    # its partials in the same scratch array
    _static_vs_workspace_twice(B=1, Hq=4, Hkv=2, T=2500, seed=1)


def test_static_scratch_decode_rejects_shapes_beyond_its_limit():
    d = 128
    Pk = tq.tq_make_rotation(synth.gaussian_matrix(d, d, 0, synth.ROT_K))
    Sk = synth.gaussian_matrix(d, d, 0, synth.QJL_K)
    hk = tq.tq_create(d, 4, tq.TQ_PROD, Pk, Sk)
    hv = tq.tq_create(d, 4, tq.TQ_MSE, Pk)
    B, Hq, Hkv, T = 64, 512, 64, 1 << 20
    assert tq.tq_attn_decode_workspace(hk, B, Hq, Hkv, T) > _lib.TQ_DECODE_STATIC_SCRATCH
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = dummy.data_ptr()
    rc = _lib.lib.tq_attn_decode_static(hk.ptr, hv.ptr, p, _lib.TQ_BF16, B, Hq, Hkv, T, T, p, p, p, p, p, p,
                                        ctypes.c_float(0.1), p, None)
    assert rc == _lib.TQ_EWORKSPACE
    assert b"scratch" in _lib.lib.tq_last_error()
