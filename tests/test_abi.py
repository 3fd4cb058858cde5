"""CPU tests of the C ABI: the library loads, exports every declared entry
point, its host-side setup (codebook, rotation) matches the oracle, and
invalid arguments are rejected with the documented status codes before any
CUDA work."""
import ctypes
import os
import re

import numpy as np
import pytest

import synth
from oracle import codebook as ocb
from oracle import turboquant as oq

tqmod = pytest.importorskip("compressed_kv_cache_turboquant_b200")
from compressed_kv_cache_turboquant_b200 import _lib  # noqa: E402

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "tq.h")


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^TQ_API\s+[\w\s\*]+?\b(tq_\w+)\s*\(", src, flags=re.M)))


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert len(names) >= 14
    for n in names:
        assert hasattr(_lib.lib, n), n
        assert n in _lib.SIGNATURES, f"binding does not declare {n}"
    assert set(_lib.SIGNATURES) == set(names)


def test_version_string():
    assert "sm_100a" in tqmod.tq_version()


@pytest.mark.parametrize("b", [1, 2, 3, 4])
@pytest.mark.parametrize("d", [3, 8, 64, 128, 200, 1536])
def test_host_codebook_matches_oracle(b, d):
    c, t = tqmod.tq_make_codebook(b, d)
    co, to = ocb.lloyd_max(b, d)
    assert np.max(np.abs(c - co) / np.abs(co)) < 1e-12
    assert np.array_equal(c, -c[::-1])
    assert np.allclose(t, 0.5 * (c[1:] + c[:-1]), rtol=0, atol=1e-18)


@pytest.mark.parametrize("d", [1, 2, 8, 64, 128, 200])
def test_host_rotation_matches_oracle(d):
    G = synth.gaussian_matrix(d, d, 7, synth.ROT_K)
    P = tqmod.tq_make_rotation(G)
    assert np.max(np.abs(P - oq.haar_rotation(G))) < 1e-12
    assert np.max(np.abs(P.T @ P - np.eye(d))) < 1e-12


def test_host_rotation_d1536_orthogonal():
    d = 1536
    G = synth.gaussian_matrix(d, d, 7, synth.ROT_K)
    P = tqmod.tq_make_rotation(G)
    assert np.max(np.abs(P - oq.haar_rotation(G))) < 1e-11


def test_codebook_rejects_bad_arguments():
    c = np.zeros(64)
    dp = c.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    assert _lib.lib.tq_make_codebook(0, 128, dp, None) == _lib.TQ_EUNSUPPORTED
    assert _lib.lib.tq_make_codebook(5, 128, dp, None) == _lib.TQ_EUNSUPPORTED
    assert _lib.lib.tq_make_codebook(2, 2, dp, None) == _lib.TQ_EUNSUPPORTED
    assert _lib.lib.tq_make_codebook(2, 5000, dp, None) == _lib.TQ_EUNSUPPORTED
    assert _lib.lib.tq_make_codebook(2, 128, None, None) == _lib.TQ_EINVAL
    assert b"tq_make_codebook" in _lib.lib.tq_last_error()
    assert _lib.lib.tq_make_rotation(0, dp, dp) == _lib.TQ_EUNSUPPORTED
    assert _lib.lib.tq_make_rotation(4, None, dp) == _lib.TQ_EINVAL


def test_create_rejects_unsupported_shapes_without_cuda():
    d = 128
    P = np.eye(d)
    pp = P.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    h = ctypes.c_void_p()
    L = _lib.lib
    assert L.tq_create(ctypes.byref(h), 100, 2, _lib.TQ_MSE, pp, None, None) == _lib.TQ_EUNSUPPORTED
    assert L.tq_create(ctypes.byref(h), 8192, 2, _lib.TQ_MSE, pp, None, None) == _lib.TQ_EUNSUPPORTED
    assert L.tq_create(ctypes.byref(h), d, 5, _lib.TQ_MSE, pp, None, None) == _lib.TQ_EUNSUPPORTED
    assert L.tq_create(ctypes.byref(h), d, 1, _lib.TQ_PROD, pp, pp, None) == _lib.TQ_EUNSUPPORTED
    assert L.tq_create(ctypes.byref(h), d, 3, _lib.TQ_PROD, pp, None, None) == _lib.TQ_EINVAL
    assert L.tq_create(ctypes.byref(h), d, 3, 7, pp, pp, None) == _lib.TQ_EUNSUPPORTED
    assert L.tq_create(None, d, 3, _lib.TQ_MSE, pp, None, None) == _lib.TQ_EINVAL
    bad = np.array([0.1, -0.1, 0.2, 0.3])
    assert L.tq_create(ctypes.byref(h), d, 2, _lib.TQ_MSE, pp, None,
                       bad.ctypes.data_as(ctypes.POINTER(ctypes.c_double))) == _lib.TQ_EINVAL


def test_hot_path_calls_reject_null_handle():
    L = _lib.lib
    assert L.tq_quant_mse(None, None, 0, 1, 128, None, None, 1, None) == _lib.TQ_EINVAL
    assert L.tq_quant_prod(None, None, 0, 1, 128, None, None, None, None, 1, None) == _lib.TQ_EINVAL
    assert L.tq_dequant_mse(None, None, None, 1, None, 0, None) == _lib.TQ_EINVAL
    assert L.tq_ip_scores(None, None, 1, None, None, None, None, 1, None, 0, None, None, None, 0,
                          None) == _lib.TQ_EINVAL
    assert L.tq_attn_decode(None, None, None, 0, 1, 1, 1, 1, 1, None, None, None, None, None, None,
                            1.0, None, None, 0, None) == _lib.TQ_EINVAL
    assert L.tq_attn_prefill(None, None, None, 0, 1, 1, 4, 1, 8, 8, None, None, None, None, None, None, 1.0, None,
                             None, 0, None) == _lib.TQ_EINVAL
    assert L.tq_ip_scores_workspace(None, 1, 1, 0) == 0
    assert L.tq_attn_decode_workspace(None, 1, 1, 1, 1) == 0
    assert L.tq_attn_prefill_workspace(None, 1, 1, 4, 1, 8) == 0
    assert L.tq_destroy(None) == _lib.TQ_OK


def test_shard_merge_calls_reject_bad_arguments_before_any_gpu_work():
    L = _lib.lib
    off = (ctypes.c_int64 * 2)(0, 10)
    p = ctypes.c_void_p(16)
    assert L.tq_topk_merge(p, p, 0, 4, 10, off, p, p, None) == _lib.TQ_EINVAL          # R = 0
    assert L.tq_topk_merge(p, p, _lib.TQ_MAX_SHARDS + 1, 4, 10, off, p, p, None) == _lib.TQ_EINVAL
    assert L.tq_topk_merge(p, p, 2, 4, 0, off, p, p, None) == _lib.TQ_EINVAL           # k = 0
    assert L.tq_topk_merge(p, p, 2, 4, _lib.TQ_MAX_TOPK + 1, off, p, p, None) == _lib.TQ_EINVAL
    assert L.tq_topk_merge(p, p, 2, 4, 10, None, p, p, None) == _lib.TQ_EINVAL         # no offsets
    neg = (ctypes.c_int64 * 2)(0, -1)
    assert L.tq_topk_merge(p, p, 2, 4, 10, neg, p, p, None) == _lib.TQ_EINVAL
    assert L.tq_topk_merge(p, p, 2, 0, 10, off, p, p, None) == _lib.TQ_OK              # nothing to do
    assert L.tq_attn_merge(None, p, 2, 4, p, None) == _lib.TQ_EINVAL
    assert L.tq_attn_decode_partial(None, None, p, 0, 1, 4, 1, 10, 10, p, p, p, p, p, p, ctypes.c_float(0.1), p, p,
                                    0, None) == _lib.TQ_EINVAL


@pytest.mark.parametrize("b,level", [(4, 1), (2, 1), (1, 2), (2, 2), (2, 5), (2, 7), (1, 6)])
def test_host_polar_codebook_matches_oracle(b, level):
    from oracle import polar as opq
    c, t = tqmod.tq_polar_codebook(b, level)
    co, to = opq.angle_codebook(b, level)
    assert np.max(np.abs(c - co)) < 1e-12 and np.max(np.abs(t - to)) < 1e-12


def test_polar_calls_reject_bad_arguments():
    L = _lib.lib
    h = ctypes.c_void_p()
    Pi = np.eye(64)
    dp = Pi.ctypes.data_as(ctypes.POINTER(ctypes.c_double))
    assert L.tq_create_polar(ctypes.byref(h), 96, 4, 2, dp) == _lib.TQ_EUNSUPPORTED     # not 64 / 128
    assert L.tq_create_polar(ctypes.byref(h), 64, 3, 2, dp) == _lib.TQ_EUNSUPPORTED     # b1 3
    assert L.tq_create_polar(ctypes.byref(h), 64, 4, 3, dp) == _lib.TQ_EUNSUPPORTED     # bh 3
    assert L.tq_create_polar(None, 64, 4, 2, dp) == _lib.TQ_EINVAL
    c = np.zeros(4)
    assert L.tq_polar_codebook(2, 0, c.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), None) == _lib.TQ_EUNSUPPORTED
