"""ctypes loader of libtq_b200.so: declares every entry point of include/tq.h.

There is no fallback: if the shared library is missing, importing this module
raises, so no caller can silently run anything but the CUDA path.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq_b200.so")

TQ_OK, TQ_EINVAL, TQ_EUNSUPPORTED, TQ_EALIGN, TQ_ECUDA, TQ_ENOMEM, TQ_EWORKSPACE = range(7)
TQ_F32, TQ_BF16, TQ_F16 = 0, 1, 2
TQ_MSE, TQ_PROD, TQ_POLAR = 0, 1, 2
TQ_MAX_DIM = 4096
TQ_MAX_TOPK = 64
TQ_STATUS_TIMEOUT, TQ_STATUS_LAYOUT = 1, 2
TQ_MAX_SHARDS = 64
TQ_DECODE_STATIC_SCRATCH = 4 * 1024 * 1024

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python compressed_kv_cache_turboquant_b200/build.py` "
        "(this package has no non-CUDA fallback)")

lib = ctypes.CDLL(LIB_PATH)

_p = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_f = ctypes.c_float
_sz = ctypes.c_size_t
_dp = ctypes.POINTER(ctypes.c_double)

# name -> (restype, argtypes); mirrors include/tq.h
SIGNATURES = {
    "tq_make_codebook": (_i, [_i, _i, _dp, _dp]),
    "tq_make_rotation": (_i, [_i, _dp, _dp]),
    "tq_create": (_i, [ctypes.POINTER(_p), _i, _i, _i, _dp, _dp, _dp]),
    "tq_destroy": (_i, [_p]),
    "tq_handle_info": (_i, [_p, ctypes.POINTER(_i), ctypes.POINTER(_i), ctypes.POINTER(_i),
                            ctypes.POINTER(_i)]),
    "tq_quant_mse": (_i, [_p, _p, _i, _i64, _i64, _p, _p, _i64, _p]),
    "tq_dequant_mse": (_i, [_p, _p, _p, _i64, _p, _i, _p]),
    "tq_quant_prod": (_i, [_p, _p, _i, _i64, _i64, _p, _p, _p, _p, _i64, _p]),
    "tq_quant_prod_ws": (_i, [_p, _p, _i, _i64, _i64, _p, _p, _p, _p, _i64, _p, _sz, _p]),
    "tq_quant_prod_workspace": (_sz, [_p, _i64]),
    "tq_ip_scores": (_i, [_p, _p, _i64, _p, _p, _p, _p, _i64, _p, _i, _p, _p, _p, _sz, _p]),
    "tq_ip_scores_workspace": (_sz, [_p, _i64, _i64, _i]),
    "tq_attn_decode": (_i, [_p, _p, _p, _i, _i, _i, _i, _i64, _i64, _p, _p, _p, _p, _p, _p, _f,
                            _p, _p, _sz, _p]),
    "tq_attn_decode_workspace": (_sz, [_p, _i, _i, _i, _i64]),
    "tq_attn_decode_static": (_i, [_p, _p, _p, _i, _i, _i, _i, _i64, _i64, _p, _p, _p, _p, _p, _p, _f,
                                   _p, _p]),
    "tq_attn_decode_partial": (_i, [_p, _p, _p, _i, _i, _i, _i, _i64, _i64, _p, _p, _p, _p, _p, _p, _f,
                                    _p, _p, _sz, _p]),
    "tq_attn_decode_partial_workspace": (_sz, [_p, _i, _i, _i, _i64]),
    "tq_attn_merge": (_i, [_p, _p, _i, _i64, _p, _p]),
    "tq_topk_merge": (_i, [_p, _p, _i, _i64, _i, ctypes.POINTER(ctypes.c_int64), _p, _p, _p]),
    "tq_quant_paged": (_i, [_p, _p, _i, _i64, _i64, _p, _p, _p, _p, _p, _p, _i, _p]),
    "tq_attn_decode_paged": (_i, [_p, _p, _p, _i, _i, _i, _i, _i64, _p, _i, _i, _p, _p, _p, _p, _i, _p, _p, _f, _p,
                                  _p, _sz, _p]),
    "tq_attn_prefill": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _i64, _i64, _p, _p, _p, _p, _p, _p, _f, _p, _p, _sz,
                             _p]),
    "tq_attn_prefill_workspace": (_sz, [_p, _i, _i, _i, _i, _i64]),
    "tq_polar_codebook": (_i, [_i, _i, _dp, _dp]),
    "tq_create_polar": (_i, [ctypes.POINTER(_p), _i, _i, _i, _dp]),
    "tq_quant_polar": (_i, [_p, _p, _i, _i64, _i64, _p, _p, _i64, _p]),
    "tq_dequant_polar": (_i, [_p, _p, _p, _i64, _p, _i, _p]),
    "tq_device_status": (_i, [_p, ctypes.POINTER(_i)]),
    "tq_quant_gather": (_i, [_p, _p, _i, _i64, _i64, _p, _p, _p, _p, _p, _i64, _p]),
    "tq_quant_gather_groups": (_i, [ctypes.POINTER(_p), _i, _p, _i, _i64, _i64, _p, ctypes.POINTER(_p),
                                    ctypes.POINTER(_p), ctypes.POINTER(_p), ctypes.POINTER(_p), _i64, _p]),
    "tq_attn_logits": (_i, [ctypes.POINTER(_p), _i, _p, _p, _i, _i, _i, _i, _i, _i64, _i64, ctypes.POINTER(_p),
                            ctypes.POINTER(_p), ctypes.POINTER(_p), ctypes.POINTER(_p), _f, _p, _p, _sz, _p]),
    "tq_attn_logits_workspace": (_sz, [ctypes.POINTER(_p), _i, _i, _i]),
    "tq_last_error": (ctypes.c_char_p, []),
    "tq_version": (ctypes.c_char_p, []),
}

for _name, (_res, _args) in SIGNATURES.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


class TQError(RuntimeError):
    def __init__(self, fn: str, code: int):
        msg = lib.tq_last_error().decode(errors="replace")
        super().__init__(f"{fn} failed with code {code}: {msg}")
        self.code = code


def check(fn: str, rc: int) -> None:
    if rc != TQ_OK:
        raise TQError(fn, rc)
