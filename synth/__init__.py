"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This module draws random numbers and nothing else: it holds none of the
quantizer's arithmetic (no QR, no codebook, no rotation, no packing).  The
random matrices that TurboQuant draws -- the Gaussian matrix whose QR factor is
the rotation, and the Gaussian QJL projection -- are produced here as raw
Gaussian draws and handed to both the oracle and the CUDA path as data.

Every generator is a pure function of ``(seed, stream, *sub)`` through
``numpy.random.default_rng([seed, stream, *sub])``, so any block of a large
workload can be regenerated on its own (the parity tests sample rows of the
full-size workloads this way).

Streams:
  0 data vectors / keys / values   1 rotation draw (K, or the only one)
  2 QJL draw (K)                    3 rotation draw (V)
  4 queries                         5 channel scales / outlier choice
"""
from __future__ import annotations

import numpy as np

DATA, ROT_K, QJL_K, ROT_V, QUERY, SCALE = 0, 1, 2, 3, 4, 5


def rng(seed: int, stream: int, *sub: int) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(stream), *[int(s) for s in sub]])


def gaussian_matrix(rows: int, cols: int, seed: int = 0, stream: int = ROT_K, *sub: int) -> np.ndarray:
    """i.i.d. N(0,1) float64 matrix (the draw behind a rotation or a QJL projection)."""
    return rng(seed, stream, *sub).standard_normal((rows, cols))


def lognormal_channel_scales(d: int, sigma: float, seed: int = 0, *sub: int) -> np.ndarray:
    """Per-channel scales exp(N(0, sigma^2)), float64 [d]."""
    return np.exp(sigma * rng(seed, SCALE, *sub).standard_normal(d))


def outlier_channels(d: int, count: int, seed: int = 0, *sub: int) -> np.ndarray:
    """``count`` distinct channel indices chosen uniformly (sorted)."""
    return np.sort(rng(seed, SCALE, 1000, *sub).choice(d, size=count, replace=False))


def to_bf16_exact(a: np.ndarray) -> np.ndarray:
    """Round float values to the nearest bfloat16 (ties to even) and return them
    as float32 values that are exactly representable in bfloat16.  Used so that a
    bf16 workload is the same numbers on the host (oracle) and the device."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    u = (u + 0x7FFF + lsb) >> 16
    out = (u.astype(np.uint32) << 16).view(np.float32)
    # keep NaN payloads out of the rounding (inputs here are finite)
    return out.reshape(a.shape)


def bf16_bits(a_bf16_exact: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of bf16-exact float32 values (for upload as bf16)."""
    f = np.ascontiguousarray(a_bf16_exact, dtype=np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


# --------------------------------------------------------------------------
# Workloads (shapes and value distributions of the pages' use cases)
# --------------------------------------------------------------------------

def scaled_gaussian_rows(n: int, d: int, sigma: float, seed: int = 0, block: int = 0,
                         outliers: int = 0, outlier_factor: float = 20.0) -> np.ndarray:
    """Rows x_i = z_i * s (elementwise), z_i ~ N(0, I_d), s = lognormal(0, sigma)
    channel scales (fixed by ``seed``); ``outliers`` channels are multiplied by
    ``outlier_factor``.  ``block`` selects an independent block of rows."""
    s = lognormal_channel_scales(d, sigma, seed)
    if outliers:
        s = s.copy()
        s[outlier_channels(d, outliers, seed)] *= outlier_factor
    z = rng(seed, DATA, block).standard_normal((n, d))
    return z * s[None, :]


def unit_rows(n: int, d: int, seed: int = 0, stream: int = DATA, block: int = 0) -> np.ndarray:
    """Gaussian rows normalised to unit length (database / query vectors of the
    nearest-neighbour search workload)."""
    z = rng(seed, stream, block).standard_normal((n, d))
    return z / np.linalg.norm(z, axis=1, keepdims=True)


def gaussian_queries(nq: int, d: int, seed: int = 0, block: int = 0) -> np.ndarray:
    return rng(seed, QUERY, block).standard_normal((nq, d))


def kv_head_rows(T: int, d: int, kind: int, b: int, h: int, sigma: float = 1.0, seed: int = 0,
                 t0: int = 0, t1: int | None = None, chunk: int = 4096) -> np.ndarray:
    """Keys (kind=0) or values (kind=1) of batch ``b``, kv-head ``h``: rows t0..t1
    of N(0,1) * lognormal(0, sigma) channel scales, the scales fixed per tensor
    kind and kv-head.  Rows are generated in chunks of ``chunk`` rows with their
    own sub-streams, so any row range regenerates identically."""
    t1 = T if t1 is None else t1
    s = lognormal_channel_scales(d, sigma, seed, 10 + kind, h)
    out = np.empty((t1 - t0, d))
    c0 = t0 // chunk
    c1 = (t1 - 1) // chunk if t1 > t0 else c0 - 1
    for c in range(c0, c1 + 1):
        z = rng(seed, DATA, 10 + kind, b, h, c).standard_normal((chunk, d))
        lo, hi = max(t0, c * chunk), min(t1, (c + 1) * chunk)
        out[lo - t0:hi - t0] = z[lo - c * chunk:hi - c * chunk] * s[None, :]
    return out


def decode_queries(B: int, Hq: int, d: int, sigma: float = 1.0, seed: int = 0) -> np.ndarray:
    """Decode-step queries [B, Hq, d]: N(0,1) * lognormal(0, sigma) channel scales."""
    s = lognormal_channel_scales(d, sigma, seed, 20)
    return rng(seed, QUERY, 20).standard_normal((B, Hq, d)) * s[None, None, :]
