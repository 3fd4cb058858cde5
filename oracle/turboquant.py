"""TurboQuant_mse / TurboQuant_prod, the inner-product estimator, packing and
attention over compressed K/V -- oracle, float64, step by step.

Page keys are listed in ``oracle/__init__.py``.  Where the pages leave a step
open, the reading taken is stated in the docstring of the function that takes
it.
"""
from __future__ import annotations

import math

import numpy as np

# ---------------------------------------------------------------------------
# Rotation
# ---------------------------------------------------------------------------


def haar_rotation(G: np.ndarray) -> np.ndarray:
    """Pi from the QR factorisation of a Gaussian matrix G
    ([ttakun, "为什么随机旋转是整个算法的底层杠杆"]; [tq.net, "实现步骤草图", 生成随机旋转矩阵]).

    Reading: the sketch keeps the bare Q of ``qr(G)``; the page on the rotation
    needs coordinates uniform on the sphere, which Q alone does not guarantee
    (its column signs follow the QR routine's conventions).  Q is multiplied
    by diag(sign(diag R)), which makes Pi Haar-distributed.  Pi is then used as
    y = Pi @ x.  Pinned by orthogonality and by R's diagonal becoming positive.
    """
    Q, R = np.linalg.qr(np.asarray(G, dtype=np.float64))
    s = np.sign(np.diag(R))
    s[s == 0] = 1.0
    return Q * s[None, :]


# ---------------------------------------------------------------------------
# Scalar quantization of rotated coordinates
# ---------------------------------------------------------------------------


def quantize_indices(y: np.ndarray, thresholds: np.ndarray) -> np.ndarray:
    """idx = #{k : y >= t_k}: the nearest Lloyd-Max centroid of each coordinate,
    found independently per coordinate against the decision thresholds
    ([ttakun, "TurboQuant_mse vs TurboQuant_prod两个变体的精确分工"]: rotate, then quantize
    each coordinate on its own with the precomputed codebook).  A value exactly on
    a threshold goes to the upper cell.  Pinned by brute-force nearest centroid."""
    y = np.asarray(y, dtype=np.float64)
    return np.sum(y[..., None] >= np.asarray(thresholds)[None, :], axis=-1).astype(np.int64)


def nearest_centroid_bruteforce(y: np.ndarray, c: np.ndarray) -> np.ndarray:
    """argmin_k |y - c_k| by exhaustive comparison; equal distances go to the larger k."""
    y = np.asarray(y, dtype=np.float64).reshape(-1)
    out = np.empty(y.shape, dtype=np.int64)
    for i, v in enumerate(y):
        best, bd = 0, abs(v - c[0])
        for k in range(1, len(c)):
            dk = abs(v - c[k])
            if dk <= bd:
                best, bd = k, dk
        out[i] = best
    return out


def near_threshold_mask(y_unit: np.ndarray, thresholds: np.ndarray, d: int, tol: float = 1e-5):
    """Coordinates whose rotated unit-frame value lies within tol/sqrt(d) of a
    decision threshold: there a float32 evaluation may legitimately pick the
    other cell, so parity excuses them."""
    gap = np.min(np.abs(np.asarray(y_unit)[..., None] - np.asarray(thresholds)[None, :]), axis=-1)
    return gap <= tol / math.sqrt(d)


def quant_mse(x: np.ndarray, Pi: np.ndarray, thresholds: np.ndarray):
    """TurboQuant_mse quantization of the rows of x
    ([ttakun, "TurboQuant_mse vs TurboQuant_prod两个变体的精确分工"]: store the norm as
    float32, rotate, quantize each coordinate with the precomputed codebook;
    [tq.net, "实现步骤草图", quant 原语]).

    n = ||x|| (float64 from the exact inputs), y = Pi @ (x / n), idx = cell of y.
    Reading for x = 0: y := 0, codes by the same rule, x_hat = 0.
    Returns (idx [N, d] int64, norms [N] float32 as stored, y [N, d] float64 unit frame).
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    n = np.sqrt(np.sum(x * x, axis=1))
    safe = np.where(n > 0, n, 1.0)
    y = (x / safe[:, None]) @ Pi.T            # y_i = Pi @ (x_i / n_i)
    y[n == 0] = 0.0
    idx = quantize_indices(y, thresholds)
    return idx, n.astype(np.float32), y


def dequant_mse(idx: np.ndarray, norms: np.ndarray, Pi: np.ndarray, centroids: np.ndarray) -> np.ndarray:
    """x_hat = n * Pi^T @ c[idx] ([ttakun, same section]: rebuild by rotating back
    and rescaling; [tq.net, "实现步骤草图", dequant 原语]).  n is the stored float32 norm."""
    y_hat = np.asarray(centroids, dtype=np.float64)[np.asarray(idx)]
    return (y_hat @ Pi) * np.asarray(norms, dtype=np.float64)[:, None]


def quant_prod(x: np.ndarray, b: int, Pi: np.ndarray, S: np.ndarray, mse_thresholds, mse_centroids,
               rn_dtype=np.float32):
    """TurboQuant_prod with b total bits per coordinate
    ([ttakun, "TurboQuant_mse vs TurboQuant_prod两个变体的精确分工"]: stage one is (b-1)-bit
    mse giving x_hat and the residual r; stage two keeps 1-bit QJL of r;
    [tmdm, "双剑合璧：PolarQuant + QJL", ✦ QJL]; [admirer, "第二步"]).

    r = x - x_hat (x_hat from the stored float32 norm), QJL bits = [ (S r)_j >= 0 ]
    (sign(0) := +1), rn = ||r|| stored as float32.
    Readings: S is m x d with m = d (the estimator's sqrt(pi/2)/d factor implies
    m = d); both norms are float32 (one page stores the norm as float32, another
    says the residual norm costs one FP16 scalar -- float32 is taken for both).
    ``rn_dtype=np.float16`` is that second page's storage of the residual norm
    ([tq.net, "工程风险与应对", 残差范数存储]): ||r|| rounded once, from float64, to
    the nearest fp16; the estimator then uses the stored value.
    b = 1 means zero mse bits: x_hat = 0 and r = x.
    """
    x = np.atleast_2d(np.asarray(x, dtype=np.float64))
    if b >= 2:
        idx, norms, y = quant_mse(x, Pi, mse_thresholds)
        x_hat = dequant_mse(idx, norms, Pi, mse_centroids)
    else:
        idx = np.zeros(x.shape, dtype=np.int64)
        norms = np.sqrt(np.sum(x * x, axis=1)).astype(np.float32)
        y = np.zeros_like(x)
        x_hat = np.zeros_like(x)
    r = x - x_hat
    v = r @ S.T
    signs = (v >= 0.0)
    rn = np.sqrt(np.sum(r * r, axis=1)).astype(rn_dtype)
    return dict(idx=idx, norms=norms, signs=signs, rnorms=rn, y=y, x_hat=x_hat, r=r, Sr=v)


def mse_estimate(q: np.ndarray, idx, norms, Pi, centroids) -> np.ndarray:
    """<q, x_hat_mse> for every (query, vector) pair: [nq, N]."""
    return np.atleast_2d(q) @ dequant_mse(idx, norms, Pi, centroids).T


def prod_estimate(q: np.ndarray, idx, norms, signs, rnorms, Pi, S, mse_centroids, b: int) -> np.ndarray:
    """Unbiased inner-product estimate
    <q, x> ~ <q, x_hat_mse> + ||r|| * sqrt(pi/2) / m * <S q, sign(S r)>
    ([tmdm, "双剑合璧", ✦ QJL]: an unbiased estimator corrects the error while the
    attention score is computed; [admirer, "第二步"]).  Pinned by unbiasedness and
    the exact variance over seeded S draws.  Returns [nq, N]."""
    q = np.atleast_2d(np.asarray(q, dtype=np.float64))
    m = S.shape[0]
    sigma = np.where(np.asarray(signs), 1.0, -1.0)
    qjl = (q @ S.T) @ sigma.T                       # <S q, sign(S r)>
    est = qjl * (np.asarray(rnorms, dtype=np.float64)[None, :] * math.sqrt(math.pi / 2.0) / m)
    if b >= 2:
        est = est + mse_estimate(q, idx, norms, Pi, mse_centroids)
    return est


# ---------------------------------------------------------------------------
# Packed storage layout (the pages only say "2- or 4-bit integers")
# ---------------------------------------------------------------------------


def code_words(b: int, d: int) -> int:
    """uint32 words per vector: ceil(d/32) groups of 32 coordinates, b words each."""
    return ((d + 31) // 32) * b


def pack_codes(idx: np.ndarray, b: int) -> np.ndarray:
    """Pack b-bit indices [N, d] into uint32 words [N, ceil(d/32) * b].

    Layout (a reading: the pages say only that 32-bit coordinates become 2- or
    4-bit integers, [ttakun, "为什么随机旋转是整个算法的底层杠杆"]).  Coordinates form
    groups of 32 (g = j // 32, i = j % 32; coordinates past d are zero); group g
    owns words g*b .. g*b+b-1.  Within a group:
      b = 1: word 0 bit i                     = idx_i
      b = 2: word k bits 2j..2j+1             = idx_{16k+j}      (k < 2, j < 16)
      b = 4: word k bits 4j..4j+3             = idx_{8k+j}       (k < 4, j < 8)
      b = 3: word k bits 4j..4j+2             = idx_{8k+j}       (k < 3, j < 8)
             word k bit  4j+3                 = bit k of idx_{24+j}
      b > 4: word k bit i = bit k of idx_i (bit planes)
    Written field by field with Python integers.  Pinned by hand-built words in
    tests/golden/packing_layout.txt."""
    idx = np.atleast_2d(np.asarray(idx, dtype=np.int64))
    N, d = idx.shape
    G = (d + 31) // 32
    out = np.zeros((N, G * b), dtype=np.uint32)
    for n in range(N):
        for g in range(G):
            grp = [int(idx[n, 32 * g + i]) if 32 * g + i < d else 0 for i in range(32)]
            words = [0] * b
            for i, v in enumerate(grp):
                if not 0 <= v < (1 << b):
                    raise ValueError("index out of range")
                if b == 1:
                    words[0] |= v << i
                elif b == 2:
                    words[i // 16] |= v << (2 * (i % 16))
                elif b == 4:
                    words[i // 8] |= v << (4 * (i % 8))
                elif b == 3:
                    if i < 24:
                        words[i // 8] |= v << (4 * (i % 8))
                    else:
                        j = i - 24
                        for k in range(3):
                            words[k] |= ((v >> k) & 1) << (4 * j + 3)
                else:
                    for k in range(b):
                        words[k] |= ((v >> k) & 1) << i
            out[n, g * b:(g + 1) * b] = words
    return out


def unpack_codes(words: np.ndarray, b: int, d: int) -> np.ndarray:
    """Inverse of ``pack_codes``: [N, ceil(d/32)*b] uint32 -> [N, d] int64."""
    words = np.atleast_2d(np.asarray(words, dtype=np.uint32))
    N = words.shape[0]
    G = (d + 31) // 32
    out = np.zeros((N, G * 32), dtype=np.int64)
    for n in range(N):
        for g in range(G):
            w = [int(v) for v in words[n, g * b:(g + 1) * b]]
            for i in range(32):
                if b == 1:
                    v = (w[0] >> i) & 1
                elif b == 2:
                    v = (w[i // 16] >> (2 * (i % 16))) & 3
                elif b == 4:
                    v = (w[i // 8] >> (4 * (i % 8))) & 15
                elif b == 3:
                    if i < 24:
                        v = (w[i // 8] >> (4 * (i % 8))) & 7
                    else:
                        j = i - 24
                        v = sum(((w[k] >> (4 * j + 3)) & 1) << k for k in range(3))
                else:
                    v = sum(((w[k] >> i) & 1) << k for k in range(b))
                out[n, 32 * g + i] = v
    return out[:, :d]


def pack_codes_vec(idx: np.ndarray, b: int) -> np.ndarray:
    """Same layout as ``pack_codes`` (b <= 4), vectorised over rows with numpy
    shifts for large inputs.  Pinned to ``pack_codes`` by equality tests."""
    idx = np.atleast_2d(np.asarray(idx)).astype(np.uint32)
    N, d = idx.shape
    G = (d + 31) // 32
    full = np.zeros((N, G * 32), dtype=np.uint32)
    full[:, :d] = idx
    grp = full.reshape(N, G, 32)
    out = np.zeros((N, G, b), dtype=np.uint32)
    if b == 1:
        for i in range(32):
            out[:, :, 0] |= grp[:, :, i] << np.uint32(i)
    elif b == 2:
        for k in range(2):
            for j in range(16):
                out[:, :, k] |= grp[:, :, 16 * k + j] << np.uint32(2 * j)
    elif b == 4:
        for k in range(4):
            for j in range(8):
                out[:, :, k] |= grp[:, :, 8 * k + j] << np.uint32(4 * j)
    elif b == 3:
        for k in range(3):
            for j in range(8):
                out[:, :, k] |= grp[:, :, 8 * k + j] << np.uint32(4 * j)
                out[:, :, k] |= ((grp[:, :, 24 + j] >> np.uint32(k)) & np.uint32(1)) << np.uint32(4 * j + 3)
    else:
        raise ValueError("pack_codes_vec handles b <= 4")
    return out.reshape(N, G * b)


def pack_signs(bits: np.ndarray) -> np.ndarray:
    """QJL sign bits [N, m] (True = non-negative) -> uint32 [N, ceil(m/32)], bit i of
    word g = coordinate 32g + i (the b = 1 layout)."""
    return pack_codes_vec(np.asarray(bits, dtype=np.int64), 1)


def unpack_signs(words: np.ndarray, m: int) -> np.ndarray:
    return unpack_codes(words, 1, m).astype(bool)


# ---------------------------------------------------------------------------
# Attention over a compressed K/V cache
# ---------------------------------------------------------------------------


def attention_decode(q: np.ndarray, k_est_fn, v_hat: np.ndarray, Hkv: int, scale: float | None = None):
    """One decode step of attention over a TurboQuant K/V cache
    ([tq.net, "实现步骤草图", 集成到 attention]: K and V are stored in TurboQuant form and
    QJL is used inside attention).

    q: [B, Hq, d]; k_est_fn(b, h, q_rows [g, d]) -> [g, T] estimated <q, k_t>
    for kv-head h of batch b; v_hat: callable (b, h) -> [T, d] dequantized values.
    Readings: logits = est / sqrt(d) unless ``scale`` is given (the pages are
    silent on the scale); q-head j uses kv-head j // (Hq / Hkv) (grouped-query
    attention); softmax and the weighted sum in float64.
    Returns (out [B, Hq, d], logits list per (b, kv-head) [g, T]).
    """
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    g = Hq // Hkv
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    out = np.zeros((B, Hq, d))
    all_logits = {}
    for b in range(B):
        for h in range(Hkv):
            qs = q[b, h * g:(h + 1) * g]
            logits = k_est_fn(b, h, qs) * scale
            mx = np.max(logits, axis=1, keepdims=True)
            p = np.exp(logits - mx)
            p /= np.sum(p, axis=1, keepdims=True)
            out[b, h * g:(h + 1) * g] = p @ v_hat(b, h)
            all_logits[(b, h)] = logits
    return out, all_logits


def attention_prefill(q: np.ndarray, k_est_fn, v_hat, Hkv: int, T: int, scale: float | None = None):
    """Attention of a block of nq new tokens (a prompt chunk) over a TurboQuant
    K/V cache that already holds them: query token i sits at position
    T - nq + i and attends the keys t <= T - nq + i (causal).  Same readings as
    ``attention_decode`` ([tq.net, "实现步骤草图", 集成到 attention]).
    q: [B, nq, Hq, d]; k_est_fn(b, h, q_rows [r, d]) -> [r, T]; v_hat(b, h) -> [T, d].
    Returns out [B, nq, Hq, d].  Pinned by scipy's softmax over each query's
    visible keys and, for nq = 1, by ``attention_decode``."""
    q = np.asarray(q, dtype=np.float64)
    B, nq, Hq, d = q.shape
    g = Hq // Hkv
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    out = np.zeros((B, nq, Hq, d))
    for b in range(B):
        for h in range(Hkv):
            rows = q[b, :, h * g:(h + 1) * g].reshape(nq * g, d)      # row = (token i, head j)
            logits = np.atleast_2d(k_est_fn(b, h, rows)) * scale     # [nq * g, T]
            pos = T - nq + np.repeat(np.arange(nq), g)               # position of each row's token
            logits = np.where(np.arange(T)[None, :] <= pos[:, None], logits, -np.inf)
            mx = np.max(logits, axis=1, keepdims=True)
            p = np.exp(logits - mx)
            p /= np.sum(p, axis=1, keepdims=True)
            out[b, :, h * g:(h + 1) * g] = (p @ v_hat(b, h)).reshape(nq, g, d)
    return out


def attention_partial(q: np.ndarray, k_est_fn, v_hat, Hkv: int, scale: float | None = None):
    """The softmax state of one decode step over a slice of the context, to be
    combined with the states of the other slices (the context split across
    devices).  Same readings as ``attention_decode``; for every (batch, q-head):
    m = max logit over the slice, l = sum_t exp(logit_t - m),
    acc = sum_t exp(logit_t - m) v_hat_t.  An empty slice gives m = -inf, l = 0,
    acc = 0.  Returns (m [B, Hq], l [B, Hq], acc [B, Hq, d]).  Pinned, through
    ``merge_attention_partials``, by the softmax of the whole context."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    g = Hq // Hkv
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    m = np.full((B, Hq), -np.inf)
    l = np.zeros((B, Hq))
    acc = np.zeros((B, Hq, d))
    for b in range(B):
        for h in range(Hkv):
            qs = q[b, h * g:(h + 1) * g]
            logits = np.atleast_2d(k_est_fn(b, h, qs)) * scale
            if logits.shape[1] == 0:
                continue
            mx = np.max(logits, axis=1)
            p = np.exp(logits - mx[:, None])
            m[b, h * g:(h + 1) * g] = mx
            l[b, h * g:(h + 1) * g] = p.sum(axis=1)
            acc[b, h * g:(h + 1) * g] = p @ v_hat(b, h)
    return m, l, acc


def merge_attention_partials(ms, ls, accs):
    """Combine the softmax states of context slices: with M = max_s m_s,
    out = sum_s e^(m_s - M) acc_s / sum_s e^(m_s - M) l_s (the log-sum-exp
    rescale).  ms, ls: [S, ...]; accs: [S, ..., d].  Returns out [..., d]."""
    ms = np.asarray(ms, dtype=np.float64)
    ls = np.asarray(ls, dtype=np.float64)
    accs = np.asarray(accs, dtype=np.float64)
    M = np.max(ms, axis=0)
    w = np.exp(ms - M[None])                     # empty slices: exp(-inf) = 0
    L = np.sum(w * ls, axis=0)
    return np.sum(w[..., None] * accs, axis=0) / L[..., None]


def topk(scores: np.ndarray, k: int):
    """The k largest scores per row, ordered by score descending then index
    ascending.  Returns (indices int64 [nq, k], values [nq, k])."""
    scores = np.atleast_2d(scores)
    N = scores.shape[1]
    order = np.lexsort((np.broadcast_to(np.arange(N), scores.shape), -scores), axis=1)[:, :k]
    return order, np.take_along_axis(scores, order, axis=1)


def channel_split(scales: np.ndarray, n_high: int):
    """Outlier channels kept at higher precision
    ([tq.net, "TurboQuant 最近的进展和外溢影响"]: ordinary parts at very low bit width,
    outliers kept separately at higher precision; [ttakun, "为什么TurboQuant..."]: 3.5
    bits per channel).  Reading: the ``n_high`` channels with the largest
    generated scale form the high-precision group, fixed before streaming; both
    groups keep ascending channel order.  Returns (high, low) index arrays."""
    order = np.argsort(-np.asarray(scales), kind="stable")
    hi = np.sort(order[:n_high])
    lo = np.sort(order[n_high:])
    return hi, lo
