#!/usr/bin/env python
"""Throughput of the TurboQuant hot path on B200 (one JSON line on rank 0).

Default workload ("sweep"): TurboQuant_mse quantize + dequantize of N = 2^20
bf16 vectors, d = 128, per-channel lognormal(0, 1) scales with 4 of 128
channels x20 outliers, for b = 1, 2, 3, 4.  One step = quantize and dequantize
the batch at every b; the metric counts vectors quantized per second.  The
decode-attention workload over a compressed K/V cache (B = 8, 32 q-heads,
8 kv-heads, d = 128, context 131072, K prod 4-bit, V mse 4-bit) is measured in
the same run and reported under "decode".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload sweep|decode]

For N > 1 (torchrun, one rank per GPU) every rank processes its own batch:
the path has no exchange step, so there is no collective in the data path
("scaling": "weak"); the time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

D = 128
SWEEP_N = 1 << 20
SWEEP_BITS = (1, 2, 3, 4)
DEC = dict(B=8, Hq=32, Hkv=8, T=131072)
METRIC = "vectors quantized/s; packed-KV logits keys/s and % of HBM-bandwidth roofline"


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the
# sweep kernels, averaged over b = 1..4, from one ncu capture (the summary file
# named in "capture").  "sources" fingerprints the kernel sources the capture
# ran: when they differ from the files in this tree the figure is stale and
# roofline.traffic is reported as null.
MEASURED_TRAFFIC = {
    "quant_mse": {"bytes": 299.5e6, "sources": "3c007b3786cd370d", "capture": "profiles/sweep_traffic_bf16_d128.md"},
    "dequant_mse": {"bytes": 519.3e6, "sources": "1e172447f3500502", "capture": "profiles/sweep_traffic_bf16_d128.md"},
}
TRAFFIC_SOURCES = {
    "quant_mse": ["quant_tc.cu", "sm100_common.cuh"],
    "dequant_mse": ["dequant_tc.cu", "sm100_common.cuh"],
}


def source_fingerprint(kernel: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in TRAFFIC_SOURCES[kernel]:
        with open(os.path.join(ROOT, "compressed_kv_cache_turboquant_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str):
    """(bytes per launch, note): the ncu figure if the kernel is unchanged since
    it was captured, else (None, why)."""
    rec = MEASURED_TRAFFIC.get(kernel)
    if not rec or rec["bytes"] is None:
        return None, "no ncu capture of the current kernel"
    if rec["sources"] != source_fingerprint(kernel):
        return None, "stale: the kernel changed since the capture"
    return rec["bytes"], rec["capture"]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9 and parts[1].isdigit():
                        rows.append(parts)
        finally:
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [int(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(int(r[2]) for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------- oracle baseline

def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] or [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_sweep_rate(n_sample: int, bits=SWEEP_BITS, seed: int = 0):
    """The oracle (as it stands) on a bounded sample of the sweep workload:
    quantize + pack + dequantize n_sample rows at each b.  Returns vectors/s."""
    from oracle import codebook as ocb
    from oracle import turboquant as oq
    G = synth.gaussian_matrix(D, D, seed, synth.ROT_K)
    Pi = oq.haar_rotation(G)
    books = {b: ocb.lloyd_max(b, D) for b in bits}
    x = synth.to_bf16_exact(synth.scaled_gaussian_rows(n_sample, D, 1.0, seed=seed, outliers=4)).astype(np.float64)
    t0 = time.perf_counter()
    for b in bits:
        c, t = books[b]
        idx, n, _ = oq.quant_mse(x, Pi, t)
        oq.pack_codes_vec(idx, b)
        oq.dequant_mse(idx, n, Pi, c)
    dt = time.perf_counter() - t0
    return n_sample * len(bits) / dt, dt


def single_thread(fn, *args):
    """fn(*args) with the BLAS thread pools held to one thread."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        return fn(*args)


def oracle_decode_rate(T_sample: int, seed: int = 0):
    """Oracle decode for one (batch, kv-head) slice of T_sample tokens and its
    4 q-heads (logits, softmax, value sum).  Returns keys/s."""
    from oracle import codebook as ocb
    from oracle import turboquant as oq
    Pk = oq.haar_rotation(synth.gaussian_matrix(D, D, seed, synth.ROT_K))
    Sk = synth.gaussian_matrix(D, D, seed, synth.QJL_K)
    Pv = oq.haar_rotation(synth.gaussian_matrix(D, D, seed, synth.ROT_V))
    c3, t3 = ocb.lloyd_max(3, D)
    c4, t4 = ocb.lloyd_max(4, D)
    k = synth.kv_head_rows(T_sample, D, 0, 0, 0, seed=seed)
    v = synth.kv_head_rows(T_sample, D, 1, 0, 0, seed=seed)
    ks = oq.quant_prod(k, 4, Pk, Sk, t3, c3)
    vi, vn, _ = oq.quant_mse(v, Pv, t4)
    q = synth.decode_queries(1, 4, D, seed=seed)
    t0 = time.perf_counter()
    vhat = oq.dequant_mse(vi, vn, Pv, c4)
    oq.attention_decode(q, lambda b, h, qs: oq.prod_estimate(qs, ks["idx"], ks["norms"], ks["signs"], ks["rnorms"],
                                                             Pk, Sk, c3, 4), lambda b, h: vhat, 1)
    dt = time.perf_counter() - t0
    return T_sample / dt, dt


def oracle_search_rate(N: int, nq: int, d: int, b: int = 4, seed: int = 0):
    """The oracle on a bounded sample of the search workload: quantize N unit
    database vectors (prod, b bits), then score nq queries against all of them
    with the estimator.  Returns (vectors/s, pairs/s, seconds)."""
    from oracle import codebook as ocb
    from oracle import turboquant as oq
    P = oq.haar_rotation(synth.gaussian_matrix(d, d, seed, synth.ROT_K))
    S = synth.gaussian_matrix(d, d, seed, synth.QJL_K)
    c, t = ocb.lloyd_max(b - 1, d)
    x = synth.unit_rows(N, d, seed)
    q = synth.unit_rows(nq, d, seed, stream=synth.QUERY)
    t0 = time.perf_counter()
    st = oq.quant_prod(x, b, P, S, t, c)
    t1 = time.perf_counter()
    oq.prod_estimate(q, st["idx"], st["norms"], st["signs"], st["rnorms"], P, S, c, b)
    t2 = time.perf_counter()
    return N / (t1 - t0), N * nq / (t2 - t1), t2 - t0


def oracle_stream_rate(T_sample: int, seed: int = 0):
    """The oracle's full-context logits for one kv-head of the split cache (64
    channels at prod 4 bits + 64 at prod 3 bits, 4 q-heads) over T_sample
    tokens.  Returns (keys/s, seconds)."""
    from oracle import codebook as ocb
    from oracle import turboquant as oq
    scales = synth.lognormal_channel_scales(D, 1.0, seed, 30)
    hi, lo = oq.channel_split(scales, 64)
    k = synth.rng(seed, synth.DATA, 40, 0).standard_normal((T_sample, D)) * scales[None, :]
    q = synth.decode_queries(1, 4, D, seed=seed)[0]
    groups = []
    for grp, (b, ch) in enumerate(((4, hi), (3, lo))):
        P = oq.haar_rotation(synth.gaussian_matrix(64, 64, seed, synth.ROT_K, grp))
        S = synth.gaussian_matrix(64, 64, seed, synth.QJL_K, grp)
        c, t = ocb.lloyd_max(b - 1, 64)
        groups.append((b, ch, P, S, c, oq.quant_prod(k[:, ch], b, P, S, t, c)))
    t0 = time.perf_counter()
    logits = np.zeros((4, T_sample))
    for b, ch, P, S, c, st in groups:
        logits += oq.prod_estimate(q[:, ch], st["idx"], st["norms"], st["signs"], st["rnorms"], P, S, c, b)
    dt = time.perf_counter() - t0
    return T_sample / dt, dt


def oracle_sub_baselines(search_d: int):
    """Oracle rates beside the decode, stream and search sub-results (bounded
    samples, all host threads); each entry says what its sample was."""
    cores = cpu_threads()
    out = {}
    r, dt = oracle_decode_rate(1 << 16)
    out["decode"] = {"value": r, "unit": "keys/s", "cores": cores, "kind": "oracle",
                     "sample": f"one (batch, kv-head) slice of 65536 tokens, 4 q-heads ({dt:.1f} s)"}
    r, dt = oracle_stream_rate(1 << 16)
    out["stream"] = {"value": r, "unit": "keys/s", "cores": cores, "kind": "oracle",
                     "sample": f"logits of one kv-head over 65536 tokens of the split cache, 4 q-heads ({dt:.1f} s)"}
    qv, pr, dt = oracle_search_rate(10 ** 5, 64, search_d)
    out["search"] = {"quantize_vectors_per_s": qv, "score_pairs_per_s": pr, "cores": cores, "kind": "oracle",
                     "sample": f"quantize 10^5 vectors, then 64 queries x 10^5 keys, d={search_d}, prod b=4 "
                               f"({dt:.1f} s)"}
    return out


# ----------------------------------------------------------------- GPU workloads

class Sweep:
    """Config: N = 2^20 bf16 vectors (256 MiB > L2), d = 128, b = 1..4."""

    def __init__(self, tq, torch, rank, dev):
        self.tq, self.torch, self.dev = tq, torch, dev
        self.N = SWEEP_N
        G = synth.gaussian_matrix(D, D, 0, synth.ROT_K)
        Pi = tq.tq_make_rotation(G)
        self.h = {b: tq.tq_create(D, b, tq.TQ_MSE, Pi) for b in SWEEP_BITS}
        g = torch.Generator(device=dev).manual_seed(1000 + rank)
        s = synth.lognormal_channel_scales(D, 1.0, 0)
        s[synth.outlier_channels(D, 4, 0)] *= 20.0
        scale = torch.tensor(s, dtype=torch.float32, device=dev)
        self.x = (torch.randn((self.N, D), generator=g, device=dev) * scale).to(torch.bfloat16)
        self.codes = {b: torch.empty((self.N, self.h[b].words), dtype=torch.int32, device=dev) for b in SWEEP_BITS}
        self.norms = {b: torch.empty(self.N, dtype=torch.float32, device=dev) for b in SWEEP_BITS}
        self.xh = torch.empty((self.N, D), dtype=torch.float32, device=dev)
        self.stream = torch.cuda.current_stream()
        self.kern = {"quant_mse": [], "dequant_mse": []}
        self.launches_per_step = 2 * len(SWEEP_BITS)

    def step(self, record=False):
        tq, torch = self.tq, self.torch
        for b in SWEEP_BITS:
            if record:
                e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
                e0.record(self.stream)
            tq.tq_quant_mse(self.h[b], self.x, self.codes[b], self.norms[b])
            if record:
                e1.record(self.stream)
            tq.tq_dequant_mse(self.h[b], self.codes[b], self.norms[b], self.xh)
            if record:
                e2.record(self.stream)
                self.kern["quant_mse"].append((e0, e1, b))
                self.kern["dequant_mse"].append((e1, e2, b))

    def launch_bytes(self, name, b):
        """Algorithmic bytes of one launch: quantize reads bf16 x and writes codes
        and norms, dequantize reads codes and norms and writes fp32 x_hat."""
        return self.N * (D * 2 + 16 * b + 4) if name == "quant_mse" else self.N * (16 * b + 4 + D * 4)

    def kernel_stats(self):
        out = {}
        for name, evs in self.kern.items():
            ms = [a.elapsed_time(bb) for a, bb, _ in evs]
            bytes_ = [self.launch_bytes(name, b) for _, _, b in evs]
            per_b = {}
            for (_, _, b), t in zip(evs, ms):
                per_b.setdefault(b, []).append(t)
            out[name] = dict(ms_total=sum(ms), launches=len(ms), bytes_total=sum(bytes_),
                             per_b={b: (sum(v) / len(v), self.launch_bytes(name, b)) for b, v in per_b.items()})
        return out

    def units_per_step(self):
        return self.N * len(SWEEP_BITS)

    # ---- end to end through host buffers
    def distortion(self):
        """Per b: the measured mean ||x - x_hat||^2 / ||x||^2 of the batch (an untimed
        round trip) beside 4^-b, the lower bound the pages compare it with."""
        out = {}
        for b in SWEEP_BITS:
            self.tq.tq_quant_mse(self.h[b], self.x, self.codes[b], self.norms[b])
            self.tq.tq_dequant_mse(self.h[b], self.codes[b], self.norms[b], self.xh)
            D = mean_relative_sq_error(self.torch, self.x, self.xh)
            out[f"b{b}"] = {"D": D, "4^-b": 4.0 ** -b, "D_times_4^b": D * 4.0 ** b}
        return out

    def e2e(self, steps, warmup, nchunk=8):
        """The step through the public API from pinned host memory: x goes up, codes
        and norms come back.  The batch is cut into `nchunk` row ranges on three
        streams (host-to-device copy, the library calls, device-to-host copy), so
        the two copy directions overlap each other and the kernels.  Returns
        (ms per step, H2D bytes, D2H bytes, check) where check says that one step
        from zeroed outputs brought back the codes of a plain call."""
        tq, torch = self.tq, self.torch
        xh_host = self.x.cpu().pin_memory()
        outs = {b: (torch.empty(self.codes[b].shape, dtype=torch.int32).pin_memory(),
                    torch.empty(self.N, dtype=torch.float32).pin_memory()) for b in SWEEP_BITS}
        xd = torch.empty_like(self.x)
        up, work, down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        E = lambda: torch.cuda.Event()
        ev_up, ev_work, ev_down = [E() for _ in range(nchunk)], [E() for _ in range(nchunk)], [E() for _ in range(nchunk)]
        rows = -(-self.N // nchunk)
        spans = [slice(k * rows, min(self.N, (k + 1) * rows)) for k in range(nchunk)]

        def one():
            for k, sl in enumerate(spans):
                with torch.cuda.stream(up):
                    up.wait_event(ev_work[k])          # the previous step's kernels have read xd[sl]
                    xd[sl].copy_(xh_host[sl], non_blocking=True)
                    ev_up[k].record(up)
                with torch.cuda.stream(work):
                    work.wait_event(ev_up[k])
                    work.wait_event(ev_down[k])        # the previous step's copies have read the outputs
                    for b in SWEEP_BITS:
                        tq.tq_quant_mse(self.h[b], xd[sl], self.codes[b][sl], self.norms[b][sl])
                        tq.tq_dequant_mse(self.h[b], self.codes[b][sl], self.norms[b][sl], self.xh[sl])
                    ev_work[k].record(work)
                with torch.cuda.stream(down):
                    down.wait_event(ev_work[k])
                    for b in SWEEP_BITS:
                        outs[b][0][sl].copy_(self.codes[b][sl], non_blocking=True)
                        outs[b][1][sl].copy_(self.norms[b][sl], non_blocking=True)
                    ev_down[k].record(down)

        def join(stream):
            for st in (up, work, down):
                stream.wait_stream(st)

        cur = torch.cuda.current_stream()
        # check: from zeroed device and host outputs, one step must bring back a plain call's codes
        tq.tq_quant_mse(self.h[SWEEP_BITS[-1]], self.x, self.codes[SWEEP_BITS[-1]], self.norms[SWEEP_BITS[-1]])
        ref = self.codes[SWEEP_BITS[-1]].cpu()
        for b in SWEEP_BITS:
            self.codes[b].zero_()
            outs[b][0].zero_()
        torch.cuda.synchronize()
        for st in (up, work, down):
            st.wait_stream(cur)
        one()
        join(cur)
        torch.cuda.synchronize()
        check = bool(torch.equal(outs[SWEEP_BITS[-1]][0], ref))
        for _ in range(warmup):
            one()
        join(cur)
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(cur)
        for st in (up, work, down):
            st.wait_stream(cur)
        for _ in range(steps):
            one()
        join(cur)
        e.record(cur)
        torch.cuda.synchronize()
        ms = s.elapsed_time(e) / steps
        h2d = self.x.numel() * 2
        d2h = sum(self.codes[b].numel() * 4 + self.N * 4 for b in SWEEP_BITS)
        return ms, h2d, d2h, check


class Decode:
    """Config: B = 8, Hq = 32, Hkv = 8, d = 128, T = 131072; K prod 4b (3+1), V mse 4b."""

    def __init__(self, tq, torch, rank, dev):
        self.tq, self.torch, self.dev = tq, torch, dev
        B, Hq, Hkv, T = DEC["B"], DEC["Hq"], DEC["Hkv"], DEC["T"]
        self.B, self.Hq, self.Hkv, self.T = B, Hq, Hkv, T
        Pk = tq.tq_make_rotation(synth.gaussian_matrix(D, D, 0, synth.ROT_K))
        Sk = synth.gaussian_matrix(D, D, 0, synth.QJL_K)
        Pv = tq.tq_make_rotation(synth.gaussian_matrix(D, D, 0, synth.ROT_V))
        self.hk = tq.tq_create(D, 4, tq.TQ_PROD, Pk, Sk)
        self.hv = tq.tq_create(D, 4, tq.TQ_MSE, Pv)
        rows = B * Hkv * T
        self.kcodes = torch.empty((rows, self.hk.words), dtype=torch.int32, device=dev)
        self.ksigns = torch.empty((rows, tq.sign_words(D)), dtype=torch.int32, device=dev)
        self.knorms = torch.empty(rows, dtype=torch.float32, device=dev)
        self.krnorms = torch.empty(rows, dtype=torch.float32, device=dev)
        self.vcodes = torch.empty((rows, self.hv.words), dtype=torch.int32, device=dev)
        self.vnorms = torch.empty(rows, dtype=torch.float32, device=dev)
        g = torch.Generator(device=dev).manual_seed(2000 + rank)
        chunk = T  # one (batch, kv-head) slice at a time: bounded temporary memory
        for bh in range(B * Hkv):
            h = bh % Hkv
            for kind in (0, 1):
                s = torch.tensor(synth.lognormal_channel_scales(D, 1.0, 0, 10 + kind, h), dtype=torch.float32,
                                 device=dev)
                x = (torch.randn((chunk, D), generator=g, device=dev) * s).to(torch.bfloat16)
                sl = slice(bh * T, (bh + 1) * T)
                if kind == 0:
                    tq.tq_quant_prod(self.hk, x, self.kcodes[sl], self.ksigns[sl], self.knorms[sl], self.krnorms[sl])
                else:
                    tq.tq_quant_mse(self.hv, x, self.vcodes[sl], self.vnorms[sl])
        sq = torch.tensor(synth.lognormal_channel_scales(D, 1.0, 0, 20), dtype=torch.float32, device=dev)
        self.q = (torch.randn((B, Hq, D), generator=g, device=dev) * sq).to(torch.bfloat16)
        self.out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
        self.ws = torch.empty(max(1, tq.tq_attn_decode_workspace(self.hk, B, Hq, Hkv, T)), dtype=torch.uint8,
                              device=dev)
        self.stream = torch.cuda.current_stream()
        self.kern = []
        self.scale = 1.0 / math.sqrt(D)

    def step(self, record=False):
        tq, torch = self.tq, self.torch
        if record:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
        tq.tq_attn_decode(self.hk, self.hv, self.q, self.Hkv, self.T, self.T, self.kcodes, self.ksigns, self.knorms,
                          self.krnorms, self.vcodes, self.vnorms, self.scale, self.out, self.ws)
        if record:
            e1.record(self.stream)
            self.kern.append((e0, e1))

    def bytes_per_step(self):
        # packed K (48 B codes + 16 B signs + 4 + 4 B norms) + V (64 B codes + 4 B norm) per token
        return self.B * self.Hkv * self.T * (48 + 16 + 8 + 64 + 4)

    def units_per_step(self):
        return self.B * self.Hkv * self.T


class Prefill:
    """Prefill over the decode configuration's cache: B = 8, Hq = 32, Hkv = 8,
    d = 128, T = 131072 (K prod 4b, V mse 4b); a block of nq = 512 new tokens
    at the end of the context attends causally.  One step = one
    tq_attn_prefill call (query prep, the tensor-core kernel, the merge)."""

    def __init__(self, tq, torch, dec, nq=512):
        self.tq, self.torch, self.dec, self.nq = tq, torch, dec, nq
        g = torch.Generator(device=dec.dev).manual_seed(5000)
        sq = torch.tensor(synth.lognormal_channel_scales(D, 1.0, 0, 21), dtype=torch.float32, device=dec.dev)
        self.q = (torch.randn((dec.B, nq, dec.Hq, D), generator=g, device=dec.dev) * sq).to(torch.bfloat16)
        self.out = torch.empty((dec.B, nq, dec.Hq, D), dtype=torch.float32, device=dec.dev)
        self.ws = torch.empty(max(1, tq.tq_attn_prefill_workspace(dec.hk, dec.B, nq, dec.Hq, dec.Hkv, dec.T)),
                              dtype=torch.uint8, device=dec.dev)
        self.ev = []

    def step(self, record=False):
        d = self.dec
        if record:
            e0, e1 = self.torch.cuda.Event(enable_timing=True), self.torch.cuda.Event(enable_timing=True)
            e0.record(d.stream)
        self.tq.tq_attn_prefill(d.hk, d.hv, self.q, d.Hkv, d.T, d.T, d.kcodes, d.ksigns, d.knorms, d.krnorms,
                                d.vcodes, d.vnorms, d.scale, self.out, self.ws)
        if record:
            e1.record(d.stream)
            self.ev.append((e0, e1))

    def flops(self):
        # 6 d FLOP per (query row, visible key): the two logit products and the value product
        d = self.dec
        vis = sum(d.T - self.nq + i + 1 for i in range(self.nq))
        return 6.0 * D * d.B * d.Hq * vis


class Stream:
    """Config: batch 1, 32 q-heads / 8 kv-heads, d = 128, context 2^20; keys split
    into the 64 largest-scale channels at prod 4 bits and 64 at prod 3 bits
    (3.5 bits per channel).  One step = append one token for every kv-head
    (per-token quantization of both channel groups) + full-context logits."""

    def __init__(self, tq, torch, rank, dev, T=1 << 20):
        from_np = lambda a: torch.tensor(a, device=dev)
        self.tq, self.torch, self.dev = tq, torch, dev
        self.Hq, self.Hkv, self.T = 32, 8, T
        scales = synth.lognormal_channel_scales(D, 1.0, 0, 30)
        order = np.argsort(-scales, kind="stable")
        hi, lo = np.sort(order[:64]), np.sort(order[64:])
        self.channels = from_np(np.concatenate([hi, lo]).astype(np.int32))
        self.h = []
        for grp, b in ((0, 4), (1, 3)):
            P = tq.tq_make_rotation(synth.gaussian_matrix(64, 64, 0, synth.ROT_K, grp))
            S = synth.gaussian_matrix(64, 64, 0, synth.QJL_K, grp)
            self.h.append(tq.tq_create(64, b, tq.TQ_PROD, P, S))
        rows = self.Hkv * T
        self.cache = []
        for h in self.h:
            self.cache.append(dict(codes=torch.empty((rows, h.words), dtype=torch.int32, device=dev),
                                   signs=torch.empty((rows, 2), dtype=torch.int32, device=dev),
                                   norms=torch.empty(rows, dtype=torch.float32, device=dev),
                                   rnorms=torch.empty(rows, dtype=torch.float32, device=dev)))
        g = torch.Generator(device=dev).manual_seed(3000 + rank)
        sc = torch.tensor(scales, dtype=torch.float32, device=dev)
        for hh in range(self.Hkv):
            x = (torch.randn((T, D), generator=g, device=dev) * sc).to(torch.bfloat16)
            sl = slice(hh * T, (hh + 1) * T)
            for k, (h, c) in enumerate(zip(self.h, self.cache)):
                tq.tq_quant_gather(h, x, self.channels[64 * k:64 * (k + 1)], c["codes"][sl], c["norms"][sl],
                                   signs=c["signs"][sl], rnorms=c["rnorms"][sl])
        self.token = (torch.randn((self.Hkv, D), generator=g, device=dev) * sc).to(torch.bfloat16)
        sq = torch.tensor(synth.lognormal_channel_scales(D, 1.0, 0, 20), dtype=torch.float32, device=dev)
        self.q = (torch.randn((1, self.Hq, D), generator=g, device=dev) * sq).to(torch.bfloat16)
        self.logits = torch.empty((1, self.Hq, T), dtype=torch.float32, device=dev)
        self.ws = torch.empty(max(1, tq.tq_attn_logits_workspace(self.h, 1, self.Hq)), dtype=torch.uint8, device=dev)
        self.stream = torch.cuda.current_stream()
        self.app, self.lgt = [], []

    def step(self, record=False):
        tq, torch = self.tq, self.torch
        E = lambda: torch.cuda.Event(enable_timing=True)
        if record:
            e0, e1, e2 = E(), E(), E()
            e0.record(self.stream)
        t = self.T - 1  # slot of the arriving token: both channel groups of every kv-head in one launch
        tq.tq_quant_gather_groups(self.h, self.token, self.channels, [c["codes"][t:] for c in self.cache],
                                  [c["norms"][t:] for c in self.cache], signs=[c["signs"][t:] for c in self.cache],
                                  rnorms=[c["rnorms"][t:] for c in self.cache], out_stride=self.T)
        if record:
            e1.record(self.stream)
        self.logits_only()
        if record:
            e2.record(self.stream)
            self.app.append((e0, e1))
            self.lgt.append((e1, e2))

    def logits_only(self):
        self.tq.tq_attn_logits(self.h, self.channels, self.q, self.Hkv, self.T, self.T,
                               [c["codes"] for c in self.cache], [c["signs"] for c in self.cache],
                               [c["norms"] for c in self.cache], [c["rnorms"] for c in self.cache],
                               1.0 / math.sqrt(D), self.logits, self.ws)

    def bytes_logits(self):
        # per token per kv-head: group A 24 B codes + 8 B signs + 8 B norms, group B 16 + 8 + 8, logits 4 x 4 B
        return self.Hkv * self.T * (40 + 32 + 16)


class Search:
    """Config: N = 10^6 unit-norm fp32 database vectors (Gaussian, normalised),
    10^4 unit queries, TurboQuant_prod at b total bits, d = 200 or 1536.  One
    step = quantize the database, then score every (query, vector) pair with a
    fused top-10 (the full score matrix is not written)."""

    def __init__(self, tq, torch, rank, dev, d=200, b=4, N=10 ** 6, nq=10 ** 4, topk=10):
        self.tq, self.torch, self.dev = tq, torch, dev
        self.d, self.b, self.N, self.nq, self.topk = d, b, N, nq, topk
        P = tq.tq_make_rotation(synth.gaussian_matrix(d, d, 0, synth.ROT_K))
        S = synth.gaussian_matrix(d, d, 0, synth.QJL_K)
        self.h = tq.tq_create(d, b, tq.TQ_PROD, P, S)
        g = torch.Generator(device=dev).manual_seed(4000 + rank)
        x = torch.randn((N, d), generator=g, device=dev)
        self.x = x / x.norm(dim=1, keepdim=True)
        q = torch.randn((nq, d), generator=g, device=dev)
        self.q = q / q.norm(dim=1, keepdim=True)
        self.codes = torch.empty((N, self.h.words), dtype=torch.int32, device=dev)
        self.signs = torch.empty((N, tq.sign_words(d)), dtype=torch.int32, device=dev)
        self.norms = torch.empty(N, dtype=torch.float32, device=dev)
        self.rnorms = torch.empty(N, dtype=torch.float32, device=dev)
        self.ti = torch.empty((nq, topk), dtype=torch.int32, device=dev)
        self.tv = torch.empty((nq, topk), dtype=torch.float32, device=dev)
        self.ws = torch.empty(max(1, tq.tq_ip_scores_workspace(self.h, nq, N, topk)), dtype=torch.uint8,
                              device=dev)
        self.stream = torch.cuda.current_stream()
        self.quant, self.score = [], []

    def step(self, record=False):
        tq, torch = self.tq, self.torch
        E = lambda: torch.cuda.Event(enable_timing=True)
        if record:
            e0, e1, e2 = E(), E(), E()
            e0.record(self.stream)
        tq.tq_quant_prod(self.h, self.x, self.codes, self.signs, self.norms, self.rnorms)
        if record:
            e1.record(self.stream)
        tq.tq_ip_scores(self.h, self.q, self.codes, self.signs, self.norms, self.rnorms, topk=self.topk,
                        top_idx=self.ti, top_val=self.tv, workspace=self.ws)
        if record:
            e2.record(self.stream)
            self.quant.append((e0, e1))
            self.score.append((e1, e2))

    def recall(self, nsample=100):
        """recall@topk of the last fused top-k against exact fp32 inner products
        <q, x> (a library GEMM, outside the timed region) for the first queries."""
        ns = min(nsample, self.nq)
        exact = self.torch.matmul(self.q[:ns], self.x.t())
        return {"recall_at_k": recall_at_k(self.torch, exact, self.ti[:ns], self.topk), "k": self.topk,
                "queries": ns, "against": "exact fp32 <q, x> of the unquantized vectors"}

    def summary(self, hbm, tc_peak):
        qms = sum(a.elapsed_time(b) for a, b in self.quant) / len(self.quant)
        sms = sum(a.elapsed_time(b) for a, b in self.score) / len(self.score)
        d = self.d
        q_flop = 2 * 2 * d * d * self.N            # two d x d contractions per vector (rotation, QJL)
        s_flop = 4 * d * self.N * self.nq          # 2d MACs per pair (codebook part + sign part)
        return {"quantize_vectors_per_s": self.N / (qms / 1e3), "quantize_ms": qms,
                "quantize_TFLOPs": q_flop / (qms / 1e3) / 1e12,
                "score_pairs_per_s": self.N * self.nq / (sms / 1e3), "score_ms": sms,
                "score_TFLOPs": s_flop / (sms / 1e3) / 1e12,
                "score_frac_tensor": s_flop / (sms / 1e3) / 1e12 / tc_peak,
                "config": f"N={self.N} unit fp32, d={d}, nq={self.nq}, prod b={self.b}, fused top-{self.topk}"}


# ----------------------------------------------------------------- driver

class Ranks:
    """One process per GPU, ranks from the torchrun environment.  The path has
    no exchange step: the only collectives are the barrier around the timed
    region and the max-over-ranks reduction of its duration."""

    def __init__(self, backend: str = "nccl", device: str | None = None, timeout_s: int = 300):
        import torch
        import torch.distributed as dist
        self.torch, self.dist = torch, dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = device
        self.cuda = device is not None and device.startswith("cuda")
        if self.world > 1 and not dist.is_initialized():
            from datetime import timedelta
            kw = {"device_id": torch.device(device)} if self.cuda else {}
            dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s), **kw)

    def max(self, v: float) -> float:
        if self.world == 1:
            return v
        t = self.torch.tensor([v], dtype=self.torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()
        if self.cuda:
            self.torch.cuda.synchronize()

    def close(self):
        if self.world > 1 and self.dist.is_initialized():
            self.dist.destroy_process_group()


def mean_relative_sq_error(torch, x, xh, chunk=1 << 16) -> float:
    """Mean over rows of ||x - xh||^2 / ||x||^2 (rows with x = 0 left out): the
    distortion of a quantize + dequantize round trip, per vector."""
    tot, cnt = 0.0, 0
    for i in range(0, x.shape[0], chunk):
        a = x[i:i + chunk].float()
        e = (a - xh[i:i + chunk].float()).pow(2).sum(1)
        n = a.pow(2).sum(1)
        m = n > 0
        tot += (e[m] / n[m]).double().sum().item()
        cnt += int(m.sum().item())
    return tot / max(cnt, 1)


def recall_at_k(torch, exact_scores, got_idx, k) -> float:
    """Share of each row's exact top-k (by score) found among the k returned
    indices, averaged over rows."""
    ex = torch.topk(exact_scores, k, dim=1).indices
    hit = (ex.unsqueeze(2) == got_idx[:, :k].long().unsqueeze(1)).any(dim=2)
    return hit.float().mean().item()


def job_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return units_per_rank * world / (ms_max / 1e3)


def run_ours(args):
    import torch
    import compressed_kv_cache_turboquant_b200 as tq

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = f"cuda:{local}"
    ranks = Ranks("nccl", dev)
    world, rank = ranks.world, ranks.rank
    max_over_ranks, barrier = ranks.max, ranks.barrier

    hbm, bf16, peak_kind = peaks()
    wl_cls = Sweep if args.workload == "sweep" else Decode
    wl = wl_cls(tq, torch, rank, dev)
    for _ in range(args.warmup):
        wl.step()
    barrier()
    with ClockSampler(local) as clk:
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(args.steps):
            wl.step(record=True)
        e.record()
        torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(s.elapsed_time(e) / args.steps)
    units = wl.units_per_step() * world
    value = job_rate(wl.units_per_step(), world, ms)

    if args.workload == "sweep":
        ks = wl.kernel_stats()
        dom = max(ks, key=lambda k: ks[k]["ms_total"])
        unit_name = "vectors/s"
        config = workload_config("sweep", world)
        launches = wl.launches_per_step * args.steps
    else:
        k_ms = sum(a.elapsed_time(b) for a, b in wl.kern)
        ks = {"attn_decode": dict(ms_total=k_ms, launches=len(wl.kern), bytes_total=wl.bytes_per_step() * len(wl.kern))}
        dom = "attn_decode"
        unit_name = "keys/s"
        config = workload_config("decode", world)
        launches = 3 * args.steps
    dk = ks[dom]
    achieved = dk["bytes_total"] / (dk["ms_total"] / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "peak_source": f"{peak_kind} hbm_gbs (copy, burst)",
                "traffic": None, "bytes_per_launch": dk["bytes_total"] / dk["launches"]}
    if args.workload == "sweep":
        roofline["traffic"], roofline["traffic_source"] = measured_traffic(dom)
    kernels = {k: {"avg_ms": v["ms_total"] / v["launches"],
                   "GBps": v["bytes_total"] / (v["ms_total"] / 1e3) / 1e9,
                   "frac_hbm": v["bytes_total"] / (v["ms_total"] / 1e3) / 1e9 / hbm} for k, v in ks.items()}
    for k, v in ks.items():
        if "per_b" in v:  # each bit width on its own: average launch time and its fraction of the peak
            kernels[k]["per_b"] = {f"b{b}": {"us": round(t * 1e3, 2), "frac_hbm": round(by / (t / 1e3) / 1e9 / hbm, 4)}
                                   for b, (t, by) in sorted(v["per_b"].items())}

    e2e = None
    if args.workload == "sweep" and not args.no_e2e:
        e_ms, h2d, d2h, check = wl.e2e(max(2, args.steps // 2), 1)
        e_ms = max_over_ranks(e_ms)
        e2e = {"value": units / (e_ms / 1e3), "unit": unit_name, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e_ms, "pipeline": "8 row ranges on copy-up / kernel / copy-down streams",
               "outputs_checked": check}

    result = {"metric": METRIC, "value": value, "unit": unit_name, "n_gpus": world, "steps": args.steps,
              "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
              "vs_baseline": None, "dtype": "f32 (bf16 in, fp32 accumulate)", "data": "synthetic",
              "config": config, "roofline": roofline, "kernels": kernels, "e2e": e2e,
              "gpu_launches": launches, "clocks": clk.summary()}

    if args.workload == "sweep":
        try:
            result["distortion"] = wl.distortion()
        except Exception as exc:  # a quality figure must not cost the bench line
            result["distortion"] = {"error": repr(exc)}

    if args.workload == "sweep" and not args.no_decode:
        del wl
        torch.cuda.empty_cache()
        dl = Decode(tq, torch, rank, dev)
        for _ in range(args.warmup):
            dl.step()
        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record()
        for _ in range(args.steps):
            dl.step(record=True)
        e2.record()
        torch.cuda.synchronize()
        dms = max_over_ranks(s2.elapsed_time(e2) / args.steps)
        kms = sum(a.elapsed_time(b) for a, b in dl.kern) / len(dl.kern)
        gbs = dl.bytes_per_step() / (kms / 1e3) / 1e9
        result["decode"] = {"value": dl.units_per_step() * world / (dms / 1e3), "unit": "keys/s",
                            "ms_per_step": dms, "GBps": gbs, "frac_hbm": gbs / hbm,
                            "bytes_per_step": dl.bytes_per_step(),
                            "config": "B=8, Hq=32, Hkv=8, d=128, T=131072, K prod 4b, V mse 4b"}
        try:
            if args.no_prefill:
                raise RuntimeError("prefill not run (--no-prefill)")
            pf = Prefill(tq, torch, dl)
            for _ in range(args.warmup):
                pf.step()
            for _ in range(max(1, args.steps // 2)):
                pf.step(record=True)
            torch.cuda.synchronize()
            pms = max_over_ranks(sum(a.elapsed_time(b) for a, b in pf.ev) / len(pf.ev))
            tfl = pf.flops() / (pms / 1e3) / 1e12
            result["prefill"] = {"ms_per_step": pms, "tokens_per_s": dl.B * pf.nq * world / (pms / 1e3),
                                 "TFLOPs": tfl, "frac_tensor": tfl / bf16,
                                 "config": "decode cache (B=8, Hq=32, Hkv=8, d=128, T=131072), a causal block of "
                                           f"nq={pf.nq} new tokens; 6 d FLOP per (query row, visible key)"}
            del pf
        except Exception as exc:  # a sub-result must not cost the bench line
            result["prefill"] = {"error": repr(exc)}

    if args.workload == "sweep" and not args.no_decode:
        torch.cuda.empty_cache()
        sw = Stream(tq, torch, rank, dev)
        for _ in range(args.warmup):
            sw.step()
        barrier()
        for _ in range(args.steps):
            sw.step(record=True)
        torch.cuda.synchronize()
        app = max_over_ranks(sum(a.elapsed_time(b) for a, b in sw.app) / len(sw.app))
        lg = max_over_ranks(sum(a.elapsed_time(b) for a, b in sw.lgt) / len(sw.lgt))
        gbs = sw.bytes_logits() / (lg / 1e3) / 1e9
        result["stream"] = {"logits_value": sw.Hkv * sw.T * world / (lg / 1e3), "unit": "keys/s",
                            "logits_ms": lg, "GBps": gbs, "frac_hbm": gbs / hbm,
                            "bytes_per_logits_call": sw.bytes_logits(),
                            "append_us_per_token": app * 1e3,
                            "config": "B=1, Hq=32, Hkv=8, d=128 split 64 ch @ prod 4b + 64 ch @ prod 3b, T=2^20"}
        del sw

    if args.workload == "sweep" and not args.no_search:
        torch.cuda.empty_cache()
        sr = Search(tq, torch, rank, dev, d=args.search_d)
        for _ in range(args.warmup):
            sr.step()
        barrier()
        for _ in range(max(1, args.steps // 2)):
            sr.step(record=True)
        torch.cuda.synchronize()
        result["search"] = sr.summary(hbm, bf16)
        try:
            result["search"]["recall"] = sr.recall()
        except Exception as exc:
            result["search"]["recall"] = {"error": repr(exc)}
        del sr

    if rank == 0 and world == 1 and not args.no_cpu:
        if args.workload == "sweep":
            rate, dt = oracle_sweep_rate(args.cpu_sample)
            sample = f"{args.cpu_sample} vectors of the sweep workload at each b=1..4 ({dt:.1f} s)"
        else:
            rate, dt = oracle_decode_rate(args.cpu_sample)
            sample = f"one (batch, kv-head) slice of {args.cpu_sample} tokens, 4 q-heads ({dt:.1f} s)"
        result["cpu_baseline"] = {"value": rate, "unit": unit_name, "cores": cpu_threads(), "kind": "oracle",
                                  "sample": sample}
        try:  # the same oracle on one core, on an eighth of the sample
            fn = oracle_sweep_rate if args.workload == "sweep" else oracle_decode_rate
            rate1, dt1 = single_thread(fn, max(1, args.cpu_sample // 8))
            result["cpu_baseline"]["single_thread"] = {"value": rate1, "unit": unit_name, "cores": 1,
                                                       "sample": f"{args.cpu_sample // 8} units ({dt1:.1f} s)"}
        except Exception as exc:
            result["cpu_baseline"]["single_thread"] = {"error": repr(exc)}
        if args.workload == "sweep":
            try:
                subs = oracle_sub_baselines(args.search_d)
                for k, v in subs.items():
                    if k in result:
                        result[k]["cpu_baseline"] = v
            except Exception as exc:
                result["cpu_baseline"]["sub_results"] = {"error": repr(exc)}
    if rank == 0:
        print(json.dumps(result), flush=True)
    ranks.close()


PROFILE_CASES = {
    "decode": "decode attention, config-4 shape at context --profile-t (default 32768)",
    "logits": "split-cache logits, config-5 shape at context --profile-t (default 2^18)",
    "search": "quantize + fused top-10 scoring: d = --search-d, --profile-n keys (default 200000), "
              "--profile-nq queries (default 1280)",
    "sweep": "the sweep step (quantize + dequantize at b = 1..4, 2^20 bf16 vectors)",
    "prefill": "prefill of --profile-nq new tokens (default 128) over the config-4 cache at context --profile-t "
               "(default 32768)",
}


def run_profile_case(args):
    """Small cases of the hot-path calls for ncu captures: set-up, then
    --profile-launches calls of the case's step, and one JSON line with each
    call's CUDA-event time.  Not a bench result."""
    import torch
    import compressed_kv_cache_turboquant_b200 as tq

    torch.cuda.set_device(0)
    dev, case = "cuda:0", args.profile_case
    if case == "decode":
        DEC["T"] = args.profile_t or 32768
        wl = Decode(tq, torch, 0, dev)
        call, size = wl.step, {"T": DEC["T"]}
    elif case == "logits":
        wl = Stream(tq, torch, 0, dev, T=args.profile_t or (1 << 18))
        call, size = wl.logits_only, {"T": wl.T}
    elif case == "prefill":
        DEC["T"] = args.profile_t or 32768
        dec = Decode(tq, torch, 0, dev)
        wl = Prefill(tq, torch, dec, nq=args.profile_nq or 128)
        call, size = wl.step, {"T": DEC["T"], "nq": wl.nq}
    elif case == "search":
        n, nq = args.profile_n or 200000, args.profile_nq or 1280
        wl = Search(tq, torch, 0, dev, d=args.search_d, N=n, nq=nq)
        call, size = wl.step, {"d": args.search_d, "N": n, "nq": nq}
    else:
        wl = Sweep(tq, torch, 0, dev)
        call, size = wl.step, {"N": SWEEP_N}
    ms = []
    for _ in range(args.profile_launches):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1))
    print(json.dumps({"profile_case": case, "what": PROFILE_CASES[case], "size": size, "ms": ms}), flush=True)


def workload_config(workload: str, world: int) -> dict:
    """The `config` object of the JSON line, the same for both arms."""
    if workload == "sweep":
        return {"workload": "TurboQuant_mse quant+dequant sweep b=1..4, N=2^20 bf16, d=128, lognormal(0,1) "
                            "channel scales, 4 channels x20 outliers",
                "N": SWEEP_N, "d": D, "bits": list(SWEEP_BITS), "input_dtype": "bf16",
                "dequant_dtype": "f32", "l2": "inputs larger than L2 (256 MiB bf16 per step per b)",
                "parallelism": f"dp{world} (independent batches, no collective)"}
    return {"workload": "decode attention over TurboQuant K/V: B=8, Hq=32, Hkv=8, d=128, T=131072, "
                        "K prod 4b (3+1 QJL), V mse 4b, bf16 queries",
            "B": DEC["B"], "Hq": DEC["Hq"], "Hkv": DEC["Hkv"], "T": DEC["T"], "d": D,
            "l2": "packed cache 1.17 GB > L2", "parallelism": f"dp{world} (independent caches)"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    times = []
    fn = oracle_sweep_rate if args.workload == "sweep" else oracle_decode_rate
    for i in range(args.warmup + args.steps):
        rate, dt = fn(args.ref_sample)
        if i >= args.warmup:
            times.append(dt)
    per = args.ref_sample * (len(SWEEP_BITS) if args.workload == "sweep" else 1)
    value = per / (sum(times) / len(times))
    unit = "vectors/s" if args.workload == "sweep" else "keys/s"
    cores = cpu_threads()
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.workload, world),
        "cpu_baseline": {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": (f"{args.ref_sample} vectors at each b = 1..4 per step (a bounded sample of the "
                                    f"sweep)" if args.workload == "sweep" else
                                    f"{args.ref_sample} tokens of one (batch, kv-head) slice, 4 q-heads, per step "
                                    f"(a bounded sample of the decode workload)")},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["sweep", "decode"], default="sweep")
    ap.add_argument("--cpu-sample", type=int, default=None)
    ap.add_argument("--ref-sample", type=int, default=None)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-search", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--search-d", type=int, default=200)
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES), default=None,
                    help="run a small case of one workload for an ncu capture instead of the bench")
    ap.add_argument("--profile-launches", type=int, default=3)
    ap.add_argument("--profile-t", type=int, default=None)
    ap.add_argument("--profile-n", type=int, default=None)
    ap.add_argument("--profile-nq", type=int, default=None)
    args = ap.parse_args()
    if args.profile_case:
        run_profile_case(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.cpu_sample is None:
        args.cpu_sample = 1 << 19 if args.workload == "sweep" else 1 << 17
    if args.ref_sample is None:
        args.ref_sample = 1 << 14 if args.workload == "sweep" else 1 << 13
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
