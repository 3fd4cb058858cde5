"""Host-side helpers of bench.py that turn GPU outputs into quality figures
(sweep distortion, search recall@k), checked on small CPU tensors."""
import os
import sys

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def test_mean_relative_sq_error_by_hand():
    x = torch.tensor([[3.0, 4.0], [1.0, 0.0], [0.0, 0.0]])
    xh = torch.tensor([[3.0, 3.0], [0.0, 0.0], [5.0, 5.0]])
    # rows: 1/25, 1/1; the zero row is left out
    got = bench.mean_relative_sq_error(torch, x, xh, chunk=2)
    assert got == pytest.approx((1 / 25 + 1.0) / 2)


def test_mean_relative_sq_error_bf16_input():
    x = torch.randn(1000, 16).to(torch.bfloat16)
    assert bench.mean_relative_sq_error(torch, x, x.float()) == 0.0


def test_recall_at_k():
    s = torch.tensor([[5.0, 4.0, 3.0, 2.0, 1.0],
                      [1.0, 2.0, 3.0, 4.0, 5.0]])
    got = torch.tensor([[0, 1, 4], [4, 3, 2]], dtype=torch.int32)
    # row 0: exact top-3 {0, 1, 2}, found {0, 1} -> 2/3; row 1: all found
    assert bench.recall_at_k(torch, s, got, 3) == pytest.approx((2 / 3 + 1) / 2)


def test_recall_order_does_not_matter():
    s = torch.randn(4, 50)
    ex = torch.topk(s, 10, dim=1).indices
    assert bench.recall_at_k(torch, s, ex.flip(1).to(torch.int32), 10) == 1.0


def test_single_thread_holds_blas_to_one_thread():
    got = bench.single_thread(bench.cpu_threads)
    assert got == 1
    rate, dt = bench.single_thread(bench.oracle_sweep_rate, 256)
    assert rate > 0 and dt > 0


def test_both_arms_share_the_workload_config():
    c = bench.workload_config("sweep", 2)
    assert c["N"] == 1 << 20 and c["bits"] == [1, 2, 3, 4] and c["parallelism"].startswith("dp2")
    d = bench.workload_config("decode", 1)
    assert (d["B"], d["Hq"], d["Hkv"], d["T"], d["d"]) == (8, 32, 8, 131072, 128)


def test_traffic_figure_is_dropped_when_the_kernel_changed(monkeypatch):
    fp = bench.source_fingerprint("dequant_mse")
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, "dequant_mse",
                        {"bytes": 5.0e8, "sources": fp, "capture": "profiles/x.md"})
    assert bench.measured_traffic("dequant_mse") == (5.0e8, "profiles/x.md")
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, "dequant_mse",
                        {"bytes": 5.0e8, "sources": "0" * 16, "capture": "profiles/x.md"})
    got, why = bench.measured_traffic("dequant_mse")
    assert got is None and "stale" in why


def test_oracle_sub_baselines_small_samples():
    r, dt = bench.oracle_stream_rate(512)
    assert r > 0 and dt > 0
    qv, pr, dt = bench.oracle_search_rate(300, 4, 64)
    assert qv > 0 and pr > 0 and dt > 0
