"""Host-side logic of the benchmark and the decoder, without a GPU: the query
walk past a workload's last step, the config both bench arms print, and the
algorithmic bytes the roofline divides by."""

import importlib.util
import os

import pytest

from kv_cache_decode_step_b200 import configs
from kv_cache_decode_step_b200.runner import Decoder

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


class _Q:
    def __init__(self, n):
        import torch
        self.q_all = torch.zeros(n)


@pytest.mark.parametrize("n", [2, 5, 256])
def test_query_walk_is_continuous(n):
    d = _Q(n)
    idx = [Decoder.q_index(d, t) for t in range(5 * n)]
    assert idx[:n] == list(range(n))                       # the workload's own steps first
    assert all(0 <= i < n for i in idx)
    assert all(abs(a - b) == 1 for a, b in zip(idx, idx[1:]))  # always a neighbouring state


def test_both_arms_print_the_same_config(bench):
    w = configs.get("offload_b64")
    a = bench.workload_config(w, "nosa", 1)
    b = bench.workload_config(w.with_(steps=9999), "nosa", 1)  # the run's step count is not part of it
    assert a == b
    for key in ("workload", "batch", "context", "k", "k_query", "k_agnostic", "min_overlap", "cache_slots",
                "n_q_heads", "n_kv_heads", "l2"):
        assert key in a
    assert not {"graph", "cpu_affinity", "calls"} & set(a)


def test_algorithmic_hbm_bytes_of_the_metric_workload(bench):
    """U·n·R·d·2 pooled keys + U·n·(8·2 + 4) scores and agnostic scores +
    U·k·P·d·4 selected K/V + F·P·d·4 cache writes + B·H_q·d·4 queries and
    outputs, for offload_b64 (U = 512, n = 64, k = 16) and F = 500 misses."""
    w = configs.get("offload_b64")
    U, n, k, F = 512, 64, 16, 500
    want = U * n * 4 * 128 * 2 + U * n * 20 + U * k * 64 * 128 * 4 + F * 64 * 128 * 4 + 64 * 32 * 128 * 4
    assert bench.hbm_bytes_per_step(w, F) == want


def test_captured_traffic_is_consistent_with_the_work(bench):
    """The ncu counters the bench line carries: the gather's link bytes exceed
    its host-memory payload only by the completions' protocol overhead, and
    its payload is at most every selected block missing (32 KiB of K and V
    each); the hits
    pass reads no more DRAM bytes per launch than the K/V of every selected
    block of the resident 8B layer (the rest is in L2 when the launch starts)."""
    ga = bench.NCU_TRAFFIC[("gather_attend_kernel", "offload_b64")]
    wb = configs.get("offload_b64")
    assert 0 < ga["payload"] <= wb.units * wb.k * 32 * 1024
    assert 1.0 < ga["pcie_read"] / ga["payload"] < 1.15
    assert ga["dram"] < 0.05 * ga["payload"]  # the cache writes stay in L2 during the launch
    w = configs.get("layer8b")
    kv_bytes = w.units * w.k * w.block * w.head_dim * 2 * 2
    hits = bench.NCU_TRAFFIC[("attend_hits_ws_kernel", "layer8b")]
    assert 0.9 * kv_bytes < hits["dram"] <= kv_bytes
