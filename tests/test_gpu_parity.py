"""GPU parity: the CUDA path, called through the C ABI, against the CPU oracle
on the same seeded inputs.  Selections, fetch lists and resident sets must be
bit-exact, and so must the bytes of every occupied cache slot (against the
host block it names); bf16 attention outputs within max-abs 2e-2 and mean-abs
2e-3 of the oracle's fp64 result.  The five workloads run at full size; on the
offloaded batch-64 workload and the long-input workload every unit's
selections and fetch lists are compared at every step, elsewhere a sample of
units."""

import numpy as np
import pytest

from kv_cache_decode_step_b200 import configs, inputs
from gpu_harness import check_all_unit_invariants, compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


def _full(w, sample, attend, graph=False, cache_steps=()):
    data = inputs.generate(w)
    rec = run_gpu(w, data, sample, attend, graph=graph, cache_steps=cache_steps)
    refs = run_oracle(w, data, sample, attend)
    err = compare(w, rec, refs, sample)
    check_all_unit_invariants(w, rec, w.steps)
    print(f"{w.name}: max-abs {err[0]:.3e} mean-abs {err[1]:.3e} stats {rec.stats}")
    return rec


@pytest.mark.parametrize("offloaded", [True, False])
def test_tiny_all_units_all_steps(offloaded):
    w = configs.get("tiny")
    if not offloaded:
        w = w.with_(offloaded=False, cache_factor=0)
    _full(w, range(w.units), range(w.steps), cache_steps=range(w.steps))


def test_layer8b_resident():
    w = configs.get("layer8b")
    _full(w, [0, 37, 64, 127], list(range(0, w.steps, 16)) + [w.steps - 1])


def test_offload_b64_graph_replay():
    """Every unit: S(t), fetch lists and n_fetch at all 256 steps; resident
    sets and cache bytes at three steps; outputs at nine."""
    w = configs.get("offload_b64")
    _full(w, range(w.units), list(range(0, w.steps, 32)) + [w.steps - 1], graph=True,
          cache_steps=[1, 100, w.steps - 1])


def test_long_input_offloaded():
    """Every unit, every step; the query resamples (t % 32 == 0) push the
    capped selection to its limit."""
    w = configs.get("long_input")
    _full(w, range(w.units), list(range(0, w.steps, 16)) + [31, 32, 33, w.steps - 1],
          cache_steps=[0, 31, 32, 33, w.steps - 1])


def test_long_generation_appends_and_closes():
    w = configs.get("long_gen")
    attend = [0, 1, 62, 63, 64, 65, 127, 128, 1000, w.steps - 1]
    rec = _full(w, [0, 77, 255], attend, cache_steps=[64, 1000])
    assert rec.stats["n_closed"] == w.n_blocks0 + w.steps // w.block


# ------------------------------------------------------------------ edge cases

@pytest.mark.parametrize("offloaded", [True, False])
def test_ragged_prompt_tail(offloaded):
    """A prompt that ends inside a block: the partial block is attended, never
    scored or fetched."""
    w = configs.get("tiny", context=4096 + 37, steps=8)
    if not offloaded:
        w = w.with_(offloaded=False, cache_factor=0)
    _full(w, range(w.units), range(w.steps), cache_steps=[0, 7])


def test_ragged_tail_with_appends_closing_a_block():
    w = configs.get("tiny", context=4096 + 60, steps=12, append=True)
    rec = _full(w, range(w.units), range(w.steps), cache_steps=[3, 4, 11])
    assert rec.stats["n_closed"] == 65 and rec.stats["tail_len"] == 8


def test_plain_topk_mode_without_agnostic_part():
    """k_e = 0 and no overlap floor: selection is the plain top-k of scores."""
    w = configs.get("tiny", k_query=16, k_agnostic=0, min_overlap=0, steps=10)
    _full(w, range(w.units), range(w.steps))


@pytest.mark.parametrize("hq", [2, 4, 16])
def test_group_sizes(hq):
    """G = 1, 2 and 8 query heads per KV head."""
    w = configs.get("tiny", n_q_heads=hq, steps=6)
    _full(w, range(w.units), range(w.steps))


def test_single_split_budget_equals_all_blocks():
    """Budget covering every block: selection is everything, output is dense."""
    w = configs.get("tiny", context=16 * 64, k_query=12, k_agnostic=4, steps=5)
    rec = _full(w, range(w.units), range(w.steps))
    assert np.array_equal(rec.sel[0, 0], np.arange(16))


@pytest.mark.parametrize("offloaded", [True, False])
def test_maximum_block_count(offloaded):
    """max_blocks = 8192 (512K tokens per unit), the largest the ABI accepts,
    with the largest cache (1024 slots)."""
    w = configs.get("tiny", context=8192 * 64, steps=4, k_query=48, k_agnostic=16, min_overlap=52,
                    cache_factor=16)
    if not offloaded:
        w = w.with_(offloaded=False, cache_factor=0)
    assert w.max_blocks == 8192
    _full(w, range(w.units), [0, 3], cache_steps=[3])


def test_side_stream_and_single_stream_agree():
    w = configs.get("tiny", steps=6)
    data = inputs.generate(w)
    a = run_gpu(w, data, range(w.units), range(w.steps), side_copy_stream=True)
    b = run_gpu(w, data, range(w.units), range(w.steps), side_copy_stream=False)
    assert np.array_equal(a.sel, b.sel) and np.array_equal(a.fetch, b.fetch)
    for t in a.out:
        assert np.array_equal(a.out[t], b.out[t])


# ------------------------------------------------------------------ fused entry point

@pytest.mark.parametrize("name,kw", [
    ("tiny", {}),
    ("tiny", {"offloaded": False, "cache_factor": 0}),
    ("layer8b", {"batch": 4, "steps": 24}),
    ("offload_b64", {"steps": 24}),
    ("long_gen", {"batch": 2, "steps": 70}),
    ("long_input", {"batch": 1, "steps": 6}),   # beyond the fused kernel: three calls
])
@pytest.mark.parametrize("graph", [False, True])
def test_fused_and_separate_calls_agree_bit_exactly(name, kw, graph):
    """nosa_score_select_fetch gives the selections, fetch lists, outputs and
    statistics of score + select + fetch, bit for bit (same arithmetic)."""
    w = configs.get(name, **kw)
    data = inputs.generate(w)
    sample = list(range(min(w.units, 8)))
    attend = list(range(w.steps))
    a = run_gpu(w, data, sample, attend, graph=graph, cache_steps=[w.steps - 1], fused=True)
    b = run_gpu(w, data, sample, attend, graph=graph, cache_steps=[w.steps - 1], fused=False)
    assert np.array_equal(a.sel, b.sel) and np.array_equal(a.fetch, b.fetch)
    assert np.array_equal(a.nfetch, b.nfetch) and np.array_equal(a.sel_all_last, b.sel_all_last)
    for t in attend:
        assert np.array_equal(a.out[t], b.out[t]), t
    for t in a.resident:
        for x, y in zip(a.resident[t], b.resident[t]):
            assert np.array_equal(x, y)
    assert a.stats == b.stats


@pytest.mark.parametrize("offloaded", [True, False])
def test_two_stage_hits_pass(offloaded, monkeypatch):
    """The hits pass built with two TMA stages (three CTAs per SM), chosen
    by NOSA_ATTN_STAGES=2 when the context is created."""
    monkeypatch.setenv("NOSA_ATTN_STAGES", "2")
    w = configs.get("layer8b", batch=2, steps=12)
    if offloaded:
        w = w.with_(offloaded=True, cache_factor=2)
    _full(w, range(w.units), range(w.steps), cache_steps=[w.steps - 1] if offloaded else ())


@pytest.mark.parametrize("offloaded", [True, False])
def test_hits_pass_without_a_producer_warp(offloaded, monkeypatch):
    """The hits pass whose thread 0 issues the loads between blocks
    (NOSA_ATTN_PRODUCER=0) gives the same outputs as the default pass with a
    producer warp, bit for bit."""
    w = configs.get("layer8b", batch=2, steps=10)
    if offloaded:
        w = w.with_(offloaded=True, cache_factor=2)
    data = inputs.generate(w)
    sample = list(range(w.units))
    a = run_gpu(w, data, sample, range(w.steps))
    monkeypatch.setenv("NOSA_ATTN_PRODUCER", "0")
    b = run_gpu(w, data, sample, range(w.steps))
    assert np.array_equal(a.sel, b.sel) and np.array_equal(a.fetch, b.fetch)
    for t in a.out:
        assert np.array_equal(a.out[t], b.out[t]), t
    refs = run_oracle(w, data, sample, range(w.steps))
    compare(w, b, refs, sample)


@pytest.mark.parametrize("gap", [0, 17])
@pytest.mark.parametrize("offloaded", [True, False])
def test_hits_pass_walk_gap(gap, offloaded, monkeypatch):
    """The hits pass with no empty positions after each unit, and with more
    empty positions than a unit has blocks (NOSA_ATTN_GAP): ranges that hold
    only empty positions still count their segments."""
    monkeypatch.setenv("NOSA_ATTN_GAP", str(gap))
    w = configs.get("tiny", steps=8)
    if not offloaded:
        w = w.with_(offloaded=False, cache_factor=0)
    _full(w, range(w.units), range(w.steps), cache_steps=[w.steps - 1] if offloaded else ())


@pytest.mark.parametrize("graph", [False, True])
def test_cache_of_exactly_k_slots(graph):
    """C = k: a full cache holds exactly S(t-1), so every miss evicts a block
    the step does not use; queries resampled every 4 steps force many misses."""
    w = configs.get("tiny", cache_factor=1, steps=24, resample_every=4)
    data = inputs.generate(w)
    sample = list(range(w.units))
    attend = list(range(w.steps))
    rec = run_gpu(w, data, sample, attend, graph=graph, cache_steps=[3, 4, 12, w.steps - 1])
    refs = run_oracle(w, data, sample, attend)
    compare(w, rec, refs, sample)
    check_all_unit_invariants(w, rec, w.steps)
    assert rec.stats["misses"] > w.units * w.steps  # the resamples made it miss
