"""Shared helpers of the GPU tests: run a workload through the C ABI, run the
oracle on a sample of units, compare."""

from __future__ import annotations

import concurrent.futures as cf
from dataclasses import dataclass, field
from typing import Dict, List, Sequence

import numpy as np
import torch

import oracle
from kv_cache_decode_step_b200 import inputs, runner

TOL_MAX = 2e-2   # max-abs error of bf16 outputs vs the fp64 oracle
TOL_MEAN = 2e-3  # mean-abs error


@dataclass
class GpuRecord:
    sel: np.ndarray                     # [steps, n_sample, k]
    fetch: np.ndarray                   # [steps, n_sample, k]
    nfetch: np.ndarray                  # [steps, n_sample]
    out: Dict[int, np.ndarray] = field(default_factory=dict)       # t -> [n_sample, G, d]
    resident: Dict[int, List[np.ndarray]] = field(default_factory=dict)
    sel_all_last: np.ndarray = None     # [U, k] at the last step
    stats: dict = None


def run_gpu(w, data, sample: Sequence[int], attend_steps, steps=None, graph=False,
            cache_steps=(), side_copy_stream=True, fused=True) -> GpuRecord:
    steps = w.steps if steps is None else steps
    sample = list(sample)
    dec = runner.Decoder(w, data, side_copy_stream=side_copy_stream, fused=fused)
    rec = GpuRecord(sel=np.zeros((steps, len(sample), w.k), np.int32),
                    fetch=np.zeros((steps, len(sample), w.k), np.int32),
                    nfetch=np.zeros((steps, len(sample)), np.int32))
    attend_steps = set(int(t) for t in attend_steps)
    idx = torch.tensor(sample, device=dec.dev)
    try:
        for t in range(steps):
            if graph and t >= 1:
                if dec.graph is None:
                    dec.capture()
                dec.replay()
            else:
                dec.step()
            dec.stream.synchronize()
            rec.sel[t] = dec.sel[idx].cpu().numpy()
            rec.fetch[t] = dec.fetch[idx].cpu().numpy()
            rec.nfetch[t] = dec.n_fetch[idx].cpu().numpy()
            if t in attend_steps:
                o = dec.out.float().cpu().numpy().reshape(w.batch, w.n_kv_heads, w.group, w.head_dim)
                rec.out[t] = np.stack([o[u // w.n_kv_heads, u % w.n_kv_heads] for u in sample])
            if t in cache_steps and w.offloaded:
                cm = dec.cache_map()
                rec.resident[t] = [np.sort(cm[u][cm[u] >= 0]) for u in sample]
                check_cache_bytes(w, data, dec, cm, sample, t)
        rec.sel_all_last = dec.sel.cpu().numpy()
        rec.stats = dec.stats()
        dec.check()
    finally:
        dec.close()
    return rec


def check_cache_bytes(w, data, dec, cache_map, sample, t, chunk=64):
    """Every occupied cache slot of the sampled units holds, byte for byte, the
    K and V rows of the block the cache map names (the input arrays: prompt
    rows, and for growing sequences the appended rows, which are the later rows
    of the same per-unit streams)."""
    P = w.block
    sample = sorted(sample)
    i = 0
    while i < len(sample):
        # contiguous runs of units, read in chunks
        j = i
        while j + 1 < len(sample) and sample[j + 1] == sample[j] + 1 and j + 1 - i < chunk:
            j += 1
        u0, n = sample[i], j - i + 1
        ck, cv = dec.cache_contents(u0, n)
        for du in range(n):
            u = u0 + du
            for slot, b in enumerate(cache_map[u]):
                if b < 0:
                    continue
                for name, got, src in (("K", ck[du, slot], data["k"][u]), ("V", cv[du, slot], data["v"][u])):
                    if not np.array_equal(got, src[b * P:(b + 1) * P]):
                        bad = np.argwhere(got != src[b * P:(b + 1) * P])
                        raise AssertionError(f"step {t} unit {u} slot {slot} block {b}: cached {name} differs "
                                             f"from the host block at {len(bad)} of {got.size} elements, first "
                                             f"(token, dim) {tuple(bad[0])}")
        i = j + 1


def run_oracle(w, data, sample, attend_steps, steps=None) -> List[oracle.UnitRun]:
    steps = w.steps if steps is None else steps
    cfg = oracle.cfg_from_workload(w, steps=steps)
    att = sorted(int(t) for t in attend_steps if t < steps)

    def one(u):
        return oracle.run_unit(cfg, data["k"][u], data["v"][u], data["a"][u], data["q"][u][:steps],
                               attend_steps=att)

    with cf.ThreadPoolExecutor(max(1, min(len(sample), 16))) as ex:
        return list(ex.map(one, list(sample)))


def compare(w, rec: GpuRecord, refs, sample, steps=None):
    steps = w.steps if steps is None else steps
    worst_max, worst_mean = 0.0, 0.0
    for i, u in enumerate(sample):
        r = refs[i]
        for t in range(steps):
            if not np.array_equal(rec.sel[t, i], r.sel[t]):
                raise AssertionError(f"unit {u} step {t}: selection\n gpu    {rec.sel[t, i].tolist()}\n"
                                     f" oracle {r.sel[t].tolist()}")
            if w.offloaded:
                if rec.nfetch[t, i] != r.nfetch[t] or not np.array_equal(rec.fetch[t, i], r.fetch[t]):
                    raise AssertionError(f"unit {u} step {t}: fetch gpu {rec.fetch[t, i].tolist()} "
                                         f"oracle {r.fetch[t].tolist()}")
        for t, o in rec.out.items():
            err = np.abs(o[i].astype(np.float64) - r.o[t])
            worst_max = max(worst_max, float(err.max()))
            worst_mean = max(worst_mean, float(err.mean()))
        for t, res in rec.resident.items():
            want = r.resident[t][r.resident[t] >= 0]
            if not np.array_equal(res[i], want):
                raise AssertionError(f"unit {u} step {t}: resident set differs")
    assert worst_max <= TOL_MAX, f"max-abs error {worst_max} > {TOL_MAX}"
    assert worst_mean <= TOL_MEAN, f"mean-abs error {worst_mean} > {TOL_MEAN}"
    return worst_max, worst_mean


def check_all_unit_invariants(w, rec: GpuRecord, steps):
    st = rec.stats
    k = w.k
    assert st["steps"] == steps
    assert st["selected"] == steps * w.units * k
    if steps > 1:
        assert st["min_overlap"] >= w.min_overlap
        if w.offloaded:
            assert st["max_fetch"] <= (k - w.min_overlap) + (1 if w.append else 0)
    if w.offloaded:
        assert st["hits"] + st["misses"] == steps * w.units * k
        assert st["fetched_bytes"] == st["misses"] * 2 * w.block * w.head_dim * 2
    s = rec.sel_all_last
    assert np.all(np.diff(s, axis=1) > 0)  # ascending, distinct
    assert s.min() >= 0
