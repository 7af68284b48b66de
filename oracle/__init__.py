"""CPU oracle of the NOSA decode step -- TEST INFRASTRUCTURE, NOT PRODUCT CODE.

A plain, slow fp64 restatement of the step in C (``nosa_oracle.c``) plus this
ctypes wrapper.  Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``
(its CPU baseline and its reference arm) may import it; the library under
``kv_cache_decode_step_b200`` never does, and the oracle never imports the
library.  Inputs come from the seeded generators as numpy arrays.

Every function is pinned by CPU tests (closed forms, brute force on tiny
inputs, invariants); the pages print no worked example, so no fixture holds a
value printed there beyond the budget arithmetic of the paper's own setting.
"""

from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nosa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, -O2, OpenMP over units)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class OrcCfg(C.Structure):
    _fields_ = [("G", C.c_int), ("d", C.c_int), ("P", C.c_int), ("Q", C.c_int),
                ("n0", C.c_int), ("tail0", C.c_int), ("max_blocks", C.c_int),
                ("k_q", C.c_int), ("k_e", C.c_int), ("m", C.c_int), ("C", C.c_int),
                ("steps", C.c_int), ("append", C.c_int), ("sink", C.c_int), ("window", C.c_int)]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = C.CDLL(_LIB_PATH)
            vp = C.c_void_p
            L.orc_bf16_to_f64.argtypes = [C.c_uint16]
            L.orc_bf16_to_f64.restype = C.c_double
            L.orc_f64_to_bf16.argtypes = [C.c_double]
            L.orc_f64_to_bf16.restype = C.c_uint16
            L.orc_pool_keys.argtypes = [vp, C.c_int, C.c_int, C.c_int, vp]
            L.orc_pool_keys.restype = None
            L.orc_score_blocks.argtypes = [vp, C.c_int, C.c_int, vp, C.c_int, C.c_int, vp]
            L.orc_score_blocks.restype = None
            L.orc_evict_update.argtypes = [vp, vp, C.c_int, C.c_int, C.c_int, C.c_int, vp]
            L.orc_evict_update.restype = C.c_int
            L.orc_select.argtypes = [vp, C.c_int, vp, C.c_int, vp, C.c_int, C.c_int,
                                     C.c_int, C.c_int, vp]
            L.orc_select.restype = C.c_int
            L.orc_select_forced.argtypes = [vp, C.c_int, vp, vp, C.c_int, vp, C.c_int, C.c_int,
                                            C.c_int, C.c_int, vp]
            L.orc_select_forced.restype = C.c_int
            L.orc_forced.argtypes = [C.c_int, C.c_int, C.c_int, vp]
            L.orc_forced.restype = C.c_int
            L.orc_cache_plan.argtypes = [vp, C.c_int, C.c_int, C.c_int, vp, vp, vp, vp]
            L.orc_cache_plan.restype = C.c_int
            L.orc_attend.argtypes = [vp, C.c_int, C.c_int, vp, vp, vp, C.c_int, vp]
            L.orc_attend.restype = None
            L.orc_run_unit.argtypes = [C.POINTER(OrcCfg)] + [vp] * 13
            L.orc_run_unit.restype = C.c_int
            L.orc_run_units.argtypes = [C.POINTER(OrcCfg), C.c_int] + [vp] * 8
            L.orc_run_units.restype = C.c_int
            _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- primitives

def bf16_to_f64(bits: int) -> float:
    return lib().orc_bf16_to_f64(int(bits))


def f64_to_bf16(x: float) -> int:
    return int(lib().orc_f64_to_bf16(float(x)))


def pool_keys(K: np.ndarray, Q: int) -> np.ndarray:
    """K bf16 bits [n_sub*Q, d] -> pooled keys bf16 bits [n_sub, d]."""
    K = _c(K, np.uint16)
    n_sub = K.shape[0] // Q
    out = np.zeros((n_sub, K.shape[1]), dtype=np.uint16)
    lib().orc_pool_keys(_p(K), n_sub, Q, K.shape[1], _p(out))
    return out


def score_blocks(q: np.ndarray, kbar: np.ndarray, R: int) -> np.ndarray:
    """q bf16 bits [G, d], kbar bf16 bits [n*R, d] -> fp64 block scores [n]."""
    q = _c(q, np.uint16)
    kbar = _c(kbar, np.uint16)
    n = kbar.shape[0] // R
    out = np.zeros(n, dtype=np.float64)
    lib().orc_score_blocks(_p(q), q.shape[0], q.shape[1], _p(kbar), n, R, _p(out))
    return out


def evict_update(a: np.ndarray, ge_prev: Sequence[int], n_from: int, n_to: int,
                 k_e: int) -> np.ndarray:
    a = _c(a, np.float32)
    gp = _c(list(ge_prev) or [0], np.int32)
    out = np.zeros(max(k_e, 1), dtype=np.int32)
    n = lib().orc_evict_update(_p(a), _p(gp), len(ge_prev), n_from, n_to, k_e, _p(out))
    return out[:n].copy()


def select(score: np.ndarray, ge: Sequence[int], prev: Sequence[int], first: bool,
           k_q: int, c_max: int) -> np.ndarray:
    score = _c(score, np.float64)
    g = _c(list(ge) or [0], np.int32)
    p = _c(list(prev) or [0], np.int32)
    out = np.zeros(len(ge) + k_q + 1, dtype=np.int32)
    n = lib().orc_select(_p(score), score.shape[0], _p(g), len(ge), _p(p), len(prev),
                         int(bool(first)), k_q, c_max, _p(out))
    return out[:n].copy()


def select_forced(score: np.ndarray, forced: Sequence[int], ge: Sequence[int], prev: Sequence[int],
                  first: bool, k_q: int, c_max: int) -> np.ndarray:
    """Selection with forced blocks (ids in `forced`)."""
    score = _c(score, np.float64)
    n = score.shape[0]
    fl = np.zeros(n + 1, dtype=np.uint8)
    for j in forced:
        fl[int(j)] = 1
    g = _c(list(ge) or [0], np.int32)
    p = _c(list(prev) or [0], np.int32)
    out = np.zeros(n + 1, dtype=np.int32)
    m = lib().orc_select_forced(_p(score), n, _p(fl), _p(g), len(ge), _p(p), len(prev),
                                int(bool(first)), k_q, c_max, _p(out))
    return out[:m].copy()


def forced_blocks(n: int, sink: int, window: int) -> np.ndarray:
    fl = np.zeros(max(n, 1), dtype=np.uint8)
    lib().orc_forced(n, sink, window, _p(fl))
    return np.nonzero(fl[:n])[0]


class Cache:
    """Per-unit cache bookkeeping state for :func:`cache_plan`."""

    def __init__(self, C_slots: int):
        self.slot_block = np.full(C_slots, -1, dtype=np.int32)
        self.last_used = np.full(C_slots, -1, dtype=np.int32)

    def plan(self, sel: Sequence[int], step: int):
        s = _c(list(sel) or [0], np.int32)
        fetch = np.zeros(max(len(sel), 1), dtype=np.int32)
        slots = np.zeros(max(len(sel), 1), dtype=np.int32)
        nf = lib().orc_cache_plan(_p(s), len(sel), step, self.slot_block.shape[0],
                                  _p(self.slot_block), _p(self.last_used), _p(fetch), _p(slots))
        if nf < 0:
            raise ValueError("cache smaller than the selection")
        return fetch[:nf].copy(), slots[:nf].copy()

    def resident(self) -> np.ndarray:
        r = self.slot_block[self.slot_block >= 0]
        return np.sort(r)


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, rows: Sequence[int]) -> np.ndarray:
    """fp64 attention of q bf16 [G, d] over the given token rows of K, V bf16 [T, d]."""
    q = _c(q, np.uint16)
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    r = _c(list(rows) or [0], np.int32)
    out = np.zeros(q.shape, dtype=np.float64)
    lib().orc_attend(_p(q), q.shape[0], q.shape[1], _p(K), _p(V), _p(r), len(rows), _p(out))
    return out


# --------------------------------------------------------------- trajectories

@dataclass
class UnitRun:
    sel: np.ndarray        # [steps, k] int32, -1 pad
    nsel: np.ndarray       # [steps]
    fetch: np.ndarray      # [steps, k] int32, -1 pad
    nfetch: np.ndarray     # [steps]
    resident: Optional[np.ndarray]  # [steps, C] sorted ids, -1 pad (offloaded)
    o: Optional[np.ndarray]         # [steps, G, d] fp64 (NaN where not requested)
    overlap: np.ndarray    # [steps]
    scores: Optional[np.ndarray]    # [steps, max_blocks]


def gather_rows(src: np.ndarray, src_idx: Sequence[int], dst: np.ndarray,
                dst_idx: Optional[Sequence[int]] = None) -> np.ndarray:
    """Transfer of missed rows (NOSA summary §4: each miss is copied from host
    memory into its GPU slot; §3.2: at block or at single-token granularity).
    For each i in order, row dst_idx[i] (row i when dst_idx is None) of a copy
    of dst takes row src_idx[i] of src; an index outside either array leaves
    that row alone.  src and dst are 2-D arrays of one row width.  Returns the
    updated copy."""
    out = np.array(dst, copy=True)
    for i, s in enumerate(src_idx):
        t = i if dst_idx is None else dst_idx[i]
        if 0 <= s < src.shape[0] and 0 <= t < out.shape[0]:
            out[t, :] = src[s, :]
    return out


def make_cfg(G, d, P, Q, n0, tail0, max_blocks, k_q, k_e, m, C_slots, steps, append, sink=0,
             window=0) -> OrcCfg:
    return OrcCfg(G, d, P, Q, n0, tail0, max_blocks, k_q, k_e, m, C_slots, steps, int(append), sink, window)


def cfg_from_workload(w, steps: Optional[int] = None) -> OrcCfg:
    return make_cfg(w.group, w.head_dim, w.block, w.sub_block, w.n_blocks0, w.tail0,
                    w.max_blocks, w.k_query, w.k_agnostic, w.min_overlap, w.cache_slots,
                    w.steps if steps is None else steps, w.append, w.sink_blocks, w.window_blocks)


def run_unit(cfg: OrcCfg, K: np.ndarray, V: np.ndarray, a: np.ndarray, q: np.ndarray,
             attend_steps=None, want_scores: bool = False) -> UnitRun:
    """Run one unit's whole trajectory.  attend_steps: iterable of step ids whose
    attention output is wanted (None = every step)."""
    steps, k = cfg.steps, cfg.k_q + cfg.k_e
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    a = _c(a, np.float32)
    q = _c(q[:steps], np.uint16)
    mask = np.zeros(steps, dtype=np.uint8)
    if attend_steps is None:
        mask[:] = 1
    else:
        for t in attend_steps:
            mask[int(t)] = 1
    sel = np.zeros((steps, k), dtype=np.int32)
    nsel = np.zeros(steps, dtype=np.int32)
    fetch = np.zeros((steps, k), dtype=np.int32)
    nfetch = np.zeros(steps, dtype=np.int32)
    resident = np.zeros((steps, cfg.C), dtype=np.int32) if cfg.C > 0 else None
    o = np.full((steps, cfg.G, cfg.d), np.nan, dtype=np.float64)
    ov = np.zeros(steps, dtype=np.int32)
    sc = np.zeros((steps, cfg.max_blocks), dtype=np.float64) if want_scores else None
    rc = lib().orc_run_unit(C.byref(cfg), _p(K), _p(V), _p(a), _p(q), _p(mask), _p(sel),
                            _p(nsel), _p(fetch), _p(nfetch), _p(resident), _p(o), _p(ov), _p(sc))
    if rc != 0:
        raise ValueError(f"orc_run_unit failed: {rc}")
    return UnitRun(sel, nsel, fetch, nfetch, resident, o, ov, sc)


def run_units(cfg: OrcCfg, K: np.ndarray, V: np.ndarray, a: np.ndarray, q: np.ndarray,
              attend_steps=None, want_o: bool = True):
    """All given units (leading axis) in parallel; returns (sel, nfetch, o, threads)."""
    n_units, steps, k = K.shape[0], cfg.steps, cfg.k_q + cfg.k_e
    K = _c(K, np.uint16)
    V = _c(V, np.uint16)
    a = _c(a, np.float32)
    q = _c(q[:, :steps], np.uint16)
    mask = np.zeros(steps, dtype=np.uint8)
    if attend_steps is None:
        mask[:] = 1
    else:
        for t in attend_steps:
            mask[int(t)] = 1
    sel = np.zeros((n_units, steps, k), dtype=np.int32)
    nfetch = np.zeros((n_units, steps), dtype=np.int32)
    o = np.full((n_units, steps, cfg.G, cfg.d), np.nan) if want_o else None
    th = lib().orc_run_units(C.byref(cfg), n_units, _p(K), _p(V), _p(a), _p(q), _p(mask),
                             _p(sel), _p(nfetch), _p(o))
    if th < 0:
        raise ValueError("orc_run_units failed")
    return sel, nfetch, o, th
