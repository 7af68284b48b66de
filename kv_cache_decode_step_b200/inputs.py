"""Seeded synthetic inputs for the NOSA decode workloads.

This module only draws random numbers and rounds them to bf16; it holds none
of the decode step's arithmetic.  Both the CUDA path (through the binding) and
the CPU oracle (in the tests and the CPU baseline) consume what it returns.

Every random quantity comes from its own numpy stream, keyed by
``SeedSequence(seed, spawn_key=(stream, unit))`` so that any subset of units can
be regenerated on its own and yields bit-identical data:

* K and V: N(0,1) drawn in fp32, rounded to bf16 with round-to-nearest-even.
  Planted blocks (the resident 8B-shaped layer) take bf16(fp32(scale * x)) of
  the same fp32 draws.  For the long-generation workload the tokens appended
  during decoding are simply the later rows of the same per-unit stream.
* Query-agnostic block scores: U(0,1) fp32, one per (unit, block), including
  the blocks that close during decoding.
* Queries: q_0 ~ N(0,1); q_t = rho * q_{t-1} + sigma * eps_t with eps_t ~ N(0,1),
  kept in fp64; a fresh N(0,1) draw replaces q_t when resampling is enabled and
  t % resample_every == 0 (t > 0).  Each q_t is rounded fp64 -> fp32 -> bf16.

Arrays of bf16 are returned as ``numpy.uint16`` bit patterns.
"""

from __future__ import annotations

import concurrent.futures as cf
import os
from typing import Dict, Iterable, Optional, Sequence

import numpy as np
import torch
from scipy.signal import lfilter

from .configs import Workload

STREAM_K, STREAM_V, STREAM_AGNOSTIC, STREAM_PLANTED, STREAM_QUERY = 0, 1, 2, 3, 4


def _rng(w: Workload, stream: int, unit: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence(w.seed, spawn_key=(stream, unit)))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even) and return the bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def unit_planted(w: Workload, u: int) -> np.ndarray:
    """Sorted block indices whose keys are scaled (empty unless planted)."""
    if w.planted_blocks <= 0:
        return np.zeros(0, dtype=np.int64)
    r = _rng(w, STREAM_PLANTED, u)
    return np.sort(r.choice(w.n_blocks0, size=w.planted_blocks, replace=False))


def unit_kv(w: Workload, u: int, which: str) -> np.ndarray:
    """bf16 bits [max_tokens, head_dim] of unit u's keys ('k') or values ('v')."""
    stream = STREAM_K if which == "k" else STREAM_V
    x = _rng(w, stream, u).standard_normal((w.max_tokens, w.head_dim), dtype=np.float32)
    if which == "k" and w.planted_blocks > 0:
        for j in unit_planted(w, u):
            rows = slice(int(j) * w.block, (int(j) + 1) * w.block)
            x[rows] = (np.float32(w.planted_scale) * x[rows]).astype(np.float32)
    return f32_to_bf16_bits(x)


def unit_agnostic(w: Workload, u: int) -> np.ndarray:
    """fp32 [max_blocks] query-agnostic scores of unit u."""
    return _rng(w, STREAM_AGNOSTIC, u).random(w.max_blocks, dtype=np.float32)


def _query_draws(w: Workload, u: int):
    """q_0 and the innovations eps_1 .. eps_{steps-1} of unit u (fp64), in the
    order the stream yields them."""
    r = _rng(w, STREAM_QUERY, u)
    shape = (w.group, w.head_dim)
    q0 = r.standard_normal(shape)
    eps = r.standard_normal((max(w.steps - 1, 0),) + shape)
    return q0, eps


def _queries_from_draws(w: Workload, q0: np.ndarray, eps: np.ndarray) -> np.ndarray:
    """AR(1) recurrence over a leading batch of units: q0 [n, G, d], eps
    [n, steps-1, G, d] -> fp64 [n, steps, G, d].

    q_t = rho*q_{t-1} + sigma*eps_t, restarted at q_t = eps_t on resample steps.
    Each segment between restarts is one linear filter along time (the same two
    fp64 products and one sum per step as the plain loop)."""
    n = q0.shape[0]
    S = w.steps
    out = np.empty((n, S) + q0.shape[1:], dtype=np.float64)
    if S == 0:
        return out
    out[:, 0] = q0
    starts = [1] + ([t for t in range(1, S) if w.resample_every and t % w.resample_every == 0])
    starts = sorted(set(starts))
    bounds = starts + [S]
    prev = q0
    for a, b in zip(bounds[:-1], bounds[1:]):
        if a >= b:
            continue
        x = eps[:, a - 1:b - 1]
        if w.resample_every and a % w.resample_every == 0:
            out[:, a] = x[:, 0]
            if b > a + 1:
                zi = (w.rho * x[:, 0])[:, None]
                out[:, a + 1:b] = lfilter([w.sigma], [1.0, -w.rho], x[:, 1:], axis=1, zi=zi)[0]
        else:
            zi = (w.rho * prev)[:, None]
            out[:, a:b] = lfilter([w.sigma], [1.0, -w.rho], x, axis=1, zi=zi)[0]
        prev = out[:, b - 1]
    return out


def _queries_loop(w: Workload, q0: np.ndarray, eps: np.ndarray) -> np.ndarray:
    """The same recurrence as a plain per-step loop (kept for cross-checks)."""
    out = np.empty((q0.shape[0], w.steps) + q0.shape[1:], dtype=np.float64)
    q = q0
    if w.steps > 0:
        out[:, 0] = q
    for t in range(1, w.steps):
        e = eps[:, t - 1]
        q = e if (w.resample_every and t % w.resample_every == 0) else w.rho * q + w.sigma * e
        out[:, t] = q
    return out


def unit_queries(w: Workload, u: int) -> np.ndarray:
    """bf16 bits [steps, group, head_dim]: the query heads of unit u, per step."""
    q0, eps = _query_draws(w, u)
    q = _queries_from_draws(w, q0[None], eps[None])[0]
    return f32_to_bf16_bits(q.astype(np.float32))


_QCHUNK = 16


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def generate(w: Workload, units: Optional[Sequence[int]] = None,
             parts: Iterable[str] = ("k", "v", "a", "q")) -> Dict[str, np.ndarray]:
    """Draw the inputs for the given units (default: all), stacked in unit order.

    Returns a dict with any of: 'k', 'v' [n_units, max_tokens, d] uint16;
    'a' [n_units, max_blocks] float32; 'q' [n_units, steps, group, d] uint16.
    """
    units = list(range(w.units)) if units is None else [int(u) for u in units]
    parts = tuple(parts)
    out: Dict[str, np.ndarray] = {}
    nu = len(units)
    if "k" in parts:
        out["k"] = np.empty((nu, w.max_tokens, w.head_dim), dtype=np.uint16)
    if "v" in parts:
        out["v"] = np.empty((nu, w.max_tokens, w.head_dim), dtype=np.uint16)
    if "a" in parts:
        out["a"] = np.empty((nu, w.max_blocks), dtype=np.float32)
    if "q" in parts:
        out["q"] = np.empty((nu, w.steps, w.group, w.head_dim), dtype=np.uint16)

    def one(i: int) -> None:
        u = units[i]
        if "k" in parts:
            out["k"][i] = unit_kv(w, u, "k")
        if "v" in parts:
            out["v"][i] = unit_kv(w, u, "v")
        if "a" in parts:
            out["a"][i] = unit_agnostic(w, u)

    def queries(i0: int) -> None:
        # the recurrence runs vectorised over a chunk of units
        chunk = list(range(i0, min(nu, i0 + _QCHUNK)))
        draws = [_query_draws(w, units[i]) for i in chunk]
        q = _queries_from_draws(w, np.stack([d[0] for d in draws]), np.stack([d[1] for d in draws]))
        out["q"][chunk[0]:chunk[-1] + 1] = f32_to_bf16_bits(q.astype(np.float32))

    jobs = [(one, i) for i in range(nu)]
    if "q" in parts:
        jobs += [(queries, i0) for i0 in range(0, nu, _QCHUNK)]
    if len(jobs) <= 2:
        for f, i in jobs:
            f(i)
    else:
        with cf.ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(lambda j: j[0](j[1]), jobs))
    return out


def queries_bhd(w: Workload, q_units: np.ndarray) -> np.ndarray:
    """Re-lay unit-major queries [U, steps, G, d] as [steps, B, H_q, d]."""
    U, S, G, d = q_units.shape
    assert U == w.units
    x = q_units.reshape(w.batch, w.n_kv_heads, S, G, d)
    return np.ascontiguousarray(x.transpose(2, 0, 1, 3, 4).reshape(S, w.batch, w.n_q_heads, d))
