"""Drive a synthetic decode workload through the C ABI on one GPU.

Holds the device and pinned-host buffers of one workload, attaches them to a
library context and runs decode steps: [append] -> score -> select -> fetch ->
decode, optionally captured once in a CUDA graph and replayed.  Used by the
GPU tests and the benchmark; it only moves data and calls the binding.
"""

from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import nosa
from .configs import Workload
from .inputs import queries_bhd


def _bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16)


class Decoder:
    """One library context over one workload's inputs.

    data: dict from ``inputs.generate(w)`` (all units): 'k', 'v' [U, T, d]
    uint16, 'a' [U, max_blocks] float32, 'q' [U, steps, G, d] uint16.
    """

    def __init__(self, w: Workload, data: Dict[str, np.ndarray], device: int = 0,
                 side_copy_stream: bool = True, pin: bool = True, fused: bool = True):
        self.w = w
        self.fused = fused  # nosa_score_select_fetch instead of the three calls
        self.dev = torch.device("cuda", device)
        torch.cuda.set_device(self.dev)
        U, d = w.units, w.head_dim
        T = w.max_tokens
        k_host = _bf16(data["k"]).reshape(U, T, d)
        v_host = _bf16(data["v"]).reshape(U, T, d)
        n_prompt = w.context
        if w.offloaded:
            # full KV in pinned host memory; tokens beyond the prompt are not
            # there yet (they arrive by appends and are written through)
            self.k_store = torch.zeros((U, T, d), dtype=torch.bfloat16, pin_memory=pin)
            self.v_store = torch.zeros((U, T, d), dtype=torch.bfloat16, pin_memory=pin)
        else:
            self.k_store = torch.zeros((U, T, d), dtype=torch.bfloat16, device=self.dev)
            self.v_store = torch.zeros((U, T, d), dtype=torch.bfloat16, device=self.dev)
        self.k_store[:, :n_prompt].copy_(k_host[:, :n_prompt])
        self.v_store[:, :n_prompt].copy_(v_host[:, :n_prompt])
        self.agnostic = torch.from_numpy(data["a"]).to(self.dev)
        self.q_all = _bf16(queries_bhd(w, data["q"])).to(self.dev)  # [steps, B, Hq, d]
        if w.append:
            # token appended at step t is row context + t of each unit
            rows = slice(n_prompt, n_prompt + w.steps)
            kn = k_host[:, rows].reshape(w.batch, w.n_kv_heads, w.steps, d).permute(2, 0, 1, 3)
            vn = v_host[:, rows].reshape(w.batch, w.n_kv_heads, w.steps, d).permute(2, 0, 1, 3)
            self.k_new = kn.contiguous().to(self.dev)
            self.v_new = vn.contiguous().to(self.dev)
            # agnostic score of the block that the append at step t closes
            a_new = np.zeros((w.steps, U), dtype=np.float32)
            for t in range(w.steps):
                tok = n_prompt + t
                if (tok + 1) % w.block == 0:
                    a_new[t] = data["a"][:, tok // w.block]
            self.a_new = torch.from_numpy(a_new).to(self.dev)
            # static per-step inputs of the append call (graph replays read these)
            self.k_in = torch.empty_like(self.k_new[0])
            self.v_in = torch.empty_like(self.v_new[0])
            self.a_in = torch.empty_like(self.a_new[0])
        self.q = torch.empty((w.batch, w.n_q_heads, d), dtype=torch.bfloat16, device=self.dev)
        self.scores = torch.zeros((U, w.max_blocks), dtype=torch.float64, device=self.dev)
        self.sel = torch.zeros((U, w.k), dtype=torch.int32, device=self.dev)
        self.fetch = torch.zeros((U, w.k), dtype=torch.int32, device=self.dev)
        self.n_fetch = torch.zeros((U,), dtype=torch.int32, device=self.dev)
        self.out = torch.zeros((w.batch, w.n_q_heads, d), dtype=torch.bfloat16, device=self.dev)
        self.stream = torch.cuda.Stream(self.dev)
        # a second stream: the attention to the cached blocks runs on it beside
        # the miss gather (which the library launches with the highest CTA
        # priority on the main stream)
        self.copy_stream = (torch.cuda.Stream(self.dev) if (side_copy_stream and w.offloaded) else self.stream)
        self.ctx = nosa.nosa_create(nosa.config_from_workload(w))
        self.graph: Optional[torch.cuda.CUDAGraph] = None
        self.t = 0
        torch.cuda.synchronize(self.dev)  # uploads above ran on the default stream
        self.attach()

    # ------------------------------------------------------------ lifecycle
    def attach(self) -> None:
        with torch.cuda.stream(self.stream):
            nosa.nosa_attach_kv(self.ctx, self.k_store, self.v_store, self.w.context, self.agnostic,
                                self.stream)
        self.stream.synchronize()
        self.t = 0

    def close(self) -> None:
        self.graph = None
        if self.ctx:
            nosa.nosa_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------ one step
    def q_index(self, t: int) -> int:
        """Row of q_all used at step t.  Past the workload's last step the
        query sequence is walked back and forth (0..N-1, N-2..0, 1..), so
        consecutive steps always get neighbouring states of the AR(1)
        sequence instead of jumping from the last query to the first."""
        n = self.q_all.shape[0]
        if t < n or n < 2:
            return t % n
        p = t % (2 * n - 2)
        return p if p < n else 2 * n - 2 - p

    def _load_inputs(self, t: int) -> None:
        """Copy step t's inputs into the static buffers (on self.stream).
        Queries are reused past the workload's last step (see q_index);
        appended tokens are not."""
        self.q.copy_(self.q_all[self.q_index(t)], non_blocking=True)
        if self.w.append:
            self.k_in.copy_(self.k_new[t], non_blocking=True)
            self.v_in.copy_(self.v_new[t], non_blocking=True)
            self.a_in.copy_(self.a_new[t], non_blocking=True)

    def _calls(self, append: bool) -> None:
        s, cs = self.stream, self.copy_stream
        if append:
            nosa.nosa_append_token(self.ctx, self.k_in, self.v_in, self.a_in, s)
        if self.fused:
            nosa.nosa_score_select_fetch(self.ctx, self.q, self.scores, self.sel, self.fetch, self.n_fetch, s, cs)
        else:
            nosa.nosa_score_blocks(self.ctx, self.q, self.scores, s)
            nosa.nosa_select(self.ctx, self.scores, self.sel, s)
            nosa.nosa_fetch_missing(self.ctx, self.sel, self.fetch, self.n_fetch, s, cs)
        nosa.nosa_sparse_decode(self.ctx, self.q, self.sel, self.out, s)

    def step_through(self, q, out) -> None:
        """Eager step t through nosa_decode_step: q and out may be device or
        pinned host tensors [B, H_q, d] bf16 (the library reads and writes
        them itself).  For growing sequences the appended token's K/V (and
        agnostic score) are copied into the static append buffers first."""
        t = self.t
        s = self.stream
        with torch.cuda.stream(s):
            if self.w.append:
                self.k_in.copy_(self.k_new[t], non_blocking=True)
                self.v_in.copy_(self.v_new[t], non_blocking=True)
                self.a_in.copy_(self.a_new[t], non_blocking=True)
                nosa.nosa_append_token(self.ctx, self.k_in, self.v_in, self.a_in, s)
            nosa.nosa_decode_step(self.ctx, q, out, self.scores, self.sel, self.fetch, self.n_fetch, s,
                                  self.copy_stream)
        self.t += 1

    def step(self) -> None:
        """Eager step t (queries of step t copied into the static q buffer)."""
        t = self.t
        with torch.cuda.stream(self.stream):
            self._load_inputs(t)
            self._calls(self.w.append)
        self.t += 1

    def capture(self) -> None:
        """Capture one step (without the input copies) in a CUDA graph.  The
        capture itself runs nothing; replays advance the device-side state
        (step counter, closed blocks, tail length)."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            self._calls(self.w.append)
        self.graph = g

    def replay(self) -> None:
        t = self.t
        with torch.cuda.stream(self.stream):
            self._load_inputs(t)
            self.graph.replay()
        self.t += 1

    # ------------------------------------------------------------ readbacks
    def stats(self) -> dict:
        return nosa.nosa_get_stats(self.ctx)

    def cache_map(self) -> np.ndarray:
        out = np.zeros((self.w.units, self.w.cache_slots), dtype=np.int32)
        nosa.nosa_read_cache_map(self.ctx, out)
        return out

    def cache_contents(self, unit_begin: int = 0, n_units: Optional[int] = None):
        """K and V of every cache slot of the given units: uint16 (bf16 bits)
        [n_units, cache_slots, block, head_dim] each."""
        w = self.w
        n_units = w.units - unit_begin if n_units is None else n_units
        shape = (n_units, w.cache_slots, w.block, w.head_dim)
        k = np.zeros(shape, dtype=np.uint16)
        v = np.zeros(shape, dtype=np.uint16)
        nosa.nosa_read_cache(self.ctx, unit_begin, n_units, k, v)
        return k, v

    def check(self) -> None:
        nosa.nosa_check_errors(self.ctx)
