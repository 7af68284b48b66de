"""nosa_decode_step: the whole step in one call, with queries and outputs in
device memory or in pinned host memory (read and written by the library's own
kernels).  It must give the selections, fetch lists and outputs of the split
calls bit for bit, on the fused path (up to 512 blocks per unit), on the
three-kernel path (more blocks), with appends, and under graph capture."""

import numpy as np
import pytest
import torch

from kv_cache_decode_step_b200 import configs, inputs, runner
from gpu_harness import compare, run_oracle

pytestmark = pytest.mark.gpu


def _trajectory(w, data, mode):
    """Per-step (sel, fetch, n_fetch, out) for every unit; mode: 'split' (the
    four calls, device buffers), 'device' or 'host' (nosa_decode_step with q
    and out in device or pinned host memory)."""
    dec = runner.Decoder(w, data)
    rec = []
    try:
        q_host = dec.q_all.cpu().pin_memory()
        out_host = torch.empty(dec.out.shape, dtype=dec.out.dtype, pin_memory=True)
        out_dev = torch.empty_like(dec.out)
        for t in range(w.steps):
            if mode == "split":
                dec.step()
                out = dec.out
            elif mode == "device":
                dec.step_through(dec.q_all[t], out_dev)
                out = out_dev
            else:
                dec.step_through(q_host[t], out_host)
                out = out_host
            torch.cuda.synchronize()
            rec.append((dec.sel.cpu().numpy().copy(), dec.fetch.cpu().numpy().copy(),
                        dec.n_fetch.cpu().numpy().copy(), out.cpu().clone()))
        dec.check()
        stats = dec.stats()
    finally:
        dec.close()
    return rec, stats


@pytest.mark.parametrize("name,kw", [
    ("tiny", {}),
    ("tiny", {"offloaded": False, "cache_factor": 0}),
    ("offload_b64", {"steps": 12}),
    ("long_input", {"batch": 1, "steps": 6}),      # beyond the fused kernel
    ("long_gen", {"batch": 2, "steps": 70}),       # appends, a block closes
])
def test_decode_step_matches_the_split_calls(name, kw):
    w = configs.get(name, **kw)
    data = inputs.generate(w)
    ref, st_ref = _trajectory(w, data, "split")
    for mode in ("device", "host"):
        got, st = _trajectory(w, data, mode)
        for t, (a, b) in enumerate(zip(ref, got)):
            for x, y in zip(a[:3], b[:3]):
                assert np.array_equal(x, y), (mode, t)
            assert torch.equal(a[3], b[3]), (mode, t)
        assert st == st_ref, mode


def test_decode_step_with_host_buffers_matches_the_oracle():
    w = configs.get("tiny")
    data = inputs.generate(w)
    got, _ = _trajectory(w, data, "host")
    refs = run_oracle(w, data, range(w.units), range(w.steps))
    for t, (sel, fetch, nf, out) in enumerate(got):
        o = out.float().numpy().reshape(w.units, w.group, w.head_dim)
        for u in range(w.units):
            assert np.array_equal(sel[u], refs[u].sel[t])
            assert np.array_equal(fetch[u], refs[u].fetch[t])
            err = np.abs(o[u] - refs[u].o[t])
            assert err.max() <= 2e-2 and err.mean() <= 2e-3


def test_decode_step_captured_in_a_graph():
    """The one-call step with host buffers, captured once and replayed: the
    queries are read from the same pinned buffer each replay."""
    w = configs.get("tiny", steps=10)
    data = inputs.generate(w)
    ref, _ = _trajectory(w, data, "split")
    dec = runner.Decoder(w, data)
    try:
        q_host = dec.q_all.cpu().pin_memory()
        q_buf = torch.empty_like(q_host[0]).pin_memory()
        out_host = torch.empty(dec.out.shape, dtype=dec.out.dtype, pin_memory=True)
        q_buf.copy_(q_host[0])
        dec.step_through(q_buf, out_host)
        torch.cuda.synchronize()
        assert torch.equal(out_host, ref[0][3])
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=dec.stream):
            from kv_cache_decode_step_b200 import nosa
            nosa.nosa_decode_step(dec.ctx, q_buf, out_host, dec.scores, dec.sel, dec.fetch, dec.n_fetch,
                                  dec.stream, dec.copy_stream)
        for t in range(1, w.steps):
            q_buf.copy_(q_host[t])
            with torch.cuda.stream(dec.stream):
                g.replay()
            torch.cuda.synchronize()
            assert np.array_equal(dec.sel.cpu().numpy(), ref[t][0]), t
            assert torch.equal(out_host, ref[t][3]), t
        del g
        dec.check()
    finally:
        dec.close()
