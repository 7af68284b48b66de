"""The launch-time choices that only change how the work is scheduled must not
change a single bit of what a step computes: the gather launched as a
programmatic dependent of the plan (NOSA_PDL), the scoring's widening of half
of the keys by bit placement (NOSA_PLACED_WIDEN), and the L2 warm-up of the
hits pass's first blocks during the selection (NOSA_WARM_BLOCKS).  Each knob
is read when a context is created; every step's selections, fetch lists,
scores and outputs are compared bit for bit with the knob off."""

import numpy as np
import pytest
import torch

from kv_cache_decode_step_b200 import configs, inputs, runner

pytestmark = pytest.mark.gpu


def _trajectory(w, data, graph):
    dec = runner.Decoder(w, data)
    rec = []
    try:
        for t in range(w.steps):
            if graph and t == 2:
                dec.capture()
            if graph and t >= 2:
                dec.replay()
            else:
                dec.step()
            torch.cuda.synchronize()
            rec.append((dec.sel.cpu().numpy().copy(), dec.fetch.cpu().numpy().copy(),
                        dec.scores.cpu().numpy().copy(), dec.out.view(torch.int16).cpu().numpy().copy()))
        dec.check()
    finally:
        dec.close()
    return rec


@pytest.mark.parametrize("knob,off", [("NOSA_PDL", "0"), ("NOSA_PLACED_WIDEN", "0"), ("NOSA_WARM_BLOCKS", "0")])
@pytest.mark.parametrize("name,kw", [
    ("layer8b", {"batch": 2, "steps": 8}),       # KV in HBM: the warm-up runs
    ("offload_b64", {"batch": 4, "steps": 8}),   # KV in host memory: the gather follows the plan
    ("long_input", {"batch": 1, "steps": 5}),    # scoring grid, then select/plan (a dependent launch)
])
def test_knob_changes_no_bit(name, kw, knob, off, monkeypatch):
    w = configs.get(name, **kw)
    data = inputs.generate(w)
    got = _trajectory(w, data, graph=True)
    monkeypatch.setenv(knob, off)
    want = _trajectory(w, data, graph=True)
    for t, (a, b) in enumerate(zip(got, want)):
        for what, x, y in zip(("sel", "fetch", "scores", "out"), a, b):
            assert np.array_equal(x.view(np.uint8), y.view(np.uint8)), f"{knob}: step {t} {what} differs"
