"""Injected transfer and launch failures, made on the host.

Each CUDA runtime call that the fetch and decode calls make (event records,
stream waits, the plan, gather and attention launches) is made to fail in turn
by nosa_debug_inject_cuda_error: the call is not made and reports a launch
failure.  The entry point must return NOSA_ERR_CUDA with a message instead of
aborting, leave the device without error bits, and after a re-attach the
context must decode the whole trajectory bit-exactly like the oracle again.
Nothing here faults or stalls the GPU: the failure exists only on the host.
"""

import numpy as np
import pytest
import torch

from kv_cache_decode_step_b200 import configs, inputs, nosa, runner
from gpu_harness import run_oracle, TOL_MAX

pytestmark = pytest.mark.gpu


def _failing_step(dec, which, skip):
    """One step whose `which` call meets an injected failure after `skip`
    successful checks; returns True if the failure fired."""
    s, cs = dec.stream, dec.copy_stream
    fired = False
    with torch.cuda.stream(s):
        dec._load_inputs(dec.t)
        calls = [("score", lambda: nosa.nosa_score_blocks(dec.ctx, dec.q, dec.scores, s)),
                 ("select", lambda: nosa.nosa_select(dec.ctx, dec.scores, dec.sel, s)),
                 ("fetch", lambda: nosa.nosa_fetch_missing(dec.ctx, dec.sel, dec.fetch, dec.n_fetch, s, cs)),
                 ("decode", lambda: nosa.nosa_sparse_decode(dec.ctx, dec.q, dec.sel, dec.out, s))]
        for name, fn in calls:
            if name == which:
                nosa.nosa_debug_inject_cuda_error(skip)
                try:
                    fn()
                except nosa.NosaError as e:
                    assert e.status == nosa.NOSA_ERR_CUDA, e
                    assert "cudaErrorLaunchFailure" in str(e) or "unspecified launch failure" in str(e), e
                    fired = True
                    break
                finally:
                    nosa.nosa_debug_inject_cuda_error(-1)
            else:
                fn()
    torch.cuda.synchronize()
    return fired


def _replay_against_oracle(dec, w, refs):
    dec.attach()
    for t in range(w.steps):
        dec.step()
        dec.stream.synchronize()
        sel = dec.sel.cpu().numpy()
        fetch = dec.fetch.cpu().numpy()
        out = dec.out.float().cpu().numpy().reshape(w.units, w.group, w.head_dim)
        for u in range(w.units):
            assert np.array_equal(sel[u], refs[u].sel[t]), (t, u)
            assert np.array_equal(fetch[u], refs[u].fetch[t]), (t, u)
            assert np.abs(out[u] - refs[u].o[t]).max() <= TOL_MAX
    dec.check()


@pytest.mark.parametrize("which", ["fetch", "decode"])
@pytest.mark.parametrize("side_stream", [True, False])
def test_injected_failure_returns_cuda_status_and_the_context_recovers(which, side_stream):
    w = configs.get("tiny", steps=6)
    data = inputs.generate(w)
    refs = run_oracle(w, data, range(w.units), range(w.steps))
    dec = runner.Decoder(w, data, side_copy_stream=side_stream, fused=False)
    try:
        fired = 0
        for skip in range(12):
            dec.attach()
            dec.step()                      # step 0 runs clean
            if not _failing_step(dec, which, skip):
                break                       # skip beyond the call's checked CUDA calls
            fired += 1
            dec.check()                     # no device-side error bits
        assert fired >= 1
        _replay_against_oracle(dec, w, refs)
    finally:
        dec.close()


def test_injected_failure_in_the_fused_first_half():
    w = configs.get("tiny", steps=6)
    data = inputs.generate(w)
    refs = run_oracle(w, data, range(w.units), range(w.steps))
    dec = runner.Decoder(w, data)
    try:
        dec.attach()
        dec.step()
        s, cs = dec.stream, dec.copy_stream
        nosa.nosa_debug_inject_cuda_error(0)
        with pytest.raises(nosa.NosaError) as e:
            nosa.nosa_score_select_fetch(dec.ctx, dec.q, dec.scores, dec.sel, dec.fetch, dec.n_fetch, s, cs)
        assert e.value.status == nosa.NOSA_ERR_CUDA
        nosa.nosa_debug_inject_cuda_error(-1)
        torch.cuda.synchronize()
        _replay_against_oracle(dec, w, refs)
    finally:
        dec.close()
