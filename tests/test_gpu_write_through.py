"""Blocks closed while decoding with KV in host memory: pooled at close,
staged in HBM and written through to the host store during the next step
(NOSA: Native and Offloadable Sparse Attention, paperlayer summary, §4 and
App. A, reading for growing sequences).

A block that is selected in the step right after it closed is a miss whose
host copy may still be in flight; the gather must then read the staged copy.
Agnostic scores above every prompt block's make each new block enter the
agnostic set at once, so that case occurs at every close."""

import numpy as np
import pytest
import torch

from gpu_harness import check_all_unit_invariants, compare, run_gpu, run_oracle
from kv_cache_decode_step_b200 import configs, inputs, nosa, runner

pytestmark = pytest.mark.gpu


def _eager_new_blocks(w):
    data = inputs.generate(w)
    data["a"][:, w.n_blocks0:] = 2.0   # prompt blocks draw U(0, 1)
    return data


@pytest.mark.parametrize("graph", [False, True])
def test_block_selected_right_after_its_close_matches_the_oracle(graph):
    # tail of 60 tokens: block 64 closes at step 3, block 65 at step 67
    w = configs.get("tiny", context=4096 + 60, steps=72, append=True)
    data = _eager_new_blocks(w)
    sample = list(range(w.units))
    attend = [2, 3, 4, 5, 66, 67, 68, 69, 71]
    rec = run_gpu(w, data, sample, attend, graph=graph, cache_steps=[4, 68])
    refs = run_oracle(w, data, sample, attend)
    compare(w, rec, refs, sample)
    check_all_unit_invariants(w, rec, w.steps)
    for i in range(len(sample)):
        assert 64 in rec.sel[4, i] and 64 in rec.fetch[4, i]
        assert 65 in rec.sel[68, i] and 65 in rec.fetch[68, i]


def _block_bits(store, b):
    """bf16 bits of block b of every unit in a [U, T, d] store."""
    return store[:, b * 64:(b + 1) * 64].contiguous().view(torch.int16).numpy().view(np.uint16)


def test_host_store_holds_the_closed_block_after_the_next_step():
    w = configs.get("tiny", context=4096 + 60, steps=8, append=True)
    data = inputs.generate(w)
    dec = runner.Decoder(w, data)
    try:
        for _ in range(5):       # the close at step 3; step 4 writes it through
            dec.step()
        dec.stream.synchronize()
        assert np.array_equal(_block_bits(dec.k_store, 64), data["k"][:, 64 * 64:65 * 64])
        assert np.array_equal(_block_bits(dec.v_store, 64), data["v"][:, 64 * 64:65 * 64])
        dec.check()
    finally:
        dec.close()


def test_checkpoint_lands_a_pending_write_through():
    w = configs.get("tiny", context=4096 + 60, steps=8, append=True)
    data = inputs.generate(w)
    dec = runner.Decoder(w, data)
    try:
        for _ in range(4):       # step 3 closes block 64; no step has written it through yet
            dec.step()
        dec.stream.synchronize()
        nosa.nosa_get_state(dec.ctx)
        assert np.array_equal(_block_bits(dec.k_store, 64), data["k"][:, 64 * 64:65 * 64])
        assert np.array_equal(_block_bits(dec.v_store, 64), data["v"][:, 64 * 64:65 * 64])
        dec.check()
    finally:
        dec.close()
