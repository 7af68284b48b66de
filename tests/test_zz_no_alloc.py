"""The allocation-free attention entry point.

Some callers of this library cannot call cudaMalloc -- for instance a serving
engine whose pool allocator already owns nearly all of HBM, or code that must
not add the device-wide synchronisation an allocation can cause.  For them
nosa_sparse_decode_noalloc runs the attention step with its split-KV scratch in
a fixed array inside the library.  Its output must match nosa_sparse_decode's
on the same inputs, on two calls in a row, and a call must not change the
device's free memory.  This file is named to be collected last.
"""

import numpy as np
import pytest
import torch

from kv_cache_decode_step_b200 import configs, inputs, nosa, runner

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN = 2e-2, 2e-3


def test_noalloc_attention_matches_the_context_path_on_two_calls():
    # resident 8B-shaped layer, 4 sequences: 32 units, 256 blocks, budget 64
    w = configs.get("layer8b", batch=4, steps=2)
    data = inputs.generate(w)
    dec = runner.Decoder(w, data)
    try:
        out = torch.empty_like(dec.out)
        free_before_second = None
        for call in range(2):
            dec.step()
            dec.stream.synchronize()
            want = dec.out.float().clone()
            if call == 1:
                torch.cuda.synchronize()
                free_before_second = torch.cuda.mem_get_info()[0]
            out.fill_(0)
            with torch.cuda.stream(dec.stream):
                nosa.nosa_sparse_decode_noalloc(dec.q, dec.k_store, dec.v_store, w.batch, w.n_q_heads,
                                                w.n_kv_heads, w.max_blocks, dec.sel, w.k, out, dec.stream)
            dec.stream.synchronize()
            if call == 1:
                assert torch.cuda.mem_get_info()[0] == free_before_second
            err = (out.float() - want).abs()
            assert err.max().item() <= TOL_MAX
            assert err.mean().item() <= TOL_MEAN
        dec.check()
    finally:
        dec.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    q = torch.zeros((512, 32, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((8, 16 * 64, 128), dtype=torch.bfloat16, device="cuda")
    sel = torch.zeros((512 * 8, 16), dtype=torch.int32, device="cuda")
    # 512 sequences x 32 query heads = 16384 > 8192: rejected before any launch
    with pytest.raises(nosa.NosaError) as e:
        nosa.nosa_sparse_decode_noalloc(q, kv, kv, 512, 32, 8, 16, sel, 16, q, None)
    assert e.value.status == nosa.NOSA_ERR_INVALID
    assert "8192" in str(e.value)
