"""The allocation-free attention entry point.

Some callers of this library cannot call cudaMalloc -- for instance a serving
engine whose pool allocator already owns nearly all of HBM, or code that must
not add the device-wide synchronisation an allocation can cause.  For them
nosa_sparse_decode_noalloc runs the attention step with its split-KV scratch in
a fixed array inside the library.  It launches the same kernel with the same
grid and walk as nosa_sparse_decode over resident KV, so its output must be
bit-identical to that path's on the same inputs, on two calls in a row; it is
also checked against the oracle's fp64 attention, a call must not change the
device's free memory, and device-side errors must reach the caller through
nosa_noalloc_check_errors.  This file is named to be collected last.
"""

import numpy as np
import pytest
import torch

import oracle
from kv_cache_decode_step_b200 import configs, inputs, nosa, runner

pytestmark = pytest.mark.gpu

TOL_MAX, TOL_MEAN = 2e-2, 2e-3


def test_noalloc_attention_matches_the_context_path_on_two_calls():
    # resident 8B-shaped layer, 4 sequences: 32 units, 256 blocks, budget 64
    w = configs.get("layer8b", batch=4, steps=2)
    data = inputs.generate(w)
    dec = runner.Decoder(w, data)
    cfg = oracle.cfg_from_workload(w)
    try:
        out = torch.empty_like(dec.out)
        free_before_second = None
        for call in range(2):
            dec.step()
            dec.stream.synchronize()
            want = dec.out.clone()
            sel = dec.sel.cpu().numpy()
            if call == 1:
                torch.cuda.synchronize()
                free_before_second = torch.cuda.mem_get_info()[0]
            out.fill_(0)
            with torch.cuda.stream(dec.stream):
                nosa.nosa_sparse_decode_noalloc(dec.q, dec.k_store, dec.v_store, w.batch, w.n_q_heads,
                                                w.n_kv_heads, w.max_blocks, dec.sel, w.k, out, dec.stream)
            nosa.nosa_noalloc_check_errors(dec.stream)
            if call == 1:
                assert torch.cuda.mem_get_info()[0] == free_before_second
            assert torch.equal(out, want), f"call {call}: output differs from nosa_sparse_decode"
            # and against the oracle's fp64 attention over the same blocks
            o = out.float().cpu().numpy().reshape(w.units, w.group, w.head_dim)
            q = dec.q.view(torch.int16).cpu().numpy().view(np.uint16).reshape(w.units, w.group, w.head_dim)
            errs = []
            for u in (0, 7, 19, w.units - 1):
                rows = np.concatenate([np.arange(b * w.block, (b + 1) * w.block) for b in sel[u]])
                ref = oracle.attend(q[u], data["k"][u], data["v"][u], rows)
                errs.append(np.abs(o[u] - ref))
            err = np.stack(errs)
            assert err.max() <= TOL_MAX and err.mean() <= TOL_MEAN, (err.max(), err.mean())
        dec.check()
    finally:
        dec.close()


def test_noalloc_reports_an_out_of_range_block_id():
    """An id outside [0, max_blocks) is flagged (and block 0 read in its
    place); the next check reports it once, then the word is clear again."""
    w = configs.get("tiny", offloaded=False, cache_factor=0)
    data = inputs.generate(w)
    kv_k = torch.from_numpy(data["k"]).view(torch.bfloat16).cuda()
    kv_v = torch.from_numpy(data["v"]).view(torch.bfloat16).cuda()
    q = torch.zeros((w.batch, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    out = torch.empty_like(q)
    sel = torch.arange(w.k, dtype=torch.int32, device="cuda").repeat(w.units, 1).contiguous()
    nosa.nosa_noalloc_check_errors(None)  # start from a clear word
    sel[1, 5] = w.max_blocks + 3
    nosa.nosa_sparse_decode_noalloc(q, kv_k, kv_v, w.batch, w.n_q_heads, w.n_kv_heads, w.max_blocks, sel, w.k,
                                    out, None)
    with pytest.raises(nosa.NosaError) as e:
        nosa.nosa_noalloc_check_errors(None)
    assert e.value.status == nosa.NOSA_ERR_INVALID
    sel[1, 5] = 5
    nosa.nosa_sparse_decode_noalloc(q, kv_k, kv_v, w.batch, w.n_q_heads, w.n_kv_heads, w.max_blocks, sel, w.k,
                                    out, None)
    nosa.nosa_noalloc_check_errors(None)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    q = torch.zeros((512, 32, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((8, 16 * 64, 128), dtype=torch.bfloat16, device="cuda")
    sel = torch.zeros((512 * 8, 16), dtype=torch.int32, device="cuda")
    # 512 sequences x 32 query heads = 16384 > 8192: rejected before any launch
    with pytest.raises(nosa.NosaError) as e:
        nosa.nosa_sparse_decode_noalloc(q, kv, kv, 512, 32, 8, 16, sel, 16, q, None)
    assert e.value.status == nosa.NOSA_ERR_INVALID
    assert "8192" in str(e.value)
