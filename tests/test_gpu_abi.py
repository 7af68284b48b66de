"""GPU behaviour of the C ABI beyond numerics: call order, pointer kinds,
bounded device waits, checkpoint/restore, graph replay determinism and the
statistics the pages' measurements need (locality, hit rate)."""

import numpy as np
import pytest
import torch

from kv_cache_decode_step_b200 import configs, inputs, nosa, runner

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tiny():
    w = configs.get("tiny", steps=12)
    return w, inputs.generate(w)


def test_step_calls_out_of_order_are_rejected(tiny):
    w, data = tiny
    dec = runner.Decoder(w, data)
    try:
        s = dec.stream
        with pytest.raises(nosa.NosaError) as e:
            nosa.nosa_select(dec.ctx, dec.scores, dec.sel, s)
        assert e.value.status == nosa.NOSA_ERR_ORDER
        with pytest.raises(nosa.NosaError):
            nosa.nosa_sparse_decode(dec.ctx, dec.q, dec.sel, dec.out, s)
        nosa.nosa_score_blocks(dec.ctx, dec.q, dec.scores, s)
        with pytest.raises(nosa.NosaError) as e:
            nosa.nosa_score_blocks(dec.ctx, dec.q, dec.scores, s)
        assert e.value.status == nosa.NOSA_ERR_ORDER
        nosa.nosa_select(dec.ctx, dec.scores, dec.sel, s)
        with pytest.raises(nosa.NosaError):  # offloaded: decode needs the fetch first
            nosa.nosa_sparse_decode(dec.ctx, dec.q, dec.sel, dec.out, s)
        with pytest.raises(nosa.NosaError):  # append only at the start of a step
            nosa.nosa_append_token(dec.ctx, dec.q, dec.q, None, s)
        nosa.nosa_fetch_missing(dec.ctx, dec.sel, dec.fetch, dec.n_fetch, s, s)
        nosa.nosa_sparse_decode(dec.ctx, dec.q, dec.sel, dec.out, s)
        dec.check()
    finally:
        dec.close()


def test_fused_first_half_follows_the_same_order(tiny):
    """nosa_score_select_fetch stands for score + select + fetch: it starts a
    step, cannot be repeated, and is followed by the decode call only."""
    w, data = tiny
    dec = runner.Decoder(w, data)
    try:
        s = dec.stream
        args = (dec.ctx, dec.q, dec.scores, dec.sel, dec.fetch, dec.n_fetch, s, s)
        nosa.nosa_score_blocks(dec.ctx, dec.q, dec.scores, s)
        with pytest.raises(nosa.NosaError) as e:  # a step is already under way
            nosa.nosa_score_select_fetch(*args)
        assert e.value.status == nosa.NOSA_ERR_ORDER
        nosa.nosa_select(dec.ctx, dec.scores, dec.sel, s)
        nosa.nosa_fetch_missing(dec.ctx, dec.sel, dec.fetch, dec.n_fetch, s, s)
        nosa.nosa_sparse_decode(dec.ctx, dec.q, dec.sel, dec.out, s)
        nosa.nosa_score_select_fetch(*args)
        with pytest.raises(nosa.NosaError) as e:
            nosa.nosa_score_select_fetch(*args)
        assert e.value.status == nosa.NOSA_ERR_ORDER
        with pytest.raises(nosa.NosaError) as e:
            nosa.nosa_select(dec.ctx, dec.scores, dec.sel, s)
        assert e.value.status == nosa.NOSA_ERR_ORDER
        nosa.nosa_sparse_decode(dec.ctx, dec.q, dec.sel, dec.out, s)
        with pytest.raises(nosa.NosaError) as e:  # NULL outputs are rejected before any launch
            nosa.nosa_score_select_fetch(dec.ctx, dec.q, dec.scores, dec.sel, None, dec.n_fetch, s, s)
        assert e.value.status == nosa.NOSA_ERR_INVALID
        dec.check()
    finally:
        dec.close()


def test_pointer_kinds_are_checked(tiny):
    w, data = tiny
    ctx = nosa.nosa_create(nosa.config_from_workload(w))
    try:
        U, T, d = w.units, w.max_tokens, w.head_dim
        dev_kv = torch.zeros((U, T, d), dtype=torch.bfloat16, device="cuda")
        pageable = torch.zeros((U, T, d), dtype=torch.bfloat16)
        a = torch.zeros((U, w.max_blocks), device="cuda")
        for kv in (dev_kv, pageable):  # offloaded KV must be pinned host memory
            with pytest.raises(nosa.NosaError) as e:
                nosa.nosa_attach_kv(ctx, kv, kv, w.context, a, None)
            assert e.value.status == nosa.NOSA_ERR_INVALID
        pinned = torch.zeros((U, T, d), dtype=torch.bfloat16, pin_memory=True)
        with pytest.raises(nosa.NosaError):  # agnostic scores must be on the device
            nosa.nosa_attach_kv(ctx, pinned, pinned, w.context, a.cpu(), None)
        with pytest.raises(nosa.NosaError):  # fewer than k blocks
            nosa.nosa_attach_kv(ctx, pinned, pinned, 64 * (w.k - 1), a, None)
        nosa.nosa_attach_kv(ctx, pinned, pinned, w.context, a, None)
    finally:
        nosa.nosa_destroy(ctx)
    wr = w.with_(offloaded=False, cache_factor=0)
    ctx = nosa.nosa_create(nosa.config_from_workload(wr))
    try:
        pinned = torch.zeros((wr.units, wr.max_tokens, wr.head_dim), dtype=torch.bfloat16, pin_memory=True)
        a = torch.zeros((wr.units, wr.max_blocks), device="cuda")
        with pytest.raises(nosa.NosaError):  # resident KV must be device memory
            nosa.nosa_attach_kv(ctx, pinned, pinned, wr.context, a, None)
        with pytest.raises(nosa.NosaError):  # no cache map when resident
            nosa.nosa_read_cache_map(ctx, np.zeros(4, np.int32))
    finally:
        nosa.nosa_destroy(ctx)


def test_bounded_wait_times_out_and_context_survives(tiny):
    w, data = tiny
    dec = runner.Decoder(w, data)
    try:
        flag = torch.zeros(1, dtype=torch.int32, device="cuda")  # nothing ever sets it
        nosa.nosa_debug_wait_flag(dec.ctx, flag, 50, dec.stream)
        with pytest.raises(nosa.NosaError) as e:
            nosa.nosa_check_errors(dec.ctx)
        assert e.value.status == nosa.NOSA_ERR_TIMEOUT
        # a set flag returns at once
        flag.fill_(1)
        torch.cuda.synchronize()
        nosa.nosa_debug_wait_flag(dec.ctx, flag, 1000, dec.stream)
        dec.stream.synchronize()
        # the context still decodes after the timeout (error bits are sticky
        # until the next attach)
        dec.attach()
        for _ in range(3):
            dec.step()
        dec.check()
    finally:
        dec.close()


@pytest.mark.parametrize("name,kw", [("offload_b64", {"batch": 8, "steps": 10}),
                                     ("tiny", {"steps": 80, "append": True, "context": 4096 + 20})])
def test_graph_replay_equals_eager(name, kw):
    w = configs.get(name, **kw)
    data = inputs.generate(w)
    outs = []
    for graph in (False, True):
        dec = runner.Decoder(w, data)
        seq = []
        try:
            for t in range(w.steps):
                if graph and t >= 1:
                    if dec.graph is None:
                        dec.capture()
                    dec.replay()
                else:
                    dec.step()
                dec.stream.synchronize()
                seq.append((dec.sel.cpu().numpy().copy(), dec.out.cpu().view(torch.int16).numpy().copy()))
            dec.check()
        finally:
            dec.close()
        outs.append(seq)
    for (s0, o0), (s1, o1) in zip(*outs):
        assert np.array_equal(s0, s1) and np.array_equal(o0, o1)


@pytest.mark.parametrize("name,kw", [("tiny", {"steps": 20}),
                                     ("tiny", {"steps": 80, "append": True, "context": 4096 + 30}),
                                     ("tiny", {"steps": 20, "offloaded": False, "cache_factor": 0})])
def test_checkpoint_restore_replays_bit_exactly(name, kw):
    w = configs.get(name, **kw)
    data = inputs.generate(w)
    dec = runner.Decoder(w, data)
    try:
        half = w.steps // 2
        for _ in range(half):
            dec.step()
        dec.stream.synchronize()
        blob = nosa.nosa_get_state(dec.ctx)
        first = []
        for _ in range(w.steps - half):
            dec.step()
            dec.stream.synchronize()
            first.append((dec.sel.cpu().numpy().copy(), dec.out.cpu().view(torch.int16).numpy().copy()))
        nosa.nosa_set_state(dec.ctx, blob)
        dec.t = half
        for i in range(w.steps - half):
            dec.step()
            dec.stream.synchronize()
            s, o = first[i]
            assert np.array_equal(dec.sel.cpu().numpy(), s)
            assert np.array_equal(dec.out.cpu().view(torch.int16).numpy(), o)
        with pytest.raises(nosa.NosaError):
            nosa.nosa_set_state(dec.ctx, blob[:-4])
        dec.check()
    finally:
        dec.close()


def test_locality_and_hit_rate_statistics():
    """gamma(t) = |S(t) ∩ S(t-1)| / |S(t)| is at least m / k every step, and
    hits + misses account for every selected block."""
    w = configs.get("offload_b64", batch=16, steps=40)
    data = inputs.generate(w)
    dec = runner.Decoder(w, data)
    try:
        fetched = []
        for t in range(w.steps):
            dec.step()
            dec.stream.synchronize()
            fetched.append(int(dec.n_fetch.sum().item()))
        st = dec.stats()
        assert fetched[0] == w.units * w.k  # cold cache
        assert st["misses"] == sum(fetched)
        assert st["min_overlap"] / w.k >= w.min_overlap / w.k
        gamma = st["overlap_sum"] / (st["overlap_terms"] * w.k)
        assert w.min_overlap / w.k <= gamma <= 1.0
        nosa.nosa_reset_stats(dec.ctx, dec.stream)
        assert dec.stats()["steps"] == 0
    finally:
        dec.close()
