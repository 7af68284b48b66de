"""Block scores written by the step (NOSA: Native and Offloadable Sparse
Attention, paperlayer summary, §3.1) against the oracle's fp64 scores, with
the pooled keys covering every finite bf16 bit pattern.

Scores are fp64 sums of exact products of bf16 keys with the group-summed
fp64 query, so the widening of every key pattern (normal, subnormal, zero)
matters.  A sub-block whose 16 keys are equal pools to that key
exactly, so the keys can be laid out so that sub-block 0 of each block holds
128 chosen patterns while sub-blocks 1-3 hold the most negative finite bf16
and never win the max over sub-blocks.  With every query 1.0 a block's score
is then 4 x the sum of its 128 patterns; patterns are sorted by sign, then magnitude, so that the terms
of one sum are alike and a wrong widening of any one term shows."""

import numpy as np
import pytest

import oracle
from kv_cache_decode_step_b200 import configs, inputs, runner

pytestmark = pytest.mark.gpu


def _finite_patterns():
    bits = np.arange(1 << 16, dtype=np.uint32)
    exp = (bits >> 7) & 0xFF
    keep = bits[exp != 0xFF].astype(np.uint16)                     # drop infinities and NaNs
    mag = keep & 0x7FFF                                            # order of |value|
    sign = keep >> 15
    return keep[np.lexsort((mag, sign))]                           # positives, then negatives


def _workload_and_data(n_units_needed):
    # resident, 2 KV heads, 64 blocks of 64 tokens per unit
    batch = (n_units_needed + 1) // 2
    w = configs.get("tiny", batch=batch, offloaded=False, cache_factor=0, steps=2)
    data = inputs.generate(w)
    return w, data


def _pattern_case():
    pats = _finite_patterns()                                   # 65,280 patterns
    blocks_needed = -(-len(pats) // 128)
    w, data = _workload_and_data(-(-blocks_needed // 64))
    U, d, n = w.units, w.head_dim, w.n_blocks0
    pad = np.full(U * n * 128 - len(pats), 0x3F80, dtype=np.uint16)  # 1.0 fills the last block
    rows = np.concatenate([pats, pad]).reshape(U, n, 128)
    neg = np.uint16(0xFF7F)                                     # -3.39e38, the most negative finite bf16
    k = np.full((U, w.max_tokens, d), neg, dtype=np.uint16)
    blk = k[:, : n * 64].reshape(U, n, 4, 16, d).copy()
    blk[:, :, 0, :, :] = rows[:, :, None, :]                    # 16 equal tokens in sub-block 0
    k[:, : n * 64] = blk.reshape(U, n * 64, d)
    data["k"] = k
    data["q"][:] = 0x3F80                                       # every query 1.0
    return w, data, rows


def _step_scores(w, data, fused):
    dec = runner.Decoder(w, data, fused=fused)
    try:
        dec.step()
        dec.stream.synchronize()
        got = dec.scores.cpu().numpy()[:, : w.n_blocks0]
        dec.check()
    finally:
        dec.close()
    return got


@pytest.mark.parametrize("fused", [True, False])
def test_scores_cover_every_finite_bf16_pattern(fused):
    w, data, rows = _pattern_case()
    U, d, n = w.units, w.head_dim, w.n_blocks0
    k = data["k"]
    got = _step_scores(w, data, fused)
    q1 = np.full((w.group, d), 0x3F80, dtype=np.uint16)
    for u in range(U):
        kbar = oracle.pool_keys(k[u, : n * 64], 16)
        want = oracle.score_blocks(q1, kbar, 4)
        vals = np.array([oracle.bf16_to_f64(int(b)) for b in rows[u].reshape(-1)]).reshape(n, 128)
        bound = 4 * np.abs(vals).sum(axis=1) * 128 * 2.0 ** -52
        assert np.all(np.abs(got[u] - want) <= bound), u
        assert np.array_equal(got[u] == 0.0, want == 0.0)


@pytest.mark.parametrize("fused", [True, False])
def test_placed_widening_gives_the_bits_of_conversions(fused, monkeypatch):
    """Half of the keys are widened by placing their bits in the fp64 high
    word (a value 2^896 smaller, the query term 2^896 larger): over every
    finite bf16 pattern the scores are bit-identical to widening every key
    by conversion (NOSA_PLACED_WIDEN=0)."""
    w, data, _ = _pattern_case()
    got = _step_scores(w, data, fused)
    monkeypatch.setenv("NOSA_PLACED_WIDEN", "0")
    want = _step_scores(w, data, fused)
    assert np.array_equal(got.view(np.uint64), want.view(np.uint64))


@pytest.mark.parametrize("fused", [True, False])
def test_queries_too_large_for_placement(fused, monkeypatch):
    """Group sums of 2^126 or more would overflow once scaled by 2^896: those
    warps widen by conversion, and the scores still match the oracle and the
    conversion-only path bit for bit."""
    w = configs.get("tiny", batch=2, offloaded=False, cache_factor=0, steps=2)
    data = inputs.generate(w)
    q = data["q"]                             # [units, steps, group, d]
    q[0, 0] = 0x7E80                          # 8.5e37 in every head of unit 0 at step 0: the group sum > 2^126
    q[0, 0, :, 1::7] = 0xFE80                 # some of them negative
    got = _step_scores(w, data, fused)
    monkeypatch.setenv("NOSA_PLACED_WIDEN", "0")
    want = _step_scores(w, data, fused)
    assert np.array_equal(got.view(np.uint64), want.view(np.uint64))

    def widen(bits):
        return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)

    n = w.n_blocks0
    for u in range(w.units):
        kbar = oracle.pool_keys(data["k"][u, : n * 64], 16)
        ref = oracle.score_blocks(q[u, 0], kbar, 4)
        # fp64 rounding of 128-term sums of exact products
        qt = widen(q[u, 0]).sum(axis=0)
        terms = np.abs(widen(kbar).reshape(n, 4, -1) * qt).sum(axis=2).max(axis=1)
        assert np.all(np.abs(got[u] - ref) <= terms * 128 * 2.0 ** -52), u
