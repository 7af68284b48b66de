"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these tests retypes the oracle's formula: each compares it with an
independent formulation (a library routine, brute-force enumeration, a closed
form, a hand-worked example) or checks an invariant the pages state.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from kv_cache_decode_step_b200 import configs, inputs

HERE = os.path.dirname(os.path.abspath(__file__))


def bits_to_f64(b):
    return inputs.bf16_bits_to_f32(np.asarray(b, dtype=np.uint16)).astype(np.float64)


# --------------------------------------------------------------- bf16 rounding

def test_bf16_rounding_matches_torch_on_fp32_values(orc):
    rng = np.random.default_rng(1)
    # random fp32 bit patterns over the whole finite range (incl. subnormals)
    raw = rng.integers(0, 2**32, size=40000, dtype=np.uint64).astype(np.uint32)
    x = raw.view(np.float32)
    x = x[np.isfinite(x)]
    # plus exact halfway cases: low 16 bits == 0x8000
    half = (rng.integers(0, 2**16, size=4000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    hx = half.view(np.float32)
    x = np.concatenate([x, hx[np.isfinite(hx)]])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.f64_to_bf16(float(v)) for v in x], dtype=np.uint16)
    # torch may produce a different NaN payload; none here, all finite
    assert np.array_equal(got, want)


def _bf16_neighbours(b):
    """bf16 values adjacent to bit pattern b (same sign side)."""
    return [(b - 1) & 0xFFFF, (b + 1) & 0xFFFF]


def test_bf16_rounding_nearest_even_on_fp64_values(orc):
    rng = np.random.default_rng(2)
    xs = np.concatenate([
        rng.standard_normal(3000) * 10.0 ** rng.integers(-40, 38, 3000),
        rng.standard_normal(500) * 2.0 ** -130,  # bf16 subnormal range
    ])
    for x in xs:
        b = orc.f64_to_bf16(float(x))
        r = orc.bf16_to_f64(b)
        err = abs(x - r)
        for nb in _bf16_neighbours(b):
            rn = orc.bf16_to_f64(nb)
            if not math.isfinite(rn) or (rn != 0 and math.copysign(1, rn) != math.copysign(1, r)):
                continue
            en = abs(x - rn)
            assert err <= en, (x, hex(b), hex(nb))
            if err == en:  # exact tie: the kept value has an even significand
                assert b % 2 == 0


def test_bf16_rounding_specials(orc):
    assert orc.f64_to_bf16(0.0) == 0x0000
    assert orc.f64_to_bf16(-0.0) == 0x8000
    assert orc.f64_to_bf16(float("inf")) == 0x7F80
    assert orc.f64_to_bf16(-float("inf")) == 0xFF80
    assert orc.f64_to_bf16(1e39) == 0x7F80            # above bf16 max -> inf
    assert orc.f64_to_bf16(3.3895313892515355e38) == 0x7F7F  # bf16 max
    assert orc.f64_to_bf16(2.0 ** -133) == 0x0001     # smallest subnormal
    assert orc.f64_to_bf16(2.0 ** -134) == 0x0000     # tie to even (zero)
    assert orc.f64_to_bf16(1.5 * 2.0 ** -133) == 0x0002  # tie to even (2)
    assert orc.f64_to_bf16(1.0 + 2.0 ** -8) == 0x3F80    # tie -> even 1.0
    assert orc.f64_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82  # tie -> even
    assert orc.f64_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81  # just above tie


# --------------------------------------------------------------- a0 pooling

def test_pool_constant_subblock_pools_to_itself(orc):
    rng = np.random.default_rng(3)
    vals = inputs.f32_to_bf16_bits(rng.standard_normal((8, 128)).astype(np.float32))
    K = np.repeat(vals, 16, axis=0)  # sub-block s is 16 copies of row s
    assert np.array_equal(orc.pool_keys(K, 16), vals)


def test_pool_matches_torch_mean(orc):
    rng = np.random.default_rng(4)
    K = inputs.f32_to_bf16_bits(rng.standard_normal((64 * 16, 128)).astype(np.float32))
    got = orc.pool_keys(K, 16)
    Kf = torch.from_numpy(bits_to_f64(K)).reshape(64, 16, 128)
    mean = Kf.mean(dim=1)  # fp64
    exact32 = (mean.to(torch.float32).to(torch.float64) == mean)
    want = mean.to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    m = exact32.numpy()
    assert m.mean() > 0.95
    assert np.array_equal(got[m], want[m])


def test_pool_grouping_and_scaling(orc):
    rng = np.random.default_rng(5)
    K = inputs.f32_to_bf16_bits(rng.standard_normal((4 * 16, 128)).astype(np.float32))
    base = orc.pool_keys(K, 16)
    # scaling all keys by a power of two scales the pooled keys exactly
    K2 = inputs.f32_to_bf16_bits(bits_to_f64(K).astype(np.float32) * 4.0)
    assert np.array_equal(bits_to_f64(orc.pool_keys(K2, 16)), 4.0 * bits_to_f64(base))
    # permuting tokens inside a sub-block does not change its mean
    perm = np.concatenate([s * 16 + rng.permutation(16) for s in range(4)])
    assert np.array_equal(orc.pool_keys(K[perm], 16), base)
    # moving a token to another sub-block does
    K3 = K.copy()
    K3[[0, 16]] = K3[[16, 0]]
    assert not np.array_equal(orc.pool_keys(K3, 16), base)


# --------------------------------------------------------------- a1 scoring

def test_scores_match_numpy_einsum(orc):
    w = configs.get("tiny")
    d = inputs.generate(w, units=[0, 1], parts=("k", "q"))
    for i in range(2):
        kbar = orc.pool_keys(d["k"][i][: w.n_blocks0 * w.block], w.sub_block)
        for t in (0, 7, 15):
            q = d["q"][i][t]
            got = orc.score_blocks(q, kbar, 4)
            sub = np.einsum("hd,sd->s", bits_to_f64(q), bits_to_f64(kbar))
            want = sub.reshape(-1, 4).max(axis=1)
            assert np.allclose(got, want, rtol=1e-12, atol=1e-12)
            # the max is over a block's own sub-blocks, not a shifted window
            shifted = np.roll(sub, 1).reshape(-1, 4).max(axis=1)
            assert not np.allclose(got, shifted)


def test_planted_blocks_rank_first_for_aligned_query(orc):
    w = configs.get("layer8b")
    u = 3
    K = inputs.unit_kv(w, u, "k")[: w.n_blocks0 * w.block]
    planted = inputs.unit_planted(w, u)
    kbar = orc.pool_keys(K, w.sub_block)
    kb = bits_to_f64(kbar).reshape(w.n_blocks0, 4, 128)
    # a query aligned with the planted blocks' pooled keys
    direction = sum(kb[j].sum(axis=0) for j in planted)
    q = inputs.f32_to_bf16_bits(np.tile(direction, (w.group, 1)).astype(np.float32))
    s = orc.score_blocks(q, kbar, 4)
    top8 = np.sort(np.argsort(-s, kind="stable")[:8])
    assert np.array_equal(top8, planted)


# --------------------------------------------------------------- a2/a3 selection

def brute_evict(a, pool, k_e):
    best, best_set = None, None
    pool = sorted(pool)
    for comb in itertools.combinations(pool, min(k_e, len(pool))):
        val = sum(float(a[j]) for j in comb)
        if best is None or val > best:
            best, best_set = val, comb
    return sorted(best_set)


def brute_select(score, n, E, prev, first, k_q, c_max):
    E = set(E)
    prev = set(prev)
    avail = [j for j in range(n) if j not in E]
    new = set(j for j in avail if j not in prev)
    c_t = 10 ** 9 if first else max(0, c_max - len(E - prev))
    size = min(k_q, len(avail) if first else len(avail))
    best, best_set = None, None
    for r in range(size, -1, -1):
        for comb in itertools.combinations(avail, r):
            if not first and len(new.intersection(comb)) > c_t:
                continue
            val = sum(score[j] for j in comb)
            if best is None or val > best:
                best, best_set = val, comb
        if best_set is not None:
            break  # largest feasible size only
    return sorted(E | set(best_set))


def test_select_equals_brute_force_max_sum(orc):
    rng = np.random.default_rng(6)
    cases = 0
    while cases < 300:
        n = int(rng.integers(6, 13))
        k_e = int(rng.integers(0, 4))
        k_q = int(rng.integers(1, 5))
        k = k_e + k_q
        if k > n:
            continue
        c_max = int(rng.integers(0, k + 1))
        score = rng.standard_normal(n)
        first = bool(rng.random() < 0.2)
        E = sorted(rng.choice(n, size=k_e, replace=False).tolist())
        if first:
            prev = []
        else:
            # previous selection: contains E except possibly one new agnostic block
            others = [j for j in range(n) if j not in E]
            prev = set(rng.choice(others, size=k - k_e, replace=False).tolist()) | set(E)
            if E and rng.random() < 0.3:
                drop = E[int(rng.integers(0, len(E)))]
                prev.discard(drop)
                extra = [j for j in range(n) if j not in prev and j not in E]
                prev.add(extra[0])
            prev = sorted(prev)
        got = orc.select(score, E, prev, first, k_q, c_max)
        want = brute_select(score, n, E, prev, first, k_q, c_max)
        assert got.tolist() == want, (n, k_e, k_q, c_max, first, E, prev)
        cases += 1


def test_evict_equals_brute_force(orc):
    rng = np.random.default_rng(7)
    for _ in range(200):
        n_to = int(rng.integers(4, 13))
        n_from = int(rng.integers(0, n_to + 1))
        k_e = int(rng.integers(1, 5))
        a = rng.random(n_to).astype(np.float32)
        prev_pool = [j for j in range(n_from)]
        ge_prev = sorted(rng.choice(prev_pool, size=min(k_e, len(prev_pool)), replace=False).tolist()) if prev_pool else []
        got = orc.evict_update(a, ge_prev, n_from, n_to, k_e)
        want = brute_evict(a, set(ge_prev) | set(range(n_from, n_to)), k_e)
        assert got.tolist() == want


def test_ties_go_to_lowest_block_id(orc):
    a = np.full(10, 0.5, dtype=np.float32)
    assert orc.evict_update(a, [], 0, 10, 3).tolist() == [0, 1, 2]
    assert orc.evict_update(a, [7, 8, 9], 10, 10, 2).tolist() == [7, 8]
    s = np.zeros(10)
    s[[3, 6, 8]] = 1.0
    assert orc.select(s, [], [], True, 2, 0).tolist() == [3, 6]
    assert orc.select(np.zeros(10), [9], [], True, 3, 0).tolist() == [0, 1, 2, 9]


def test_signed_zeros_are_equal_scores(orc):
    """-0.0 and +0.0 are the same value: their order falls to the block ids."""
    a = np.array([0.0, -0.0, 0.0, -0.0, 1.0, -0.0], dtype=np.float32)
    assert orc.evict_update(a, [], 0, 6, 3).tolist() == [0, 1, 4]
    a2 = np.array([-0.0, 0.0, -0.0, 0.0, 1.0, 0.0], dtype=np.float32)
    assert orc.evict_update(a2, [], 0, 6, 3).tolist() == [0, 1, 4]
    s = np.array([-0.0, 0.0, -0.0, 2.0, 0.0])
    assert orc.select(s, [], [], True, 2, 0).tolist() == [0, 3]
    assert orc.select(-s, [], [], True, 2, 0).tolist() == [0, 1]


def test_no_agnostic_no_cap_is_plain_topk(orc):
    rng = np.random.default_rng(8)
    for _ in range(50):
        n = int(rng.integers(20, 200))
        k = int(rng.integers(1, 20))
        s = rng.standard_normal(n)
        prev = sorted(rng.choice(n, size=k, replace=False).tolist())
        got = orc.select(s, [], prev, False, k, k)  # c_max = k: no cap
        want = np.sort(np.argsort(-s, kind="stable")[:k])
        assert got.tolist() == want.tolist()
        got0 = orc.select(s, [], [], True, k, 0)
        assert got0.tolist() == want.tolist()


def _drive(orc, rng, n, k_q, k_e, m, steps, closing=False, C_slots=0):
    """Random-score trajectory through evict/select/plan, returning per-step records."""
    k = k_q + k_e
    a = rng.random(n + steps).astype(np.float32)
    ge, prev, n_cur, n_last = [], [], n, 0
    cache = orc.Cache(C_slots) if C_slots else None
    recs = []
    for t in range(steps):
        if closing and t > 0 and rng.random() < 0.3:
            n_cur += 1
        s = rng.standard_normal(n_cur)
        first = t == 0
        ge_new = orc.evict_update(a[:n_cur], [] if first else ge, 0 if first else n_last, n_cur, k_e)
        n_last = n_cur
        sel = orc.select(s, ge_new, prev, first, k_q, k - m)
        rec = dict(t=t, sel=sel, ge=ge_new, ge_prev=list(ge), prev=list(prev), n=n_cur)
        if cache is not None:
            res_before = set(cache.resident().tolist())
            fetch, slots = cache.plan(sel, t)
            rec.update(fetch=fetch, res_before=res_before, res_after=set(cache.resident().tolist()))
        recs.append(rec)
        ge, prev = ge_new.tolist(), sel.tolist()
    return recs


@pytest.mark.parametrize("closing", [False, True])
def test_selection_invariants(orc, closing):
    """Overlap >= m (gamma0), |S| = k, Gamma_e never readmits an evicted block,
    gamma(t) >= k_e / k (App. E)."""
    rng = np.random.default_rng(9)
    for trial in range(20):
        n, k_q, k_e = 64, 12, 4
        k = k_q + k_e
        m = 13
        recs = _drive(orc, rng, n, k_q, k_e, m, 60, closing=closing)
        ever_out = set()
        for r in recs:
            S = set(r["sel"].tolist())
            assert len(S) == k
            assert set(r["ge"].tolist()) <= S
            ge_prev = set(r["ge_prev"])
            # eviction: nothing that ever left Gamma_e comes back
            assert not (set(r["ge"].tolist()) & ever_out)
            if r["t"] > 0:
                ever_out |= ge_prev - set(r["ge"].tolist())
                prev = set(r["prev"])
                e_new = len(set(r["ge"].tolist()) - prev)
                assert len(S & prev) >= min(m, k - e_new)
                if e_new == 0:
                    assert len(S & prev) >= k_e  # App. E guarantee
                    assert len(S & prev) / k >= k_e / k


# --------------------------------------------------------------- a4 cache

def test_cache_hand_worked_lru_example(orc):
    """C = 3 slots; selections of 2 blocks; the expected fetch lists, slots and
    resident sets below follow the replacement rule by hand."""
    c = orc.Cache(3)
    f, s = c.plan([1, 2], 0)
    assert f.tolist() == [1, 2] and s.tolist() == [0, 1]
    f, s = c.plan([2, 3], 1)
    assert f.tolist() == [3] and s.tolist() == [2]
    assert c.resident().tolist() == [1, 2, 3]
    f, s = c.plan([3, 4], 2)          # evict 1 (last used at step 0)
    assert f.tolist() == [4] and s.tolist() == [0]
    assert c.resident().tolist() == [2, 3, 4]
    f, s = c.plan([1, 2], 3)          # 3 and 4 both last used at 2: evict the lower id, 3
    assert f.tolist() == [1] and s.tolist() == [2]
    assert c.resident().tolist() == [1, 2, 4]
    f, s = c.plan([0, 5], 4)          # victims in order 4 (step 2), 1 (step 3), 2 (step 3)
    assert f.tolist() == [0, 5] and s.tolist() == [0, 2]
    assert c.resident().tolist() == [0, 2, 5]
    f, s = c.plan([0, 2], 5)          # all hits
    assert f.tolist() == [] and c.resident().tolist() == [0, 2, 5]


def naive_lru(steps_sel, C_slots):
    """Independent model: a dict block -> last step, capacity C."""
    last = {}
    out = []
    for t, sel in enumerate(steps_sel):
        S = set(sel)
        misses = sorted(b for b in S if b not in last)
        for b in S:
            if b in last:
                last[b] = t
        for b in misses:
            if len(last) >= C_slots:
                victim = min((lu, bb) for bb, lu in last.items() if bb not in S)[1]
                del last[victim]
            last[b] = t
        out.append((misses, sorted(last)))
    return out


def test_cache_matches_naive_model_and_invariants(orc):
    rng = np.random.default_rng(10)
    for trial in range(10):
        C_slots = int(rng.choice([16, 17, 32, 48]))
        recs = _drive(orc, rng, 64, 12, 4, 13, 80, C_slots=C_slots)
        model = naive_lru([r["sel"].tolist() for r in recs], C_slots)
        for r, (misses, resident) in zip(recs, model):
            S = set(r["sel"].tolist())
            assert r["fetch"].tolist() == misses
            assert sorted(r["res_after"]) == resident
            assert S <= r["res_after"]
            assert len(r["res_after"]) <= C_slots
            evicted = r["res_before"] - r["res_after"]
            assert not (evicted & S)                 # only unused blocks swapped out
            assert set(r["fetch"].tolist()) == S - r["res_before"]
            if r["t"] > 0:
                assert len(r["fetch"]) <= len(S - set(r["prev"]))


def test_cache_too_small_is_an_error(orc):
    c = orc.Cache(2)
    with pytest.raises(ValueError):
        c.plan([1, 2, 3], 0)


# --------------------------------------------------------------- a6 attention

def _rand_bf16(rng, shape, scale=1.0):
    return inputs.f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def test_attention_dense_equals_sdpa(orc):
    rng = np.random.default_rng(11)
    G, d, T = 4, 128, 320
    q, K, V = _rand_bf16(rng, (G, d)), _rand_bf16(rng, (T, d)), _rand_bf16(rng, (T, d))
    got = orc.attend(q, K, V, list(range(T)))
    qt = torch.from_numpy(bits_to_f64(q)).view(1, G, 1, d)
    kt = torch.from_numpy(bits_to_f64(K)).view(1, 1, T, d).expand(1, G, T, d)
    vt = torch.from_numpy(bits_to_f64(V)).view(1, 1, T, d).expand(1, G, T, d)
    want = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).view(G, d).numpy()
    assert np.allclose(got, want, rtol=1e-12, atol=1e-12)


def test_attention_closed_forms(orc):
    rng = np.random.default_rng(12)
    G, d, T = 2, 128, 128
    q, K = _rand_bf16(rng, (G, d)), _rand_bf16(rng, (T, d))
    V = np.tile(_rand_bf16(rng, (1, d)), (T, 1))
    got = orc.attend(q, K, V, list(range(T)))
    assert np.allclose(got, np.tile(bits_to_f64(V[0]), (G, 1)), rtol=0, atol=1e-14)
    # one key aligned with q and scaled 1e3 takes all the weight
    K2 = K.copy()
    V2 = _rand_bf16(rng, (T, d))
    K2[17] = inputs.f32_to_bf16_bits((bits_to_f64(q[0]) * 1000.0).astype(np.float32))
    out = orc.attend(q[:1], K2, V2, list(range(T)))
    assert np.allclose(out[0], bits_to_f64(V2[17]), atol=1e-9)
    # only the listed rows take part
    rows = [5, 9, 40]
    sub = orc.attend(q, K, V2, rows)
    dense = orc.attend(q, K[rows], V2[rows], [0, 1, 2])
    assert np.array_equal(sub, dense)


# --------------------------------------------------------------- trajectories

def test_tiny_trajectory_invariants(orc):
    w = configs.get("tiny")
    d = inputs.generate(w)
    cfg = orc.cfg_from_workload(w)
    k, c_max = w.k, w.k - w.min_overlap
    for u in range(w.units):
        r = orc.run_unit(cfg, d["k"][u], d["v"][u], d["a"][u], d["q"][u])
        assert np.all(r.nsel == k)
        assert np.all(r.overlap[1:] >= w.min_overlap)
        assert r.nfetch[0] == k  # cold cache
        for t in range(1, w.steps):
            assert r.nfetch[t] <= c_max
            S = set(r.sel[t].tolist())
            res = set(r.resident[t][r.resident[t] >= 0].tolist())
            assert S <= res and len(res) <= w.cache_slots
            assert set(r.fetch[t][: r.nfetch[t]].tolist()) <= S - set(r.sel[t - 1].tolist())
        assert np.all(np.isfinite(r.o))


@pytest.mark.parametrize("append", [False, True])
def test_budget_covering_all_blocks_is_dense_attention(orc, append):
    """When k equals the number of blocks, every step attends every token (plus
    the open tail), so the output is dense softmax attention."""
    rng = np.random.default_rng(13)
    G, d, P, n0, steps = 4, 128, 64, 6, 70 if append else 5
    max_blocks = n0 + (2 if append else 0)
    T = max_blocks * P
    K, V = _rand_bf16(rng, (T, d)), _rand_bf16(rng, (T, d))
    a = rng.random(max_blocks).astype(np.float32)
    q = _rand_bf16(rng, (steps, G, d))
    # k = n0 blocks; once a block closes n > k, so only check steps before that
    cfg = orc.make_cfg(G, d, P, 16, n0, 0, max_blocks, 4, 2, 0, 0, steps, append)
    r = orc.run_unit(cfg, K, V, a, q)
    for t in range(min(steps, 64)):
        tokens = n0 * P + (t + 1 if append else 0)
        qt = torch.from_numpy(bits_to_f64(q[t])).view(1, G, 1, d)
        kt = torch.from_numpy(bits_to_f64(K[:tokens])).view(1, 1, tokens, d).expand(1, G, tokens, d)
        vt = torch.from_numpy(bits_to_f64(V[:tokens])).view(1, 1, tokens, d).expand(1, G, tokens, d)
        want = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt).view(G, d).numpy()
        assert np.allclose(r.o[t], want, rtol=1e-12, atol=1e-12), t


def test_long_generation_closes_blocks(orc):
    """With appends, a block closes every P steps; it becomes a candidate at the
    next step and may enter Gamma_e (at most one new agnostic block per step)."""
    rng = np.random.default_rng(14)
    G, d, P, n0, steps = 2, 128, 64, 20, 200
    max_blocks = n0 + 4
    K, V = _rand_bf16(rng, (max_blocks * P, d)), _rand_bf16(rng, (max_blocks * P, d))
    a = rng.random(max_blocks).astype(np.float32)
    a[n0:] = 2.0  # closing blocks outrank every prompt block
    q = _rand_bf16(rng, (steps, G, d))
    cfg = orc.make_cfg(G, d, P, 16, n0, 0, max_blocks, 6, 4, 7, 20, steps, True)
    r = orc.run_unit(cfg, K, V, a, q, attend_steps=[])
    for t in range(steps):
        S = set(r.sel[t].tolist())
        n_closed = n0 + t // P  # blocks closed before step t's selection
        assert max(S) < n_closed
        if t >= P:
            # the most recently closed block (agnostic score 2.0) is selected
            assert (n_closed - 1) in S
        if t > 0:
            assert r.overlap[t] >= 7


# --------------------------------------------------------------- the pages' budget

def test_paper_budget_fixture(orc):
    g = json.load(open(os.path.join(HERE, "golden", "paper_budget.json")))
    P = g["transfer_block_bytes"] // (g["d_kv"] * 2)
    assert P == 64  # a 16 KiB bf16 block at d_kv = 128 holds 64 tokens
    assert g["k_tokens"] // P == g["query_aware_blocks"] + g["agnostic_blocks"]
    assert g["k_q_tokens"] // P == g["query_aware_blocks"]
    assert g["infllmv2_sink_blocks"] + g["infllmv2_window_blocks"] + g["infllmv2_dynamic_blocks"] == g["k_tokens"] // P
    # App. E with the paper's split: no gamma0 cap beyond the split itself
    rng = np.random.default_rng(15)
    k_q, k_e = g["query_aware_blocks"], g["agnostic_blocks"]
    k = k_q + k_e
    recs = _drive(orc, rng, 256, k_q, k_e, 0, 40)
    for r in recs[1:]:
        ov = len(set(r["sel"].tolist()) & set(r["prev"]))
        assert ov >= k_e
        assert ov / k >= g["locality_lower_bound"]


# --------------------------------------------------------------- forced blocks (sink, window)

def brute_select_forced(score, n, F, E, prev, first, k_q, c_max):
    F, E, prev = set(F), set(E), set(prev)
    fixed = F | E
    avail = [j for j in range(n) if j not in fixed]
    new = set(j for j in avail if j not in prev)
    c_t = 10 ** 9 if first else max(0, c_max - len(fixed - prev))
    for r in range(min(k_q, len(avail)), -1, -1):
        best, best_set = None, None
        for comb in itertools.combinations(avail, r):
            if not first and len(new.intersection(comb)) > c_t:
                continue
            val = sum(score[j] for j in comb)
            if best is None or val > best:
                best, best_set = val, comb
        if best_set is not None:
            return sorted(fixed | set(best_set))
    return sorted(fixed)


def test_forced_blocks_definition(orc):
    assert orc.forced_blocks(10, 1, 3).tolist() == [0, 7, 8, 9]
    assert orc.forced_blocks(10, 0, 0).tolist() == []
    assert orc.forced_blocks(3, 1, 4).tolist() == [0, 1, 2]   # sink and window overlap


def test_select_with_forced_blocks_equals_brute_force(orc):
    rng = np.random.default_rng(16)
    cases = 0
    while cases < 200:
        n = int(rng.integers(8, 13))
        sink, window = int(rng.integers(0, 2)), int(rng.integers(0, 3))
        F = orc.forced_blocks(n, sink, window).tolist()
        k_e_dyn = int(rng.integers(0, 3))
        k_q = int(rng.integers(1, 4))
        free = [j for j in range(n) if j not in F]
        if len(free) < k_e_dyn + k_q:
            continue
        E = sorted(rng.choice(free, size=k_e_dyn, replace=False).tolist())
        k = len(F) + k_e_dyn + k_q
        c_max = int(rng.integers(0, k + 1))
        first = bool(rng.random() < 0.2)
        prev = [] if first else sorted(rng.choice(n, size=min(k, n), replace=False).tolist())
        score = rng.standard_normal(n)
        got = orc.select_forced(score, F, E, prev, first, k_q, c_max)
        assert got.tolist() == brute_select_forced(score, n, F, E, prev, first, k_q, c_max)
        cases += 1


def _run_policy(orc, n0, steps, k_q, k_e, m, sink, window, append, seed):
    rng = np.random.default_rng(seed)
    G, d, P = 2, 128, 64
    max_blocks = n0 + (steps + P - 1) // P + 1 if append else n0
    K = _rand_bf16(rng, (max_blocks * P, d))
    V = _rand_bf16(rng, (max_blocks * P, d))
    a = rng.random(max_blocks).astype(np.float32)
    q = _rand_bf16(rng, (steps, G, d))
    cfg = orc.make_cfg(G, d, P, 16, n0, 0, max_blocks, k_q, k_e, m, 0, steps, append, sink, window)
    return orc.run_unit(cfg, K, V, a, q, attend_steps=[], want_scores=True), max_blocks


def test_sliding_window_invariants_with_closing_blocks(orc):
    """The sink and the last `window` closed blocks are in every S(t); the
    window slides as blocks close; |S| = k; overlap >= m whenever the new
    forced and agnostic blocks fit in the allowance."""
    n0, steps, sink, window, k_q, k_e, m = 40, 300, 1, 6, 8, 12, 16
    r, _ = _run_policy(orc, n0, steps, k_q, k_e, m, sink, window, True, 17)
    k = k_q + k_e
    for t in range(steps):
        n = n0 + t // 64  # blocks closed before step t's selection
        S = set(r.sel[t].tolist())
        assert len(S) == k
        assert set(orc.forced_blocks(n, sink, window).tolist()) <= S
        if t > 0:
            assert r.overlap[t] >= min(m, k - 2)


def test_infllmv2_policy_is_forced_plus_plain_topk(orc):
    """Sink + window + the query-aware top-k of the rest, with no agnostic set
    and no overlap floor, is what InfLLMv2 selects (paperlayer summary,
    App. B.2.2: 1 sink block, 16 window blocks, 47 dynamic blocks)."""
    n0, steps = 200, 12
    r, _ = _run_policy(orc, n0, steps, 47, 17, 0, 1, 16, False, 18)
    F = set(orc.forced_blocks(n0, 1, 16).tolist())
    for t in range(steps):
        s = r.scores[t][:n0]
        rest = np.array([j for j in range(n0) if j not in F])
        top = rest[np.argsort(-s[rest], kind="stable")[:47]]
        assert r.sel[t].tolist() == sorted(F | set(top.tolist()))


def test_paper_split_with_sink_and_window_keeps_75_percent(orc):
    """NOSA's own budget (App. B.2.2): 16 query-aware + 48 agnostic blocks, the
    48 counting one sink and 16 window blocks; App. E: consecutive selections
    share at least k_e = 48 of the 64 blocks."""
    g = json.load(open(os.path.join(HERE, "golden", "paper_budget.json")))
    r, _ = _run_policy(orc, 256, 40, g["query_aware_blocks"], g["agnostic_blocks"], 0,
                       g["infllmv2_sink_blocks"], g["infllmv2_window_blocks"], False, 19)
    for t in range(1, 40):
        assert r.overlap[t] >= g["agnostic_blocks"]
        assert r.overlap[t] / 64 >= g["locality_lower_bound"]


def test_block_leaving_the_window_joins_the_agnostic_pool(orc):
    """A block that slides out of the window becomes eligible for Gamma_e; with
    the highest agnostic score it is selected at every later step."""
    rng = np.random.default_rng(20)
    G, d, P, n0, steps = 2, 128, 64, 10, 190
    max_blocks = 14
    K = _rand_bf16(rng, (max_blocks * P, d))
    V = _rand_bf16(rng, (max_blocks * P, d))
    a = np.full(max_blocks, 0.1, dtype=np.float32)
    a[10] = 2.0  # block 10 closes at step 63 and leaves the 1-block window at step 128
    q = _rand_bf16(rng, (steps, G, d))
    cfg = orc.make_cfg(G, d, P, 16, n0, 0, max_blocks, 3, 2, 0, 0, steps, True, 0, 1)
    r = orc.run_unit(cfg, K, V, a, q, attend_steps=[])
    for t in range(64, 128):
        assert 10 in r.sel[t].tolist()          # in the window
    for t in range(128, steps):
        assert 10 in r.sel[t].tolist()          # now through Gamma_e
        assert 11 in r.sel[t].tolist()          # the new window block


# ---------------------------------------------------------------- row transfer

def test_gather_rows_hand_example(orc):
    """Rows move by their indices, source and destination not swapped."""
    src = np.array([[1, 2], [3, 4], [5, 6]], dtype=np.uint8)
    dst = np.zeros((4, 2), dtype=np.uint8)
    got = orc.gather_rows(src, [2, 0], dst, [1, 3])
    assert got.tolist() == [[0, 0], [5, 6], [0, 0], [1, 2]]
    assert dst.sum() == 0  # the input is not modified
    assert orc.gather_rows(src, [1, 2], dst).tolist() == [[3, 4], [5, 6], [0, 0], [0, 0]]


def test_gather_rows_skips_out_of_range(orc):
    src = np.arange(6, dtype=np.uint8).reshape(3, 2)
    dst = np.full((2, 2), 9, dtype=np.uint8)
    got = orc.gather_rows(src, [3, -1, 0], dst, [0, 1, 5])
    assert got.tolist() == [[9, 9], [9, 9]]


def test_block_rows_equal_their_token_rows(orc):
    """A 64-token block row is the same bytes as its 64 token rows: moving a
    block whole or token by token yields the same cache."""
    rng = np.random.default_rng(3)
    tok = rng.integers(0, 256, size=(4 * 64, 256), dtype=np.uint8)   # 4 blocks of 64 tokens
    blk = tok.reshape(4, 64 * 256)
    cache_b = orc.gather_rows(blk, [2, 0], np.zeros((2, 64 * 256), np.uint8))
    tok_idx = [2 * 64 + i for i in range(64)] + [i for i in range(64)]
    cache_t = orc.gather_rows(tok, tok_idx, np.zeros((128, 256), np.uint8))
    assert np.array_equal(cache_b.reshape(128, 256), cache_t)
