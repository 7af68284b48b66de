"""GPU parity where the selection has to break ties.

The rule (NOSA: Native and Offloadable Sparse Attention, paperlayer summary,
§2.1 and §3.1; ties read as "the lower block id wins"): query-aware scores are
ordered by fp64 value, agnostic scores by fp32 value, and equal values by
ascending block id; -0.0 and +0.0 are equal values.  Seeded N(0,1) and U(0,1)
inputs almost never tie at a selection boundary, so these tests plant ties:

- blocks whose keys are copies of another block's keys (equal pooled keys,
  hence bit-equal scores on both sides), four copies of each key pattern, so
  the top-k_q and top-c boundaries fall inside groups of equal scores;
- agnostic scores drawn from a handful of values, with signed zeros at the
  Gamma_e boundary.

Each case runs every unit and every step through the C ABI and the oracle and
asks for bit-exact S(t), fetch lists and resident sets.  It also checks, on the
oracle's own scores, that ties did sit on a boundary, so the case cannot pass
vacuously.
"""

import numpy as np
import pytest

import oracle
from kv_cache_decode_step_b200 import configs, inputs
from gpu_harness import check_all_unit_invariants, compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


def plant_key_copies(w, data, copies=4, seed=1):
    """Every block j of every unit takes the keys of template block
    perm[j // copies] (the templates are a random quarter of the blocks);
    values stay as drawn.  Blocks closed by appends are left alone."""
    rng = np.random.default_rng(seed)
    n = w.n_blocks0
    P = w.block
    for u in range(w.units):
        order = rng.permutation(n)
        templates = order[: (n + copies - 1) // copies]
        K = data["k"][u]
        src = K[: n * P].reshape(n, P, -1).copy()
        for i, j in enumerate(order):
            K[j * P:(j + 1) * P] = src[templates[i // copies]]


def plant_agnostic_ties(w, data, seed=2):
    """Agnostic scores take one of 5 values; in every unit k_e - 1 blocks get
    1.0 and every other block a signed zero (alternating sign from a random
    start), so Gamma_e takes the lowest-id zero whatever its sign."""
    rng = np.random.default_rng(seed)
    a = data["a"]
    for u in range(w.units):
        m = a.shape[1]
        vals = rng.choice(np.array([0.25, 0.5, 0.75], np.float32), size=m)
        a[u] = vals
        if w.k_agnostic >= 1:
            top = rng.permutation(w.n_blocks0)[: max(0, w.k_agnostic - 1)]
            zeros = np.setdiff1d(np.arange(w.n_blocks0), top)
            sign = rng.integers(0, 2)
            for i, j in enumerate(zeros):
                a[u, j] = np.float32(-0.0) if (i + sign) % 2 else np.float32(0.0)
            a[u, top] = 1.0


def boundary_ties(w, data, units, steps):
    """Count (unit, step) pairs where a selected query-aware block ties in
    score with a block left out (from the oracle's own fp64 scores)."""
    cfg = oracle.cfg_from_workload(w, steps=steps)
    hits = 0
    for u in units:
        r = oracle.run_unit(cfg, data["k"][u], data["v"][u], data["a"][u], data["q"][u][:steps],
                            attend_steps=[], want_scores=True)
        for t in range(steps):
            n = w.n_blocks0
            sel = set(int(x) for x in r.sel[t][: r.nsel[t]])
            sc = r.scores[t][:n]
            chosen = {float(sc[j]) for j in sel}
            left = {float(sc[j]) for j in range(n) if j not in sel}
            hits += bool(chosen & left)
    return hits


def _run(w, data, cache_steps=None, fused=True):
    units = list(range(w.units))
    steps = list(range(w.steps))
    if cache_steps is None:
        cache_steps = steps
    rec = run_gpu(w, data, units, steps, cache_steps=cache_steps if w.offloaded else (), fused=fused)
    refs = run_oracle(w, data, units, steps)
    compare(w, rec, refs, units)
    check_all_unit_invariants(w, rec, w.steps)
    return rec


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("offloaded", [True, False])
def test_tied_scores_tiny(offloaded, fused):
    """n = 64: the fused kernel (fused=True) and the register selection kernel
    (fused=False) on groups of four equal scores."""
    w = configs.get("tiny", steps=24, resample_every=6)
    if not offloaded:
        w = w.with_(offloaded=False, cache_factor=0)
    data = inputs.generate(w)
    plant_key_copies(w, data)
    plant_agnostic_ties(w, data)
    assert boundary_ties(w, data, range(w.units), w.steps) > 0
    _run(w, data, fused=fused)


def test_tied_scores_long_input_shape_register_path():
    """n = 1024 blocks, budget 48 + 16 (the long-input shape with 2 sequences):
    the register selection with 32 rows per lane."""
    w = configs.get("long_input", batch=2, steps=20, resample_every=5)
    data = inputs.generate(w)
    plant_key_copies(w, data)
    plant_agnostic_ties(w, data)
    assert boundary_ties(w, data, [0], w.steps) > 0
    _run(w, data, cache_steps=[0, 5, w.steps - 1])


def test_tied_scores_beyond_the_register_path():
    """n = 1536 blocks (> 1024): the shared-memory selection kernel."""
    w = configs.get("long_input", batch=1, context=1536 * 64, steps=12, resample_every=4)
    data = inputs.generate(w)
    plant_key_copies(w, data)
    plant_agnostic_ties(w, data)
    assert boundary_ties(w, data, [0], w.steps) > 0
    _run(w, data, cache_steps=[0, 4, w.steps - 1])


def test_tied_agnostic_scores_with_growth():
    """Blocks closing during decoding join Gamma_e's pool with tied agnostic
    scores (signed zeros included): eviction ties go to the lower block id."""
    w = configs.get("long_gen", batch=1, context=100 * 64 + 40, steps=100)
    data = inputs.generate(w)
    plant_key_copies(w, data)
    a = data["a"]
    rng = np.random.default_rng(5)
    for u in range(w.units):
        a[u] = rng.choice(np.array([-0.0, 0.0, 0.5, 1.0], np.float32), size=a.shape[1])
    _run(w, data, cache_steps=[0, 23, 24, 88, w.steps - 1])
