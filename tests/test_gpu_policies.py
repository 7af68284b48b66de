"""GPU parity of the selection policies built on the same kernels: forced
sink / sliding-window blocks (NOSA's own split and InfLLMv2's), including a
window that slides as blocks close, and dense attention."""

import numpy as np
import pytest

from kv_cache_decode_step_b200 import configs, inputs
from gpu_harness import check_all_unit_invariants, compare, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


def _run(w, sample, attend, cache_steps=()):
    data = inputs.generate(w)
    rec = run_gpu(w, data, sample, attend, cache_steps=cache_steps)
    refs = run_oracle(w, data, sample, attend)
    err = compare(w, rec, refs, sample)
    print(f"{w.name}: max-abs {err[0]:.3e} mean-abs {err[1]:.3e} stats {rec.stats}")
    return rec


@pytest.mark.parametrize("offloaded", [True, False])
def test_tiny_with_sink_and_window(offloaded):
    w = configs.get("tiny", sink_blocks=1, window_blocks=2, steps=12)
    if not offloaded:
        w = w.with_(offloaded=False, cache_factor=0)
    rec = _run(w, range(w.units), range(w.steps), cache_steps=[0, 11])
    s = rec.sel_all_last
    assert np.all(s[:, 0] == 0) and np.all(s[:, -1] == w.n_blocks0 - 1) and np.all(s[:, -2] == w.n_blocks0 - 2)


def test_sliding_window_moves_as_blocks_close():
    w = configs.get("tiny", context=4096 + 40, steps=200, append=True, sink_blocks=1, window_blocks=3,
                    k_query=10, k_agnostic=6, min_overlap=12)
    rec = _run(w, range(w.units), range(0, w.steps, 7), cache_steps=[23, 24, 150])
    assert rec.stats["n_closed"] == 64 + 3


@pytest.mark.parametrize("policy", ["paper", "infllmv2", "full"])
def test_layer8b_policies(policy):
    w = configs.with_policy(configs.get("layer8b", steps=64), policy)
    rec = _run(w, [0, 57, 127], list(range(0, w.steps, 16)) + [w.steps - 1])
    check_all_unit_invariants(w, rec, w.steps)


@pytest.mark.parametrize("policy", ["paper", "infllmv2"])
def test_long_generation_policies(policy):
    w = configs.with_policy(configs.get("long_gen", steps=400), policy)
    rec = _run(w, [0, 131, 255], [0, 63, 64, 65, 200, 399], cache_steps=[64, 399])
    check_all_unit_invariants(w, rec, w.steps)
