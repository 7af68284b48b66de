"""The five synthetic NOSA decode workloads.

Each workload is a batch of decoding sequences over one attention layer.  A
*unit* is one (sequence b, KV head g) pair, laid out u = b * n_kv_heads + g.
Every size below is a plain parameter: nothing here is derived from the
method's arithmetic, and both the CUDA path and the CPU oracle receive these
integers as inputs.

Budget notation (NOSA: Native and Offloadable Sparse Attention, paperlayer
summary, §3.1 and App. A): the selection budget is k = k_q + k_e blocks, k_q of
them query-aware and k_e query-agnostic.  The minimum overlap with the previous
step's selection is gamma0; it is handed to the library as the integer
m = ceil(gamma0 * k), written out literally below (16 * 0.8 = 12.8 -> 13,
64 * 0.8 = 51.2 -> 52, 64 * 0.85 = 54.4 -> 55).
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    context: int            # prompt tokens present at attach time
    k_query: int            # k_q
    k_agnostic: int         # k_e
    gamma0: float           # documented value; the library takes min_overlap
    min_overlap: int        # m = ceil(gamma0 * k), literal
    steps: int              # decode steps
    rho: float              # AR(1) coefficient of the queries
    sigma: float            # AR(1) innovation scale
    offloaded: bool         # KV in pinned host memory (True) or resident in HBM
    cache_factor: int       # GPU cache slots per unit = cache_factor * k (offloaded)
    append: bool = False    # one new token per step is appended (growing tail)
    resample_every: int = 0  # queries replaced by fresh N(0,1) every this many steps
    planted_blocks: int = 0  # blocks per unit whose keys are scaled
    planted_scale: float = 1.0
    sink_blocks: int = 0     # forced: the first closed blocks (attention sink)
    window_blocks: int = 0   # forced: the last closed blocks (sliding window)
    head_dim: int = 128
    block: int = 64         # P, tokens per block
    sub_block: int = 16     # Q, tokens per pooled sub-block
    seed: int = 0

    # ---- derived sizes (plain bookkeeping) ----
    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def units(self) -> int:
        return self.batch * self.n_kv_heads

    @property
    def k(self) -> int:
        return self.k_query + self.k_agnostic

    @property
    def n_blocks0(self) -> int:
        """Closed blocks at attach time."""
        return self.context // self.block

    @property
    def tail0(self) -> int:
        """Tokens of the open tail block at attach time."""
        return self.context % self.block

    @property
    def max_tokens(self) -> int:
        """Token capacity per unit (prompt plus every appended token)."""
        t = self.context + (self.steps if self.append else 0)
        return int(math.ceil(t / self.block)) * self.block

    @property
    def max_blocks(self) -> int:
        return self.max_tokens // self.block

    @property
    def cache_slots(self) -> int:
        return self.cache_factor * self.k if self.offloaded else 0

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _sigma(rho: float) -> float:
    return math.sqrt(1.0 - rho * rho)


WORKLOADS: Dict[str, Workload] = {
    # Tiny decode: parity case, run both resident and offloaded.
    "tiny": Workload(
        name="tiny", batch=1, n_q_heads=8, n_kv_heads=2, context=4096,
        k_query=12, k_agnostic=4, gamma0=0.8, min_overlap=13, steps=16,
        rho=0.9, sigma=0.44, offloaded=True, cache_factor=2),
    # 8B-shaped decode layer, all KV resident in HBM, 8 planted x3 blocks per unit.
    "layer8b": Workload(
        name="layer8b", batch=16, n_q_heads=32, n_kv_heads=8, context=16384,
        k_query=48, k_agnostic=16, gamma0=0.8, min_overlap=52, steps=128,
        rho=0.95, sigma=_sigma(0.95), offloaded=False, cache_factor=0,
        planted_blocks=8, planted_scale=3.0),
    # Offloaded batch decode at B=64: the throughput workload.
    "offload_b64": Workload(
        name="offload_b64", batch=64, n_q_heads=32, n_kv_heads=8, context=4096,
        k_query=12, k_agnostic=4, gamma0=0.8, min_overlap=13, steps=256,
        rho=0.95, sigma=_sigma(0.95), offloaded=True, cache_factor=2),
    # Long input (64K), offloaded, cache 4x budget, query resampled every 32 steps.
    "long_input": Workload(
        name="long_input", batch=8, n_q_heads=16, n_kv_heads=4, context=65536,
        k_query=48, k_agnostic=16, gamma0=0.85, min_overlap=55, steps=128,
        rho=0.9, sigma=_sigma(0.9), offloaded=True, cache_factor=4,
        resample_every=32),
    # Long generation: 16K prompt growing by one token per step for 2048 steps.
    "long_gen": Workload(
        name="long_gen", batch=32, n_q_heads=32, n_kv_heads=8, context=16384,
        k_query=48, k_agnostic=16, gamma0=0.8, min_overlap=52, steps=2048,
        rho=0.97, sigma=_sigma(0.97), offloaded=True, cache_factor=2,
        append=True),
}

ORDER = ["tiny", "layer8b", "offload_b64", "long_input", "long_gen"]


def get(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return w.with_(**overrides) if overrides else w


def describe(w: Workload) -> str:
    mode = "offloaded" if w.offloaded else "resident"
    return (f"{w.name}: B={w.batch} Hq/Hkv={w.n_q_heads}/{w.n_kv_heads} ctx={w.context} "
            f"n={w.n_blocks0} k={w.k}({w.k_query}+{w.k_agnostic}) m={w.min_overlap} "
            f"steps={w.steps} {mode}" + (f" C={w.cache_slots}" if w.offloaded else "")
            + (" append" if w.append else ""))


# Selection policies on the same kernels (NOSA: Native and Offloadable Sparse
# Attention, paperlayer summary, App. B.2.2, for a 64-block = 4096-token budget):
#   nosa     -- the workload's own split and overlap floor
#   paper    -- NOSA's own split: 16 query-aware + 48 agnostic blocks, the 48
#               counting one sink block and 16 sliding-window blocks, no floor
#               beyond what the split guarantees (App. E: 48 of 64)
#   infllmv2 -- 1 sink + 16 window + 47 query-aware blocks, no agnostic set,
#               no overlap floor
#   full     -- every closed block, KV resident (dense attention)
POLICIES = ("nosa", "paper", "infllmv2", "full")


def with_policy(w: Workload, policy: str, k_query: Optional[int] = None) -> Workload:
    """k_query (paper policy only) moves the query-aware share of the 64-block
    budget; the rest stays query-agnostic, sink and window included."""
    if policy == "nosa":
        return w
    if policy == "paper":
        kq = 16 if k_query is None else int(k_query)
        if not 0 <= kq <= 64 - 17:
            raise ValueError("the paper split keeps 1 sink + 16 window blocks: k_query in [0, 47]")
        return w.with_(name=f"{w.name}/paper" + ("" if k_query is None else f"-kq{kq}"), k_query=kq,
                       k_agnostic=64 - kq, sink_blocks=1, window_blocks=16, min_overlap=0, gamma0=0.0)
    if policy == "infllmv2":
        return w.with_(name=f"{w.name}/infllmv2", k_query=47, k_agnostic=17, sink_blocks=1, window_blocks=16,
                       min_overlap=0, gamma0=0.0)
    if policy == "full":
        if w.append:
            raise ValueError("the dense policy covers fixed-length workloads")
        return w.with_(name=f"{w.name}/full", k_query=w.n_blocks0, k_agnostic=0, min_overlap=0, gamma0=0.0,
                       offloaded=False, cache_factor=0)
    raise ValueError(f"unknown policy {policy!r}")
