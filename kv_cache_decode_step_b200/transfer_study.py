"""Block-wise against element-wise KV transfer over PCIe.

NOSA: Native and Offloadable Sparse Attention (paperlayer summary, §3.2)
compares moving selected KV as whole blocks with moving it token by token, at
batch 64 with 4096-token sequences, 128-dim keys and values and two KV heads, as locality rises;
§4 describes the block transfer as a zero-copy kernel over 16 KiB blocks.

This module measures both with one kernel (``nosa_gather_rows``) on the same
miss volume, and again with TMA bulk copies (``nosa_gather_rows_bulk``).  Per unit (sequence, KV head) the selection budget is 16 blocks
(1024 tokens, a quarter of the sequence); at locality gamma the step misses
(1 - gamma) * 1024 tokens, i.e. 8, 4, 2 or 1 blocks for gamma = 0.5, 0.75,
0.875, 0.9375.  Block-wise, each missed block is a 16 KiB row of K and one of
V; element-wise, the same number of tokens is missed at random positions of
the sequence and each token is a 256-byte row of K and one of V.  Rows of 4 and
16 tokens fill in the curve between the two.

    python -m kv_cache_decode_step_b200.transfer_study [--reps 20] [--json FILE]

Every launch is timed alone with CUDA events on its stream, after a write of
256 MiB that flushes L2, over ``reps`` different random miss sets.
"""

from __future__ import annotations

import argparse
import json
import statistics
import sys
import time

import numpy as np

from . import build, nosa

BATCH, KV_HEADS, SEQ, D = 64, 2, 4096, 128
UNITS = BATCH * KV_HEADS
TOKEN_BYTES = D * 2                 # one token's K (or V) row, bf16
BUDGET_TOKENS = 16 * 64             # k = 16 blocks of 64 tokens
GAMMAS = (0.5, 0.75, 0.875, 0.9375)
GRANULARITIES = (1, 4, 16, 64)      # tokens per transferred row
SUB_TOKEN_ROWS = (16, 32, 64, 128)  # bytes: pieces of one token's row


def miss_sets(rng, gamma: float, row_bytes: int, reps: int):
    """Source and destination rows for `reps` random miss sets: per unit,
    (1 - gamma) * 1024 missed tokens, moved as distinct aligned rows of
    row_bytes (a token is 256 bytes; rows below that split a token)."""
    m = int(round((1.0 - gamma) * BUDGET_TOKENS))
    runs = m * TOKEN_BYTES // row_bytes
    per_seq = SEQ * TOKEN_BYTES // row_bytes
    slots = BUDGET_TOKENS * TOKEN_BYTES // row_bytes
    out = []
    for _ in range(reps):
        chunk = np.stack([rng.choice(per_seq, size=runs, replace=False) for _ in range(UNITS)])  # [U, runs]
        u = np.arange(UNITS)[:, None]
        src = np.concatenate([(kv * UNITS + u) * per_seq + chunk for kv in (0, 1)]).reshape(-1)
        dst = np.concatenate([(kv * UNITS + u) * slots + np.arange(runs)[None, :] for kv in (0, 1)]
                             ).reshape(-1)
        out.append((src.astype(np.int64), dst.astype(np.int64)))
    return m, out


def time_gathers(torch, host, cache, sets, row_bytes: int, ctas: int, flush, stream, fn=None):
    fn = fn or nosa.nosa_gather_rows
    src_rows = host.numel() // row_bytes
    dst_rows = cache.numel() // row_bytes
    dev_sets = [(torch.from_numpy(s).cuda(), torch.from_numpy(d).cuda()) for s, d in sets]
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    ms = []
    with torch.cuda.stream(stream):
        for i in range(3 + len(dev_sets)):        # 3 untimed launches first
            s, d = dev_sets[i % len(dev_sets)]
            flush.fill_(i & 0xFF)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn(host, src_rows, cache, dst_rows, row_bytes, s, d, s.numel(), ctas, flags, stream)
            e1.record(stream)
            if i >= 3:
                ms.append((e0, e1))
    stream.synchronize()
    if flags.item() != 0:
        raise RuntimeError("row gather reported an out-of-range index")
    return [a.elapsed_time(b) for a, b in ms]


def torch_index_copy(torch, host, sets, row_bytes: int, reps: int):
    """Context only: the obvious PyTorch route for element-wise transfer (index
    the pinned host tensor on the CPU, then one host-to-device copy)."""
    rows = host.view(-1, row_bytes)
    t = []
    for s, _ in sets[:reps]:
        idx = torch.from_numpy(s)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        staged = rows.index_select(0, idx)
        staged.to("cuda", non_blocking=False)
        torch.cuda.synchronize()
        t.append((time.perf_counter() - t0) * 1e3)
    return t


def main(argv=None) -> int:
    p = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    p.add_argument("--reps", type=int, default=20)
    p.add_argument("--json", default=None, help="also write the rows to this file")
    p.add_argument("--seed", type=int, default=0)
    args = p.parse_args(argv)

    import torch
    build.build()
    if not torch.cuda.is_available():
        raise RuntimeError("the transfer study needs a GPU")
    props = torch.cuda.get_device_properties(0)
    sms = props.multi_processor_count
    rng = np.random.default_rng(args.seed)

    host = torch.empty(2 * UNITS * SEQ * TOKEN_BYTES, dtype=torch.uint8).pin_memory()
    host.view(torch.int32).random_(generator=torch.Generator().manual_seed(args.seed))
    cache = torch.zeros(2 * UNITS * BUDGET_TOKENS * TOKEN_BYTES, dtype=torch.uint8, device="cuda")
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()

    # host-to-device ceiling of this link: one large pinned copy
    big = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for _ in range(2):
        big.copy_(host[: 256 << 20], non_blocking=True)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(4):
        big.copy_(host[: 256 << 20], non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    h2d = 4 * (256 << 20) / (e0.elapsed_time(e1) * 1e-3) / 1e9
    del big

    rows = []

    def record(kind, gamma, row_bytes, ctas, m, ms):
        nbytes = 2 * UNITS * m * TOKEN_BYTES
        med = statistics.median(ms)
        r = {"kind": kind, "gamma": gamma, "tokens_per_row": row_bytes / TOKEN_BYTES, "row_bytes": row_bytes,
             "ctas": ctas,
             "missed_tokens_per_unit": m, "bytes": nbytes, "median_us": med * 1e3,
             "min_us": min(ms) * 1e3, "gbs": nbytes / (med * 1e-3) / 1e9, "of_h2d_copy": None}
        r["of_h2d_copy"] = r["gbs"] / h2d
        rows.append(r)
        print(json.dumps(r), flush=True)

    default_ctas = (sms + 3) // 4
    for gamma in GAMMAS:
        for g in GRANULARITIES:
            rb = g * TOKEN_BYTES
            m, sets = miss_sets(rng, gamma, rb, args.reps)
            record("gather_rows", gamma, rb, default_ctas, m,
                   time_gathers(torch, host, cache, sets, rb, default_ctas, flush, stream))
            record("gather_rows_bulk", gamma, rb, default_ctas, m,
                   time_gathers(torch, host, cache, sets, rb, default_ctas, flush, stream,
                                nosa.nosa_gather_rows_bulk))
    # the TMA bulk arm at other grid widths (block rows and token rows)
    for g in (1, 64):
        rb = g * TOKEN_BYTES
        m, sets = miss_sets(rng, 0.75, rb, args.reps)
        for ctas in (default_ctas // 2, 2 * default_ctas, sms, 2 * sms):
            record("gather_rows_bulk", 0.75, rb, ctas, m,
                   time_gathers(torch, host, cache, sets, rb, ctas, flush, stream, nosa.nosa_gather_rows_bulk))
    # rows below one token: where does the request size start to cost?
    for rb in SUB_TOKEN_ROWS:
        m, sets = miss_sets(rng, 0.75, rb, args.reps)
        for ctas in (default_ctas, 4 * sms):
            record("gather_rows", 0.75, rb, ctas, m, time_gathers(torch, host, cache, sets, rb, ctas, flush, stream))
    # grid width: does more parallelism rescue small rows?
    for g in (1, 64):
        rb = g * TOKEN_BYTES
        m, sets = miss_sets(rng, 0.75, rb, args.reps)
        for ctas in (default_ctas // 2, 2 * default_ctas, sms, 2 * sms, 4 * sms):
            record("gather_rows", 0.75, rb, ctas, m, time_gathers(torch, host, cache, sets, rb, ctas, flush, stream))
    # context: PyTorch index + copy, token rows and block rows
    for g in (1, 64):
        rb = g * TOKEN_BYTES
        m, sets = miss_sets(rng, 0.75, rb, min(args.reps, 5))
        record("torch_index_select_then_copy", 0.75, rb, 0, m, torch_index_copy(torch, host, sets, rb, 5))

    summary = {"h2d_copy_gbs": h2d, "sms": sms, "device": props.name, "units": UNITS, "seq": SEQ,
               "budget_tokens": BUDGET_TOKENS, "rows": rows}
    if args.json:
        with open(args.json, "w") as f:
            json.dump(summary, f, indent=1)
    print(json.dumps({"h2d_copy_gbs": h2d}), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
