"""Row gather at block and token granularity (NOSA: Native and Offloadable
Sparse Attention, paperlayer summary, §3.2 and §4) against the oracle's row
transfer: bit-exact, from pinned host memory and from device memory, through
SM loads (nosa_gather_rows) and through TMA bulk copies (nosa_gather_rows_bulk)."""

import numpy as np
import pytest
import torch

import oracle
from kv_cache_decode_step_b200 import nosa

pytestmark = pytest.mark.gpu

GATHERS = [pytest.param(nosa.nosa_gather_rows, id="loads"), pytest.param(nosa.nosa_gather_rows_bulk, id="bulk")]


def _case(rng, src_rows, dst_rows, n):
    src_idx = rng.integers(0, src_rows, size=n).astype(np.int64)
    dst_idx = rng.permutation(dst_rows)[:n].astype(np.int64)
    return src_idx, dst_idx


@pytest.mark.parametrize("gather", GATHERS)
@pytest.mark.parametrize("row_bytes", [16, 256, 1024, 16384, 65536])
@pytest.mark.parametrize("pinned", [True, False])
def test_gather_rows_matches_the_oracle(row_bytes, pinned, gather):
    rng = np.random.default_rng(row_bytes)
    src_rows = max(8, (8 << 20) // row_bytes)
    dst_rows = max(4, src_rows // 2)
    n = dst_rows - 3          # ragged: not a multiple of any tile
    src_np = rng.integers(0, 256, size=(src_rows, row_bytes), dtype=np.uint8)
    src_idx, dst_idx = _case(rng, src_rows, dst_rows, n)
    dst0 = rng.integers(0, 256, size=(dst_rows, row_bytes), dtype=np.uint8)
    want = oracle.gather_rows(src_np, src_idx, dst0, dst_idx)

    src = torch.from_numpy(src_np)
    src = src.pin_memory() if pinned else src.cuda()
    dst = torch.from_numpy(dst0).cuda()
    si, di = torch.from_numpy(src_idx).cuda(), torch.from_numpy(dst_idx).cuda()
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    gather(src, src_rows, dst, dst_rows, row_bytes, si, di, n, 0, flags)
    torch.cuda.synchronize()
    assert flags.item() == 0
    assert np.array_equal(dst.cpu().numpy(), want)


@pytest.mark.parametrize("gather", GATHERS)
@pytest.mark.parametrize("ctas", [1, 7, 148])
def test_gather_rows_identity_destination_and_grid_widths(ctas, gather):
    rng = np.random.default_rng(ctas)
    src_np = rng.integers(0, 256, size=(4096, 256), dtype=np.uint8)
    src_idx = rng.integers(0, 4096, size=1001).astype(np.int64)
    want = oracle.gather_rows(src_np, src_idx, np.zeros((1001, 256), np.uint8))
    src = torch.from_numpy(src_np).pin_memory()
    dst = torch.zeros((1001, 256), dtype=torch.uint8, device="cuda")
    gather(src, 4096, dst, 1001, 256, torch.from_numpy(src_idx).cuda(), None, 1001, ctas)
    torch.cuda.synchronize()
    assert np.array_equal(dst.cpu().numpy(), want)


@pytest.mark.parametrize("gather", GATHERS)
def test_gather_rows_flags_and_skips_out_of_range_indices(gather):
    src_np = np.arange(64 * 16, dtype=np.uint8).reshape(64, 16)
    src_idx = np.array([0, 64, 5, -2, 63], dtype=np.int64)
    dst_idx = np.array([0, 1, 9, 3, 4], dtype=np.int64)   # row 9 is past the 8-row destination
    dst0 = np.full((8, 16), 7, dtype=np.uint8)
    want = oracle.gather_rows(src_np, src_idx, dst0, dst_idx)
    dst = torch.from_numpy(dst0).cuda()
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    gather(torch.from_numpy(src_np).pin_memory(), 64, dst, 8, 16, torch.from_numpy(src_idx).cuda(),
           torch.from_numpy(dst_idx).cuda(), 5, 0, flags)
    torch.cuda.synchronize()
    assert flags.item() == 1
    assert np.array_equal(dst.cpu().numpy(), want)


@pytest.mark.parametrize("gather", GATHERS)
def test_block_and_token_granularity_fill_the_same_cache(gather):
    """The transfer study's two arms move the same bytes: K of 2 KV heads at
    d = 128, 64 sequences of 4096 tokens, 4 missed blocks per unit, gathered as
    16 KiB block rows and as 256-byte token rows."""
    rng = np.random.default_rng(11)
    U, T, blocks = 128, 4096, 4
    host = torch.from_numpy(rng.integers(0, 256, size=(U * T, 256), dtype=np.uint8)).pin_memory()
    miss = np.stack([np.sort(rng.permutation(T // 64)[:blocks]) for _ in range(U)])       # [U, 4]
    blk_src = (np.arange(U)[:, None] * (T // 64) + miss).reshape(-1).astype(np.int64)
    tok_src = (blk_src[:, None] * 64 + np.arange(64)[None, :]).reshape(-1).astype(np.int64)
    a = torch.zeros((U * blocks, 64 * 256), dtype=torch.uint8, device="cuda")
    b = torch.zeros((U * blocks * 64, 256), dtype=torch.uint8, device="cuda")
    gather(host, U * T // 64, a, U * blocks, 16384, torch.from_numpy(blk_src).cuda(), None, len(blk_src))
    gather(host, U * T, b, U * blocks * 64, 256, torch.from_numpy(tok_src).cuda(), None, len(tok_src))
    torch.cuda.synchronize()
    assert torch.equal(a.view(-1), b.view(-1))
