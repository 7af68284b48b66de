"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point declared in include/nosa.h, and rejects bad configurations
and NULL arguments with status codes before touching CUDA."""

import ctypes as C
import os
import re

import pytest

from kv_cache_decode_step_b200 import build as nbuild
from kv_cache_decode_step_b200 import configs, nosa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    nbuild.build()
    return nosa.lib()


def declared_entry_points():
    src = open(os.path.join(ROOT, "include", "nosa.h")).read()
    return sorted(set(re.findall(r"^NOSA_API\s+[\w\s\*]*?\b(nosa_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_binding_entry_points():
    assert declared_entry_points() == sorted(nosa.ENTRY_POINTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_entry_points():
        assert hasattr(L, name), name
    assert "sm_100a" in nosa.nosa_version()


def test_library_needs_no_cuda_shared_libraries():
    import subprocess
    out = subprocess.run(["ldd", nosa.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libcudart.so" not in out


def _cfg(**kw):
    w = configs.get("tiny")
    c = nosa.config_from_workload(w)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 64, nosa.NOSA_ERR_UNIMPLEMENTED),
    ("block", 32, nosa.NOSA_ERR_UNIMPLEMENTED),
    ("sub_block", 8, nosa.NOSA_ERR_UNIMPLEMENTED),
    ("n_q_heads", 7, nosa.NOSA_ERR_INVALID),          # not a multiple of n_kv_heads = 2
    ("n_q_heads", 36, nosa.NOSA_ERR_UNIMPLEMENTED),   # group of 18 > 8
    ("batch", 0, nosa.NOSA_ERR_INVALID),
    ("k_query", -1, nosa.NOSA_ERR_INVALID),
    ("k_query", 253, nosa.NOSA_ERR_UNIMPLEMENTED),    # k = 257 > 256
    ("min_overlap", 17, nosa.NOSA_ERR_INVALID),       # > k = 16
    ("min_overlap", -1, nosa.NOSA_ERR_INVALID),
    ("max_blocks", 15, nosa.NOSA_ERR_INVALID),        # < k
    ("max_blocks", 9000, nosa.NOSA_ERR_INVALID),
    ("cache_slots", 15, nosa.NOSA_ERR_INVALID),       # 0 < C < k
    ("cache_slots", 2000, nosa.NOSA_ERR_INVALID),
    ("sink_blocks", -1, nosa.NOSA_ERR_INVALID),
    ("window_blocks", 5, nosa.NOSA_ERR_INVALID),     # sink + window > k_agnostic = 4
])
def test_create_rejects_bad_configs(L, field, value, status):
    out = C.c_void_p()
    rc = L.nosa_create(C.byref(_cfg(**{field: value})), C.byref(out))
    assert rc == status
    assert out.value is None
    assert nosa.nosa_last_error() != ""


def test_zero_budget_is_rejected(L):
    out = C.c_void_p()
    assert L.nosa_create(C.byref(_cfg(k_query=0, k_agnostic=0)), C.byref(out)) == nosa.NOSA_ERR_INVALID


def test_null_arguments_are_rejected(L):
    out = C.c_void_p()
    assert L.nosa_create(None, C.byref(out)) == nosa.NOSA_ERR_INVALID
    assert L.nosa_create(C.byref(_cfg()), None) == nosa.NOSA_ERR_INVALID
    L.nosa_destroy(None)  # ignored
    for name, nargs in [("nosa_score_blocks", 4), ("nosa_select", 4), ("nosa_sparse_decode", 5),
                        ("nosa_fetch_missing", 6), ("nosa_check_errors", 1), ("nosa_reset_stats", 2),
                        ("nosa_read_cache_map", 2), ("nosa_attach_kv", 6), ("nosa_append_token", 5),
                        ("nosa_debug_wait_flag", 4)]:
        args = [None] * nargs
        if name in ("nosa_attach_kv",):
            args = [None, None, None, 0, None, None]
        if name == "nosa_debug_wait_flag":
            args = [None, None, 10, None]
        assert getattr(L, name)(*args) == nosa.NOSA_ERR_INVALID, name
    st = nosa.nosa_stats()
    assert L.nosa_get_stats(None, C.byref(st)) == nosa.NOSA_ERR_INVALID
    size = C.c_size_t(0)
    assert L.nosa_get_state(None, None, C.byref(size)) == nosa.NOSA_ERR_INVALID


def test_valid_config_without_gpu_fails_cleanly(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    out = C.c_void_p()
    rc = L.nosa_create(C.byref(_cfg()), C.byref(out))
    assert rc in (nosa.NOSA_ERR_CUDA, nosa.NOSA_ERR_NOMEM)
    assert out.value is None


def test_binding_raises_with_status():
    with pytest.raises(nosa.NosaError) as ei:
        nosa.nosa_create(_cfg(head_dim=64))
    assert ei.value.status == nosa.NOSA_ERR_UNIMPLEMENTED


def test_every_workload_config_validates_host_side(L):
    """The five workloads pass every host-side check (the create call then
    fails only for lack of a device when there is none)."""
    import torch
    for name in configs.ORDER:
        out = C.c_void_p()
        rc = L.nosa_create(C.byref(nosa.config_from_workload(configs.get(name))), C.byref(out))
        if torch.cuda.is_available():
            assert rc == nosa.NOSA_OK
            L.nosa_destroy(out)
        else:
            assert rc in (nosa.NOSA_ERR_CUDA, nosa.NOSA_ERR_NOMEM), (name, nosa.nosa_last_error())


@pytest.mark.parametrize("row_bytes,n,ctas", [(24, 1, 0), (8, 1, 0), (131072, 1, 0), (256, -1, 0),
                                              (256, 1, -1), (256, 1, 70000)])
def test_gather_rows_rejects_bad_sizes(L, row_bytes, n, ctas):
    rc = L.nosa_gather_rows(None, 0, None, 0, row_bytes, None, None, n, ctas, None, None)
    assert rc == nosa.NOSA_ERR_INVALID


def test_gather_rows_with_no_rows_is_a_no_op(L):
    assert L.nosa_gather_rows(None, 0, None, 0, 256, None, None, 0, 0, None, None) == nosa.NOSA_OK


def test_gather_rows_rejects_pageable_memory(L):
    import numpy as np
    src = np.zeros((4, 64), dtype=np.uint32)     # pageable host memory
    dst = np.zeros((4, 64), dtype=np.uint32)
    idx = np.arange(4, dtype=np.int64)
    with pytest.raises(nosa.NosaError) as e:
        nosa.nosa_gather_rows(src, 4, dst, 4, 256, idx, None, 4)
    assert e.value.status == nosa.NOSA_ERR_INVALID
