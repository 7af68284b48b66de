"""ctypes binding of libnosa.so: one Python function per C entry point, same
names, argument marshalling only (tensors and arrays become raw pointers,
statuses become exceptions).  Every computation happens in the library's CUDA
kernels; there is no Python or CPU fallback, and loading fails loudly when the
library has not been built.
"""

from __future__ import annotations

import ctypes as C
import os
import threading
from typing import Any, Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnosa.so")

NOSA_OK = 0
NOSA_ERR_INVALID = -1
NOSA_ERR_CUDA = -2
NOSA_ERR_NOMEM = -3
NOSA_ERR_ORDER = -4
NOSA_ERR_TIMEOUT = -5
NOSA_ERR_UNIMPLEMENTED = -6
_NAMES = {0: "NOSA_OK", -1: "NOSA_ERR_INVALID", -2: "NOSA_ERR_CUDA", -3: "NOSA_ERR_NOMEM",
          -4: "NOSA_ERR_ORDER", -5: "NOSA_ERR_TIMEOUT", -6: "NOSA_ERR_UNIMPLEMENTED"}

# every symbol declared in include/nosa.h
ENTRY_POINTS = (
    "nosa_create", "nosa_destroy", "nosa_attach_kv", "nosa_append_token", "nosa_score_blocks",
    "nosa_select", "nosa_fetch_missing", "nosa_sparse_decode", "nosa_get_stats", "nosa_reset_stats",
    "nosa_check_errors", "nosa_read_cache_map", "nosa_get_state", "nosa_set_state",
    "nosa_debug_wait_flag", "nosa_last_error", "nosa_version", "nosa_sparse_decode_noalloc",
    "nosa_gather_rows", "nosa_score_select_fetch", "nosa_gather_rows_bulk", "nosa_noalloc_check_errors",
    "nosa_read_cache", "nosa_debug_inject_cuda_error", "nosa_decode_step",
)


class NosaError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_NAMES.get(status, status)}: {msg}")
        self.status = status


class nosa_config(C.Structure):
    _fields_ = [(n, C.c_int) for n in (
        "batch", "n_q_heads", "n_kv_heads", "head_dim", "block", "sub_block", "k_query",
        "k_agnostic", "min_overlap", "max_blocks", "cache_slots", "sink_blocks", "window_blocks")]


class nosa_stats(C.Structure):
    _fields_ = [("steps", C.c_int64), ("selected", C.c_int64), ("hits", C.c_int64),
                ("misses", C.c_int64), ("fetched_bytes", C.c_int64), ("overlap_sum", C.c_int64),
                ("overlap_terms", C.c_int64), ("min_overlap", C.c_int32), ("max_fetch", C.c_int32),
                ("error_bits", C.c_uint32), ("n_closed", C.c_int32), ("tail_len", C.c_int32),
                ("reserved", C.c_int32)]

    def as_dict(self):
        return {n: getattr(self, n) for n, _ in self._fields_ if n != "reserved"}


_lock = threading.Lock()
_lib: Optional[C.CDLL] = None


def lib() -> C.CDLL:
    """Load libnosa.so (built in-tree); raise if it is missing."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m kv_cache_decode_step_b200.build`")
        L = C.CDLL(LIB_PATH)
        vp, i32, st = C.c_void_p, C.c_int, C.c_int
        sig = {
            "nosa_create": ([C.POINTER(nosa_config), C.POINTER(vp)], st),
            "nosa_destroy": ([vp], None),
            "nosa_attach_kv": ([vp, vp, vp, i32, vp, vp], st),
            "nosa_append_token": ([vp, vp, vp, vp, vp], st),
            "nosa_score_blocks": ([vp, vp, vp, vp], st),
            "nosa_select": ([vp, vp, vp, vp], st),
            "nosa_fetch_missing": ([vp, vp, vp, vp, vp, vp], st),
            "nosa_sparse_decode": ([vp, vp, vp, vp, vp], st),
            "nosa_get_stats": ([vp, C.POINTER(nosa_stats)], st),
            "nosa_reset_stats": ([vp, vp], st),
            "nosa_check_errors": ([vp], st),
            "nosa_read_cache_map": ([vp, vp], st),
            "nosa_get_state": ([vp, vp, C.POINTER(C.c_size_t)], st),
            "nosa_set_state": ([vp, vp, C.c_size_t], st),
            "nosa_debug_wait_flag": ([vp, vp, i32, vp], st),
            "nosa_last_error": ([], C.c_char_p),
            "nosa_version": ([], C.c_char_p),
            "nosa_sparse_decode_noalloc": ([vp, vp, vp, i32, i32, i32, i32, vp, i32, vp, vp], st),
            "nosa_noalloc_check_errors": ([vp], st),
            "nosa_read_cache": ([vp, i32, i32, vp, vp], st),
            "nosa_debug_inject_cuda_error": ([i32], st),
            "nosa_gather_rows": ([vp, C.c_int64, vp, C.c_int64, i32, vp, vp, i32, i32, vp, vp], st),
            "nosa_gather_rows_bulk": ([vp, C.c_int64, vp, C.c_int64, i32, vp, vp, i32, i32, vp, vp], st),
            "nosa_score_select_fetch": ([vp, vp, vp, vp, vp, vp, vp, vp], st),
            "nosa_decode_step": ([vp, vp, vp, vp, vp, vp, vp, vp, vp], st),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
        return L


def _ptr(x: Any) -> Optional[int]:
    """Raw address of a torch tensor, numpy array, int or None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):
        return x.ctypes.data
    raise TypeError(f"cannot take the address of {type(x)!r}")


def _stream(s: Any) -> Optional[int]:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream  # torch.cuda.Stream


def _check(status: int, name: str) -> None:
    if status != NOSA_OK:
        raise NosaError(status, f"{name}: {nosa_last_error()}")


# ------------------------------------------------------------------ entry points

def nosa_last_error() -> str:
    r = lib().nosa_last_error()
    return r.decode() if r else ""


def nosa_version() -> str:
    return lib().nosa_version().decode()


def nosa_create(cfg: nosa_config) -> int:
    out = C.c_void_p()
    _check(lib().nosa_create(C.byref(cfg), C.byref(out)), "nosa_create")
    return out.value


def nosa_destroy(ctx: Optional[int]) -> None:
    if ctx:
        lib().nosa_destroy(ctx)


def nosa_attach_kv(ctx, k, v, n_tokens: int, agnostic, stream=None) -> None:
    _check(lib().nosa_attach_kv(ctx, _ptr(k), _ptr(v), int(n_tokens), _ptr(agnostic), _stream(stream)),
           "nosa_attach_kv")


def nosa_append_token(ctx, k_new, v_new, agnostic_if_close=None, stream=None) -> None:
    _check(lib().nosa_append_token(ctx, _ptr(k_new), _ptr(v_new), _ptr(agnostic_if_close),
                                   _stream(stream)), "nosa_append_token")


def nosa_score_blocks(ctx, q, scores, stream=None) -> None:
    _check(lib().nosa_score_blocks(ctx, _ptr(q), _ptr(scores), _stream(stream)), "nosa_score_blocks")


def nosa_select(ctx, scores, sel, stream=None) -> None:
    _check(lib().nosa_select(ctx, _ptr(scores), _ptr(sel), _stream(stream)), "nosa_select")


def nosa_fetch_missing(ctx, sel, fetch, n_fetch, compute=None, copy=None) -> None:
    _check(lib().nosa_fetch_missing(ctx, _ptr(sel), _ptr(fetch), _ptr(n_fetch), _stream(compute),
                                    _stream(copy)), "nosa_fetch_missing")


def nosa_score_select_fetch(ctx, q, scores, sel, fetch, n_fetch, compute=None, copy=None) -> None:
    _check(lib().nosa_score_select_fetch(ctx, _ptr(q), _ptr(scores), _ptr(sel), _ptr(fetch), _ptr(n_fetch),
                                         _stream(compute), _stream(copy if copy is not None else compute)),
           "nosa_score_select_fetch")


def nosa_decode_step(ctx, q, out, scores=None, sel=None, fetch=None, n_fetch=None, compute=None,
                     copy=None) -> None:
    _check(lib().nosa_decode_step(ctx, _ptr(q), _ptr(scores), _ptr(sel), _ptr(fetch), _ptr(n_fetch), _ptr(out),
                                  _stream(compute), _stream(copy if copy is not None else compute)),
           "nosa_decode_step")


def nosa_sparse_decode(ctx, q, sel, out, stream=None) -> None:
    _check(lib().nosa_sparse_decode(ctx, _ptr(q), _ptr(sel), _ptr(out), _stream(stream)),
           "nosa_sparse_decode")


def nosa_get_stats(ctx) -> dict:
    s = nosa_stats()
    _check(lib().nosa_get_stats(ctx, C.byref(s)), "nosa_get_stats")
    return s.as_dict()


def nosa_reset_stats(ctx, stream=None) -> None:
    _check(lib().nosa_reset_stats(ctx, _stream(stream)), "nosa_reset_stats")


def nosa_check_errors(ctx) -> None:
    _check(lib().nosa_check_errors(ctx), "nosa_check_errors")


def nosa_read_cache_map(ctx, out) -> None:
    _check(lib().nosa_read_cache_map(ctx, _ptr(out)), "nosa_read_cache_map")


def nosa_read_cache(ctx, unit_begin: int, n_units: int, k_out, v_out) -> None:
    _check(lib().nosa_read_cache(ctx, int(unit_begin), int(n_units), _ptr(k_out), _ptr(v_out)), "nosa_read_cache")


def nosa_debug_inject_cuda_error(skip: int) -> None:
    _check(lib().nosa_debug_inject_cuda_error(int(skip)), "nosa_debug_inject_cuda_error")


def nosa_get_state(ctx) -> bytes:
    size = C.c_size_t(0)
    _check(lib().nosa_get_state(ctx, None, C.byref(size)), "nosa_get_state")
    buf = (C.c_ubyte * size.value)()
    _check(lib().nosa_get_state(ctx, C.addressof(buf), C.byref(size)), "nosa_get_state")
    return bytes(buf)


def nosa_set_state(ctx, blob: bytes) -> None:
    buf = (C.c_ubyte * len(blob)).from_buffer_copy(blob)
    _check(lib().nosa_set_state(ctx, C.addressof(buf), len(blob)), "nosa_set_state")


def nosa_debug_wait_flag(ctx, flag, timeout_ms: int, stream=None) -> None:
    _check(lib().nosa_debug_wait_flag(ctx, _ptr(flag), int(timeout_ms), _stream(stream)),
           "nosa_debug_wait_flag")


def nosa_sparse_decode_noalloc(q, k, v, batch: int, n_q_heads: int, n_kv_heads: int, max_blocks: int,
                               sel, k_sel: int, out, stream=None) -> None:
    _check(lib().nosa_sparse_decode_noalloc(_ptr(q), _ptr(k), _ptr(v), int(batch), int(n_q_heads),
                                            int(n_kv_heads), int(max_blocks), _ptr(sel), int(k_sel),
                                            _ptr(out), _stream(stream)), "nosa_sparse_decode_noalloc")


def nosa_noalloc_check_errors(stream=None) -> None:
    _check(lib().nosa_noalloc_check_errors(_stream(stream)), "nosa_noalloc_check_errors")


def nosa_gather_rows(src, src_rows: int, dst, dst_rows: int, row_bytes: int, src_idx, dst_idx, n: int,
                     ctas: int = 0, flags=None, stream=None) -> None:
    _check(lib().nosa_gather_rows(_ptr(src), int(src_rows), _ptr(dst), int(dst_rows), int(row_bytes),
                                  _ptr(src_idx), _ptr(dst_idx), int(n), int(ctas), _ptr(flags),
                                  _stream(stream)), "nosa_gather_rows")


def nosa_gather_rows_bulk(src, src_rows: int, dst, dst_rows: int, row_bytes: int, src_idx, dst_idx, n: int,
                          ctas: int = 0, flags=None, stream=None) -> None:
    _check(lib().nosa_gather_rows_bulk(_ptr(src), int(src_rows), _ptr(dst), int(dst_rows), int(row_bytes),
                                       _ptr(src_idx), _ptr(dst_idx), int(n), int(ctas), _ptr(flags),
                                       _stream(stream)), "nosa_gather_rows_bulk")


def config_from_workload(w) -> nosa_config:
    return nosa_config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.block, w.sub_block,
                       w.k_query, w.k_agnostic, w.min_overlap, w.max_blocks, w.cache_slots,
                       w.sink_blocks, w.window_blocks)
