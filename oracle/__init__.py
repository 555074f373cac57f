"""The oracle: a plain, slow fp64 CPU reference of the paged KV hot path.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` leg of ``bench.py`` (and its ``--impl reference`` arm) may
import this package.  The product library and its Python binding never do.

The arithmetic lives in ``mg_oracle.c`` (plain C, double precision, loops over
requests x heads x positions that dereference the page table).  This module
only compiles it with gcc, loads it with ctypes and marshals numpy arrays.
bf16 tensors cross this boundary as their raw uint16 bit patterns.

Functions and what pins them (see ``tests/test_oracle_pins.py``):

* ``store_kv``  -- pinned against ``torch.Tensor.index_copy_`` (bit-exact).
* ``decode``    -- pinned against dense fp64 ``scaled_dot_product_attention`` on
  tiny inputs, slot-permutation invariance and closed forms.
* ``extend``    -- pinned against dense causal fp64 SDPA with an explicit mask,
  against ``decode`` row by row, and by the same invariants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "mg_oracle.c")
LIBRARY = os.path.join(_HERE, "liboracle.so")

ERRORS = {
    0: "ok",
    1: "bad argument",
    2: "slot out of range",
    3: "page-table row out of range",
    4: "length out of range",
    5: "out of memory",
}

_lock = threading.Lock()
_lib = None


class OracleError(RuntimeError):
    pass


def build(source: str = SOURCE, output: str = LIBRARY, force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math: IEEE double, fixed order)."""
    if not force and os.path.exists(output) and os.path.getmtime(output) >= os.path.getmtime(source):
        return output
    tmp = output + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", tmp, source, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, output)
    return output


def load(path: str | None = None):
    """Load the compiled oracle (building it first if needed)."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
        return _lib


def _bind(lib):
    p, i64, i32, dbl = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double
    lib.oracle_store_kv.argtypes = [p, p, p, i64, p, p, i64, i64, i64]
    lib.oracle_store_kv.restype = i32
    lib.oracle_decode.argtypes = [p, p, p, i64, p, i64, i64, p, p, i64, i64, i64, i64, dbl, p, i32, p]
    lib.oracle_decode.restype = i32
    lib.oracle_extend.argtypes = [p, p, p, i64, p, i64, i64, p, p, p, p, i64, i64, i64, i64, i64,
                                  dbl, p, i32, p]
    lib.oracle_extend.restype = i32
    return lib


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16 data crosses as uint16 bit patterns"
    return a


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _mask(requests, batch: int):
    if requests is None:
        return None
    m = np.zeros(batch, dtype=np.uint8)
    m[np.asarray(list(requests), dtype=np.int64)] = 1
    return m


def _check(code: int, what: str):
    if code != 0:
        raise OracleError(f"oracle {what}: {ERRORS.get(code, code)}")


def store_kv(k, v, out_loc, k_pool, v_pool, lib=None) -> None:
    """In-place: k_pool[out_loc[t]] = k[t], v_pool[out_loc[t]] = v[t] (uint16 bits)."""
    lib = lib or load()
    k, v, out_loc = _u16(k), _u16(v), _i32(out_loc)
    assert k_pool.flags["C_CONTIGUOUS"] and v_pool.flags["C_CONTIGUOUS"]
    num_slots, hkv, d = k_pool.shape
    _check(lib.oracle_store_kv(_ptr(k), _ptr(v), _ptr(out_loc), out_loc.shape[0], _ptr(k_pool),
                               _ptr(v_pool), num_slots, hkv, d), "store_kv")


def decode(q, k_pool, v_pool, page_table, table_idx, seq_len, scale: float,
           requests=None, threads: int = 0, lib=None) -> np.ndarray:
    """fp64 decode attention: returns [B, Hq, D] float64 (NaN for skipped requests)."""
    lib = lib or load()
    q, k_pool, v_pool = _u16(q), _u16(k_pool), _u16(v_pool)
    page_table, table_idx, seq_len = _i32(page_table), _i32(table_idx), _i32(seq_len)
    batch, hq, d = q.shape
    num_slots, hkv, _ = k_pool.shape
    out = np.full((batch, hq, d), np.nan, dtype=np.float64)
    mask = _mask(requests, batch)
    _check(lib.oracle_decode(_ptr(q), _ptr(k_pool), _ptr(v_pool), num_slots, _ptr(page_table),
                             page_table.shape[0], page_table.shape[1], _ptr(table_idx),
                             _ptr(seq_len), batch, hq, hkv, d, float(scale), _ptr(mask),
                             int(threads), _ptr(out)), "decode")
    return out


def extend(q, k_pool, v_pool, page_table, table_idx, cached_len, seq_len, q_offset,
           scale: float, requests=None, threads: int = 0, lib=None) -> np.ndarray:
    """fp64 causal extend attention: returns [total_q, Hq, D] float64."""
    lib = lib or load()
    q, k_pool, v_pool = _u16(q), _u16(k_pool), _u16(v_pool)
    page_table, table_idx = _i32(page_table), _i32(table_idx)
    cached_len, seq_len, q_offset = _i32(cached_len), _i32(seq_len), _i32(q_offset)
    total_q, hq, d = q.shape
    num_slots, hkv, _ = k_pool.shape
    batch = seq_len.shape[0]
    out = np.full((total_q, hq, d), np.nan, dtype=np.float64)
    mask = _mask(requests, batch)
    _check(lib.oracle_extend(_ptr(q), _ptr(k_pool), _ptr(v_pool), num_slots, _ptr(page_table),
                             page_table.shape[0], page_table.shape[1], _ptr(table_idx),
                             _ptr(cached_len), _ptr(seq_len), _ptr(q_offset), batch, total_q,
                             hq, hkv, d, float(scale), _ptr(mask), int(threads), _ptr(out)),
           "extend")
    return out
