"""Python binding of libmg (include/mg.h): argument marshalling only.

Every operation runs in the CUDA library; this module checks tensor dtypes,
shapes and devices, passes raw pointers and the current CUDA stream through
ctypes, and raises ``MgError`` on a non-OK status.  There is no fallback: if
libmg.so is missing, the first call raises.  PyTorch is used for device
memory and streams only.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

LIBRARY = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmg.so")

STATUS = {
    0: "MG_OK",
    1: "MG_ERR_INVALID_ARGUMENT",
    2: "MG_ERR_UNSUPPORTED_SHAPE",
    3: "MG_ERR_MISALIGNED",
    4: "MG_ERR_WORKSPACE_TOO_SMALL",
    5: "MG_ERR_CUDA",
    6: "MG_ERR_DEVICE_CHECK",
    7: "MG_ERR_DEVICE_TIMEOUT",
}
DEVERR_SLOT_RANGE = 0x1
DEVERR_ROW_RANGE = 0x2
DEVERR_LENGTH = 0x4
DEVERR_WAIT_TIMEOUT = 0x8
DEVERR_INTERNAL = 0x10

# name -> (restype, argtypes), the exact list of include/mg.h
_P, _I32, _I64, _F32, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "mg_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mg_abi_version": (_I32, []),
    "mg_store_kv": (ctypes.c_int, [_P, _P, _P, _I32, _P, _P, _I64, _I32, _I32, _P]),
    "mg_decode_plan": (ctypes.c_int, [_I32, _I32, _I32, _I32, ctypes.POINTER(_I32), ctypes.POINTER(_I64)]),
    "mg_decode_workspace_bytes": (_SZ, [_I32, _I32, _I32, _I32, _I32, _I32]),
    "mg_decode_attn": (ctypes.c_int, [_P, _P, _P, _I64, _P, _I32, _I32, _P, _P, _I32, _I32, _I32, _I32,
                                      _I32, _F32, _I32, _P, _P, _SZ, _P]),
    "mg_store_decode_attn": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _P, _I32, _I32, _P, _P, _I32, _I32,
                                            _I32, _I32, _I32, _F32, _I32, _P, _P, _SZ, _P]),
    "mg_decode_shared_prefix_workspace_bytes": (_SZ, [_I32, _I32, _I32, _I32, _I32, _I32, _I32]),
    "mg_decode_attn_shared_prefix": (ctypes.c_int, [_P, _P, _P, _I64, _P, _I32, _I32, _P, _P, _I32, _I32, _P, _P,
                                                    _I32, _I32, _I32, _I32, _F32, _I32, _P, _P, _SZ, _P]),
    "mg_store_decode_attn_shared_prefix": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I64, _P, _I32, _I32, _P, _P,
                                                          _I32, _I32, _P, _P, _I32, _I32, _I32, _I32, _F32, _I32,
                                                          _P, _P, _SZ, _P]),
    "mg_extend_attn": (ctypes.c_int, [_P, _P, _P, _I64, _P, _I32, _I32, _P, _P, _P, _P, _I32, _I32, _I32,
                                      _I32, _I32, _I32, _I32, _F32, _P, _P]),
    "mg_mixed_workspace_bytes": (_SZ, [_I32, _I32, _I32, _I32, _I32, _I32]),
    "mg_mixed_attn": (ctypes.c_int, [_P, _P, _P, _I64, _P, _I32, _I32, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32,
                                     _I32, _I32, _F32, _I32, _I32, _P, _P, _SZ, _P]),
    "mg_decode_attn_static_workspace": (ctypes.c_int, [_P, _P, _P, _I64, _P, _I32, _I32, _P, _P, _I32, _I32,
                                                       _I32, _I32, _I32, _F32, _I32, _P, _P]),
    "mg_set_extend_wait_limit": (ctypes.c_int, [ctypes.c_uint64, _I32]),
    "mg_read_device_error": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_uint32)]),
}

_lock = threading.Lock()
_lib = None


class MgError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


def load(path: str = LIBRARY):
    """Load libmg.so once; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(path):
                raise RuntimeError(f"libmg.so not built ({path}); run python -m paged_kv_attention_mg_b200.build")
            lib = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
        return _lib


def _check(status: int, what: str):
    if status != 0:
        raise MgError(status, what)


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, dtype, name: str) -> int:
    """Device pointer of a dense tensor of `dtype` on the current CUDA device
    (the library launches on the current device)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name} is on {t.device}, not on the current CUDA device "
                         f"(cuda:{torch.cuda.current_device()}), where the library launches")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _shape(t: torch.Tensor, shape, what: str) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{what} must be a tensor")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{what}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def _attention_shapes(op: str, q, k_cache, v_cache, page_table, out, per_request) -> None:
    """The sizes the library takes on trust: q [rows, Hq, D]; pools [slots, Hkv, D],
    V like K; a 2-D page table; out like q; [batch] metadata per request."""
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("page_table", page_table)):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{op}: {name} must be a tensor")
    if q.dim() != 3:
        raise ValueError(f"{op}: q must be [rows, num_q_heads, head_dim]")
    if k_cache.dim() != 3 or k_cache.shape[2] != q.shape[2]:
        raise ValueError(f"{op}: k_cache must be [num_slots, num_kv_heads, head_dim]")
    _shape(v_cache, k_cache.shape, f"{op}: v_cache")
    if page_table.dim() != 2:
        raise ValueError(f"{op}: page_table must be [rows, stride]")
    if out is not None:
        _shape(out, q.shape, f"{op}: out")
    for name, (t, shape) in per_request.items():
        _shape(t, shape, f"{op}: {name}")


def store_kv(k: torch.Tensor, v: torch.Tensor, out_loc: torch.Tensor, k_cache: torch.Tensor,
             v_cache: torch.Tensor, stream=None) -> None:
    """k_cache[out_loc[t]] = k[t]; v_cache[out_loc[t]] = v[t] (bf16 rows)."""
    if k.dim() != 3 or k_cache.dim() != 3:
        raise ValueError("store_kv: k must be [num_tokens, num_kv_heads, head_dim], k_cache [num_slots, ...]")
    t, hkv, d = k.shape
    if v.shape != k.shape or k_cache.shape[1:] != (hkv, d) or v_cache.shape != k_cache.shape:
        raise ValueError("store_kv: shape mismatch")
    if out_loc.shape != (t,):
        raise ValueError("store_kv: out_loc must be [num_tokens]")
    _check(load().mg_store_kv(_dev(k, torch.bfloat16, "k"), _dev(v, torch.bfloat16, "v"),
                              _dev(out_loc, torch.int32, "out_loc"), t,
                              _dev(k_cache, torch.bfloat16, "k_cache"),
                              _dev(v_cache, torch.bfloat16, "v_cache"), k_cache.shape[0], hkv, d,
                              _stream(stream)), "mg_store_kv")


def decode_plan(batch: int, num_kv_heads: int, max_seq_len: int, num_partitions: int = 0):
    """(workers, partial slots) that mg_decode_attn will use."""
    workers, slots = _I32(), _I64()
    _check(load().mg_decode_plan(batch, num_kv_heads, max_seq_len, num_partitions, ctypes.byref(workers),
                                 ctypes.byref(slots)), "mg_decode_plan")
    return workers.value, slots.value


def decode_workspace_bytes(batch: int, num_q_heads: int, num_kv_heads: int, max_seq_len: int,
                           num_partitions: int = 0, head_dim: int = 128) -> int:
    return int(load().mg_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_seq_len,
                                                 num_partitions))


def decode_attn(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, page_table: torch.Tensor,
                table_idx: torch.Tensor, seq_len: torch.Tensor, max_seq_len: int, scale: float,
                num_partitions: int = 0, out: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Paged decode attention; returns out [B, Hq, D] bf16."""
    b = q.shape[0] if isinstance(q, torch.Tensor) and q.dim() == 3 else -1
    _attention_shapes("decode_attn", q, k_cache, v_cache, page_table, out,
                      {"table_idx": (table_idx, (b,)), "seq_len": (seq_len, (b,))})
    b, hq, d = q.shape
    hkv = k_cache.shape[1]
    if out is None:
        out = torch.empty_like(q)
    need = decode_workspace_bytes(b, hq, hkv, max_seq_len, num_partitions, d)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, torch.uint8, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(load().mg_decode_attn(_dev(q, torch.bfloat16, "q"), _dev(k_cache, torch.bfloat16, "k_cache"),
                                 _dev(v_cache, torch.bfloat16, "v_cache"), k_cache.shape[0],
                                 _dev(page_table, torch.int32, "page_table"), page_table.shape[0],
                                 page_table.shape[1], _dev(table_idx, torch.int32, "table_idx"),
                                 _dev(seq_len, torch.int32, "seq_len"), b, max_seq_len, hq, hkv, d,
                                 float(scale), num_partitions, _dev(out, torch.bfloat16, "out"), ws_ptr, ws_bytes,
                                 _stream(stream)), "mg_decode_attn")
    return out


def store_decode_attn(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor, out_loc: torch.Tensor,
                      k_cache: torch.Tensor, v_cache: torch.Tensor, page_table: torch.Tensor,
                      table_idx: torch.Tensor, seq_len: torch.Tensor, max_seq_len: int, scale: float,
                      num_partitions: int = 0, out: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """store_kv(k_new, v_new, out_loc) then decode_attn, fused into one decode launch."""
    b = q.shape[0] if isinstance(q, torch.Tensor) and q.dim() == 3 else -1
    _attention_shapes("store_decode_attn", q, k_cache, v_cache, page_table, out,
                      {"table_idx": (table_idx, (b,)), "seq_len": (seq_len, (b,))})
    b, hq, d = q.shape
    hkv = k_cache.shape[1]
    if k_new.shape != (b, hkv, d) or v_new.shape != k_new.shape or out_loc.shape != (b,):
        raise ValueError("store_decode_attn: one new token per request expected")
    if out is None:
        out = torch.empty_like(q)
    need = decode_workspace_bytes(b, hq, hkv, max_seq_len, num_partitions, d)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, torch.uint8, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(load().mg_store_decode_attn(_dev(q, torch.bfloat16, "q"), _dev(k_new, torch.bfloat16, "k_new"),
                                       _dev(v_new, torch.bfloat16, "v_new"), _dev(out_loc, torch.int32, "out_loc"),
                                       _dev(k_cache, torch.bfloat16, "k_cache"),
                                       _dev(v_cache, torch.bfloat16, "v_cache"), k_cache.shape[0],
                                       _dev(page_table, torch.int32, "page_table"), page_table.shape[0],
                                       page_table.shape[1], _dev(table_idx, torch.int32, "table_idx"),
                                       _dev(seq_len, torch.int32, "seq_len"), b, max_seq_len, hq, hkv, d,
                                       float(scale), num_partitions, _dev(out, torch.bfloat16, "out"), ws_ptr,
                                       ws_bytes, _stream(stream)), "mg_store_decode_attn")
    return out


def decode_shared_prefix_workspace_bytes(batch: int, num_groups: int, num_q_heads: int, num_kv_heads: int,
                                         max_seq_len: int, num_partitions: int = 0, head_dim: int = 128) -> int:
    return int(load().mg_decode_shared_prefix_workspace_bytes(batch, num_groups, num_q_heads, num_kv_heads,
                                                               head_dim, max_seq_len, num_partitions))


def decode_attn_shared_prefix(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                              page_table: torch.Tensor, table_idx: torch.Tensor, seq_len: torch.Tensor,
                              group_first: torch.Tensor, prefix_len: torch.Tensor, max_seq_len: int,
                              scale: float, num_partitions: int = 0, out: Optional[torch.Tensor] = None,
                              workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """decode_attn where groups of consecutive requests share a prefix of their
    page-table rows (group_first [G+1], prefix_len [G]); the shared K/V rows are
    read once per group.  Returns out [B, Hq, D] bf16."""
    b = q.shape[0] if isinstance(q, torch.Tensor) and q.dim() == 3 else -1
    if not isinstance(prefix_len, torch.Tensor) or prefix_len.dim() != 1:
        raise ValueError("decode_attn_shared_prefix: prefix_len must be [num_groups]")
    ng = prefix_len.shape[0]
    _attention_shapes("decode_attn_shared_prefix", q, k_cache, v_cache, page_table, out,
                      {"table_idx": (table_idx, (b,)), "seq_len": (seq_len, (b,)),
                       "group_first": (group_first, (ng + 1,))})
    b, hq, d = q.shape
    hkv = k_cache.shape[1]
    if out is None:
        out = torch.empty_like(q)
    need = decode_shared_prefix_workspace_bytes(b, ng, hq, hkv, max_seq_len, num_partitions, d)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, torch.uint8, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(load().mg_decode_attn_shared_prefix(
        _dev(q, torch.bfloat16, "q"), _dev(k_cache, torch.bfloat16, "k_cache"),
        _dev(v_cache, torch.bfloat16, "v_cache"), k_cache.shape[0], _dev(page_table, torch.int32, "page_table"),
        page_table.shape[0], page_table.shape[1], _dev(table_idx, torch.int32, "table_idx"),
        _dev(seq_len, torch.int32, "seq_len"), b, max_seq_len, _dev(group_first, torch.int32, "group_first"),
        _dev(prefix_len, torch.int32, "prefix_len"), ng, hq, hkv, d, float(scale), num_partitions,
        _dev(out, torch.bfloat16, "out"), ws_ptr, ws_bytes, _stream(stream)), "mg_decode_attn_shared_prefix")
    return out


def store_decode_attn_shared_prefix(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                                    out_loc: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                                    page_table: torch.Tensor, table_idx: torch.Tensor, seq_len: torch.Tensor,
                                    group_first: torch.Tensor, prefix_len: torch.Tensor, max_seq_len: int,
                                    scale: float, num_partitions: int = 0, out: Optional[torch.Tensor] = None,
                                    workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """store_kv(k_new, v_new, out_loc) then decode_attn_shared_prefix, fused
    into one decode launch."""
    b = q.shape[0] if isinstance(q, torch.Tensor) and q.dim() == 3 else -1
    if not isinstance(prefix_len, torch.Tensor) or prefix_len.dim() != 1:
        raise ValueError("store_decode_attn_shared_prefix: prefix_len must be [num_groups]")
    ng = prefix_len.shape[0]
    _attention_shapes("store_decode_attn_shared_prefix", q, k_cache, v_cache, page_table, out,
                      {"table_idx": (table_idx, (b,)), "seq_len": (seq_len, (b,)),
                       "group_first": (group_first, (ng + 1,))})
    b, hq, d = q.shape
    hkv = k_cache.shape[1]
    if k_new.shape != (b, hkv, d) or v_new.shape != k_new.shape or out_loc.shape != (b,):
        raise ValueError("store_decode_attn_shared_prefix: one new token per request expected")
    if out is None:
        out = torch.empty_like(q)
    need = decode_shared_prefix_workspace_bytes(b, ng, hq, hkv, max_seq_len, num_partitions, d)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, torch.uint8, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(load().mg_store_decode_attn_shared_prefix(
        _dev(q, torch.bfloat16, "q"), _dev(k_new, torch.bfloat16, "k_new"), _dev(v_new, torch.bfloat16, "v_new"),
        _dev(out_loc, torch.int32, "out_loc"), _dev(k_cache, torch.bfloat16, "k_cache"),
        _dev(v_cache, torch.bfloat16, "v_cache"), k_cache.shape[0], _dev(page_table, torch.int32, "page_table"),
        page_table.shape[0], page_table.shape[1], _dev(table_idx, torch.int32, "table_idx"),
        _dev(seq_len, torch.int32, "seq_len"), b, max_seq_len, _dev(group_first, torch.int32, "group_first"),
        _dev(prefix_len, torch.int32, "prefix_len"), ng, hq, hkv, d, float(scale), num_partitions,
        _dev(out, torch.bfloat16, "out"), ws_ptr, ws_bytes, _stream(stream)), "mg_store_decode_attn_shared_prefix")
    return out


def extend_attn(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, page_table: torch.Tensor,
                table_idx: torch.Tensor, cached_len: torch.Tensor, seq_len: torch.Tensor,
                q_offset: torch.Tensor, max_q_len: int, max_seq_len: int, scale: float,
                out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Chunked-prefill extend attention; returns out [total_q, Hq, D] bf16."""
    if not isinstance(seq_len, torch.Tensor) or seq_len.dim() != 1:
        raise ValueError("extend_attn: seq_len must be [batch]")
    b = seq_len.shape[0]
    _attention_shapes("extend_attn", q, k_cache, v_cache, page_table, out,
                      {"table_idx": (table_idx, (b,)), "cached_len": (cached_len, (b,)),
                       "q_offset": (q_offset, (b + 1,))})
    total_q, hq, d = q.shape
    hkv = k_cache.shape[1]
    if out is None:
        out = torch.empty_like(q)
    _check(load().mg_extend_attn(_dev(q, torch.bfloat16, "q"), _dev(k_cache, torch.bfloat16, "k_cache"),
                                 _dev(v_cache, torch.bfloat16, "v_cache"), k_cache.shape[0],
                                 _dev(page_table, torch.int32, "page_table"), page_table.shape[0],
                                 page_table.shape[1], _dev(table_idx, torch.int32, "table_idx"),
                                 _dev(cached_len, torch.int32, "cached_len"),
                                 _dev(seq_len, torch.int32, "seq_len"), _dev(q_offset, torch.int32, "q_offset"),
                                 b, total_q, max_q_len, max_seq_len, hq, hkv, d, float(scale),
                                 _dev(out, torch.bfloat16, "out"), _stream(stream)), "mg_extend_attn")
    return out


def mixed_workspace_bytes(batch: int, num_q_heads: int, num_kv_heads: int, max_seq_len: int,
                          num_partitions: int = 0, head_dim: int = 128) -> int:
    return int(load().mg_mixed_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_seq_len,
                                               num_partitions))


def mixed_attn(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, page_table: torch.Tensor,
               table_idx: torch.Tensor, cached_len: torch.Tensor, seq_len: torch.Tensor, q_offset: torch.Tensor,
               max_q_len: int, max_seq_len: int, scale: float, num_partitions: int = 0,
               extend_ctas: int = 0, out: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """extend_attn for a mixed batch: one-token requests through the decode
    kernel, the others through the extend kernel; returns out [total_q, Hq, D].
    extend_ctas > 0 runs the extend kernel on that many SMs at the same time as
    the decode kernel on the rest (see mixed_extend_ctas)."""
    if not isinstance(seq_len, torch.Tensor) or seq_len.dim() != 1:
        raise ValueError("mixed_attn: seq_len must be [batch]")
    b = seq_len.shape[0]
    _attention_shapes("mixed_attn", q, k_cache, v_cache, page_table, out,
                      {"table_idx": (table_idx, (b,)), "cached_len": (cached_len, (b,)),
                       "q_offset": (q_offset, (b + 1,))})
    total_q, hq, d = q.shape
    hkv = k_cache.shape[1]
    if out is None:
        out = torch.empty_like(q)
    need = mixed_workspace_bytes(b, hq, hkv, max_seq_len, num_partitions, d)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, torch.uint8, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(load().mg_mixed_attn(_dev(q, torch.bfloat16, "q"), _dev(k_cache, torch.bfloat16, "k_cache"),
                                _dev(v_cache, torch.bfloat16, "v_cache"), k_cache.shape[0],
                                _dev(page_table, torch.int32, "page_table"), page_table.shape[0], page_table.shape[1],
                                _dev(table_idx, torch.int32, "table_idx"), _dev(cached_len, torch.int32, "cached_len"),
                                _dev(seq_len, torch.int32, "seq_len"), _dev(q_offset, torch.int32, "q_offset"),
                                b, total_q, max_q_len, max_seq_len, hq, hkv, d, float(scale), num_partitions,
                                extend_ctas, _dev(out, torch.bfloat16, "out"), ws_ptr, ws_bytes, _stream(stream)),
           "mg_mixed_attn")
    return out


# Rates the split estimate works with, measured on B200 with this library's
# kernels: a 128-key tile of an extend item (two Q tiles, causal edge tiles
# counted whole) every ~3.6 us per SM; the decode kernel's K/V stream at up to
# ~52 GB/s per SM and ~5.6 TB/s in all (HBM).
_EXTEND_TILE_S = 3.6e-6
_DECODE_SM_BYTES_PER_S = 52e9
_DECODE_HBM_BYTES_PER_S = 5.6e12


def mixed_extend_ctas(cached_len, seq_len, num_q_heads: int, num_kv_heads: int, sms: int,
                      head_dim: int = 128) -> int:
    """How many SMs mg_mixed_attn should give the extend kernel so that it and
    the decode kernel finish together, from the batch's host-side lengths (the
    scheduler that formed the batch has them): the extend items' KV tiles
    against the one-token requests' K/V bytes at the rates above; the split
    whose later kernel ends first.  0 when the batch has no prompt chunk or no
    one-token request."""
    g = num_q_heads // num_kv_heads
    span = 2 * (128 // g)  # tokens of a q block
    tiles, dec_bytes = 0, 0
    for c, L in zip(cached_len, seq_len):
        c, L = int(c), int(L)
        n = L - c
        if n == 1:
            dec_bytes += L * num_kv_heads * head_dim * 2 * 2
        elif n > 1:
            for t0 in range(0, n, span):
                tiles += -(-(c + min(t0 + span, n)) // 128) * num_kv_heads
    if tiles == 0 or dec_bytes == 0:
        return 0

    def finish(e):  # when the later of the two kernels ends with e SMs for extend
        ext = tiles * _EXTEND_TILE_S / e
        dec = dec_bytes / min(_DECODE_HBM_BYTES_PER_S, (sms - e) * _DECODE_SM_BYTES_PER_S)
        return max(ext, dec)
    return min(range(1, sms), key=finish)


STATIC_WORKSPACE_BYTES = 16 << 20  # MG_DECODE_STATIC_WORKSPACE_BYTES in include/mg.h


def decode_attn_static_workspace(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                                 page_table: torch.Tensor, table_idx: torch.Tensor, seq_len: torch.Tensor,
                                 max_seq_len: int, scale: float, num_partitions: int = 0,
                                 out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """decode_attn for callers that cannot pass device scratch memory: the
    library's own fixed workspace is used (shared by all calls; overlapping
    calls race).  Raises MgError(MG_ERR_WORKSPACE_TOO_SMALL) when the plan
    needs more than STATIC_WORKSPACE_BYTES.  Allocates nothing on the device
    except `out` when it is not given."""
    b = q.shape[0] if isinstance(q, torch.Tensor) and q.dim() == 3 else -1
    _attention_shapes("decode_attn_static_workspace", q, k_cache, v_cache, page_table, out,
                      {"table_idx": (table_idx, (b,)), "seq_len": (seq_len, (b,))})
    b, hq, d = q.shape
    hkv = k_cache.shape[1]
    if out is None:
        out = torch.empty_like(q)
    _check(load().mg_decode_attn_static_workspace(
        _dev(q, torch.bfloat16, "q"), _dev(k_cache, torch.bfloat16, "k_cache"),
        _dev(v_cache, torch.bfloat16, "v_cache"), k_cache.shape[0], _dev(page_table, torch.int32, "page_table"),
        page_table.shape[0], page_table.shape[1], _dev(table_idx, torch.int32, "table_idx"),
        _dev(seq_len, torch.int32, "seq_len"), b, max_seq_len, hq, hkv, d, float(scale), num_partitions,
        _dev(out, torch.bfloat16, "out"), _stream(stream)), "mg_decode_attn_static_workspace")
    return out


def set_extend_wait_limit(limit_ns: int = 0, inject_stall: bool = False) -> None:
    """Bound of extend's pipeline waits (0 = the default 2 s) and the
    fault-injection hook that withholds one hand-off (tests only)."""
    _check(load().mg_set_extend_wait_limit(int(limit_ns), 1 if inject_stall else 0), "mg_set_extend_wait_limit")


def read_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error bits."""
    bits = ctypes.c_uint32(0)
    st = load().mg_read_device_error(_stream(stream), ctypes.byref(bits))
    if st not in (0, 6, 7):
        raise MgError(st, "mg_read_device_error")
    return bits.value
