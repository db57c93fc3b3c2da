"""ctypes binding of libcsa2.so: argument marshalling only.

Every function here converts torch tensors to raw pointers and calls the C entry
point of the same name; all computation runs in the library's CUDA kernels.
There is no fallback: if the library is missing or fails to load, the import
raises.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa2.so")

CSA2_OP_INDEX_FULL = 1
CSA2_OP_INDEX_REINDEX = 2
CSA2_OP_SPARSE_ATTN = 3

STATUS = {0: "CSA2_OK", 1: "CSA2_ERR_INVALID_ARG", 2: "CSA2_ERR_CAPACITY",
          3: "CSA2_ERR_WORKSPACE", 4: "CSA2_ERR_UNSUPPORTED", 5: "CSA2_ERR_CUDA",
          6: "CSA2_ERR_DEVICE_BOUNDS"}

DEVERR_SLOT, DEVERR_INDEX, DEVERR_NMAX, DEVERR_RANGE, DEVERR_TIMEOUT = 0x1, 0x2, 0x4, 0x8, 0x10
DEFAULT_WAIT_LIMIT_NS = 500_000_000
DEVERR_ROPE = 0x20
DEVERR_PAGE = 0x40

# every symbol declared in include/csa2.h
EXPORTS = ("csa2_quantize_append", "csa2_quantize_append_rope", "csa2_workspace_size",
           "csa2_index_full", "csa2_index_full_tc", "csa2_index_full_noalloc",
           "csa2_index_reindex", "csa2_sparse_attn_decode", "csa2_sparse_attn_decode_append",
           "csa2_sparse_attn_decode_append_rope", "csa2_read_device_error",
           "csa2_status_string", "csa2_abi_version", "csa2_debug_set_waits",
           "csa2_index_full_slice", "csa2_index_merge", "csa2_attn_combine",
           "csa2_quantize_append_paged", "csa2_index_full_paged", "csa2_index_reindex_paged",
           "csa2_sparse_attn_decode_paged", "csa2_sparse_attn_decode_reuse",
           "csa2_index_reindex_settled", "csa2_index_reindex_paged_settled",
           "csa2_sparse_attn_decode_paged_reuse")


class Csa2Error(RuntimeError):
    def __init__(self, fn: str, status: int, lib):
        self.status = status
        msg = lib.csa2_status_string(status).decode()
        super().__init__(f"{fn} -> {STATUS.get(status, status)} ({msg})")


class CSA2GlobalKV(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scales", C.c_void_p), ("idx_codes", C.c_void_p),
                ("idx_scale", C.c_void_p), ("batch", C.c_int32), ("cap", C.c_int32),
                ("d_idx", C.c_int32), ("ratio", C.c_int32)]


class CSA2SWA(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scale", C.c_void_p), ("batch", C.c_int32),
                ("window_cap", C.c_int32)]


class CSA2PagedKV(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scales", C.c_void_p), ("idx_codes", C.c_void_p),
                ("idx_scale", C.c_void_p), ("block_table", C.c_void_p), ("batch", C.c_int32),
                ("max_pages", C.c_int32), ("page_size", C.c_int32), ("n_pages", C.c_int32),
                ("d_idx", C.c_int32), ("ratio", C.c_int32)]


class CSA2Rope(C.Structure):
    _fields_ = [("cos_sin", C.c_void_p), ("n_pos", C.c_int32), ("start", C.c_int32),
                ("pairs", C.c_int32)]


class Rope:
    """A RoPE table on the device ([n_pos][pairs][2] fp32 (cos, sin)) with its channel
    range, and the csa2_rope descriptor that points at it (kept alive together)."""

    def __init__(self, cos_sin, start: int, pairs: int, device="cuda"):
        t = torch.as_tensor(cos_sin, dtype=torch.float32).to(device).contiguous()
        assert t.dim() == 3 and t.shape[1] == pairs and t.shape[2] == 2
        self.table = t
        self.struct = CSA2Rope(t.data_ptr(), t.shape[0], start, pairs)


_lib = None


def load_library(path: str = LIB_PATH):
    """Load libcsa2.so (building it first only if the sources are newer)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        from .build import build
        build()
    L = C.CDLL(path)
    P, i32, sz = C.c_void_p, C.c_int32, C.c_size_t
    L.csa2_quantize_append.argtypes = [P, P, P, i32, P, P, P, i32, P, P, P]
    L.csa2_quantize_append_rope.argtypes = [P, P, P, i32, P, P, P, i32, P, P, P, P]
    L.csa2_workspace_size.argtypes = [i32] * 7
    L.csa2_workspace_size.restype = sz
    L.csa2_index_full.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, P, P, P, P, sz, P, P]
    L.csa2_index_full_tc.argtypes = L.csa2_index_full.argtypes
    L.csa2_index_reindex.argtypes = [P, P, P, P, i32, i32, P, i32, i32, P, P, P, sz, P, P]
    L.csa2_sparse_attn_decode.argtypes = [P, P, P, P, i32, i32, P, i32, i32, C.c_float, P, P, P,
                                          sz, P, P]
    L.csa2_sparse_attn_decode_append.argtypes = [P, P, P, P, P, i32, i32, P, i32, i32, C.c_float,
                                                 P, P, P, sz, P, P]
    L.csa2_sparse_attn_decode_append_rope.argtypes = [P, P, P, P, P, i32, i32, P, i32, i32,
                                                      C.c_float, P, P, P, P, sz, P, P]
    L.csa2_read_device_error.argtypes = [P, P, P]
    L.csa2_status_string.argtypes = [C.c_int]
    L.csa2_status_string.restype = C.c_char_p
    L.csa2_abi_version.restype = i32
    L.csa2_debug_set_waits.argtypes = [C.c_uint64, i32]
    L.csa2_debug_set_waits.restype = None
    i64 = C.c_int64
    L.csa2_index_full_slice.argtypes = [P, i64, P, P, P, i32, i32, i32, i32, i32, P, P, P, sz, P, P]
    L.csa2_index_merge.argtypes = [P, i32, i32, i32, i32, i64, i64, P, P, P, P]
    L.csa2_attn_combine.argtypes = [P, P, i32, i64, P, P, P]
    for fn in ("csa2_index_full_slice", "csa2_index_merge", "csa2_attn_combine"):
        getattr(L, fn).restype = C.c_int
    L.csa2_quantize_append_paged.argtypes = [P, P, P, i32, P, P, P, i32, P, P, P, P]
    L.csa2_index_full_paged.argtypes = [P, P, P, P, i32, i32, i32, i32, i32, P, P, P, P, sz, P, P]
    L.csa2_index_reindex_paged.argtypes = [P, P, P, P, i32, i32, P, i32, i32, P, P, P, sz, P, P]
    L.csa2_sparse_attn_decode_paged.argtypes = [P, P, P, P, P, i32, i32, P, i32, i32, C.c_float,
                                                P, P, P, P, P]
    L.csa2_sparse_attn_decode_reuse.argtypes = L.csa2_sparse_attn_decode_paged.argtypes
    L.csa2_index_reindex_settled.argtypes = L.csa2_index_reindex.argtypes
    L.csa2_index_reindex_paged_settled.argtypes = L.csa2_index_reindex_paged.argtypes
    L.csa2_sparse_attn_decode_paged_reuse.argtypes = L.csa2_sparse_attn_decode_paged.argtypes
    for fn in ("csa2_quantize_append_paged", "csa2_index_full_paged", "csa2_index_reindex_paged",
               "csa2_sparse_attn_decode_paged", "csa2_sparse_attn_decode_reuse",
               "csa2_index_reindex_settled", "csa2_index_reindex_paged_settled",
               "csa2_sparse_attn_decode_paged_reuse"):
        getattr(L, fn).restype = C.c_int
    for fn in ("csa2_quantize_append", "csa2_quantize_append_rope", "csa2_index_full",
               "csa2_index_full_tc", "csa2_index_reindex", "csa2_sparse_attn_decode",
               "csa2_sparse_attn_decode_append", "csa2_sparse_attn_decode_append_rope",
               "csa2_read_device_error"):
        getattr(L, fn).restype = C.c_int
    _lib = L
    return L


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    assert t.is_contiguous(), "tensors passed to libcsa2 must be contiguous"
    return C.c_void_p(t.data_ptr())


def _stream(stream) -> C.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return C.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn: str, status: int):
    if status != 0:
        raise Csa2Error(fn, status, load_library())


def csa2_workspace_size(op: int, B: int, Tq: int, n_max: int, H: int, top_k: int,
                        pool_blocks: int) -> int:
    return load_library().csa2_workspace_size(op, B, Tq, n_max, H, top_k, pool_blocks)


def csa2_quantize_append(kv: CSA2GlobalKV | None, kv_bf16, idxk_bf16, T_kv: int, kv_start,
                         swa: CSA2SWA | None, swa_bf16, T_swa: int, swa_start, dev_err=None,
                         stream=None):
    L = load_library()
    st = L.csa2_quantize_append(C.byref(kv) if kv is not None else None, _ptr(kv_bf16),
                                _ptr(idxk_bf16), T_kv, _ptr(kv_start),
                                C.byref(swa) if swa is not None else None, _ptr(swa_bf16),
                                T_swa, _ptr(swa_start), _ptr(dev_err), _stream(stream))
    _check("csa2_quantize_append", st)


def csa2_quantize_append_rope(kv: CSA2GlobalKV | None, kv_bf16, idxk_bf16, T_kv: int, kv_start,
                              swa: CSA2SWA | None, swa_bf16, T_swa: int, swa_start,
                              rope: CSA2Rope | None, dev_err=None, stream=None):
    """csa2_quantize_append with RoPE applied to the main-KV and SWA rows first."""
    L = load_library()
    st = L.csa2_quantize_append_rope(C.byref(kv) if kv is not None else None, _ptr(kv_bf16),
                                     _ptr(idxk_bf16), T_kv, _ptr(kv_start),
                                     C.byref(swa) if swa is not None else None, _ptr(swa_bf16),
                                     T_swa, _ptr(swa_start),
                                     C.byref(rope) if rope is not None else None, _ptr(dev_err),
                                     _stream(stream))
    _check("csa2_quantize_append_rope", st)


def csa2_index_full(kv: CSA2GlobalKV, q_idx, w, q_pos, Tq: int, H_I: int, n_max: int,
                    pool_blocks: int, top_k: int, pool_out, topk_out, topk_count, workspace,
                    dev_err=None, stream=None):
    L = load_library()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = L.csa2_index_full(C.byref(kv), _ptr(q_idx), _ptr(w), _ptr(q_pos), Tq, H_I, n_max,
                           pool_blocks, top_k, _ptr(pool_out), _ptr(topk_out), _ptr(topk_count),
                           _ptr(workspace), ws_bytes, _ptr(dev_err), _stream(stream))
    _check("csa2_index_full", st)


def csa2_index_full_tc(kv: CSA2GlobalKV, q_idx, w, q_pos, Tq: int, H_I: int, n_max: int,
                       pool_blocks: int, top_k: int, pool_out, topk_out, topk_count, workspace,
                       dev_err=None, stream=None):
    """csa2_index_full with the scan on the tensor cores (prefill chunks)."""
    L = load_library()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = L.csa2_index_full_tc(C.byref(kv), _ptr(q_idx), _ptr(w), _ptr(q_pos), Tq, H_I, n_max,
                              pool_blocks, top_k, _ptr(pool_out), _ptr(topk_out),
                              _ptr(topk_count), _ptr(workspace), ws_bytes, _ptr(dev_err),
                              _stream(stream))
    _check("csa2_index_full_tc", st)


def csa2_index_full_slice(kv: CSA2GlobalKV, entry_lo: int, q_idx, w, q_pos, Tq: int, H_I: int,
                          n_max: int, pool_blocks: int, top_k: int, pool_keys_out, topk_keys_out,
                          workspace, dev_err=None, stream=None):
    """Context parallel: the Full layer on a slice of the entries, its local selections
    as candidate keys."""
    L = load_library()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = L.csa2_index_full_slice(C.byref(kv), entry_lo, _ptr(q_idx), _ptr(w), _ptr(q_pos), Tq, H_I,
                                 n_max, pool_blocks, top_k, _ptr(pool_keys_out), _ptr(topk_keys_out),
                                 _ptr(workspace), ws_bytes, _ptr(dev_err), _stream(stream))
    _check("csa2_index_full_slice", st)


def csa2_index_merge(lists, BT: int, n_lists: int, list_len: int, k: int, local_lo: int,
                     local_hi: int, ids_out, count_out, local_out, stream=None):
    """Context parallel: the exact selection from the shards' candidate lists."""
    L = load_library()
    st = L.csa2_index_merge(_ptr(lists), BT, n_lists, list_len, k, local_lo, local_hi,
                            _ptr(ids_out), _ptr(count_out), _ptr(local_out), _stream(stream))
    _check("csa2_index_merge", st)


def csa2_attn_combine(o_parts, lse_parts, n_parts: int, rows: int, out, lse_out, stream=None):
    """Context parallel: one softmax from the shards' partial attention results."""
    L = load_library()
    st = L.csa2_attn_combine(_ptr(o_parts), _ptr(lse_parts), n_parts, rows, _ptr(out),
                             _ptr(lse_out), _stream(stream))
    _check("csa2_attn_combine", st)


def csa2_quantize_append_paged(kv: CSA2PagedKV | None, kv_bf16, idxk_bf16, T_kv: int, kv_start,
                               swa: CSA2SWA | None, swa_bf16, T_swa: int, swa_start, rope=None,
                               dev_err=None, stream=None):
    """csa2_quantize_append(_rope) on a paged cache."""
    L = load_library()
    st = L.csa2_quantize_append_paged(C.byref(kv) if kv is not None else None, _ptr(kv_bf16),
                                      _ptr(idxk_bf16), T_kv, _ptr(kv_start),
                                      C.byref(swa) if swa is not None else None, _ptr(swa_bf16),
                                      T_swa, _ptr(swa_start),
                                      C.byref(rope) if rope is not None else None, _ptr(dev_err),
                                      _stream(stream))
    _check("csa2_quantize_append_paged", st)


def csa2_index_full_paged(kv: CSA2PagedKV, q_idx, w, q_pos, Tq: int, H_I: int, n_max: int,
                          pool_blocks: int, top_k: int, pool_out, topk_out, topk_count, workspace,
                          dev_err=None, stream=None):
    """csa2_index_full on a paged cache."""
    L = load_library()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = L.csa2_index_full_paged(C.byref(kv), _ptr(q_idx), _ptr(w), _ptr(q_pos), Tq, H_I, n_max,
                                 pool_blocks, top_k, _ptr(pool_out), _ptr(topk_out),
                                 _ptr(topk_count), _ptr(workspace), ws_bytes, _ptr(dev_err),
                                 _stream(stream))
    _check("csa2_index_full_paged", st)


def csa2_index_reindex_paged(kv: CSA2PagedKV, q_idx, w, q_pos, Tq: int, H_I: int, pool,
                             pool_blocks: int, top_k: int, topk_out, topk_count, workspace,
                             dev_err=None, stream=None):
    """csa2_index_reindex on a paged cache."""
    L = load_library()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = L.csa2_index_reindex_paged(C.byref(kv), _ptr(q_idx), _ptr(w), _ptr(q_pos), Tq, H_I,
                                    _ptr(pool), pool_blocks, top_k, _ptr(topk_out),
                                    _ptr(topk_count), _ptr(workspace), ws_bytes, _ptr(dev_err),
                                    _stream(stream))
    _check("csa2_index_reindex_paged", st)


def csa2_sparse_attn_decode_reuse(kv: CSA2GlobalKV, swa: CSA2SWA | None, swa_bf16, q, q_pos,
                                  Tq: int, H: int, topk, top_k: int, swa_len: int,
                                  softmax_scale: float, rope, out, lse, dev_err=None, stream=None):
    """The sparse attention of a Reuse layer (swa_bf16 None: no fused append), whose
    inputs were all written two or more launches earlier on the stream."""
    L = load_library()
    st = L.csa2_sparse_attn_decode_reuse(
        C.byref(kv), C.byref(swa) if swa is not None else None, _ptr(swa_bf16), _ptr(q), _ptr(q_pos),
        Tq, H, _ptr(topk), top_k, swa_len, softmax_scale, C.byref(rope) if rope is not None else None,
        _ptr(out), _ptr(lse), _ptr(dev_err), _stream(stream))
    _check("csa2_sparse_attn_decode_reuse", st)


def csa2_sparse_attn_decode_paged(kv: CSA2PagedKV, swa: CSA2SWA | None, swa_bf16, q, q_pos,
                                  Tq: int, H: int, topk, top_k: int, swa_len: int,
                                  softmax_scale: float, rope, out, lse, dev_err=None, stream=None):
    """csa2_sparse_attn_decode (swa_bf16 None) or its fused-append form on a paged cache."""
    L = load_library()
    st = L.csa2_sparse_attn_decode_paged(C.byref(kv), C.byref(swa) if swa is not None else None,
                                         _ptr(swa_bf16), _ptr(q), _ptr(q_pos), Tq, H, _ptr(topk),
                                         top_k, swa_len, softmax_scale,
                                         C.byref(rope) if rope is not None else None, _ptr(out),
                                         _ptr(lse), _ptr(dev_err), _stream(stream))
    _check("csa2_sparse_attn_decode_paged", st)


def csa2_index_reindex(kv: CSA2GlobalKV, q_idx, w, q_pos, Tq: int, H_I: int, pool,
                       pool_blocks: int, top_k: int, topk_out, topk_count, workspace,
                       dev_err=None, stream=None):
    L = load_library()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = L.csa2_index_reindex(C.byref(kv), _ptr(q_idx), _ptr(w), _ptr(q_pos), Tq, H_I,
                              _ptr(pool), pool_blocks, top_k, _ptr(topk_out), _ptr(topk_count),
                              _ptr(workspace), ws_bytes, _ptr(dev_err), _stream(stream))
    _check("csa2_index_reindex", st)


def csa2_index_reindex_paged_settled(kv: CSA2PagedKV, q_idx, w, q_pos, Tq: int, H_I: int, pool,
                                     pool_blocks: int, top_k: int, topk_out, topk_count, workspace,
                                     dev_err=None, stream=None):
    """csa2_index_reindex_settled on a paged cache."""
    L = load_library()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = L.csa2_index_reindex_paged_settled(C.byref(kv), _ptr(q_idx), _ptr(w), _ptr(q_pos), Tq, H_I,
                                            _ptr(pool), pool_blocks, top_k, _ptr(topk_out),
                                            _ptr(topk_count), _ptr(workspace), ws_bytes, _ptr(dev_err),
                                            _stream(stream))
    _check("csa2_index_reindex_paged_settled", st)


def csa2_sparse_attn_decode_paged_reuse(kv: CSA2PagedKV, swa: CSA2SWA | None, swa_bf16, q, q_pos,
                                        Tq: int, H: int, topk, top_k: int, swa_len: int,
                                        softmax_scale: float, rope, out, lse, dev_err=None, stream=None):
    """csa2_sparse_attn_decode_reuse on a paged cache."""
    L = load_library()
    st = L.csa2_sparse_attn_decode_paged_reuse(
        C.byref(kv), C.byref(swa) if swa is not None else None, _ptr(swa_bf16), _ptr(q), _ptr(q_pos),
        Tq, H, _ptr(topk), top_k, swa_len, softmax_scale, C.byref(rope) if rope is not None else None,
        _ptr(out), _ptr(lse), _ptr(dev_err), _stream(stream))
    _check("csa2_sparse_attn_decode_paged_reuse", st)


def csa2_index_reindex_settled(kv: CSA2GlobalKV, q_idx, w, q_pos, Tq: int, H_I: int, pool,
                               pool_blocks: int, top_k: int, topk_out, topk_count, workspace,
                               dev_err=None, stream=None):
    """csa2_index_reindex whose scoring overlaps the previous launch on the stream (every
    input written two or more launches earlier)."""
    L = load_library()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = L.csa2_index_reindex_settled(C.byref(kv), _ptr(q_idx), _ptr(w), _ptr(q_pos), Tq, H_I,
                                      _ptr(pool), pool_blocks, top_k, _ptr(topk_out), _ptr(topk_count),
                                      _ptr(workspace), ws_bytes, _ptr(dev_err), _stream(stream))
    _check("csa2_index_reindex_settled", st)


def csa2_sparse_attn_decode(kv: CSA2GlobalKV, swa: CSA2SWA | None, q, q_pos, Tq: int, H: int,
                            topk, top_k: int, swa_len: int, softmax_scale: float, out, lse,
                            workspace=None, dev_err=None, stream=None):
    L = load_library()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = L.csa2_sparse_attn_decode(C.byref(kv), C.byref(swa) if swa is not None else None,
                                   _ptr(q), _ptr(q_pos), Tq, H, _ptr(topk), top_k, swa_len,
                                   softmax_scale, _ptr(out), _ptr(lse), _ptr(workspace),
                                   ws_bytes, _ptr(dev_err), _stream(stream))
    _check("csa2_sparse_attn_decode", st)


def csa2_sparse_attn_decode_append(kv: CSA2GlobalKV, swa: CSA2SWA, swa_bf16, q, q_pos, Tq: int,
                                   H: int, topk, top_k: int, swa_len: int, softmax_scale: float,
                                   out, lse, workspace=None, dev_err=None, stream=None):
    """SWA append of the query token (Tq = 1) fused with csa2_sparse_attn_decode."""
    L = load_library()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = L.csa2_sparse_attn_decode_append(C.byref(kv), C.byref(swa) if swa is not None else None,
                                          _ptr(swa_bf16), _ptr(q), _ptr(q_pos), Tq, H, _ptr(topk),
                                          top_k, swa_len, softmax_scale, _ptr(out), _ptr(lse),
                                          _ptr(workspace), ws_bytes, _ptr(dev_err), _stream(stream))
    _check("csa2_sparse_attn_decode_append", st)


def csa2_debug_set_waits(limit_ns: int, stuck_wait: bool) -> None:
    """Test hook of the kernels' bounded waits (see include/csa2.h)."""
    load_library().csa2_debug_set_waits(int(limit_ns), 1 if stuck_wait else 0)


def csa2_read_device_error(dev_err, stream=None) -> int:
    """Synchronises the stream; returns the device error bits (0 = none) and resets them."""
    L = load_library()
    bits = C.c_int32(0)
    st = L.csa2_read_device_error(_ptr(dev_err), C.byref(bits), _stream(stream))
    if st not in (0, 6):
        _check("csa2_read_device_error", st)
    return bits.value


def csa2_sparse_attn_decode_append_rope(kv: CSA2GlobalKV, swa: CSA2SWA, swa_bf16, q, q_pos,
                                        Tq: int, H: int, topk, top_k: int, swa_len: int,
                                        softmax_scale: float, rope: CSA2Rope | None, out, lse,
                                        workspace=None, dev_err=None, stream=None):
    """csa2_sparse_attn_decode_append with RoPE applied to the new SWA row first."""
    L = load_library()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = L.csa2_sparse_attn_decode_append_rope(
        C.byref(kv), C.byref(swa), _ptr(swa_bf16), _ptr(q), _ptr(q_pos), Tq, H, _ptr(topk), top_k,
        swa_len, softmax_scale, C.byref(rope) if rope is not None else None, _ptr(out), _ptr(lse),
        _ptr(workspace), ws_bytes, _ptr(dev_err), _stream(stream))
    _check("csa2_sparse_attn_decode_append_rope", st)
