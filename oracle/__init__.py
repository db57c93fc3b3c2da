"""CPU oracle of the CSA2 decode path (ctypes front end of csa2_oracle.c).

TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU
baseline leg may import this package.  It shares no code with the CUDA path:
it takes bf16 inputs and computes the quantised caches, index scores,
selections and attention outputs itself.

All arrays are numpy; bf16 tensors travel as uint16 bit patterns.
"""
from __future__ import annotations

import ctypes as C

import numpy as np

from .build import build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = build()
        L = C.CDLL(path)
        P = C.c_void_p
        i32, i64, f32, f64 = C.c_int32, C.c_int64, C.c_float, C.c_double
        sig = {
            "csa2o_bf16_to_f32": (f32, [C.c_uint16]),
            "csa2o_f32_to_bf16": (C.c_uint16, [f32]),
            "csa2o_rope_rows": (i64, [P, i64, C.c_int, P, P, i64, C.c_int, C.c_int, P]),
            "csa2o_e2m1_value": (f64, [C.c_int]),
            "csa2o_e4m3_value": (f64, [C.c_int]),
            "csa2o_e2m1_encode": (C.c_int, [f32]),
            "csa2o_e4m3_encode": (C.c_int, [f32]),
            "csa2o_quantize_fp4": (None, [P, i64, C.c_int, P, P]),
            "csa2o_quantize_fp8": (None, [P, i64, C.c_int, P, P]),
            "csa2o_dequant_fp4": (None, [P, P, i64, C.c_int, P]),
            "csa2o_dequant_fp8": (None, [P, P, i64, C.c_int, P]),
            "csa2o_visible": (i64, [i64, C.c_int]),
            "csa2o_scores": (None, [P, P, C.c_int, P, i64, P, P, C.c_int, P]),
            "csa2o_scores_f64": (None, [P, P, C.c_int, P, i64, P, P, C.c_int, P, P]),
            "csa2o_block_max": (None, [P, i64, P]),
            "csa2o_select_topk": (i64, [P, P, i64, i64, P]),
            "csa2o_index_full_one": (i32, [P, P, C.c_int, i64, P, P, C.c_int, C.c_int, C.c_int,
                                           P, P, P]),
            "csa2o_index_reindex_one": (i32, [P, P, C.c_int, i64, P, P, C.c_int, P, C.c_int,
                                              C.c_int, P]),
            "csa2o_attention_one": (None, [P, P, P, P, C.c_int, P, C.c_int, i64, P, C.c_int,
                                           C.c_int, f64, P, P]),
            "csa2o_index_full": (None, [P, P, C.c_int, i64, C.c_int, C.c_int, P, P, P, C.c_int,
                                        C.c_int, C.c_int, C.c_int, P, P, P]),
            "csa2o_index_reindex": (None, [P, P, C.c_int, i64, C.c_int, C.c_int, P, P, P,
                                           C.c_int, C.c_int, P, C.c_int, C.c_int, P, P]),
            "csa2o_attention": (None, [P, P, C.c_int, i64, P, P, C.c_int, P, P, C.c_int, C.c_int,
                                       P, C.c_int, C.c_int, f64, P, P]),
            "csa2o_num_threads": (C.c_int, []),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def as_bf16_bits(x) -> np.ndarray:
    """torch bf16 tensor or uint16 array -> contiguous uint16 numpy array."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy()
                                .view(np.uint16))


# ---- formats --------------------------------------------------------------------------------
def e2m1_value(code: int) -> float:
    return lib().csa2o_e2m1_value(code)


def e4m3_value(code: int) -> float:
    return lib().csa2o_e4m3_value(code)


def e2m1_encode(r: float) -> int:
    return lib().csa2o_e2m1_encode(r)


def e4m3_encode(x: float) -> int:
    return lib().csa2o_e4m3_encode(x)


def f32_to_bf16(v: float) -> int:
    return lib().csa2o_f32_to_bf16(v)


def rope_rows(x, pos, cos_sin: np.ndarray, start: int, pairs: int) -> tuple[np.ndarray, int]:
    """bf16 rows [..., W] at token positions pos [...] -> (rotated bf16 rows as uint16,
    number of rows whose position is outside the table and stay unrotated)."""
    xb = as_bf16_bits(x)
    shape = xb.shape
    W = shape[-1]
    xb = np.ascontiguousarray(xb.reshape(-1, W))
    pos = np.ascontiguousarray(np.asarray(pos, np.int64).reshape(-1))
    assert len(pos) == xb.shape[0]
    cs = np.ascontiguousarray(cos_sin, np.float32)
    assert cs.shape[1:] == (pairs, 2)
    out = np.zeros_like(xb)
    n_out = lib().csa2o_rope_rows(_p(xb), xb.shape[0], W, _p(pos), _p(cs), cs.shape[0], start,
                                  pairs, _p(out))
    return out.reshape(shape), n_out


# ---- a1 / a2 --------------------------------------------------------------------------------
def quantize_fp4(x) -> tuple[np.ndarray, np.ndarray]:
    """bf16 [..., W] -> (codes u8 [..., W/2], scales u8 [..., W/16])."""
    xb = as_bf16_bits(x)
    W = xb.shape[-1]
    rows = xb.size // W
    codes = np.zeros(xb.shape[:-1] + (W // 2,), np.uint8)
    scales = np.zeros(xb.shape[:-1] + (W // 16,), np.uint8)
    lib().csa2o_quantize_fp4(_p(xb), rows, W, _p(codes), _p(scales))
    return codes, scales


def quantize_fp8(x) -> tuple[np.ndarray, np.ndarray]:
    """bf16 [..., W] -> (codes u8 [..., W], sigma f32 [...])."""
    xb = as_bf16_bits(x)
    W = xb.shape[-1]
    rows = xb.size // W
    codes = np.zeros(xb.shape, np.uint8)
    scale = np.zeros(xb.shape[:-1], np.float32)
    lib().csa2o_quantize_fp8(_p(xb), rows, W, _p(codes), _p(scale))
    return codes, scale


def dequant_fp4(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes)
    scales = np.ascontiguousarray(scales)
    W = codes.shape[-1] * 2
    rows = codes.size // codes.shape[-1]
    out = np.zeros(codes.shape[:-1] + (W,), np.float64)
    lib().csa2o_dequant_fp4(_p(codes), _p(scales), rows, W, _p(out))
    return out


def dequant_fp8(codes: np.ndarray, scale: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes)
    scale = np.ascontiguousarray(scale, dtype=np.float32)
    W = codes.shape[-1]
    out = np.zeros(codes.shape, np.float64)
    lib().csa2o_dequant_fp8(_p(codes), _p(scale), codes.size // W, W, _p(out))
    return out


def visible(t: int, ratio: int) -> int:
    return lib().csa2o_visible(t, ratio)


# ---- a3 - a6 --------------------------------------------------------------------------------
def scores(kc: np.ndarray, ks: np.ndarray, q, w: np.ndarray, pos: np.ndarray | None = None,
           n: int | None = None) -> np.ndarray:
    """Canonical fp32 index scores of positions `pos` (or 0..n-1) for one query."""
    kc = np.ascontiguousarray(kc, np.uint8)
    ks = np.ascontiguousarray(ks, np.float32)
    qb = as_bf16_bits(q)
    w = np.ascontiguousarray(w, np.float32)
    H_I, d = qb.shape
    if pos is not None:
        pos = np.ascontiguousarray(pos, np.int32)
        n = len(pos)
    out = np.zeros(n, np.float32)
    lib().csa2o_scores(_p(kc), _p(ks), d, _p(pos), n, _p(qb), _p(w), H_I, _p(out))
    return out


def scores_f64(kc: np.ndarray, ks: np.ndarray, q, w: np.ndarray, pos: np.ndarray | None = None,
               n: int | None = None) -> tuple[np.ndarray, np.ndarray]:
    """Index scores without fp32 rounding, for one query: (score f64 [n], magnitude
    f64 [n]), magnitude = sigma_s * sum_h w_h * sum_c |q_hc * k_sc|, which bounds the
    rounding error of any fp32 summation order of the score."""
    kc = np.ascontiguousarray(kc, np.uint8)
    ks = np.ascontiguousarray(ks, np.float32)
    qb = as_bf16_bits(q)
    w = np.ascontiguousarray(w, np.float32)
    H_I, d = qb.shape
    if pos is not None:
        pos = np.ascontiguousarray(pos, np.int32)
        n = len(pos)
    out = np.zeros(n, np.float64)
    mag = np.zeros(n, np.float64)
    lib().csa2o_scores_f64(_p(kc), _p(ks), d, _p(pos), n, _p(qb), _p(w), H_I, _p(out), _p(mag))
    return out, mag


def block_max(sc: np.ndarray) -> np.ndarray:
    sc = np.ascontiguousarray(sc, np.float32)
    out = np.zeros((len(sc) + 7) // 8, np.float32)
    lib().csa2o_block_max(_p(sc), len(sc), _p(out))
    return out


def select_topk(vals: np.ndarray, k: int, ids: np.ndarray | None = None) -> np.ndarray:
    vals = np.ascontiguousarray(vals, np.float32)
    if ids is not None:
        ids = np.ascontiguousarray(ids, np.int32)
    out = np.zeros(max(k, 1), np.int32)
    m = lib().csa2o_select_topk(_p(vals), _p(ids), len(vals), k, _p(out))
    return out[:m].copy()


def index_full_one(kc, ks, q, w, N: int, pool_blocks: int, top_k: int):
    """One query: returns (pool [pool_blocks] or None, topk [top_k], count, scores [N])."""
    kc = np.ascontiguousarray(kc, np.uint8)
    ks = np.ascontiguousarray(ks, np.float32)
    qb = as_bf16_bits(q)
    w = np.ascontiguousarray(w, np.float32)
    H_I, d = qb.shape
    pool = np.full(max(pool_blocks, 1), -1, np.int32)
    topk = np.full(max(top_k, 1), -1, np.int32)
    sc = np.zeros(max(N, 1), np.float32)
    cnt = lib().csa2o_index_full_one(_p(kc), _p(ks), d, N, _p(qb), _p(w), H_I, pool_blocks,
                                     top_k, _p(pool) if pool_blocks else None, _p(topk), _p(sc))
    return (pool[:pool_blocks] if pool_blocks else None), topk[:top_k], cnt, sc[:N]


def index_reindex_one(kc, ks, q, w, N: int, pool: np.ndarray, top_k: int):
    kc = np.ascontiguousarray(kc, np.uint8)
    ks = np.ascontiguousarray(ks, np.float32)
    qb = as_bf16_bits(q)
    w = np.ascontiguousarray(w, np.float32)
    pool = np.ascontiguousarray(pool, np.int32)
    H_I, d = qb.shape
    topk = np.full(max(top_k, 1), -1, np.int32)
    cnt = lib().csa2o_index_reindex_one(_p(kc), _p(ks), d, N, _p(qb), _p(w), H_I, _p(pool),
                                        len(pool), top_k, _p(topk))
    return topk[:top_k], cnt


def attention_one(main_codes, main_scales, swa_codes, swa_scale, q, t: int, topk,
                  swa_len: int, softmax_scale: float):
    """One query: returns (o [H][512] fp64, lse [H] fp64)."""
    mc = np.ascontiguousarray(main_codes, np.uint8)
    ms = np.ascontiguousarray(main_scales, np.uint8)
    sc = np.ascontiguousarray(swa_codes, np.uint8)
    ss = np.ascontiguousarray(swa_scale, np.float32)
    qb = as_bf16_bits(q)
    topk = np.ascontiguousarray(topk, np.int32)
    H = qb.shape[0]
    W = sc.shape[0]
    out = np.zeros((H, 512), np.float64)
    lse = np.zeros(H, np.float64)
    lib().csa2o_attention_one(_p(mc), _p(ms), _p(sc), _p(ss), W, _p(qb), H, t, _p(topk),
                              len(topk), swa_len, softmax_scale, _p(out), _p(lse))
    return out, lse


# ---- batched, in the library's layout -------------------------------------------------------
def index_full(kc, ks, ratio: int, q, w, q_pos, pool_blocks: int, top_k: int):
    """kc u8 [B][cap][d], ks f32 [B][cap], q bf16 [B][Tq][H_I][d], w f32 [B][Tq][H_I],
    q_pos i32 [B][Tq] -> (pool [B][Tq][P] or None, topk [B][Tq][K], count [B][Tq])."""
    kc = np.ascontiguousarray(kc, np.uint8)
    ks = np.ascontiguousarray(ks, np.float32)
    qb = as_bf16_bits(q)
    w = np.ascontiguousarray(w, np.float32)
    q_pos = np.ascontiguousarray(q_pos, np.int32)
    B, cap, d = kc.shape
    _, Tq, H_I, _ = qb.shape
    pool = np.full((B, Tq, max(pool_blocks, 1)), -1, np.int32)
    topk = np.full((B, Tq, top_k), -1, np.int32)
    cnt = np.zeros((B, Tq), np.int32)
    lib().csa2o_index_full(_p(kc), _p(ks), B, cap, d, ratio, _p(qb), _p(w), _p(q_pos), Tq, H_I,
                           pool_blocks, top_k, _p(pool) if pool_blocks else None, _p(topk),
                           _p(cnt))
    return (pool if pool_blocks else None), topk, cnt


def index_reindex(kc, ks, ratio: int, q, w, q_pos, pool, top_k: int):
    kc = np.ascontiguousarray(kc, np.uint8)
    ks = np.ascontiguousarray(ks, np.float32)
    qb = as_bf16_bits(q)
    w = np.ascontiguousarray(w, np.float32)
    q_pos = np.ascontiguousarray(q_pos, np.int32)
    pool = np.ascontiguousarray(pool, np.int32)
    B, cap, d = kc.shape
    _, Tq, H_I, _ = qb.shape
    topk = np.full((B, Tq, top_k), -1, np.int32)
    cnt = np.zeros((B, Tq), np.int32)
    lib().csa2o_index_reindex(_p(kc), _p(ks), B, cap, d, ratio, _p(qb), _p(w), _p(q_pos), Tq,
                              H_I, _p(pool), pool.shape[-1], top_k, _p(topk), _p(cnt))
    return topk, cnt


def attention(main_codes, main_scales, swa_codes, swa_scale, q, q_pos, topk, swa_len: int,
              softmax_scale: float):
    """main_codes [B][cap][256], main_scales [B][cap][32], swa_codes [B][W][512],
    swa_scale [B][W], q bf16 [B][Tq][H][512], q_pos [B][Tq], topk [B][Tq][K]
    -> (o f64 [B][Tq][H][512], lse f64 [B][Tq][H])."""
    mc = np.ascontiguousarray(main_codes, np.uint8)
    ms = np.ascontiguousarray(main_scales, np.uint8)
    sc = np.ascontiguousarray(swa_codes, np.uint8)
    ss = np.ascontiguousarray(swa_scale, np.float32)
    qb = as_bf16_bits(q)
    q_pos = np.ascontiguousarray(q_pos, np.int32)
    topk = np.ascontiguousarray(topk, np.int32)
    B, cap, _ = mc.shape
    W = sc.shape[1]
    _, Tq, H, _ = qb.shape
    out = np.zeros((B, Tq, H, 512), np.float64)
    lse = np.zeros((B, Tq, H), np.float64)
    lib().csa2o_attention(_p(mc), _p(ms), B, cap, _p(sc), _p(ss), W, _p(qb), _p(q_pos), Tq, H,
                          _p(topk), topk.shape[-1], swa_len, softmax_scale, _p(out), _p(lse))
    return out, lse


def num_threads() -> int:
    return lib().csa2o_num_threads()
