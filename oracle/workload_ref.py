"""Oracle-side reference of one request of a workload (host only).

TEST INFRASTRUCTURE, like the rest of this package: only the tests, the smoke
check and the benchmark's CPU baseline leg / reference arm use it.

Regenerates the request's bf16 inputs with the seeded generator and runs the
CPU oracle on them: caches, every selector layer's pool / Top-K, and the
attention of the requested layers.  Imports nothing of the CUDA path.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle as orc
from synth.workloads import Workload

SOFTMAX_SCALE = 1.0 / math.sqrt(512)


def reuse_sources(wl: Workload) -> list[tuple[int, str, int]]:
    """(group, mode, source layer) per layer: a Reuse layer attends with the
    selection of the nearest preceding Full/Reindex layer of its group."""
    out, layer = [], 0
    for g, grp in enumerate(wl.groups):
        last = None
        for m in grp.schedule:
            if m in "FX":
                last = layer
            out.append((g, m, last))
            layer += 1
    return out


def request_caches(wl: Workload, b: int, main_rows: dict[int, np.ndarray] | None = None):
    """Index caches (full), main-KV caches (all rows, or only `main_rows[g]`), and the
    SWA rings of request b as they stand after the step."""
    groups = []
    for g, grp in enumerate(wl.groups):
        N = wl.entries(g)
        kc, ks = orc.quantize_fp8(wl.idx_k(g, b, 0, N))
        codes = np.zeros((N, 256), np.uint8)
        scales = np.zeros((N, 32), np.uint8)
        rows = np.arange(N) if main_rows is None else np.unique(main_rows[g])
        rows = rows[(rows >= 0) & (rows < N)]
        if main_rows is None:
            c, s = orc.quantize_fp4(wl.main_kv(g, b, 0, N))
            codes[:], scales[:] = c, s
        else:
            for r in rows:
                c, s = orc.quantize_fp4(wl.main_kv(g, b, int(r), 1))
                codes[r], scales[r] = c[0], s[0]
        groups.append(dict(N=N, idx_codes=kc, idx_scale=ks, codes=codes, scales=scales,
                           rows=rows))
    return groups


def swa_ring(wl: Workload, layer: int, b: int):
    W = wl.window_cap
    t_first = wl.first_q_pos
    t_last = wl.ctx - 1
    p0 = max(0, t_first - wl.swa_len + 1)
    codes = np.zeros((W, 512), np.uint8)
    scale = np.zeros(W, np.float32)
    rows = wl.swa(layer, b, p0, t_last - p0 + 1)
    c, s = orc.quantize_fp8(rows)
    for i, p in enumerate(range(p0, t_last + 1)):
        codes[p % W], scale[p % W] = c[i], s[i]
    return codes, scale


def index_layers(wl: Workload, b: int, caches, q_pos: np.ndarray | None = None,
                 qsel: np.ndarray | None = None):
    """Pool / Top-K / count of every Full and Reindex layer of request b (of the query
    tokens qsel only, when given: queries are independent given the caches)."""
    q_pos = np.asarray(wl.q_positions() if q_pos is None else q_pos, np.int32)
    sel = slice(None) if qsel is None else np.asarray(qsel)
    q_pos = np.ascontiguousarray(q_pos[sel])
    res = {"topk": {}, "count": {}, "pool": {}}
    pool = {}
    for layer, (g, m, src) in enumerate(reuse_sources(wl)):
        grp = wl.groups[g]
        c = caches[g]
        if m in "FX":
            qi = wl.q_idx(layer, b)[sel].contiguous()
            w = np.ascontiguousarray(wl.w(layer, b)[sel].numpy())
        if m == "F":
            p, t, n = orc.index_full(c["idx_codes"][None], c["idx_scale"][None], grp.ratio,
                                     qi[None], w[None], q_pos[None], grp.pool_blocks, wl.top_k)
            if p is not None:
                pool[g] = p
                res["pool"][g] = p[0]
            res["topk"][layer], res["count"][layer] = t[0], n[0]
        elif m == "X":
            t, n = orc.index_reindex(c["idx_codes"][None], c["idx_scale"][None], grp.ratio,
                                     qi[None], w[None], q_pos[None], pool[g], wl.top_k)
            res["topk"][layer], res["count"][layer] = t[0], n[0]
    return res


def attention_layer(wl: Workload, b: int, layer: int, caches, topk: np.ndarray,
                    q_pos: np.ndarray | None = None, qsel: np.ndarray | None = None):
    """Attention of one layer for request b (query tokens qsel only, when given; topk
    then holds those queries' selections)."""
    q_pos = np.asarray(wl.q_positions() if q_pos is None else q_pos, np.int32)
    sel = slice(None) if qsel is None else np.asarray(qsel)
    q_pos = np.ascontiguousarray(q_pos[sel])
    g = reuse_sources(wl)[layer][0]
    c = caches[g]
    ring_c, ring_s = swa_ring(wl, layer, b)
    o, lse = orc.attention(c["codes"][None], c["scales"][None], ring_c[None], ring_s[None],
                           wl.q(layer, b)[sel].contiguous()[None], q_pos[None],
                           np.ascontiguousarray(topk)[None], wl.swa_len, SOFTMAX_SCALE)
    return o[0], lse[0]


def rel_err_rows(o: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Norm-wise error per row: max_c |o - ref| / max_c |ref| (rows = leading dims)."""
    o = o.reshape(-1, o.shape[-1]).astype(np.float64)
    ref = ref.reshape(-1, ref.shape[-1])
    den = np.abs(ref).max(-1)
    num = np.abs(o - ref).max(-1)
    return np.where(den > 0, num / np.where(den > 0, den, 1), num)


def rel_err_elems(o: np.ndarray, ref: np.ndarray) -> float:
    """Largest elementwise relative error |o - ref| / |ref| over the elements whose
    |ref| is at least the RMS of their row (the companion figure of the norm-wise
    error; rows = leading dims).  0.0 when no element qualifies."""
    o = o.reshape(-1, o.shape[-1]).astype(np.float64)
    ref = ref.reshape(-1, ref.shape[-1]).astype(np.float64)
    rms = np.sqrt((ref * ref).mean(-1, keepdims=True))
    big = (np.abs(ref) >= rms) & (rms > 0)
    if not big.any():
        return 0.0
    return float((np.abs(o - ref)[big] / np.abs(ref)[big]).max())
