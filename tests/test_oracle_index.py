"""Pins of the oracle's index path: score, block key, pool, Top-K, Reindex, Reuse.

The score's fp32 order is checked against exact rational arithmetic with one
correct rounding per operation; the formula against fp64 within the fp32 error
bound and one-hot special cases; selection against numpy's lexsort brute force;
and the Full / Reindex / Reuse structure against the bounds the pages print
(pool <= 2048 x 8 = 16384 positions, <= 512 selected) and the pool lemma.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

from conftest import golden_lines
from exact_fp32 import add32, f, fma32, mul32

import synth
from synth.workloads import WORKLOADS, small_variant


def e4m3_exact(code: int) -> Fraction:
    v = torch.tensor([code], dtype=torch.uint8).view(torch.float8_e4m3fn).double().item()
    return Fraction(v)


def random_index_rows(n, d, seed, scale=1.0):
    x = synth.rows_normal_bf16(seed, "k", 0, 0, n, d)
    return (x.float() * scale).to(torch.bfloat16)


def exact_score(q, w, kcodes, sigma):
    """The stated fp32 order, evaluated in exact rationals with one rounding per op."""
    H_I, d = q.shape
    t = Fraction(0)
    for h in range(H_I):
        e = Fraction(0)
        o = Fraction(0)
        for c in range(0, d, 2):
            e = fma32(f(q[h, c]), e4m3_exact(int(kcodes[c])), e)
            o = fma32(f(q[h, c + 1]), e4m3_exact(int(kcodes[c + 1])), o)
        a = add32(e, o)
        r = a if a > 0 else Fraction(0)
        t = fma32(f(w[h]), r, t)
    return mul32(t, f(sigma))


def test_score_order_exact_rational(orc):
    d, H_I, n = 64, 4, 24
    k = random_index_rows(n, d, 21, 2.0)
    kc, ks = orc.quantize_fp8(k)
    q = synth.rows_normal_bf16(22, "q", 0, 0, H_I, d)
    w = synth.rows_uniform_f32(23, "w", 0, 0, 1, H_I)[0].numpy()
    sc = orc.scores(kc, ks, q, w, n=n)
    qf = q.float().numpy()
    for s in range(n):
        assert Fraction(float(sc[s])) == exact_score(qf, w, kc[s], ks[s]), s


def test_score_formula_fp64_bound_and_one_hot(orc):
    d, H_I, n = 128, 4, 256
    k = random_index_rows(n, d, 31)
    kc, ks = orc.quantize_fp8(k)
    q = synth.rows_normal_bf16(32, "q", 0, 0, H_I, d)
    w = synth.rows_uniform_f32(33, "w", 0, 0, 1, H_I)[0].numpy()
    sc = orc.scores(kc, ks, q, w, n=n).astype(np.float64)
    kd = orc.dequant_fp8(kc, ks)                        # exact dequantised values
    dots = q.double().numpy() @ kd.T                    # [H_I][n] fp64
    ref = (w[:, None].astype(np.float64) * np.maximum(dots, 0)).sum(0)
    absdot = (np.abs(q.double().numpy()) @ np.abs(kd.T))
    bound = (d + 8) * 2 ** -24 * (w[:, None] * absdot).sum(0) * 1.01
    assert np.all(np.abs(sc - ref) <= bound + 1e-30)
    # one-hot: k = e_c (code 0x38 = 1.0, sigma 1), w = e_h -> score = relu(q[h,c])
    for h in range(H_I):
        for c in (0, 1, 63, 126, 127):
            kc1 = np.zeros((1, d), np.uint8)
            kc1[0, c] = 0x38
            w1 = np.zeros(H_I, np.float32)
            w1[h] = 1.0
            s = orc.scores(kc1, np.ones(1, np.float32), q, w1, n=1)[0]
            assert s == max(float(q[h, c]), 0.0)


def test_scores_f64_exact_rational_and_bound(orc):
    """The unrounded score (used for scans that sum in another order) equals the
    exact rational score of the definition, its magnitude equals the exact sum of
    |products|, and the canonical fp32 score lies within (d + H_I + 1) * 2^-24 of
    that magnitude from it."""
    d, H_I, n = 64, 4, 16
    k = random_index_rows(n, d, 24, 3.0)
    kc, ks = orc.quantize_fp8(k)
    q = synth.rows_normal_bf16(25, "q", 0, 0, H_I, d)
    q[2, 5] = -q[2, 5]
    w = synth.rows_uniform_f32(26, "w", 0, 0, 1, H_I)[0].numpy()
    sc, mag = orc.scores_f64(kc, ks, q, w, n=n)
    qf = q.float().numpy()
    for s in range(n):
        t = Fraction(0)
        m = Fraction(0)
        for h in range(H_I):
            prods = [f(qf[h, c]) * e4m3_exact(int(kc[s, c])) for c in range(d)]
            a = sum(prods, Fraction(0))
            t += f(w[h]) * max(a, Fraction(0))
            m += f(w[h]) * sum((abs(p) for p in prods), Fraction(0))
        t *= f(ks[s])
        m *= f(ks[s])
        assert abs(Fraction(float(sc[s])) - t) <= abs(t) * Fraction(1, 2 ** 50), s
        assert abs(Fraction(float(mag[s])) - m) <= m * Fraction(1, 2 ** 50), s
    sc32 = orc.scores(kc, ks, q, w, n=n).astype(np.float64)
    assert np.all(np.abs(sc32 - sc) <= (d + H_I + 1) * 2.0 ** -24 * mag * 1.001 + 1e-300)
    # a subset of positions gives the same values
    pos = np.array([15, 0, 7], np.int32)
    sp, mp = orc.scores_f64(kc, ks, q, w, pos=pos)
    assert np.array_equal(sp, sc[pos]) and np.array_equal(mp, mag[pos])


def test_block_max(orc):
    sc = np.random.default_rng(1).standard_normal(83).astype(np.float32)
    bm = orc.block_max(sc)
    pad = np.concatenate([sc, np.full(88 - 83, -np.inf, np.float32)])
    assert np.array_equal(bm, pad.reshape(11, 8).max(1))


@pytest.mark.parametrize("n,k", [(0, 4), (5, 8), (100, 17), (4096, 512)])
def test_select_matches_lexsort(orc, n, k):
    rng = np.random.default_rng(n + k)
    v = rng.standard_normal(n).astype(np.float32)
    v[rng.random(n) < 0.3] = 0.0                        # heavy ties at zero
    v[rng.random(n) < 0.05] = -0.0                      # -0 ties with +0
    if n > 10:
        v[3] = np.nan
    out = orc.select_topk(v, k)
    key = np.where(np.isnan(v), -np.inf, v)
    order = np.lexsort((np.arange(n), -key))            # value desc, index asc
    assert np.array_equal(out, np.sort(order[:min(k, n)]))


def _decoder_small(ctx=2048, B=2, seed_cfg="decoder_group_32k"):
    return small_variant(WORKLOADS[seed_cfg], B=B, ctx=ctx)


def test_full_pool_bounds_and_lemma(orc):
    inv = dict(ln.split() for ln in golden_lines("format_invariants.txt"))
    assert int(inv["pool_blocks"]) * int(inv["block_positions"]) == int(inv["pool_positions"])
    # the lemma needs pool_blocks >= top_k (2048 >= 512 on the pages)
    for N, P, K in [(1000, 64, 64), (5000, 64, 16), (20000, 2048, 512), (7, 4, 3), (1, 2, 1)]:
        k = random_index_rows(N, 64, N)
        kc, ks = orc.quantize_fp8(k)
        q = synth.rows_normal_bf16(N + 1, "q", 0, 0, 4, 64)
        w = synth.rows_uniform_f32(N + 2, "w", 0, 0, 1, 4)[0].numpy()
        pool, topk, cnt, sc = orc.index_full_one(kc, ks, q, w, N, P, K)
        nb = (N + 7) // 8
        assert (pool >= 0).sum() == min(P, nb)
        assert 8 * (pool >= 0).sum() <= 8 * P
        assert cnt == min(K, N) and (topk >= 0).sum() == cnt
        valid = topk[:cnt]
        assert np.all(np.diff(valid) > 0)
        assert set((valid // 8).tolist()) <= set(pool[pool >= 0].tolist())   # Top-K in pool
        # Top-K from the pool alone equals Top-K over everything
        cand = np.concatenate([np.arange(8 * b, min(8 * b + 8, N)) for b in pool[pool >= 0]])
        sub = orc.select_topk(sc[cand], K, cand.astype(np.int32))
        assert np.array_equal(sub, valid)


def test_full_flat_top_k_cap(orc):
    inv = dict(ln.split() for ln in golden_lines("format_invariants.txt"))
    kmax = int(inv["top_k_max"])
    N = 3000
    k = random_index_rows(N, 128, 77)
    kc, ks = orc.quantize_fp8(k)
    q = synth.rows_normal_bf16(78, "q", 0, 0, 4, 128)
    w = synth.rows_uniform_f32(79, "w", 0, 0, 1, 4)[0].numpy()
    pool, topk, cnt, sc = orc.index_full_one(kc, ks, q, w, N, 0, kmax)
    assert pool is None and cnt == kmax
    assert np.array_equal(topk, orc.select_topk(sc, kmax))


def test_planted_positions_selected(orc):
    wl = _decoder_small(ctx=4096, B=2)
    g = wl.decoder_group
    L = wl.decoder_full_layer
    for b in range(wl.B):
        N = wl.entries(g)
        kc, ks = orc.quantize_fp8(wl.idx_k(g, b, 0, N))
        q = wl.q_idx(L, b)[0]
        w = wl.w(L, b)[0].numpy()
        pool, topk, cnt, _ = orc.index_full_one(kc, ks, q, w, N, 2048, 512)
        pos, _ = wl.planted_rows(b)
        assert len(pos) == 8
        assert set(pos) <= set(topk[:cnt].tolist())
        assert {p // 8 for p in pos} <= set(pool[pool >= 0].tolist())


def test_reindex_searches_only_the_pool(orc):
    N = 6000
    kc, ks = orc.quantize_fp8(random_index_rows(N, 128, 91))
    q1 = synth.rows_normal_bf16(92, "q", 0, 0, 4, 128)
    q2 = synth.rows_normal_bf16(93, "q", 0, 0, 4, 128)
    w = synth.rows_uniform_f32(94, "w", 0, 0, 1, 4)[0].numpy()
    pool, _, _, _ = orc.index_full_one(kc, ks, q1, w, N, 64, 64)
    topk, cnt = orc.index_reindex_one(kc, ks, q2, w, N, pool, 64)
    assert cnt == 64
    assert set((topk // 8).tolist()) <= set(pool.tolist())
    # equals a brute-force Top-64 of the pool positions under the second query
    cand = np.concatenate([np.arange(8 * b, min(8 * b + 8, N)) for b in pool if b >= 0])
    sc = orc.scores(kc, ks, q2, w, pos=cand.astype(np.int32))
    order = np.lexsort((cand, -sc))
    assert np.array_equal(topk, np.sort(cand[order[:64]]))
    # with every block in the pool, Reindex equals the flat Full Top-K
    nb = (N + 7) // 8
    allpool = np.arange(nb, dtype=np.int32)
    t_all, _ = orc.index_reindex_one(kc, ks, q2, w, N, allpool, 64)
    _, t_flat, _, _ = orc.index_full_one(kc, ks, q2, w, N, 0, 64)
    assert np.array_equal(t_all, t_flat)


def test_partial_last_block_and_visibility(orc):
    assert orc.visible(0, 1) == 1 and orc.visible(4095, 1) == 4096
    assert orc.visible(0, 2) == 0 and orc.visible(1, 2) == 1 and orc.visible(2, 2) == 1
    N = 13                                       # last block holds positions 8..12
    kc, ks = orc.quantize_fp8(random_index_rows(16, 64, 5))
    q = synth.rows_normal_bf16(6, "q", 0, 0, 4, 64)
    w = np.ones(4, np.float32)
    pool, topk, cnt, sc = orc.index_full_one(kc, ks, q, w, N, 4, 16)
    assert cnt == 13 and np.array_equal(topk[:13], np.arange(13)) and np.all(topk[13:] == -1)
    assert np.array_equal(pool, np.array([0, 1, -1, -1]))


def test_batched_drivers_match_single(orc):
    B, cap, d, Tq, H_I = 2, 700, 64, 3, 4
    k = synth.rows_normal_bf16(41, "k", 0, 0, B * cap, d).view(B, cap, d)
    kc, ks = orc.quantize_fp8(k)
    q = synth.rows_normal_bf16(42, "q", 0, 0, B * Tq * H_I, d).view(B, Tq, H_I, d)
    w = synth.rows_uniform_f32(43, "w", 0, 0, B * Tq, H_I).view(B, Tq, H_I).numpy()
    q_pos = np.array([[100, 399, 698], [0, 7, 650]], np.int32)
    for ratio in (1, 2):
        pool, topk, cnt = orc.index_full(kc, ks, ratio, q, w, q_pos, 8, 16)
        for b in range(B):
            for t in range(Tq):
                N = orc.visible(int(q_pos[b, t]), ratio)
                p1, t1, c1, _ = orc.index_full_one(kc[b], ks[b], q[b, t], w[b, t], N, 8, 16)
                assert np.array_equal(pool[b, t], p1) and np.array_equal(topk[b, t], t1)
                assert cnt[b, t] == c1
        t2, c2 = orc.index_reindex(kc, ks, ratio, q, w, q_pos, pool, 16)
        for b in range(B):
            for t in range(Tq):
                N = orc.visible(int(q_pos[b, t]), ratio)
                t1, c1 = orc.index_reindex_one(kc[b], ks[b], q[b, t], w[b, t], N, pool[b, t], 16)
                assert np.array_equal(t2[b, t], t1) and c2[b, t] == c1
