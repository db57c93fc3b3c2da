"""Pins of the oracle's sparse attention.

Special cases that reduce to textbook dense softmax attention (numpy fp64),
a single key (o = v exactly), two equal logits (o = mean), order invariance of
the selected set, the window ring slots, and the union without de-duplication.
"""
import math

import numpy as np
import torch

import synth


def fp4_cache(orc, n, seed, scale=1.0):
    x = (synth.rows_normal_bf16(seed, "kv", 0, 0, n, 512).float() * scale).to(torch.bfloat16)
    codes, scales = orc.quantize_fp4(x)
    return codes, scales, orc.dequant_fp4(codes, scales)


def swa_ring(orc, W, seed):
    x = synth.rows_normal_bf16(seed, "swa", 0, 0, W, 512)
    codes, sigma = orc.quantize_fp8(x)
    return codes, sigma, orc.dequant_fp8(codes, sigma)


def dense(q, keys, scale):
    """Textbook softmax attention in fp64, K = V = keys."""
    logits = q @ keys.T * scale
    m = logits.max(1, keepdims=True)
    p = np.exp(logits - m)
    den = p.sum(1, keepdims=True)
    return (p / den) @ keys, (m + np.log(den))[:, 0]


def test_reduces_to_dense_attention_over_all_entries(orc):
    N, H = 40, 8
    codes, scales, kv = fp4_cache(orc, N, 1)
    swc, sws, _ = swa_ring(orc, 128, 2)
    q = synth.rows_normal_bf16(3, "q", 0, 0, H, 512)
    topk = np.arange(N, dtype=np.int32)
    sc = 1 / math.sqrt(512)
    o, lse = orc.attention_one(codes, scales, swc, sws, q, N - 1, topk, 0, sc)
    ref_o, ref_lse = dense(q.double().numpy(), kv, sc)
    assert np.allclose(o, ref_o, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_window_only_and_ring_slots(orc):
    W, H, t = 128, 4, 300
    codes, scales, _ = fp4_cache(orc, 8, 4)
    swc, sws, swv = swa_ring(orc, W, 5)
    q = synth.rows_normal_bf16(6, "q", 0, 0, H, 512)
    topk = np.full(16, -1, np.int32)
    sc = 0.05
    o, lse = orc.attention_one(codes, scales, swc, sws, q, t, topk, 128, sc)
    slots = [p % W for p in range(t - 127, t + 1)]
    ref_o, ref_lse = dense(q.double().numpy(), swv[slots], sc)
    assert np.allclose(o, ref_o, rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)
    # early positions: the window is clipped at position 0
    o2, _ = orc.attention_one(codes, scales, swc, sws, q, 5, topk, 128, sc)
    ref2, _ = dense(q.double().numpy(), swv[:6], sc)
    assert np.allclose(o2, ref2, rtol=1e-12, atol=1e-12)


def test_single_key_and_equal_logits(orc):
    codes, scales, kv = fp4_cache(orc, 4, 7)
    swc, sws, _ = swa_ring(orc, 128, 8)
    q = synth.rows_normal_bf16(9, "q", 0, 0, 2, 512)
    o, lse = orc.attention_one(codes, scales, swc, sws, q, 3, np.array([2, -1], np.int32), 0,
                               0.1)
    assert np.array_equal(o, np.stack([kv[2], kv[2]]))
    assert np.allclose(lse, 0.1 * (q.double().numpy() @ kv[2]), rtol=1e-14)
    # the same entry twice: the union is not de-duplicated, the result is unchanged
    # with one other key the weight of the duplicated key doubles
    o3, _ = orc.attention_one(codes, scales, swc, sws, torch.zeros(1, 512, dtype=torch.bfloat16),
                              3, np.array([1, 1, 2], np.int32), 0, 0.1)
    assert np.allclose(o3[0], (2 * kv[1] + kv[2]) / 3, rtol=1e-14, atol=1e-14)


def test_order_of_selection_is_irrelevant_and_union(orc):
    N, H, t, W = 64, 4, 63, 128
    codes, scales, kv = fp4_cache(orc, N, 10)
    swc, sws, swv = swa_ring(orc, W, 11)
    q = synth.rows_normal_bf16(12, "q", 0, 0, H, 512)
    sel = np.array([5, 17, 40, 41, 63, -1, 9], np.int32)
    perm = np.array([63, -1, 9, 41, 5, 40, 17], np.int32)
    o1, l1 = orc.attention_one(codes, scales, swc, sws, q, t, sel, 16, 0.04)
    o2, l2 = orc.attention_one(codes, scales, swc, sws, q, t, perm, 16, 0.04)
    assert np.allclose(o1, o2, rtol=1e-13, atol=1e-13) and np.allclose(l1, l2, rtol=1e-13)
    keys = np.concatenate([kv[[5, 17, 40, 41, 63, 9]], swv[[p % W for p in range(48, 64)]]])
    ref_o, ref_l = dense(q.double().numpy(), keys, 0.04)
    assert np.allclose(o1, ref_o, rtol=1e-12, atol=1e-12)
    assert np.allclose(l1, ref_l, rtol=1e-12, atol=1e-12)


def test_no_keys(orc):
    codes, scales, _ = fp4_cache(orc, 2, 13)
    swc, sws, _ = swa_ring(orc, 128, 14)
    q = synth.rows_normal_bf16(15, "q", 0, 0, 2, 512)
    o, lse = orc.attention_one(codes, scales, swc, sws, q, 0, np.full(4, -1, np.int32), 0, 0.1)
    assert not o.any() and np.all(np.isneginf(lse))


def test_batched_attention_matches_single(orc):
    B, cap, W, Tq, H, K = 2, 50, 130, 3, 4, 8
    x = synth.rows_normal_bf16(20, "kv", 0, 0, B * cap, 512).view(B, cap, 512)
    codes, scales = orc.quantize_fp4(x)
    s = synth.rows_normal_bf16(21, "swa", 0, 0, B * W, 512).view(B, W, 512)
    swc, sws = orc.quantize_fp8(s)
    q = synth.rows_normal_bf16(22, "q", 0, 0, B * Tq * H, 512).view(B, Tq, H, 512)
    q_pos = np.array([[10, 20, 49], [0, 1, 2]], np.int32)
    rng = np.random.default_rng(0)
    topk = rng.integers(-1, 10, (B, Tq, K)).astype(np.int32)
    o, lse = orc.attention(codes, scales, swc, sws, q, q_pos, topk, 3, 0.05)
    for b in range(B):
        for t in range(Tq):
            o1, l1 = orc.attention_one(codes[b], scales[b], swc[b], sws[b], q[b, t],
                                       int(q_pos[b, t]), topk[b, t], 3, 0.05)
            assert np.array_equal(o[b, t], o1) and np.array_equal(lse[b, t], l1)
