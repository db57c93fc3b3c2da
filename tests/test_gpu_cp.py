"""GPU parity of the context-parallel path (one request's entries split across shards):
the merged pool / Top-K must equal the single-cache csa2_index_full bit for bit, and the
combined attention must match the oracle within 2e-3.  The shards are virtual: S slices
of the same cache on one GPU, their candidate lists stacked in slice order (exactly what
an all-gather delivers), run through the same calls a rank makes."""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import workload_ref as R

pytestmark = pytest.mark.gpu

ATTN_TOL = 2e-3
LSE_TOL = 1e-3


@pytest.fixture(scope="module")
def pkg():
    import fp4_kv_compressed_b200 as p
    assert torch.cuda.is_available()
    return p


def _case(pkg, orc, *, B, N, ratio, q_pos, pool_blocks, top_k, S, H=64, H_I=4, d=128, seed=61,
          swa_len=128):
    from fp4_kv_compressed_b200.context_parallel import ContextShard, LibraryBackend, slice_bounds
    dev = "cuda"
    Tq = len(q_pos[0])
    rows = torch.stack([synth.rows_normal_bf16(seed, "ik", b, 0, N, d) for b in range(B)])
    kvr = torch.stack([synth.rows_normal_bf16(seed, "kv", b, 0, N, 512) for b in range(B)])
    kv = pkg.GlobalKV(B, N, d, ratio, dev)
    z = torch.zeros(B, dtype=torch.int32, device=dev)
    pkg.csa2_quantize_append(kv.struct, kvr.cuda(), rows.cuda(), N, z, None, None, 0, None)
    W = swa_len + Tq - 1
    ring = pkg.SwaRing(B, W, dev)
    sw = torch.stack([synth.rows_normal_bf16(seed, "swa", b, 0, W, 512) for b in range(B)])
    ring_start = torch.full((B,), max(0, int(q_pos[0][0]) - swa_len + 1), dtype=torch.int32, device=dev)
    pkg.csa2_quantize_append(None, None, None, 0, None, ring.struct, sw.cuda(), W, ring_start)
    q_idx = torch.stack([synth.rows_normal_bf16(seed, "qi", b, 0, Tq * H_I, d)
                         for b in range(B)]).view(B, Tq, H_I, d).cuda()
    w = torch.stack([synth.rows_uniform_f32(seed, "w", b, 0, Tq, H_I) for b in range(B)]).cuda()
    q = torch.stack([synth.rows_normal_bf16(seed, "q", b, 0, Tq * H, 512, stride=synth.Q_STRIDE)
                     for b in range(B)]).view(B, Tq, H, 512).cuda()
    qp = torch.tensor(q_pos, dtype=torch.int32, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    # the single-cache reference
    P = max(pool_blocks, 1)
    pool_ref = torch.full((B, Tq, P), -7, dtype=torch.int32, device=dev)
    topk_ref = torch.full((B, Tq, top_k), -7, dtype=torch.int32, device=dev)
    cnt_ref = torch.zeros(B, Tq, dtype=torch.int32, device=dev)
    ws = torch.empty(pkg.csa2_workspace_size(pkg.CSA2_OP_INDEX_FULL, B, Tq, N, 0, top_k, pool_blocks),
                     dtype=torch.uint8, device=dev)
    pkg.csa2_index_full(kv.struct, q_idx, w, qp, Tq, H_I, N, pool_blocks, top_k,
                        pool_ref if pool_blocks else None, topk_ref, cnt_ref, ws, err)
    # S shards over [0, N)
    bounds = slice_bounds(N, S)
    shards = []
    for r, (lo, hi) in enumerate(bounds):
        n = max(hi - lo, 1)
        kv_s = pkg.GlobalKV(B, n, d, ratio, dev)
        for src, dst in ((kv.codes, kv_s.codes), (kv.scales, kv_s.scales),
                         (kv.idx_codes, kv_s.idx_codes), (kv.idx_scale, kv_s.idx_scale)):
            dst[:, :hi - lo].copy_(src[:, lo:hi])
        shards.append(ContextShard(kv_s, lo, hi, r, S, window=(r == S - 1), gather=None,
                                   backend=LibraryBackend))
    scans = []
    for sh in shards:
        n_max = sh.local_n_max(qp)
        ws_s = torch.empty(max(256, pkg.csa2_workspace_size(pkg.CSA2_OP_INDEX_FULL, B, Tq, max(n_max, 1),
                                                            0, top_k, pool_blocks)),
                           dtype=torch.uint8, device=dev)
        scans.append(sh.scan(q_idx, w, qp, Tq, H_I, pool_blocks, top_k, ws_s, dev_err=err))
    pool_lists = torch.stack([p for p, _ in scans]) if pool_blocks else None
    topk_lists = torch.stack([t for _, t in scans])
    results = [sh.merge(pool_lists, topk_lists) for sh in shards]
    assert pkg.csa2_read_device_error(err) == 0
    for res in results:
        assert torch.equal(res.topk, topk_ref) and torch.equal(res.count, cnt_ref)
        if pool_blocks:
            assert torch.equal(res.pool, pool_ref)
    # each shard's part is its slice's share of the Top-K, as local ids
    for sh, res in zip(shards, results):
        g = res.topk
        inside = (g >= sh.lo) & (g < sh.hi)
        assert torch.equal(res.topk_local, torch.where(inside, g - sh.lo, torch.full_like(g, -1)))
    # attention: partials on every shard, stacked, combined
    scale = 1 / math.sqrt(512)
    parts = [sh.attend_partial(ring, q, qp, Tq, H, res.topk_local, top_k, swa_len, scale, dev_err=err)
             for sh, res in zip(shards, results)]
    out, lse = shards[0].combine(torch.stack([o for o, _ in parts]), torch.stack([l for _, l in parts]))
    assert pkg.csa2_read_device_error(err) == 0
    mc, ms = orc.quantize_fp4(kvr)
    sc, ss = orc.quantize_fp8(sw)
    ring_c = np.zeros((B, W, 512), np.uint8)
    ring_s = np.zeros((B, W), np.float32)
    p0 = int(ring_start[0])
    for i in range(W):
        ring_c[:, (p0 + i) % W], ring_s[:, (p0 + i) % W] = sc[:, i], ss[:, i]
    o_ref, l_ref = orc.attention(mc, ms, ring_c, ring_s, q.cpu(), np.asarray(q_pos, np.int32),
                                 topk_ref.cpu().numpy(), swa_len, scale)
    err_rows = R.rel_err_rows(out.cpu().numpy(), o_ref)
    assert err_rows.max() <= ATTN_TOL, f"max row error {err_rows.max():.3e}"
    assert np.abs(lse.cpu().numpy() - l_ref).max() <= LSE_TOL


@pytest.mark.parametrize("S", [2, 4, 8])
def test_cp_decoder_pool(pkg, orc, S):
    """Ratio 1 with the hierarchical pool (20000 entries: more than 2048 blocks), two
    requests at different positions, split over S shards."""
    N = 20000
    _case(pkg, orc, B=2, N=N, ratio=1, q_pos=[[N - 1], [N - 3000]], pool_blocks=2048, top_k=512, S=S)


@pytest.mark.parametrize("S", [2, 3])
def test_cp_flat_ratio2(pkg, orc, S):
    """Ratio 2, flat Top-512, a long row (40000 entries: the multi-level selection) and
    uneven slices."""
    N = 40000
    _case(pkg, orc, B=1, N=N, ratio=2, q_pos=[[2 * N - 1]], pool_blocks=0, top_k=512, S=S, seed=62)


def test_cp_empty_and_short_shards(pkg, orc):
    """A query that sees only the first slice (the later shards see nothing) and a
    Top-K larger than what some shards hold."""
    N = 3000
    _case(pkg, orc, B=2, N=N, ratio=1, q_pos=[[700], [N - 1]], pool_blocks=512, top_k=256, S=4,
          seed=63)
