"""GPU parity of the tensor-core Full-layer scan (csa2_index_full_tc) against the oracle.

The tensor cores sum the channel products in their own order, so the scores are
compared with the unrounded oracle score within the fp32 error bound of any
summation order, (d + H_I + 2) * 2^-23 of the score's magnitude (2^-23: room for
an accumulator that truncates instead of rounding to nearest).  The selection
that follows is the exact path's: given the kernel's own scores, pool and Top-K
must equal the oracle's selection over those scores bit for bit, and the Top-K
can differ from the oracle's exact one only between positions whose scores lie
within the bound of each other."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkg():
    import fp4_kv_compressed_b200 as p
    assert torch.cuda.is_available()
    return p


def _score_stride(n_max: int) -> int:
    # workspace layout of the Full call: scores [B*Tq][align_up(n_max, 64)] fp32 first
    return (max(n_max, 1) + 63) // 64 * 64


def _tc_case(pkg, orc, rows, ratio, q_pos, pool_blocks, top_k, H_I, seed, check=None):
    """rows [B][N][d] bf16 index-K rows, q_pos [B][Tq]; runs csa2_index_full_tc and
    checks every query (or the (b, t) pairs in `check`)."""
    B, N, d = rows.shape
    Tq = len(q_pos[0])
    kv = pkg.GlobalKV(B, N, d, ratio, "cuda")
    z = torch.zeros(B, dtype=torch.int32, device="cuda")
    pkg.csa2_quantize_append(kv.struct, None, rows.cuda(), N, z, None, None, 0, None)
    q = torch.stack([synth.rows_normal_bf16(seed, "q", b, 0, Tq * H_I, d) for b in range(B)])
    q = q.view(B, Tq, H_I, d)
    w = torch.stack([synth.rows_uniform_f32(seed, "w", b, 0, Tq, H_I) for b in range(B)])
    qp = torch.tensor(q_pos, dtype=torch.int32).view(B, Tq)
    P = max(pool_blocks, 1)
    pool = torch.full((B, Tq, P), -7, dtype=torch.int32, device="cuda")
    topk = torch.full((B, Tq, top_k), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((B, Tq), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(pkg.csa2_workspace_size(pkg.CSA2_OP_INDEX_FULL, B, Tq, N, 0, top_k, pool_blocks),
                     dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkg.csa2_index_full_tc(kv.struct, q.cuda(), w.cuda(), qp.cuda(), Tq, H_I, N, pool_blocks,
                           top_k, pool if pool_blocks else None, topk, cnt, ws, err)
    torch.cuda.synchronize()
    assert pkg.csa2_read_device_error(err) == 0
    kc, ks = orc.quantize_fp8(rows.reshape(B * N, d))
    kc, ks = kc.reshape(B, N, d), ks.reshape(B, N)
    stride = _score_stride(N)
    sc_all = ws[:B * Tq * stride * 4].view(torch.float32).view(B, Tq, stride).cpu().numpy()
    topk, cnt, pool = topk.cpu().numpy(), cnt.cpu().numpy(), pool.cpu().numpy()
    pairs = check if check is not None else [(b, t) for b in range(B) for t in range(Tq)]
    n_diff = 0
    for b, t in pairs:
        n = min(orc.visible(int(q_pos[b][t]), ratio), N)
        g = sc_all[b, t, :n].astype(np.float32)
        ex, mag = orc.scores_f64(kc[b], ks[b], q[b, t], w[b, t].numpy(), n=n)
        tol = (d + H_I + 2) * 2.0 ** -23 * mag
        err_abs = np.abs(g.astype(np.float64) - ex)
        assert np.all(err_abs <= tol), f"({b},{t}) score off by {np.max(err_abs - tol):.3e} beyond bound"
        # the selection over the kernel's own scores is exact
        if pool_blocks:
            p_ref = orc.select_topk(orc.block_max(g), pool_blocks)
            p_row = np.full(pool_blocks, -1, np.int32)
            p_row[:len(p_ref)] = p_ref
            assert np.array_equal(pool[b, t], p_row), f"({b},{t}) pool"
            ids = (p_ref[:, None] * 8 + np.arange(8)[None, :]).ravel()
            ids = ids[ids < n].astype(np.int32)
            t_ref = orc.select_topk(g[ids], top_k, ids)
        else:
            t_ref = orc.select_topk(g, top_k)
        row = np.full(top_k, -1, np.int32)
        row[:len(t_ref)] = t_ref
        assert np.array_equal(topk[b, t], row), f"({b},{t}) Top-K over the kernel's scores"
        assert cnt[b, t] == min(n, top_k)
        # against the exact Top-K: differences only between near-tied positions
        order = np.lexsort((np.arange(n), -ex))
        exact = set(order[:min(n, top_k)].tolist())
        got = set(t_ref.tolist())
        for p_in in got - exact:
            for u in exact - got:
                assert ex[u] - ex[p_in] <= tol[u] + tol[p_in], f"({b},{t}) {p_in} chosen over {u}"
        n_diff += len(got - exact)
    return n_diff


def test_tc_prefill_flat_ratio2(pkg, orc):
    """Encoder shape (ratio 2, flat Top-512, H_I = 4, d = 128): 100 causal query tokens
    (4 query blocks, the last ragged), one request far into its cache and one at its
    first tokens (0 and 1 visible entries, then fewer than top_k)."""
    B, N, d = 2, 3000, 128
    rows = torch.stack([synth.rows_normal_bf16(51, "rows", b, 0, N, d) for b in range(B)])
    q_pos = [[5800 + t for t in range(100)], [t for t in range(100)]]
    _tc_case(pkg, orc, rows, 2, q_pos, 0, 512, 4, 52)


def test_tc_decoder_hierarchical_pool(pkg, orc):
    """Decoder shape (ratio 1, pool 2048 x 8, H_I = 8): N = 20000 > 16384 so the pool
    really selects, 20 query tokens in two query blocks."""
    B, N, d = 1, 20000, 128
    rows = synth.rows_normal_bf16(53, "rows", 0, 0, N, d).view(1, N, d)
    q_pos = [[N - 20 + t for t in range(20)]]
    _tc_case(pkg, orc, rows, 1, q_pos, 2048, 512, 8, 54)


@pytest.mark.parametrize("H_I", [1, 16])
def test_tc_head_counts_d64(pkg, orc, H_I):
    """d = 64 with 1 and 16 index heads (128 and 8 query tokens per block): 130 query
    tokens, N = 1500 (a ragged last tile), Top-64."""
    B, N, d = 1, 1500, 64
    rows = synth.rows_normal_bf16(55, "rows", 0, 0, N, d).view(1, N, d)
    q_pos = [[N - 130 + t for t in range(130)]]
    _tc_case(pkg, orc, rows, 1, q_pos, 0, 64, H_I, 56 + H_I)


def test_tc_identical_rows_take_the_lowest_positions(pkg, orc):
    """Every index-K row identical: the products and their sums are the same for every
    entry, so all scores of a query are equal and the Top-K is the lowest positions."""
    B, N, d = 1, 5000, 128
    row = synth.rows_normal_bf16(57, "row", 0, 0, 1, d)
    rows = row.expand(N, d).contiguous().view(1, N, d)
    kv = pkg.GlobalKV(B, N, d, 1, "cuda")
    z = torch.zeros(B, dtype=torch.int32, device="cuda")
    pkg.csa2_quantize_append(kv.struct, None, rows.cuda(), N, z, None, None, 0, None)
    Tq, H_I = 40, 4
    q = synth.rows_normal_bf16(58, "q", 0, 0, Tq * H_I, d).view(1, Tq, H_I, d).cuda()
    w = synth.rows_uniform_f32(58, "w", 0, 0, Tq, H_I).view(1, Tq, H_I).cuda()
    qp = torch.arange(N - Tq, N, dtype=torch.int32, device="cuda").view(1, Tq)
    for pool_blocks in (0, 2048):
        pool = torch.full((1, Tq, max(pool_blocks, 1)), -7, dtype=torch.int32, device="cuda")
        topk = torch.full((1, Tq, 512), -7, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(1, Tq, dtype=torch.int32, device="cuda")
        ws = torch.empty(pkg.csa2_workspace_size(pkg.CSA2_OP_INDEX_FULL, 1, Tq, N, 0, 512,
                                                 pool_blocks), dtype=torch.uint8, device="cuda")
        pkg.csa2_index_full_tc(kv.struct, q, w, qp, Tq, H_I, N, pool_blocks, 512,
                               pool if pool_blocks else None, topk, cnt, ws)
        torch.cuda.synchronize()
        sc = ws[:Tq * _score_stride(N) * 4].view(torch.float32).view(Tq, -1).cpu().numpy()
        for t in range(Tq):
            n = N - Tq + t + 1
            assert np.unique(sc[t, :n]).size == 1
        assert (topk[0].cpu().numpy() == np.arange(512)[None, :]).all()
        if pool_blocks:
            pl = pool[0].cpu().numpy()
            for t in range(Tq):
                nb = (N - Tq + t + 1 + 7) // 8
                assert (pl[t, :nb] == np.arange(nb)).all() and (pl[t, nb:] == -1).all()


def test_tc_full_size_prefill_chunk_sampled(pkg, orc):
    """The 2048-token prefill chunk after a 65536-token prefix (ratio 2: 32768 .. 33792
    visible entries, H_I = 4, d = 128, flat Top-512) in one call, the launch the
    benchmark times; sampled queries are checked against the oracle."""
    from synth.workloads import WORKLOADS
    wl = WORKLOADS["prefill_chunk_enc"]
    N = wl.ctx // 2
    d, H_I, Tq = wl.d_I, wl.H_I, wl.Tq
    rows = synth.rows_normal_bf16(59, "rows", 0, 0, N, d).view(1, N, d)
    q_pos = [[wl.ctx - Tq + t for t in range(Tq)]]
    check = [(0, t) for t in (0, 1, 31, 32, 1000, 2047)]
    _tc_case(pkg, orc, rows, 2, q_pos, 0, 512, H_I, 60, check=check)


def test_tc_stack_prefill_chunk(pkg, orc):
    """The encoder stack (ratio 2, F + 5 U) on a 64-token prefill chunk with the
    tensor-core scan: every query's Top-K is valid against the unrounded scores (a
    position is left out only for one within the error bound of it), and every layer's
    attention over the kernel's own selection matches the oracle."""
    import csa2_harness
    from oracle import workload_ref as R
    from synth.workloads import WORKLOADS, small_variant
    wl = small_variant(WORKLOADS["prefill_chunk_enc"], B=1, ctx=3000 + 64, Tq=64)
    dw = csa2_harness.DeviceWorkload(wl, index_scan="tc")
    dw.step()
    torch.cuda.synchronize()
    assert dw.stack.dev_err.item() == 0
    gpu = dw.request_state(0)
    plan = R.reuse_sources(wl)
    L = [layer for layer, (_, m, _) in enumerate(plan) if m == "F"][0]
    caches = R.request_caches(wl, 0, main_rows={0: gpu["topk"][L].ravel()})
    c = caches[0]
    d = wl.d_I
    for t, pos in enumerate(wl.q_positions()):
        n = orc.visible(pos, wl.groups[0].ratio)
        ex, mag = orc.scores_f64(c["idx_codes"], c["idx_scale"], wl.q_idx(L, 0)[t],
                                 wl.w(L, 0)[t].numpy(), n=n)
        tol = (d + wl.H_I + 2) * 2.0 ** -23 * mag
        got = gpu["topk"][L][t]
        k = min(n, wl.top_k)
        assert gpu["count"][L][t] == k and (got[k:] == -1).all()
        chosen = got[:k]
        assert (np.diff(chosen) > 0).all() and chosen.min(initial=0) >= 0 and chosen.max(initial=0) < n
        left = np.setdiff1d(np.arange(n), chosen)
        if len(left):
            # every left-out position scores at most the lowest chosen one, up to the bound
            i = np.argmin(ex[chosen] + tol[chosen])
            assert (ex[left] - tol[left] <= ex[chosen][i] + tol[chosen][i]).all(), t
    for layer in range(len(plan)):
        o_ref, l_ref = R.attention_layer(wl, 0, layer, caches, gpu["topk"][plan[layer][2]])
        assert R.rel_err_rows(gpu["out"][layer], o_ref).max() <= 2e-3
        fin = np.isfinite(l_ref)
        assert np.array_equal(np.isfinite(gpu["lse"][layer]), fin)
        assert np.abs(gpu["lse"][layer][fin] - l_ref[fin]).max(initial=0) <= 1e-3
