"""GPU parity of the index path (a3-a7): scores, block pool, Top-K (Full, flat,
hierarchical, ratio 2), Reindex and Reuse -- bit-exact against the oracle."""
import numpy as np
import pytest
import torch

from oracle import workload_ref as R
from synth.workloads import WORKLOADS, small_variant

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def harness():
    import csa2_harness
    assert torch.cuda.is_available()
    return csa2_harness


def _check_request_index(dw, b, q_pos=None):
    wl = dw.wl
    ref_caches = R.request_caches(wl, b, main_rows={g: np.zeros(0, np.int64)
                                                    for g in range(len(wl.groups))})
    st = dw.stack.kv
    for g, c in enumerate(ref_caches):
        assert np.array_equal(st[g].idx_codes[b].cpu().numpy(), c["idx_codes"]), f"group {g}"
        assert np.array_equal(st[g].idx_scale[b].cpu().numpy(), c["idx_scale"]), f"group {g}"
    ref = R.index_layers(wl, b, ref_caches, q_pos)
    for layer, t in ref["topk"].items():
        got = dw.stack.topk[layer][b].cpu().numpy()
        cnt = dw.stack.count[layer][b].cpu().numpy()
        assert np.array_equal(cnt, ref["count"][layer]), f"layer {layer} count"
        for tq in range(t.shape[0]):
            assert np.array_equal(got[tq], t[tq]), f"layer {layer} query {tq} Top-K differs"
    for g, p in ref["pool"].items():
        assert np.array_equal(dw.stack.pool[g][b].cpu().numpy(), p), f"group {g} pool"
    return ref


def test_tiny_full_layer_and_scores(harness, orc):
    """The tiny workload at its own size: pool 64x8 of 512 blocks, Top-64, and the
    workspace scores themselves, bit for bit."""
    wl = WORKLOADS["tiny_full_layer"]
    dw = harness.DeviceWorkload(wl)
    dw.step()
    assert dw.stack.dev_err.item() == 0
    _check_request_index(dw, 0)
    N = wl.entries(0)
    c = R.request_caches(wl, 0, main_rows={0: np.zeros(0, np.int64)})[0]
    ref_scores = orc.scores(c["idx_codes"], c["idx_scale"], wl.q_idx(0, 0)[0], wl.w(0, 0)[0].numpy(),
                            n=N)
    ws = dw.stack.workspace.view(torch.float32)[:N].cpu().numpy()
    assert np.array_equal(ws.view(np.uint32), ref_scores.view(np.uint32))


def test_decoder_group_pool_active(harness):
    """N = 20000 > 2048 x 8: the pool really selects; Full + 4 Reindex layers."""
    wl = small_variant(WORKLOADS["decoder_group_32k"], B=2, ctx=20000)
    dw = harness.DeviceWorkload(wl)
    dw.step()
    assert dw.stack.dev_err.item() == 0
    for b in range(wl.B):
        _check_request_index(dw, b)
        # Reuse layers alias their source's selection
        for layer, (g, m, src) in enumerate(R.reuse_sources(wl)):
            if m == "U":
                assert dw.stack.topk_of(layer).data_ptr() == dw.stack.topk[src].data_ptr()
        # planted positions survive into the Full layer's Top-512
        pos, _ = wl.planted_rows(b)
        top = set(dw.stack.topk[wl.decoder_full_layer][b, 0].cpu().numpy().tolist())
        assert set(pos) <= top


def test_flat_ratio2_prefill_causal(harness):
    """Encoder group (ratio 2, flat Top-512) with 64 causal query tokens."""
    wl = small_variant(WORKLOADS["prefill_chunk_enc"], B=1, ctx=6000 + 64, Tq=64)
    dw = harness.DeviceWorkload(wl)
    dw.step()
    assert dw.stack.dev_err.item() == 0
    _check_request_index(dw, 0)


@pytest.mark.parametrize("ctx", [40000, 110000])
def test_flat_unstaged_and_hierarchical_million_shape(harness, ctx):
    """Encoder groups (flat) with N = ctx / 2 next to a decoder group with N = ctx:
    20000 keys (> 16384: the wide shared-memory stage) and 55000 keys (> 49152: the
    selection streams its keys from global memory in every radix pass)."""
    wl = small_variant(WORKLOADS["decode_1m"], B=2, ctx=ctx)
    dw = harness.DeviceWorkload(wl)
    dw.step()
    assert dw.stack.dev_err.item() == 0
    for b in range(wl.B):
        _check_request_index(dw, b)


def test_ragged_positions(harness):
    """Requests at different positions (one with fewer than top_k visible entries)."""
    import fp4_kv_compressed_b200 as pkg
    wl = small_variant(WORKLOADS["decoder_group_32k"], B=3, ctx=3000)
    dw = harness.DeviceWorkload(wl)
    st = dw.stack
    q_pos = torch.tensor([[2999], [1234], [300]], dtype=torch.int32, device="cuda")
    L = wl.decoder_full_layer
    inp = dw.inputs
    pkg.csa2_index_full(st.kv[0].struct, inp["q_idx"][L], inp["w"][L], q_pos, 1, wl.H_I, 3000,
                        2048, 512, st.pool[0], st.topk[L], st.count[L], st.workspace, st.dev_err)
    torch.cuda.synchronize()
    assert st.dev_err.item() == 0
    for b in range(3):
        caches = R.request_caches(wl, b, main_rows={0: np.zeros(0, np.int64)})
        c = caches[0]
        p, t, n = __import__("oracle").index_full(
            c["idx_codes"][None], c["idx_scale"][None], 1, wl.q_idx(L, b)[None],
            wl.w(L, b)[None].numpy(), q_pos[b:b + 1].cpu().numpy(), 2048, 512)
        assert np.array_equal(st.topk[L][b].cpu().numpy(), t[0])
        assert np.array_equal(st.pool[0][b].cpu().numpy(), p[0])
        assert st.count[L][b].item() == n[0, 0]
    assert st.count[L][2].item() == 301 and (st.topk[L][2, 0, 301:] == -1).all()


def test_device_bounds_flags(harness):
    """n_max smaller than a query's visible count, and a pool id past the visible
    range, are flagged on the device (no fault, no hang)."""
    import fp4_kv_compressed_b200 as pkg
    wl = small_variant(WORKLOADS["decoder_group_32k"], B=1, ctx=3000)
    dw = harness.DeviceWorkload(wl)
    st = dw.stack
    inp = dw.inputs
    L = wl.decoder_full_layer
    pkg.csa2_index_full(st.kv[0].struct, inp["q_idx"][L], inp["w"][L], inp["q_pos"], 1, wl.H_I,
                        1000, 2048, 512, st.pool[0], st.topk[L], st.count[L], st.workspace,
                        st.dev_err)
    assert pkg.csa2_read_device_error(st.dev_err) & pkg.DEVERR_NMAX
    bad_pool = torch.full((1, 1, 2048), -1, dtype=torch.int32, device="cuda")
    bad_pool[0, 0, 0] = 5000          # block 5000 = positions 40000.. > visible 3000
    pkg.csa2_index_reindex(st.kv[0].struct, inp["q_idx"][L], inp["w"][L], inp["q_pos"], 1,
                           wl.H_I, bad_pool, 2048, 512, st.topk[L], st.count[L], st.workspace,
                           st.dev_err)
    assert pkg.csa2_read_device_error(st.dev_err) & pkg.DEVERR_INDEX
    assert st.count[L][0].item() == 0


@pytest.mark.parametrize("qscale", [1.0, 300.0])
def test_scores_wide_dynamic_range(harness, orc, qscale):
    """Index-K rows whose magnitudes span about 40 binades (so the E4M3 codes reach
    the subnormals and the top of the range) against a small and a large query:
    the fp32 scores match the oracle's bit for bit."""
    import fp4_kv_compressed_b200 as pkg
    import synth
    N, d, H_I = 3000, 128, 4
    kv = pkg.GlobalKV(1, N, d, 1, "cuda")
    g = torch.Generator().manual_seed(9)
    mags = torch.exp2(torch.randint(-30, 12, (N, 1), generator=g).float())
    rows = (synth.rows_normal_bf16(4, "k", 0, 0, N, d).float() * mags).to(torch.bfloat16)
    z = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkg.csa2_quantize_append(kv.struct, None, rows.view(1, N, d).cuda(), N, z, None, None, 0, None)
    q = (synth.rows_normal_bf16(5, "q", 0, 0, H_I, d).float() * qscale).to(torch.bfloat16)
    q[1, 7] = -q[1, 7]
    w = synth.rows_uniform_f32(6, "w", 0, 0, 1, H_I)
    topk = torch.zeros(1, 1, 64, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, 1, dtype=torch.int32, device="cuda")
    ws = torch.empty(pkg.csa2_workspace_size(pkg.CSA2_OP_INDEX_FULL, 1, 1, N, 0, 64, 0),
                     dtype=torch.uint8, device="cuda")
    qpos = torch.tensor([[N - 1]], dtype=torch.int32, device="cuda")
    pkg.csa2_index_full(kv.struct, q.view(1, 1, H_I, d).cuda(), w.view(1, 1, H_I).cuda(), qpos, 1,
                        H_I, N, 0, 64, None, topk, cnt, ws)
    torch.cuda.synchronize()
    kc, ks = orc.quantize_fp8(rows)
    ref = orc.scores(kc, ks, q, w[0].numpy(), n=N)
    got = ws.view(torch.float32)[:N].cpu().numpy()
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    assert np.array_equal(topk[0, 0].cpu().numpy(), orc.select_topk(ref, 64))


def _index_case(pkg, orc, rows, ratio, q_pos, pool_blocks, top_k, H_I=4, seed=41):
    """Runs csa2_index_full over per-request index-K rows [B][N][d] and compares pool,
    Top-K and counts with the oracle, bit for bit."""
    import synth
    B, N, d = rows.shape
    kv = pkg.GlobalKV(B, N, d, ratio, "cuda")
    z = torch.zeros(B, dtype=torch.int32, device="cuda")
    pkg.csa2_quantize_append(kv.struct, None, rows.cuda(), N, z, None, None, 0, None)
    q = torch.stack([synth.rows_normal_bf16(seed, "q", b, 0, H_I, d) for b in range(B)]).view(B, 1, H_I, d)
    w = torch.stack([synth.rows_uniform_f32(seed, "w", b, 0, 1, H_I) for b in range(B)]).view(B, 1, H_I)
    qp = torch.tensor(q_pos, dtype=torch.int32).view(B, 1)
    P = max(pool_blocks, 1)
    pool = torch.full((B, 1, P), -1, dtype=torch.int32, device="cuda")
    topk = torch.full((B, 1, top_k), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((B, 1), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(pkg.csa2_workspace_size(pkg.CSA2_OP_INDEX_FULL, B, 1, N, 0, top_k, pool_blocks),
                     dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkg.csa2_index_full(kv.struct, q.cuda(), w.cuda(), qp.cuda(), 1, H_I, N, pool_blocks, top_k,
                        pool if pool_blocks else None, topk, cnt, ws, err)
    torch.cuda.synchronize()
    assert pkg.csa2_read_device_error(err) == 0
    kc, ks = orc.quantize_fp8(rows.reshape(B * N, d))
    p_ref, t_ref, n_ref = orc.index_full(kc.reshape(B, N, d), ks.reshape(B, N), ratio, q, w.numpy(),
                                         qp.numpy(), pool_blocks, top_k)
    assert np.array_equal(topk.cpu().numpy(), t_ref)
    assert np.array_equal(cnt.cpu().numpy(), n_ref)
    if pool_blocks:
        assert np.array_equal(pool.cpu().numpy(), p_ref)
    return topk.cpu().numpy(), cnt.cpu().numpy(), (pool.cpu().numpy() if pool_blocks else None)


@pytest.mark.parametrize("N,pool_blocks", [(5000, 0), (5000, 2048), (20000, 2048)])
def test_exact_ties_take_the_lowest_positions(harness, orc, N, pool_blocks):
    """Every index-K row identical, so every score and every block maximum is equal: the
    selection falls back to the position order (lowest first), flat and hierarchical,
    including a pool smaller than the block count."""
    import fp4_kv_compressed_b200 as pkg
    import synth
    row = synth.rows_normal_bf16(40, "row", 0, 0, 1, 128)
    rows = row.expand(2, N, 128).contiguous()
    topk, cnt, pool = _index_case(pkg, orc, rows, 1, [N - 1, N - 1], pool_blocks, 512)
    assert (topk[:, 0] == np.arange(512)).all() and (cnt == 512).all()
    if pool_blocks:
        nb = (N + 7) // 8
        assert (pool[:, 0, :min(nb, 2048)] == np.arange(min(nb, 2048))).all()


def test_zero_scores_and_mixed(harness, orc):
    """A third of the rows are zero (sigma 0, score exactly 0) and tie below every
    positive score; the rest include scores clipped to 0 by the relu."""
    import fp4_kv_compressed_b200 as pkg
    import synth
    N = 3000
    rows = synth.rows_normal_bf16(42, "rows", 0, 0, N, 128).view(1, N, 128).clone()
    rows[0, ::3] = 0
    _index_case(pkg, orc, rows, 1, [N - 1], 0, 512)
    t, c, _ = _index_case(pkg, orc, rows, 1, [N - 1], 2048, 2048 // 4)
    assert c[0, 0] == 512


def test_ratio2_earliest_positions(harness, orc):
    """Ratio-2 entries at the first token positions: t = 0 sees no entry, t = 1 and 2 one,
    t = 3 two; counts and padded Top-K match the oracle."""
    import fp4_kv_compressed_b200 as pkg
    import synth
    rows = torch.stack([synth.rows_normal_bf16(43, "rows", b, 0, 8, 128) for b in range(4)])
    topk, cnt, _ = _index_case(pkg, orc, rows, 2, [0, 1, 2, 3], 0, 16)
    assert cnt[:, 0].tolist() == [0, 1, 1, 2]
    assert (topk[0, 0] == -1).all() and (topk[3, 0, 2:] == -1).all()


@pytest.mark.parametrize("paged", [False, True])
def test_reindex_many_pool_tiles(harness, orc, paged):
    """24 queries x 128 pool tiles of 128 positions: more scoring CTAs than the SMs hold
    at once.  The query positions are ragged (some pool blocks only partly visible) and
    each pool is a random set of 2048 visible blocks, the last one included; Top-K and
    counts bit-exact against the oracle, on the contiguous and on a paged layout with
    shuffled pages."""
    import fp4_kv_compressed_b200 as pkg
    import synth
    B, cap, d, H_I, P, K, page = 24, 20480, 128, 4, 2048, 512, 256
    rng = np.random.default_rng(81)
    codes = rng.integers(0, 256, size=(B, cap, d), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3C                  # E4M3 NaN codes -> 1.5
    sigma = rng.uniform(0.01, 2.0, size=(B, cap)).astype(np.float32)
    q_pos = np.array([cap - 1 - 13 * b - (b % 3) for b in range(B)], np.int32)
    pool = np.zeros((B, 1, P), np.int32)
    for b in range(B):
        nb = (int(q_pos[b]) + 8) // 8                     # blocks with a visible position
        blocks = rng.choice(nb - 1, size=P - 1, replace=False)
        pool[b, 0] = np.sort(np.append(blocks, nb - 1))   # the last, partly visible block too
    q = torch.stack([synth.rows_normal_bf16(82, "qi", b, 0, H_I, d) for b in range(B)]).view(B, 1, H_I, d)
    w = torch.stack([synth.rows_uniform_f32(82, "w", b, 0, 1, H_I) for b in range(B)]).view(B, 1, H_I)
    if paged:
        max_pages = cap // page
        n_pages = B * max_pages + 5
        perm = torch.randperm(n_pages, generator=torch.Generator().manual_seed(83)).to(torch.int32)
        table = perm[:B * max_pages].view(B, max_pages).contiguous()
        kv = pkg.PagedKV(B, max_pages, page, n_pages, d, 1, table, "cuda")
        for b in range(B):
            r = kv.rows_of(b, cap)
            kv.idx_codes[r] = torch.from_numpy(codes[b]).cuda()
            kv.idx_scale[r] = torch.from_numpy(sigma[b]).cuda()
        call = pkg.csa2_index_reindex_paged
    else:
        kv = pkg.GlobalKV(B, cap, d, 1, "cuda")
        kv.idx_codes.copy_(torch.from_numpy(codes))
        kv.idx_scale.copy_(torch.from_numpy(sigma))
        call = pkg.csa2_index_reindex
    topk = torch.full((B, 1, K), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, 1, dtype=torch.int32, device="cuda")
    ws = torch.empty(pkg.csa2_workspace_size(pkg.CSA2_OP_INDEX_REINDEX, B, 1, 0, 0, K, P),
                     dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    call(kv.struct, q.cuda(), w.cuda(), torch.from_numpy(q_pos).view(B, 1).cuda(), 1, H_I,
         torch.from_numpy(pool).cuda(), P, K, topk, cnt, ws, err)
    torch.cuda.synchronize()
    assert pkg.csa2_read_device_error(err) == 0
    t_ref, c_ref = orc.index_reindex(codes, sigma, 1, q, w.numpy(), q_pos.reshape(B, 1), pool, K)
    assert np.array_equal(cnt.cpu().numpy(), c_ref)
    assert np.array_equal(topk.cpu().numpy(), t_ref)
