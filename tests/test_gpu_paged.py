"""GPU parity of the paged global KV (pages of the cache in a shuffled pool, requests of
different lengths): every call on the paged layout must give the same bytes and results
as on the contiguous layout, bit for bit, and touch no page beyond a request's length
(those block-table entries are -1, and no CSA2_DEVERR_PAGE may appear)."""
import math

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


def _layouts(pkg, lens, page, d=128, ratio=1, seed=71, spare=7):
    """A contiguous cache and a paged one holding the same entries."""
    B = len(lens)
    cap = max(lens)
    max_pages = -(-cap // page)
    need = [-(-n // page) for n in lens]
    n_pages = sum(need) + spare
    perm = torch.randperm(n_pages, generator=torch.Generator().manual_seed(seed)).to(torch.int32)
    table = torch.full((B, max_pages), -1, dtype=torch.int32)
    k = 0
    for b, n in enumerate(need):
        table[b, :n] = perm[k:k + n]
        k += n
    dev = "cuda"
    kv = pkg.GlobalKV(B, cap, d, ratio, dev)
    pk = pkg.PagedKV(B, max_pages, page, n_pages, d, ratio, table, dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    for b, n in enumerate(lens):
        rows = synth.rows_normal_bf16(seed, "kv", b, 0, n, 512).view(1, n, 512).cuda()
        ik = synth.rows_normal_bf16(seed, "ik", b, 0, n, d).view(1, n, d).cuda()
        # one request at a time: the call appends T_kv rows to every request, so the
        # others start past any capacity and are skipped (CSA2_DEVERR_SLOT)
        full = torch.zeros(B, n, 512, dtype=torch.bfloat16, device=dev)
        fik = torch.zeros(B, n, d, dtype=torch.bfloat16, device=dev)
        full[b], fik[b] = rows[0], ik[0]
        start = torch.full((B,), 1 << 30, dtype=torch.int32, device=dev)   # past any cap: skipped
        start[b] = 0
        pkg.csa2_quantize_append(kv.struct, full, fik, n, start, None, None, 0, None, err)
        pkg.csa2_quantize_append_paged(pk.struct, full, fik, n, start, None, None, 0, None, None, err)
    bits = pkg.csa2_read_device_error(err)
    # the skipped rows of the other requests flag CSA2_DEVERR_SLOT only
    assert bits & ~pkg.DEVERR_SLOT == 0
    return kv, pk, table


def test_paged_bytes_and_index_calls(pkg):
    lens, page, d, H_I = [20000, 5000, 900], 256, 128, 4
    kv, pk, table = _layouts(pkg, lens, page)
    B = len(lens)
    for b, n in enumerate(lens):
        r = pk.rows_of(b, n)
        assert torch.equal(pk.codes[r], kv.codes[b, :n]) and torch.equal(pk.scales[r], kv.scales[b, :n])
        assert torch.equal(pk.idx_codes[r], kv.idx_codes[b, :n])
        assert torch.equal(pk.idx_scale[r], kv.idx_scale[b, :n])
    q_idx = torch.stack([synth.rows_normal_bf16(72, "qi", b, 0, H_I, d) for b in range(B)]).view(B, 1, H_I, d).cuda()
    w = torch.stack([synth.rows_uniform_f32(72, "w", b, 0, 1, H_I) for b in range(B)]).cuda()
    qp = torch.tensor([[n - 1] for n in lens], dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    N = max(lens)
    ws = torch.empty(pkg.csa2_workspace_size(pkg.CSA2_OP_INDEX_FULL, B, 1, N, 0, 512, 2048),
                     dtype=torch.uint8, device="cuda")
    out = {}
    for name, full, reidx, st in (("flat", pkg.csa2_index_full, pkg.csa2_index_reindex, kv.struct),
                                  ("paged", pkg.csa2_index_full_paged, None, pk.struct)):
        pool = torch.full((B, 1, 2048), -7, dtype=torch.int32, device="cuda")
        topk = torch.full((B, 1, 512), -7, dtype=torch.int32, device="cuda")
        cnt = torch.zeros(B, 1, dtype=torch.int32, device="cuda")
        full(st, q_idx, w, qp, 1, H_I, N, 2048, 512, pool, topk, cnt, ws, err)
        rt = torch.full((B, 1, 512), -7, dtype=torch.int32, device="cuda")
        rc = torch.zeros(B, 1, dtype=torch.int32, device="cuda")
        rws = torch.empty(pkg.csa2_workspace_size(pkg.CSA2_OP_INDEX_REINDEX, B, 1, 0, 0, 512, 2048),
                          dtype=torch.uint8, device="cuda")
        if reidx is not None:
            reidx(st, q_idx, w, qp, 1, H_I, pool, 2048, 512, rt, rc, rws, err)
        else:
            pkg.csa2_index_reindex_paged(st, q_idx, w, qp, 1, H_I, pool, 2048, 512, rt, rc, rws, err)
        out[name] = [x.cpu() for x in (pool, topk, cnt, rt, rc)]
    assert pkg.csa2_read_device_error(err) == 0
    for a, b in zip(out["flat"], out["paged"]):
        assert torch.equal(a, b)


@pytest.mark.parametrize("fused", [False, True])
def test_paged_attention(pkg, fused):
    lens, page, H = [3000, 1800], 512, 64
    kv, pk, table = _layouts(pkg, lens, page, seed=73)
    B = len(lens)
    W = 128
    dev = "cuda"
    rings = [pkg.SwaRing(B, W, dev) for _ in range(2)]
    t = torch.tensor([[n - 1] for n in lens], dtype=torch.int32, device=dev)
    for ring in rings:
        for b, n in enumerate(lens):
            rows = torch.zeros(B, W, 512, dtype=torch.bfloat16, device=dev)
            rows[b] = synth.rows_normal_bf16(74, "swa", b, 0, W, 512).cuda()
            st = torch.full((B,), -1, dtype=torch.int32, device=dev)       # negative: skipped
            st[b] = n - W
            pkg.csa2_quantize_append(None, None, None, 0, None, ring.struct, rows, W, st)
    g = torch.Generator().manual_seed(75)
    topk = torch.stack([torch.sort(torch.randperm(n, generator=g)[:512]).values for n in lens]).to(torch.int32)
    topk = topk.view(B, 1, 512).cuda()
    q = torch.stack([synth.rows_normal_bf16(76, "q", b, 0, H, 512, stride=synth.Q_STRIDE)
                     for b in range(B)]).view(B, 1, H, 512).cuda()
    new = torch.stack([synth.rows_normal_bf16(77, "new", b, 0, 1, 512) for b in range(B)]).view(B, 512).cuda()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    res = []
    for i, paged in enumerate((False, True)):
        o = torch.zeros(B, 1, H, 512, device=dev)
        l = torch.zeros(B, 1, H, device=dev)
        if paged:
            pkg.csa2_sparse_attn_decode_paged(pk.struct, rings[i].struct, new if fused else None, q, t, 1, H,
                                              topk, 512, W, 1 / math.sqrt(512), None, o, l, err)
        elif fused:
            pkg.csa2_sparse_attn_decode_append(kv.struct, rings[i].struct, new, q, t, 1, H, topk, 512, W,
                                               1 / math.sqrt(512), o, l, None, err)
        else:
            pkg.csa2_sparse_attn_decode(kv.struct, rings[i].struct, q, t, 1, H, topk, 512, W,
                                        1 / math.sqrt(512), o, l, None, err)
        res.append((o.cpu(), l.cpu(), rings[i].codes.cpu(), rings[i].scale.cpu()))
    assert pkg.csa2_read_device_error(err) == 0
    for a, b in zip(res[0], res[1]):
        assert torch.equal(a, b)


def test_bad_page_is_flagged_not_read(pkg):
    """A block-table entry outside the pool: the append skips the row and the attention
    drops the entries of that page, each with CSA2_DEVERR_PAGE."""
    lens, page = [1024], 256
    kv, pk, table = _layouts(pkg, lens, page, seed=78)
    bad = table.clone()
    bad[0, 1] = pk.n_pages + 3
    pk.block_table.copy_(bad)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    rows = synth.rows_normal_bf16(79, "kv", 0, 0, 512, 512).view(1, 512, 512).cuda()
    pkg.csa2_quantize_append_paged(pk.struct, rows, None, 512, torch.zeros(1, dtype=torch.int32, device="cuda"),
                                   None, None, 0, None, None, err)
    assert pkg.csa2_read_device_error(err) & pkg.DEVERR_PAGE
    topk = torch.arange(0, 512, dtype=torch.int32, device="cuda").view(1, 1, 512)
    q = synth.rows_normal_bf16(80, "q", 0, 0, 16, 512).view(1, 1, 16, 512).cuda()
    o = torch.zeros(1, 1, 16, 512, device="cuda")
    l = torch.zeros(1, 1, 16, device="cuda")
    t = torch.tensor([[1023]], dtype=torch.int32, device="cuda")
    pkg.csa2_sparse_attn_decode_paged(pk.struct, None, None, q, t, 1, 16, topk, 512, 0, 0.05, None, o, l, err)
    assert pkg.csa2_read_device_error(err) & pkg.DEVERR_PAGE
    assert torch.isfinite(o).all() and torch.isfinite(l).all()


@pytest.mark.parametrize("name,B,ctx,page", [("decoder_group_32k", 3, 20005, 256), ("decode_1m", 2, 6001, 1024)])
def test_paged_stack_equals_contiguous(pkg, name, B, ctx, page):
    """One decode step of the whole layer loop on paged caches (each group's pages handed
    to the requests in a shuffled order) equals the same step on contiguous caches, bit
    for bit: every layer's Top-K, counts, outputs and lse, and every group's pool."""
    import csa2_harness
    from synth.workloads import WORKLOADS, small_variant
    wl = small_variant(WORKLOADS[name], B=B, ctx=ctx)
    res = []
    for page_size in (0, page):
        dw = csa2_harness.DeviceWorkload(wl, page_size=page_size)
        dw.step()
        torch.cuda.synchronize()
        st = dw.stack
        assert st.dev_err.item() == 0
        res.append(({l: t.cpu() for l, t in st.topk.items()}, {l: c.cpu() for l, c in st.count.items()},
                    {g: p.cpu() for g, p in st.pool.items()}, [o.cpu() for o in st.out],
                    [x.cpu() for x in st.lse]))
        del dw, st
    (t0, c0, p0, o0, l0), (t1, c1, p1, o1, l1) = res
    for l in t0:
        assert torch.equal(t0[l], t1[l]) and torch.equal(c0[l], c1[l]), f"layer {l}"
    for g in p0:
        assert torch.equal(p0[g], p1[g]), f"group {g}"
    for l in range(len(o0)):
        assert torch.equal(o0[l], o1[l]) and torch.equal(l0[l], l1[l]), f"layer {l} output"
