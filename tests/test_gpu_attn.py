"""GPU parity of sparse attention (a8) and of whole stack steps (a1-a9) against
the oracle: Top-K bit-exact, attention within 2e-3 (norm-wise per head row)."""
import math

import numpy as np
import pytest
import torch

from oracle import workload_ref as R
import synth
from synth.workloads import WORKLOADS, small_variant

pytestmark = pytest.mark.gpu

ATTN_TOL = 2e-3      # max_c |o - o_ref| / max_c |o_ref| per (request, query, head)
LSE_TOL = 1e-3       # absolute, natural-log units


@pytest.fixture(scope="module")
def pkg():
    import fp4_kv_compressed_b200 as p
    assert torch.cuda.is_available()
    return p


def _attn_case(pkg, orc, *, B, H, cap, W, q_pos, topk, swa_len, seed):
    kv = pkg.GlobalKV(B, cap, 128, 1, "cuda")
    ring = pkg.SwaRing(B, W, "cuda")
    x = torch.stack([synth.rows_normal_bf16(seed, "kv", b, 0, cap, 512) for b in range(B)])
    s = torch.stack([(synth.rows_normal_bf16(seed, "swa", b, 0, W, 512).float() * 3)
                     .to(torch.bfloat16) for b in range(B)])
    z = torch.zeros(B, dtype=torch.int32, device="cuda")
    pkg.csa2_quantize_append(kv.struct, x.cuda(), None, cap, z, ring.struct, s.cuda(), W, z)
    Tq = q_pos.shape[1]
    q = torch.stack([synth.rows_normal_bf16(seed, "q", b, 0, Tq * H, 512, stride=synth.Q_STRIDE)
                     for b in range(B)]).view(B, Tq, H, 512)
    out = torch.zeros(B, Tq, H, 512, device="cuda")
    lse = torch.zeros(B, Tq, H, device="cuda")
    dev_err = torch.zeros(1, dtype=torch.int32, device="cuda")
    top_k = topk.shape[-1]
    pkg.csa2_sparse_attn_decode(kv.struct, ring.struct if swa_len else None, q.cuda(),
                                q_pos.cuda(), Tq, H, topk.cuda() if top_k else None, top_k,
                                swa_len, 1 / math.sqrt(512), out, lse, None, dev_err)
    bits = pkg.csa2_read_device_error(dev_err)
    mc, ms = orc.quantize_fp4(x)
    sc, ss = orc.quantize_fp8(s)
    tk = topk.numpy() if top_k else np.full((B, Tq, 1), -1, np.int32)
    o_ref, l_ref = orc.attention(mc, ms, sc, ss, q, q_pos.numpy(), tk, swa_len, 1 / math.sqrt(512))
    return out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, bits


def _assert_close(o, l, o_ref, l_ref):
    err = R.rel_err_rows(o, o_ref)
    # reported beside the norm-wise figure: the elementwise relative error of the
    # elements at least as large as their row's RMS
    print(f"attention: norm-wise row error {err.max():.2e}, "
          f"elementwise (|o_ref| >= row RMS) {R.rel_err_elems(o, o_ref):.2e}")
    assert err.max() <= ATTN_TOL, f"max row error {err.max():.3e}"
    fin = np.isfinite(l_ref)
    assert np.array_equal(np.isfinite(l), fin)
    assert np.abs(l[fin] - l_ref[fin]).max(initial=0) <= LSE_TOL


@pytest.mark.parametrize("H", [16, 64])
def test_attention_random_sets(pkg, orc, H):
    B, cap, W = 2, 700, 128
    g = torch.Generator().manual_seed(H)
    q_pos = torch.tensor([[699], [450]], dtype=torch.int32)
    topk = torch.randint(-1, 451, (B, 1, 96), generator=g, dtype=torch.int32)
    topk[0, 0, :10] = torch.arange(690, 700, dtype=torch.int32)      # recent entries, duplicates w/ window
    o, l, o_ref, l_ref, bits = _attn_case(pkg, orc, B=B, H=H, cap=cap, W=W, q_pos=q_pos,
                                          topk=topk, swa_len=128, seed=H)
    assert bits == 0
    _assert_close(o, l, o_ref, l_ref)


def test_attention_edges(pkg, orc):
    B, cap, W = 2, 300, 130
    # window only, early position (window clipped at 0), ring wider than the window
    q_pos = torch.tensor([[5], [200]], dtype=torch.int32)
    o, l, o_ref, l_ref, _ = _attn_case(pkg, orc, B=B, H=16, cap=cap, W=W, q_pos=q_pos,
                                       topk=torch.zeros(B, 1, 0, dtype=torch.int32),
                                       swa_len=128, seed=1)
    _assert_close(o, l, o_ref, l_ref)
    # selected entries only (no window), with -1 padding
    topk = torch.full((B, 1, 64), -1, dtype=torch.int32)
    topk[0, 0, :3] = torch.tensor([0, 1, 5])
    topk[1, 0, :40] = torch.arange(100, 140)
    o, l, o_ref, l_ref, _ = _attn_case(pkg, orc, B=B, H=32, cap=cap, W=W, q_pos=q_pos,
                                       topk=topk, swa_len=0, seed=2)
    _assert_close(o, l, o_ref, l_ref)
    # nothing at all: o = 0, lse = -inf
    topk = torch.full((B, 1, 8), -1, dtype=torch.int32)
    o, l, o_ref, l_ref, _ = _attn_case(pkg, orc, B=B, H=16, cap=cap, W=W, q_pos=q_pos,
                                       topk=topk, swa_len=0, seed=3)
    assert not o.any() and np.isneginf(l).all()
    # an id past the visible range is skipped and flagged
    topk = torch.full((B, 1, 8), 250, dtype=torch.int32)
    _, _, _, _, bits = _attn_case(pkg, orc, B=B, H=16, cap=cap, W=W, q_pos=q_pos,
                                  topk=topk, swa_len=4, seed=4)
    assert bits & pkg.DEVERR_INDEX


@pytest.mark.parametrize("B,top_k", [(1, 384), (1, 512), (12, 512), (38, 512)])
def test_attention_running_max_moves_every_tile(pkg, orc, B, top_k):
    """Entry e is c_e times head 0 of the query, c_e growing along the key order, so the
    logits of every later 64-key tile exceed the running max by more than 8 (log2 units):
    the max moves and O is rescaled on every tile, by each worker set in turn (after the
    other set's output MMAs of the previous tile).  B = 1 and 12: 4 CTAs per query, 2 or
    3 tiles each; B = 38: 2 CTAs per query, 5 tiles each.  Within the tolerance of the
    oracle."""
    H, cap, W = 64, 700, 128
    q_pos = torch.full((B, 1), 699, dtype=torch.int32)
    q = torch.stack([synth.rows_normal_bf16(9, "q", b, 0, H, 512, stride=synth.Q_STRIDE)
                     for b in range(B)]).view(B, 1, H, 512)
    c = torch.arange(cap, dtype=torch.float32) * 0.006
    x = (c.view(1, cap, 1) * q[:, 0, 0].float().view(B, 1, 512)).to(torch.bfloat16)
    sw = torch.stack([synth.rows_normal_bf16(9, "swa", b, 0, W, 512) for b in range(B)])
    kv = pkg.GlobalKV(B, cap, 128, 1, "cuda")
    ring = pkg.SwaRing(B, W, "cuda")
    z = torch.zeros(B, dtype=torch.int32, device="cuda")
    pkg.csa2_quantize_append(kv.struct, x.cuda(), None, cap, z, ring.struct, sw.cuda(), W, z)
    topk = torch.arange(top_k, dtype=torch.int32).view(1, 1, top_k).expand(B, 1, top_k).contiguous()
    out = torch.zeros(B, 1, H, 512, device="cuda")
    lse = torch.zeros(B, 1, H, device="cuda")
    dev_err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkg.csa2_sparse_attn_decode(kv.struct, ring.struct, q.cuda(), q_pos.cuda(), 1, H, topk.cuda(), top_k,
                                128, 1 / math.sqrt(512), out, lse, None, dev_err)
    assert pkg.csa2_read_device_error(dev_err) == 0
    mc, ms = orc.quantize_fp4(x)
    sc, ss = orc.quantize_fp8(sw)
    o_ref, l_ref = orc.attention(mc, ms, sc, ss, q, q_pos.numpy(), topk.numpy(), 128, 1 / math.sqrt(512))
    # the premise: head 0's logits (log2 units) rise by more than 8 per 64 entries
    qq = q[0, 0, 0].double()
    step = float((qq * qq).sum()) * 0.006 * 64 / math.sqrt(512) / math.log(2)
    assert step > 8
    _assert_close(out.cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref)


@pytest.mark.parametrize("name,rope,ctx", [("decode_128k", False, 6000), ("decode_1m", False, 6000),
                                           ("decode_128k", True, 6000), ("decode_128k", False, 12)])
def test_reuse_launch_matches_ordinary_calls(pkg, name, rope, ctx):
    """Reuse layers launched with csa2_sparse_attn_decode_reuse and Reindex layers with
    csa2_index_reindex_settled (loads before the wait for the previous launch) give the
    same outputs and lse on every layer, bit for bit, as the ordinary calls: whole decode
    stacks, so that every such launch follows another layer's launch on the stream; with
    RoPE, the fused append's rotation goes through the same call.  A 12-token context
    leaves two of each query's four CTAs without keys (their wait is the combine's)."""
    import csa2_harness
    wl = small_variant(WORKLOADS[name], B=4, ctx=ctx)
    res = []
    for reuse in (False, True):
        dw = csa2_harness.DeviceWorkload(wl, rope=rope)
        dw.stack.reuse_launch = reuse
        st = torch.cuda.Stream()      # a real stream, where launches may overlap
        st.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(st):
            dw.step(stream=st)
        torch.cuda.synchronize()
        assert dw.stack.dev_err.item() == 0
        res.append([t.clone() for t in dw.stack.out] + [t.clone() for t in dw.stack.lse])
    assert len(res[0]) > 0
    for a, b in zip(*res):
        assert torch.equal(a, b)


def _stack_check(wl, requests, layers=None):
    import csa2_harness
    dw = csa2_harness.DeviceWorkload(wl)
    dw.step()
    torch.cuda.synchronize()
    assert dw.stack.dev_err.item() == 0
    plan = R.reuse_sources(wl)
    for b in requests:
        gpu = dw.request_state(b)
        # main rows needed: every selected entry of every selector layer
        rows = {g: [] for g in range(len(wl.groups))}
        for layer, t in gpu["topk"].items():
            rows[plan[layer][0]].append(t.ravel())
        rows = {g: np.concatenate(v) if v else np.zeros(0, np.int64) for g, v in rows.items()}
        caches = R.request_caches(wl, b, main_rows=rows)
        for g, c in enumerate(caches):
            assert np.array_equal(gpu["kv"][g]["codes"][c["rows"]], c["codes"][c["rows"]])
            assert np.array_equal(gpu["kv"][g]["scales"][c["rows"]], c["scales"][c["rows"]])
        ref = R.index_layers(wl, b, caches)
        for layer, t in ref["topk"].items():
            assert np.array_equal(gpu["topk"][layer], t), f"request {b} layer {layer}"
        for layer in (range(len(plan)) if layers is None else layers):
            src = plan[layer][2]
            o_ref, l_ref = R.attention_layer(wl, b, layer, caches, ref["topk"][src])
            _assert_close(gpu["out"][layer], gpu["lse"][layer], o_ref, l_ref)


def test_stack_decoder_group(pkg):
    """Decoder group (F + 4X + 15U) on 2 requests at N = 20000, every layer."""
    _stack_check(small_variant(WORKLOADS["decoder_group_32k"], B=2, ctx=20000), [0, 1])


def test_stack_tiny(pkg):
    _stack_check(WORKLOADS["tiny_full_layer"], [0])


def test_stack_prefill_chunk(pkg):
    """Encoder group, ratio 2, 64 causal queries sharing the cache, every layer."""
    _stack_check(small_variant(WORKLOADS["prefill_chunk_enc"], B=1, ctx=3000 + 64, Tq=64), [0])


def test_stack_scaled_channels(pkg):
    """Per-channel log-uniform scales on the main KV and SWA (the 128K workload's inputs)."""
    _stack_check(small_variant(WORKLOADS["decode_128k"], B=2, ctx=5000), [1],
                 layers=[0, 3, 4, 19])


def test_fused_swa_append_matches_separate(pkg):
    """csa2_sparse_attn_decode_append == csa2_quantize_append (SWA row) followed by
    csa2_sparse_attn_decode: the same ring bytes and the same outputs, bit for bit,
    for H = 64 and H = 128 (two head groups), and at a position where the window is
    still filling (t < swa_len - 1)."""
    import synth
    for H, t_last in ((64, 2999), (128, 2999), (64, 40)):
        B, cap, W = 3, 3000, 160
        kv = pkg.GlobalKV(B, cap, 128, 1, "cuda")
        x = torch.stack([synth.rows_normal_bf16(31, "kv", b, 0, cap, 512) for b in range(B)])
        z = torch.zeros(B, dtype=torch.int32, device="cuda")
        pkg.csa2_quantize_append(kv.struct, x.cuda(), None, cap, z, None, None, 0, None)
        rings = [pkg.SwaRing(B, W, "cuda") for _ in range(2)]
        n_old = min(t_last, W - 1)          # the ring holds the previous W - 1 tokens
        p_old = t_last - n_old
        old = torch.stack([synth.rows_normal_bf16(32, "swa", b, p_old, n_old, 512) for b in range(B)])
        s_old = torch.full((B,), p_old, dtype=torch.int32, device="cuda")
        if n_old > 0:
            for r in rings:
                pkg.csa2_quantize_append(None, None, None, 0, None, r.struct, old.cuda(), n_old, s_old)
        new = torch.stack([synth.rows_normal_bf16(33, "new", b, 0, 1, 512) for b in range(B)]).cuda()
        q = torch.stack([synth.rows_normal_bf16(34, "q", b, 0, H, 512, stride=synth.Q_STRIDE)
                         for b in range(B)]).view(B, 1, H, 512).cuda()
        q_pos = torch.full((B, 1), t_last, dtype=torch.int32, device="cuda")
        g = torch.Generator().manual_seed(35)
        vis = min(t_last + 1, cap)
        topk = torch.stack([torch.sort(torch.randperm(vis, generator=g)[:min(512, vis)]).values
                            for _ in range(B)]).view(B, 1, -1).int().cuda()
        K = topk.shape[-1]
        outs = [torch.zeros(B, 1, H, 512, device="cuda") for _ in range(2)]
        lses = [torch.zeros(B, 1, H, device="cuda") for _ in range(2)]
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        start = torch.full((B,), t_last, dtype=torch.int32, device="cuda")
        pkg.csa2_quantize_append(None, None, None, 0, None, rings[0].struct, new.view(B, 1, 512), 1,
                                 start, err)
        pkg.csa2_sparse_attn_decode(kv.struct, rings[0].struct, q, q_pos, 1, H, topk, K, 128,
                                    512 ** -0.5, outs[0], lses[0], None, err)
        pkg.csa2_sparse_attn_decode_append(kv.struct, rings[1].struct, new, q, q_pos, 1, H, topk, K,
                                           128, 512 ** -0.5, outs[1], lses[1], None, err)
        torch.cuda.synchronize()
        assert pkg.csa2_read_device_error(err) == 0
        assert torch.equal(rings[0].codes, rings[1].codes)
        assert torch.equal(rings[0].scale.view(torch.int32), rings[1].scale.view(torch.int32))
        assert torch.equal(outs[0].view(torch.int32), outs[1].view(torch.int32))
        assert torch.equal(lses[0].view(torch.int32), lses[1].view(torch.int32))
