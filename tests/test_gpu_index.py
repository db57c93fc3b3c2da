"""GPU parity of the index path (a3-a7): scores, block pool, Top-K (Full, flat,
hierarchical, ratio 2), Reindex and Reuse -- bit-exact against the oracle."""
import numpy as np
import pytest
import torch

import oracle_ref as R
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


def test_flat_unstaged_and_hierarchical_million_shape(harness):
    """Encoder groups with N = 20000 (> 16384: selection streams keys from global
    memory) next to a decoder group with N = 40000."""
    wl = small_variant(WORKLOADS["decode_1m"], B=2, ctx=40000)
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
