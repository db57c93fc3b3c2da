"""The kernels' bounded waits, driven to run out on purpose (no fault, no hang).

csa2_debug_set_waits(limit, stuck) makes the first wait of every CTA of the
tensor-core kernels wait on a barrier that nothing signals, for `limit` ns of wall
time.  The call must then come back with CSA2_DEVERR_TIMEOUT in the device error
word, and the CTA must have waited for the MMAs it issued and freed its tensor
memory: the next ordinary call on the same stream must give the same results, bit
for bit, as a call made before the timeout.
"""
import math

import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000      # 2 ms: each stuck CTA gives up after this long


@pytest.fixture(scope="module")
def pkg():
    import fp4_kv_compressed_b200 as p
    assert torch.cuda.is_available()
    yield p
    p.csa2_debug_set_waits(p.DEFAULT_WAIT_LIMIT_NS, False)


def _run_tc_scan(pkg, kv, q, w, qp, Tq, H_I, N, pool_blocks, top_k):
    B = qp.shape[0]
    pool = torch.full((B, Tq, pool_blocks), -7, dtype=torch.int32, device="cuda")
    topk = torch.full((B, Tq, top_k), -7, dtype=torch.int32, device="cuda")
    cnt = torch.full((B, Tq), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(pkg.csa2_workspace_size(pkg.CSA2_OP_INDEX_FULL, B, Tq, N, 0, top_k,
                                             pool_blocks), dtype=torch.uint8, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkg.csa2_index_full_tc(kv.struct, q, w, qp, Tq, H_I, N, pool_blocks, top_k, pool, topk, cnt,
                           ws, err)
    bits = pkg.csa2_read_device_error(err)
    return bits, pool.cpu(), topk.cpu(), cnt.cpu()


def test_tc_scan_wait_runs_out_then_recovers(pkg):
    B, N, d, H_I, Tq = 2, 4000, 128, 4, 96
    rows = torch.stack([synth.rows_normal_bf16(81, "rows", b, 0, N, d) for b in range(B)])
    kv = pkg.GlobalKV(B, N, d, 1, "cuda")
    z = torch.zeros(B, dtype=torch.int32, device="cuda")
    pkg.csa2_quantize_append(kv.struct, None, rows.cuda(), N, z, None, None, 0, None)
    q = torch.stack([synth.rows_normal_bf16(82, "q", b, 0, Tq * H_I, d)
                     for b in range(B)]).view(B, Tq, H_I, d).cuda()
    w = torch.stack([synth.rows_uniform_f32(82, "w", b, 0, Tq, H_I) for b in range(B)]).cuda()
    qp = torch.tensor([[N - Tq + t for t in range(Tq)]] * B, dtype=torch.int32, device="cuda")
    args = (pkg, kv, q, w, qp, Tq, H_I, N, 512, 512)

    bits0, *ref = _run_tc_scan(*args)
    assert bits0 == 0
    pkg.csa2_debug_set_waits(LIMIT_NS, True)
    try:
        bits1, *_ = _run_tc_scan(*args)
    finally:
        pkg.csa2_debug_set_waits(pkg.DEFAULT_WAIT_LIMIT_NS, False)
    assert bits1 & pkg.DEVERR_TIMEOUT, f"device error bits {bits1:#x}: the wait did not run out"
    # the context is usable and the tensor memory was freed: the same call again
    for _ in range(2):
        bits2, *got = _run_tc_scan(*args)
        assert bits2 == 0
        for a, b in zip(ref, got):
            assert torch.equal(a, b)


def test_attention_wait_runs_out_then_recovers(pkg):
    """The same for the sparse attention: a stuck wait in every CTA of every
    cluster (after the first score MMAs were issued) must end the call with the timeout
    bit, every CTA still meeting at the cluster barriers of the combine, and leave the
    tensor memory free for the next call."""
    import math
    B, cap, H, W = 3, 1500, 64, 128
    kv = pkg.GlobalKV(B, cap, 128, 1, "cuda")
    ring = pkg.SwaRing(B, W, "cuda")
    x = torch.stack([synth.rows_normal_bf16(83, "kv", b, 0, cap, 512) for b in range(B)]).cuda()
    sw = torch.stack([synth.rows_normal_bf16(83, "swa", b, 0, W, 512) for b in range(B)]).cuda()
    z = torch.zeros(B, dtype=torch.int32, device="cuda")
    pkg.csa2_quantize_append(kv.struct, x, None, cap, z, ring.struct, sw, W, z)
    g = torch.Generator().manual_seed(84)
    topk = torch.stack([torch.sort(torch.randperm(cap, generator=g)[:512]).values
                        for _ in range(B)]).to(torch.int32).view(B, 1, 512).cuda()
    q = torch.stack([synth.rows_normal_bf16(85, "q", b, 0, H, 512, stride=synth.Q_STRIDE)
                     for b in range(B)]).view(B, 1, H, 512).cuda()
    qp = torch.full((B, 1), cap - 1, dtype=torch.int32, device="cuda")

    def run():
        o = torch.full((B, 1, H, 512), 7.0, device="cuda")
        l = torch.full((B, 1, H), 7.0, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        pkg.csa2_sparse_attn_decode(kv.struct, ring.struct, q, qp, 1, H, topk, 512, W,
                                    1 / math.sqrt(512), o, l, None, err)
        return pkg.csa2_read_device_error(err), o.cpu(), l.cpu()

    bits0, o0, l0 = run()
    assert bits0 == 0
    pkg.csa2_debug_set_waits(LIMIT_NS, True)
    try:
        bits1, _, _ = run()
    finally:
        pkg.csa2_debug_set_waits(pkg.DEFAULT_WAIT_LIMIT_NS, False)
    assert bits1 & pkg.DEVERR_TIMEOUT, f"device error bits {bits1:#x}: the wait did not run out"
    for _ in range(2):
        bits2, o2, l2 = run()
        assert bits2 == 0 and torch.equal(o2, o0) and torch.equal(l2, l0)
