"""GPU parity of RoPE inside the append (csa2_quantize_append_rope and the fused
decode append) against the oracle: rotate (oracle.rope_rows), then quantise -- codes,
scales and ring bytes bit-exact."""
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


def _rows(seed, name, B, T, W):
    return torch.stack([synth.rows_normal_bf16(seed, name, b, 0, T, W) for b in range(B)])


def _append_case(pkg, orc, ratio, start, pairs, n_pos, kv_start, swa_start, seed):
    B, cap, T, d, W = len(kv_start), 400, 40, 128, 64
    kv = pkg.GlobalKV(B, cap, d, ratio, "cuda")
    ring = pkg.SwaRing(B, W, "cuda")
    x, ik, sw = _rows(seed, "kv", B, T, 512), _rows(seed, "ik", B, T, d), _rows(seed, "sw", B, T, 512)
    table = synth.rope_table(n_pos, pairs)
    rope = pkg.Rope(table, start, pairs)
    ks = torch.tensor(kv_start, dtype=torch.int32, device="cuda")
    ss = torch.tensor(swa_start, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkg.csa2_quantize_append_rope(kv.struct, x.cuda(), ik.cuda(), T, ks, ring.struct, sw.cuda(), T,
                                  ss, rope.struct, err)
    bits = pkg.csa2_read_device_error(err)
    n_outside = 0
    for b in range(B):
        e = kv_start[b] + np.arange(T)
        rot, n = orc.rope_rows(x[b], e * ratio + ratio - 1, table, start, pairs)
        n_outside += n
        c, s = orc.quantize_fp4(rot)
        assert np.array_equal(kv.codes[b, e].cpu().numpy(), c), b
        assert np.array_equal(kv.scales[b, e].cpu().numpy(), s), b
        c, s = orc.quantize_fp8(ik[b])                          # indexer K: not rotated
        assert np.array_equal(kv.idx_codes[b, e].cpu().numpy(), c), b
        assert np.array_equal(kv.idx_scale[b, e].cpu().numpy().view(np.uint32), s.view(np.uint32)), b
        p = swa_start[b] + np.arange(T)
        rot, n = orc.rope_rows(sw[b], p, table, start, pairs)
        n_outside += n
        c, s = orc.quantize_fp8(rot)
        assert np.array_equal(ring.codes[b, p % W].cpu().numpy(), c), b
        assert np.array_equal(ring.scale[b, p % W].cpu().numpy().view(np.uint32), s.view(np.uint32)), b
    return bits, n_outside


@pytest.mark.parametrize("ratio,start,pairs", [(1, 448, 32), (2, 0, 256), (1, 6, 5)])
def test_quantize_append_rope_matches_oracle(pkg, orc, ratio, start, pairs):
    """Main-KV entries (at position ratio * slot + ratio - 1) and SWA rows (at their
    token position) are rotated then quantised; the indexer K is left as given."""
    bits, n_out = _append_case(pkg, orc, ratio, start, pairs, 4000, [0, 100, 300], [0, 3000, 77],
                               seed=80 + pairs)
    assert bits == 0 and n_out == 0


def test_rope_position_outside_table_is_flagged(pkg, orc):
    """Rows past the end of the table are stored unrotated and flag CSA2_DEVERR_ROPE."""
    bits, n_out = _append_case(pkg, orc, 1, 448, 32, 120, [0, 100], [10, 90], seed=90)
    assert n_out > 0 and bits == pkg.DEVERR_ROPE


def test_fused_swa_append_rope_matches_separate(pkg, orc):
    """csa2_sparse_attn_decode_append_rope == csa2_quantize_append_rope (SWA row) then
    csa2_sparse_attn_decode: the same ring bytes (those of the oracle) and the same
    outputs, bit for bit, for H = 64 and 128."""
    for H in (64, 128):
        B, cap, W, t_last = 3, 3000, 160, 2999
        kv = pkg.GlobalKV(B, cap, 128, 1, "cuda")
        x = _rows(91, "kv", B, cap, 512)
        z = torch.zeros(B, dtype=torch.int32, device="cuda")
        pkg.csa2_quantize_append(kv.struct, x.cuda(), None, cap, z, None, None, 0, None)
        table = synth.rope_table(4096, 32)
        rope = pkg.Rope(table, 448, 32)
        rings = [pkg.SwaRing(B, W, "cuda") for _ in range(2)]
        n_old = W - 1
        p_old = t_last - n_old
        old = torch.stack([synth.rows_normal_bf16(92, "swa", b, p_old, n_old, 512) for b in range(B)])
        s_old = torch.full((B,), p_old, dtype=torch.int32, device="cuda")
        for r in rings:
            pkg.csa2_quantize_append_rope(None, None, None, 0, None, r.struct, old.cuda(), n_old,
                                          s_old, rope.struct)
        new = _rows(93, "new", B, 1, 512).cuda()
        q = torch.stack([synth.rows_normal_bf16(94, "q", b, 0, H, 512, stride=synth.Q_STRIDE)
                         for b in range(B)]).view(B, 1, H, 512).cuda()
        q_pos = torch.full((B, 1), t_last, dtype=torch.int32, device="cuda")
        g = torch.Generator().manual_seed(95)
        topk = torch.stack([torch.sort(torch.randperm(cap, generator=g)[:512]).values
                            for _ in range(B)]).view(B, 1, -1).int().cuda()
        outs = [torch.zeros(B, 1, H, 512, device="cuda") for _ in range(2)]
        lses = [torch.zeros(B, 1, H, device="cuda") for _ in range(2)]
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        start = torch.full((B,), t_last, dtype=torch.int32, device="cuda")
        pkg.csa2_quantize_append_rope(None, None, None, 0, None, rings[0].struct, new.view(B, 1, 512), 1,
                                      start, rope.struct, err)
        pkg.csa2_sparse_attn_decode(kv.struct, rings[0].struct, q, q_pos, 1, H, topk, 512, 128,
                                    512 ** -0.5, outs[0], lses[0], None, err)
        pkg.csa2_sparse_attn_decode_append_rope(kv.struct, rings[1].struct, new, q, q_pos, 1, H, topk,
                                                512, 128, 512 ** -0.5, rope.struct, outs[1], lses[1],
                                                None, err)
        torch.cuda.synchronize()
        assert pkg.csa2_read_device_error(err) == 0
        assert torch.equal(rings[0].codes, rings[1].codes)
        assert torch.equal(rings[0].scale.view(torch.int32), rings[1].scale.view(torch.int32))
        assert torch.equal(outs[0].view(torch.int32), outs[1].view(torch.int32))
        assert torch.equal(lses[0].view(torch.int32), lses[1].view(torch.int32))
        rot, _ = orc.rope_rows(new.cpu().view(B, 512), np.full(B, t_last), table, 448, 32)
        c, s = orc.quantize_fp8(rot)
        slot = t_last % W
        assert np.array_equal(rings[1].codes[:, slot].cpu().numpy(), c)
        assert np.array_equal(rings[1].scale[:, slot].cpu().numpy().view(np.uint32), s.view(np.uint32))
