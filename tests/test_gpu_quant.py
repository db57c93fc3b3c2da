"""GPU parity of quantise-append (a1/a2): FP4 codes and E4M3 scales, FP8 index-K and
SWA rows, slots and the SWA ring -- bit-exact against the oracle."""
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


def _all_bf16_rows():
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    x = bits[torch.isfinite(bits.float())]
    pad = (-x.numel()) % 512
    x = torch.cat([x, torch.zeros(pad, dtype=torch.bfloat16)])
    return x.view(-1, 512)


def _sweep_rows():
    """Every finite bf16 value, in groups whose amax varies over the full range, plus the
    same values scaled by powers of two (scale sweep), plus N(0,1) rows."""
    base = _all_bf16_rows()
    g = torch.Generator().manual_seed(0)
    perm = base.flatten()[torch.randperm(base.numel(), generator=g)].view(-1, 512)
    scaled = [(perm.float() * 2.0 ** e).to(torch.bfloat16) for e in (-30, -12, -4, 3, 9)]
    normal = synth.rows_normal_bf16(9, "q", 0, 0, 256, 512)
    rows = torch.cat([base, perm, *scaled, normal])
    rows = torch.where(torch.isfinite(rows.float()), rows, torch.zeros_like(rows))
    return rows.contiguous()


def test_fp4_quantise_exhaustive(pkg, orc):
    rows = _sweep_rows()
    n = rows.shape[0]
    kv = pkg.GlobalKV(1, n, 128, 1, "cuda")
    dev_err = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = rows.view(1, n, 512).cuda()
    start = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkg.csa2_quantize_append(kv.struct, x, None, n, start, None, None, 0, None, dev_err)
    assert pkg.csa2_read_device_error(dev_err) == 0
    codes, scales = orc.quantize_fp4(rows)
    gc = kv.codes[0].cpu().numpy()
    gs = kv.scales[0].cpu().numpy()
    bad_s = np.argwhere(gs != scales)
    assert bad_s.size == 0, f"{len(bad_s)} scale mismatches, first {bad_s[:4]}"
    bad_c = np.argwhere(gc != codes)
    assert bad_c.size == 0, f"{len(bad_c)} code-byte mismatches, first {bad_c[:4]}"


@pytest.mark.parametrize("d", [64, 128])
def test_fp8_index_rows(pkg, orc, d):
    n = 4096
    g = torch.Generator().manual_seed(d)
    mags = torch.exp2(torch.randint(-40, 20, (n, 1), generator=g).float())
    rows = (synth.rows_normal_bf16(3, "k", 0, 0, n, d).float() * mags).to(torch.bfloat16)
    rows[0] = 0
    rows[1, :5] = torch.tensor([-0.0, 1e-30, -1e-30, 3.0, -448.0])
    kv = pkg.GlobalKV(1, n, d, 1, "cuda")
    start = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkg.csa2_quantize_append(kv.struct, None, rows.view(1, n, d).cuda(), n, start, None, None,
                             0, None)
    kc, ks = orc.quantize_fp8(rows)
    assert np.array_equal(kv.idx_scale[0].cpu().numpy(), ks)
    assert np.array_equal(kv.idx_codes[0].cpu().numpy(), kc)


def test_swa_ring_and_slots(pkg, orc):
    B, W, T = 3, 130, 7
    ring = pkg.SwaRing(B, W, "cuda")
    kv = pkg.GlobalKV(B, 50, 128, 1, "cuda")
    dev_err = torch.zeros(1, dtype=torch.int32, device="cuda")
    swa_rows = torch.stack([synth.rows_normal_bf16(5, "s", b, 0, T, 512) for b in range(B)])
    kv_rows = torch.stack([synth.rows_normal_bf16(6, "kv", b, 0, T, 512) for b in range(B)])
    ik_rows = torch.stack([synth.rows_normal_bf16(7, "ik", b, 0, T, 128) for b in range(B)])
    swa_start = torch.tensor([0, 126, 1000], dtype=torch.int32, device="cuda")   # wraps the ring
    kv_start = torch.tensor([0, 40, 45], dtype=torch.int32, device="cuda")       # last overflows
    pkg.csa2_quantize_append(kv.struct, kv_rows.cuda(), ik_rows.cuda(), T, kv_start, ring.struct,
                             swa_rows.cuda(), T, swa_start, dev_err)
    bits = pkg.csa2_read_device_error(dev_err)
    assert bits == pkg.DEVERR_SLOT
    for b in range(B):
        c, s = orc.quantize_fp8(swa_rows[b])
        for i in range(T):
            slot = (int(swa_start[b]) + i) % W
            assert np.array_equal(ring.codes[b, slot].cpu().numpy(), c[i])
            assert ring.scale[b, slot].item() == s[i]
        mc, ms = orc.quantize_fp4(kv_rows[b])
        kc, ks = orc.quantize_fp8(ik_rows[b])
        for i in range(T):
            e = int(kv_start[b]) + i
            if e >= 50:
                continue
            assert np.array_equal(kv.codes[b, e].cpu().numpy(), mc[i])
            assert np.array_equal(kv.scales[b, e].cpu().numpy(), ms[i])
            assert np.array_equal(kv.idx_codes[b, e].cpu().numpy(), kc[i])
            assert kv.idx_scale[b, e].item() == ks[i]
    # rows past the cache were skipped: slots 45..49 written, nothing else touched
    assert not kv.codes[0, T:].any()
