"""Pins of the oracle's number formats (E2M1, E4M3) and its FP4/FP8 quantisers.

Each check ties the oracle to something other than itself: the printed format
invariants, the formats' value tables, PyTorch's independent float8_e4m3fn
conversion, hand-worked groups, and properties (nearest value, ties to even,
monotonicity, exact round trip, error bound).
"""
import math

import numpy as np
import pytest
import torch

from conftest import golden_lines

E2M1_MAGS = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def all_finite_bf16() -> torch.Tensor:
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    x = bits.view(torch.bfloat16)
    return x[torch.isfinite(x.float())]


# ---- value tables -----------------------------------------------------------------------------
def test_e2m1_table_matches_golden(orc):
    rows = [ln.split() for ln in golden_lines("e2m1_values.txt")]
    assert len(rows) == 16
    for code, val in rows:
        v = orc.e2m1_value(int(code))
        assert v == float(val) and math.copysign(1, v) == math.copysign(1, float(val))


def test_e4m3_anchors_match_golden(orc):
    for code, val in (ln.split() for ln in golden_lines("e4m3_anchor_values.txt")):
        v = orc.e4m3_value(int(code, 16))
        assert v == float(val) and math.copysign(1, v) == math.copysign(1, float(val))


def test_e4m3_table_matches_torch_float8():
    """All 256 codes decoded by the oracle equal PyTorch's float8_e4m3fn decode."""
    import oracle
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).float().double().numpy()
    for c in range(256):
        v = oracle.e4m3_value(c)
        if c in (0x7F, 0xFF):
            assert math.isnan(v) and math.isnan(ref[c])
        else:
            assert v == ref[c], hex(c)


def test_invariant_bits_per_value():
    inv = dict(ln.split() for ln in golden_lines("format_invariants.txt"))
    group = int(inv["group"])
    bits = 4 + 8 / group
    assert bits == float(inv["bits_per_value"])
    # a 512-channel entry: 256 code bytes + 32 scale bytes = 288 B = 4.5 bits/value
    assert (512 // 2 + 512 // group) * 8 / 512 == float(inv["bits_per_value"])


# ---- E4M3 encoder -----------------------------------------------------------------------------
def test_e4m3_encode_equals_torch_rne_on_all_bf16(orc):
    x = all_finite_bf16().float()
    ours = np.array([orc.e4m3_encode(float(v)) for v in x], dtype=np.int64)
    inside = x.abs() < 448
    ref = x[inside].to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(np.int64)
    assert np.array_equal(ours[inside.numpy()], ref)
    # saturation: |x| >= 448 -> +-448, sign kept
    sat = ours[~inside.numpy()]
    sgn = torch.signbit(x[~inside]).numpy()
    assert np.all(sat == np.where(sgn, 0xFE, 0x7E))


def test_e4m3_encode_equals_torch_rne_on_fp32_sweep(orc):
    g = torch.Generator().manual_seed(7)
    x = torch.exp2(torch.empty(20000).uniform_(-12, 8.8, generator=g)) * \
        torch.where(torch.rand(20000, generator=g) < 0.5, -1.0, 1.0)
    x = x.float()
    ours = np.array([orc.e4m3_encode(float(v)) for v in x], dtype=np.int64)
    inside = (x.abs() < 448).numpy()
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy().astype(np.int64)
    assert np.array_equal(ours[inside], ref[inside])


# ---- E2M1 encoder -----------------------------------------------------------------------------
def test_e2m1_worked_ties():
    import oracle
    # ties go to the even mantissa (round-to-nearest-even)
    expect = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for r, v in expect.items():
        assert oracle.e2m1_value(oracle.e2m1_encode(r)) == v
        assert oracle.e2m1_value(oracle.e2m1_encode(-r)) == -v


def test_e2m1_encode_nearest_monotone_saturating(orc):
    r = np.concatenate([np.linspace(-8, 8, 40001), np.array([6.0, -6.0, 6.5, -100.0, 100.0])])
    r = r.astype(np.float32)
    codes = np.array([orc.e2m1_encode(float(v)) for v in r])
    vals = np.array([orc.e2m1_value(int(c)) for c in codes])
    grid = np.array(E2M1_MAGS + [-m for m in E2M1_MAGS])
    clipped = np.clip(r.astype(np.float64), -6, 6)
    best = np.min(np.abs(clipped[:, None] - grid[None, :]), axis=1)
    assert np.all(np.abs(clipped - vals) == best)           # nearest after saturation
    assert np.all(np.diff(vals[:40001]) >= 0)              # monotone in r
    assert np.all((codes >> 3) == (np.signbit(r)).astype(int))   # sign bit kept
    for c in range(8):                                       # exact round trip on the grid
        assert orc.e2m1_encode(E2M1_MAGS[c]) == c
        assert orc.e2m1_encode(-E2M1_MAGS[c]) == (8 | c)


# ---- FP4 quantiser ----------------------------------------------------------------------------
def test_fp4_worked_examples(orc):
    for ln in golden_lines("fp4_worked_examples.txt"):
        name, xs, sc, cs = [t.strip() for t in ln.split("|")]
        x = torch.tensor([float(v) for v in xs.split()], dtype=torch.bfloat16).view(1, 16)
        codes, scales = orc.quantize_fp4(x)
        assert scales[0, 0] == int(sc, 16), name
        nib = [int(c, 16) for c in cs.split()]
        packed = [nib[2 * j] | (nib[2 * j + 1] << 4) for j in range(8)]
        assert list(codes[0]) == packed, name


def test_fp4_layout_and_round_trip(orc):
    """Entries built from grid values x scale, with amax = 6 * scale, decode exactly."""
    rng = np.random.default_rng(3)
    rows = []
    for _ in range(64):
        grp = []
        for g in range(32):
            s = 2.0 ** int(rng.integers(-6, 4))
            v = rng.choice(E2M1_MAGS + [-m for m in E2M1_MAGS], 16) * s
            v[int(rng.integers(16))] = 6 * s * rng.choice([-1, 1])
            grp.append(v)
        rows.append(np.concatenate(grp))
    x = torch.tensor(np.array(rows), dtype=torch.float32).to(torch.bfloat16)
    codes, scales = orc.quantize_fp4(x)
    assert codes.shape == (64, 256) and scales.shape == (64, 32)
    assert codes.nbytes + scales.nbytes == 64 * 288
    back = orc.dequant_fp4(codes, scales)
    assert np.array_equal(back, x.double().numpy())


def test_fp4_scale_rule_and_error_bound(orc):
    """scale = E4M3_RNE(amax/6) (checked with torch's cast); |x - v| <= half the local
    E2M1 gap times the scale, unless the input saturates."""
    x = torch.randn(256, 512, generator=torch.Generator().manual_seed(11)) * \
        torch.exp2(torch.randint(-3, 4, (256, 1), generator=torch.Generator().manual_seed(12)))
    x = x.to(torch.bfloat16)
    codes, scales = orc.quantize_fp4(x)
    xf = x.float().view(256, 32, 16)
    amax = xf.abs().amax(-1)
    ref_scale = (amax / 6.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(scales, ref_scale)
    sd = torch.from_numpy(scales).view(torch.float8_e4m3fn).double()
    v = torch.from_numpy(orc.dequant_fp4(codes, scales)).view(256, 32, 16)
    r = (xf.double() / sd[..., None]).abs()
    mags = torch.tensor(E2M1_MAGS, dtype=torch.float64)
    gaps = torch.tensor([0.5, 0.5, 0.5, 0.5, 1.0, 1.0, 2.0, 2.0], dtype=torch.float64)
    idx = torch.clamp(torch.searchsorted(mags, r.contiguous(), right=True) - 1, 0, 7)
    half_gap = gaps[idx] / 2
    err = (xf.double() - v).abs()
    ok = (err <= half_gap * sd[..., None] + 1e-12) | (r > 6)
    assert bool(ok.all())


def test_fp4_zero_and_negative_zero(orc):
    x = torch.zeros(1, 512, dtype=torch.bfloat16)
    codes, scales = orc.quantize_fp4(x)
    assert not codes.any() and not scales.any()
    x = torch.ones(1, 512, dtype=torch.bfloat16)
    x[0, 0] = -0.0
    codes, _ = orc.quantize_fp4(x)
    assert codes[0, 0] & 0xF == 0x8          # -0 keeps its sign


# ---- FP8 rows ---------------------------------------------------------------------------------
def test_fp8_rows_match_torch(orc):
    x = (torch.randn(300, 128, generator=torch.Generator().manual_seed(5)) * 3).to(torch.bfloat16)
    codes, sigma = orc.quantize_fp8(x)
    xf = x.float()
    ref_sigma = xf.abs().amax(-1) / 448.0
    assert np.array_equal(sigma, ref_sigma.numpy())
    r = xf / ref_sigma[:, None]
    ref = torch.clamp(r, -448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)
    # dequantised error bound: half an E4M3 ulp of the scaled value, times sigma
    back = orc.dequant_fp8(codes, sigma)
    rel = np.abs(back - xf.double().numpy()) / np.maximum(np.abs(xf.double().numpy()), 1e-30)
    small = np.abs(r.numpy()) >= 2 ** -6
    assert np.all(rel[small] <= 2 ** -4 + 1e-9)


def test_fp8_zero_row(orc):
    codes, sigma = orc.quantize_fp8(torch.zeros(2, 512, dtype=torch.bfloat16))
    assert not codes.any() and not sigma.any()
