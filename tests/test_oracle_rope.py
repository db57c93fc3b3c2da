"""Pins of the oracle's RoPE-inside-the-append step and its fp32 -> bf16 rounding.

The rounding is checked against torch's bf16 cast (round to nearest, ties to even)
on ties, subnormals and random values; the rotation against exact rational
arithmetic with one correct rounding per operation (the products, the fma, the
bf16 rounding), and against the plain rotations it must reduce to: the identity
and a quarter turn.  Channels outside the range and rows outside the table are
left as they are.
"""
from fractions import Fraction

import numpy as np
import torch

import synth
from exact_fp32 import f, fma32, mul32


def round_bf16(x: Fraction) -> Fraction:
    """Nearest bf16 value (8 significant bits, ties to even), normal and subnormal."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    ulp_e = max(e - 7, -133)
    scaled = a / Fraction(2) ** ulp_e
    n = scaled.numerator // scaled.denominator
    rem = scaled - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * n * Fraction(2) ** ulp_e


def bf16_value(bits: int) -> float:
    return float(torch.tensor([bits], dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float())


def test_f32_to_bf16_matches_torch(orc):
    rng = np.random.default_rng(7)
    vals = [0.0, -0.0, 1.0, -1.5, 3.4e38, -3.4e38, 1e-40, -1e-42, np.inf, -np.inf]
    # exact ties: low 16 bits 0x8000 with an even and an odd kept lsb
    for hi in (0x3F80, 0x3F81, 0xBF80, 0xBF81, 0x0001, 0x7F7F):
        vals.append(np.uint32((hi << 16) | 0x8000).view(np.float32).item())
        vals.append(np.uint32((hi << 16) | 0x7FFF).view(np.float32).item())
    vals += list(rng.standard_normal(2000).astype(np.float32) * np.float32(2.0) ** rng.integers(-130, 120, 2000).astype(np.float32))
    x = torch.tensor(np.array(vals, np.float32))
    ref = x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.f32_to_bf16(float(v)) for v in x.numpy()], np.uint16)
    assert np.array_equal(got, ref)


def test_rope_exact_rational(orc):
    """Every rotated value equals round_bf16(fma(x0, c, -(x1 s))) and
    round_bf16(fma(x0, s, x1 c)) evaluated exactly, one rounding per operation."""
    W, pairs, start = 64, 9, 10
    rows = synth.rows_normal_bf16(71, "x", 0, 0, 6, W)
    rows[2, 11] = -rows[2, 11]
    cs = synth.rope_table(5000, pairs)
    pos = np.array([0, 1, 17, 999, 4321, 4999])
    out, n_out = orc.rope_rows(rows, pos, cs, start, pairs)
    assert n_out == 0
    xb = rows.float().numpy()
    for r in range(len(pos)):
        for i in range(pairs):
            j = start + 2 * i
            x0, x1 = f(xb[r, j]), f(xb[r, j + 1])
            c, s = f(cs[pos[r], i, 0]), f(cs[pos[r], i, 1])
            y0 = round_bf16(fma32(x0, c, -mul32(x1, s)))
            y1 = round_bf16(fma32(x0, s, mul32(x1, c)))
            assert Fraction(bf16_value(int(out[r, j]))) == y0, (r, i)
            assert Fraction(bf16_value(int(out[r, j + 1]))) == y1, (r, i)


def test_rope_identity_quarter_turn_and_passthrough(orc):
    W, pairs, start = 512, 32, 448
    rows = synth.rows_normal_bf16(72, "x", 0, 0, 4, W)
    xb = rows.view(torch.int16).numpy().view(np.uint16)
    xf = rows.float().numpy()
    ident = np.zeros((3, pairs, 2), np.float32)
    ident[..., 0] = 1.0
    out, n_out = orc.rope_rows(rows, [0, 1, 2, 2], ident, start, pairs)
    assert n_out == 0
    assert np.array_equal(np.array([[bf16_value(int(v)) for v in r] for r in out]), xf)
    quarter = np.zeros((3, pairs, 2), np.float32)
    quarter[..., 1] = 1.0                                      # angle pi/2: (x0, x1) -> (-x1, x0)
    out, _ = orc.rope_rows(rows, [0, 1, 2, 2], quarter, start, pairs)
    of = np.array([[bf16_value(int(v)) for v in r] for r in out])
    assert np.array_equal(of[:, start::2], -xf[:, start + 1::2])
    assert np.array_equal(of[:, start + 1::2], xf[:, start::2])
    # channels before the range are copied bit for bit; a row past the table stays as is
    cs = synth.rope_table(3, pairs)
    out, n_out = orc.rope_rows(rows, [0, 2, 3, -1], cs, start, pairs)
    assert n_out == 2
    assert np.array_equal(out[:, :start], xb[:, :start])
    assert np.array_equal(out[2:], xb[2:])
    assert not np.array_equal(out[1, start:], xb[1, start:])
