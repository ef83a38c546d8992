"""Pins for the oracle's number codecs against what the format definitions fix and
against independent library conversions (numpy binary16, torch bf16 / E4M3)."""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e2m1_e4m3_fp16_points.txt")


def _golden():
    rows = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        fmt, x, code = line.split()
        rows.append((fmt, float(x), int(code, 16)))
    return rows


@pytest.mark.parametrize("fmt,x,code", _golden())
def test_golden_points(fmt, x, code):
    enc = {"e2m1": oracle.f32_to_e2m1, "e4m3": oracle.f32_to_e4m3, "fp16": oracle.f32_to_f16}[fmt]
    assert int(enc(np.array([x], np.float32))[0]) == code


def _grid(p, emin, emax_val):
    """All non-negative finite values of a binary format (brute force)."""
    vals = {Fraction(0)}
    sub_q = Fraction(2) ** (emin - p + 1)
    for m in range(1, 2 ** (p - 1)):
        vals.add(m * sub_q)
    E = emin
    while True:
        q = Fraction(2) ** (E - p + 1)
        for m in range(2 ** (p - 1), 2 ** p):
            v = m * q
            if v > emax_val:
                return sorted(vals)
            vals.add(v)
        E += 1


def _brute_rne(x: Fraction, grid):
    """Nearest grid value to |x|; on a tie the one whose significand is even
    (index parity in the grid: consecutive grid values alternate last bit)."""
    a = abs(x)
    best = None
    for i, g in enumerate(grid):
        d = abs(a - g)
        if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
            best = (d, i, g)
    return best[2]


def test_e2m1_bruteforce_dense():
    grid = _grid(2, 0, Fraction(6))
    assert [float(g) for g in grid] == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    xs = np.concatenate([np.linspace(-7, 7, 2801, dtype=np.float32),
                         np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], np.float32)])
    codes = oracle.f32_to_e2m1(xs)
    dec = oracle.e2m1_to_f32(codes)
    for x, c, d in zip(xs, codes, dec):
        want = _brute_rne(Fraction(float(x)), grid)
        if want > 6:
            want = Fraction(6)
        assert Fraction(float(abs(d))) == want, (x, c, d)
        assert (c >> 3) == (1 if np.signbit(x) else 0)


def test_e2m1_decode_table():
    codes = np.arange(16, dtype=np.uint8)
    dec = oracle.e2m1_to_f32(codes)
    assert list(dec[:8]) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    assert list(-dec[8:]) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]


def test_e4m3_against_torch_all_midpoints():
    codes = np.arange(256, dtype=np.uint8)
    dec = oracle.e4m3_to_f32(codes)
    tdec = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    both_nan = np.isnan(dec) & np.isnan(tdec)
    assert np.all(both_nan | (dec == tdec))
    pos = np.sort(dec[(~np.isnan(dec)) & (dec >= 0)])
    pos = np.unique(pos)
    mids = (pos[:-1].astype(np.float64) + pos[1:]) / 2
    xs = np.concatenate([pos, mids, mids * (1 + 1e-6), mids * (1 - 1e-6)]).astype(np.float32)
    xs = np.concatenate([xs, -xs])
    ours = oracle.f32_to_e4m3(xs)
    theirs = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, theirs)


def test_e4m3_saturates():
    xs = np.array([448.0, 449.0, 463.9, 464.0, 500.0, 1e30, np.inf, -1e30], np.float32)
    assert list(oracle.f32_to_e4m3(xs)) == [0x7E] * 7 + [0xFE]


def test_fp16_against_numpy():
    rng = np.random.default_rng(1)
    allh = np.arange(65536, dtype=np.uint16)
    f = allh.view(np.float16).astype(np.float32)
    ours = oracle.f16_to_f32(allh)
    fin = np.isfinite(f)
    assert np.array_equal(ours[fin], f[fin])
    assert np.all(np.isnan(ours[np.isnan(f)]))
    # every finite fp16 value, all midpoints and their float32 neighbours, and random values
    pos = np.unique(f[fin & (f >= 0)]).astype(np.float64)
    mids = (pos[:-1] + pos[1:]) / 2
    m32 = mids.astype(np.float32)
    xs = np.concatenate([pos.astype(np.float32), m32, np.nextafter(m32, np.float32(np.inf)),
                         np.nextafter(m32, np.float32(-np.inf)),
                         (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 12, 200000))).astype(np.float32),
                         np.array([65519.0, 65520.0, 70000.0], np.float32)])
    xs = np.concatenate([xs, -xs])
    assert np.array_equal(oracle.f32_to_f16(xs), xs.astype(np.float16).view(np.uint16))


def test_bf16_against_torch():
    rng = np.random.default_rng(2)
    allh = np.arange(65536, dtype=np.uint16)
    f = oracle.bf16_to_f32(allh)
    fin = np.isfinite(f)
    # decode/encode round trip on every finite bf16
    assert np.array_equal(oracle.f32_to_bf16(f[fin]), allh[fin])
    # ties, near-ties and random values
    base = rng.integers(0, 2**31 - 2**24, 100000, dtype=np.uint64).astype(np.uint32) & np.uint32(0xFFFF0000)
    ties = (base | np.uint32(0x8000)).view(np.float32)
    near = (base | np.uint32(0x7FFF)).view(np.float32)
    xs = np.concatenate([ties, near, rng.standard_normal(100000).astype(np.float32) * 37.0])
    xs = xs[np.isfinite(xs)]
    xs = np.concatenate([xs, -xs])
    theirs = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16(xs), theirs)


def test_f64_to_bf16_single_rounding():
    # 1 + 2^-8 + 2^-30 lies above the bf16 tie at 1 + 2^-8, so it rounds up; a
    # detour through binary32 would land exactly on the tie and round to 1.0.
    x = 1.0 + 2.0**-8 + 2.0**-30
    assert int(oracle.f64_to_bf16(np.array([x]))[0]) == 0x3F81
    assert int(oracle.f32_to_bf16(np.array([x], np.float32))[0]) == 0x3F80
    # brute force against the grid for random doubles in a few binades
    rng = np.random.default_rng(3)
    xs = rng.uniform(-4, 4, 2000)
    got = oracle.bf16_to_f32(oracle.f64_to_bf16(xs)).astype(np.float64)
    for x, g in zip(xs, got):
        a = abs(Fraction(float(x)))
        E = a.numerator.bit_length() - a.denominator.bit_length()
        if Fraction(2) ** E > a:
            E -= 1
        q = Fraction(2) ** (E - 7)
        lo = (a // q) * q
        hi = lo + q
        if a - lo < hi - a:
            want = lo
        elif a - lo > hi - a:
            want = hi
        else:
            want = lo if (lo / q) % 2 == 0 else hi
        assert Fraction(float(abs(g))) == want
