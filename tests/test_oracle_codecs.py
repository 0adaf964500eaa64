"""Pins of the oracle's number formats against their definitions.

e2m1 and e4m3 values come from the format specifications (fixtures under
tests/golden/, with citations) and from PyTorch's float8_e4m3fn dtype; the
encoders are checked against brute-force nearest-even search on the decoded
grids.  These formats are the pages' NVFP4 weights ("Expert Weight
Quantization") and fp8 KV cache ("Key points").
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _table(name):
    rows = []
    for line in open(os.path.join(GOLD, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            c, v = line.split()
            rows.append((int(c), float(v)))
    return rows


def test_e2m1_decode_matches_spec_table():
    L = oracle.lib()
    for code, val in _table("e2m1_values.txt"):
        got = L.msk_or_e2m1_decode(code)
        assert got == val and math.copysign(1, got) == math.copysign(1, val)


def test_e4m3_decode_landmarks():
    L = oracle.lib()
    for code, val in _table("e4m3_points.txt"):
        got = L.msk_or_e4m3_decode(code)
        if math.isnan(val):
            assert math.isnan(got)
        else:
            assert got == val


def test_e4m3_decode_all_codes_vs_torch():
    L = oracle.lib()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().double().numpy()
    for c in range(256):
        got = L.msk_or_e4m3_decode(c)
        if math.isnan(ref[c]):
            assert math.isnan(got)
        else:
            assert got == ref[c], c


def _finite_grid():
    L = oracle.lib()
    return np.array([L.msk_or_e4m3_decode(c) for c in range(127)])  # codes 0..126, >= 0


def _nearest_even(a, grid):
    """Brute force: nearest grid value, ties to the even code (mantissa lsb 0)."""
    d = np.abs(grid - a)
    best = np.flatnonzero(d == d.min())
    if len(best) > 1:
        best = [b for b in best if b % 2 == 0]
    return int(best[0])


def test_e4m3_encode_round_trip_and_saturation():
    L = oracle.lib()
    for c in range(1, 127):
        v = L.msk_or_e4m3_decode(c)
        assert L.msk_or_e4m3_encode(v) == c
        assert L.msk_or_e4m3_encode(-v) == 128 | c
    for x in (448.0, 449.0, 463.9, 464.0, 500.0, 1e9):
        assert L.msk_or_e4m3_encode(x) == 0x7E
        assert L.msk_or_e4m3_encode(-x) == 0xFE
    assert L.msk_or_e4m3_encode(0.0) == 0
    # OFP8 E4M3 has a signed zero (S.0000.000) and one NaN pattern per sign
    # (S.1111.111): -0 and negative values that round to zero keep the sign
    # bit, NaN stays NaN, infinities saturate
    assert L.msk_or_e4m3_encode(-0.0) == 0x80
    assert L.msk_or_e4m3_encode(-2.0 ** -11) == 0x80
    assert L.msk_or_e4m3_encode(float("nan")) & 0x7F == 0x7F
    assert L.msk_or_e4m3_encode(float("inf")) == 0x7E
    assert L.msk_or_e4m3_encode(float("-inf")) == 0xFE


def test_e4m3_encode_ties_and_random_vs_brute_force():
    L = oracle.lib()
    grid = _finite_grid()
    # every midpoint between neighbours: a tie, resolved to the even code
    for c in range(0, 126):
        mid = 0.5 * (grid[c] + grid[c + 1])
        want = c if c % 2 == 0 else c + 1
        assert L.msk_or_e4m3_encode(mid) == want, (c, mid)
    rng = np.random.default_rng(1)
    xs = np.concatenate([rng.standard_normal(3000) * s for s in (1e-3, 0.1, 1.0, 30.0, 150.0)])
    for x in xs:
        a = abs(x)
        want = _nearest_even(min(a, 448.0), grid)
        got = L.msk_or_e4m3_encode(float(x))
        assert got == (want | (128 if x < 0 else 0)), x  # sign kept, also on -0


def test_e4m3_encode_matches_torch_in_range():
    L = oracle.lib()
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(20000) * 8).astype(np.float32)
    x = x[np.abs(x) < 440]
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([L.msk_or_e4m3_encode(float(v)) for v in x])
    assert np.array_equal(got, ref)  # signed zeros included


def test_bf16_encode_matches_torch():
    L = oracle.lib()
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(20000), rng.standard_normal(2000) * 1e3]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([L.msk_or_bf16_encode(float(v)) for v in x], np.uint16)
    assert np.array_equal(got, ref)
    # ties: halfway between two bf16 values goes to the even one
    for b in (0x3F80, 0x3F81, 0x4000, 0xBF85):
        lo = L.msk_or_bf16_decode(b)
        hi = L.msk_or_bf16_decode(b + 1)
        want = b if b % 2 == 0 else b + 1
        assert L.msk_or_bf16_encode(0.5 * (lo + hi)) == want
