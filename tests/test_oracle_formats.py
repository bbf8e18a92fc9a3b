"""Pins for the oracle's format decoding and its fp64 -> bf16 rounding.

Every check compares against something other than the oracle itself: the published format
definitions (golden fixtures), torch's float8_e4m3fn / bf16 conversions (library routines), or
exact properties of the formats (monotonicity, sign symmetry, double-rounding cases).
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        code, val = line.split()
        rows.append((int(code, 16), float(val)))
    return rows


def _same(a, b):
    if math.isnan(b):
        return math.isnan(a)
    return a == b and math.copysign(1, a) == math.copysign(1, b)


def test_e2m1_all_codes_match_definition():
    rows = _read("e2m1_codes.txt")
    assert len(rows) == 16
    for code, val in rows:
        assert _same(oracle.e2m1(code), val), (code, oracle.e2m1(code), val)


def test_e4m3_named_points():
    for code, val in _read("e4m3_points.txt"):
        assert _same(oracle.e4m3(code), val), (hex(code), oracle.e4m3(code), val)


def test_e4m3_all_codes_match_torch_float8_e4m3fn():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    ours = oracle.e4m3_table()
    for c in range(256):
        assert _same(ours[c], ref[c]), (hex(c), ours[c], ref[c])


def test_e4m3_structure():
    t = oracle.e4m3_table()
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0), "strictly increasing on 0x00..0x7E"
    for c in range(0x7F):
        assert _same(t[c | 0x80], -t[c])
    assert math.isnan(t[0x7F]) and math.isnan(t[0xFF])
    # subnormals are exact multiples of 2^-9; normals have 4 significant bits
    for c in range(1, 8):
        assert t[c] == c * 2.0 ** -9
    for c in range(8, 0x7F):
        m, e = math.frexp(t[c])
        assert (m * 16).is_integer()


def test_e2m1_structure():
    t = oracle.e2m1_table()
    assert np.all(np.diff(t[:8]) > 0)
    for c in range(8):
        assert _same(t[c | 8], -t[c])
    # every value times 2 is an integer (multiples of 0.5)
    assert np.all((t * 2) == np.round(t * 2))


def test_bf16_value_matches_torch():
    bits = np.arange(65536, dtype=np.uint16)
    ours = oracle.bf16_value(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    finite = np.isfinite(ref)
    assert np.array_equal(ours[finite], ref[finite])
    assert np.array_equal(np.isnan(ours), np.isnan(ref))


def test_bf16_rne_matches_torch_on_fp32_values():
    """On values exact in fp32, rounding straight from fp64 equals torch's fp32->bf16 RNE."""
    rng = np.random.default_rng(11)
    raw = rng.integers(0, 2 ** 32, 20000, dtype=np.uint64).astype(np.uint32)
    f = raw.view(np.float32)
    f = f[np.isfinite(f)]
    # ties and near-ties: low 16 bits 0x8000 (exact tie), 0x7FFF, 0x8001
    hi = rng.integers(0, 2 ** 16, 3000, dtype=np.uint64).astype(np.uint32) << 16
    ties = np.concatenate([hi | 0x8000, hi | 0x7FFF, hi | 0x8001]).astype(np.uint32).view(np.float32)
    ties = ties[np.isfinite(ties)]
    vals = np.concatenate([f, ties, np.float32([1e-40, -1e-40, 3.0e38, -3.4e38, 0.0, -0.0])])
    ours = oracle.bf16_rne(vals.astype(np.float64))
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(vals[i]), hex(ours[i]), hex(ref[i])) for i in bad[:5]]


def test_bf16_rne_single_rounding_from_fp64():
    # just above the tie between 1 and 1+2^-7: direct rounding goes up; via fp32 it would tie to 1
    assert oracle.bf16_rne(1 + 2 ** -8 + 2 ** -30) == 0x3F81
    assert oracle.bf16_rne(1 + 2 ** -8) == 0x3F80          # exact tie -> even
    assert oracle.bf16_rne(1 + 3 * 2 ** -8) == 0x3F82      # exact tie -> even (up)
    assert oracle.bf16_rne(-(1 + 2 ** -8 + 2 ** -30)) == 0xBF81
    # overflow threshold: (2 - 2^-8) * 2^127 is the tie between max finite and 2^128 -> inf
    assert oracle.bf16_rne(255.5 * 2.0 ** 120) == 0x7F80
    assert oracle.bf16_rne(255.4 * 2.0 ** 120) == 0x7F7F
    # subnormal quantum 2^-133; half of it rounds to even (zero)
    assert oracle.bf16_rne(2.0 ** -133) == 0x0001
    assert oracle.bf16_rne(2.0 ** -134) == 0x0000
    assert oracle.bf16_rne(1.5 * 2.0 ** -133) == 0x0002
    assert oracle.bf16_rne(float("nan")) & 0x7FFF > 0x7F80


def test_ulp_distance():
    a = np.array([0x3F80, 0x0000, 0x8000, 0x0001, 0x8001], np.uint16)
    b = np.array([0x3F81, 0x8000, 0x0001, 0x8001, 0x8002], np.uint16)
    assert list(oracle.bf16_ulp_distance(a, b)) == [1, 0, 1, 2, 1]


def test_bf16_rounding_interval_and_tolerance_rule():
    lo, hi = oracle.bf16_rounding_interval(np.array([0x3F80, 0x4492, 0x0000], np.uint16))
    assert lo[0] == 1 - 2 ** -9 and hi[0] == 1 + 2 ** -8
    assert lo[1] == 1164.0 and hi[1] == 1172.0      # bf16 1168, spacing 8
    assert lo[2] == -(2.0 ** -134) and hi[2] == 2.0 ** -134
    # a correctly rounded output passes even where |y - y_ref| exceeds 2e-3 A (|y| close to A)
    assert oracle.within_tolerance(np.array([0x4492]), np.array([1164.0138]), np.array([1438.5]))[0]
    assert not oracle.within_tolerance(np.array([0x4494]), np.array([1164.0138]),
                                       np.array([1438.5]))[0]
