"""Pins for the oracle GEMV and the fused dual.

Independent anchors: closed-form sums on hand-built matrices, exact single-term cases, a library
cross-check (dequantise through the published E2M1 table and torch's float8_e4m3fn, then
numpy float64 matmul), and exact invariants (sign flip, power-of-two scaling, permutations,
row invariance).  A dropped term, wrong sign, wrong nibble order, wrong scale index or a
transposed operand fails at least one of these.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _e2m1_golden():
    t = np.zeros(16)
    for line in open(os.path.join(GOLDEN, "e2m1_codes.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            c, v = line.split()
            t[int(c, 16)] = float(v)
    return t


E2M1 = _e2m1_golden()
E4M3 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()


def pack(nibs):
    """[n][k] nibble codes -> [n][k/2] bytes, low nibble = even k."""
    nibs = np.asarray(nibs, np.uint8)
    return (nibs[:, 0::2] | (nibs[:, 1::2] << 4)).astype(np.uint8)


def bf16_bits(vals):
    return torch.tensor(np.asarray(vals, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def library_reference(nibs, scales, g, x_bits):
    w = E2M1[np.asarray(nibs)] * np.repeat(E4M3[np.asarray(scales)], 16, axis=1) * float(g)
    x = oracle.bf16_value(x_bits)
    return np.matmul(x, w.T)


def test_closed_form_ones():
    n, k = 5, 64
    nibs = np.full((n, k), 0x2)
    sc = np.full((n, k // 16), 0x38)
    xv = np.arange(k, dtype=np.float32) % 7 - 3  # small integers, exact in bf16
    y, a = oracle.gemv(pack(nibs), sc, 1.0, bf16_bits(xv)[None, :])
    assert np.all(y == xv.sum())
    assert np.all(a == np.abs(xv).sum())


def test_one_hot_terms_are_exact():
    rng = np.random.default_rng(3)
    n, k = 40, 96
    nibs = np.zeros((n, k), np.uint8)
    sc = rng.integers(0, 0x7F, (n, k // 16)).astype(np.uint8)
    ks = rng.integers(0, k, n)
    codes = rng.integers(0, 16, n)
    nibs[np.arange(n), ks] = codes
    xb = bf16_bits(rng.standard_normal((3, k)).astype(np.float32))
    g = 0.0375
    y, _ = oracle.gemv(pack(nibs), sc, g, xb)
    xv = oracle.bf16_value(xb)
    for j in range(n):
        expect = E2M1[codes[j]] * E4M3[sc[j, ks[j] // 16]] * np.float64(np.float32(g)) * xv[:, ks[j]]
        assert np.array_equal(y[:, j], expect + 0.0)


def test_every_scale_code_once():
    """N=1, one group per finite non-negative scale code, nibbles 1.0, x = 1: y = 16 * sum(scales)."""
    codes = np.arange(0x7F, dtype=np.uint8)
    k = 16 * codes.size
    nibs = np.full((1, k), 0x2)
    y, a = oracle.gemv(pack(nibs), codes[None, :], 1.0, bf16_bits(np.ones(k))[None, :])
    assert y[0, 0] == 16.0 * E4M3[:0x7F].sum()
    assert a[0, 0] == y[0, 0]


def test_every_nibble_code_times_every_scale():
    """Row n = scale code n (0..126); x row r = one-hot at k = r: y[r][n] = e2m1(code at k=r) * e4m3(n)."""
    n, k = 127, 32
    nibs = np.tile(np.arange(16, dtype=np.uint8), (n, 2))
    sc = np.repeat(np.arange(n, dtype=np.uint8)[:, None], 2, axis=1)
    x = np.zeros((16, k), np.float32)
    x[np.arange(16), np.arange(16)] = 1.0
    y, _ = oracle.gemv(pack(nibs), sc, 1.0, bf16_bits(x))
    assert np.array_equal(y, (E2M1[:, None] * E4M3[None, :n]) + 0.0)


def test_plus_minus_pairs_cancel():
    rng = np.random.default_rng(5)
    n, k = 9, 128
    c = rng.integers(0, 8, (n, k // 2)).astype(np.uint8)
    nibs = np.empty((n, k), np.uint8)
    nibs[:, 0::2] = c
    nibs[:, 1::2] = c | 8
    sc = rng.integers(0, 0x7F, (n, k // 16)).astype(np.uint8)
    xv = np.repeat(rng.standard_normal((2, k // 2)).astype(np.float32), 2, axis=1)
    y, a = oracle.gemv(pack(nibs), sc, 0.5, bf16_bits(xv))
    assert np.all(y == 0.0)
    assert np.all(a >= 0.0)


@pytest.mark.parametrize("n", list(range(1, 18)))
@pytest.mark.parametrize("k", [32, 48, 96])
def test_brute_force_against_library_matmul(n, k):
    rng = np.random.default_rng(n * 1000 + k)
    nibs = rng.integers(0, 16, (n, k)).astype(np.uint8)
    sc = rng.integers(0, 0x7F, (n, k // 16)).astype(np.uint8)
    m = int(rng.integers(1, 9))
    xb = bf16_bits(rng.standard_normal((m, k)).astype(np.float32) * 3)
    g = float(np.float32(rng.uniform(1e-3, 2.0)))
    y, a = oracle.gemv(pack(nibs), sc, g, xb)
    ref = library_reference(nibs, sc, g, xb)
    assert y.shape == (m, n)
    assert np.all(np.abs(y - ref) <= 1e-13 * a + 1e-300)


def test_synthetic_matrix_against_library_matmul():
    wl = synth.make("tiny")
    p = wl.projections[0]
    nib = np.empty((p.n, p.k), np.uint8)
    nib[:, 0::2] = p.w.packed & 15
    nib[:, 1::2] = p.w.packed >> 4
    y, a = oracle.gemv(p.w.packed, p.w.scales, p.w.g, p.x)
    ref = library_reference(nib, p.w.scales, p.w.g, p.x)
    assert np.all(np.abs(y - ref) <= 1e-12 * a)


def _rand_case(seed, n=33, k=160, m=4):
    rng = np.random.default_rng(seed)
    nibs = rng.integers(0, 16, (n, k)).astype(np.uint8)
    sc = rng.integers(0, 0x7F, (n, k // 16)).astype(np.uint8)
    xb = bf16_bits(rng.standard_normal((m, k)).astype(np.float32))
    return nibs, sc, xb


def test_sign_flip_negates_exactly():
    nibs, sc, xb = _rand_case(7)
    y1, a1 = oracle.gemv(pack(nibs), sc, 0.25, xb)
    y2, a2 = oracle.gemv(pack(nibs ^ 8), sc, 0.25, xb)
    assert np.array_equal(y2, -y1)
    assert np.array_equal(a1, a2)


def test_power_of_two_global_scale_is_exact():
    nibs, sc, xb = _rand_case(8)
    y1, _ = oracle.gemv(pack(nibs), sc, 0.3, xb)
    y2, _ = oracle.gemv(pack(nibs), sc, 0.6, xb)
    assert np.array_equal(y2, 2 * y1)


def test_permutations():
    nibs, sc, xb = _rand_case(9)
    perm = np.random.default_rng(1).permutation(nibs.shape[0])
    y1, _ = oracle.gemv(pack(nibs), sc, 1.0, xb)
    y2, _ = oracle.gemv(pack(nibs[perm]), sc[perm], 1.0, xb)
    assert np.array_equal(y2, y1[:, perm])
    y3, _ = oracle.gemv(pack(nibs), sc, 1.0, xb[::-1].copy())
    assert np.array_equal(y3, y1[::-1])


def test_nibble_order_low_is_even_k():
    # a single nonzero nibble in the LOW half of byte 0 must pair with x[0], not x[1]
    nibs = np.zeros((1, 32), np.uint8)
    nibs[0, 0] = 0x2
    x = np.zeros(32, np.float32)
    x[0], x[1] = 3.0, 5.0
    y, _ = oracle.gemv(pack(nibs), np.full((1, 2), 0x38, np.uint8), 1.0, bf16_bits(x)[None])
    assert y[0, 0] == 3.0
    assert pack(nibs)[0, 0] == 0x02


def test_scale_index_follows_group():
    # nibbles in group 1 must use scales[:,1]
    nibs = np.zeros((1, 32), np.uint8)
    nibs[0, 16] = 0x2
    sc = np.array([[0x38, 0x40]], np.uint8)  # 1.0, 2.0
    y, _ = oracle.gemv(pack(nibs), sc, 1.0, bf16_bits(np.ones(32))[None])
    assert y[0, 0] == 2.0


def test_row_invariance():
    nibs, sc, xb = _rand_case(10, m=8)
    full, _ = oracle.gemv(pack(nibs), sc, 0.7, xb)
    for r in range(8):
        one, _ = oracle.gemv(pack(nibs), sc, 0.7, xb[r:r + 1])
        assert np.array_equal(one[0], full[r])


def test_rows_subset_and_threads():
    nibs, sc, xb = _rand_case(12, n=50)
    full, a = oracle.gemv(pack(nibs), sc, 1.0, xb, threads=1)
    rows = [49, 0, 17, 17, 3]
    sub, asub = oracle.gemv(pack(nibs), sc, 1.0, xb, rows=rows, threads=4)
    assert np.array_equal(sub, full[:, rows])
    assert np.array_equal(asub, a[:, rows])


def test_absum_bounds():
    nibs, sc, xb = _rand_case(13)
    y, a = oracle.gemv(pack(nibs), sc, 1.0, xb)
    assert np.all(a >= np.abs(y))
    y2, a2 = oracle.gemv(pack(nibs & 7), sc, 1.0, bf16_bits(np.abs(oracle.bf16_value(xb))))
    assert np.allclose(y2, a2, rtol=1e-15, atol=0)


def test_empty_and_bad_shapes():
    y, a = oracle.gemv(np.zeros((0, 16), np.uint8), np.zeros((0, 2), np.uint8), 1.0,
                       np.zeros((2, 32), np.uint16))
    assert y.shape == (2, 0)
    y, a = oracle.gemv(np.zeros((3, 0), np.uint8), np.zeros((3, 0), np.uint8), 1.0,
                       np.zeros((1, 0), np.uint16))
    assert np.all(y == 0)
    with pytest.raises(ValueError):
        oracle.gemv(np.zeros((3, 16), np.uint8), np.zeros((3, 1), np.uint8), 1.0,
                    np.zeros((1, 32), np.uint16))


# ------------------------------------------------------------------------------------------
# fused dual

def test_dual_zero_gate_gives_zero():
    nibs, sc, xb = _rand_case(20)
    z = pack(np.zeros_like(nibs))
    o, yg, yu, ag, au = oracle.gemv_dual(z, sc, 1.0, pack(nibs), sc, 1.0, xb)
    assert np.all(yg == 0) and np.all(o == 0)


def test_dual_closed_form_silu():
    """Gate row n = t_n via one-hot, up row = 1: o = t / (1 + e^-t)."""
    ts = np.array([-6.0, -3.0, -1.0, -0.5, 0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    n, k = ts.size, 32
    code = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}
    gn = np.zeros((n, k), np.uint8)
    for j, t in enumerate(ts):
        gn[j, 0] = code[abs(t)] | (8 if t < 0 else 0)
    un = np.zeros((n, k), np.uint8)
    un[:, 0] = 0x2
    sc = np.full((n, 2), 0x38, np.uint8)
    x = np.zeros(k, np.float32)
    x[0] = 1.0
    o, yg, yu, _, _ = oracle.gemv_dual(pack(gn), sc, 1.0, pack(un), sc, 1.0, bf16_bits(x)[None])
    expect = np.array([t / (1 + math.exp(-t)) for t in ts])
    assert np.allclose(o[0], expect, rtol=1e-15, atol=0)
    assert np.array_equal(yg[0], ts)
    assert np.all(yu == 1.0)


def test_dual_is_silu_of_gate_times_up():
    ng, sg, xb = _rand_case(21)
    nu, su, _ = _rand_case(22)
    o, yg, yu, ag, au = oracle.gemv_dual(pack(ng), sg, 0.01, pack(nu), su, 0.02, xb)
    yg1, ag1 = oracle.gemv(pack(ng), sg, 0.01, xb)
    yu1, au1 = oracle.gemv(pack(nu), su, 0.02, xb)
    assert np.array_equal(yg, yg1) and np.array_equal(yu, yu1)
    assert np.array_equal(ag, ag1) and np.array_equal(au, au1)
    assert np.allclose(o, yg1 / (1 + np.exp(-yg1)) * yu1, rtol=1e-15, atol=0)
    # gate and up are not interchangeable
    o2, *_ = oracle.gemv_dual(pack(nu), su, 0.02, pack(ng), sg, 0.01, xb)
    assert not np.allclose(o, o2)
