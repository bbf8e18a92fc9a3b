"""Pins of the oracle's input prologues (residual add + RMS norm, sigmoid gate) against facts
that do not come from the oracle: hand-derived values, closed forms of the mean square and of
eps, the one rounding of the residual sum, invariants, and a 50-digit decimal evaluation with
its own bf16 rounding."""
import decimal
from decimal import Decimal

import numpy as np
import pytest

import oracle


def bf(vals):
    return oracle.bf16_rne(np.asarray(vals, np.float64))


def val(bits):
    return oracle.bf16_value(bits)


# ---- an independent bf16 rounding of a Decimal: nearest of the bf16 values that bracket it,
# ties to the even significand (found through the float32 grid, not through oracle code)

def decimal_digits(prec):
    def wrap(fn):
        def run(*a, **kw):
            with decimal.localcontext() as ctx:
                ctx.prec = prec
                return fn(*a, **kw)
        run.__name__ = fn.__name__
        return run
    return wrap


def dec_to_bf16(d: Decimal) -> int:
    if d == 0:
        return 0x8000 if d.is_signed() else 0
    sign = 0x8000 if d < 0 else 0
    a = abs(d)
    f = np.float32(float(a))
    u = int(np.array([f], np.float32).view(np.uint32)[0])
    lo_bits = (u >> 16) & 0x7FFF
    cands = [lo_bits - 1, lo_bits, lo_bits + 1, lo_bits + 2]
    best = None
    for c in cands:
        if c < 0 or c >= 0x7F80:
            continue
        v = Decimal(float(np.array([c << 16], np.uint32).view(np.float32)[0]))
        dist = abs(v - a)
        key = (dist, c & 1)  # nearer first, then the even significand
        if best is None or key < best[0]:
            best = (key, c)
    return sign | best[1]


def test_independent_rounding_agrees_with_the_oracle_on_easy_cases():
    for v in (1.0, 1.5, -3.25, 1 + 2 ** -8, 1 + 3 * 2 ** -8, 6.4, -4.8, 1e-30, 3e38):
        assert dec_to_bf16(Decimal(v)) == int(bf([v])[0]), v


# ---- residual add + RMS norm

def test_hand_derived_values():
    # h = [3, 4, 0 x 62], K = 64, gamma = 1, eps = 0: mean(h^2) = 25/64, rms = 5/8, so
    # xn = [24/5, 32/5, 0...] = [4.8, 6.4, 0...].  4.8 = 1.0011001100..b x 4 rounds up to
    # 1.0011010b x 4 = 4.8125; 6.4 = 1.1001100110..b x 4 rounds up to 1.1001101b x 4 = 6.40625.
    x = bf([[3, 4] + [0] * 62])
    r = bf([[0] * 64])
    h, xn, near = oracle.add_rmsnorm(x, r, bf([1] * 64), 0.0)
    assert np.array_equal(h, x)
    assert list(val(xn[0, :2])) == [4.8125, 6.40625]
    assert not val(xn[0, 2:]).any()


@pytest.mark.parametrize("c", [1.75, -0.375, 2.0 ** -60, -96.0])
def test_constant_row_normalises_to_gamma(c):
    # x + r = c everywhere, eps = 0: rms = |c|, so xn = sign(c) * gamma exactly
    k = 48
    rng = np.random.default_rng(1)
    gamma = bf(rng.uniform(0.25, 2.0, k))
    x = bf([[c / 2] * k])
    r = bf([[c / 2] * k])
    h, xn, _ = oracle.add_rmsnorm(x, r, gamma, 0.0)
    assert np.array_equal(val(h[0]), np.full(k, c))
    assert np.array_equal(val(xn[0]), np.sign(c) * val(gamma))


def test_eps_inside_the_square_root():
    # constant c with eps = 3 c^2: rms = sqrt(4 c^2) = 2|c|, xn = gamma / 2
    c = 2.0 ** -10
    k = 32
    gamma = bf(np.linspace(0.5, 3.0, k))
    h, xn, _ = oracle.add_rmsnorm(bf([[c] * k]), bf([[0.0] * k]), gamma, 3 * c * c)
    assert np.array_equal(val(xn[0]), val(gamma) / 2)
    # the mean, not the sum: the same row twice as long gives the same xn
    h2, xn2, _ = oracle.add_rmsnorm(bf([[c] * 2 * k]), bf([[0.0] * 2 * k]),
                                    bf(np.tile(val(gamma), 2)), 3 * c * c)
    assert np.array_equal(xn2[0, :k], xn[0])


def test_residual_sum_is_rounded_once_to_even():
    k = 16
    x = bf([[1.0, 1 + 2 ** -7, 1.0, -1.0] + [0.0] * (k - 4)])
    r = np.array([[bf([2 ** -8])[0]] * 3 + [bf([-2 ** -8])[0]] + [0] * (k - 4)], np.uint16)
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: even significand 1.0; (1 + 2^-7) + 2^-8 is
    # halfway between 1 + 2^-7 and 1 + 2^-6: even 1 + 2^-6; -1 - 2^-8: -1.0
    r[0, 2] = bf([2 ** -8 + 2 ** -14])[0]  # exact in bf16, just above the tie: 1 + 2^-7
    h, _, _ = oracle.add_rmsnorm(x, r, bf([1.0] * k), 1e-6)
    assert list(val(h[0, :4])) == [1.0, 1 + 2 ** -6, 1 + 2 ** -7, -1.0]


def test_scale_sign_and_permutation_invariants():
    rng = np.random.default_rng(2)
    m, k = 3, 64
    x = bf(rng.normal(0, 1, (m, k)))
    r = bf(rng.normal(0, 1, (m, k)))
    gamma = bf(rng.uniform(0.5, 1.5, k))
    h, xn, _ = oracle.add_rmsnorm(x, r, gamma, 0.0)
    # scaling x and r by 2^j leaves xn unchanged (eps = 0)
    hs, xns, _ = oracle.add_rmsnorm(bf(val(x) * 2.0 ** 40), bf(val(r) * 2.0 ** 40), gamma, 0.0)
    assert np.array_equal(xns, xn)
    assert np.array_equal(val(hs), val(h) * 2.0 ** 40)
    # negating x and r negates h and xn
    hn, xnn, _ = oracle.add_rmsnorm(x ^ np.uint16(0x8000), r ^ np.uint16(0x8000), gamma, 0.0)
    assert np.array_equal(val(xnn), -val(xn))
    # permuting k (with gamma) permutes xn; rows are independent
    p = rng.permutation(k)
    _, xnp, _ = oracle.add_rmsnorm(x[:, p], r[:, p], gamma[p], 0.0)
    assert np.array_equal(xnp, xn[:, p])
    _, xn1, _ = oracle.add_rmsnorm(x[1:2], r[1:2], gamma, 0.0)
    assert np.array_equal(xn1[0], xn[1])


@decimal_digits(50)
def test_add_rmsnorm_decimal_brute_force():
    rng = np.random.default_rng(3)
    m, k = 2, 32
    x = bf(rng.normal(0, 1, (m, k)))
    r = bf(rng.normal(0, 0.5, (m, k)))
    gamma = bf(rng.uniform(0.5, 1.5, k))
    eps = float(np.float32(1e-5))
    h, xn, near = oracle.add_rmsnorm(x, r, gamma, eps)
    for i in range(m):
        hd = [Decimal(float(a)) + Decimal(float(b)) for a, b in zip(val(x[i]), val(r[i]))]
        hb = [dec_to_bf16(t) for t in hd]
        assert hb == [int(t) for t in h[i]]
        hv = [Decimal(float(val(np.uint16(t)))) for t in hb]
        ms = sum(t * t for t in hv) / k
        inv = 1 / (ms + Decimal(eps)).sqrt()
        for j in range(k):
            want = dec_to_bf16(hv[j] * Decimal(float(val(gamma[j]))) * inv)
            got = int(xn[i, j])
            if near[i, j]:
                assert abs(oracle.bf16_ordinal(got) - oracle.bf16_ordinal(want)) <= 1
            else:
                assert got == want, (i, j)


# ---- sigmoid gate

def test_sigmoid_gate_closed_forms():
    rng = np.random.default_rng(4)
    a = bf(rng.normal(0, 3, (2, 32)))
    zero = np.zeros_like(a)
    xo, _ = oracle.sigmoid_gate(a, zero)             # sigmoid(0) = 1/2: exact halving
    assert np.array_equal(val(xo), val(a) / 2)
    xo, _ = oracle.sigmoid_gate(a, np.full_like(a, bf([100.0])[0]))   # saturates to a
    assert np.array_equal(xo, a)
    xo, _ = oracle.sigmoid_gate(a, np.full_like(a, bf([-100.0])[0]))  # a * e^-100 -> +-0
    assert not val(xo).any()
    assert np.array_equal(xo & 0x8000, a & 0x8000)


def test_sigmoid_symmetry():
    # sigmoid(t) + sigmoid(-t) = 1, so the two gated values add up to a within one ulp of a
    rng = np.random.default_rng(5)
    a = bf(rng.normal(0, 1, (4, 64)))
    t = bf(rng.normal(0, 2, (4, 64)))
    xp, _ = oracle.sigmoid_gate(a, t)
    xm, _ = oracle.sigmoid_gate(a, t ^ np.uint16(0x8000))
    av = val(a)
    ulp = np.abs(val(bf(av * (1 + 2 ** -7))) - av)
    assert (np.abs(val(xp) + val(xm) - av) <= ulp).all()


@decimal_digits(50)
def test_sigmoid_gate_decimal_brute_force():
    rng = np.random.default_rng(6)
    a = bf(rng.normal(0, 1, (2, 32)))
    t = bf(rng.normal(0, 3, (2, 32)))
    xo, near = oracle.sigmoid_gate(a, t)
    for i in range(2):
        for j in range(32):
            td = Decimal(float(val(t[i, j])))
            want = dec_to_bf16(Decimal(float(val(a[i, j]))) / (1 + (-td).exp()))
            got = int(xo[i, j])
            if near[i, j]:
                assert abs(oracle.bf16_ordinal(got) - oracle.bf16_ordinal(want)) <= 1
            else:
                assert got == want, (i, j)


def test_rounding_slack_is_the_neighbour_gap_where_near():
    xq = bf([[1.0, 1.0, -3.0, 0.0]])
    near = np.array([[1, 0, 1, 0]], np.uint8)
    s = val(oracle.rounding_slack(xq, near))
    assert list(s[0]) == [2 ** -7, 0.0, 2 ** -6, 0.0]


# ---- gated RMS norm (per group of channels, fp32 input, SiLU gate)

def test_gated_rmsnorm_closed_forms():
    # a constant group normalises to +-1; gate 100 passes through silu(100) = 100 (to fp64);
    # gamma 1/4: x' = +-25 exactly, group by group
    g = 128
    x = np.array([[1.5] * g + [-0.25] * g + [3e-3] * g], np.float32)
    z = bf(np.full((1, 3 * g), 100.0))
    gamma = bf(np.full(g, 0.25))
    xo, _ = oracle.gated_rmsnorm(x, z, gamma, g, 0.0)
    assert list(np.unique(val(xo[0, :g]))) == [25.0]
    assert list(np.unique(val(xo[0, g:2 * g]))) == [-25.0]
    assert list(np.unique(val(xo[0, 2 * g:]))) == [25.0]
    # gate 0: silu(0) = 0 gives signed zeros
    xo, _ = oracle.gated_rmsnorm(x, np.zeros_like(z), gamma, g, 0.0)
    assert not val(xo).any()
    # eps inside the square root: constant c with eps = 3 c^2 halves the result
    c = 2.0 ** -6
    xo, _ = oracle.gated_rmsnorm(np.full((1, g), c, np.float32), bf(np.full((1, g), 100.0)),
                                 gamma, g, 3 * c * c)
    assert list(np.unique(val(xo))) == [12.5]


def test_gated_rmsnorm_groups_are_independent_and_scale_free():
    rng = np.random.default_rng(7)
    g, m = 128, 2
    x = rng.normal(0, 1, (m, 4 * g)).astype(np.float32)
    z = bf(rng.normal(0, 2, (m, 4 * g)))
    gamma = bf(rng.uniform(0.5, 1.5, g))
    xo, _ = oracle.gated_rmsnorm(x, z, gamma, g, 0.0)
    # changing group 2 leaves the other groups unchanged
    x2 = x.copy()
    x2[:, 2 * g:3 * g] *= 7.0
    xo2, _ = oracle.gated_rmsnorm(x2, z, gamma, g, 0.0)
    keep = np.r_[0:2 * g, 3 * g:4 * g]
    assert np.array_equal(xo2[:, keep], xo[:, keep])
    # scaling a group by a power of two leaves its x' unchanged (eps = 0)
    x3 = x.copy()
    x3[:, g:2 * g] *= np.float32(2.0 ** 20)
    xo3, _ = oracle.gated_rmsnorm(x3, z, gamma, g, 0.0)
    assert np.array_equal(xo3, xo)
    # one group of a wider row equals the same values as a row of their own
    xo4, _ = oracle.gated_rmsnorm(x[:, g:2 * g], z[:, g:2 * g], gamma, g, 0.0)
    assert np.array_equal(xo4, xo[:, g:2 * g])


@decimal_digits(50)
def test_gated_rmsnorm_decimal_brute_force():
    rng = np.random.default_rng(8)
    g, m = 32, 2
    x = rng.normal(0, 1, (m, 2 * g)).astype(np.float32)
    z = bf(rng.normal(0, 2, (m, 2 * g)))
    gamma = bf(rng.uniform(0.5, 1.5, g))
    eps = float(np.float32(1e-5))
    xo, near = oracle.gated_rmsnorm(x, z, gamma, g, eps)
    for i in range(m):
        for q in range(2):
            xs = [Decimal(float(v)) for v in x[i, q * g:(q + 1) * g]]
            inv = 1 / (sum(v * v for v in xs) / g + Decimal(eps)).sqrt()
            for j in range(g):
                t = Decimal(float(val(z[i, q * g + j])))
                silu = t / (1 + (-t).exp())
                want = dec_to_bf16(xs[j] * Decimal(float(val(gamma[j]))) * silu * inv)
                got = int(xo[i, q * g + j])
                if near[i, q * g + j]:
                    assert abs(oracle.bf16_ordinal(got) - oracle.bf16_ordinal(want)) <= 1
                else:
                    assert got == want, (i, q, j)
