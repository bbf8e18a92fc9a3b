"""GPU parity: the CUDA library, called through the C ABI, against the fp64 oracle.

Tolerance (per element): |y_gpu - y_ref| <= 2e-3 * sum_k |w_k x_k| + 1e-6, and the bf16 output
within 1 ulp of bf16(y_ref) wherever the fp32 accumulation error cannot reach half an ulp.
Row invariance and determinism are bitwise.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import nvfp4_weight_only_03_b200 as nv
from gpu_util import (assert_ws_clean, bits, bf16_bits_of, check_dual, check_single, dev_weight,
                      dev_x, pack_nibbles, random_weight)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ws():
    return torch.zeros(nv.workspace_bytes(), dtype=torch.uint8, device="cuda")


def run(w, x_bits, ws, m=None):
    m = x_bits.shape[0] if m is None else m
    W, S, g = dev_weight(w)
    y = nv.gemv(W, S, g, dev_x(x_bits[:m]), ws=ws)
    torch.cuda.synchronize()
    return bits(y)


# ------------------------------------------------------------------------------------------
# the workloads


def test_tiny_all_rows(ws):
    wl = synth.make("tiny")
    p = wl.projections[0]
    for m in range(1, 9):
        y = run(p.w, p.x, ws, m)
        ref, a = oracle.gemv(p.w.packed, p.w.scales, p.w.g, p.x[:m])
        check_single(y, ref, a, f"tiny M={m}")
    assert_ws_clean(ws)


def test_inproj_full(ws):
    wl = synth.make("inproj")
    p = wl.projections[0]
    y = run(p.w, p.x, ws, 1)
    ref, a = oracle.gemv(p.w.packed, p.w.scales, p.w.g, p.x[:1])
    check_single(y, ref, a, "inproj")
    assert_ws_clean(ws)


def test_gateup_full(ws):
    wl = synth.make("gateup")
    p = wl.projections[0]
    Wg, Sg, gg = dev_weight(p.w)
    Wu, Su, gu = dev_weight(p.w_up)
    o = bits(nv.gemv_dual(Wg, Sg, gg, Wu, Su, gu, dev_x(p.x[:1]), ws=ws))
    o_ref, yg, yu, ag, au = oracle.gemv_dual(p.w.packed, p.w.scales, p.w.g, p.w_up.packed,
                                             p.w_up.scales, p.w_up.g, p.x[:1])
    check_dual(o, o_ref, yg, yu, ag, au, "gateup")
    assert_ws_clean(ws)


def test_down_full_and_row_invariance(ws):
    wl = synth.make("down")
    p = wl.projections[0]
    y8 = run(p.w, p.x, ws, 8)
    ref, a = oracle.gemv(p.w.packed, p.w.scales, p.w.g, p.x)
    check_single(y8, ref, a, "down M=8")
    for m in range(1, 8):
        ym = run(p.w, p.x, ws, m)
        assert np.array_equal(ym, y8[:m]), f"rows differ between M={m} and M=8"
    for r in range(8):
        y1 = run(p.w, p.x[r:r + 1], ws, 1)
        assert np.array_equal(y1[0], y8[r]), f"row {r} of M=8 differs from its M=1 call"
    assert_ws_clean(ws)


@pytest.mark.parametrize("layer", [0, 3])
def test_sweep_layer_sampled(ws, layer):
    """Full-size sweep shapes at the bench's launch configuration: every M in {1,2,4,8}
    bitwise row-invariant; sampled outputs against the oracle at M=8."""
    wl = synth.make("sweep")
    rng = np.random.default_rng(layer)
    for p in wl.projections[4 * layer:4 * layer + 4]:
        rows = np.unique(np.concatenate([rng.integers(0, p.n, 192), [0, p.n - 1]]))
        if p.dual:
            Wg, Sg, gg = dev_weight(p.w)
            Wu, Su, gu = dev_weight(p.w_up)
            outs = {m: bits(nv.gemv_dual(Wg, Sg, gg, Wu, Su, gu, dev_x(p.x[:m]), ws=ws))
                    for m in (1, 2, 4, 8)}
            o_ref, yg, yu, ag, au = oracle.gemv_dual(p.w.packed, p.w.scales, p.w.g,
                                                     p.w_up.packed, p.w_up.scales, p.w_up.g,
                                                     p.x, rows=rows)
            check_dual(outs[8][:, rows], o_ref, yg, yu, ag, au, p.name)
        else:
            outs = {m: run(p.w, p.x, ws, m) for m in (1, 2, 4, 8)}
            ref, a = oracle.gemv(p.w.packed, p.w.scales, p.w.g, p.x, rows=rows)
            check_single(outs[8][:, rows], ref, a, p.name)
        for m in (1, 2, 4):
            assert np.array_equal(outs[m], outs[8][:m]), f"{p.name}: M={m} rows differ"
    assert_ws_clean(ws)


# ------------------------------------------------------------------------------------------
# ragged shapes, strides, edge cases


@pytest.mark.parametrize("n,k", [(1, 32), (15, 96), (17, 160), (255, 224), (257, 544),
                                 (300, 4096 + 32), (1000, 1056), (4097, 2080), (37, 12800 + 96)])
def test_ragged_shapes(ws, n, k):
    rng = np.random.default_rng(n * 7 + k)
    w = random_weight(rng, n, k)
    x = bf16_bits_of(rng.standard_normal((8, k)).astype(np.float32))
    for m in (1, 3, 8):
        y = run(w, x, ws, m)
        ref, a = oracle.gemv(w.packed, w.scales, w.g, x[:m])
        check_single(y, ref, a, f"n={n} k={k} M={m}")
        if m == 8:
            y8 = y
    for r in (0, 5, 7):
        assert np.array_equal(run(w, x[r:r + 1], ws, 1)[0], y8[r])
    assert_ws_clean(ws)


def test_split_launch_large_n_large_k(ws):
    """N and K large enough that the host splits the rows into several launches (the staged
    activations of one CTA would not fit shared memory otherwise)."""
    rng = np.random.default_rng(41)
    n, k = 37120 + 300, 12928
    w = random_weight(rng, n, k)
    x = bf16_bits_of(rng.standard_normal((2, k)).astype(np.float32))
    y = run(w, x, ws, 2)
    rows = np.unique(np.concatenate([rng.integers(0, n, 64), [0, 37119, 37120, n - 1]]))
    ref, a = oracle.gemv(w.packed, w.scales, w.g, x, rows=rows)
    check_single(y[:, rows], ref, a, "split")
    assert np.array_equal(run(w, x[1:2], ws, 1)[0], y[1])
    assert_ws_clean(ws)


def test_many_row_groups_small_k(ws):
    """N large enough that each CTA owns several whole row groups (no cut segments)."""
    rng = np.random.default_rng(77)
    n, k = 148 * 256 * 3 + 40, 64
    w = random_weight(rng, n, k)
    x = bf16_bits_of(rng.standard_normal((4, k)).astype(np.float32))
    y = run(w, x, ws, 4)
    ref, a = oracle.gemv(w.packed, w.scales, w.g, x)
    check_single(y, ref, a, "wide")
    assert_ws_clean(ws)


def test_strided_x_and_y(ws):
    rng = np.random.default_rng(5)
    n, k, m = 777, 640, 5
    w = random_weight(rng, n, k)
    x = bf16_bits_of(rng.standard_normal((m, k)).astype(np.float32))
    W, S, g = dev_weight(w)
    xs = dev_x(x, ldx=k + 24)
    assert xs.stride(0) == k + 24
    ybuf = torch.full((m, n + 13), 7.0, dtype=torch.bfloat16, device="cuda")
    nv.gemv(W, S, g, xs, y=ybuf[:, :n], ws=ws)
    torch.cuda.synchronize()
    ref, a = oracle.gemv(w.packed, w.scales, w.g, x)
    check_single(bits(ybuf[:, :n]), ref, a, "strided")
    assert torch.all(ybuf[:, n:] == 7.0), "wrote past the row end"
    assert np.array_equal(bits(ybuf[:, :n]), run(w, x, ws, m))


def test_stacked_dual_layout(ws):
    """A [gate; up] buffer passed as w_up = w_gate + N*K/2 equals separate tensors."""
    rng = np.random.default_rng(9)
    n, k = 513, 384
    wg, wu = random_weight(rng, n, k), random_weight(rng, n, k)
    x = bf16_bits_of(rng.standard_normal((2, k)).astype(np.float32))
    Wst = torch.from_numpy(np.concatenate([wg.packed, wu.packed])).cuda()
    Sst = torch.from_numpy(np.concatenate([wg.scales, wu.scales])).cuda()
    o_sep = bits(nv.gemv_dual(*dev_weight(wg), *dev_weight(wu), dev_x(x), ws=ws))
    o_st = bits(nv.gemv_dual(Wst[:n], Sst[:n], wg.g, Wst[n:], Sst[n:], wu.g, dev_x(x), ws=ws))
    assert np.array_equal(o_sep, o_st)
    o_ref, yg, yu, ag, au = oracle.gemv_dual(wg.packed, wg.scales, wg.g, wu.packed, wu.scales,
                                             wu.g, x)
    check_dual(o_sep, o_ref, yg, yu, ag, au, "stacked")


def test_k_zero_writes_zeros_and_noops(ws):
    W = torch.zeros((10, 0), dtype=torch.uint8, device="cuda")
    S = torch.zeros((10, 0), dtype=torch.uint8, device="cuda")
    x = torch.zeros((3, 0), dtype=torch.bfloat16, device="cuda")
    y = torch.full((3, 10), 5.0, dtype=torch.bfloat16, device="cuda")
    nv.gemv(W, S, 1.0, x, y=y, ws=ws)
    o = torch.full((3, 10), 5.0, dtype=torch.bfloat16, device="cuda")
    nv.gemv_dual(W, S, 1.0, W, S, 1.0, x, y=o, ws=ws)
    torch.cuda.synchronize()
    assert torch.all(y == 0) and torch.all(o == 0)
    # N == 0 and M == 0: nothing written, OK returned
    L = nv.lib()
    assert L.nvfp4_gemv(W.data_ptr(), S.data_ptr(), 1.0, x.data_ptr(), 0, y.data_ptr(), 10, 0,
                        10, 0, ws.data_ptr(), ws.numel(), None) == 0


# ------------------------------------------------------------------------------------------
# exact cases: decode tables through the real kernel, invariants, determinism


def test_every_nibble_times_every_scale_is_exact(ws):
    """Row n carries scale code n (0..126) and nibbles 0..15; x row r is one-hot at k=r:
    y[r][n] = e2m1(r) * e4m3(n) exactly (single-term sums, exact in bf16)."""
    n, k = 127, 32
    nibs = np.tile(np.arange(16, dtype=np.uint8), (n, 2))
    sc = np.repeat(np.arange(n, dtype=np.uint8)[:, None], 2, axis=1)
    w = synth.Weight(n, k, pack_nibbles(nibs), sc, 1.0)
    t2, t4 = oracle.e2m1_table(), oracle.e4m3_table()
    for r0 in (0, 8):
        x = np.zeros((8, k), np.float32)
        x[np.arange(8), r0 + np.arange(8)] = 1.0
        y = oracle.bf16_value(run(w, bf16_bits_of(x), ws, 8))
        expect = t2[r0:r0 + 8, None] * t4[None, :n]
        assert np.array_equal(y, expect + 0.0), np.argwhere(y != expect)[:5]


def test_closed_form_sum(ws):
    n, k = 64, 1024
    nibs = np.full((n, k), 0x2, np.uint8)
    sc = np.full((n, k // 16), 0x38, np.uint8)
    w = synth.Weight(n, k, pack_nibbles(nibs), sc, 1.0)
    xv = (np.arange(k) % 5 - 2).astype(np.float32)
    y = oracle.bf16_value(run(w, bf16_bits_of(xv[None]), ws, 1))
    assert np.all(y == xv.sum())


def test_sign_flip_and_power_of_two_scale_are_bitwise(ws):
    rng = np.random.default_rng(31)
    n, k = 2048, 3072
    w = random_weight(rng, n, k)
    x = bf16_bits_of(rng.standard_normal((8, k)).astype(np.float32))
    y = run(w, x, ws, 8)
    wneg = synth.Weight(n, k, w.packed ^ 0x88, w.scales, w.g)
    yn = run(wneg, x, ws, 8)
    assert np.array_equal(oracle.bf16_value(yn), -oracle.bf16_value(y))
    nz = (y & 0x7FFF) != 0
    assert np.array_equal(yn[nz], y[nz] ^ 0x8000)
    w2 = synth.Weight(n, k, w.packed, w.scales, w.g * 2)
    assert np.array_equal(oracle.bf16_value(run(w2, x, ws, 8)), 2 * oracle.bf16_value(y))


def test_deterministic(ws):
    wl = synth.make("inproj")
    p = wl.projections[0]
    W, S, g = dev_weight(p.w)
    x = dev_x(p.x)
    outs = [bits(nv.gemv(W, S, g, x, ws=ws)) for _ in range(5)]
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])


def test_zero_scale_with_nonzero_nibbles(ws):
    rng = np.random.default_rng(3)
    n, k = 100, 256
    w = random_weight(rng, n, k)
    w.scales[:, 3] = 0
    w.scales[7, :] = 0
    x = bf16_bits_of(rng.standard_normal((2, k)).astype(np.float32))
    y = run(w, x, ws, 2)
    ref, a = oracle.gemv(w.packed, w.scales, w.g, x)
    check_single(y, ref, a, "zero scales")
    assert np.all(oracle.bf16_value(y[:, 7]) == 0)


# ------------------------------------------------------------------------------------------
# error statuses with a real device (host checks; nothing is launched)


def test_error_statuses_on_device(ws):
    W = torch.zeros((64, 32), dtype=torch.uint8, device="cuda")
    S = torch.zeros((64, 4), dtype=torch.uint8, device="cuda")
    x = torch.zeros((9, 64), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((9, 64), dtype=torch.bfloat16, device="cuda")
    L = nv.lib()
    args = lambda **o: (o.get("w", W.data_ptr()), o.get("s", S.data_ptr()), 1.0,
                        o.get("x", x.data_ptr()), o.get("ldx", 64), o.get("y", y.data_ptr()),
                        o.get("ldy", 64), o.get("m", 1), 64, 64, o.get("ws", ws.data_ptr()),
                        o.get("wsb", ws.numel()), None)
    assert L.nvfp4_gemv(*args()) == 0
    assert L.nvfp4_gemv(*args(m=129)) == -3
    assert L.nvfp4_gemv(*args(x=x.data_ptr() + 2)) == -4
    assert L.nvfp4_gemv(*args(w=W.data_ptr() + 1)) == -4
    assert L.nvfp4_gemv(*args(wsb=1024)) == -7
    assert L.nvfp4_gemv(*args(ws=None)) == -7
    with pytest.raises(nv.Nvfp4Error):
        nv.gemv(W, S, 1.0, x[:1], ws=ws[:100])
    torch.cuda.synchronize()
    assert nv.workspace_error(ws) == 0


# ------------------------------------------------------------------------------------------
# launch flags and the scale-copy paths


def test_prefetch_flag_matches_plain_launch(ws):
    """Programmatic dependent launch changes only when the weights stream, not the result."""
    wl = synth.make("tiny")
    rng = np.random.default_rng(17)
    for n, k in ((4000, 5120), (700, 1056)):
        w = random_weight(rng, n, k)
        x = bf16_bits_of(rng.standard_normal((8, k)).astype(np.float32))
        W, S, g = dev_weight(w)
        xd = dev_x(x)
        a = bits(nv.gemv(W, S, g, xd, ws=ws))
        # a chain of prefetching launches on one stream, back to back
        outs = [nv.gemv(W, S, g, xd, ws=ws, prefetch_weights=True) for _ in range(4)]
        torch.cuda.synchronize()
        for o in outs:
            assert np.array_equal(bits(o), a)
        wu = random_weight(rng, n, k)
        Wu, Su, gu = dev_weight(wu)
        d0 = bits(nv.gemv_dual(W, S, g, Wu, Su, gu, xd, ws=ws))
        d1 = bits(nv.gemv_dual(W, S, g, Wu, Su, gu, xd, ws=ws, prefetch_weights=True))
        assert np.array_equal(d0, d1)
    assert_ws_clean(ws)


@pytest.mark.parametrize("k,offset", [(5120, 0), (5120, 2), (5120, 8), (384, 0), (160, 0)])
def test_scale_copy_paths(ws, k, offset):
    """TMA scale boxes (K % 256 == 0, 16-byte aligned scales), 8-byte cp.async (K % 128 == 0,
    8-byte aligned) and the 2-byte copy (otherwise) give identical results."""
    rng = np.random.default_rng(k + offset)
    n = 1000
    w = random_weight(rng, n, k)
    x = bf16_bits_of(rng.standard_normal((3, k)).astype(np.float32))
    W = torch.from_numpy(w.packed).cuda()
    buf = torch.zeros(n * (k // 16) + 64, dtype=torch.uint8, device="cuda")
    S = buf[offset:offset + n * (k // 16)].view(n, k // 16)
    S.copy_(torch.from_numpy(w.scales).cuda())
    y = bits(nv.gemv(W, S, w.g, dev_x(x), ws=ws))
    ref, a = oracle.gemv(w.packed, w.scales, w.g, x)
    check_single(y, ref, a, f"k={k} offset={offset}")
    y0 = bits(nv.gemv(W, torch.from_numpy(w.scales).cuda(), w.g, dev_x(x), ws=ws))
    assert np.array_equal(y, y0)


def amax_trap_rows(m, k, k0=1000):
    """x rows whose largest magnitude sits in the low half of a bf16 pair while other words of
    the same lane have a larger high half: 1.0 at even k, 3.0 at odd k, and in the 8-element
    chunk holding k0 (even) 2.0 at odd k and 1000 at k0.  A per-row maximum that compared
    packed pairs as whole words would miss the 1000 and overflow f16."""
    v = np.where(np.arange(k) % 2 == 0, 1.0, 3.0)
    c0 = k0 - k0 % 8
    v[c0 + 1:c0 + 8:2] = 2.0
    v[k0] = 1000.0
    return oracle.bf16_rne(np.tile(v, (m, 1)))


@pytest.mark.parametrize("m", [1, 5, 8])
def test_row_maximum_in_a_low_half_word(m):
    n, k = 1000, 5120
    w = synth.nvfp4_weight(55, 0, n, k)
    x = amax_trap_rows(m, k)
    W, S, g = dev_weight(w)
    y = bits(nv.gemv(W, S, g, dev_x(x)))
    torch.cuda.synchronize()
    assert np.isfinite(oracle.bf16_value(y)).all()
    ref, a = oracle.gemv(w.packed, w.scales, w.g, x)
    check_single(y, ref, a, f"row maximum in a low half, M={m}")
    y1 = bits(nv.gemv(W, S, g, dev_x(x[:1])))
    torch.cuda.synchronize()
    assert np.array_equal(y1[0], y[m - 1])


def test_row_maximum_in_a_low_half_word_on_the_tier():
    n, k, m = 1000, 5120, 16
    w = synth.nvfp4_weight(56, 0, n, k)
    x = amax_trap_rows(m, k)
    W, S, g = dev_weight(w)
    y = bits(nv.gemv(W, S, g, dev_x(x), wide_tensor=True))
    torch.cuda.synchronize()
    assert np.isfinite(oracle.bf16_value(y)).all()
    ref, a = oracle.gemv(w.packed, w.scales, w.g, x)
    check_single(y, ref, a, "row maximum in a low half, tier")


def heavy_tailed_rows(seed, m, k):
    """x rows of N(0, 1) draws times e^N(0, 3^2): magnitudes spread over ~30 binades, the shape
    of a gated activation; the largest values of a row are far from the next ones."""
    a = synth.normal_f32(seed, 0, m * k, 1.0).astype(np.float64)
    s = synth.normal_f32(seed, 2 * m * k, m * k, 3.0).astype(np.float64)
    return oracle.bf16_rne((a * np.exp(s)).reshape(m, k))


def test_heavy_tailed_rows_on_every_path():
    n, k = 1000, 5120
    w = synth.nvfp4_weight(57, 0, n, k)
    wu = synth.nvfp4_weight(57, 10_000_000, n, k)
    W, S, g = dev_weight(w)
    Wu, Su, gu = dev_weight(wu)
    for m, wide in ((8, False), (19, False), (24, True)):
        x = heavy_tailed_rows(57 + m, m, k)
        ref, a = oracle.gemv(w.packed, w.scales, w.g, x)
        y = bits(nv.gemv(W, S, g, dev_x(x), wide_tensor=wide))
        torch.cuda.synchronize()
        check_single(y, ref, a, f"heavy tails, single, M={m}, tier={wide}")
        o = bits(nv.gemv_dual(W, S, g, Wu, Su, gu, dev_x(x), wide_tensor=wide))
        torch.cuda.synchronize()
        o_ref, yg, yu, ag, au = oracle.gemv_dual(w.packed, w.scales, w.g, wu.packed, wu.scales,
                                                 wu.g, x)
        check_dual(o, o_ref, yg, yu, ag, au, f"heavy tails, dual, M={m}, tier={wide}")
        # two outputs share one split (not the single call's), so compare with the oracle
        ys = [bits(t) for t in nv.gemv_multi([(W, S, g), (Wu, Su, gu)], dev_x(x),
                                             wide_tensor=wide)]
        torch.cuda.synchronize()
        check_single(ys[0], ref, a, f"heavy tails, multi output 0, M={m}, tier={wide}")
        check_single(ys[1], yu, au, f"heavy tails, multi output 1, M={m}, tier={wide}")
        if not wide:
            # rows as in calls of their own
            for r in (0, m - 1):
                y1 = bits(nv.gemv(W, S, g, dev_x(x[r:r + 1])))
                torch.cuda.synchronize()
                assert np.array_equal(y1[0], y[r]), f"row {r} of M={m}"
