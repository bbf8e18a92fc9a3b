"""The tensor-core tier for 9..128 rows (NVFP4_FLAG_WIDE_TENSOR) through the C ABI against the
fp64 oracle under the acceptance rules; bitwise row invariance over M = 9..128 and determinism;
both ways of finishing a tile (direct, or fp32 partials of a K split added in order); the fused
dual (gate and up through the tier in fp32, then SiLU(gate)*up); and the fall-back to 8-row
passes where the tier does not apply."""
import numpy as np
import pytest
import torch

import oracle
import synth
import nvfp4_weight_only_03_b200 as nv
from gpu_util import bits, check_dual, check_single, dev_weight, dev_x

pytestmark = pytest.mark.gpu


def wide(W, S, g, x_dev, ws=None):
    y = nv.gemv(W, S, g, x_dev, ws=ws, wide_tensor=True)
    torch.cuda.synchronize()
    return bits(y)


@pytest.mark.parametrize("n,k,m", [
    (4096, 5120, 128),       # K split in 4: fp32 partials added by the reduce kernel
    (4096, 5120, 9),
    (1000 + 77, 1024, 40),   # ragged N
    (512, 17408, 64),        # long K
    (148 * 128, 512, 16),    # one tile per SM, no K split: the tier writes y itself
])
def test_tier_matches_oracle(n, k, m):
    w = synth.nvfp4_weight(30, 0, n, k)
    x = synth.activations(30, 200_000_000, m, k)
    W, S, g = dev_weight(w)
    y = wide(W, S, g, dev_x(x))
    rows = None if n <= 2048 else np.unique(
        np.concatenate([np.random.default_rng(n).integers(0, n, 200), [0, 127, 128, n - 1]]))
    ref, a = oracle.gemv(w.packed, w.scales, w.g, x, rows=rows)
    check_single(y if rows is None else y[:, rows], ref, a, f"tier n={n} k={k} M={m}")
    err = nv.workspace_error(nv.wide_workspace(n, k, m))
    assert err == 0


def test_tier_rows_invariant_and_deterministic():
    n, k = 4096, 5120
    w = synth.nvfp4_weight(31, 0, n, k)
    x = synth.activations(31, 100_000_000, 128, k)
    W, S, g = dev_weight(w)
    y128 = wide(W, S, g, dev_x(x))
    for m in (9, 33, 100):
        assert np.array_equal(wide(W, S, g, dev_x(x[:m])), y128[:m]), f"M={m}"
    assert np.array_equal(wide(W, S, g, dev_x(x[50:70])), y128[50:70])
    assert np.array_equal(wide(W, S, g, dev_x(x)), y128)


def test_tier_strided_x_and_y():
    n, k, m = 2000, 2048, 24
    w = synth.nvfp4_weight(32, 0, n, k)
    x = synth.activations(32, 10_000_000, m, k)
    W, S, g = dev_weight(w)
    ybuf = torch.full((m, n + 40), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = nv.gemv(W, S, g, dev_x(x, ldx=k + 256), y=ybuf[:, :n], wide_tensor=True)
    torch.cuda.synchronize()
    ref, a = oracle.gemv(w.packed, w.scales, w.g, x)
    check_single(bits(y), ref, a, "tier strided")
    assert torch.isnan(ybuf[:, n:].float()).all()


def test_tier_falls_back_to_passes_where_it_does_not_apply():
    # K % 256 != 0: the flag is ignored, the call runs as 8-row passes (bitwise)
    n, k, m = 700, 5120 + 32, 12
    w = synth.nvfp4_weight(33, 0, n, k)
    x = synth.activations(33, 10_000_000, m, k)
    W, S, g = dev_weight(w)
    y_flag = wide(W, S, g, dev_x(x))
    y_pass = bits(nv.gemv(W, S, g, dev_x(x)))
    torch.cuda.synchronize()
    assert np.array_equal(y_flag, y_pass)
    # 1..8 rows never use the tier
    assert np.array_equal(wide(W, S, g, dev_x(x[:8])), bits(nv.gemv(W, S, g, dev_x(x[:8]))))


def test_tier_rejects_a_small_workspace():
    n, k, m = 4096, 5120, 32
    assert nv.workspace_bytes_wide(n, k, m) > nv.workspace_bytes()
    ws = torch.zeros(nv.workspace_bytes(), dtype=torch.uint8, device="cuda")
    W = torch.zeros((n, k // 2), dtype=torch.uint8, device="cuda")
    S = torch.zeros((n, k // 16), dtype=torch.uint8, device="cuda")
    x = torch.zeros((m, k), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nv.Nvfp4Error) as e:
        nv.gemv(W, S, 1.0, x, ws=ws, wide_tensor=True)
    assert e.value.status == -7


def wide_dual(Wg, Sg, gg, Wu, Su, gu, x_dev):
    o = nv.gemv_dual(Wg, Sg, gg, Wu, Su, gu, x_dev, wide_tensor=True)
    torch.cuda.synchronize()
    return bits(o)


@pytest.mark.parametrize("n,k,m", [
    (2048, 5120, 24),        # K split: both streams reduced into fp32 before the combine
    (1000 + 77, 1024, 40),   # ragged N
    (148 * 128, 512, 128),   # no K split: the tier writes the fp32 results itself
])
def test_dual_tier_matches_oracle(n, k, m):
    wg = synth.nvfp4_weight(34, 0, n, k)
    wu = synth.nvfp4_weight(34, 40_000_000, n, k)
    x = synth.activations(34, 80_000_000, m, k)
    Wg, Sg, gg = dev_weight(wg)
    Wu, Su, gu = dev_weight(wu)
    o = wide_dual(Wg, Sg, gg, Wu, Su, gu, dev_x(x))
    rows = None if n <= 2048 else np.unique(
        np.concatenate([np.random.default_rng(n).integers(0, n, 150), [0, 127, 128, n - 1]]))
    o_ref, yg, yu, ag, au = oracle.gemv_dual(wg.packed, wg.scales, wg.g, wu.packed, wu.scales,
                                             wu.g, x, rows=rows)
    check_dual(o if rows is None else o[:, rows], o_ref, yg, yu, ag, au,
               f"dual tier n={n} k={k} M={m}")
    assert nv.workspace_error(nv.wide_workspace(n, k, m)) == 0


def test_dual_tier_rows_invariant_and_deterministic():
    n, k = 2048, 5120
    wg = synth.nvfp4_weight(35, 0, n, k)
    wu = synth.nvfp4_weight(35, 20_000_000, n, k)
    x = synth.activations(35, 40_000_000, 128, k)
    Wg, Sg, gg = dev_weight(wg)
    Wu, Su, gu = dev_weight(wu)
    o128 = wide_dual(Wg, Sg, gg, Wu, Su, gu, dev_x(x))
    for m in (9, 64):
        assert np.array_equal(wide_dual(Wg, Sg, gg, Wu, Su, gu, dev_x(x[:m])), o128[:m]), m
    assert np.array_equal(wide_dual(Wg, Sg, gg, Wu, Su, gu, dev_x(x[30:47])), o128[30:47])
    assert np.array_equal(wide_dual(Wg, Sg, gg, Wu, Su, gu, dev_x(x)), o128)


def test_dual_tier_strided_and_fallback():
    n, k, m = 900, 2048, 20
    wg = synth.nvfp4_weight(36, 0, n, k)
    wu = synth.nvfp4_weight(36, 4_000_000, n, k)
    x = synth.activations(36, 8_000_000, m, k)
    Wg, Sg, gg = dev_weight(wg)
    Wu, Su, gu = dev_weight(wu)
    ybuf = torch.full((m, n + 24), float("nan"), dtype=torch.bfloat16, device="cuda")
    o = nv.gemv_dual(Wg, Sg, gg, Wu, Su, gu, dev_x(x, ldx=k + 128), y=ybuf[:, :n],
                     wide_tensor=True)
    torch.cuda.synchronize()
    o_ref, yg, yu, ag, au = oracle.gemv_dual(wg.packed, wg.scales, wg.g, wu.packed, wu.scales,
                                             wu.g, x)
    check_dual(bits(o), o_ref, yg, yu, ag, au, "dual tier strided")
    assert torch.isnan(ybuf[:, n:].float()).all()
    # 1..8 rows ignore the flag (bitwise the fused dual kernel)
    o8 = wide_dual(Wg, Sg, gg, Wu, Su, gu, dev_x(x[:8]))
    assert np.array_equal(o8, bits(nv.gemv_dual(Wg, Sg, gg, Wu, Su, gu, dev_x(x[:8]))))


def test_multi_on_the_tier_matches_single_calls_and_oracle():
    # the attention's q and gate (6144 x 5120 each) and k, v (1024 x 5120) sharing x at M = 24
    k, m = 5120, 24
    ws_ = [synth.nvfp4_weight(37, off, n, k) for off, n in
           ((0, 6144), (40_000_000, 1024), (50_000_000, 1024))]
    x = synth.activations(37, 80_000_000, m, k)
    devs = [dev_weight(w) for w in ws_]
    ys = [bits(y) for y in nv.gemv_multi(devs, dev_x(x), wide_tensor=True)]
    torch.cuda.synchronize()
    for o, (w, d) in enumerate(zip(ws_, devs)):
        assert np.array_equal(ys[o], wide(*d, dev_x(x))), f"output {o} vs its own call"
        rows = np.unique(np.concatenate([np.random.default_rng(o).integers(0, w.n, 120),
                                         [0, 127, w.n - 1]]))
        ref, a = oracle.gemv(w.packed, w.scales, w.g, x, rows=rows)
        check_single(ys[o][:, rows], ref, a, f"multi tier output {o}")
    # rows invariant over M within the tier
    ys9 = [bits(y) for y in nv.gemv_multi(devs, dev_x(x[:9]), wide_tensor=True)]
    torch.cuda.synchronize()
    for o in range(3):
        assert np.array_equal(ys9[o], ys[o][:9])
    # 1..8 rows ignore the flag
    y8 = [bits(y) for y in nv.gemv_multi(devs, dev_x(x[:8]), wide_tensor=True)]
    p8 = [bits(y) for y in nv.gemv_multi(devs, dev_x(x[:8]))]
    torch.cuda.synchronize()
    for o in range(3):
        assert np.array_equal(y8[o], p8[o])
