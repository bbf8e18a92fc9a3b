"""More than 8 rows (the plan's wider multi_seq arms, up to 128 rows): one kernel pass per 8-row
block of x and y, each row computed exactly as in a call of its own, so rows stay bitwise
invariant over M = 1..128.  Results against the fp64 oracle under the acceptance rules."""
import numpy as np
import pytest
import torch

import oracle
import synth
import nvfp4_weight_only_03_b200 as nv
from gpu_util import bits, check_dual, check_single, dev_weight, dev_x

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ws():
    return torch.zeros(nv.workspace_bytes(), dtype=torch.uint8, device="cuda")


def assert_ws_clean(ws):
    torch.cuda.synchronize()
    head = ws[:256 + 4 * torch.cuda.get_device_properties(0).multi_processor_count]
    assert int(head.count_nonzero()) == 0, "workspace flags / error word not left zero"


def test_single_128_rows(ws):
    n, k = 4096, 5120
    w = synth.nvfp4_weight(20, 0, n, k)
    x = synth.activations(20, 100_000_000, 128, k)
    W, S, g = dev_weight(w)
    y128 = bits(nv.gemv(W, S, g, dev_x(x), ws=ws))
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.random.default_rng(1).integers(0, n, 150), [0, n - 1]]))
    ref, a = oracle.gemv(w.packed, w.scales, w.g, x, rows=rows)
    check_single(y128[:, rows], ref, a, "M=128")
    # every row bitwise as in calls of 1, 8 and 37 rows
    for r in (0, 7, 8, 63, 127):
        y1 = bits(nv.gemv(W, S, g, dev_x(x[r:r + 1]), ws=ws))
        assert np.array_equal(y1[0], y128[r]), f"row {r}"
    assert np.array_equal(bits(nv.gemv(W, S, g, dev_x(x[:8]), ws=ws)), y128[:8])
    assert np.array_equal(bits(nv.gemv(W, S, g, dev_x(x[:37]), ws=ws)), y128[:37])
    assert_ws_clean(ws)


def test_strided_rows_beyond_one_pass(ws):
    # 19 rows (three passes, the last of 3 rows) with row strides larger than K and N
    n, k = 1000, 1024
    w = synth.nvfp4_weight(21, 0, n, k)
    x = synth.activations(21, 2_000_000, 19, k)
    W, S, g = dev_weight(w)
    xs = dev_x(x, ldx=k + 64)
    ybuf = torch.full((19, n + 8), float("nan"), dtype=torch.bfloat16, device="cuda")
    y = nv.gemv(W, S, g, xs, y=ybuf[:, :n], ws=ws)
    torch.cuda.synchronize()
    ref, a = oracle.gemv(w.packed, w.scales, w.g, x)
    check_single(bits(y), ref, a, "strided M=19")
    assert torch.isnan(ybuf[:, n:].float()).all(), "wrote past the rows' N outputs"
    assert_ws_clean(ws)


def test_dual_24_rows(ws):
    n, k = 2048, 5120
    wg = synth.nvfp4_weight(22, 0, n, k)
    wu = synth.nvfp4_weight(22, 20_000_000, n, k)
    x = synth.activations(22, 40_000_000, 24, k)
    Wg, Sg, gg = dev_weight(wg)
    Wu, Su, gu = dev_weight(wu)
    o24 = bits(nv.gemv_dual(Wg, Sg, gg, Wu, Su, gu, dev_x(x), ws=ws))
    torch.cuda.synchronize()
    rows = np.arange(0, n, 13)
    o_ref, yg, yu, ag, au = oracle.gemv_dual(wg.packed, wg.scales, wg.g, wu.packed, wu.scales,
                                             wu.g, x, rows=rows)
    check_dual(o24[:, rows], o_ref, yg, yu, ag, au, "dual M=24")
    for r in (0, 9, 23):
        o1 = bits(nv.gemv_dual(Wg, Sg, gg, Wu, Su, gu, dev_x(x[r:r + 1]), ws=ws))
        assert np.array_equal(o1[0], o24[r]), f"row {r}"
    assert_ws_clean(ws)


def test_multi_20_rows(ws):
    wl = synth.make("attn_kv", generate_x=False)
    weights = [p.w for p in wl.projections]
    k = weights[0].k
    x = synth.activations(23, 0, 20, k)
    devs = [dev_weight(w) for w in weights]
    ys = [bits(y) for y in nv.gemv_multi(devs, dev_x(x), ws=ws)]
    torch.cuda.synchronize()
    for o, (w, y) in enumerate(zip(weights, ys)):
        ref, a = oracle.gemv(w.packed, w.scales, w.g, x)
        check_single(y, ref, a, f"multi M=20 output {o}")
    for r in (3, 19):
        y1 = [bits(y) for y in nv.gemv_multi(devs, dev_x(x[r:r + 1]), ws=ws)]
        for o in range(len(weights)):
            assert np.array_equal(y1[o][0], ys[o][r]), f"output {o} row {r}"
    assert_ws_clean(ws)


def test_noalloc_17_rows_match_nvfp4_gemv(ws):
    n, k = 3000, 2048
    w = synth.nvfp4_weight(24, 0, n, k)
    x = synth.activations(24, 10_000_000, 17, k)
    W, S, g = dev_weight(w)
    y_ws = bits(nv.gemv(W, S, g, dev_x(x), ws=ws))
    y_na = bits(nv.gemv_noalloc(W, S, g, dev_x(x)))
    torch.cuda.synchronize()
    assert np.array_equal(y_ws, y_na)
