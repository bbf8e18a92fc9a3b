"""Input prologues through the C ABI against the oracle: residual add + RMS norm (single, dual,
multi-output, 8-row passes, the tensor-core tier) and the sigmoid gate.

The GPU forms x' in fp32 and rounds it to bf16; the oracle forms it in fp64.  Where the fp64
value lies within a relative 2^-16 of a bf16 rounding midpoint the two may round apart, so the
tolerance of each output grows by sum_k |w_k| * (one bf16 step of x'_k) over those elements
(oracle.rounding_slack); everywhere else the acceptance rules are unchanged.  The residual sum h
is exactly rounded on both sides and compared bitwise."""
import numpy as np
import pytest
import torch

import oracle
import synth
import nvfp4_weight_only_03_b200 as nv
from gpu_util import bits, check_dual, check_single, dev_weight, dev_x

pytestmark = pytest.mark.gpu


def dev_vec(v_bits):
    return torch.from_numpy(np.ascontiguousarray(v_bits).view(np.int16)).view(torch.bfloat16).cuda()


def check_pro_single(y_bits, w, xq, near, where, rows=None):
    ref, a = oracle.gemv(w.packed, w.scales, w.g, xq, rows=rows)
    _, extra = oracle.gemv(w.packed, w.scales, w.g, oracle.rounding_slack(xq, near), rows=rows)
    return check_single(y_bits, ref, a + extra / 2e-3, where)


def check_pro_dual(o_bits, wg, wu, xq, near, where, rows=None):
    o_ref, yg, yu, ag, au = oracle.gemv_dual(wg.packed, wg.scales, wg.g, wu.packed, wu.scales,
                                             wu.g, xq, rows=rows)
    slack = oracle.rounding_slack(xq, near)
    _, eg = oracle.gemv(wg.packed, wg.scales, wg.g, slack, rows=rows)
    _, eu = oracle.gemv(wu.packed, wu.scales, wu.g, slack, rows=rows)
    return check_dual(o_bits, o_ref, yg, yu, ag + eg / 2e-3, au + eu / 2e-3, where)


def norm_inputs(seed, m, k, x_scale=1.0):
    x = synth.activations(seed, 300_000_000, m, k)
    r = synth.residual_stream(seed, 310_000_000, m, k)
    if x_scale != 1.0:  # exact power-of-two scaling of both (bf16 exponent shift)
        x = oracle.bf16_rne(oracle.bf16_value(x) * x_scale)
        r = oracle.bf16_rne(oracle.bf16_value(r) * x_scale)
    gamma = synth.norm_gains(seed, 320_000_000, k)
    return x, r, gamma


def sample_rows(n, count=160):
    if n <= 2048:
        return None
    return np.unique(np.concatenate([np.random.default_rng(n).integers(0, n, count),
                                     [0, 127, 128, n - 1]]))


@pytest.mark.parametrize("m", [1, 8])
def test_add_rmsnorm_single(m):
    n, k, eps = 4096 + 77, 5120, 1e-6
    w = synth.nvfp4_weight(40, 0, n, k)
    x, r, gamma = norm_inputs(40, m, k)
    W, S, g = dev_weight(w)
    h_out = torch.full((m, k), float("nan"), dtype=torch.bfloat16, device="cuda")
    pro = nv.AddRmsNorm(dev_x(r), dev_vec(gamma), eps, h_out)
    y = bits(nv.gemv(W, S, g, dev_x(x), prologue=pro))
    h_ref, xn, near = oracle.add_rmsnorm(x, r, gamma, eps)
    assert np.array_equal(bits(h_out), h_ref), "residual sum h"
    rows = sample_rows(n)
    check_pro_single(y if rows is None else y[:, rows], w, xn, near, f"add_rmsnorm M={m}", rows)
    # determinism, and each row as in a call of its own
    assert np.array_equal(bits(nv.gemv(W, S, g, dev_x(x), prologue=pro)), y)
    for i in (0, m - 1):
        y1 = bits(nv.gemv(W, S, g, dev_x(x[i:i + 1]),
                          prologue=nv.AddRmsNorm(dev_x(r[i:i + 1]), dev_vec(gamma), eps)))
        assert np.array_equal(y1[0], y[i]), f"row {i}"


@pytest.mark.parametrize("scale,eps", [(2.0 ** -14, 1e-6), (1.0, 0.5), (2.0 ** 20, 0.0)])
def test_add_rmsnorm_eps_and_magnitudes(scale, eps):
    # eps dominating the mean square, a large eps, and large magnitudes with eps = 0
    n, k, m = 1000, 2048, 3
    w = synth.nvfp4_weight(41, 0, n, k)
    x, r, gamma = norm_inputs(41, m, k, x_scale=scale)
    W, S, g = dev_weight(w)
    y = bits(nv.gemv(W, S, g, dev_x(x), prologue=nv.AddRmsNorm(dev_x(r), dev_vec(gamma), eps)))
    _, xn, near = oracle.add_rmsnorm(x, r, gamma, eps)
    check_pro_single(y, w, xn, near, f"scale={scale} eps={eps}")


def test_add_rmsnorm_dual():
    n, k, m, eps = 2048, 5120, 4, 1e-6
    wg = synth.nvfp4_weight(42, 0, n, k)
    wu = synth.nvfp4_weight(42, 20_000_000, n, k)
    x, r, gamma = norm_inputs(42, m, k)
    Wg, Sg, gg = dev_weight(wg)
    Wu, Su, gu = dev_weight(wu)
    h_out = torch.empty((m, k), dtype=torch.bfloat16, device="cuda")
    o = bits(nv.gemv_dual(Wg, Sg, gg, Wu, Su, gu, dev_x(x),
                          prologue=nv.AddRmsNorm(dev_x(r), dev_vec(gamma), eps, h_out)))
    h_ref, xn, near = oracle.add_rmsnorm(x, r, gamma, eps)
    assert np.array_equal(bits(h_out), h_ref)
    check_pro_dual(o, wg, wu, xn, near, "dual add_rmsnorm")


def test_add_rmsnorm_multi():
    # the attention projections sharing the normed x: q (6144) and k, v (1024 each)
    k, m, eps = 5120, 3, 1e-6
    ws_ = [synth.nvfp4_weight(43, off, n, k) for off, n in
           ((0, 6144), (40_000_000, 1024), (50_000_000, 1024))]
    x, r, gamma = norm_inputs(43, m, k)
    devs = [dev_weight(w) for w in ws_]
    h_out = torch.empty((m, k), dtype=torch.bfloat16, device="cuda")
    ys = [bits(y) for y in nv.gemv_multi(devs, dev_x(x), prologue=nv.AddRmsNorm(
        dev_x(r), dev_vec(gamma), eps, h_out))]
    h_ref, xn, near = oracle.add_rmsnorm(x, r, gamma, eps)
    assert np.array_equal(bits(h_out), h_ref)
    for o, (w, y) in enumerate(zip(ws_, ys)):
        rows = sample_rows(w.n)
        check_pro_single(y if rows is None else y[:, rows], w, xn, near, f"multi output {o}", rows)


@pytest.mark.parametrize("m", [1, 8])
def test_sigmoid_gate_single(m):
    # the attention output projection: o 5120 x 6144 after the sigmoid gate
    n, k = 5120, 6144
    w = synth.nvfp4_weight(44, 0, n, k)
    a = synth.activations(44, 300_000_000, m, k)
    t = synth.gate_logits(44, 310_000_000, m, k)
    W, S, g = dev_weight(w)
    y = bits(nv.gemv(W, S, g, dev_x(a), prologue=nv.SigmoidGate(dev_x(t))))
    xo, near = oracle.sigmoid_gate(a, t)
    rows = sample_rows(n)
    check_pro_single(y[:, rows], w, xo, near, f"sigmoid gate M={m}", rows)
    if m > 1:
        y1 = bits(nv.gemv(W, S, g, dev_x(a[m - 1:]), prologue=nv.SigmoidGate(dev_x(t[m - 1:]))))
        assert np.array_equal(y1[0], y[m - 1])


def test_prologue_with_ragged_k_and_passes():
    # K % 256 != 0 (partial last unit), 19 rows (three 8-row passes), strided arrays
    n, k, m, eps = 700, 5120 + 96, 19, 1e-5
    w = synth.nvfp4_weight(45, 0, n, k)
    x, r, gamma = norm_inputs(45, m, k)
    W, S, g = dev_weight(w)
    hbuf = torch.full((m, k + 40), float("nan"), dtype=torch.bfloat16, device="cuda")
    pro = nv.AddRmsNorm(dev_x(r, ldx=k + 64), dev_vec(gamma), eps, hbuf[:, :k])
    y = bits(nv.gemv(W, S, g, dev_x(x, ldx=k + 128), prologue=pro))
    h_ref, xn, near = oracle.add_rmsnorm(x, r, gamma, eps)
    assert np.array_equal(bits(hbuf[:, :k]), h_ref)
    assert torch.isnan(hbuf[:, k:].float()).all(), "wrote past K in residual_out"
    check_pro_single(y, w, xn, near, "ragged K, 19 rows")
    for i in (0, 8, 18):
        y1 = bits(nv.gemv(W, S, g, dev_x(x[i:i + 1]),
                          prologue=nv.AddRmsNorm(dev_x(r[i:i + 1]), dev_vec(gamma), eps)))
        assert np.array_equal(y1[0], y[i]), f"row {i}"
    # a gate prologue at the same ragged K
    t = synth.gate_logits(45, 330_000_000, m, k)
    y = bits(nv.gemv(W, S, g, dev_x(x), prologue=nv.SigmoidGate(dev_x(t))))
    xo, near = oracle.sigmoid_gate(x, t)
    check_pro_single(y, w, xo, near, "gate, ragged K, 19 rows")


def test_kind_none_is_the_plain_call():
    n, k, m = 1500, 2048, 5
    w = synth.nvfp4_weight(46, 0, n, k)
    x = synth.activations(46, 300_000_000, m, k)
    W, S, g = dev_weight(w)

    class NoneKind:
        def struct(self, m_, k_):
            return nv.Prologue(kind=nv.PROLOGUE_NONE)

    assert np.array_equal(bits(nv.gemv(W, S, g, dev_x(x), prologue=NoneKind())),
                          bits(nv.gemv(W, S, g, dev_x(x))))


def test_prologue_on_the_tensor_core_tier():
    n, k, m, eps = 4096, 5120, 24, 1e-6
    w = synth.nvfp4_weight(47, 0, n, k)
    wu = synth.nvfp4_weight(47, 30_000_000, n, k)
    x, r, gamma = norm_inputs(47, m, k)
    W, S, g = dev_weight(w)
    Wu, Su, gu = dev_weight(wu)
    h_out = torch.empty((m, k), dtype=torch.bfloat16, device="cuda")
    pro = nv.AddRmsNorm(dev_x(r), dev_vec(gamma), eps, h_out)
    y = bits(nv.gemv(W, S, g, dev_x(x), prologue=pro, wide_tensor=True))
    h_ref, xn, near = oracle.add_rmsnorm(x, r, gamma, eps)
    assert np.array_equal(bits(h_out), h_ref)
    rows = sample_rows(n)
    check_pro_single(y[:, rows], w, xn, near, "tier add_rmsnorm", rows)
    # rows invariant within the tier (9..24 rows)
    y9 = bits(nv.gemv(W, S, g, dev_x(x[:9]), wide_tensor=True,
                      prologue=nv.AddRmsNorm(dev_x(r[:9]), dev_vec(gamma), eps)))
    assert np.array_equal(y9, y[:9])
    o = bits(nv.gemv_dual(W, S, g, Wu, Su, gu, dev_x(x), wide_tensor=True,
                          prologue=nv.AddRmsNorm(dev_x(r), dev_vec(gamma), eps)))
    check_pro_dual(o[:, rows], w, wu, xn, near, "tier dual add_rmsnorm", rows)
    t = synth.gate_logits(47, 330_000_000, m, k)
    y = bits(nv.gemv(W, S, g, dev_x(x), prologue=nv.SigmoidGate(dev_x(t)), wide_tensor=True))
    xo, near = oracle.sigmoid_gate(x, t)
    check_pro_single(y[:, rows], w, xo, near, "tier sigmoid gate", rows)
    assert nv.workspace_error(nv.wide_workspace(n, k, m)) == 0


def test_prologue_needs_the_larger_workspace():
    n, k, m = 256, 512, 2
    w = synth.nvfp4_weight(48, 0, n, k)
    x, r, gamma = norm_inputs(48, m, k)
    W, S, g = dev_weight(w)
    small = torch.zeros(nv.workspace_bytes(), dtype=torch.uint8, device="cuda")
    assert nv.workspace_bytes_wide(n, k, m) > nv.workspace_bytes()
    with pytest.raises(nv.Nvfp4Error) as e:
        nv.gemv(W, S, g, dev_x(x), ws=small,
                prologue=nv.AddRmsNorm(dev_x(r), dev_vec(gamma), 1e-6))
    assert e.value.status == -7
    big = torch.zeros(nv.workspace_bytes_wide(n, k, m), dtype=torch.uint8, device="cuda")
    y = bits(nv.gemv(W, S, g, dev_x(x), ws=big,
                     prologue=nv.AddRmsNorm(dev_x(r), dev_vec(gamma), 1e-6)))
    _, xn, near = oracle.add_rmsnorm(x, r, gamma, 1e-6)
    check_pro_single(y, w, xn, near, "explicit workspace")


def test_prologue_beyond_one_register_round():
    # K = 17408 > 4 x 512 chunks of 8: the norm re-reads x, the residual and gamma for x', and
    # the gate walks its row in several rounds; 12 rows run as two 8-row GEMV passes
    n, k, m, eps = 640, 17408, 12, 1e-6
    w = synth.nvfp4_weight(49, 0, n, k)
    x, r, gamma = norm_inputs(49, m, k)
    W, S, g = dev_weight(w)
    h_out = torch.empty((m, k), dtype=torch.bfloat16, device="cuda")
    y = bits(nv.gemv(W, S, g, dev_x(x), prologue=nv.AddRmsNorm(dev_x(r), dev_vec(gamma), eps,
                                                                h_out)))
    h_ref, xn, near = oracle.add_rmsnorm(x, r, gamma, eps)
    assert np.array_equal(bits(h_out), h_ref)
    check_pro_single(y, w, xn, near, "norm, K = 17408")
    y1 = bits(nv.gemv(W, S, g, dev_x(x[5:6]),
                      prologue=nv.AddRmsNorm(dev_x(r[5:6]), dev_vec(gamma), eps)))
    assert np.array_equal(y1[0], y[5])
    t = synth.gate_logits(49, 330_000_000, m, k)
    y = bits(nv.gemv(W, S, g, dev_x(x), prologue=nv.SigmoidGate(dev_x(t))))
    xo, near = oracle.sigmoid_gate(x, t)
    check_pro_single(y, w, xo, near, "gate, K = 17408")


def test_prologue_chain_with_programmatic_launch_and_graphs():
    # a layer's chain: qkv-like GEMV after a norm (writes h1), an o-like GEMV after the sigmoid
    # gate, whose output feeds the dual after a norm with h1 as the residual (writes h2); run
    # plain, with programmatic dependent launch, and as a replayed CUDA graph: all bitwise equal
    k, m, eps = 1024, 4, 1e-6
    wq = synth.nvfp4_weight(50, 0, 1536, k)
    wo = synth.nvfp4_weight(50, 10_000_000, k, k)
    wg = synth.nvfp4_weight(50, 20_000_000, 2048, k)
    wu = synth.nvfp4_weight(50, 30_000_000, 2048, k)
    x, r, gamma1 = norm_inputs(50, m, k)
    gamma2 = synth.norm_gains(50, 340_000_000, k)
    a = synth.activations(50, 350_000_000, m, k)
    t = synth.gate_logits(50, 360_000_000, m, k)
    Wq, Wo, Wg, Wu = (dev_weight(w) for w in (wq, wo, wg, wu))
    dx, dr, da, dt = dev_x(x), dev_x(r), dev_x(a), dev_x(t)
    g1, g2 = dev_vec(gamma1), dev_vec(gamma2)
    ws = torch.zeros(nv.workspace_bytes_wide(2048, k, m), dtype=torch.uint8, device="cuda")
    outs = {n_: torch.empty(shape, dtype=torch.bfloat16, device="cuda") for n_, shape in
            (("q", (m, 1536)), ("o", (m, k)), ("gu", (m, 2048)), ("h1", (m, k)), ("h2", (m, k)))}

    def chain(pdl, stream=None):
        nv.gemv(*Wq, dx, y=outs["q"], ws=ws, stream=stream, prefetch_weights=pdl,
                prologue=nv.AddRmsNorm(dr, g1, eps, outs["h1"]))
        nv.gemv(*Wo, da, y=outs["o"], ws=ws, stream=stream, prefetch_weights=pdl,
                prologue=nv.SigmoidGate(dt))
        nv.gemv_dual(*Wg, *Wu, outs["o"], y=outs["gu"], ws=ws, stream=stream,
                     prefetch_weights=pdl, prologue=nv.AddRmsNorm(outs["h1"], g2, eps, outs["h2"]))

    def snapshot():
        torch.cuda.synchronize()
        return {n_: bits(v) for n_, v in outs.items()}

    chain(False)
    ref = snapshot()
    for v in outs.values():
        v.fill_(float("nan"))
    chain(True)
    assert all(np.array_equal(ref[n_], got) for n_, got in snapshot().items()), "with PDL"
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        chain(True, s)  # warm-up on the capture stream
    s.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        chain(True, torch.cuda.current_stream())
    for v in outs.values():
        v.fill_(float("nan"))
    for _ in range(3):
        graph.replay()
    assert all(np.array_equal(ref[n_], got) for n_, got in snapshot().items()), "graph replay"
    del graph
    # the chain against the oracle: h1, then the gate's GEMV, then the dual on its output
    h1, xn1, near1 = oracle.add_rmsnorm(x, r, gamma1, eps)
    assert np.array_equal(ref["h1"], h1)
    check_pro_single(ref["q"], wq, xn1, near1, "chain q")
    xo, neargate = oracle.sigmoid_gate(a, t)
    check_pro_single(ref["o"], wo, xo, neargate, "chain o")
    h2, xn2, near2 = oracle.add_rmsnorm(ref["o"], h1, gamma2, eps)
    assert np.array_equal(ref["h2"], h2)
    check_pro_dual(ref["gu"], wg, wu, xn2, near2, "chain gate_up")


def test_prologue_with_multi_on_the_tier():
    # q, k, v sharing the normed x at M = 24 on the tier: each output bitwise its own
    # single-output call with the same prologue, and within tolerance of the oracle
    k, m, eps = 5120, 24, 1e-6
    ws_ = [synth.nvfp4_weight(51, off, n, k) for off, n in
           ((0, 2048), (20_000_000, 1024), (30_000_000, 1024))]
    x, r, gamma = norm_inputs(51, m, k)
    devs = [dev_weight(w) for w in ws_]
    h_out = torch.empty((m, k), dtype=torch.bfloat16, device="cuda")
    ys = [bits(y) for y in nv.gemv_multi(devs, dev_x(x), wide_tensor=True, prologue=nv.AddRmsNorm(
        dev_x(r), dev_vec(gamma), eps, h_out))]
    h_ref, xn, near = oracle.add_rmsnorm(x, r, gamma, eps)
    assert np.array_equal(bits(h_out), h_ref)
    for o, (w, d) in enumerate(zip(ws_, devs)):
        single = bits(nv.gemv(*d, dev_x(x), wide_tensor=True,
                              prologue=nv.AddRmsNorm(dev_x(r), dev_vec(gamma), eps)))
        assert np.array_equal(ys[o], single), f"output {o}"
        rows = sample_rows(w.n, 100) if w.n > 2048 else None
        check_pro_single(ys[o] if rows is None else ys[o][:, rows], w, xn, near,
                         f"multi tier output {o}", rows)


def gated_inputs(seed, m, k, g):
    x = synth.normal_f32(seed, 400_000_000, m * k, 1.0).reshape(m, k)
    z = synth.gate_logits(seed, 410_000_000, m, k)
    gamma = synth.norm_gains(seed, 420_000_000, g)
    return x, z, gamma


def dev_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


@pytest.mark.parametrize("m", [1, 8, 19])
def test_gated_rmsnorm_single(m):
    # the GatedDeltaNet's output projection: K = 48 heads x 128 channels, fp32 x
    n, k, g, eps = 2000, 6144, 128, 1e-6
    w = synth.nvfp4_weight(52, 0, n, k)
    x, z, gamma = gated_inputs(52, m, k, g)
    W, S, gs = dev_weight(w)
    y = bits(nv.gemv(W, S, gs, dev_f32(x), prologue=nv.GatedRmsNorm(dev_x(z), dev_vec(gamma), g,
                                                                     eps)))
    xo, near = oracle.gated_rmsnorm(x, z, gamma, g, eps)
    check_pro_single(y, w, xo, near, f"gated rmsnorm M={m}")
    r = m - 1
    y1 = bits(nv.gemv(W, S, gs, dev_f32(x[r:r + 1]),
                      prologue=nv.GatedRmsNorm(dev_x(z[r:r + 1]), dev_vec(gamma), g, eps)))
    assert np.array_equal(y1[0], y[r]), f"row {r}"


@pytest.mark.parametrize("g", [256, 512])
def test_gated_rmsnorm_group_sizes(g):
    n, k, m, eps = 700, 2048, 3, 1e-5
    w = synth.nvfp4_weight(53, 0, n, k)
    x, z, gamma = gated_inputs(53, m, k, g)
    W, S, gs = dev_weight(w)
    y = bits(nv.gemv(W, S, gs, dev_f32(x), prologue=nv.GatedRmsNorm(dev_x(z), dev_vec(gamma), g,
                                                                     eps)))
    xo, near = oracle.gated_rmsnorm(x, z, gamma, g, eps)
    check_pro_single(y, w, xo, near, f"gated rmsnorm G={g}")


def test_gated_rmsnorm_ignores_the_wide_flag():
    n, k, m, g = 1024, 5120, 24, 128
    w = synth.nvfp4_weight(54, 0, n, k)
    x, z, gamma = gated_inputs(54, m, k, g)
    W, S, gs = dev_weight(w)
    pro = nv.GatedRmsNorm(dev_x(z), dev_vec(gamma), g)
    y_wide = bits(nv.gemv(W, S, gs, dev_f32(x), prologue=pro, wide_tensor=True))
    y_pass = bits(nv.gemv(W, S, gs, dev_f32(x), prologue=pro))
    assert np.array_equal(y_wide, y_pass)
