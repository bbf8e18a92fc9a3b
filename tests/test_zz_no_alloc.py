"""nvfp4_gemv_noalloc, the entry point that runs on the library's compiled-in scratch instead
of a caller workspace, against nvfp4_gemv (and the oracle) through the C ABI.

Collected last on purpose: it must pass both alone and after every other GPU test, when the
device and the library's per-device state have already been used by the workspace path.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import nvfp4_weight_only_03_b200 as nv
from gpu_util import bits, check_single, dev_weight, dev_x

pytestmark = pytest.mark.gpu


def noalloc(W, S, g, x, m, n, k):
    y = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = nv.lib().nvfp4_gemv_noalloc(W.data_ptr(), S.data_ptr(), float(g), x.data_ptr(), k,
                                     y.data_ptr(), n, m, n, k,
                                     torch.cuda.current_stream().cuda_stream)
    assert st == 0, nv.lib().nvfp4_status_string(st).decode()
    return y


def with_workspace(W, S, g, x, m, n, k):
    ws = torch.zeros(nv.workspace_bytes(), dtype=torch.uint8, device="cuda")
    y = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = nv.lib().nvfp4_gemv(W.data_ptr(), S.data_ptr(), float(g), x.data_ptr(), k,
                             y.data_ptr(), n, m, n, k, ws.data_ptr(), ws.numel(),
                             torch.cuda.current_stream().cuda_stream)
    assert st == 0, nv.lib().nvfp4_status_string(st).decode()
    return y


def agree_within_tolerance(y_a, y_b, a_ref, where):
    """Both outputs as reals, |a - b| within the acceptance tolerance 2e-3 A + 1e-6."""
    va, vb = oracle.bf16_value(y_a), oracle.bf16_value(y_b)
    tol = oracle.tolerance(a_ref)
    bad = np.argwhere(~(np.abs(va - vb) <= tol))
    assert bad.size == 0, f"{where}: {bad.shape[0]} elements differ beyond tolerance"


@pytest.mark.parametrize("m", [1, 8])
def test_two_calls_in_a_row_match_the_workspace_path(m):
    # 10240 x 5120: 80 row groups over the persistent grid, so CTAs hand partial sums to each
    # other through the scratch's flags on every call.
    p = synth.make("inproj").projections[0]
    W, S, g = dev_weight(p.w)
    n, k = p.w.n, p.w.k
    x = dev_x(p.x[:m])
    ref, a = oracle.gemv(p.w.packed, p.w.scales, p.w.g, p.x[:m])
    y_ws = bits(with_workspace(W, S, g, x, m, n, k))
    first = bits(noalloc(W, S, g, x, m, n, k))
    second = bits(noalloc(W, S, g, x, m, n, k))
    torch.cuda.synchronize()
    for name, y in (("first", first), ("second", second)):
        agree_within_tolerance(y, y_ws, a, f"{name} call vs nvfp4_gemv, M={m}")
        check_single(y, ref, a, f"{name} noalloc call vs oracle, M={m}")
    # the same kernel and work split as nvfp4_gemv: identical bits, call after call
    assert np.array_equal(first, y_ws) and np.array_equal(second, y_ws)


def test_24_rows_run_as_passes_on_the_shared_scratch():
    # 24 rows: three 8-row kernel passes in stream order, all on the one compiled-in scratch
    p = synth.make("inproj").projections[0]
    W, S, g = dev_weight(p.w)
    n, k = p.w.n, p.w.k
    rng = np.random.default_rng(24)
    xb = oracle.bf16_rne(rng.standard_normal((24, k)))
    x = dev_x(xb)
    y_ws = bits(with_workspace(W, S, g, x, 24, n, k))
    first = bits(noalloc(W, S, g, x, 24, n, k))
    second = bits(noalloc(W, S, g, x, 24, n, k))
    torch.cuda.synchronize()
    assert np.array_equal(first, y_ws) and np.array_equal(second, y_ws)
    rows = np.arange(0, n, 61)
    ref, a = oracle.gemv(p.w.packed, p.w.scales, p.w.g, xb, rows=rows)
    check_single(first[:, rows], ref, a, "noalloc M=24 vs oracle (sampled rows)")


def test_consecutive_shapes_share_the_scratch():
    # a split-heavy shape, then a small one, then the first again: each call starts from the
    # flags the previous one left and must still be exact
    rng = np.random.default_rng(7)
    cases = []
    for n, k in ((37420, 1024), (256, 512), (37420, 1024)):
        w = synth.Weight(n, k, rng.integers(0, 256, (n, k // 2), dtype=np.uint8),
                         rng.integers(0x20, 0x50, (n, k // 16), dtype=np.uint8),
                         float(np.float32(0.37)))
        xb = oracle.bf16_rne(rng.standard_normal((4, k)))
        cases.append((w, xb))
    outs = []
    for w, xb in cases:
        W, S, g = dev_weight(w)
        outs.append((w, xb, bits(noalloc(W, S, g, dev_x(xb), 4, w.n, w.k)),
                     bits(with_workspace(W, S, g, dev_x(xb), 4, w.n, w.k))))
    torch.cuda.synchronize()
    for i, (w, xb, y_na, y_ws) in enumerate(outs):
        rows = np.arange(0, w.n, 97)
        ref, a = oracle.gemv(w.packed, w.scales, w.g, xb, rows=rows)
        check_single(y_na[:, rows], ref, a, f"case {i} vs oracle (sampled rows)")
        assert np.array_equal(y_na, y_ws), f"case {i}: noalloc differs from nvfp4_gemv"


def test_rejects_bad_arguments_before_launch():
    L = nv.lib()
    h = torch.cuda.current_stream().cuda_stream
    buf = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    p = buf.data_ptr()
    assert L.nvfp4_gemv_noalloc(p, p, 1.0, p, 64, p, 64, 129, 64, 64, h) == -3
    assert L.nvfp4_gemv_noalloc(p, p, 1.0, p + 8, 64, p, 64, 1, 64, 64, h) == -4
    assert L.nvfp4_gemv_noalloc(p, p, 1.0, p, 64, p, 64, 1, 64, 48, h) == -2
