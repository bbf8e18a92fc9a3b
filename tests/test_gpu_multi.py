"""nvfp4_gemv_multi through the C ABI against the fp64 oracle: several NVFP4 weights that share
x and K, computed in one pass.

Every output is checked against the oracle's plain GEMV of its own weight under the acceptance
rules (|y_gpu - y_ref| <= 2e-3 * sum_k |w_k x_k| + 1e-6, and within 1 bf16 ulp where the fp32
accumulation cannot reach half an ulp).  Row invariance over M = 1..8 and determinism are
bitwise; a single output is bitwise nvfp4_gemv's result.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import nvfp4_weight_only_03_b200 as nv
from gpu_util import assert_ws_clean, bits, check_single, dev_weight, dev_x

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ws():
    return torch.zeros(nv.workspace_bytes(), dtype=torch.uint8, device="cuda")


def multi(weights, x_bits, ws):
    ys = nv.gemv_multi([dev_weight(w) for w in weights], dev_x(x_bits), ws=ws)
    torch.cuda.synchronize()
    return [bits(y) for y in ys]


def check_outputs(weights, x_bits, ys, where, rows=None):
    for o, (w, y) in enumerate(zip(weights, ys)):
        ref, a = oracle.gemv(w.packed, w.scales, w.g, x_bits, rows=rows)
        got = y if rows is None else y[:, rows]
        check_single(got, ref, a, f"{where}, output {o}")


@pytest.mark.parametrize("name", ["attn_kv", "attn_qgate"])
@pytest.mark.parametrize("m", [1, 8])
def test_attention_pairs_match_the_oracle(name, m, ws):
    # the decode plan's two-output groups: k/v (1024 + 1024 rows) and q/gate (6144 + 6144)
    wl = synth.make(name)
    weights = [p.w for p in wl.projections]
    x = wl.projections[0].x[:m]
    ys = multi(weights, x, ws)
    check_outputs(weights, x, ys, f"{name} M={m}")
    assert_ws_clean(ws)


def ragged_weights(seed=11, k=512):
    # heights that are not multiples of the 128-row unit, one output shorter than a unit
    return [synth.nvfp4_weight(seed, i * 1_000_000, n, k) for i, n in enumerate((200, 77, 1000, 128))]


def test_four_ragged_outputs_every_row_count(ws):
    weights = ragged_weights()
    x = synth.activations(12, 0, 8, 512)
    per_m = {}
    for m in range(1, 9):
        ys = multi(weights, x[:m], ws)
        check_outputs(weights, x[:m], ys, f"ragged M={m}")
        per_m[m] = ys
    # row r of every output is bitwise the same for every M that includes it
    for m in range(1, 8):
        for o in range(len(weights)):
            assert np.array_equal(per_m[m][o], per_m[8][o][:m]), f"output {o}: M={m} vs M=8"
    assert_ws_clean(ws)


def test_deterministic(ws):
    wl = synth.make("attn_kv")
    weights = [p.w for p in wl.projections]
    x = wl.projections[0].x[:4]
    first = multi(weights, x, ws)
    for _ in range(3):
        again = multi(weights, x, ws)
        for a, b in zip(first, again):
            assert np.array_equal(a, b)


def test_single_output_is_nvfp4_gemv(ws):
    # one output runs the same split and arithmetic as nvfp4_gemv: identical bits
    w = synth.nvfp4_weight(13, 0, 3000, 5120)
    x = synth.activations(13, 98, 8, 5120)
    (y_multi,) = multi([w], x, ws)
    W, S, g = dev_weight(w)
    y_single = bits(nv.gemv(W, S, g, dev_x(x), ws=ws))
    torch.cuda.synchronize()
    assert np.array_equal(y_multi, y_single)


def test_empty_output_between_others(ws):
    k = 512
    a = synth.nvfp4_weight(14, 0, 300, k)
    b = synth.nvfp4_weight(14, 10_000_000, 260, k)
    x = synth.activations(14, 4, 3, k)
    W0 = (torch.zeros((0, k // 2), dtype=torch.uint8, device="cuda"),
          torch.zeros((0, k // 16), dtype=torch.uint8, device="cuda"), 1.0)
    ys = nv.gemv_multi([dev_weight(a), W0, dev_weight(b)], dev_x(x), ws=ws)
    torch.cuda.synchronize()
    assert tuple(ys[1].shape) == (3, 0)
    check_outputs([a, b], x, [bits(ys[0]), bits(ys[2])], "outputs around an empty one")


def test_outputs_beyond_one_launch_at_large_k(ws):
    # K = 17408: three 5120-row outputs hold more row groups than one launch can stage x for,
    # so each output runs as nvfp4_gemv would run it -- bitwise equal to that call
    k = 17408
    weights = [synth.nvfp4_weight(15, i * 100_000_000, 5120, k) for i in range(3)]
    x = synth.activations(15, 6, 2, k)
    ys = multi(weights, x, ws)
    rows = np.arange(0, 5120, 37)
    check_outputs(weights, x, ys, "large K", rows=rows)
    for w, y in zip(weights, ys):
        W, S, g = dev_weight(w)
        y1 = bits(nv.gemv(W, S, g, dev_x(x), ws=ws))
        torch.cuda.synchronize()
        assert np.array_equal(y, y1)
    assert_ws_clean(ws)


def test_two_outputs_in_one_launch_at_large_k(ws):
    # K = 17408 with two 5120-row outputs: 80 row groups fit one launch
    k = 17408
    weights = [synth.nvfp4_weight(16, i * 100_000_000, 5120, k) for i in range(2)]
    x = synth.activations(16, 6, 8, k)
    ys = multi(weights, x, ws)
    rows = np.arange(3, 5120, 41)
    check_outputs(weights, x, ys, "large K, one launch", rows=rows)
    assert_ws_clean(ws)
