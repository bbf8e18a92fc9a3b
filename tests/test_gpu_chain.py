"""GPU parity of nvfp4_gemv_chain: several projections in one persistent launch.

Every operation of a chain keeps its own work split, so its result must be bitwise that of the
same call made alone (nvfp4_gemv_multi / nvfp4_gemv_dual on the same x), and the standalone
calls are checked against the fp64 oracle here too.  A dependent operation (x_from) reads the
earlier operation's output; the oracle side of that check runs the whole chain in fp64 itself
(the dual's output rounded to bf16 becomes down's x) and widens down's tolerance by what a
1-ulp difference in each of those x elements can move it.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
import nvfp4_weight_only_03_b200 as nv
from gpu_util import (bits, bf16_bits_of, check_dual, check_single, dev_weight, dev_x,
                      random_weight)

pytestmark = pytest.mark.gpu


def sample_rows(rng, n, count=160):
    return np.unique(np.concatenate([rng.integers(0, n, count), [0, n - 1]]))


def chain_bits(ops, **kw):
    outs = nv.gemv_chain(ops, check=True, **kw)
    torch.cuda.synchronize()
    return [bits(o) if torch.is_tensor(o) else [bits(t) for t in o] for o in outs]


@pytest.fixture(scope="module")
def layer0():
    wl = synth.make("sweep")
    return wl.projections[:4]  # qkv, o, gate_up, down


def layer_ops(projs, m, dev):
    qkv, o, gu, down = projs
    return [nv.ChainOp.single([dev_weight(qkv.w)], x=dev_x(qkv.x[:m])),
            nv.ChainOp.single([dev_weight(o.w)], x=dev_x(o.x[:m])),
            nv.ChainOp.dual(*dev_weight(gu.w), *dev_weight(gu.w_up), x=dev_x(gu.x[:m])),
            nv.ChainOp.single([dev_weight(down.w)], x=dev_x(down.x[:m]))]


@pytest.mark.parametrize("m", [1, 8])
def test_layer_as_one_chain_is_bitwise_the_separate_calls(layer0, m):
    """The sweep's first layer (qkv, o, gate_up dual, down; each its own x) as one launch."""
    qkv, o, gu, down = layer0
    got = chain_bits(layer_ops(layer0, m, "cuda"))
    want = []
    for p in (qkv, o):
        want.append(bits(nv.gemv(*dev_weight(p.w), dev_x(p.x[:m]))))
    want.append(bits(nv.gemv_dual(*dev_weight(gu.w), *dev_weight(gu.w_up), dev_x(gu.x[:m]))))
    want.append(bits(nv.gemv(*dev_weight(down.w), dev_x(down.x[:m]))))
    torch.cuda.synchronize()
    for p, a, b in zip(layer0, got, want):
        assert np.array_equal(a, b), f"{p.name} M={m}: chain differs from the separate call"
    rng = np.random.default_rng(m)
    for p, y in zip(layer0, got):
        rows = sample_rows(rng, p.n)
        if p.dual:
            o_ref, yg, yu, ag, au = oracle.gemv_dual(p.w.packed, p.w.scales, p.w.g, p.w_up.packed,
                                                     p.w_up.scales, p.w_up.g, p.x[:m], rows=rows)
            check_dual(y[:, rows], o_ref, yg, yu, ag, au, f"chain {p.name} M={m}")
        else:
            ref, a = oracle.gemv(p.w.packed, p.w.scales, p.w.g, p.x[:m], rows=rows)
            check_single(y[:, rows], ref, a, f"chain {p.name} M={m}")


def mlp_reference(gu, down, x_bits, rows):
    """fp64 oracle of the chained MLP: o = silu(gate) * up rounded to bf16 is down's x.  Returns
    (y_ref, tolerance) for the sampled down rows: the accumulation bound on down's own sum plus
    sum_k |w_k| times the dual's per-element tolerance (how far the GPU's x may sit from the
    oracle's, rounded up to bf16)."""
    o_ref, yg, yu, ag, au = oracle.gemv_dual(gu.w.packed, gu.w.scales, gu.w.g, gu.w_up.packed,
                                             gu.w_up.scales, gu.w_up.g, x_bits)
    xo = oracle.bf16_rne(o_ref)
    t = oracle.dual_tolerance(yg, yu, ag, au, o_ref)
    # the GPU's x element lies within t of o_ref, and bf16(o_ref) within half an ulp (<= t) of
    # it: 2t bounds their distance; rounded up to a bf16 value, as bf16 bits
    t_bits = oracle.bf16_rne(2 * t * (1 + 2.0 ** -7))
    y_ref, a = oracle.gemv(down.w.packed, down.w.scales, down.w.g, xo, rows=rows)
    _, spread = oracle.gemv(down.w.packed, down.w.scales, abs(down.w.g), t_bits, rows=rows)
    return y_ref, oracle.tolerance(a) + spread, a


@pytest.mark.parametrize("m", [1, 3, 8])
def test_mlp_chain_down_reads_the_dual_output(layer0, m):
    """gate_up -> down in one launch, down's x being the dual's output (x_from)."""
    _, _, gu, down = layer0
    Wd, Sd, gd = dev_weight(down.w)
    ops = [nv.ChainOp.dual(*dev_weight(gu.w), *dev_weight(gu.w_up), x=dev_x(gu.x[:m])),
           nv.ChainOp.single([(Wd, Sd, gd)], x_from=0)]
    o_chain, y_chain = chain_bits(ops)
    # the same two calls made one after the other
    o_sep = nv.gemv_dual(*dev_weight(gu.w), *dev_weight(gu.w_up), dev_x(gu.x[:m]))
    y_sep = nv.gemv(Wd, Sd, gd, o_sep)
    torch.cuda.synchronize()
    assert np.array_equal(o_chain, bits(o_sep)), f"M={m}: chained dual differs"
    assert np.array_equal(y_chain, bits(y_sep)), f"M={m}: chained down differs"
    rows = sample_rows(np.random.default_rng(100 + m), down.n, 96)
    y_ref, tol, a = mlp_reference(gu, down, gu.x[:m], rows)
    y = oracle.bf16_value(y_chain[:, rows])
    lo, hi = oracle.bf16_rounding_interval(y_chain[:, rows])
    dist = np.maximum(0.0, np.maximum(lo - y_ref, y_ref - hi))
    bad = np.argwhere(~(dist <= tol))
    assert bad.size == 0, f"M={m}: {bad.shape[0]} down outputs outside the propagated tolerance"
    if m == 8:
        for r in (0, 5, 7):
            o1, y1 = chain_bits([nv.ChainOp.dual(*dev_weight(gu.w), *dev_weight(gu.w_up),
                                                 x=dev_x(gu.x[r:r + 1])),
                                 nv.ChainOp.single([(Wd, Sd, gd)], x_from=0)])
            assert np.array_equal(o1[0], o_chain[r]) and np.array_equal(y1[0], y_chain[r]), \
                f"row {r}: the chain is not row invariant"


def test_chain_replays_and_rows_beyond_one_pass(layer0):
    """20 rows (three 8-row passes), run twice on one workspace: bitwise the separate calls
    both times (the arrival and completion counts are reset by every launch)."""
    _, _, gu, down = layer0
    rng = np.random.default_rng(7)
    x = bf16_bits_of(rng.standard_normal((20, gu.k)).astype(np.float32))
    Wd, Sd, gd = dev_weight(down.w)
    ops = [nv.ChainOp.dual(*dev_weight(gu.w), *dev_weight(gu.w_up), x=dev_x(x)),
           nv.ChainOp.single([(Wd, Sd, gd)], x_from=0)]
    first = chain_bits(ops)
    second = chain_bits(ops)
    o_sep = nv.gemv_dual(*dev_weight(gu.w), *dev_weight(gu.w_up), dev_x(x))
    y_sep = nv.gemv(Wd, Sd, gd, o_sep)
    torch.cuda.synchronize()
    for run in (first, second):
        assert np.array_equal(run[0], bits(o_sep)) and np.array_equal(run[1], bits(y_sep))


def test_chain_multi_output_ragged_and_strided():
    """A two-output operation, ragged heights, K = 512, a strided x, then an operation reading a
    ragged single output."""
    rng = np.random.default_rng(5)
    wk = random_weight(rng, 200, 512)
    wv = random_weight(rng, 77, 512)
    w2 = random_weight(rng, 1000, 256)
    wa = random_weight(rng, 256, 512)  # feeds wb, whose K is wa's 256 rows
    wb = random_weight(rng, 130, 256)
    x = bf16_bits_of(rng.standard_normal((5, 512)).astype(np.float32))
    x2 = bf16_bits_of(rng.standard_normal((5, 256)).astype(np.float32))
    xs = dev_x(x, ldx=520)
    ops = [nv.ChainOp.single([dev_weight(wk), dev_weight(wv)], x=xs),
           nv.ChainOp.single([dev_weight(w2)], x=dev_x(x2)),
           nv.ChainOp.single([dev_weight(wa)], x=xs),
           nv.ChainOp.single([dev_weight(wb)], x_from=2)]
    got = chain_bits(ops)
    kv = nv.gemv_multi([dev_weight(wk), dev_weight(wv)], xs)
    y2 = nv.gemv(*dev_weight(w2), dev_x(x2))
    ya = nv.gemv(*dev_weight(wa), xs)
    yb = nv.gemv(*dev_weight(wb), ya)
    torch.cuda.synchronize()
    assert np.array_equal(got[0][0], bits(kv[0])) and np.array_equal(got[0][1], bits(kv[1]))
    assert np.array_equal(got[1], bits(y2))
    assert np.array_equal(got[2], bits(ya)) and np.array_equal(got[3], bits(yb))
    for w, y, xx in ((wk, got[0][0], x), (wv, got[0][1], x), (w2, got[1], x2), (wa, got[2], x)):
        ref, a = oracle.gemv(w.packed, w.scales, w.g, xx)
        check_single(y, ref, a, f"chain ragged n={w.n}")


def test_chain_cuts_a_tall_operation_into_row_chunks():
    """K = 17408 and 10,752 rows: more row groups than one launch holds at that K, so the chain
    runs the operation as row chunks, exactly as nvfp4_gemv does."""
    rng = np.random.default_rng(9)
    n, k = 10752, 17408
    w = random_weight(rng, n, k)
    x = bf16_bits_of(rng.standard_normal((2, k)).astype(np.float32))
    got = chain_bits([nv.ChainOp.single([dev_weight(w)], x=dev_x(x))])[0]
    want = bits(nv.gemv(*dev_weight(w), dev_x(x)))
    assert np.array_equal(got, want)
    rows = sample_rows(rng, n, 64)
    ref, a = oracle.gemv(w.packed, w.scales, w.g, x, rows=rows)
    check_single(got[:, rows], ref, a, "chain row chunks")


def test_bounded_wait_gives_up_and_the_device_stays_usable():
    """The test form of the chain never reports the dual's completion: down's CTAs wait 1 ms,
    give up, record error 4 and finish the launch.  A normal chain on a fresh workspace then
    gives the right results."""
    rng = np.random.default_rng(13)
    g = random_weight(rng, 512, 256)
    u = random_weight(rng, 512, 256)
    d = random_weight(rng, 256, 512)
    x = bf16_bits_of(rng.standard_normal((2, 256)).astype(np.float32))
    Wd = dev_weight(d)
    ops = [nv.ChainOp.dual(*dev_weight(g), *dev_weight(u), x=dev_x(x)),
           nv.ChainOp.single([Wd], x_from=0)]
    arr, m, results, keep = nv._chain_structs(ops)
    need = nv.chain_workspace_bytes(ops)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    st = nv.lib().nvfp4_gemv_chain_unsignalled(arr, len(ops), m, ws.data_ptr(), ws.numel(),
                                               1_000_000, stream)
    assert st == 0, nv.STATUS.get(st, st)
    assert nv.workspace_error(ws) == 4
    with pytest.raises(RuntimeError, match="bounded wait"):
        nv._check_error(ws, None, "chain")
    # the device still works: a normal chain on a fresh workspace
    fresh = torch.zeros(need, dtype=torch.uint8, device="cuda")
    o, y = nv.gemv_chain(ops, ws=fresh, check=True)
    o_sep = nv.gemv_dual(*dev_weight(g), *dev_weight(u), dev_x(x))
    y_sep = nv.gemv(*Wd, o_sep)
    torch.cuda.synchronize()
    assert np.array_equal(bits(o), bits(o_sep)) and np.array_equal(bits(y), bits(y_sep))
    o_ref, yg, yu, ag, au = oracle.gemv_dual(g.packed, g.scales, g.g, u.packed, u.scales, u.g, x)
    check_dual(bits(o), o_ref, yg, yu, ag, au, "dual, fresh workspace after a timed-out launch")


def test_chain_argument_checks():
    rng = np.random.default_rng(3)
    w = random_weight(rng, 256, 512)
    W, S, g = dev_weight(w)
    x = dev_x(bf16_bits_of(rng.standard_normal((1, 512)).astype(np.float32)))
    ok = [nv.ChainOp.single([(W, S, g)], x=x)]
    arr, m, _, _ = nv._chain_structs(ok)
    ws = torch.zeros(nv.chain_workspace_bytes(ok), dtype=torch.uint8, device="cuda")
    L = nv.lib()
    s = torch.cuda.current_stream().cuda_stream

    def call(a, count=1, mm=1, flags=0, wsp=ws.data_ptr(), wsn=ws.numel()):
        return L.nvfp4_gemv_chain(a, count, mm, wsp, wsn, flags, s)

    assert call(arr) == 0
    assert call(arr, count=0) == -2 and call(arr, count=17) == -2
    assert call(arr, mm=0) == -3 and call(arr, mm=129) == -3
    assert call(arr, flags=2) == -2
    assert call(arr, wsn=1024) == -7 and call(arr, wsp=None) == -7
    bad = (nv.ChainOpStruct * 1)()
    ctypes.memmove(ctypes.addressof(bad), ctypes.addressof(arr), ctypes.sizeof(bad))
    bad[0].k = 480  # not a multiple of 256
    assert call(bad) == -2
    bad[0].k = 512
    bad[0].x_from = 0  # an operation cannot read its own result
    assert call(bad) == -2
    bad[0].x_from = -1
    bad[0].kind = 7
    assert call(bad) == -2
    torch.cuda.synchronize()


def test_concurrent_streams_with_default_workspaces():
    """The same GEMV issued alternately on two streams that run at the same time, each call on
    its stream's default workspace: every result is bitwise the single-stream one."""
    p = synth.make("inproj").projections[0]
    W, S, g = dev_weight(p.w)
    xs = [dev_x(p.x[i:i + 1]) for i in range(4)]
    want = [bits(nv.gemv(W, S, g, x)) for x in xs]
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    outs = []
    torch.cuda.synchronize()
    for it in range(24):
        st = s1 if it % 2 == 0 else s2
        with torch.cuda.stream(st):
            outs.append((it % 4, nv.gemv(W, S, g, xs[it % 4])))
    torch.cuda.synchronize()
    assert nv.workspace(stream=s1).data_ptr() != nv.workspace(stream=s2).data_ptr()
    for i, y in outs:
        assert np.array_equal(bits(y), want[i]), "a call on a second stream changed the result"
    ref, a = oracle.gemv(p.w.packed, p.w.scales, p.w.g, p.x[:1])
    check_single(want[0], ref, a, "inproj, two streams")
    for st in (s1, s2):
        assert nv.workspace_error(nv.workspace(stream=st), st) == 0


@pytest.mark.parametrize("m", [1, 8])
def test_owner_handoff_is_bitwise_the_normal_path(layer0, m):
    """Owners that do not wait at all (test hook, limit 0) publish their own partial tile and
    leave nearly every cut row group to the last of its later CTAs, which finishes it.  Results
    must be bitwise those of the normal chain, for the layer (single and dual operations) and for
    the MLP pair reading the dual's output, launch after launch on one workspace (a hand-off
    word left non-zero would break the next launch)."""
    from gpu_util import assert_ws_clean
    qkv, o, gu, down = layer0
    Wd, Sd, gd = dev_weight(down.w)
    mlp = [nv.ChainOp.dual(*dev_weight(gu.w), *dev_weight(gu.w_up), x=dev_x(gu.x[:m])),
           nv.ChainOp.single([(Wd, Sd, gd)], x_from=0)]
    stream = torch.cuda.current_stream().cuda_stream
    for chain in (layer_ops(layer0, m, "cuda"), mlp):
        want = chain_bits(chain)
        arr, mm, results, keep = nv._chain_structs(chain)
        ws = torch.zeros(nv.chain_workspace_bytes(chain), dtype=torch.uint8, device="cuda")
        for limit in (0, 0, 0, 50000):
            for r in results:
                for t in r:
                    t.fill_(0)
            st = nv.lib().nvfp4_gemv_chain_owner_wait(arr, len(chain), mm, ws.data_ptr(),
                                                       ws.numel(), limit, stream)
            assert st == 0, nv.STATUS.get(st, st)
            torch.cuda.synchronize()
            assert nv.workspace_error(ws) == 0
            got = [bits(r[0]) if len(r) == 1 else [bits(t) for t in r] for r in results]
            for i, (a, b) in enumerate(zip(got, want)):
                assert np.array_equal(np.asarray(a), np.asarray(b)), \
                    f"operation {i}, owner limit {limit} ns, M={m}: differs from the normal chain"
            assert_ws_clean(ws)
