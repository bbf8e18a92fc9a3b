"""C ABI checks that need no GPU: the library loads, exports every function include/nvfp4.h
declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re
import subprocess

import pytest

from conftest import ROOT, cuda_ok
import nvfp4_weight_only_03_b200 as nv
from nvfp4_weight_only_03_b200 import build as nvbuild

HEADER = os.path.join(ROOT, "include", "nvfp4.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(nvfp4_\w+)\s*\(", text, re.M)))


@pytest.fixture(scope="module")
def L():
    nvbuild.build()
    return nv.lib()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("nvfp4_pack_info", "nvfp4_gemv", "nvfp4_gemv_dual", "nvfp4_gemv_multi",
                     "nvfp4_workspace_bytes", "nvfp4_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol(L):
    out = subprocess.check_output(["nm", "-D", "--defined-only", nv.library_path()], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        getattr(L, n)  # resolvable through ctypes


def test_library_targets_sm100a_only(L):
    # the build flags pin the architecture; the ELF carries a CUDA fatbin section
    assert "arch=compute_100a,code=sm_100a" in " ".join(nvbuild.NVCC_FLAGS)
    out = subprocess.check_output(["readelf", "-S", nv.library_path()], text=True)
    assert ".nv_fatbin" in out


def test_pack_info():
    info = nv.pack_info(10240, 5120)
    assert info["weight_bytes"] == 10240 * 2560
    assert info["scale_bytes"] == 10240 * 320
    assert info["weight_row_bytes"] == 2560 and info["scale_row_bytes"] == 320
    assert info["group"] == 16 and info["max_rows"] == 128
    assert info["align_bytes"] == 16 and info["layout_version"] == 1
    for bad in ((10, 48), (-1, 32), (4, -32)):
        with pytest.raises(nv.Nvfp4Error) as e:
            nv.pack_info(*bad)
        assert e.value.status == -2
    assert nv.lib().nvfp4_pack_info(1, 32, None) == -1


def test_status_strings(L):
    for code, name in nv.STATUS.items():
        assert L.nvfp4_status_string(code).decode() == name
    assert L.nvfp4_status_string(12345).decode() == "NVFP4_ERR_UNKNOWN"


# Fake, never-dereferenced addresses: every case below is rejected by the host checks, which
# run before any CUDA call, so the pointers are only inspected for alignment / NULL.
A16 = 0x10000


def call(L, m=1, n=64, k=64, w=A16, s=A16, x=A16, ldx=None, y=A16, ldy=None, ws=A16,
         wsb=1 << 30):
    ldx = k if ldx is None else ldx
    ldy = n if ldy is None else ldy
    return L.nvfp4_gemv(w, s, 1.0, x, ldx, y, ldy, m, n, k, ws, wsb, None)


def call_dual(L, m=1, n=64, k=64, wu=A16, su=A16, **kw):
    return L.nvfp4_gemv_dual(A16, A16, 1.0, wu, su, 1.0, A16, k, A16, n, m, n, k, A16, 1 << 30,
                             None)


@pytest.mark.parametrize("kw,status", [
    (dict(m=129), -3), (dict(m=-1), -3),
    (dict(k=48), -2), (dict(k=-32), -2), (dict(n=-1), -2),
    (dict(ldx=32), -2), (dict(ldy=10), -2),
    (dict(w=None), -1), (dict(s=None), -1), (dict(x=None), -1), (dict(y=None), -1),
    (dict(w=A16 + 8), -4), (dict(x=A16 + 8), -4), (dict(s=A16 + 1), -4), (dict(y=A16 + 1), -4),
    (dict(k=64, ldx=68), -4),
    (dict(ws=None), -7), (dict(ws=A16 + 4), -7),
])
def test_host_argument_checks(L, kw, status):
    assert call(L, **kw) == status


def test_noops_return_ok_without_cuda(L):
    assert call(L, m=0) == 0
    assert call(L, n=0) == 0
    assert call(L, m=0, w=None, x=None, y=None) == 0


def test_dual_host_checks(L):
    assert L.nvfp4_gemv_dual(A16, A16, 1.0, None, A16, 1.0, A16, 64, A16, 64, 1, 64, 64, A16,
                             1 << 30, None) == -1
    assert L.nvfp4_gemv_dual(A16, A16, 1.0, A16 + 4, A16, 1.0, A16, 64, A16, 64, 1, 64, 64,
                             A16, 1 << 30, None) == -4
    assert L.nvfp4_gemv_dual(A16, A16, 1.0, A16, A16, 1.0, A16, 64, A16, 64, 130, 64, 64, A16,
                             1 << 30, None) == -3


@pytest.mark.skipif(cuda_ok(), reason="only meaningful on a host without a CUDA device")
def test_valid_call_without_device_reports_arch(L):
    assert call(L) == -5
    b = ctypes.c_size_t()
    assert L.nvfp4_workspace_bytes(ctypes.byref(b)) == -5


def test_noalloc_host_checks(L):
    assert L.nvfp4_gemv_noalloc(A16, A16, 1.0, A16, 64, A16, 64, 129, 64, 64, None) == -3
    assert L.nvfp4_gemv_noalloc(A16, A16, 1.0, A16 + 8, 64, A16, 64, 1, 64, 64, None) == -4
    assert L.nvfp4_gemv_noalloc(None, A16, 1.0, A16, 64, A16, 64, 1, 64, 64, None) == -1
    assert L.nvfp4_gemv_noalloc(A16, A16, 1.0, A16, 64, A16, 64, 0, 64, 64, None) == 0
    if not cuda_ok():
        assert L.nvfp4_gemv_noalloc(A16, A16, 1.0, A16, 64, A16, 64, 1, 64, 64, None) == -5


def _outputs(*specs):
    """nvfp4_output_t array from (w, s, g, y, ldy, n) tuples."""
    arr = (nv.Output * len(specs))()
    for o, (w, s, g, y, ldy, n) in enumerate(specs):
        arr[o].w, arr[o].s, arr[o].global_scale = w, s, g
        arr[o].y, arr[o].ldy, arr[o].n = y, ldy, n
    return arr


def test_multi_host_checks(L):
    good = (A16, A16, 1.0, A16, 64, 64)
    ok2 = _outputs(good, good)
    # count out of range, descriptor array missing
    assert L.nvfp4_gemv_multi(ok2, 0, A16, 64, 1, 64, A16, 1 << 30, 0, None) == -2
    assert L.nvfp4_gemv_multi(_outputs(*[good] * 5), 5, A16, 64, 1, 64, A16, 1 << 30, 0,
                              None) == -2
    assert L.nvfp4_gemv_multi(None, 1, A16, 64, 1, 64, A16, 1 << 30, 0, None) == -1
    # every output is vetted like nvfp4_gemv: rows, alignment, null weight, ldy < n, flags
    assert L.nvfp4_gemv_multi(ok2, 2, A16, 64, 129, 64, A16, 1 << 30, 0, None) == -3
    assert L.nvfp4_gemv_multi(_outputs(good, (A16 + 4, A16, 1.0, A16, 64, 64)), 2, A16, 64, 1,
                              64, A16, 1 << 30, 0, None) == -4
    assert L.nvfp4_gemv_multi(_outputs(good, (None, A16, 1.0, A16, 64, 64)), 2, A16, 64, 1, 64,
                              A16, 1 << 30, 0, None) == -1
    assert L.nvfp4_gemv_multi(_outputs(good, (A16, A16, 1.0, A16, 32, 64)), 2, A16, 64, 1, 64,
                              A16, 1 << 30, 0, None) == -2
    assert L.nvfp4_gemv_multi(ok2, 2, A16, 64, 1, 64, A16, 1 << 30, 4, None) == -2
    # nothing to do: M = 0, or every output empty
    assert L.nvfp4_gemv_multi(ok2, 2, A16, 64, 0, 64, A16, 1 << 30, 0, None) == 0
    empty = (A16, A16, 1.0, A16, 64, 0)
    assert L.nvfp4_gemv_multi(_outputs(empty, empty), 2, A16, 64, 1, 64, A16, 1 << 30, 0,
                              None) == 0
    if not cuda_ok():
        assert L.nvfp4_gemv_multi(ok2, 2, A16, 64, 1, 64, A16, 1 << 30, 0, None) == -5


def test_multi_binding_argument_checks():
    import torch
    w = torch.zeros((64, 32), dtype=torch.uint8)
    s = torch.zeros((64, 4), dtype=torch.uint8)
    x = torch.zeros((1, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        nv.gemv_multi([], x)
    with pytest.raises(ValueError):
        nv.gemv_multi([(w, s, 1.0)] * 5, x)
    w2 = torch.zeros((64, 16), dtype=torch.uint8)
    s2 = torch.zeros((64, 2), dtype=torch.uint8)
    with pytest.raises(ValueError):  # K differs between outputs
        nv.gemv_multi([(w, s, 1.0), (w2, s2, 1.0)], x)


def test_wide_tensor_flag_host_checks(L):
    # the flag is accepted; an unknown bit is not
    ex = lambda m, flags: L.nvfp4_gemv_ex(A16, A16, 1.0, A16, 64, A16, 64, m, 64, 64, A16,
                                          1 << 30, flags, None)
    assert ex(0, nv.FLAG_WIDE_TENSOR) == 0
    assert ex(1, 4) == -2
    if not cuda_ok():
        assert ex(16, nv.FLAG_WIDE_TENSOR) == -5
    b = ctypes.c_size_t()
    assert L.nvfp4_workspace_bytes_wide(64, 64, 16, None) == -1
    assert L.nvfp4_workspace_bytes_wide(64, 48, 16, ctypes.byref(b)) == -2
    assert L.nvfp4_workspace_bytes_wide(64, 64, 129, ctypes.byref(b)) == -3
    if not cuda_ok():
        assert L.nvfp4_workspace_bytes_wide(64, 64, 16, ctypes.byref(b)) == -5


# ---- input prologues: host checks (distinct fake addresses so that only the planted overlap
# counts as one)
PX, PY, PR, PG, PH, PT, PW, PWS = (0x100000 * i for i in range(1, 9))


def pro(kind=nv.PROLOGUE_ADD_RMSNORM, eps=1e-6, residual=PR, ld_residual=64, gamma=PG,
        residual_out=PH, ld_residual_out=64, gate=PT, ld_gate=64):
    return nv.Prologue(kind=kind, eps=eps, residual=residual, ld_residual=ld_residual,
                       gamma=gamma, residual_out=residual_out, ld_residual_out=ld_residual_out,
                       gate=gate, ld_gate=ld_gate)


def call_pro(L, p, m=2, n=64, k=64):
    return L.nvfp4_gemv_pro(ctypes.byref(p) if p is not None else None, PW, PW, 1.0, PX, k, PY,
                            n, m, n, k, PWS, 1 << 30, 0, None)


@pytest.mark.parametrize("kw,status", [
    (dict(kind=7), -2), (dict(kind=-1), -2),
    (dict(eps=-1.0), -2), (dict(eps=float("nan")), -2), (dict(eps=float("inf")), -2),
    (dict(residual=None), -1), (dict(gamma=None), -1),
    (dict(ld_residual=32), -2), (dict(ld_residual_out=32), -2),
    (dict(ld_residual=68), -4), (dict(residual=PR + 8), -4), (dict(gamma=PG + 8), -4),
    (dict(residual_out=PH + 8), -4), (dict(ld_residual_out=72 + 4), -4),
    (dict(residual_out=PX), -8),            # h written over x
    (dict(residual_out=PR + 64), -8),       # ... over the residual's second row
    (dict(residual_out=PG - 32), -8),       # ... over gamma
    (dict(residual_out=PY + 2 * 64), -8),   # ... over y's second row
    (dict(residual=PY), -8),                # y written over the residual
    (dict(kind=nv.PROLOGUE_SIGMOID_GATE, gate=None), -1),
    (dict(kind=nv.PROLOGUE_SIGMOID_GATE, ld_gate=8), -2),
    (dict(kind=nv.PROLOGUE_SIGMOID_GATE, gate=PT + 2), -4),
    (dict(kind=nv.PROLOGUE_SIGMOID_GATE, gate=PY), -8),
])
def test_prologue_host_checks(L, kw, status):
    assert call_pro(L, pro(**kw)) == status


def test_prologue_valid_calls_and_noops(L):
    # no prologue or kind NONE is the plain call; a gate prologue ignores the norm fields
    expect = 0 if cuda_ok() else -5
    for p in (None, pro(kind=nv.PROLOGUE_NONE, residual=None, gamma=None),
              pro(), pro(residual_out=None),
              pro(kind=nv.PROLOGUE_SIGMOID_GATE, residual=None, gamma=None, eps=-5.0)):
        if not cuda_ok():
            assert call_pro(L, p) == expect
    # M == 0: nothing is read; the kind and eps are still checked
    assert call_pro(L, pro(residual=None, gamma=None), m=0) == 0
    assert call_pro(L, pro(kind=9), m=0) == -2
    # the tensors of the prologue stay clear of x where x's rows are strided past K
    assert call_pro(L, pro(residual_out=PX + 2 * 64 * 2), m=1) == (0 if cuda_ok() else -5)


def test_dual_and_multi_prologue_host_checks(L):
    p = pro(residual_out=PY)
    st = L.nvfp4_gemv_dual_pro(ctypes.byref(p), PW, PW, 1.0, PW, PW, 1.0, PX, 64, PY, 64, 2, 64,
                               64, PWS, 1 << 30, 0, None)
    assert st == -8
    outs = _outputs((PW, PW, 1.0, PY, 64, 64), (PW, PW, 1.0, PY + 0x10000, 64, 64))
    p2 = pro(residual_out=PY + 0x10000 + 64)  # overlaps the second output
    assert L.nvfp4_gemv_multi_pro(ctypes.byref(p2), outs, 2, PX, 64, 2, 64, PWS, 1 << 30, 0,
                                  None) == -8
    p3 = pro(kind=3)
    assert L.nvfp4_gemv_multi_pro(ctypes.byref(p3), outs, 2, PX, 64, 2, 64, PWS, 1 << 30, 0,
                                  None) == -2
    if not cuda_ok():
        p4 = pro()
        assert L.nvfp4_gemv_multi_pro(ctypes.byref(p4), outs, 2, PX, 64, 2, 64, PWS, 1 << 30, 0,
                                      None) == -5


def test_prologue_binding_argument_checks():
    import torch
    w = torch.zeros((64, 32), dtype=torch.uint8)
    s = torch.zeros((64, 4), dtype=torch.uint8)
    x = torch.zeros((2, 64), dtype=torch.bfloat16)
    r = torch.zeros((2, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):  # gamma of the wrong length
        nv.gemv(w, s, 1.0, x, prologue=nv.AddRmsNorm(r, torch.ones(32, dtype=torch.bfloat16)))
    with pytest.raises(ValueError):  # residual of the wrong shape
        nv.gemv(w, s, 1.0, x, prologue=nv.AddRmsNorm(r[:1], torch.ones(64, dtype=torch.bfloat16)))
    with pytest.raises(TypeError):   # gate not bf16
        nv.gemv(w, s, 1.0, x, prologue=nv.SigmoidGate(torch.zeros((2, 64))))


def gated(group=128, eps=1e-6, gate=PT, ld_gate=256, gamma=PG):
    return nv.Prologue(kind=nv.PROLOGUE_GATED_RMSNORM, eps=eps, gate=gate, ld_gate=ld_gate,
                       gamma=gamma, group=group)


@pytest.mark.parametrize("kw,k,status", [
    (dict(group=64), 256, -2), (dict(group=192), 384, -2), (dict(group=640), 1280, -2),
    (dict(group=256), 384, -2),              # K % G != 0
    (dict(eps=-1.0), 256, -2), (dict(eps=float("nan")), 256, -2),
    (dict(gate=None), 256, -1), (dict(gamma=None), 256, -1),
    (dict(ld_gate=128), 256, -2), (dict(ld_gate=260), 256, -4),
    (dict(gate=PT + 8), 256, -4), (dict(gamma=PG + 8), 256, -4),
])
def test_gated_rmsnorm_host_checks(L, kw, k, status):
    p = gated(**kw)
    if "ld_gate" not in kw:
        p.ld_gate = k
    assert L.nvfp4_gemv_pro(ctypes.byref(p), PW, PW, 1.0, PX, k, PY, 64, 2, 64, k, PWS, 1 << 30,
                            0, None) == status


def test_gated_rmsnorm_valid_call_reaches_the_device(L):
    p = gated()
    expect = 0 if cuda_ok() else -5
    if not cuda_ok():
        assert L.nvfp4_gemv_pro(ctypes.byref(p), PW, PW, 1.0, PX, 256, PY, 64, 2, 64, 256, PWS,
                                1 << 30, 0, None) == expect


# ---- nvfp4_gemv_chain / nvfp4_chain_workspace_bytes: host checks (no CUDA call is reached)

def chain_op(kind=0, outputs=1, n=256, k=256, x=A16, ldx=None, x_from=-1, y=A16, ldy=None,
             w=A16, s=A16, up=None):
    op = nv.ChainOpStruct()
    op.kind, op.outputs, op.k, op.x_from = kind, outputs, k, x_from
    op.x, op.ldx = x, (k if ldx is None else ldx)
    for o in range(min(outputs, nv.MAX_OUTPUTS) if kind == 0 else 2):
        op.out[o].w, op.out[o].s, op.out[o].global_scale = w, s, 1.0
        op.out[o].y, op.out[o].ldy, op.out[o].n = y, (n if ldy is None else ldy), n
    if kind == 1 and up is not None:
        op.out[1].n = up
    return op


def run_chain(L, ops, m=1, ws=A16, wsb=1 << 30, flags=0):
    arr = (nv.ChainOpStruct * max(1, len(ops)))(*ops)
    return L.nvfp4_gemv_chain(arr, len(ops), m, ws, wsb, flags, None)


@pytest.mark.parametrize("ops,kw,status", [
    ([chain_op()], dict(m=0), -3),
    ([chain_op()], dict(m=129), -3),
    ([chain_op()] * 17, {}, -2),                                   # more than 16 operations
    ([chain_op(kind=2)], {}, -2),                                  # unknown kind
    ([chain_op(outputs=0)], {}, -2),
    ([chain_op(outputs=5)], {}, -2),
    ([chain_op(k=128)], {}, -2),                                   # K % 256 != 0
    ([chain_op(x_from=0)], {}, -2),                                # reads itself
    ([chain_op(), chain_op(x_from=2)], {}, -2),                    # reads a later operation
    ([chain_op(n=512), chain_op(k=256, x_from=0)], {}, -2),        # source N != this K
    ([chain_op(outputs=2), chain_op(k=256, x_from=0)], {}, -2),    # source has two outputs
    ([chain_op(y=A16 + 2), chain_op(x_from=0)], {}, -4),           # source y not 16-byte aligned
    ([chain_op(ldy=260), chain_op(x_from=0)], {}, -4),             # source ldy % 8 != 0
    ([chain_op(x=None)], {}, -1),
    ([chain_op(ldx=128)], {}, -2),
    ([chain_op(x=A16 + 8)], {}, -4),
    ([chain_op(w=None)], {}, -1),
    ([chain_op(y=None)], {}, -1),
    ([chain_op(s=A16 + 2)], {}, -4),                               # scales move by TMA
    ([chain_op(kind=1, up=128)], {}, -2),                          # dual: up N != gate N
    ([chain_op()], dict(flags=4), -2),                             # unknown flag
    ([chain_op()], dict(ws=None), -7),
    ([chain_op()], dict(ws=A16 + 4), -7),
])
def test_chain_host_argument_checks(L, ops, kw, status):
    assert run_chain(L, ops, **kw) == status


def test_chain_null_ops_and_workspace_query_checks(L):
    assert L.nvfp4_gemv_chain(None, 1, 1, A16, 1 << 30, 0, None) == -1
    b = ctypes.c_size_t()
    assert L.nvfp4_chain_workspace_bytes(None, 1, 1, ctypes.byref(b)) == -1
    arr = (nv.ChainOpStruct * 1)(chain_op())
    assert L.nvfp4_chain_workspace_bytes(arr, 1, 1, None) == -1
    assert L.nvfp4_chain_workspace_bytes(arr, 0, 1, ctypes.byref(b)) == -2
    assert L.nvfp4_chain_workspace_bytes(arr, 1, 200, ctypes.byref(b)) == -3
    # the test hook checks its limit before anything else
    assert L.nvfp4_gemv_chain_unsignalled(arr, 1, 1, A16, 1 << 30, 0, None) == -2
    assert L.nvfp4_gemv_chain_unsignalled(arr, 1, 1, A16, 1 << 30, 2 * 10 ** 9, None) == -2


@pytest.mark.skipif(cuda_ok(), reason="only meaningful on a host without a CUDA device")
def test_valid_chain_without_device_reports_arch(L):
    assert run_chain(L, [chain_op(), chain_op(n=256, x_from=0)]) == -5


def test_chain_binding_argument_checks():
    t = torch_cpu_bf16((1, 256))
    w = torch_cpu_u8((256, 128))
    s = torch_cpu_u8((256, 16))
    with pytest.raises((ValueError, TypeError)):
        nv.ChainOp.single([(w, s, 1.0)], x=t, x_from=0)          # both x and x_from
    with pytest.raises((ValueError, TypeError)):
        nv._chain_structs([nv.ChainOp.single([(w, s, 1.0)], x_from=0)])  # reads itself


def torch_cpu_bf16(shape):
    import torch
    return torch.zeros(shape, dtype=torch.bfloat16)


def torch_cpu_u8(shape):
    import torch
    return torch.zeros(shape, dtype=torch.uint8)


def test_owner_wait_hook_checks_its_limit(L):
    arr = (nv.ChainOpStruct * 1)(chain_op())
    assert L.nvfp4_gemv_chain_owner_wait(arr, 1, 1, A16, 1 << 30, -1, None) == -2
    assert L.nvfp4_gemv_chain_owner_wait(arr, 1, 1, A16, 1 << 30, 50001, None) == -2
    assert L.nvfp4_gemv_chain_owner_wait(arr, 1, 0, A16, 1 << 30, 0, None) == -3
