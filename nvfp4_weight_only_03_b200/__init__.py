"""Weight-only NVFP4 GEMV for NVIDIA B200 -- thin Python binding over the C ABI in include/nvfp4.h.

Every step of the computation runs in the CUDA library (libnvfp4gemv.so, built in-tree for
sm_100a).  This module only marshals torch tensors into device pointers, sizes and the current
CUDA stream; PyTorch provides memory and streams.  There is no fallback: if the library is
missing or the device is not a B200 the calls raise.

    y = gemv(w, s, g, x)                      # y[m][n] = bf16(g * sum_k e2m1(w) e4m3(s) x)
    o = gemv_dual(wg, sg, gg, wu, su, gu, x)  # o = bf16(silu(gate) * up)
    k_, v_ = gemv_multi([(wk, sk, gk), (wv, sv, gv)], x)  # several outputs sharing x, one pass
    q = gemv(w, s, g, x, prologue=AddRmsNorm(r, gamma, 1e-6, h))  # x' = rmsnorm(x + r) first
    o, d = gemv_chain([ChainOp.dual(wg, sg, gg, wu, su, gu, x=x),    # one launch: gate_up ...
                       ChainOp.single([(wd, sd, gd)], x_from=0)])   # ... feeding down

w: uint8 [N][K/2] packed e2m1 (low nibble = even k), s: uint8 [N][K/16] e4m3 scale codes,
g: float global scale, x: bfloat16 [M][K] (M = 1..128, one kernel pass per 8 rows; row stride
may exceed K).
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

_LIB_PATH = _build.LIB
_lib = None

STATUS = {0: "NVFP4_OK", -1: "NVFP4_ERR_NULL", -2: "NVFP4_ERR_SHAPE", -3: "NVFP4_ERR_ROWS",
          -4: "NVFP4_ERR_ALIGN", -5: "NVFP4_ERR_ARCH", -6: "NVFP4_ERR_LAUNCH",
          -7: "NVFP4_ERR_WORKSPACE", -8: "NVFP4_ERR_ALIAS"}
MAX_ROWS = 128
PASS_ROWS = 8
MAX_OUTPUTS = 4
GROUP = 16
FLAG_PREFETCH_WEIGHTS = 1
FLAG_WIDE_TENSOR = 2
CHAIN_MAX_OPS = 16
OP_SINGLE, OP_DUAL = 0, 1


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class Output(ctypes.Structure):
    """nvfp4_output_t: one output of nvfp4_gemv_multi."""
    _fields_ = [("w", ctypes.c_void_p), ("s", ctypes.c_void_p), ("global_scale", ctypes.c_float),
                ("y", ctypes.c_void_p), ("ldy", ctypes.c_int64), ("n", ctypes.c_int64)]


class ChainOpStruct(ctypes.Structure):
    """nvfp4_chain_op_t: one operation of nvfp4_gemv_chain."""
    _fields_ = [("kind", ctypes.c_int32), ("outputs", ctypes.c_int32),
                ("out", Output * MAX_OUTPUTS), ("x", ctypes.c_void_p), ("ldx", ctypes.c_int64),
                ("k", ctypes.c_int64), ("x_from", ctypes.c_int32)]


class Prologue(ctypes.Structure):
    """nvfp4_prologue_t: the transform of x a call applies before its GEMV."""
    _fields_ = [("kind", ctypes.c_int32), ("eps", ctypes.c_float),
                ("residual", ctypes.c_void_p), ("ld_residual", ctypes.c_int64),
                ("gamma", ctypes.c_void_p),
                ("residual_out", ctypes.c_void_p), ("ld_residual_out", ctypes.c_int64),
                ("gate", ctypes.c_void_p), ("ld_gate", ctypes.c_int64),
                ("group", ctypes.c_int32)]


PROLOGUE_NONE, PROLOGUE_ADD_RMSNORM, PROLOGUE_SIGMOID_GATE, PROLOGUE_GATED_RMSNORM = 0, 1, 2, 3


def _rows_arg(t: torch.Tensor, m: int, k: int, name: str):
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16")
    if t.dim() == 1:
        t = t.unsqueeze(0)
    if t.dim() != 2 or t.shape != (m, k) or t.stride(1) != 1:
        raise ValueError(f"{name} must be [{m}][{k}] with unit inner stride")
    return t, t.stride(0) if m > 1 else k


class AddRmsNorm:
    """Prologue: h = bf16(x + residual), x' = bf16(h / sqrt(mean(h^2) + eps) * gamma); h is
    written to residual_out when given (it may not overlap x, residual, gamma or y)."""

    def __init__(self, residual: torch.Tensor, gamma: torch.Tensor, eps: float = 1e-6,
                 residual_out: torch.Tensor = None):
        self.residual, self.gamma, self.eps, self.residual_out = residual, gamma, eps, residual_out

    def struct(self, m: int, k: int) -> Prologue:
        r, ldr = _rows_arg(self.residual, m, k, "residual")
        if self.gamma.dtype != torch.bfloat16 or self.gamma.shape != (k,) or \
                not self.gamma.is_contiguous():
            raise ValueError(f"gamma must be contiguous bfloat16 [{k}]")
        p = Prologue(kind=PROLOGUE_ADD_RMSNORM, eps=float(self.eps), residual=r.data_ptr(),
                     ld_residual=ldr, gamma=self.gamma.data_ptr())
        if self.residual_out is not None:
            h, ldh = _rows_arg(self.residual_out, m, k, "residual_out")
            p.residual_out, p.ld_residual_out = h.data_ptr(), ldh
        return p


class GatedRmsNorm:
    """Prologue for an fp32 x (pass x as float32): every group of `group` channels is normalised
    alone, x' = bf16(x / sqrt(mean_group(x^2) + eps) * gamma[k % group] * silu(gate)).
    group % 128 == 0, group <= 512; gamma is bfloat16 [group], gate bfloat16 [M][K]."""

    x_dtype = torch.float32

    def __init__(self, gate: torch.Tensor, gamma: torch.Tensor, group: int, eps: float = 1e-6):
        self.gate, self.gamma, self.group, self.eps = gate, gamma, group, eps

    def struct(self, m: int, k: int) -> Prologue:
        t, ldt = _rows_arg(self.gate, m, k, "gate")
        if self.gamma.dtype != torch.bfloat16 or self.gamma.shape != (self.group,) or \
                not self.gamma.is_contiguous():
            raise ValueError(f"gamma must be contiguous bfloat16 [{self.group}]")
        return Prologue(kind=PROLOGUE_GATED_RMSNORM, eps=float(self.eps), gate=t.data_ptr(),
                        ld_gate=ldt, gamma=self.gamma.data_ptr(), group=int(self.group))


class SigmoidGate:
    """Prologue: x' = bf16(x * sigmoid(gate))."""

    def __init__(self, gate: torch.Tensor):
        self.gate = gate

    def struct(self, m: int, k: int) -> Prologue:
        t, ldt = _rows_arg(self.gate, m, k, "gate")
        return Prologue(kind=PROLOGUE_SIGMOID_GATE, gate=t.data_ptr(), ld_gate=ldt)


class PackInfo(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int64), ("k", ctypes.c_int64),
                ("weight_bytes", ctypes.c_int64), ("scale_bytes", ctypes.c_int64),
                ("weight_row_bytes", ctypes.c_int64), ("scale_row_bytes", ctypes.c_int64),
                ("group", ctypes.c_int32), ("max_rows", ctypes.c_int32),
                ("align_bytes", ctypes.c_int32), ("layout_version", ctypes.c_int32)]


def library_path() -> str:
    return _LIB_PATH


def lib():
    """The loaded C library (ctypes).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m nvfp4_weight_only_03_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        i64, vp, c_int, sz = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.nvfp4_pack_info.argtypes = [i64, i64, ctypes.POINTER(PackInfo)]
        L.nvfp4_workspace_bytes.argtypes = [ctypes.POINTER(sz)]
        L.nvfp4_gemv.argtypes = [vp, vp, ctypes.c_float, vp, i64, vp, i64, c_int, i64, i64,
                                 vp, sz, vp]
        L.nvfp4_gemv_dual.argtypes = [vp, vp, ctypes.c_float, vp, vp, ctypes.c_float, vp, i64,
                                      vp, i64, c_int, i64, i64, vp, sz, vp]
        L.nvfp4_gemv_ex.argtypes = [vp, vp, ctypes.c_float, vp, i64, vp, i64, c_int, i64, i64,
                                    vp, sz, ctypes.c_uint32, vp]
        L.nvfp4_gemv_dual_ex.argtypes = [vp, vp, ctypes.c_float, vp, vp, ctypes.c_float, vp, i64,
                                         vp, i64, c_int, i64, i64, vp, sz, ctypes.c_uint32, vp]
        L.nvfp4_gemv_noalloc.argtypes = [vp, vp, ctypes.c_float, vp, i64, vp, i64, c_int, i64,
                                         i64, vp]
        L.nvfp4_gemv_multi.argtypes = [ctypes.POINTER(Output), c_int, vp, i64, c_int, i64, vp,
                                       sz, ctypes.c_uint32, vp]
        pp = ctypes.POINTER(Prologue)
        L.nvfp4_gemv_pro.argtypes = [pp] + L.nvfp4_gemv_ex.argtypes
        L.nvfp4_gemv_dual_pro.argtypes = [pp] + L.nvfp4_gemv_dual_ex.argtypes
        L.nvfp4_gemv_multi_pro.argtypes = [pp] + L.nvfp4_gemv_multi.argtypes
        L.nvfp4_workspace_error.argtypes = [vp, sz, vp, ctypes.POINTER(ctypes.c_int32)]
        L.nvfp4_workspace_bytes_wide.argtypes = [i64, i64, c_int, ctypes.POINTER(sz)]
        cp = ctypes.POINTER(ChainOpStruct)
        L.nvfp4_chain_workspace_bytes.argtypes = [cp, c_int, c_int, ctypes.POINTER(sz)]
        L.nvfp4_gemv_chain.argtypes = [cp, c_int, c_int, vp, sz, ctypes.c_uint32, vp]
        L.nvfp4_gemv_chain_unsignalled.argtypes = [cp, c_int, c_int, vp, sz, i64, vp]
        L.nvfp4_gemv_chain_owner_wait.argtypes = [cp, c_int, c_int, vp, sz, i64, vp]
        L.nvfp4_status_string.argtypes = [c_int]
        L.nvfp4_status_string.restype = ctypes.c_char_p
        for f in (L.nvfp4_pack_info, L.nvfp4_workspace_bytes, L.nvfp4_gemv, L.nvfp4_gemv_dual,
                  L.nvfp4_gemv_ex, L.nvfp4_gemv_dual_ex, L.nvfp4_gemv_noalloc,
                  L.nvfp4_gemv_multi, L.nvfp4_workspace_error, L.nvfp4_workspace_bytes_wide,
                  L.nvfp4_gemv_pro, L.nvfp4_gemv_dual_pro, L.nvfp4_gemv_multi_pro,
                  L.nvfp4_chain_workspace_bytes, L.nvfp4_gemv_chain,
                  L.nvfp4_gemv_chain_unsignalled, L.nvfp4_gemv_chain_owner_wait):
            f.restype = c_int
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise Nvfp4Error(status, where)


def pack_info(n: int, k: int) -> dict:
    info = PackInfo()
    _check(lib().nvfp4_pack_info(n, k, ctypes.byref(info)), "nvfp4_pack_info")
    return {name: getattr(info, name) for name, _ in PackInfo._fields_}


def workspace_bytes() -> int:
    b = ctypes.c_size_t()
    _check(lib().nvfp4_workspace_bytes(ctypes.byref(b)), "nvfp4_workspace_bytes")
    return int(b.value)


def workspace_bytes_wide(n: int, k: int, m: int) -> int:
    b = ctypes.c_size_t()
    _check(lib().nvfp4_workspace_bytes_wide(n, k, m, ctypes.byref(b)), "nvfp4_workspace_bytes_wide")
    return int(b.value)


# Default workspaces, one per (device, stream, kind): calls on different streams may run at
# the same time, and two calls sharing a workspace at the same time would mix their arrival
# counts and partial sums.  Calls on one stream run in order, so they share one.  The cache
# keeps a reference to each torch stream, so its handle cannot be reused by a new stream while
# the workspace is in the cache.
_workspaces: dict = {}


def _device_of(device) -> torch.device:
    return torch.device("cuda", torch.cuda.current_device() if device is None else
                        torch.device(device).index or 0)


def _stream_obj(stream, dev):
    if stream is None:
        return torch.cuda.current_stream(dev)
    if hasattr(stream, "cuda_stream"):
        return stream
    return torch.cuda.ExternalStream(int(stream), device=dev)


def _cached_workspace(kind: str, need: int, device, stream) -> torch.Tensor:
    dev = _device_of(device)
    st = _stream_obj(stream, dev)
    key = (dev, st.cuda_stream, kind)
    ent = _workspaces.get(key)
    if ent is None or ent[0].numel() < need:
        # allocated (and zero-filled) on the stream that uses it: when a grown workspace
        # replaces it, the caching allocator reuses the old block only in that stream's order
        with torch.cuda.device(dev), torch.cuda.stream(st):
            ws = torch.zeros(need, dtype=torch.uint8, device=dev)
        ent = (ws, st)
        _workspaces[key] = ent
    return ent[0]


def workspace(device=None, stream=None) -> torch.Tensor:
    """The zero-filled default workspace of (device, stream): cached, one per stream, so calls
    on different streams never share one."""
    return _cached_workspace("plain", workspace_bytes(), device, stream)


def workspace_error(ws: torch.Tensor, stream=None) -> int:
    err = ctypes.c_int32()
    st = _stream(stream)
    _check(lib().nvfp4_workspace_error(ws.data_ptr(), ws.numel(), st, ctypes.byref(err)),
           "nvfp4_workspace_error")
    return int(err.value)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _weight_args(w: torch.Tensor, s: torch.Tensor):
    if w.dtype != torch.uint8 or s.dtype != torch.uint8:
        raise TypeError("w and s must be uint8")
    if w.dim() != 2 or s.dim() != 2 or not w.is_contiguous() or not s.is_contiguous():
        raise ValueError("w [N][K/2] and s [N][K/16] must be contiguous 2-D tensors")
    n, k = w.shape[0], w.shape[1] * 2
    if s.shape[0] != n or s.shape[1] * 16 != k:
        raise ValueError(f"scale shape {tuple(s.shape)} does not match weight {tuple(w.shape)}")
    return n, k


def _x_args(x: torch.Tensor, k: int, dtype=torch.bfloat16):
    if x.dtype != dtype:
        raise TypeError(f"x must be {dtype}")
    if x.dim() == 1:
        x = x.unsqueeze(0)
    if x.dim() != 2 or x.shape[1] != k or x.stride(1) != 1:
        raise ValueError(f"x must be [M][{k}] with unit inner stride")
    return x, x.shape[0], x.stride(0) if x.shape[0] > 1 else k


def _out(y, m, n, x):
    if y is None:
        y = torch.empty((m, n), dtype=torch.bfloat16, device=x.device)
    if y.dtype != torch.bfloat16 or y.dim() != 2 or y.shape != (m, n) or y.stride(1) != 1:
        raise ValueError(f"y must be bfloat16 [{m}][{n}] with unit inner stride")
    return y, y.stride(0) if m > 1 else n


def wide_workspace(n: int, k: int, m: int, device=None, stream=None) -> torch.Tensor:
    """The default workspace of (device, stream) for a wide_tensor or prologue call of this
    shape (grown when a larger one is needed)."""
    return _cached_workspace("wide", workspace_bytes_wide(n, k, m), device, stream)


def _check_error(ws: torch.Tensor, stream, where: str):
    """Opt-in check after a call: synchronises the stream and raises if a bounded wait in the
    call's kernels gave up (the results are then invalid)."""
    err = workspace_error(ws, stream)
    if err != 0:
        raise RuntimeError(f"{where}: a bounded wait gave up (workspace error word {err}); "
                           "the results are invalid")


def gemv(w: torch.Tensor, s: torch.Tensor, g: float, x: torch.Tensor, y: torch.Tensor = None,
         ws: torch.Tensor = None, stream=None, prefetch_weights: bool = False,
         wide_tensor: bool = False, prologue=None, check: bool = False) -> torch.Tensor:
    """y[m][n] = bf16(g * sum_k e2m1(w[n][k]) * e4m3(s[n][k/16]) * x[m][k]) on the GPU.

    prefetch_weights: stream w and s before earlier work on the stream has finished
    (programmatic dependent launch); only valid when that work does not write w or s.
    wide_tensor: calls of 9..128 rows run on the tensor-core tier (one pass over the weights;
    rows invariant over 9..128, equal to 1..8-row calls within the tolerance).
    prologue: AddRmsNorm or SigmoidGate, applied to x inside the call (its x' lives in the
    workspace, so a caller's ws must hold workspace_bytes_wide(n, k, m)).
    ws: the workspace; by default the cached one of (x's device, stream).
    check: synchronise after the call and raise if a bounded wait in its kernels gave up."""
    n, k = _weight_args(w, s)
    x, m, ldx = _x_args(x, k, getattr(prologue, "x_dtype", torch.bfloat16))
    pro = None if prologue is None else prologue.struct(m, k)
    y, ldy = _out(y, m, n, x)
    if ws is None:
        ws = wide_workspace(n, k, m, x.device, stream) if (wide_tensor or pro) else \
            workspace(x.device, stream)
    flags = (FLAG_PREFETCH_WEIGHTS if prefetch_weights else 0) | \
        (FLAG_WIDE_TENSOR if wide_tensor else 0)
    args = (w.data_ptr(), s.data_ptr(), float(g), x.data_ptr(), ldx, y.data_ptr(), ldy, m, n, k,
            ws.data_ptr(), ws.numel(), flags, _stream(stream))
    if pro is None:
        st = lib().nvfp4_gemv_ex(*args)
    else:
        st = lib().nvfp4_gemv_pro(ctypes.byref(pro), *args)
    _check(st, "nvfp4_gemv")
    if check:
        _check_error(ws, stream, "nvfp4_gemv")
    return y


def gemv_noalloc(w: torch.Tensor, s: torch.Tensor, g: float, x: torch.Tensor,
                 y: torch.Tensor = None, stream=None) -> torch.Tensor:
    """gemv through nvfp4_gemv_noalloc: the library's own scratch replaces the workspace.

    Calls on one device share that scratch, so they must not overlap in time."""
    n, k = _weight_args(w, s)
    x, m, ldx = _x_args(x, k)
    y, ldy = _out(y, m, n, x)
    st = lib().nvfp4_gemv_noalloc(w.data_ptr(), s.data_ptr(), float(g), x.data_ptr(), ldx,
                                  y.data_ptr(), ldy, m, n, k, _stream(stream))
    _check(st, "nvfp4_gemv_noalloc")
    return y


def gemv_dual(wg: torch.Tensor, sg: torch.Tensor, gg: float, wu: torch.Tensor, su: torch.Tensor,
              gu: float, x: torch.Tensor, y: torch.Tensor = None, ws: torch.Tensor = None,
              stream=None, prefetch_weights: bool = False,
              wide_tensor: bool = False, prologue=None, check: bool = False) -> torch.Tensor:
    """o[m][n] = bf16(silu(gate) * up), gate/up the two NVFP4 GEMVs of the same x.

    wide_tensor: calls of 9..128 rows run gate and up on the tensor-core tier, kept in fp32
    and combined by one final pass.  prologue, ws, check: as for gemv."""
    n, k = _weight_args(wg, sg)
    if _weight_args(wu, su) != (n, k):
        raise ValueError("gate and up weights must have the same shape")
    x, m, ldx = _x_args(x, k, getattr(prologue, "x_dtype", torch.bfloat16))
    pro = None if prologue is None else prologue.struct(m, k)
    y, ldy = _out(y, m, n, x)
    if ws is None:
        ws = wide_workspace(n, k, m, x.device, stream) if (wide_tensor or pro) else \
            workspace(x.device, stream)
    flags = (FLAG_PREFETCH_WEIGHTS if prefetch_weights else 0) | \
        (FLAG_WIDE_TENSOR if wide_tensor else 0)
    args = (wg.data_ptr(), sg.data_ptr(), float(gg), wu.data_ptr(), su.data_ptr(), float(gu),
            x.data_ptr(), ldx, y.data_ptr(), ldy, m, n, k, ws.data_ptr(), ws.numel(), flags,
            _stream(stream))
    if pro is None:
        st = lib().nvfp4_gemv_dual_ex(*args)
    else:
        st = lib().nvfp4_gemv_dual_pro(ctypes.byref(pro), *args)
    _check(st, "nvfp4_gemv_dual")
    if check:
        _check_error(ws, stream, "nvfp4_gemv_dual")
    return y


def gemv_multi(weights, x: torch.Tensor, ys=None, ws: torch.Tensor = None, stream=None,
               prefetch_weights: bool = False, prologue=None, wide_tensor: bool = False,
               check: bool = False) -> list:
    """Several GEMVs sharing x in one pass (nvfp4_gemv_multi): weights is a list of up to
    MAX_OUTPUTS (w, s, g) triples with the same K; returns [y_0, y_1, ...], y_o the GEMV of
    weight o as gemv computes it.  ys: optional preallocated outputs, one per weight.
    prologue: as for gemv, applied once to the shared x.  wide_tensor: 9..128 rows on the
    tensor-core tier, each output bitwise as gemv(..., wide_tensor=True) computes it.
    ws, check: as for gemv."""
    weights = list(weights)
    if not 1 <= len(weights) <= MAX_OUTPUTS:
        raise ValueError(f"1..{MAX_OUTPUTS} weights, got {len(weights)}")
    shapes = [_weight_args(w, s) for w, s, _ in weights]
    k = shapes[0][1]
    if any(kk != k for _, kk in shapes):
        raise ValueError("all weights must have the same K")
    x, m, ldx = _x_args(x, k, getattr(prologue, "x_dtype", torch.bfloat16))
    pro = None if prologue is None else prologue.struct(m, k)
    ys = [None] * len(weights) if ys is None else list(ys)
    if len(ys) != len(weights):
        raise ValueError("one output per weight")
    outs = (Output * len(weights))()
    result = []
    for o, ((w, s, g), (n, _), y) in enumerate(zip(weights, shapes, ys)):
        y, ldy = _out(y, m, n, x)
        result.append(y)
        outs[o].w, outs[o].s, outs[o].global_scale = w.data_ptr(), s.data_ptr(), float(g)
        outs[o].y, outs[o].ldy, outs[o].n = y.data_ptr(), ldy, n
    if ws is None:
        if pro is not None or wide_tensor:
            ws = wide_workspace(max(shapes, key=lambda nk: workspace_bytes_wide(nk[0], k, m))[0],
                                k, m, x.device, stream)
        else:
            ws = workspace(x.device, stream)
    flags = (FLAG_PREFETCH_WEIGHTS if prefetch_weights else 0) | \
        (FLAG_WIDE_TENSOR if wide_tensor else 0)
    args = (outs, len(weights), x.data_ptr(), ldx, m, k, ws.data_ptr(), ws.numel(), flags,
            _stream(stream))
    if pro is None:
        st = lib().nvfp4_gemv_multi(*args)
    else:
        st = lib().nvfp4_gemv_multi_pro(ctypes.byref(pro), *args)
    _check(st, "nvfp4_gemv_multi")
    if check:
        _check_error(ws, stream, "nvfp4_gemv_multi")
    return result


class ChainOp:
    """One operation of gemv_chain: NVFP4 weights sharing an x, which is either a bf16 tensor
    or the result of an earlier operation of the chain (x_from = its index)."""

    def __init__(self, kind, weights, x=None, x_from=None, ys=None):
        if (x is None) == (x_from is None):
            raise ValueError("give exactly one of x and x_from")
        self.kind, self.weights, self.x, self.x_from = kind, list(weights), x, x_from
        self.ys = ys

    @classmethod
    def single(cls, weights, x=None, x_from=None, ys=None):
        """1..MAX_OUTPUTS (w, s, g) weights sharing x (as gemv_multi)."""
        return cls(OP_SINGLE, weights, x, x_from, ys)

    @classmethod
    def dual(cls, wg, sg, gg, wu, su, gu, x=None, x_from=None, y=None):
        """o = silu(gate x) * (up x) (as gemv_dual)."""
        return cls(OP_DUAL, [(wg, sg, gg), (wu, su, gu)], x, x_from, None if y is None else [y])


def _chain_structs(ops, m_hint=None):
    """Marshals a list of ChainOp into nvfp4_chain_op_t structs and allocates the outputs."""
    n_ops = len(ops)
    if not 1 <= n_ops <= CHAIN_MAX_OPS:
        raise ValueError(f"1..{CHAIN_MAX_OPS} operations, got {n_ops}")
    m = m_hint
    xs = []
    for i, op in enumerate(ops):
        if op.x_from is not None and not 0 <= int(op.x_from) < i:
            raise ValueError(f"operation {i}: x_from must name an earlier operation")
        if op.x is not None:
            k = _weight_args(*op.weights[0][:2])[1]
            x, mm, ldx = _x_args(op.x, k)
            if m is not None and mm != m:
                raise ValueError("every x of a chain must have the same number of rows")
            m = mm
            xs.append((x, ldx))
        else:
            xs.append((None, 0))
    if m is None:
        raise ValueError("the first operation needs an x")
    arr = (ChainOpStruct * n_ops)()
    results, keep = [], []
    for i, (op, (x, ldx)) in enumerate(zip(ops, xs)):
        shapes = [_weight_args(w, s) for w, s, _ in op.weights]
        k = shapes[0][1]
        if any(kk != k for _, kk in shapes):
            raise ValueError(f"operation {i}: all weights must have the same K")
        c = arr[i]
        c.kind, c.k = op.kind, k
        c.x_from = -1 if op.x_from is None else int(op.x_from)
        if x is not None:
            c.x, c.ldx = x.data_ptr(), ldx
            keep.append(x)
        n_out = 1 if op.kind == OP_DUAL else len(op.weights)
        c.outputs = n_out
        dev = x.device if x is not None else results[op.x_from][0].device
        ys = op.ys if op.ys is not None else [None] * n_out
        outs = []
        for o in range(n_out):
            y, ldy = _out(ys[o], m, shapes[o][0], torch.empty(0, device=dev))
            outs.append(y)
            c.out[o].y, c.out[o].ldy, c.out[o].n = y.data_ptr(), ldy, shapes[o][0]
        for j, (w, s, g) in enumerate(op.weights):
            c.out[j].w, c.out[j].s, c.out[j].global_scale = w.data_ptr(), s.data_ptr(), float(g)
            if op.kind == OP_DUAL and j == 1:
                c.out[j].n = shapes[1][0]
        results.append(outs)
    return arr, m, results, keep


def chain_workspace_bytes(ops, m: int = None) -> int:
    arr, m, _, _ = _chain_structs(ops, m)
    b = ctypes.c_size_t()
    _check(lib().nvfp4_chain_workspace_bytes(arr, len(ops), m, ctypes.byref(b)),
           "nvfp4_chain_workspace_bytes")
    return int(b.value)


class Chain:
    """A chain marshalled once for repeated launches (a serving loop's fixed plan): the ChainOp
    list's pointers, shapes and outputs are fixed at construction; every call enqueues the whole
    chain (nvfp4_gemv_chain) on `stream` and returns the outputs, as gemv_chain does."""

    def __init__(self, ops, ws: torch.Tensor = None, stream=None, prefetch_weights: bool = False):
        ops = list(ops)
        self._arr, self.m, results, self._keep = _chain_structs(ops)
        self._count = len(ops)
        self._keep_ops = ops
        b = ctypes.c_size_t()
        _check(lib().nvfp4_chain_workspace_bytes(self._arr, self._count, self.m, ctypes.byref(b)),
               "nvfp4_chain_workspace_bytes")
        self.workspace_bytes = int(b.value)
        dev = results[0][0].device
        self.ws = ws if ws is not None else _cached_workspace("chain", self.workspace_bytes, dev,
                                                              stream)
        if self.ws.numel() < self.workspace_bytes:
            raise ValueError(f"workspace of {self.ws.numel()} bytes, need {self.workspace_bytes}")
        self.flags = FLAG_PREFETCH_WEIGHTS if prefetch_weights else 0
        self.outputs = [r[0] if len(r) == 1 else r for r in results]

    def __call__(self, stream=None, check: bool = False) -> list:
        st = lib().nvfp4_gemv_chain(self._arr, self._count, self.m, self.ws.data_ptr(),
                                    self.ws.numel(), self.flags, _stream(stream))
        _check(st, "nvfp4_gemv_chain")
        if check:
            _check_error(self.ws, stream, "nvfp4_gemv_chain")
        return self.outputs


def gemv_chain(ops, ws: torch.Tensor = None, stream=None, prefetch_weights: bool = False,
               check: bool = False) -> list:
    """Runs the ChainOp list in one persistent launch per 8-row pass (nvfp4_gemv_chain).
    Returns, per operation, its output (a tensor) or, for a single operation with several
    weights, the list of its outputs.  Each is bitwise what gemv_multi / gemv_dual gives for
    the same x.  ws, check: as for gemv (the default workspace is grown to the chain's size)."""
    return Chain(ops, ws=ws, stream=stream, prefetch_weights=prefetch_weights)(stream, check)

