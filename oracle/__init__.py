"""CPU fp64 oracle for the weight-only NVFP4 GEMV -- TEST INFRASTRUCTURE ONLY.

Only `tests/`, `__graft_entry__.smoke()` and the CPU-baseline leg of `bench.py` may import this
package.  The CUDA library never calls it; the two share no code, headers, tables or constants.
Only the seeded input generator (`synth`) serves both.

The arithmetic is in `oracle.c` (plain C, fp64, decoding each stored code from its bit-layout
definition and summing in increasing k).  This module only marshals numpy arrays.

Parity status of each function (what pins it is listed in the tests named here):
  e2m1 / e4m3 decode ....... pinned: format definitions, exhaustive (tests/test_oracle_formats.py)
  bf16_rne (fp64 -> bf16) .. pinned: exhaustive against fp32 rounding + hand cases (same file)
  gemv ..................... pinned: closed-form sums, brute force, invariants, library matmul
                             cross-check (tests/test_oracle_gemv.py)
  gemv_dual ................ pinned: SiLU closed forms + reduction to gemv (tests/test_oracle_gemv.py)
  add_rmsnorm .............. pinned: hand-derived values, closed forms of the mean square and eps,
                             tie rounding of the residual sum, scale and sign invariants, a
                             50-digit decimal brute force (tests/test_oracle_prologue.py)
  sigmoid_gate ............. pinned: sigmoid(0) = 1/2, saturation, the symmetry
                             sigmoid(t) + sigmoid(-t) = 1, decimal brute force (same file)
  gated_rmsnorm ............ pinned: closed forms of a constant group and of the gate, group
                             independence, scale invariance per group, decimal brute force
                             (same file)
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source (plain C, OpenMP over output rows)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        vp, i64, c_int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        lib.oracle_e2m1.argtypes = [ctypes.c_uint8]
        lib.oracle_e2m1.restype = ctypes.c_double
        lib.oracle_e4m3.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3.restype = ctypes.c_double
        lib.oracle_bf16_value.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_value.restype = ctypes.c_double
        lib.oracle_bf16_rne.argtypes = [ctypes.c_double]
        lib.oracle_bf16_rne.restype = ctypes.c_uint16
        lib.oracle_gemv.argtypes = [vp, vp, ctypes.c_float, vp, i64, c_int, i64, i64, vp, i64,
                                    vp, vp, c_int]
        lib.oracle_gemv.restype = c_int
        lib.oracle_gemv_dual.argtypes = [vp, vp, ctypes.c_float, vp, vp, ctypes.c_float, vp, i64,
                                         c_int, i64, i64, vp, i64, vp, vp, vp, vp, vp, c_int]
        lib.oracle_gemv_dual.restype = c_int
        lib.oracle_add_rmsnorm.argtypes = [vp, i64, vp, i64, vp, ctypes.c_float, c_int, i64, vp,
                                           vp, vp]
        lib.oracle_add_rmsnorm.restype = c_int
        lib.oracle_sigmoid_gate.argtypes = [vp, i64, vp, i64, c_int, i64, vp, vp]
        lib.oracle_sigmoid_gate.restype = c_int
        lib.oracle_gated_rmsnorm.argtypes = [vp, i64, vp, i64, vp, c_int, ctypes.c_float, c_int,
                                             i64, vp, vp]
        lib.oracle_gated_rmsnorm.restype = c_int
        _lib = lib
    return _lib


def e2m1(nibble: int) -> float:
    return float(_load().oracle_e2m1(nibble))


def e4m3(code: int) -> float:
    return float(_load().oracle_e4m3(code))


def e2m1_table() -> np.ndarray:
    return np.array([e2m1(i) for i in range(16)], np.float64)


def e4m3_table() -> np.ndarray:
    return np.array([e4m3(i) for i in range(256)], np.float64)


def bf16_value(bits) -> np.ndarray:
    """bf16 bit patterns -> fp64 values (vectorised)."""
    b = np.asarray(bits, np.uint16)
    # widening a signalling-NaN pattern raises the invalid flag; the result is a NaN either way
    with np.errstate(invalid="ignore"):
        return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_rne(values) -> np.ndarray:
    """fp64 -> bf16 bit patterns, nearest-even, one rounding straight from fp64."""
    v = np.asarray(values, np.float64)
    f = _load().oracle_bf16_rne
    out = np.fromiter((f(float(t)) for t in v.ravel()), np.uint16, count=v.size)
    return out.reshape(v.shape)


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data


def _shape(packed, scales, x):
    n, kh = packed.shape
    k = 2 * kh
    if scales.shape != (n, k // 16):
        raise ValueError("scales must be [n][k/16]")
    if x.ndim != 2 or x.shape[1] != k:
        raise ValueError("x must be [m][k] bf16 bits")
    return n, k, x.shape[0]


def gemv(packed: np.ndarray, scales: np.ndarray, g: float, x: np.ndarray, rows=None,
         threads: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """y[m][j], A[m][j] (fp64) for outputs j = rows (all when None); x is bf16 bits [m][k]."""
    n, k, m = _shape(packed, scales, x)
    packed, pw = _c(packed, np.uint8)
    scales, ps = _c(scales, np.uint8)
    x, px = _c(x, np.uint16)
    if rows is None:
        count, prow, ridx = n, None, None
    else:
        ridx, prow = _c(np.asarray(rows, np.int64), np.int64)
        count = ridx.size
    y = np.zeros((m, count), np.float64)
    a = np.zeros((m, count), np.float64)
    rc = _load().oracle_gemv(pw, ps, g, px, k, m, n, k, prow, count, y.ctypes.data,
                             a.ctypes.data, threads)
    if rc:
        raise ValueError("oracle_gemv rejected its arguments")
    return y, a


def gemv_dual(pg, sg, gg, pu, su, gu, x, rows=None, threads: int = 0):
    """(o, yg, yu, Ag, Au) with o = silu(yg) * yu, all fp64 [m][j]."""
    n, k, m = _shape(pg, sg, x)
    if pu.shape != pg.shape or su.shape != sg.shape:
        raise ValueError("gate and up must have the same shape")
    pg, p1 = _c(pg, np.uint8)
    sg, p2 = _c(sg, np.uint8)
    pu, p3 = _c(pu, np.uint8)
    su, p4 = _c(su, np.uint8)
    x, px = _c(x, np.uint16)
    if rows is None:
        count, prow, ridx = n, None, None
    else:
        ridx, prow = _c(np.asarray(rows, np.int64), np.int64)
        count = ridx.size
    outs = [np.zeros((m, count), np.float64) for _ in range(5)]
    rc = _load().oracle_gemv_dual(p1, p2, gg, p3, p4, gu, px, k, m, n, k, prow, count,
                                  *[o.ctypes.data for o in outs], threads)
    if rc:
        raise ValueError("oracle_gemv_dual rejected its arguments")
    return tuple(outs)


def add_rmsnorm(x, r, gamma, eps: float):
    """Residual add, then RMS norm with gain (x, r: bf16 bits [m][k]; gamma: bf16 bits [k]).
    Returns (h, xn, near): h = bf16(x + r), xn = bf16(h * gamma / sqrt(mean(h^2) + eps)), both
    bf16 bits [m][k], and near[m][k] = 1 where xn's fp64 value lies within a relative 2^-16 of a
    bf16 rounding midpoint."""
    x, px = _c(np.atleast_2d(x), np.uint16)
    r, pr = _c(np.atleast_2d(r), np.uint16)
    gamma, pg = _c(gamma, np.uint16)
    m, k = x.shape
    if r.shape != (m, k) or gamma.shape != (k,):
        raise ValueError("x and r must be [m][k], gamma [k]")
    h = np.zeros((m, k), np.uint16)
    xn = np.zeros((m, k), np.uint16)
    near = np.zeros((m, k), np.uint8)
    rc = _load().oracle_add_rmsnorm(px, k, pr, k, pg, eps, m, k, h.ctypes.data, xn.ctypes.data,
                                    near.ctypes.data)
    if rc:
        raise ValueError("oracle_add_rmsnorm rejected its arguments")
    return h, xn, near


def sigmoid_gate(a, gate):
    """xo = bf16(a * sigmoid(gate)) (bf16 bits [m][k] in and out) and its near-midpoint mask."""
    a, pa = _c(np.atleast_2d(a), np.uint16)
    gate, pg = _c(np.atleast_2d(gate), np.uint16)
    m, k = a.shape
    if gate.shape != (m, k):
        raise ValueError("a and gate must be [m][k]")
    xo = np.zeros((m, k), np.uint16)
    near = np.zeros((m, k), np.uint8)
    rc = _load().oracle_sigmoid_gate(pa, k, pg, k, m, k, xo.ctypes.data, near.ctypes.data)
    if rc:
        raise ValueError("oracle_sigmoid_gate rejected its arguments")
    return xo, near


def gated_rmsnorm(x, z, gamma, group: int, eps: float):
    """Gated RMS norm per group of channels (x: fp32 [m][k]; z: bf16 bits [m][k]; gamma: bf16
    bits [group]).  Returns (xo, near): xo = bf16(x gamma silu(z) / sqrt(mean_group(x^2) + eps))
    as bf16 bits [m][k], and the near-midpoint mask."""
    x, px = _c(np.atleast_2d(x), np.float32)
    z, pz = _c(np.atleast_2d(z), np.uint16)
    gamma, pg = _c(gamma, np.uint16)
    m, k = x.shape
    if z.shape != (m, k) or gamma.shape != (group,):
        raise ValueError("x and z must be [m][k], gamma [group]")
    xo = np.zeros((m, k), np.uint16)
    near = np.zeros((m, k), np.uint8)
    rc = _load().oracle_gated_rmsnorm(px, k, pz, k, pg, group, eps, m, k, xo.ctypes.data,
                                      near.ctypes.data)
    if rc:
        raise ValueError("oracle_gated_rmsnorm rejected its arguments")
    return xo, near


def rounding_slack(xq, near) -> np.ndarray:
    """bf16 bits [m][k]: the larger gap from each near-midpoint element of xq to a bf16
    neighbour (a power of two), zero elsewhere.  The GEMV of these (its absolute-sum output)
    bounds how far y moves when those elements round the other way."""
    xq = np.asarray(xq, np.uint16)
    o = bf16_ordinal(xq)

    def from_ordinal(v):
        v = np.asarray(v, np.int64)
        mag = np.abs(v).astype(np.uint16)
        return np.where(v < 0, mag | 0x8000, mag).astype(np.uint16)

    v = bf16_value(xq)
    gap = np.maximum(np.abs(bf16_value(from_ordinal(o + 1)) - v),
                     np.abs(v - bf16_value(from_ordinal(o - 1))))
    gap = np.where(np.asarray(near) != 0, gap, 0.0)
    return bf16_rne(gap)


# ----------------------------------------------------------------------------------------------
# acceptance rules (the tolerance the GPU result is held to)

def tolerance(absum: np.ndarray) -> np.ndarray:
    """|y_gpu - y_ref| <= 2e-3 * sum_k |w_k x_k| + 1e-6 per element."""
    return 2e-3 * np.asarray(absum) + 1e-6


def bf16_rounding_interval(bits) -> tuple[np.ndarray, np.ndarray]:
    """[lo, hi]: the reals that round (nearest) to each finite bf16 value -- halfway to its
    neighbours on either side."""
    b = np.asarray(bits, np.uint16)
    o = bf16_ordinal(b)

    def from_ordinal(v):
        v = np.asarray(v, np.int64)
        mag = np.abs(v).astype(np.uint16)
        return np.where(v < 0, mag | 0x8000, mag).astype(np.uint16)

    v = bf16_value(b)
    lo = (v + bf16_value(from_ordinal(o - 1))) / 2
    hi = (v + bf16_value(from_ordinal(o + 1))) / 2
    return lo, hi


def within_tolerance(y_bits, y_ref, absum) -> np.ndarray:
    """The accumulation bound on the observable bf16 output: some real within
    2e-3 * A + 1e-6 of y_ref rounds to y_bits (y_ref's distance to the rounding interval of
    y_bits is within the tolerance)."""
    lo, hi = bf16_rounding_interval(y_bits)
    y_ref = np.asarray(y_ref, np.float64)
    dist = np.maximum(np.maximum(lo - y_ref, y_ref - hi), 0.0)
    return dist <= tolerance(absum)


def bf16_ordinal(bits) -> np.ndarray:
    """Monotone integer image of bf16 bit patterns (adjacent values differ by 1; +0 == -0)."""
    b = np.asarray(bits, np.uint16).astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def bf16_ulp_distance(a_bits, b_bits) -> np.ndarray:
    return np.abs(bf16_ordinal(a_bits) - bf16_ordinal(b_bits))


def silu(t):
    t = np.asarray(t, np.float64)
    with np.errstate(over="ignore"):  # e^-t = inf for t < -709 gives the exact limit, -0
        return t / (1.0 + np.exp(-t))


def silu_grad(t):
    t = np.asarray(t, np.float64)
    with np.errstate(over="ignore"):  # e^-t = inf gives s = 0, the exact limit
        s = 1.0 / (1.0 + np.exp(-t))
    return s * (1.0 + t * (1.0 - s))


def dual_tolerance(yg, yu, ag, au, o_ref) -> np.ndarray:
    """Propagated bound for o = silu(g) u:  |silu'(g)| |u| Eg + |silu(g)| Eu + 1/2 ulp_bf16(o)."""
    eg = tolerance(ag)
    eu = tolerance(au)
    o_ref = np.asarray(o_ref, np.float64)
    mag = np.abs(o_ref)
    e = np.floor(np.log2(np.where(mag > 0, mag, 2.0 ** -133)))
    half_ulp = np.ldexp(1.0, (np.maximum(e, -126) - 8).astype(np.int64))
    return np.abs(silu_grad(yg)) * (np.abs(yu) + eu) * eg + np.abs(silu(yg)) * eu + half_ulp
