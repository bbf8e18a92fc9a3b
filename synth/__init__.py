"""Seeded synthetic inputs for the weight-only NVFP4 GEMV (shared by tests, bench and oracle runs).

Only input manufacture lives here: splitmix64 counter stream -> Box-Muller normals -> fp32 / bf16,
and the NVFP4 quantisation recipe that turns fp32 weights into the stored bytes (e2m1 nibbles, one
e4m3 scale per 16 along K, fp32 per-tensor global scale).  No GEMV arithmetic and no decoding of
stored codes: the oracle and the CUDA library each do their own.

Workload recipes (the projection shapes of a 27B hybrid GatedDeltaNet + gated-attention decoder,
"Blueprint - circuit executor" page for qwen3.8-27b-nvfp4 on GB10, "Kernels the plan launches"):

  tiny      N=256,   K=512,   M=1, seed 0                 (correctness case)
  inproj    N=10240, K=5120,  M=1, seed 1                 (attention / GDN input projection)
  gateup    gate, up each N=17408, K=5120, M=1, seed 2    (fused SiLU(gate)*up dual GEMV)
  down      N=5120,  K=17408, M=8, seed 3                 (down projection at draft/verify width)
  sweep     4 layers x {qkv 10240x5120, o 5120x6144, gate_up 2x17408x5120, down 5120x17408},
            M in {1,2,4,8}, seed 4

Input prologues (the residual add + RMS norm before a projection, the sigmoid gate before the
attention output projection): a residual stream of N(0, 4^2) bf16 draws, norm gains
1 + N(0, 0.1^2) rounded to bf16, gate logits N(0, 2^2) bf16, each from its own offset.

Stream order inside one seed: every weight tensor (row-major, in the order listed; for the dual,
gate then up), then every activation tensor (row-major).  Activations are always drawn with 8 rows
and an M-row call uses the first M, so row r of x is the same for every M.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libsynth.so")
_lib = None

W_SIGMA = 0.02
X_SIGMA = 1.0
X_ROWS = 8  # activations are drawn with the largest row count


def build(force: bool = False) -> str:
    """Compile libsynth.so next to its source (plain C, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        u64, i64, dbl = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double
        vp = ctypes.c_void_p
        lib.synth_draw.argtypes = [u64, u64]
        lib.synth_draw.restype = u64
        lib.synth_normal_f64.argtypes = [u64, u64, i64, dbl, vp]
        lib.synth_normal_f32.argtypes = [u64, u64, i64, dbl, vp]
        lib.synth_normal_bf16.argtypes = [u64, u64, i64, dbl, vp]
        for f in (lib.synth_normal_f64, lib.synth_normal_f32, lib.synth_normal_bf16):
            f.restype = ctypes.c_int
        lib.synth_f32_to_bf16.argtypes = [ctypes.c_float]
        lib.synth_f32_to_bf16.restype = ctypes.c_uint16
        lib.synth_e4m3_round.argtypes = [ctypes.c_float, ctypes.POINTER(ctypes.c_float)]
        lib.synth_e4m3_round.restype = ctypes.c_uint8
        lib.synth_e2m1_round.argtypes = [ctypes.c_float]
        lib.synth_e2m1_round.restype = ctypes.c_uint8
        lib.synth_quantize_nvfp4.argtypes = [vp, i64, i64, vp, vp, ctypes.POINTER(ctypes.c_float)]
        lib.synth_quantize_nvfp4.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def draw(seed: int, i: int) -> int:
    """Raw 64-bit draw i of the splitmix64 stream seeded with `seed`."""
    return int(_load().synth_draw(seed, i))


def normal_f64(seed: int, offset: int, count: int, sigma: float = 1.0) -> np.ndarray:
    out = np.empty(count, np.float64)
    if _load().synth_normal_f64(seed, offset, count, sigma, _ptr(out)) != 0:
        raise ValueError("offset must be even and count >= 0")
    return out


def normal_f32(seed: int, offset: int, count: int, sigma: float = 1.0) -> np.ndarray:
    out = np.empty(count, np.float32)
    if _load().synth_normal_f32(seed, offset, count, sigma, _ptr(out)) != 0:
        raise ValueError("offset must be even and count >= 0")
    return out


def normal_bf16(seed: int, offset: int, count: int, sigma: float = 1.0) -> np.ndarray:
    """bf16 bit patterns (uint16) of fp32 normal draws, rounded to nearest even."""
    out = np.empty(count, np.uint16)
    if _load().synth_normal_bf16(seed, offset, count, sigma, _ptr(out)) != 0:
        raise ValueError("offset must be even and count >= 0")
    return out


def f32_to_bf16(v: float) -> int:
    return int(_load().synth_f32_to_bf16(v))


def e4m3_round(v: float) -> tuple[int, float]:
    val = ctypes.c_float()
    code = _load().synth_e4m3_round(v, ctypes.byref(val))
    return int(code), float(val.value)


def e2m1_round(r: float) -> int:
    return int(_load().synth_e2m1_round(r))


def quantize_nvfp4(w: np.ndarray) -> tuple[np.ndarray, np.ndarray, float]:
    """fp32 [n][k] -> (packed uint8 [n][k/2], scale codes uint8 [n][k/16], fp32 global scale)."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    if k % 16:
        raise ValueError("k must be a multiple of 16")
    packed = np.empty((n, k // 2), np.uint8)
    scales = np.empty((n, k // 16), np.uint8)
    g = ctypes.c_float()
    if _load().synth_quantize_nvfp4(_ptr(w), n, k, _ptr(packed), _ptr(scales), ctypes.byref(g)) != 0:
        raise ValueError("bad shape")
    return packed, scales, float(g.value)


@dataclass
class Weight:
    """One NVFP4 weight tensor as stored: packed nibbles, scale codes, global scale."""
    n: int
    k: int
    packed: np.ndarray  # uint8 [n][k/2]
    scales: np.ndarray  # uint8 [n][k/16]
    g: float


def nvfp4_weight(seed: int, offset: int, n: int, k: int, sigma: float = W_SIGMA) -> Weight:
    w = normal_f32(seed, offset, n * k, sigma).reshape(n, k)
    p, s, g = quantize_nvfp4(w)
    return Weight(n, k, p, s, g)


def activations(seed: int, offset: int, m: int, k: int) -> np.ndarray:
    """bf16 bits [m][k] of N(0, 1) draws."""
    return normal_bf16(seed, offset, m * k, X_SIGMA).reshape(m, k)


def residual_stream(seed: int, offset: int, m: int, k: int, sigma: float = 4.0) -> np.ndarray:
    """bf16 bits [m][k] of N(0, sigma^2) draws: the residual stream a norm prologue adds."""
    return normal_bf16(seed, offset, m * k, sigma).reshape(m, k)


def norm_gains(seed: int, offset: int, k: int, sigma: float = 0.1) -> np.ndarray:
    """bf16 bits [k] of 1 + N(0, sigma^2): an RMS norm's per-channel gains."""
    v = normal_f32(seed, offset, k, sigma) + np.float32(1.0)
    return np.array([f32_to_bf16(float(t)) for t in v], np.uint16)


def gate_logits(seed: int, offset: int, m: int, k: int, sigma: float = 2.0) -> np.ndarray:
    """bf16 bits [m][k] of N(0, sigma^2): the pre-sigmoid gate of a gated output."""
    return normal_bf16(seed, offset, m * k, sigma).reshape(m, k)


# ----------------------------------------------------------------------------------------------
# workload recipes


@dataclass
class Projection:
    """One GEMV of a workload: a single weight, or a gate/up pair for the fused dual."""
    name: str
    n: int
    k: int
    dual: bool = False
    w: Weight | None = None
    w_up: Weight | None = None
    x: np.ndarray | None = None  # bf16 bits [X_ROWS][k]


@dataclass
class Workload:
    name: str
    seed: int
    rows: tuple[int, ...]
    projections: list[Projection] = field(default_factory=list)

    def weight_bytes(self) -> int:
        b = 0
        for p in self.projections:
            b += (2 if p.dual else 1) * (p.n * p.k // 2 + p.n * p.k // 16)
        return b


# (name, [(projection name, N, K, dual)], seed, rows)
_RECIPES = {
    "tiny": ([("tiny", 256, 512, False)], 0, (1,)),
    "inproj": ([("inproj", 10240, 5120, False)], 1, (1,)),
    "gateup": ([("gate_up", 17408, 5120, True)], 2, (1,)),
    "down": ([("down", 5120, 17408, False)], 3, (8,)),
    "sweep": ([(f"L{l}.{nm}", n, k, d) for l in range(4) for (nm, n, k, d) in
               (("qkv", 10240, 5120, False), ("o", 5120, 6144, False),
                ("gate_up", 17408, 5120, True), ("down", 5120, 17408, False))], 4, (1, 2, 4, 8)),
    # several weights sharing one x (nvfp4_gemv_multi): the gated attention's key/value and
    # query/gate projections over the 5120-wide hidden state; every projection's x is drawn,
    # the multi-output GEMV uses the first one's
    "attn_kv": ([("k", 1024, 5120, False), ("v", 1024, 5120, False)], 5, (1, 8)),
    "attn_qgate": ([("q", 6144, 5120, False), ("gate", 6144, 5120, False)], 6, (1, 8)),
}

WORKLOADS = tuple(_RECIPES)


def describe(name: str) -> Workload:
    """Shapes of a workload without generating data."""
    projs, seed, rows = _RECIPES[name]
    return Workload(name, seed, rows, [Projection(nm, n, k, d) for (nm, n, k, d) in projs])


def make(name: str, generate_x: bool = True) -> Workload:
    """Generate every tensor of a workload from its seed (deterministic, parallel)."""
    wl = describe(name)
    off = 0
    for p in wl.projections:
        p.w = nvfp4_weight(wl.seed, off, p.n, p.k)
        off += p.n * p.k
        if p.dual:
            p.w_up = nvfp4_weight(wl.seed, off, p.n, p.k)
            off += p.n * p.k
    if generate_x:
        for p in wl.projections:
            p.x = activations(wl.seed, off, X_ROWS, p.k)
            off += X_ROWS * p.k
    return wl
