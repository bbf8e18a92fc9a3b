"""Helpers shared by the GPU tests: upload synthetic inputs, run the library, compare with the
oracle under the acceptance rules."""
import numpy as np
import torch

# One entry per checked call: where, elements, elements more than 1 bf16 ulp from bf16(y_ref)
# (all of them, near-zero ones included), the largest ulp distance, and the largest error over
# the tolerance.  conftest.py prints them at the end of the run.
ULP_RECORDS: list = []

import oracle
import synth
import nvfp4_weight_only_03_b200 as nv


def dev_weight(w: synth.Weight):
    return (torch.from_numpy(w.packed).cuda(), torch.from_numpy(w.scales).cuda(), w.g)


def dev_x(x_bits: np.ndarray, ldx: int = None):
    """bf16 bits [m][k] -> device bf16 tensor, optionally with a row stride ldx > k."""
    m, k = x_bits.shape
    t = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16)
    if ldx is None or ldx == k:
        return t.cuda()
    buf = torch.zeros((m, ldx), dtype=torch.bfloat16, device="cuda")
    buf[:, :k] = t.cuda()
    return buf[:, :k]


def bits(y: torch.Tensor) -> np.ndarray:
    return y.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def check_single(y_bits, y_ref, a_ref, where=""):
    """Accumulation bound: some real within 2e-3 A + 1e-6 of y_ref rounds to the bf16 output;
    and the output is within 1 bf16 ulp of bf16(y_ref) wherever the fp32 accumulation error
    cannot reach half an ulp (|y_ref| >= A / 16)."""
    y = oracle.bf16_value(y_bits)
    ok = oracle.within_tolerance(y_bits, y_ref, a_ref)
    bad = np.argwhere(~ok)
    tol = oracle.tolerance(a_ref)
    assert bad.size == 0, f"{where}: {bad.shape[0]} outside tolerance, e.g. {bad[:3].tolist()} " \
                          f"gpu={y[tuple(bad[0])]} ref={y_ref[tuple(bad[0])]} tol={tol[tuple(bad[0])]}"
    ulp = oracle.bf16_ulp_distance(y_bits, oracle.bf16_rne(y_ref))
    strict = np.abs(y_ref) >= a_ref / 16
    worst = int(ulp[strict].max()) if strict.any() else 0
    assert worst <= 1, f"{where}: bf16 ulp distance {worst} on a well-conditioned output"
    err = np.abs(y - y_ref)
    res = {"max_err_over_tol": float((err / tol).max()) if err.size else 0.0,
           "ulp_gt1_total": int((ulp > 1).sum()), "ulp_max": int(ulp.max()) if ulp.size else 0}
    ULP_RECORDS.append((where or "single", int(ulp.size), res["ulp_gt1_total"], res["ulp_max"],
                        res["max_err_over_tol"]))
    return res


def check_dual(o_bits, o_ref, yg, yu, ag, au, where=""):
    """Propagated tolerance on every element, and within 1 bf16 ulp of bf16(o_ref) wherever both
    pre-activations are well conditioned (each at least 1/16 of its absolute-value sum, as for
    the single GEMV, and the gate away from zero)."""
    o = oracle.bf16_value(o_bits)
    tol = oracle.dual_tolerance(yg, yu, ag, au, o_ref)
    err = np.abs(o - o_ref)
    bad = np.argwhere(~(err <= tol))
    assert bad.size == 0, f"{where}: {bad.shape[0]} outside tolerance, e.g. {bad[:3].tolist()}"
    ulp = oracle.bf16_ulp_distance(o_bits, oracle.bf16_rne(o_ref))
    well = (np.abs(yg) >= ag / 16) & (np.abs(yu) >= au / 16) & (np.abs(yg) > 1e-3)
    worst = int(ulp[well].max()) if well.any() else 0
    assert worst <= 1, f"{where}: bf16 ulp distance {worst} on a well-conditioned output"
    res = {"max_err_over_tol": float((err / tol).max()) if err.size else 0.0,
           "ulp_gt1_total": int((ulp > 1).sum()), "ulp_max": int(ulp.max()) if ulp.size else 0}
    ULP_RECORDS.append((where or "dual", int(ulp.size), res["ulp_gt1_total"], res["ulp_max"],
                        res["max_err_over_tol"]))
    return res


def assert_ws_clean(ws):
    """Error word, completion and arrival counts all back at zero after the calls (the partial
    sums are scratch and may stay): the header's 512 bytes, then one count per SM."""
    torch.cuda.synchronize()
    head = ws[:512 + 4 * torch.cuda.get_device_properties(ws.device).multi_processor_count]
    assert int(head.count_nonzero()) == 0, "workspace counts / error word not left zero"


def pack_nibbles(nibs: np.ndarray) -> np.ndarray:
    nibs = np.asarray(nibs, np.uint8)
    return (nibs[:, 0::2] | (nibs[:, 1::2] << 4)).astype(np.uint8)


def bf16_bits_of(vals) -> np.ndarray:
    return torch.tensor(np.asarray(vals, np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def random_weight(rng, n, k, scale_hi=0x7F):
    nibs = rng.integers(0, 16, (n, k)).astype(np.uint8)
    sc = rng.integers(0, scale_hi, (n, k // 16)).astype(np.uint8)
    return synth.Weight(n, k, pack_nibbles(nibs), sc, float(np.float32(rng.uniform(0.01, 1.0))))
