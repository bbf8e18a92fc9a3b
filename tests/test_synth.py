"""Checks of the seeded input generator and the NVFP4 quantisation recipe (input side)."""
import numpy as np
import pytest
import torch

import oracle
import synth

MASK = (1 << 64) - 1


def splitmix64_sequential(seed, count):
    """The generator in its textbook sequential form (state += gamma; mix)."""
    out, state = [], seed
    for _ in range(count):
        state = (state + 0x9E3779B97F4A7C15) & MASK
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK
        out.append(z ^ (z >> 31))
    return out


def test_splitmix64_published_vectors():
    # first outputs of splitmix64 seeded with 0 (widely published test vector)
    assert synth.draw(0, 0) == 0xE220A8397B1DCDAF
    assert synth.draw(0, 1) == 0x6E789E6AA1B965F4
    assert synth.draw(0, 2) == 0x06C45D188009454F


@pytest.mark.parametrize("seed", [0, 1, 4, 0xDEADBEEF])
def test_counter_form_equals_sequential_form(seed):
    seq = splitmix64_sequential(seed, 50)
    assert [synth.draw(seed, i) for i in range(50)] == seq


def test_normals_statistics_and_offsets():
    z = synth.normal_f64(1, 0, 400000)
    assert abs(z.mean()) < 5 / np.sqrt(z.size)
    assert abs(z.var() - 1) < 0.01
    # counter form: a window at an even offset equals the same slice of a longer draw
    assert np.array_equal(synth.normal_f64(1, 1000, 64), z[1000:1064])
    with pytest.raises(ValueError):
        synth.normal_f64(1, 3, 4)


def test_bf16_rounding_of_draws_matches_torch():
    f = synth.normal_f32(7, 0, 10001, 1.0)
    b = synth.normal_bf16(7, 0, 10001, 1.0)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(b, ref)


def test_e2m1_rounding_ties_to_even_and_saturates():
    cases = {0.0: 0, 0.2: 0, 0.25: 0, 0.26: 1, 0.75: 2, 1.25: 2, 1.3: 3, 1.75: 4, 2.5: 4,
             2.6: 5, 3.5: 6, 5.0: 6, 5.01: 7, 6.0: 7, 100.0: 7}
    for v, c in cases.items():
        assert synth.e2m1_round(v) == c, v
        assert synth.e2m1_round(-v) == c | 8, -v


def test_e4m3_rounding_matches_torch_in_range():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(0, 448, 5000), np.exp(rng.uniform(-13, 6, 5000)),
                        oracle.e4m3_table()[:0x7F]]).astype(np.float32)
    v = v[v <= 448]
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for x, r in zip(v, ref):
        code, val = synth.e4m3_round(float(x))
        assert code == r, (float(x), code, r)
        assert val == oracle.e4m3(code)
    assert synth.e4m3_round(1000.0)[0] == 0x7E


def test_quantiser_recipe():
    wl = synth.make("tiny")
    w = synth.normal_f32(0, 0, 256 * 512, synth.W_SIGMA).reshape(256, 512)
    p = wl.projections[0].w
    amax = np.abs(w).max()
    assert p.g == np.float32(amax) / np.float32(6 * 448)
    # the group holding the tensor amax gets the top scale code
    r, c = np.unravel_index(np.abs(w).argmax(), w.shape)
    assert p.scales[r, c // 16] == 0x7E
    # dequantised weights are within half a grid step of the originals (nearest rounding)
    nib = np.empty_like(w, dtype=np.uint8)
    nib[:, 0::2] = p.packed & 15
    nib[:, 1::2] = p.packed >> 4
    t2, t4 = oracle.e2m1_table(), oracle.e4m3_table()
    s = np.repeat(t4[p.scales], 16, axis=1)
    deq = t2[nib] * s * p.g
    step = s * p.g  # largest e2m1 grid gap is 2 (between 4 and 6) -> half step <= 1 * scale
    assert np.all(np.abs(deq - w) <= step * 1.0 + 1e-12)
    # the e2m1 value never exceeds 6 and nibbles follow the sign of w (or are zero)
    nz = t2[nib] != 0
    assert np.all(np.sign(t2[nib][nz]) == np.sign(w[nz]))


def test_zero_group_quantises_to_zero():
    w = np.zeros((2, 32), np.float32)
    w[1, 16:] = np.linspace(-1, 1, 16)
    packed, scales, g = synth.quantize_nvfp4(w)
    assert scales[0, 0] == 0 and scales[0, 1] == 0 and scales[1, 0] == 0
    assert np.all(packed[0] == 0) and np.all(packed[1, :8] == 0)
    assert scales[1, 1] == 0x7E
    w0 = np.zeros((1, 16), np.float32)
    assert synth.quantize_nvfp4(w0)[2] == 1.0


def test_workload_shapes_and_row_prefix():
    wl = synth.describe("sweep")
    assert len(wl.projections) == 16
    assert wl.rows == (1, 2, 4, 8)
    assert wl.weight_bytes() == 790364160
    gu = synth.describe("gateup").projections[0]
    assert gu.dual and (gu.n, gu.k) == (17408, 5120)
    d = synth.describe("down").projections[0]
    assert (d.n, d.k) == (5120, 17408) and synth.describe("down").rows == (8,)
