"""The seeded input generator (free_sparse_attention_block_b200/inputs.py): the threaded
whole-workload path, a head subset and caller-provided output arrays all give the same values as
generating each head alone; the separable field equals its direct definition
F_c(t, y, x) = sum_s sin(2*pi*(f_t t/T + f_h y/H + f_w x/W) + phi); the bf16 rounding is
round-to-nearest-even."""
import math

import numpy as np

from free_sparse_attention_block_b200 import inputs


def test_workload_paths_agree_head_by_head():
    wl = inputs.Workload("t", 1, 3, 2 * 16 * 32, (2, 16, 32), (), seed=9)
    q, k, v = inputs.gen_workload(wl, processes=3)
    q1, k1, v1 = inputs.gen_workload(wl, processes=1)
    assert np.array_equal(q, q1) and np.array_equal(k, k1) and np.array_equal(v, v1)
    out = tuple(np.full(q.shape, 7, np.uint16) for _ in range(3))
    inputs.gen_workload(wl, heads=[(0, 2)], out=out)
    assert np.array_equal(out[0][0, 2], q[0, 2]) and np.array_equal(out[2][0, 2], v[0, 2])
    assert np.all(out[0][0, :2] == 7)                  # heads not asked for are left as they were
    for h in range(3):
        qh, kh, vh = inputs.gen_head(wl.seed, 0, h, wl.grid, wl.d, wl.f_max)
        assert np.array_equal(qh, q[0, h]) and np.array_equal(kh, k[0, h]) and np.array_equal(vh, v[0, h])


def test_field_equals_its_direct_definition():
    grid, d, f_max = (3, 5, 7), 4, 4.0
    rng = np.random.Generator(np.random.PCG64([1, 2, 3]))
    F = inputs._field(rng, grid, d, f_max)
    rng = np.random.Generator(np.random.PCG64([1, 2, 3]))
    f = rng.uniform(0.0, f_max, size=(d, 4, 3))
    phi = rng.uniform(0.0, 2.0 * math.pi, size=(d, 4))
    T, H, W = grid
    ref = np.zeros((T * H * W, d))
    for t in range(T):
        for y in range(H):
            for x in range(W):
                n = (t * H + y) * W + x
                for c in range(d):
                    ref[n, c] = sum(math.sin(2 * math.pi * (f[c, s, 0] * t / T + f[c, s, 1] * y / H +
                                                            f[c, s, 2] * x / W) + phi[c, s])
                                    for s in range(4))
    np.testing.assert_allclose(F, ref.astype(np.float32), rtol=0, atol=2e-6)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 3.0e38, np.inf, -np.inf, np.nan],
                 np.float32)
    b = inputs.f32_to_bf16_bits(x)
    back = inputs.bf16_bits_to_f32(b)
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties go to the even mantissa (1.0); 1 + 3*2^-8
    # is halfway between 1 + 2^-7 and 1 + 2^-6: even is 1 + 2^-6
    assert back[0] == 1.0 and back[1] == 1.0 and back[2] == 1.0 + 2.0 ** -6
    assert back[3] == -2.5 and back[5] == np.inf and back[6] == -np.inf and np.isnan(back[7])
    assert np.isfinite(back[4]) and abs(back[4] / 3.0e38 - 1.0) <= 2.0 ** -8   # below the bf16 maximum
