"""The seeded input generator: its published primitives and the recipe's structure."""
import math

import numpy as np

import synth


def test_splitmix64_published_sequence():
    # splitmix64 reference generator seeded with 1234567 (state advanced by the golden gamma)
    gamma = 0x9E3779B97F4A7C15
    x = 1234567
    got = [synth.splitmix64((x + i * gamma) & (2**64 - 1)) for i in range(3)]
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423]


def test_normals_have_unit_moments():
    w = synth.Workload("m", [4096], 4, 4, 64, 128, 3, seed=7, draw_dtype="f32")
    x = w.fill("v", kind="f32").astype(np.float64).ravel()
    n = x.size
    assert abs(x.mean()) < 5.0 / math.sqrt(n)
    assert abs(x.var() - 1.0) < 8.0 * math.sqrt(2.0 / n)
    # fourth moment of a normal is 3
    assert abs((x**4).mean() - 3.0) < 0.05


def test_rows_equal_fill_and_seeds_differ():
    w = synth.CONFIGS["gqa128k"]
    q = w.fill("q", 4090, 4100)
    tok = np.array([4090, 4095, 4099])
    hd = np.array([0, 17, 31])
    np.testing.assert_array_equal(w.rows("q", tok, hd), q[tok - 4090, hd])
    w2 = synth.Workload("x", [8192], 32, 8, 128, 2048, 3, seed=1, rope_theta=5e5, plant=0.5)
    assert not np.array_equal(w2.fill("q", 4090, 4100), q)


def test_rotary_is_a_rotation_and_identity_at_position_zero():
    base = synth.Workload("a", [300], 2, 2, 16, 64, 3, seed=3, draw_dtype="f32")
    rot = synth.Workload("a", [300], 2, 2, 16, 64, 3, seed=3, rope_theta=500000.0, draw_dtype="f32")
    x = base.fill("q", kind="f32").astype(np.float64)
    y = rot.fill("q", kind="f32").astype(np.float64)
    np.testing.assert_array_equal(x[0], y[0])
    # pairs (d, d + D/2) keep their norm
    nx = x[:, :, :8] ** 2 + x[:, :, 8:] ** 2
    ny = y[:, :, :8] ** 2 + y[:, :, 8:] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-5, atol=1e-6)
    # pair d rotates by p * theta^(-2d/D): check the angle of one pair at p = 5
    p, d = 5, 1
    a = math.atan2(x[p, 0, d + 8], x[p, 0, d])
    b = math.atan2(y[p, 0, d + 8], y[p, 0, d])
    want = p * 500000.0 ** (-2.0 * d / 16)
    assert abs(math.remainder(b - a - want, 2 * math.pi)) < 1e-5


def test_plant_adds_the_recipe_offsets():
    kw = dict(seed=11, rope_theta=0.0, draw_dtype="f32")
    plain = synth.Workload("p", [64, 40], 4, 2, 8, 8, 3, **kw)
    plant = synth.Workload("p", [64, 40], 4, 2, 8, 8, 3, plant=0.5, **kw)
    dq = plant.fill("q", kind="f32").astype(np.float64) - plain.fill("q", kind="f32")
    dk = plant.fill("k", kind="f32").astype(np.float64) - plain.fill("k", kind="f32")
    dv = plant.fill("v", kind="f32").astype(np.float64) - plain.fill("v", kind="f32")
    assert not dv.any()
    cu = plant.cu_seqlens
    for s in range(2):
        nb = plant.blocks_of(s)
        for g in range(2):
            # queries: block 0 untouched, every later block shifted by 0.5 * the same unit vector
            u = None
            for i in range(nb):
                for t in range(cu[s] + 8 * i, min(cu[s + 1], cu[s] + 8 * i + 8)):
                    for h in (2 * g, 2 * g + 1):
                        if i == 0:
                            assert not dq[t, h].any()
                        else:
                            v = dq[t, h] / 0.5
                            assert abs(np.linalg.norm(v) - 1.0) < 1e-5
                            u = v if u is None else u
                            np.testing.assert_allclose(v, u, atol=1e-5)
            # keys: block r shifted by 0.5 * (number of query blocks targeting r) * u
            count = np.zeros(nb)
            for i in range(1, nb):
                r = plant.plant_target(s, i, g)
                assert 0 <= r < i
                count[r] += 1
            for r in range(nb):
                t = cu[s] + 8 * r
                np.testing.assert_allclose(dk[t, g], 0.5 * count[r] * u, atol=1e-5)


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.0e-5, 65504.0], dtype=np.float32)
    b = synth.f32_to_bf16_bits(x)
    back = synth.bf16_bits_to_f32(b)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1.0) wins
    assert back[1] == 1.0
    # 1 + 3*2^-8 is a tie between 1+2^-7 and 1+2^-6: even mantissa wins
    assert back[2] == np.float32(1.015625)
    assert back[0] == 1.0 and back[3] == -2.5
