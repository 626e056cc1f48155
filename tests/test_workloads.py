"""The seeded generators: shapes, determinism and the stated distributions."""
import numpy as np

from decode_split12_b200 import workloads as wl


def test_bf16_rounding_is_nearest_even():
    f = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, np.inf], np.float32)
    b = wl.to_bf16_bits(f)
    assert list(b) == [0x3F80, 0x3F80, 0x3F82, 0xC020, 0x0000, 0x7F80]
    assert np.array_equal(wl.bf16_bits_to_f32(b)[[0, 3, 4]], f[[0, 3, 4]])


def test_generators_are_deterministic():
    a = wl.normal_with_outliers(16, 256, 0.02, 0.01, 0)
    b = wl.normal_with_outliers(16, 256, 0.02, 0.01, 0)
    c = wl.normal_with_outliers(16, 256, 0.02, 0.01, 1)
    assert np.array_equal(a, b) and not np.array_equal(a, c)


def test_student_t_scale():
    w = wl.bf16_bits_to_f32(wl.student_t_scaled(512, 4096, 0)).astype(np.float64)
    assert abs(w.std() * np.sqrt(4096) - 1.0) < 0.05


def test_escape_recipe_planted_exponents():
    w, n = wl.escape_stress(0.02, 0, rows=64, cols=512)
    e = (w.astype(np.int64) >> 7) & 0xFF
    assert n == round(0.02 * w.size)
    assert int(((e >= 140) & (e <= 150)).sum()) == n
    assert int(((e >= 109) & (e <= 123)).sum()) == w.size - n


def test_routing_distinct_experts():
    r = wl.moe_routing()
    assert r.shape == (64, 2)
    assert all(len(set(row)) == 2 for row in r)
    assert r.min() >= 0 and r.max() < 8


def test_llama8b_shapes():
    assert sum(r * c for r, c in wl.LLAMA8B_SHAPES.values()) == 218103808
