"""Pins for the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a
hand-derived container, exhaustive round trips, brute force on tiny inputs,
closed forms, special cases with exact answers, an independent FP64 routine,
and the entropy figure the pages print.
"""
import math

import numpy as np
import pytest

from conftest import golden_expected_bytes, golden_two_tiles_weights, load_golden
from decode_split12_b200 import workloads as wl


# ---------------------------------------------------------------- golden

def test_golden_two_tiles_bytes(oracle):
    """Hand-derived container (tests/golden/two_tiles.json): header, both
    planes' nibble order, the tie-break to the smallest base, escape order and
    all plane offsets."""
    d = load_golden("two_tiles.json")
    w = golden_two_tiles_weights(d)
    blob = oracle.encode(w)
    exp = golden_expected_bytes(d)
    assert blob.size == d["total_bytes"]
    bad = np.nonzero(blob != exp)[0]
    assert bad.size == 0, f"first mismatching byte offsets {bad[:10]}"
    assert np.array_equal(oracle.decode(blob), w)
    st = oracle.stats(blob)
    assert st["n_esc"] == d["n_esc"]


def test_golden_tile_bases(oracle):
    d = load_golden("two_tiles.json")
    w = golden_two_tiles_weights(d)
    for r in range(2):
        b, n_esc = oracle.tile_base(w[r])
        assert b == d["base"][r]
    assert oracle.tile_base(w[0])[1] == 2
    assert oracle.tile_base(w[1])[1] == 64


# ---------------------------------------------------------------- exhaustive

def _all_patterns():
    return np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)


def _bitrev16(a):
    a = a.astype(np.uint32)
    r = np.zeros_like(a)
    for i in range(16):
        r |= ((a >> i) & 1) << (15 - i)
    return r.astype(np.uint16)


def test_roundtrip_all_patterns_natural_order(oracle):
    """All 65,536 BF16 patterns (NaNs, infinities, zeros, subnormals); in
    natural order every 128-weight tile shares sign and exponent, so no tile
    needs an escape."""
    w = _all_patterns().reshape(512, 128)
    blob = oracle.encode(w)
    assert np.array_equal(oracle.decode(blob), w)
    assert oracle.stats(blob)["n_esc"] == 0


@pytest.mark.parametrize("order", ["shuffled", "bitreversed"])
def test_roundtrip_all_patterns_scrambled(oracle, order):
    p = _all_patterns()
    if order == "shuffled":
        p = p[wl.rng_for(0, 1).permutation(p.size)]
    else:
        p = _bitrev16(p)
    w = p.reshape(512, 128)
    blob = oracle.encode(w)
    assert np.array_equal(oracle.decode(blob), w)
    st = oracle.stats(blob)
    assert st["n_esc"] > 10000  # uniform exponents: most weights escape
    # every decoded exponent histogram bin holds 256 patterns
    assert np.all(st["exp_hist"] == 256)


# ---------------------------------------------------------------- brute force

def _escapes_for_base(tile, b):
    e = (tile.astype(np.int64) >> 7) & 0xFF
    return int(np.sum((e < b) | (e > b + 14)))


@pytest.mark.parametrize("seed", range(40))
def test_base_minimises_escapes_brute_force(oracle, seed):
    """For tiny tensors the chosen base must minimise the escape count over
    every admissible base, and be the smallest base doing so."""
    g = wl.rng_for(seed, 3)
    kind = seed % 4
    if kind == 0:
        tile = g.integers(0, 1 << 16, size=128).astype(np.uint16)
    elif kind == 1:
        e = g.integers(100, 140, size=128)
        tile = ((g.integers(0, 2, 128) << 15) | (e << 7) | g.integers(0, 128, 128)).astype(np.uint16)
    elif kind == 2:
        e = np.concatenate([g.integers(0, 15, 64), g.integers(200, 215, 64)])
        tile = ((e << 7) | g.integers(0, 128, 128)).astype(np.uint16)
    else:
        tile = wl.normal_with_outliers(1, 128, 0.02, 0.05, seed)[0]
    counts = [_escapes_for_base(tile, b) for b in range(242)]
    best = min(counts)
    b, n_esc = oracle.tile_base(tile)
    assert n_esc == best
    assert b == counts.index(best)


@pytest.mark.parametrize("seed", range(8))
def test_tiny_tensor_escape_total(oracle, seed):
    g = wl.rng_for(seed, 4)
    w = g.integers(0, 1 << 16, size=(2, 256)).astype(np.uint16)
    blob = oracle.encode(w)
    expect = sum(min(_escapes_for_base(w.reshape(-1, 128)[t], b) for b in range(242)) for t in range(4))
    assert oracle.stats(blob)["n_esc"] == expect
    assert np.array_equal(oracle.decode(blob), w)


@pytest.mark.parametrize("spread", [0, 1, 5, 14])
def test_narrow_exponent_spread_never_escapes(oracle, spread):
    """A tile whose exponents span at most 15 values fits one window."""
    g = wl.rng_for(spread, 5)
    for lo in (0, 60, 127, 241, 255 - spread):
        e = g.integers(lo, lo + spread + 1, size=128)
        tile = ((g.integers(0, 2, 128) << 15) | (e << 7) | g.integers(0, 128, 128)).astype(np.uint16)
        assert oracle.tile_base(tile)[1] == 0


def test_sixteen_exponents_escape_once(oracle):
    """Exponents spanning 16 values: the least common one must escape."""
    e = np.concatenate([np.arange(120, 136), np.full(112, 125)])  # 120..135: 16 distinct
    tile = ((e << 7) | 3).astype(np.uint16)
    b, n = oracle.tile_base(tile)
    assert n == 1 and b == 120  # drop 135 (smallest base wins over dropping 120)


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("rows,cols", [(1, 128), (3, 256), (4096, 4096), (8192, 28672), (7, 1152)])
def test_payload_rate_twelve_bits(oracle, rows, cols):
    """The payload (raw + codes) is 12 bits per weight, 0.75 of BF16, i.e.
    1.33x smaller (setupai.cc key points); the rest is per-tile header
    (1 base byte + 4 offset bytes), escapes and alignment padding."""
    n = rows * cols
    for n_esc in (0, 1, 1000):
        total = oracle.container_bytes(rows, cols, n_esc)
        overhead = total - 1.5 * n
        assert total % 256 == 0
        assert overhead >= 5 * (n // 128) + 4 + 2 * n_esc + 64
        assert overhead < 5 * (n // 128) + 4 + 2 * n_esc + 64 + 6 * 256
    big = oracle.container_bytes(1 << 14, 1 << 14, 0)
    assert abs(big / (2 << 28) - (0.75 + 5 / 256)) < 1e-4


def test_shape_errors(oracle):
    assert oracle.container_bytes(4, 100, 0) < 0
    assert oracle.container_bytes(0, 128, 0) < 0


def test_escape_generator_count_exact(oracle):
    """The escape-stress recipe plants an exact escape count; the oracle must
    find exactly those (reduced size, same recipe)."""
    for rate in wl.ESCAPE_RATES:
        w, planted = wl.escape_stress(rate, seed=0, rows=512, cols=1024)
        blob = oracle.encode(w)
        assert oracle.stats(blob)["n_esc"] == planted
        assert np.array_equal(oracle.decode(blob), w)


# ---------------------------------------------------------------- entropy

@pytest.mark.parametrize("kind", ["normal", "student_t"])
def test_exponent_entropy_near_page_figure(oracle, kind):
    """The exponent field of trained weights carries about 2.6 of its 8 bits
    (meowlab section 1 table: 2.59-2.64 bits on Qwen3-8B).  Normal-like
    synthetic weights land in the same range."""
    if kind == "normal":
        w = wl.normal_with_outliers(256, 4096, 0.02, 0.0, 0)
    else:
        w = wl.student_t_scaled(256, 4096, 0)
    blob = oracle.encode(w)
    st = oracle.stats(blob)
    assert 2.4 <= st["exp_entropy_bits"] <= 2.8
    # the oracle's histogram must equal the raw tensor's exponent histogram
    direct = np.bincount(((w.astype(np.int64) >> 7) & 0xFF).ravel(), minlength=256)
    assert np.array_equal(st["exp_hist"].astype(np.int64), direct)
    # fully charged size: 12 bits + header (0.3125 bit) + escapes
    assert 12.3 < st["bits_per_weight"] < 12.4
    assert st["payload_ratio"] == 0.75


# ---------------------------------------------------------------- products

def test_bf16_exact_values(oracle):
    assert oracle.bf16_to_double(0x3F80) == 1.0
    assert oracle.bf16_to_double(0xBFC0) == -1.5
    assert oracle.bf16_to_double(0x0001) == 2.0 ** -133
    assert math.isinf(oracle.bf16_to_double(0x7F80))
    assert math.isnan(oracle.bf16_to_double(0x7FC0))
    assert oracle.bf16_to_double(0x3C00) == 2.0 ** -7


def test_gemv_one_hot_returns_column(oracle):
    """x = e_j gives y = W[:, j] exactly (a single product of BF16 values)."""
    w = wl.normal_with_outliers(67, 384, 0.02, 0.01, 3)
    blob = oracle.encode(w)
    for j in (0, 1, 127, 128, 383):
        x = np.zeros((1, 384), np.uint16)
        x[0, j] = 0x3F80
        y, s = oracle.gemv_f64(blob, x)
        col = wl.bf16_bits_to_f32(w[:, j]).astype(np.float64)
        assert np.array_equal(y[0], col)
        assert np.array_equal(s[0], np.abs(col))


def test_gemv_integer_sums_exact(oracle):
    """Small-integer W with an all-ones x: row sums are exact integers, and
    the tolerance scale is the sum of magnitudes."""
    g = wl.rng_for(9, 0)
    vals = g.integers(-8, 9, size=(50, 640)).astype(np.float32)
    w = wl.to_bf16_bits(vals)
    x = np.full((2, 640), 0x3F80, np.uint16)
    x[1] = 0xBF80  # -1
    blob = oracle.encode(w)
    y, s = oracle.gemv_f64(blob, x)
    assert np.array_equal(y[0], vals.sum(1).astype(np.float64))
    assert np.array_equal(y[1], -vals.sum(1).astype(np.float64))
    assert np.array_equal(s[0], np.abs(vals).sum(1).astype(np.float64))


def test_gemv_matches_independent_fp64(oracle):
    """The oracle's FP64 product against numpy float64 on the same decoded
    values (an independent routine, not the oracle)."""
    w = wl.student_t_scaled(96, 1024, 1)
    x = wl.activations(3, 1024, 1)
    blob = oracle.encode(w)
    y, s = oracle.gemv_f64(blob, x)
    wf = wl.bf16_bits_to_f32(w).astype(np.float64)
    xf = wl.bf16_bits_to_f32(x).astype(np.float64)
    ref = xf @ wf.T
    assert np.allclose(y, ref, rtol=0, atol=1e-12 * (np.abs(xf) @ np.abs(wf).T).max())
    assert np.allclose(s, np.abs(xf) @ np.abs(wf).T, rtol=1e-14)
    yr, sr = oracle.gemv_rows_f64(blob, x, [5, 0, 95])
    assert np.array_equal(yr, y[:, [5, 0, 95]])
    assert np.array_equal(sr, s[:, [5, 0, 95]])


# ---------------------------------------------------------------- corruption

def test_silu_mul_textbook_values(oracle):
    """The gated-MLP activation h = silu(g) * u against values fixed by the
    logistic function itself: silu(0) = 0; silu(1) = e / (1 + e); silu(t)
    -> t for large t and -> 0 for large negative t; silu(t) - silu(-t) = t
    (because the logistic satisfies s(t) + s(-t) = 1).  A flipped sign in
    the exponent, a dropped factor or swapped operands fails one of them."""
    e = math.e
    g = np.array([0.0, 1.0, 1.0, 2.0, 64.0, -64.0, 3.5, -3.5, 0.25, -0.25])
    u = np.array([5.0, 1.0, 2.0, 1.0, 3.0, 3.0, 1.0, 1.0, 1.0, 1.0])
    h = oracle.silu_mul_f64(g, u)
    assert h[0] == 0.0
    assert h[1] == pytest.approx(e / (1 + e), rel=1e-15)
    assert h[2] == pytest.approx(2 * e / (1 + e), rel=1e-15)          # gate 1, up 2
    assert h[3] == pytest.approx(2 * e * e / (1 + e * e), rel=1e-15)  # gate 2, up 1: not the same
    assert h[4] == pytest.approx(192.0, rel=1e-25)
    assert abs(h[5]) < 1e-24
    assert h[6] - h[7] == pytest.approx(3.5, rel=1e-15)
    assert h[8] - h[9] == pytest.approx(0.25, rel=1e-15)


def test_swiglu_one_hot_uses_gate_and_up_columns(oracle):
    """x = e_j: g and u are column j of each matrix exactly, and h applies
    the activation to the gate column only."""
    wg = wl.normal_with_outliers(40, 256, 0.5, 0.0, 5)
    wu = wl.normal_with_outliers(40, 256, 0.5, 0.0, 6)
    bg, bu = oracle.encode(wg), oracle.encode(wu)
    j = 77
    x = np.zeros((1, 256), np.uint16)
    x[0, j] = 0x3F80
    h, g, u, s_g, s_u = oracle.swiglu_f64(bg, bu, x)
    cg = wl.bf16_bits_to_f32(wg[:, j]).astype(np.float64)
    cu = wl.bf16_bits_to_f32(wu[:, j]).astype(np.float64)
    assert np.array_equal(g[0], cg) and np.array_equal(u[0], cu)
    assert np.array_equal(s_g[0], np.abs(cg)) and np.array_equal(s_u[0], np.abs(cu))
    assert np.array_equal(h[0], oracle.silu_mul_f64(cg, cu))
    assert not np.allclose(h[0], oracle.silu_mul_f64(cu, cg))


def test_corruption_detected(oracle):
    """Flipping bytes must make the decoder fail closed (wavect, 14-day pilot,
    step 2: inject corruption and confirm it is detected)."""
    w = wl.normal_with_outliers(8, 512, 0.02, 0.01, 4)
    blob = oracle.encode(w)
    assert oracle.decode_rc(blob) == 0
    st = oracle.stats(blob)
    assert st["n_esc"] > 0
    b = blob.copy(); b[0] ^= 1
    assert oracle.decode_rc(b) != 0                      # magic
    b = blob.copy(); b[32] ^= 1
    assert oracle.decode_rc(b) != 0                      # n_esc
    off_esc_off = 256 + 4096 + 2048 + 256
    b = blob.copy(); b[off_esc_off + 4] ^= 0x7F
    assert oracle.decode_rc(b) != 0                      # esc_off
    # turn an ordinary code into an escape code: count mismatch
    code = blob[256 + 4096: 256 + 4096 + 2048]
    k = int(np.nonzero((code & 0x0F) != 0x0F)[0][0])
    b = blob.copy(); b[256 + 4096 + k] |= 0x0F
    assert oracle.decode_rc(b) != 0
    # turn an escape code into an ordinary one: fewer escapes than offsets say
    k = int(np.nonzero((code & 0x0F) == 0x0F)[0][0])
    b = blob.copy(); b[256 + 4096 + k] &= 0xF0
    assert oracle.decode_rc(b) != 0
