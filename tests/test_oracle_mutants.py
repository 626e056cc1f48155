"""Planted mistakes: each plausible slip in the oracle must fail a pin.

Every case edits a copy of oracle/split12_oracle.c (the committed oracle is
never touched), compiles it with gcc into a temporary directory, binds it and
runs a quick battery of the same pins as test_oracle_pins.py.  A mutant that
passes the battery would mean the pins cannot see that mistake.
"""
import os

import numpy as np
import pytest

from conftest import golden_expected_bytes, golden_two_tiles_weights, load_golden
from decode_split12_b200 import workloads as wl
from oracle import build_oracle
from oracle.oracle import Oracle, load

SRC = build_oracle.SRC

MUTANTS = {
    "window_14_wide": [("e <= b + ORACLE_WINDOW - 1", "e <= b + ORACLE_WINDOW - 2")],
    "ties_to_largest_base": [("if (!have || c > best_count)", "if (!have || c >= best_count)")],
    "base_241_excluded": [("for (uint32_t b = 0; b <= ORACLE_MAX_BASE; b++)",
                           "for (uint32_t b = 0; b < ORACLE_MAX_BASE; b++)")],
    "nibbles_swapped_consistently": [
        ("code[pos / 2] = (uint8_t)c;", "code[pos / 2] = (uint8_t)(c << 4);"),
        ("code[pos / 2] |= (uint8_t)(c << 4);", "code[pos / 2] |= (uint8_t)c;"),
        ("return (pos % 2 == 0) ? (byte & 0x0Fu) : (uint32_t)(byte >> 4);",
         "return (pos % 2 == 1) ? (byte & 0x0Fu) : (uint32_t)(byte >> 4);"),
    ],
    "sign_dropped_from_raw": [("(oracle_bf16_sign(v) << 7)", "(0u << 7)")],
    "mantissa_mask_6_bits": [("return w & 0x7Fu; }", "return w & 0x3Fu; }")],
    "decode_exponent_off_by_one": [("uint32_t e = b + c;", "uint32_t e = b + c + 1;")],
    "decode_sign_wrong_bit": [("((uint32_t)(r & 0x80) << 8)", "((uint32_t)(r & 0x80) << 7)")],
    "escapes_read_backwards": [("get_u16(V->esc + 2 * (uint64_t)(lo + k))",
                                "get_u16(V->esc + 2 * (uint64_t)(hi - 1 - k))")],
    "escape_count_check_dropped": [("if (lo + k != hi) return ORACLE_ERR_CORRUPT;", "")],
    "magnitude_without_abs": [("mag += fabs(p);", "mag += p;")],
    "weight_operand_transposed": [("oracle_bf16_to_double(w[n * cols + k])",
                                   "oracle_bf16_to_double(w[k * rows + n])")],
    "bf16_widened_by_15": [("uint32_t bits = (uint32_t)w << 16;", "uint32_t bits = (uint32_t)w << 15;")],
    "last_plane_unpadded": [("L->total = L->off_esc + pad_to_align(2 * n_esc);",
                             "L->total = L->off_esc + 2 * n_esc;")],
    "entropy_in_nats": [("h -= p * log2(p);", "h -= p * log(p);")],
    "silu_exp_sign_flipped": [("h[i] = g[i] / (1.0 + exp(-g[i])) * u[i];",
                               "h[i] = g[i] / (1.0 + exp(g[i])) * u[i];")],
    "silu_applied_to_up": [("h[i] = g[i] / (1.0 + exp(-g[i])) * u[i];",
                            "h[i] = u[i] / (1.0 + exp(-u[i])) * g[i];")],
    "sigmoid_instead_of_silu": [("h[i] = g[i] / (1.0 + exp(-g[i])) * u[i];",
                                 "h[i] = 1.0 / (1.0 + exp(-g[i])) * u[i];")],
    "v2_count_check_dropped": [("            if (seen != count) return ORACLE_ERR_CORRUPT;\n", "")],
    "v2_row_offset_ignored": [("        uint64_t k = lo; /* next escape of this row */",
                               "        uint64_t k = 0; /* next escape of this row */")],
    "v2_base_and_count_bytes_swapped": [
        ("        tmeta[2 * t] = (uint8_t)b;\n        tmeta[2 * t + 1] = (uint8_t)count;",
         "        tmeta[2 * t + 1] = (uint8_t)b;\n        tmeta[2 * t] = (uint8_t)count;"),
        ("uint32_t b = tmeta[2 * t], count = tmeta[2 * t + 1], seen = 0;",
         "uint32_t b = tmeta[2 * t + 1], count = tmeta[2 * t], seen = 0;")],
    "v3_pair_raw_bytes_swapped": [("            pt[3 * i] = raw_t[2 * i];\n            pt[3 * i + 1] = raw_t[2 * i + 1];",
                                   "            pt[3 * i] = raw_t[2 * i + 1];\n            pt[3 * i + 1] = raw_t[2 * i];")],
    "v3_pair_nibbles_swapped_consistently": [
        ("            pt[3 * i + 2] = code_t[i];",
         "            pt[3 * i + 2] = (uint8_t)((code_t[i] >> 4) | (code_t[i] << 4));"),
        ("(pos % 2 == 0) ? (pair[3 * p + 2] & 0x0Fu) : (uint32_t)(pair[3 * p + 2] >> 4)",
         "(pos % 2 == 1) ? (pair[3 * p + 2] & 0x0Fu) : (uint32_t)(pair[3 * p + 2] >> 4)")],
    "v3_pair_plane_unpadded": [("L->off_base = L->off_pair + pad_to_align(rows * cols / 2 * 3);",
                                "L->off_base = L->off_pair + rows * cols / 2 * 3;")],
    "v4_ties_to_larger_symbol": [("if (best < 0 || count[s] > count[best]) best = s;",
                                  "if (best < 0 || count[s] >= count[best]) best = s;")],
    "v4_table_of_30_symbols": [("    for (uint32_t k = 0; k < ORACLE_SYM_CODES; k++) {\n        int best = -1;",
                                "    for (uint32_t k = 0; k + 1 < ORACLE_SYM_CODES; k++) {\n        int best = -1;")],
    "v4_code_bit_dropped_from_raw": [("raw[pos] = (uint8_t)(((c & 1u) << 7) | oracle_bf16_mantissa(v));",
                                      "raw[pos] = (uint8_t)oracle_bf16_mantissa(v);")],
    "escape_stored_byte_swapped": [("esc[2 * *written] = (uint8_t)(v & 0xFF);\n            esc[2 * *written + 1] = (uint8_t)(v >> 8);",
                                    "esc[2 * *written] = (uint8_t)(v >> 8);\n            esc[2 * *written + 1] = (uint8_t)(v & 0xFF);")],
}


def _battery(o: Oracle):
    """Raises AssertionError (or an oracle error) when any pin fails."""
    d = load_golden("two_tiles.json")
    w = golden_two_tiles_weights(d)
    blob = o.encode(w)
    assert blob.size == d["total_bytes"]
    assert np.array_equal(blob, golden_expected_bytes(d))
    # exhaustive round trips
    allp = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    for p in (allp, allp[wl.rng_for(0, 1).permutation(allp.size)]):
        wt = p.reshape(512, 128)
        b2 = o.encode(wt)
        assert np.array_equal(o.decode(b2), wt)
    assert o.stats(o.encode(allp.reshape(512, 128)))["n_esc"] == 0
    # brute-force bases
    for seed in range(12):
        tile = wl.rng_for(seed, 3).integers(0, 1 << 16, size=128).astype(np.uint16)
        e = (tile.astype(np.int64) >> 7) & 0xFF
        counts = [int(np.sum((e < b) | (e > b + 14))) for b in range(242)]
        b, n = o.tile_base(tile)
        assert n == min(counts) and b == counts.index(min(counts))
    # exact escape count of the stress recipe
    ws, planted = wl.escape_stress(0.02, seed=0, rows=64, cols=1024)
    assert o.stats(o.encode(ws))["n_esc"] == planted
    # products: one-hot column, integer sums, magnitudes
    wn = wl.normal_with_outliers(33, 384, 0.02, 0.01, 3)
    bn = o.encode(wn)
    x = np.zeros((1, 384), np.uint16)
    x[0, 200] = 0x3F80
    y, s = o.gemv_f64(bn, x)
    col = wl.bf16_bits_to_f32(wn[:, 200]).astype(np.float64)
    assert np.array_equal(y[0], col) and np.array_equal(s[0], np.abs(col))
    vals = wl.rng_for(9, 0).integers(-8, 9, size=(20, 256)).astype(np.float32)
    bi = o.encode(wl.to_bf16_bits(vals))
    y, s = o.gemv_f64(bi, np.full((1, 256), 0x3F80, np.uint16))
    assert np.array_equal(y[0], vals.sum(1)) and np.array_equal(s[0], np.abs(vals).sum(1))
    # container version 2: round trip, agreement with version 1's metadata,
    # a corrupted tile count refused
    wv = allp[wl.rng_for(0, 1).permutation(allp.size)].reshape(512, 128)
    assert np.array_equal(o.decode_v2(o.encode_v2(wv)), wv)
    w2, _ = wl.escape_stress(0.05, seed=2, rows=16, cols=1024)
    b1, b2 = o.encode(w2), o.encode_v2(w2)
    n_t = 16 * 1024 // 128
    off_t = 256 + 16 * 1024 + 8192        # both versions: header, raw, code planes first
    assert np.array_equal(b2[off_t:off_t + 2 * n_t:2], b1[off_t:off_t + n_t])
    e1 = b1[off_t + 256:off_t + 256 + 4 * (n_t + 1)].view(np.uint32)
    assert np.array_equal(b2[off_t + 1:off_t + 2 * n_t:2].astype(np.uint32), np.diff(e1))
    k = int(np.flatnonzero(b2[off_t + 1:off_t + 2 * n_t:2])[0])
    bad = b2.copy()
    bad[off_t + 2 * k + 1] += 1
    assert o.decode_v2_rc(bad) != 0
    # container version 3: the hand-derived golden, round trip, agreement
    # with version 1's planes
    g3 = load_golden("two_tiles_v3.json")
    e3 = golden_expected_bytes(d)
    for lo, hi in g3["clear"]:
        e3[lo:hi] = 0
    for item in g3["patch"]:
        chunk = np.frombuffer(bytes.fromhex(item[1]) * (item[2] if len(item) > 2 else 1), np.uint8)
        e3[item[0]:item[0] + chunk.size] = chunk
    assert np.array_equal(o.encode_v3(w), e3)
    assert np.array_equal(o.decode_v3(o.encode_v3(wv)), wv)
    b3 = o.encode_v3(w2)
    pr = b3[256:256 + 16 * 1024 * 3 // 2].reshape(-1, 3)
    assert np.array_equal(pr[:, 2], b1[256 + 16 * 1024:256 + 16 * 1024 + 8192])
    assert np.array_equal(pr[:, 0], b1[256:256 + 16 * 1024:2])
    # container version 4: the hand-derived golden and a round trip
    d4 = load_golden("one_tile_v4.json")
    w4 = np.array([int(x, 16) for x in d4["weights"]], np.uint16).reshape(1, 128)
    assert np.array_equal(o.encode_v4(w4), golden_expected_bytes(d4))
    assert np.array_equal(o.decode_v4(o.encode_v4(wv)), wv)
    # gated-MLP activation: textbook values of t * logistic(t)
    e = np.e
    h = o.silu_mul_f64(np.array([1.0, 2.0, 64.0, -64.0, 0.0]), np.array([2.0, 1.0, 3.0, 3.0, 5.0]))
    assert abs(h[0] - 2 * e / (1 + e)) < 1e-14 and abs(h[1] - 2 * e * e / (1 + e * e)) < 1e-14
    assert abs(h[2] - 192.0) < 1e-10 and abs(h[3]) < 1e-20 and h[4] == 0.0
    # entropy near the pages' ~2.6 bits
    st = o.stats(o.encode(wl.normal_with_outliers(64, 2048, 0.02, 0.0, 0)))
    assert 2.4 <= st["exp_entropy_bits"] <= 2.8
    # corruption: a flipped code nibble must be refused
    wc = wl.normal_with_outliers(8, 512, 0.02, 0.01, 4)
    bc = o.encode(wc)
    code = bc[256 + 4096: 256 + 4096 + 2048]
    k = int(np.nonzero((code & 0x0F) != 0x0F)[0][0])
    bc[256 + 4096 + k] |= 0x0F
    assert o.decode_rc(bc) != 0
    # ... and so must an escape code turned into an ordinary one
    bc = o.encode(wc)
    code = bc[256 + 4096: 256 + 4096 + 2048]
    k = int(np.nonzero((code & 0x0F) == 0x0F)[0][0])
    bc[256 + 4096 + k] &= 0xF0
    assert o.decode_rc(bc) != 0


def test_unmutated_oracle_passes_battery(oracle):
    _battery(oracle)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    src = open(SRC).read()
    for old, new in MUTANTS[name]:
        assert src.count(old) == 1, f"mutation anchor not unique/missing: {old!r}"
        src = src.replace(old, new)
    path = tmp_path / "mutant.c"
    path.write_text(src)
    lib = build_oracle.build(str(path), str(tmp_path / f"lib_{name}.so"), extra=("-w",))
    o = Oracle(load(lib))
    with pytest.raises(Exception):
        _battery(o)
    assert os.path.exists(lib)
