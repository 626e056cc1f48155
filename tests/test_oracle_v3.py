"""Container version 3 (packed 24-bit pairs; [T] technical deep dive: the
12-bit representation packed into 3-byte words, two weights per word) in
the oracle: exhaustive bit-exact round trips, a hand-derived golden
container, byte-for-byte agreement with the pinned version 1 (the pair plane
is version 1's raw and code planes regrouped; every other plane is the
same), the closed-form size and corruption checks."""
import numpy as np
import pytest

from conftest import golden_expected_bytes, golden_two_tiles_weights, load_golden
from decode_split12_b200 import workloads as wl

ALIGN = 256


def _pad(n):
    return (n + ALIGN - 1) // ALIGN * ALIGN


def _planes(sizes):
    out, off = [], ALIGN
    for sz in sizes:
        out.append((off, off + sz))
        off += _pad(sz)
    return out, off


def _v1_planes(rows, cols, n_esc):
    n_t = rows * cols // 128
    return _planes([rows * cols, rows * cols // 2, n_t, 4 * (n_t + 1), 2 * n_esc])


def _v3_planes(rows, cols, n_esc):
    n_t = rows * cols // 128
    return _planes([rows * cols * 3 // 2, n_t, 4 * (n_t + 1), 2 * n_esc])


@pytest.mark.parametrize("order", ["natural", "shuffled", "reversed_bits"])
def test_v3_roundtrip_all_patterns(oracle, order):
    p = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    if order == "shuffled":
        p = p[wl.rng_for(7, 3).permutation(p.size)]
    elif order == "reversed_bits":
        p = np.array([int(f"{i:016b}"[::-1], 2) for i in range(1 << 16)], np.uint16)
    w = p.reshape(512, 128)
    assert np.array_equal(oracle.decode_v3(oracle.encode_v3(w)), w)


@pytest.mark.parametrize("shape,kind", [((1, 128), "normal"), ((37, 640), "normal"), ((64, 1024), "stress"),
                                        ((16, 4096), "student")])
def test_v3_agrees_with_v1(oracle, shape, kind):
    r, c = shape
    if kind == "stress":
        w, _ = wl.escape_stress(0.02, 1, r, c)
    elif kind == "student":
        w = wl.student_t_scaled(r, c, 2)
    else:
        w = wl.normal_with_outliers(r, c, 0.02, 0.01, r + c)
    b1, b3 = oracle.encode(w), oracle.encode_v3(w)
    n_esc = int(b1[32:40].view(np.uint64)[0])
    assert int(b3[4:8].view(np.uint32)[0]) == 3
    h1, h3 = b1[:256].copy(), b3[:256].copy()
    h1[4:8] = h3[4:8] = 0
    assert np.array_equal(h1, h3)
    p1, t1 = _v1_planes(r, c, n_esc)
    p3, t3 = _v3_planes(r, c, n_esc)
    assert b3.size == t3 == oracle.container_bytes_v3(r, c, n_esc)
    pair = b3[p3[0][0]:p3[0][1]].reshape(-1, 3)
    raw = b1[p1[0][0]:p1[0][1]]
    code = b1[p1[1][0]:p1[1][1]]
    assert np.array_equal(pair[:, 0], raw[0::2]) and np.array_equal(pair[:, 1], raw[1::2])
    assert np.array_equal(pair[:, 2], code)
    for i in (1, 2, 3):     # base, esc_off, escapes
        assert np.array_equal(b1[p1[i + 1][0]:p1[i + 1][1]], b3[p3[i][0]:p3[i][1]])
    assert np.array_equal(oracle.decode_v3(b3), w)


def test_v3_payload_is_12_bits(oracle):
    """The pair plane holds exactly 1.5 bytes per weight, the fixed 12-bit
    rate ([T] key points: 1.33x smaller than BF16)."""
    for r, c in [(2, 128), (4096, 4096), (14336, 4096)]:
        p3, _ = _v3_planes(r, c, 0)
        assert (p3[0][1] - p3[0][0]) * 8 == 12 * r * c


def test_v3_golden_two_tiles_bytes(oracle):
    g1 = load_golden("two_tiles.json")
    g3 = load_golden("two_tiles_v3.json")
    expect = golden_expected_bytes(g1)
    for a, b in g3["clear"]:
        expect[a:b] = 0
    for item in g3["patch"]:
        off, hexs = item[0], item[1]
        reps = item[2] if len(item) > 2 else 1
        chunk = np.frombuffer(bytes.fromhex(hexs) * reps, np.uint8)
        expect[off:off + chunk.size] = chunk
    w = golden_two_tiles_weights(g1)
    assert np.array_equal(oracle.encode_v3(w), expect)
    assert np.array_equal(oracle.decode_v3(expect), w)


def test_v3_corruptions_detected(oracle):
    w, _ = wl.escape_stress(0.05, 4, 16, 1024)
    b = oracle.encode_v3(w)
    n_esc = int(b[32:40].view(np.uint64)[0])
    p3, _ = _v3_planes(16, 1024, n_esc)
    (q0, q1), (b0, _), (o0, _) = p3[0], p3[1], p3[2]
    pair = b[q0:q1].reshape(-1, 3)
    k_plain = int(np.flatnonzero((pair[:, 2] & 0x0F) != 0x0F)[7])
    k_esc = int(np.flatnonzero((pair[:, 2] & 0x0F) == 0x0F)[0])

    def bad(mutate):
        c = b.copy()
        mutate(c)
        return oracle.decode_v3_rc(c) != 0

    assert not bad(lambda c: None)
    assert bad(lambda c: c.__setitem__(q0 + 3 * k_plain + 2, c[q0 + 3 * k_plain + 2] | 0x0F))  # code -> escape
    assert bad(lambda c: c.__setitem__(q0 + 3 * k_esc + 2, c[q0 + 3 * k_esc + 2] & 0xF0))      # escape -> code
    assert bad(lambda c: c.__setitem__(b0 + 3, 242))                                             # base
    assert bad(lambda c: c.__setitem__(slice(o0, o0 + 4), np.frombuffer(np.uint32(1).tobytes(), np.uint8)))
    assert bad(lambda c: c.__setitem__(4, 1))                                                    # version
    # a version 1 container is not a version 3 one
    assert oracle.decode_v3_rc(oracle.encode(w)) != 0
