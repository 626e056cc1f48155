"""Container version 2 (compact tile header) in the oracle, pinned before any
kernel reads it: exhaustive bit-exact round trips, byte-for-byte agreement
with the pinned version 1 on the planes they share (raw, code, escapes) and
on the metadata version 2 derives from version 1's (base, per-tile escape
counts, per-row offsets), the closed-form size, and corruption checks."""
import numpy as np
import pytest

from conftest import golden_expected_bytes, golden_two_tiles_weights, load_golden
from decode_split12_b200 import workloads as wl

ALIGN = 256


def _pad(n):
    return (n + ALIGN - 1) // ALIGN * ALIGN


def _v1_planes(rows, cols, n_esc):
    n_t = rows * cols // 128
    sizes = [rows * cols, rows * cols // 2, n_t, 4 * (n_t + 1), 2 * n_esc]
    out, off = [], ALIGN
    for sz in sizes:
        out.append((off, off + sz))
        off += _pad(sz)
    return out, off


def _v2_planes(rows, cols, n_esc):
    n_t = rows * cols // 128
    sizes = [rows * cols, rows * cols // 2, 2 * n_t, 4 * (rows + 1), 2 * n_esc]
    out, off = [], ALIGN
    for sz in sizes:
        out.append((off, off + sz))
        off += _pad(sz)
    return out, off


@pytest.mark.parametrize("order", ["natural", "shuffled"])
def test_v2_roundtrip_all_patterns(oracle, order):
    p = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    if order == "shuffled":
        p = p[wl.rng_for(7, 2).permutation(p.size)]
    w = p.reshape(512, 128)
    assert np.array_equal(oracle.decode_v2(oracle.encode_v2(w)), w)


@pytest.mark.parametrize("shape,kind", [((1, 128), "normal"), ((37, 640), "normal"), ((64, 1024), "stress"),
                                        ((16, 4096), "student")])
def test_v2_agrees_with_v1(oracle, shape, kind):
    r, c = shape
    if kind == "stress":
        w, _ = wl.escape_stress(0.02, 1, r, c)
    elif kind == "student":
        w = wl.student_t_scaled(r, c, 2)
    else:
        w = wl.normal_with_outliers(r, c, 0.02, 0.01, r + c)
    b1, b2 = oracle.encode(w), oracle.encode_v2(w)
    n_esc = int(b1[32:40].view(np.uint64)[0])
    assert int(b2[32:40].view(np.uint64)[0]) == n_esc
    assert int(b2[4:8].view(np.uint32)[0]) == 2 and int(b1[4:8].view(np.uint32)[0]) == 1
    p1, t1 = _v1_planes(r, c, n_esc)
    p2, t2 = _v2_planes(r, c, n_esc)
    assert b1.size == t1 and b2.size == t2 == oracle.container_bytes_v2(r, c, n_esc)
    for i in (0, 1, 4):     # raw, code, esc: byte for byte
        assert np.array_equal(b1[p1[i][0]:p1[i][1]], b2[p2[i][0]:p2[i][1]])
    base1 = b1[p1[2][0]:p1[2][1]]
    off1 = b1[p1[3][0]:p1[3][1]].view(np.uint32)
    tmeta = b2[p2[2][0]:p2[2][1]].reshape(-1, 2)
    row_esc = b2[p2[3][0]:p2[3][1]].view(np.uint32)
    assert np.array_equal(tmeta[:, 0], base1)
    assert np.array_equal(tmeta[:, 1].astype(np.uint32), np.diff(off1))
    T = c // 128
    assert np.array_equal(row_esc, np.append(off1[::T][:r], off1[-1]))
    assert np.array_equal(oracle.decode_v2(b2), w)


def test_v2_metadata_saving_closed_form(oracle):
    """Unpadded metadata: version 1 has 5 bytes per tile + 4, version 2 has 2
    per tile + 4 per row + 4, so version 2 saves 3 bytes per tile minus 4 per
    row; for the 8B-style layer's shapes that is 0.1875 - 32/cols bits per
    weight."""
    for r, c in [(4096, 4096), (1024, 4096), (14336, 4096), (4096, 14336)]:
        n_t = r * c // 128
        v1 = 5 * n_t + 4
        v2 = 2 * n_t + 4 * (r + 1)
        assert (v1 - v2) * 8 / (r * c) == pytest.approx(3 * 8 / 128 - 32 / c)
        assert oracle.container_bytes_v2(r, c, 0) <= oracle.container_bytes(r, c, 0)


def test_v2_corruptions_detected(oracle):
    w, _ = wl.escape_stress(0.05, 4, 16, 1024)
    b = oracle.encode_v2(w)
    n_esc = int(b[32:40].view(np.uint64)[0])
    p2, _ = _v2_planes(16, 1024, n_esc)
    (t0, _), (r0, _) = p2[2], p2[3]
    tmeta = b[t0:t0 + 2 * 128].reshape(-1, 2)
    t_esc = int(np.flatnonzero(tmeta[:, 1] > 0)[0])

    def bad(mutate):
        c = b.copy()
        mutate(c)
        return oracle.decode_v2_rc(c) != 0

    assert not bad(lambda c: None)
    assert bad(lambda c: c.__setitem__(t0 + 2 * t_esc + 1, c[t0 + 2 * t_esc + 1] + 1))   # tile count
    assert bad(lambda c: c.__setitem__(t0 + 2 * 3, 242))                                  # base
    assert bad(lambda c: c.__setitem__(slice(r0, r0 + 4), np.frombuffer(np.uint32(1).tobytes(), np.uint8)))
    assert bad(lambda c: c.__setitem__(slice(r0 + 4 * 16, r0 + 4 * 17),
                                       np.frombuffer(np.uint32(n_esc + 1).tobytes(), np.uint8)))
    assert bad(lambda c: c.__setitem__(slice(r0 + 4 * 5, r0 + 4 * 6),
                                       np.frombuffer(np.uint32(0).tobytes(), np.uint8)))       # row offsets
    assert bad(lambda c: c.__setitem__(4, 1))                                               # version 1 header
    # a version 1 container is not a version 2 one
    assert oracle.decode_v2_rc(oracle.encode(w)) != 0


def test_v2_golden_two_tiles_bytes(oracle):
    """The hand-derived version 2 container of the two-tile golden tensor
    (tests/golden/two_tiles_v2.json: the version 1 golden bytes with the
    version field and the two tile headers changed)."""
    g1 = load_golden("two_tiles.json")
    g2 = load_golden("two_tiles_v2.json")
    expect = golden_expected_bytes(g1)
    for off, hexs in g2["patch"]:
        chunk = np.frombuffer(bytes.fromhex(hexs), np.uint8)
        expect[off:off + chunk.size] = chunk
    w = golden_two_tiles_weights(g1)
    assert np.array_equal(oracle.encode_v2(w), expect)
    assert np.array_equal(oracle.decode_v2(expect), w)
