"""Host-side container validation and plane hashes, with a corruption-
injection suite (no GPU needed): every corruption is judged the same way by
the library's validator and by the oracle's decoder (an independent
implementation of the container definition), with the expected problem
named; byte changes that leave the structure intact (raw bytes, escape
values) are caught by the plane hashes instead."""
import numpy as np
import pytest

from decode_split12_b200 import s12
from decode_split12_b200 import workloads as wl

ALIGN = 256


def _pad(n):
    return (n + ALIGN - 1) // ALIGN * ALIGN


def _planes(rows, cols, n_esc):
    """Byte ranges of the planes, from the container layout (256-byte header,
    then raw, code, base, esc_off, esc, each padded to 256 bytes)."""
    n_t = rows * cols // 128
    sizes = [rows * cols, rows * cols // 2, n_t, 4 * (n_t + 1), 2 * n_esc]
    out, off = [], ALIGN
    for sz in sizes:
        out.append((off, off + sz))
        off += _pad(sz)
    return out


def test_fnv1a64_published_vectors():
    """The FNV-1a 64-bit test vectors of the function's published
    definition."""
    assert s12.s12_fnv1a64(b"") == 0xCBF29CE484222325
    assert s12.s12_fnv1a64(b"a") == 0xAF63DC4C8601EC8C
    assert s12.s12_fnv1a64(b"foobar") == 0x85944171F73967E8


@pytest.fixture(scope="module")
def blob(oracle):
    w, n = wl.escape_stress(0.02, 3, 64, 512)   # escapes in most tiles
    b = oracle.encode(w)
    return b, w.shape, n


def test_valid_containers(oracle):
    for i, (r, c) in enumerate([(1, 128), (37, 640), (64, 4096)]):
        b = oracle.encode(wl.normal_with_outliers(r, c, 0.02, 0.01, i))
        rc, rep = s12.s12_validate_host(b)
        assert rc == s12.S12_OK and rep["problem"] is None and rep["notes"] == 0
        assert rep["n_esc_counted"] == int(np.frombuffer(b[32:40].tobytes(), np.uint64)[0])


def _corrupt_and_judge(oracle, b, mutate):
    c = b.copy()
    mutate(c)
    rc, rep = s12.s12_validate_host(c)
    orc_bad = oracle.decode_rc(c) != 0
    assert (rc != s12.S12_OK) == orc_bad, (rc, rep)
    return rc, rep


def _u32_at(c, off, v):
    c[off:off + 4] = np.frombuffer(np.uint32(v).tobytes(), np.uint8)


def test_header_corruptions(oracle, blob):
    b, _, _ = blob
    cases = {
        "magic": lambda c: c.__setitem__(1, ord("X")),
        "version": lambda c: _u32_at(c, 4, 2),
        "tile": lambda c: _u32_at(c, 24, 64),
        "flags": lambda c: _u32_at(c, 28, 1),
        "reserved": lambda c: c.__setitem__(50, 7),
        "cols": lambda c: c.__setitem__(16, 100),
    }
    for name, f in cases.items():
        rc, rep = _corrupt_and_judge(oracle, b, f)
        assert rc == s12.S12_ERR_CORRUPT and rep["problem"] == "header", name


def test_size_and_offset_corruptions(oracle, blob):
    b, (rows, cols), n_esc = blob
    (_, _), (_, _), (_, _), (o0, o1), _ = _planes(rows, cols, n_esc)
    n_t = rows * cols // 128
    rc, rep = _corrupt_and_judge(oracle, b[:-1], lambda c: None)
    assert rep["problem"] == "size"
    rc, rep = _corrupt_and_judge(oracle, b, lambda c: _u32_at(c, o0, 1))
    assert rep["problem"] == "offsets"
    rc, rep = _corrupt_and_judge(oracle, b, lambda c: _u32_at(c, o0 + 4 * n_t, n_esc + 1))
    assert rep["problem"] == "offsets"
    # a middle offset moved below its predecessor: tile t-1 now ends before it starts
    t = n_t // 2
    rc, rep = _corrupt_and_judge(oracle, b, lambda c: _u32_at(c, o0 + 4 * t, 0))
    assert rc == s12.S12_ERR_CORRUPT and rep["problem"] in ("tile_offsets", "esc_count")
    # a middle offset moved past the end of the stream
    rc, rep = _corrupt_and_judge(oracle, b, lambda c: _u32_at(c, o0 + 4 * t, n_esc + 5))
    assert rep["problem"] == "tile_offsets"


def test_base_and_code_corruptions(oracle, blob):
    b, (rows, cols), n_esc = blob
    _, (c0, _), (b0, _), _, _ = _planes(rows, cols, n_esc)
    rc, rep = _corrupt_and_judge(oracle, b, lambda c: c.__setitem__(b0 + 5, 242))
    assert rep["problem"] == "base" and rep["tile"] == 5
    # a code nibble turned into an escape, and an escape turned into a code
    codes = b[c0:c0 + rows * cols // 2]
    lo_nib = codes & 0x0F
    k_plain = int(np.flatnonzero(lo_nib != 0x0F)[10])
    k_esc = int(np.flatnonzero(lo_nib == 0x0F)[0])
    rc, rep = _corrupt_and_judge(oracle, b, lambda c: c.__setitem__(c0 + k_plain, (c[c0 + k_plain] & 0xF0) | 0x0F))
    assert rep["problem"] == "esc_count" and rep["tile"] == (2 * k_plain) // 128
    rc, rep = _corrupt_and_judge(oracle, b, lambda c: c.__setitem__(c0 + k_esc, (c[c0 + k_esc] & 0xF0) | 0x03))
    assert rep["problem"] == "esc_count" and rep["tile"] == (2 * k_esc) // 128


def test_structure_free_bytes_caught_by_hashes(oracle, blob):
    """A raw byte, an escape value or a padding byte changed: the container
    stays valid for both implementations, but the changed plane's hash (and
    only that one) differs; padding only raises the note."""
    b, (rows, cols), n_esc = blob
    planes = _planes(rows, cols, n_esc)
    h0 = s12.s12_plane_hashes_host(b)
    for i, (lo, hi) in enumerate(planes):
        assert h0[i] == s12.s12_fnv1a64(b[lo:hi].tobytes())
    for plane, pos in ((0, 1000), (4, 6)):
        rc, rep = _corrupt_and_judge(oracle, b, lambda c: c.__setitem__(planes[plane][0] + pos,
                                                                         c[planes[plane][0] + pos] ^ 0x40))
        assert rc == s12.S12_OK
        c = b.copy()
        c[planes[plane][0] + pos] ^= 0x40
        h1 = s12.s12_plane_hashes_host(c)
        assert [h1[i] != h0[i] for i in range(5)] == [i == plane for i in range(5)]
    assert planes[3][1] + 3 < planes[4][0]   # inside esc_off's padding
    rc, rep = _corrupt_and_judge(oracle, b, lambda c: c.__setitem__(planes[3][1] + 3, 9))
    assert rc == s12.S12_OK and rep["notes"] == 1
    rc, rep = _corrupt_and_judge(oracle, b, lambda c: c.__setitem__(100, 1))   # header padding
    assert rc == s12.S12_OK and rep["notes"] == 1


@pytest.mark.parametrize("shape,kind", [((1, 128), "normal"), ((37, 640), "normal"), ((64, 1024), "stress"),
                                        ((16, 4096), "student")])
def test_v2_conversion_matches_oracle_and_round_trips(oracle, shape, kind):
    """The library's host conversion to container version 2 equals the
    oracle's version 2 encoder byte for byte, and converting back gives the
    version 1 container byte for byte."""
    r, c = shape
    if kind == "stress":
        w, _ = wl.escape_stress(0.02, 1, r, c)
    elif kind == "student":
        w = wl.student_t_scaled(r, c, 2)
    else:
        w = wl.normal_with_outliers(r, c, 0.02, 0.01, r + c)
    v1 = oracle.encode(w)
    v2 = s12.to_v2_host(v1)
    assert np.array_equal(v2, oracle.encode_v2(w))
    assert v2.size <= v1.size
    assert np.array_equal(s12.from_v2_host(v2), v1)


def test_v2_conversion_refuses_corrupt_sources(oracle):
    w, _ = wl.escape_stress(0.05, 4, 16, 1024)
    v1 = oracle.encode(w)
    bad = v1.copy()
    bad[1] = ord("X")
    with pytest.raises(s12.S12Error):
        s12.to_v2_host(bad)
    v2 = oracle.encode_v2(w)
    n_esc = int(v2[32:40].view(np.uint64)[0])
    n_t = 16 * 1024 // 128
    off_t = 256 + 16 * 1024 + 8192
    k = int(np.flatnonzero(v2[off_t + 1:off_t + 2 * n_t:2])[0])
    bad2 = v2.copy()
    bad2[off_t + 2 * k + 1] += 1            # a tile count that no longer adds up to its row's span
    with pytest.raises(s12.S12Error):
        s12.from_v2_host(bad2)
    with pytest.raises(s12.S12Error):
        s12.from_v2_host(v1)                # a version 1 container is not version 2
    assert n_esc > 0


def test_v2_conversion_of_the_golden_container():
    """The library's conversion of the hand-derived version 1 golden
    container gives the hand-derived version 2 bytes, and back."""
    from conftest import golden_expected_bytes, load_golden
    g1, g2 = load_golden("two_tiles.json"), load_golden("two_tiles_v2.json")
    v1 = golden_expected_bytes(g1)
    v2 = v1.copy()
    for off, hexs in g2["patch"]:
        chunk = np.frombuffer(bytes.fromhex(hexs), np.uint8)
        v2[off:off + chunk.size] = chunk
    assert np.array_equal(s12.to_v2_host(v1), v2)
    assert np.array_equal(s12.from_v2_host(v2), v1)


# ---------------------------------------------------------------------------
# container version 3 (packed 24-bit pairs) as a storage format

@pytest.mark.parametrize("shape,kind", [((1, 128), "normal"), ((37, 640), "normal"), ((64, 1024), "stress"),
                                        ((16, 4096), "student")])
def test_v3_conversion_matches_oracle(oracle, shape, kind):
    """The library's host conversion to version 3 equals the oracle's
    version 3 encoder byte for byte, and converting back gives the version
    1 container byte for byte."""
    r, c = shape
    if kind == "stress":
        w, _ = wl.escape_stress(0.02, 2, r, c)
    elif kind == "student":
        w = wl.student_t_scaled(r, c, 3)
    else:
        w = wl.normal_with_outliers(r, c, 0.02, 0.01, 2 * r + c)
    v1 = oracle.encode(w)
    v3 = s12.to_v3_host(v1)
    assert np.array_equal(v3, oracle.encode_v3(w))
    assert np.array_equal(s12.from_v3_host(v3), v1)


def test_v3_conversion_of_the_golden_container():
    from conftest import golden_expected_bytes, load_golden
    g1, g3 = load_golden("two_tiles.json"), load_golden("two_tiles_v3.json")
    v1 = golden_expected_bytes(g1)
    v3 = v1.copy()
    for a, b in g3["clear"]:
        v3[a:b] = 0
    for item in g3["patch"]:
        chunk = np.frombuffer(bytes.fromhex(item[1]) * (item[2] if len(item) > 2 else 1), np.uint8)
        v3[item[0]:item[0] + chunk.size] = chunk
    assert np.array_equal(s12.to_v3_host(v1), v3)
    assert np.array_equal(s12.from_v3_host(v3), v1)


def test_v3_conversion_refuses_corrupt_sources(oracle):
    w, _ = wl.escape_stress(0.05, 5, 16, 1024)
    v3 = oracle.encode_v3(w)
    pair0 = 256
    codes = v3[pair0 + 2:pair0 + 16 * 1024 * 3 // 2:3]
    k = int(np.flatnonzero((codes & 0x0F) != 0x0F)[3])
    bad = v3.copy()
    bad[pair0 + 3 * k + 2] |= 0x0F          # a code turned into an escape: the tile's count no longer matches
    with pytest.raises(s12.S12Error):
        s12.from_v3_host(bad)
    with pytest.raises(s12.S12Error):
        s12.from_v3_host(oracle.encode(w))  # a version 1 container is not version 3
    with pytest.raises(s12.S12Error):
        s12.to_v3_host(v3)                  # nor is a version 3 one version 1
