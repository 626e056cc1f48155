"""Container version 4 (sign-and-exponent symbol codes; [W] "What did the
GLM-5.2 experiment actually prove?": short fixed codes for a tensor's common
sign-and-exponent symbols, rare ones to an escape stream) in the oracle:
a hand-derived golden container, exhaustive bit-exact round trips, the
symbol table and every code against brute force, the 12-bit payload and
corruption checks."""
import numpy as np
import pytest

from conftest import golden_expected_bytes, load_golden
from decode_split12_b200 import workloads as wl

ALIGN = 256


def _pad(n):
    return (n + ALIGN - 1) // ALIGN * ALIGN


def _v4_planes(rows, cols, n_esc):
    n_t = rows * cols // 128
    out, off = [], ALIGN
    for sz in [64, rows * cols, rows * cols // 2, 4 * (n_t + 1), 2 * n_esc]:
        out.append((off, off + sz))
        off += _pad(sz)
    return out, off


def _brute_table(w):
    """The 31 most frequent symbols (w >> 7), count descending, ties to the
    smaller symbol."""
    sym = (w.reshape(-1).astype(np.int64) >> 7)
    counts = np.bincount(sym, minlength=512)
    order = sorted(range(512), key=lambda s: (-counts[s], s))
    used = [s for s in order if counts[s] > 0][:31]
    return used, int(w.size - sum(counts[s] for s in used))


def test_v4_golden_one_tile(oracle):
    d = load_golden("one_tile_v4.json")
    w = np.array([int(h, 16) for h in d["weights"]], np.uint16).reshape(1, 128)
    expect = golden_expected_bytes(d)
    assert np.array_equal(oracle.encode_v4(w), expect)
    assert np.array_equal(oracle.decode_v4(expect), w)


@pytest.mark.parametrize("order", ["natural", "shuffled", "reversed_bits"])
def test_v4_roundtrip_all_patterns(oracle, order):
    p = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    if order == "shuffled":
        p = p[wl.rng_for(7, 4).permutation(p.size)]
    elif order == "reversed_bits":
        p = np.array([int(f"{i:016b}"[::-1], 2) for i in range(1 << 16)], np.uint16)
    w = p.reshape(512, 128)
    assert np.array_equal(oracle.decode_v4(oracle.encode_v4(w)), w)


@pytest.mark.parametrize("kind", ["normal", "student", "stress", "few_symbols", "random_bits"])
def test_v4_table_and_codes_brute_force(oracle, kind):
    if kind == "normal":
        w = wl.normal_with_outliers(64, 512, 0.02, 0.01, 3)
    elif kind == "student":
        w = wl.student_t_scaled(32, 1024, 4)
    elif kind == "stress":
        w, _ = wl.escape_stress(0.02, 5, 32, 1024)
    elif kind == "few_symbols":
        w = np.tile(np.array([0x3F80, 0xBF80, 0x4000, 0x0000], np.uint16), (8, 64))
    else:
        w = wl.rng_for(6, 0).integers(0, 1 << 16, size=(16, 256)).astype(np.uint16)
    used, n_out = _brute_table(w)
    table, n_o = oracle.symbol_table(w)
    assert n_o == n_out
    assert list(table[:len(used)]) == used and all(t == 0xFFFF for t in table[len(used):31]) and table[31] == 0
    b = oracle.encode_v4(w)
    r, c = w.shape
    n_esc = int(b[32:40].view(np.uint64)[0])
    assert n_esc == n_out
    planes, total = _v4_planes(r, c, n_esc)
    assert b.size == total == oracle.container_bytes_v4(r, c, n_esc)
    raw = b[planes[1][0]:planes[1][1]]
    nib = b[planes[2][0]:planes[2][1]]
    nibs = np.stack([nib & 0x0F, nib >> 4], axis=1).reshape(-1)
    code = (nibs.astype(np.int64) << 1) | (raw >> 7)
    idx = {s: i for i, s in enumerate(used)}
    want = np.array([idx.get(int(s), 31) for s in (w.reshape(-1).astype(np.int64) >> 7)])
    assert np.array_equal(code, want)
    assert np.array_equal(raw & 0x7F, (w.reshape(-1) & 0x7F).astype(np.uint8))
    esc = b[planes[4][0]:planes[4][1]].view(np.uint16)
    assert np.array_equal(esc, w.reshape(-1)[want == 31])
    assert np.array_equal(oracle.decode_v4(b), w)


def test_v4_payload_is_12_bits():
    """Raw and code planes: exactly 1.5 bytes per weight."""
    for r, c in [(1, 128), (4096, 4096)]:
        planes, _ = _v4_planes(r, c, 0)
        assert ((planes[1][1] - planes[1][0]) + (planes[2][1] - planes[2][0])) * 8 == 12 * r * c


def test_v4_corruptions_detected(oracle):
    w, _ = wl.escape_stress(0.05, 7, 16, 1024)
    b = oracle.encode_v4(w)
    n_esc = int(b[32:40].view(np.uint64)[0])
    planes, _ = _v4_planes(16, 1024, n_esc)
    (t0, _), (r0, _), (c0, _), (o0, _) = planes[0], planes[1], planes[2], planes[3]

    def bad(mutate):
        c = b.copy()
        mutate(c)
        return oracle.decode_v4_rc(c) != 0

    codes = ((np.stack([b[c0:c0 + 8192] & 0x0F, b[c0:c0 + 8192] >> 4], 1).reshape(-1).astype(np.int64) << 1)
             | (b[r0:r0 + 16384] >> 7))
    k_plain = int(np.flatnonzero(codes < 31)[11])
    assert not bad(lambda c: None)
    # a plain weight turned into an escape (nibble 15 and code bit 1)
    def to_escape(c):
        c[r0 + k_plain] |= 0x80
        c[c0 + k_plain // 2] |= 0x0F if k_plain % 2 == 0 else 0xF0
    assert bad(to_escape)
    assert bad(lambda c: c.__setitem__(slice(t0, t0 + 2), np.frombuffer(np.uint16(600).tobytes(), np.uint8)))
    assert bad(lambda c: c.__setitem__(slice(o0, o0 + 4), np.frombuffer(np.uint32(1).tobytes(), np.uint8)))
    assert bad(lambda c: c.__setitem__(4, 1))
    assert oracle.decode_v4_rc(oracle.encode(w)) != 0


def test_v4_code_of_unused_entry_refused(oracle):
    """A code that points at an unused table entry (a tensor with 4 symbols
    has 27) is corruption, not a weight."""
    w = np.tile(np.array([0x3F80, 0xBF80, 0x4000, 0x0000], np.uint16), (2, 64))
    b = oracle.encode_v4(w)
    planes, _ = _v4_planes(2, 256, 0)
    c = b.copy()
    c[planes[2][0]] = (c[planes[2][0]] & 0xF0) | 0x03   # weight 0: code 6 or 7
    assert oracle.decode_v4_rc(c) != 0
