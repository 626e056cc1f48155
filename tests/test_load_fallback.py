"""Whole-tensor load with fallback to the original BF16 weights ([W] "A
14-day production-readiness pilot": check what was loaded, keep the original
weights, serve a failing tensor from them).

The corruption is injected into the HOST copy of a container (never on a
GPU).  The CPU tests cover every rejection, which s12_load_bf16 decides on
the host before any device work; the GPU tests cover the decode of a clean
container and the fallback copy."""
import numpy as np
import pytest
import torch

from decode_split12_b200 import s12
from decode_split12_b200 import workloads as wl

ALIGN = 256
# stand-in device addresses for rejections, which never touch device memory
FAKE_DEV = (1 << 40, 1 << 41, 1 << 42)


def _pad(n):
    return (n + ALIGN - 1) // ALIGN * ALIGN


def _planes(rows, cols, n_esc):
    """Byte ranges of the planes (256-byte header, then raw, code, base,
    esc_off, esc, each padded to 256 bytes)."""
    n_t = rows * cols // 128
    out, off = [], ALIGN
    for sz in [rows * cols, rows * cols // 2, n_t, 4 * (n_t + 1), 2 * n_esc]:
        out.append((off, off + sz))
        off += _pad(sz)
    return out


@pytest.fixture(scope="module")
def tensor(oracle):
    w, n_esc = wl.escape_stress(0.02, 11, 96, 1024)
    blob = oracle.encode(w)
    hashes = s12.s12_plane_hashes_host(blob)
    return w, blob, hashes, n_esc


def _reject(blob, rows, cols, hashes=None):
    d_c, d_o, d_e = FAKE_DEV
    return s12.s12_load_bf16(blob, rows, cols, d_c, d_o, d_e, expected_hashes=hashes, fallback=None)


def test_rejections_decided_on_the_host(tensor):
    """Every corruption the host checks see gives "rejected" without a BF16
    copy, with the finding named: a code nibble turned into an escape (count
    check), a base above 241, a raw byte and an escape value changed (plane
    hashes), and a header that describes another shape."""
    w, blob, hashes, n_esc = tensor
    rows, cols = w.shape
    (r0, _), (c0, _), (b0, _), _, (e0, _) = _planes(rows, cols, n_esc)

    c = blob.copy()
    k = int(np.flatnonzero((c[c0:c0 + rows * cols // 2] & 0x0F) != 0x0F)[3])
    c[c0 + k] = (c[c0 + k] & 0xF0) | 0x0F
    res = _reject(c, rows, cols)
    assert res["outcome"] == "rejected" and res["problem"] == "esc_count"

    c = blob.copy()
    c[b0 + 7] = 250
    res = _reject(c, rows, cols)
    assert res["outcome"] == "rejected" and res["problem"] == "base"

    c = blob.copy()
    c[r0 + 12345] ^= 0x01
    res = _reject(c, rows, cols, hashes)
    assert res["outcome"] == "rejected" and res["problem"] is None and res["hash_mismatch"] == 0b00001

    c = blob.copy()
    c[e0 + 2 * (n_esc // 2)] ^= 0x40
    res = _reject(c, rows, cols, hashes)
    assert res["outcome"] == "rejected" and res["hash_mismatch"] == 0b10000

    res = _reject(blob, rows + 1, cols)
    assert res["outcome"] == "rejected" and res["problem"] == "header"

    # without expected hashes a raw-byte change passes the structural checks
    # (it would be decoded): the hashes are what catch it
    c = blob.copy()
    c[r0 + 12345] ^= 0x01
    assert s12.s12_validate_host(c)[0] == s12.S12_OK


def test_argument_checks(tensor):
    w, blob, hashes, _ = tensor
    rows, cols = w.shape
    d_c, d_o, d_e = FAKE_DEV
    with pytest.raises(s12.S12Error):
        s12.s12_load_bf16(blob, rows, 100, d_c, d_o, d_e)          # cols % 128
    with pytest.raises(s12.S12Error):
        s12.s12_load_bf16(blob, rows, cols, d_c + 8, d_o, d_e)      # container not 256-aligned
    with pytest.raises(s12.S12Error):
        s12.s12_load_bf16(blob, 0, cols, d_c, d_o, d_e)


@pytest.mark.gpu
def test_clean_container_is_decoded(cuda_ok, tensor):
    w, blob, hashes, _ = tensor
    rows, cols = w.shape
    d_c = torch.empty(blob.size, dtype=torch.uint8, device="cuda")
    d_o = torch.zeros((rows, cols), dtype=torch.int16, device="cuda")
    d_e = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = s12.s12_load_bf16(blob, rows, cols, d_c, d_o, d_e, expected_hashes=hashes, fallback=w)
    assert res == {"outcome": "decoded", "problem": None, "hash_mismatch": 0, "device_flags": 0}
    assert np.array_equal(d_o.cpu().numpy().view(np.uint16), w)


@pytest.mark.gpu
@pytest.mark.parametrize("where", ["raw", "code", "escape"])
def test_corrupt_container_falls_back(cuda_ok, tensor, where):
    """A corrupted host copy is never decoded into the output: the output
    holds the caller's BF16 copy, bit for bit."""
    w, blob, hashes, n_esc = tensor
    rows, cols = w.shape
    (r0, _), (c0, _), _, _, (e0, _) = _planes(rows, cols, n_esc)
    c = blob.copy()
    if where == "raw":
        c[r0 + 777] ^= 0x80
    elif where == "code":
        k = int(np.flatnonzero((c[c0:c0 + rows * cols // 2] & 0x0F) != 0x0F)[5])
        c[c0 + k] = (c[c0 + k] & 0xF0) | 0x0F
    else:
        c[e0] ^= 0x01
    d_c = torch.empty(c.size, dtype=torch.uint8, device="cuda")
    d_o = torch.zeros((rows, cols), dtype=torch.int16, device="cuda")
    d_e = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = s12.s12_load_bf16(c, rows, cols, d_c, d_o, d_e, expected_hashes=hashes, fallback=w)
    assert res["outcome"] == "fallback"
    assert np.array_equal(d_o.cpu().numpy().view(np.uint16), w)
    res = s12.s12_load_bf16(c, rows, cols, d_c, d_o, d_e, expected_hashes=hashes, fallback=None)
    assert res["outcome"] == "rejected"
