"""GPU parity of the encoder, the standalone decoder and the statistics
against the CPU oracle: containers byte-for-byte, decodes bit-exact."""
import numpy as np
import pytest
import torch

from conftest import golden_expected_bytes, golden_two_tiles_weights, load_golden
from decode_split12_b200 import workloads as wl
from gpu_util import blob_to_dev, blob_to_host, from_dev_u16, new_flag, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def s12(cuda_ok):
    from decode_split12_b200 import s12 as mod
    mod.device_check()
    return mod


def _all_patterns(order):
    p = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    if order == "shuffled":
        p = p[wl.rng_for(0, 1).permutation(p.size)]
    elif order == "bitreversed":
        a = p.astype(np.uint32)
        r = np.zeros_like(a)
        for i in range(16):
            r |= ((a >> i) & 1) << (15 - i)
        p = r.astype(np.uint16)
    return p.reshape(512, 128)


def _roundtrip(s12, oracle, w, check_oracle=True):
    wd = to_dev(w)
    blob = s12.s12_encode(wd)
    host = blob_to_host(blob)
    if check_oracle:
        ref = oracle.encode(w)
        assert host.size == ref.size
        diff = np.nonzero(host != ref)[0]
        assert diff.size == 0, f"{diff.size} container bytes differ, first at {diff[:8]}"
    view = s12.s12_open(blob)
    flag = new_flag()
    out = s12.s12_decode(view, err_flag=flag)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev_u16(out), w)
    assert int(flag.item()) == 0
    return blob, view


def test_golden_two_tiles(s12, oracle):
    d = load_golden("two_tiles.json")
    w = golden_two_tiles_weights(d)
    blob, _ = _roundtrip(s12, oracle, w)
    assert np.array_equal(blob_to_host(blob), golden_expected_bytes(d))


@pytest.mark.parametrize("order", ["natural", "shuffled", "bitreversed"])
def test_all_bf16_patterns(s12, oracle, order):
    _roundtrip(s12, oracle, _all_patterns(order))


@pytest.mark.parametrize("shape", [(1, 128), (3, 256), (2, 384), (67, 384), (300, 1152), (33, 4096), (5, 14336)])
@pytest.mark.parametrize("kind", ["normal", "uniform_bits", "student_t"])
def test_small_shapes(s12, oracle, shape, kind):
    r, c = shape
    if kind == "normal":
        w = wl.normal_with_outliers(r, c, 0.02, 0.01, 11)
    elif kind == "uniform_bits":
        w = wl.rng_for(12, 0).integers(0, 1 << 16, size=(r, c)).astype(np.uint16)
    else:
        w = wl.student_t_scaled(r, c, 13)
    _roundtrip(s12, oracle, w)


def test_every_exponent_base_extreme(s12, oracle):
    """Tiles pinned at exponent 0 and 255 (zeros, subnormals, Inf/NaN) and
    tiles whose best base is 241."""
    g = wl.rng_for(21, 0)
    rows = []
    for lo in (0, 1, 120, 240, 241, 250):
        e = g.integers(lo, min(lo + 15, 256), size=128)
        rows.append(((g.integers(0, 2, 128) << 15) | (e << 7) | g.integers(0, 128, 128)).astype(np.uint16))
    w = np.stack(rows)
    _roundtrip(s12, oracle, w)


@pytest.mark.parametrize("rate", wl.ESCAPE_RATES)
def test_escape_stress_reduced(s12, oracle, rate):
    w, planted = wl.escape_stress(rate, seed=0, rows=512, cols=2048)
    _, view = _roundtrip(s12, oracle, w)
    assert view.n_esc == planted


def test_single_tensor_full_size(s12, oracle):
    """4096 x 4096, N(0, 0.02) with 0.1 % outliers: container byte-for-byte."""
    w, _ = wl.single_tensor(0)
    _roundtrip(s12, oracle, w)


_FULL_SHAPES = {
    "llama8b_kv_1024x4096": lambda: wl.llama8b_layer(0, 1, names=["k"])[0]["k"],
    "llama8b_q_4096x4096": lambda: wl.llama8b_layer(0, 1, names=["q"])[0]["q"],
    "llama8b_gate_14336x4096": lambda: wl.llama8b_layer(0, 1, names=["gate"])[0]["gate"],
    "llama8b_down_4096x14336": lambda: wl.llama8b_layer(0, 1, names=["down"])[0]["down"],
    "mlp70b_up_28672x8192": lambda: wl.mlp70b("up", 0),
    "mlp70b_down_8192x28672": lambda: wl.mlp70b("down", 0),
}


@pytest.mark.parametrize("name", list(_FULL_SHAPES))
def test_encode_full_shapes_byte_exact(s12, oracle, name):
    """Every full-size matrix the GEMV and GEMM parity tests and the bench
    use: the GPU encoder's container equals the oracle's byte for byte, and
    the GPU decode gives W back bit for bit ("What does 'lossless' mean for
    LLM weights?": the exact round trip is the definition)."""
    w = _FULL_SHAPES[name]()
    _roundtrip(s12, oracle, w)


@pytest.mark.parametrize("rate", wl.ESCAPE_RATES)
def test_escape_stress_full_size_decode(s12, oracle, rate):
    """8192 x 8192 at each escape rate: exact escape count and bit-exact
    decode; the container is compared with the oracle at one rate."""
    w, planted = wl.escape_stress(rate, seed=0)
    _, view = _roundtrip(s12, oracle, w, check_oracle=(rate == 0.02))
    assert view.n_esc == planted


def test_decode_is_deterministic_and_idempotent(s12, oracle):
    w = wl.normal_with_outliers(64, 1024, 0.02, 0.01, 5)
    blob, view = _roundtrip(s12, oracle, w)
    a = s12.s12_decode(view)
    b = s12.s12_decode(view)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_corruption_sets_flag_without_hanging(s12, oracle):
    """A flipped code nibble and a wrong offset raise the error flag; the
    kernel still finishes (wavect, 14-day pilot step 2: inject corruption and
    confirm it is detected)."""
    w = wl.normal_with_outliers(16, 1024, 0.02, 0.01, 4)
    ref = oracle.encode(w)
    code_off = 256 + 16 * 1024
    code = ref[code_off: code_off + 8 * 1024]
    k = int(np.nonzero((code & 0x0F) != 0x0F)[0][0])
    bad = ref.copy()
    bad[code_off + k] |= 0x0F
    for blob_np in (bad,):
        blob = blob_to_dev(blob_np)
        view = s12.s12_open(blob)
        flag = new_flag()
        s12.s12_decode(view, err_flag=flag)
        y = s12.s12_gemv(view, to_dev(wl.activations(1, 1024, 0)), err_flag=flag)
        torch.cuda.synchronize()
        assert int(flag.item()) & s12.S12_FLAG_ESC_COUNT
        assert y.shape == (1, 16)
    # an escape code turned into an ordinary one
    k = int(np.nonzero((code & 0x0F) == 0x0F)[0][0])
    bad = ref.copy()
    bad[code_off + k] &= 0xF0
    view = s12.s12_open(blob_to_dev(bad))
    flag = new_flag()
    s12.s12_decode(view, err_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) & s12.S12_FLAG_ESC_COUNT
    # a header the opener must refuse
    hdr = ref.copy()
    hdr[0] ^= 1
    with pytest.raises(s12.S12Error):
        s12.s12_open(blob_to_dev(hdr))


def test_stats_match_oracle(s12, oracle):
    for w in (wl.student_t_scaled(256, 4096, 0), wl.escape_stress(0.0023, 0, 256, 2048)[0],
              _all_patterns("shuffled")):
        blob, view = _roundtrip(s12, oracle, w, check_oracle=False)
        got = s12.s12_stats(view)
        ref = oracle.stats(blob_to_host(blob))
        assert list(ref["exp_hist"]) == got["exp_hist"]
        for key in ("rows", "cols", "n_tiles", "n_esc", "container_bytes", "payload_bytes", "header_bytes",
                    "escape_bytes"):
            assert got[key] == ref[key], key
        for key in ("escape_rate", "bits_per_weight", "ratio_vs_bf16", "payload_ratio", "exp_entropy_bits"):
            assert abs(got[key] - ref[key]) <= 1e-12 * max(1.0, abs(ref[key])), key


def test_size_query_and_capacity(s12, oracle):
    import ctypes as C
    w = wl.normal_with_outliers(8, 256, 0.02, 0.05, 2)
    wd = to_dev(w)
    lib = s12.lib()
    ws = torch.empty(lib.s12_encode_ws_bytes(8, 256), dtype=torch.uint8, device="cuda")
    n = C.c_size_t(0)
    st = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.s12_encode(C.c_void_p(wd.data_ptr()), 8, 256, None, 0, C.byref(n), C.c_void_p(ws.data_ptr()),
                          ws.numel(), st) == 0
    assert n.value == oracle.encode_size(w)
    exact = n.value
    # too small for the escapes only, and smaller than the escape-free size:
    # both report S12_ERR_CAPACITY with the size needed
    for cap in (exact - 256, 512):
        small = torch.zeros(cap, dtype=torch.uint8, device="cuda")
        n2 = C.c_size_t(0)
        rc = lib.s12_encode(C.c_void_p(wd.data_ptr()), 8, 256, C.c_void_p(small.data_ptr()), small.numel(),
                            C.byref(n2), C.c_void_p(ws.data_ptr()), ws.numel(), st)
        assert rc == s12.S12_ERR_CAPACITY and n2.value == exact
    # and a destination of the reported size gets the oracle's container
    blob = torch.zeros(exact, dtype=torch.uint8, device="cuda")
    assert lib.s12_encode(C.c_void_p(wd.data_ptr()), 8, 256, C.c_void_p(blob.data_ptr()), exact, C.byref(n),
                          C.c_void_p(ws.data_ptr()), ws.numel(), st) == 0
    assert np.array_equal(blob.cpu().numpy(), oracle.encode(w))


# ---------------------------------------------------------------------------
# container version 2 on the GPU: the decoder and the statistics read it

@pytest.mark.parametrize("order", ["natural", "shuffled"])
def test_v2_decode_all_patterns(s12, oracle, order):
    """All 65,536 BF16 patterns as a version 2 container built by the oracle:
    the GPU decode gives every bit back and raises no flag."""
    w = _all_patterns(order)
    blob = blob_to_dev(oracle.encode_v2(w))
    view = s12.s12_open(blob)
    assert view.version == 2
    flag = new_flag()
    out = s12.s12_decode(view, err_flag=flag)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev_u16(out), w)
    assert int(flag.item()) == 0


@pytest.mark.parametrize("shape", [(1, 128), (3, 384), (67, 384), (300, 1152), (33, 4096), (5, 14336)])
@pytest.mark.parametrize("rate", [0.0003, 0.10])
def test_v2_decode_shapes_and_escape_rates(s12, oracle, shape, rate):
    """Version 2 decode at a low and a high escape rate, over chunks that
    cross row boundaries and ragged final chunks (n_tiles not a multiple of
    32): bit-exact against the source matrix."""
    r, c = shape
    w, _ = wl.escape_stress(rate, r + c, r, c)
    blob = blob_to_dev(oracle.encode_v2(w))
    view = s12.s12_open(blob)
    flag = new_flag()
    out = s12.s12_decode(view, err_flag=flag)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev_u16(out), w)
    assert int(flag.item()) == 0


def test_v2_decode_full_size_escape_stress(s12, oracle):
    """8192 x 8192 at 2 % escapes as a version 2 container: bit-exact."""
    w, planted = wl.escape_stress(0.02, seed=0)
    blob = blob_to_dev(oracle.encode_v2(w))
    view = s12.s12_open(blob)
    assert view.n_esc == planted
    flag = new_flag()
    out = s12.s12_decode(view, err_flag=flag)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), to_dev(w))
    assert int(flag.item()) == 0


def test_v2_stats_match_v1(s12, oracle):
    """The statistics of a version 2 container: the same exponent histogram
    and entropy as the oracle's statistics of the version 1 container, and
    the header bytes of version 2 (2 per tile + 4 per row)."""
    w = wl.student_t_scaled(300, 1152, 5)
    ref = oracle.stats(oracle.encode(w))
    view = s12.s12_open(blob_to_dev(oracle.encode_v2(w)))
    st = s12.s12_stats(view)
    assert st["exp_hist"] == [int(h) for h in ref["exp_hist"]]
    assert st["exp_entropy_bits"] == pytest.approx(ref["exp_entropy_bits"], abs=1e-12)
    assert st["header_bytes"] == 2 * view.n_tiles + 4 * (view.rows + 1)
    assert st["n_esc"] == ref["n_esc"]


# ---------------------------------------------------------------------------
# container version 3 (packed 24-bit pairs), built by the oracle

@pytest.mark.parametrize("order", ["natural", "shuffled"])
def test_v3_decode_all_patterns(s12, oracle, order):
    """All 65,536 BF16 patterns as a version 3 container (two weights per
    3 bytes; [T] technical deep dive): the GPU decode gives every bit back."""
    w = _all_patterns(order)
    view = s12.s12_open(blob_to_dev(oracle.encode_v3(w)))
    assert view.version == 3
    flag = new_flag()
    out = s12.s12_decode(view, err_flag=flag)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev_u16(out), w)
    assert int(flag.item()) == 0


@pytest.mark.parametrize("shape", [(1, 128), (3, 384), (67, 384), (300, 1152), (5, 14336)])
@pytest.mark.parametrize("rate", [0.0003, 0.10])
def test_v3_decode_shapes_and_escape_rates(s12, oracle, shape, rate):
    r, c = shape
    w, _ = wl.escape_stress(rate, 3 * r + c, r, c)
    view = s12.s12_open(blob_to_dev(oracle.encode_v3(w)))
    flag = new_flag()
    out = s12.s12_decode(view, err_flag=flag)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev_u16(out), w)
    assert int(flag.item()) == 0


def test_v3_decode_full_size_and_stats(s12, oracle):
    """8192 x 8192 at 2 % escapes as a version 3 container: bit-exact; its
    statistics equal the oracle's of the version 1 container; the fused
    products refuse version 3 (they read versions 1 and 2)."""
    w, planted = wl.escape_stress(0.02, seed=1)
    view = s12.s12_open(blob_to_dev(oracle.encode_v3(w)))
    assert view.n_esc == planted
    flag = new_flag()
    out = s12.s12_decode(view, err_flag=flag)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), to_dev(w))
    assert int(flag.item()) == 0
    small = wl.student_t_scaled(300, 1152, 6)
    ref = oracle.stats(oracle.encode(small))
    v3 = s12.s12_open(blob_to_dev(oracle.encode_v3(small)))
    st = s12.s12_stats(v3)
    assert st["exp_hist"] == [int(h) for h in ref["exp_hist"]]
    assert st["n_esc"] == ref["n_esc"]
    with pytest.raises(s12.S12Error):
        s12.s12_gemv(v3, to_dev(wl.activations(1, 1152, 0)))
    with pytest.raises(s12.S12Error):
        s12.s12_gemm_skinny(v3, to_dev(wl.activations(16, 1152, 0)))


# ---------------------------------------------------------------------------
# container version 4 (sign-and-exponent symbol codes), built by the oracle

@pytest.mark.parametrize("order", ["natural", "shuffled"])
def test_v4_decode_all_patterns(s12, oracle, order):
    """All 65,536 BF16 patterns as a version 4 container (a tensor table of
    31 sign+exponent symbols; [W] "What did the GLM-5.2 experiment actually
    prove?"): the GPU decode gives every bit back."""
    w = _all_patterns(order)
    view = s12.s12_open(blob_to_dev(oracle.encode_v4(w)))
    assert view.version == 4
    flag = new_flag()
    out = s12.s12_decode(view, err_flag=flag)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev_u16(out), w)
    assert int(flag.item()) == 0


@pytest.mark.parametrize("shape", [(1, 128), (3, 384), (67, 384), (300, 1152), (5, 14336)])
@pytest.mark.parametrize("kind", ["student", "stress"])
def test_v4_decode_shapes(s12, oracle, shape, kind):
    r, c = shape
    w = wl.student_t_scaled(r, c, r + c) if kind == "student" else wl.escape_stress(0.05, r + 2 * c, r, c)[0]
    view = s12.s12_open(blob_to_dev(oracle.encode_v4(w)))
    flag = new_flag()
    out = s12.s12_decode(view, err_flag=flag)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev_u16(out), w)
    assert int(flag.item()) == 0


def test_v4_decode_full_size_and_stats(s12, oracle):
    """The 8B-style gate projection (14336 x 4096) as a version 4 container:
    bit-exact; its statistics equal the oracle's of the version 1 container;
    the fused products refuse version 4."""
    w = wl.student_t_scaled(14336, 4096, 0, 4)
    view = s12.s12_open(blob_to_dev(oracle.encode_v4(w)))
    flag = new_flag()
    out = s12.s12_decode(view, err_flag=flag)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), to_dev(w))
    assert int(flag.item()) == 0
    small = wl.student_t_scaled(300, 1152, 7)
    ref = oracle.stats(oracle.encode(small))
    v4 = s12.s12_open(blob_to_dev(oracle.encode_v4(small)))
    st = s12.s12_stats(v4)
    assert st["exp_hist"] == [int(h) for h in ref["exp_hist"]]
    with pytest.raises(s12.S12Error):
        s12.s12_gemv(v4, to_dev(wl.activations(1, 1152, 0)))
    with pytest.raises(s12.S12Error):
        s12.s12_gemm_skinny(v4, to_dev(wl.activations(16, 1152, 0)))
