"""GPU parity of the fused decode-skinny-GEMM (tcgen05 tensor cores) against
the FP64 oracle: |y - y_ref| <= 1e-3 * sum_j |W_ij x_j| for every output."""
import numpy as np
import pytest
import torch

from decode_split12_b200 import workloads as wl
from gpu_util import assert_within_tolerance, new_flag, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def s12(cuda_ok):
    from decode_split12_b200 import s12 as mod
    mod.device_check()
    return mod


def _gemm(s12, w, x, flag=None, ws=None):
    blob = s12.s12_encode(to_dev(w))
    view = s12.s12_open(blob)
    y = s12.s12_gemm_skinny(view, to_dev(x), ws=ws, err_flag=flag)
    torch.cuda.synchronize()
    return blob, view, y.cpu().numpy()


@pytest.mark.parametrize("checked", [True, False])
@pytest.mark.parametrize("shape,M", [((128, 128), 16), ((256, 512), 16), ((300, 1152), 17), ((16, 256), 32),
                                     ((1000, 4096), 64), ((512, 2048), 256), ((130, 14336), 48),
                                     ((640, 1024), 200)])
def test_gemm_small_shapes(s12, oracle, shape, M, checked):
    """Ragged 128-row tiles, M not a multiple of 16 (zero-padded token rows),
    tiles split across CTAs (stream-K fix-up), long rows, every M class."""
    r, c = shape
    w = wl.normal_with_outliers(r, c, 0.02, 0.002, r + c + M)
    x = wl.activations(M, c, M)
    flag = new_flag() if checked else None
    _, view, y = _gemm(s12, w, x, flag)
    yr, sr = oracle.gemv_f64(oracle.encode(w), x)
    assert y.shape == (M, r)
    assert_within_tolerance(y, yr, sr)
    if checked:
        assert int(flag.item()) == 0


def test_gemm_escape_heavy(s12, oracle):
    """10 % escapes (every tile has some) plus a row of random exponents."""
    w, _ = wl.escape_stress(0.10, 0, 256, 2048)
    g = wl.rng_for(5, 0)
    e = g.integers(0, 161, size=2048)
    w[7] = ((g.integers(0, 2, 2048) << 15) | (e << 7) | g.integers(0, 128, 2048)).astype(np.uint16)
    x = wl.activations(32, 2048, 6)
    flag = new_flag()
    _, _, y = _gemm(s12, w, x, flag)
    yr, sr = oracle.gemv_f64(oracle.encode(w), x)
    assert_within_tolerance(y, yr, sr)
    assert int(flag.item()) == 0


def test_gemm_one_hot_is_exact(s12):
    """x = e_j returns column j of W exactly (one product per output)."""
    w = wl.normal_with_outliers(384, 1024, 0.02, 0.01, 9)
    cols = [0, 63, 64, 127, 128, 500, 777, 1023] * 2
    x = np.zeros((16, 1024), np.uint16)
    for b, j in enumerate(cols):
        x[b, j] = 0x3F80
    _, _, y = _gemm(s12, w, x)
    for b, j in enumerate(cols):
        assert np.array_equal(y[b], wl.bf16_bits_to_f32(w[:, j]))


def test_gemm_deterministic_and_workspace_clean(s12):
    w = wl.student_t_scaled(1024, 4096, 3)
    x = to_dev(wl.activations(64, 4096, 3))
    view = s12.s12_open(s12.s12_encode(to_dev(w)))
    need = s12.s12_gemm_ws_bytes(view, 64)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    a = s12.s12_gemm_skinny(view, x, ws=ws)
    b = s12.s12_gemm_skinny(view, x, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    n_cnt = -(-((1024 + 127) // 128) * 4 // 256) * 256
    assert int(ws[-n_cnt:].count_nonzero()) == 0


@pytest.mark.parametrize("name", ["up", "down"])
@pytest.mark.parametrize("M", [16, 64, 256])
def test_gemm_70b_mlp_full_size_sampled(s12, oracle, name, M):
    """The 70B-style MLP matrices at full size in the launch configuration
    the benchmark times; 48 sampled rows checked against the FP64 oracle."""
    w = wl.mlp70b(name, 0)
    x = wl.activations(M, w.shape[1], M)
    blob, view, y = _gemm(s12, w, x)
    rows = np.unique(np.concatenate([[0, w.shape[0] - 1], wl.rng_for(8, M).choice(w.shape[0], 46, replace=False)]))
    # the reference starts from W: the oracle encodes the sampled rows itself
    yr, sr = oracle.gemv_f64(oracle.encode(w[rows]), x)
    assert_within_tolerance(y[:, rows], yr, sr)


# ---------------------------------------------------------------------------
# grouped launch (s12_gemm_skinny_multi)

@pytest.mark.parametrize("checked", [True, False])
def test_gemm_multi_mixed_shapes_and_tokens(s12, oracle, checked):
    """Six matrices of different shapes (ragged 128-row tiles, long rows,
    a matrix smaller than one tile) and different token counts (one below
    16) in one launch:
    every y_i matches the FP64 oracle, and the rows of the shared padded
    token count beyond M_i are never written."""
    shapes = [(300, 1152), (128, 128), (77, 4096), (640, 1024), (16, 2048), (200, 512)]
    Ms = [17, 32, 16, 29, 24, 3]
    ws_, xs, views, blobs = [], [], [], []
    for i, ((r, c), m) in enumerate(zip(shapes, Ms)):
        w = wl.normal_with_outliers(r, c, 0.02, 0.002, 40 + i)
        ws_.append(w)
        xs.append(wl.activations(m, c, 50 + i))
        blobs.append(s12.s12_encode(to_dev(w)))
        views.append(s12.s12_open(blobs[-1]))
    ys = [torch.full((m, r), float("nan"), dtype=torch.float32, device="cuda") for m, (r, _) in zip(Ms, shapes)]
    flag = new_flag() if checked else None
    s12.s12_gemm_skinny_multi(views, [to_dev(x) for x in xs], ys, err_flag=flag)
    torch.cuda.synchronize()
    for w, x, y in zip(ws_, xs, ys):
        yr, sr = oracle.gemv_f64(oracle.encode(w), x)
        assert_within_tolerance(y.cpu().numpy(), yr, sr)
    if checked:
        assert int(flag.item()) == 0


def test_gemm_multi_moe_experts_full_size(s12, oracle):
    """An 8-expert block's gate projections (14336 x 4096 each) with the
    token counts of a top-2 routing of 64 tokens, in one launch; 24 sampled
    rows per expert against the FP64 oracle, and the result equals the
    per-expert single calls within the tolerance."""
    Ms = [14, 15, 13, 14, 17, 20, 15, 20]
    views, blobs, refs, xs, samples = [], [], [], [], []
    for e, m in enumerate(Ms):
        w = wl.student_t_scaled(14336, 4096, 100 + e)
        blobs.append(s12.s12_encode(to_dev(w)))
        views.append(s12.s12_open(blobs[-1]))
        rows = np.unique(np.concatenate([[0, 14335], wl.rng_for(9, e).choice(14336, 22, replace=False)]))
        samples.append(rows)
        # the reference starts from W: the oracle encodes the sampled rows itself
        refs.append(oracle.encode(w[rows]))
        xs.append(wl.activations(m, 4096, 200 + e))
        del w
    ys = s12.s12_gemm_skinny_multi(views, [to_dev(x) for x in xs])
    torch.cuda.synchronize()
    for e, m in enumerate(Ms):
        rows = samples[e]
        yr, sr = oracle.gemv_f64(refs[e], xs[e])
        assert_within_tolerance(ys[e][:, rows].cpu().numpy(), yr, sr)


def test_gemm_multi_deterministic_and_workspace_clean(s12):
    """Two identical grouped calls give identical outputs and leave the
    workspace's arrival counters at zero."""
    mats = [wl.student_t_scaled(1024, 4096, 3), wl.student_t_scaled(512, 2048, 4)]
    views = [s12.s12_open(s12.s12_encode(to_dev(w))) for w in mats]
    xs = [to_dev(wl.activations(48, 4096, 3)), to_dev(wl.activations(40, 2048, 4))]
    need = s12.s12_gemm_multi_ws_bytes(views, [48, 40])
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    a = s12.s12_gemm_skinny_multi(views, xs, ws=ws)
    b = s12.s12_gemm_skinny_multi(views, xs, ws=ws)
    torch.cuda.synchronize()
    for ya, yb in zip(a, b):
        assert torch.equal(ya, yb)
    n_tiles = (1024 + 127) // 128 + (512 + 127) // 128
    n_cnt = -(-n_tiles * 4 // 256) * 256
    assert int(ws[-n_cnt:].count_nonzero()) == 0


def test_gemm_multi_rejects_bad_groups(s12):
    """More than S12_GEMM_MAX_PROBLEMS matrices, or an M above 256 in any
    entry, fails the whole call before any launch."""
    w = wl.normal_with_outliers(128, 256, 0.02, 0.0, 1)
    v = s12.s12_open(s12.s12_encode(to_dev(w)))
    x = to_dev(wl.activations(16, 256, 0))
    with pytest.raises(s12.S12Error):
        s12.s12_gemm_skinny_multi([v] * 17, [x] * 17)
    with pytest.raises(s12.S12Error):
        s12.s12_gemm_skinny_multi([v, v], [x, to_dev(wl.activations(257, 256, 0))])


# ---------------------------------------------------------------------------
# container version 2 (compact tile header) and the BF16 output

def _v2_blob(oracle, w):
    """A version 2 container built by the oracle from W, on the device."""
    from gpu_util import blob_to_dev
    return blob_to_dev(oracle.encode_v2(w))


@pytest.mark.parametrize("checked", [True, False])
@pytest.mark.parametrize("shape,M", [((128, 128), 16), ((300, 1152), 17), ((1000, 4096), 64),
                                     ((130, 14336), 48), ((640, 1024), 200), ((512, 2048), 256)])
def test_gemm_v2_small_shapes(s12, oracle, shape, M, checked):
    """The fused GEMM reading a version 2 container (per tile one u16 of
    base | escape count, per row one u32 escape offset; [W] English
    edition, opening summary) matches the FP64 oracle.  CTAs whose range
    starts in the middle of a tile row sum the earlier tiles' counts; the
    stream-K split tiles and ragged last tiles are covered."""
    r, c = shape
    w = wl.normal_with_outliers(r, c, 0.02, 0.004, r + 3 * c + M)
    x = wl.activations(M, c, M + 2)
    view = s12.s12_open(_v2_blob(oracle, w))
    assert view.version == 2
    flag = new_flag() if checked else None
    y = s12.s12_gemm_skinny(view, to_dev(x), err_flag=flag)
    torch.cuda.synchronize()
    yr, sr = oracle.gemv_f64(oracle.encode(w), x)
    assert_within_tolerance(y.cpu().numpy(), yr, sr)
    if checked:
        assert int(flag.item()) == 0


def test_gemm_v2_escape_heavy_and_multi(s12, oracle):
    """Version 2 at 10 % escapes (every tile, a row of random exponents)
    grouped with a second version 2 matrix; a call that mixes container
    versions is refused before any launch."""
    w0, _ = wl.escape_stress(0.10, 3, 256, 2048)
    g = wl.rng_for(6, 0)
    e = g.integers(0, 161, size=2048)
    w0[5] = ((g.integers(0, 2, 2048) << 15) | (e << 7) | g.integers(0, 128, 2048)).astype(np.uint16)
    w1 = wl.student_t_scaled(300, 1152, 4)
    x0, x1 = wl.activations(32, 2048, 7), wl.activations(20, 1152, 8)
    v0, v1 = s12.s12_open(_v2_blob(oracle, w0)), s12.s12_open(_v2_blob(oracle, w1))
    flag = new_flag()
    ys = s12.s12_gemm_skinny_multi([v0, v1], [to_dev(x0), to_dev(x1)], err_flag=flag)
    torch.cuda.synchronize()
    for w, x, y in ((w0, x0, ys[0]), (w1, x1, ys[1])):
        yr, sr = oracle.gemv_f64(oracle.encode(w), x)
        assert_within_tolerance(y.cpu().numpy(), yr, sr)
    assert int(flag.item()) == 0
    v_one = s12.s12_open(s12.s12_encode(to_dev(w1)))
    with pytest.raises(s12.S12Error):
        s12.s12_gemm_skinny_multi([v0, v_one], [to_dev(x0), to_dev(x1)])


def test_gemm_v2_70b_down_full_size_sampled(s12, oracle):
    """The 70B-style down projection (8192 x 28672) as a version 2 container
    at M = 16, 48 sampled rows against the FP64 oracle."""
    w = wl.mlp70b("down", 0)
    x = wl.activations(16, w.shape[1], 16)
    view = s12.s12_open(_v2_blob(oracle, w))
    y = s12.s12_gemm_skinny(view, to_dev(x))
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, w.shape[0] - 1], wl.rng_for(10, 1).choice(w.shape[0], 46, replace=False)]))
    yr, sr = oracle.gemv_f64(oracle.encode(w[rows]), x)
    assert_within_tolerance(y.cpu().numpy()[:, rows], yr, sr)


@pytest.mark.parametrize("shape,M", [((128, 256), 16), ((300, 1152), 33), ((1024, 4096), 128), ((640, 2048), 256)])
def test_gemm_bf16_output(s12, oracle, shape, M):
    """The BF16-output GEMM: each y is the FP32 sum rounded to BF16, within
    1e-3 * sum|W x| + 2^-9 |y_ref| of the FP64 oracle (rounding to BF16 adds
    at most half an ulp, 2^-9 relative); stream-K split tiles included."""
    r, c = shape
    w = wl.normal_with_outliers(r, c, 0.02, 0.002, r + c + M)
    x = wl.activations(M, c, 60 + M)
    view = s12.s12_open(s12.s12_encode(to_dev(w)))
    flag = new_flag()
    yb = s12.s12_gemm_skinny_bf16(view, to_dev(x), err_flag=flag)
    torch.cuda.synchronize()
    y = wl.bf16_bits_to_f32(yb.cpu().numpy().view(np.uint16)).astype(np.float64)
    yr, sr = oracle.gemv_f64(oracle.encode(w), x)
    err = np.abs(y - yr)
    bound = 1e-3 * sr + 2.0 ** -9 * np.abs(yr)
    assert (err <= bound).all(), float((err / np.maximum(bound, 1e-300)).max())
    assert int(flag.item()) == 0
