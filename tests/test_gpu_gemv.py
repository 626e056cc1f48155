"""GPU parity of the fused decode-GEMV (and the plain BF16 GEMV baseline)
against the FP64 oracle: |y - y_ref| <= 1e-3 * sum_j |W_ij x_j|."""
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


def _gemv(s12, w, x, flag=None, ws=None):
    blob = s12.s12_encode(to_dev(w))
    view = s12.s12_open(blob)
    y = s12.s12_gemv(view, to_dev(x), ws=ws, err_flag=flag)
    torch.cuda.synchronize()
    return blob, view, y.cpu().numpy()


@pytest.mark.parametrize("checked", [True, False])
@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("shape", [(1, 128), (3, 384), (149, 640), (300, 1152), (77, 4096), (19, 14336)])
def test_gemv_small_shapes_all_batches(s12, oracle, B, shape, checked):
    """Ragged 16-row groups, row groups split across many warps (stream-K
    fix-up), x staged in shared memory or (B=8, K=14336) read from global
    memory; with the error word (every tile checked) and without it."""
    r, c = shape
    w = wl.normal_with_outliers(r, c, 0.02, 0.002, r + c)
    x = wl.activations(B, c, B)
    flag = new_flag() if checked else None
    ws = torch.zeros(s12.s12_gemv_ws_bytes(s12.s12_open(s12.s12_encode(to_dev(w))), B), dtype=torch.uint8,
                     device="cuda")
    blob, view, y = _gemv(s12, w, x, flag, ws)
    yr, sr = oracle.gemv_f64(oracle.encode(w), x)
    assert_within_tolerance(y, yr, sr)
    if checked:
        assert int(flag.item()) == 0
    # the arrival counters (the workspace's tail, one per 16-row group) are
    # back at zero for the next call
    n_cnt = -(-((view.rows + 15) // 16) * 4 // 256) * 256
    assert int(ws[-n_cnt:].count_nonzero()) == 0


def test_gemv_one_hot_is_exact(s12, oracle):
    """x = e_j returns column j exactly: one BF16 product is exact in FP32."""
    w = wl.normal_with_outliers(300, 1152, 0.02, 0.01, 8)
    x = np.zeros((8, 1152), np.uint16)
    cols = [0, 127, 128, 511, 512, 700, 1100, 1151]
    for b, j in enumerate(cols):
        x[b, j] = 0x3F80
    _, _, y = _gemv(s12, w, x)
    for b, j in enumerate(cols):
        assert np.array_equal(y[b], wl.bf16_bits_to_f32(w[:, j]))


def test_gemv_integer_matrix_is_exact(s12, oracle):
    vals = wl.rng_for(3, 0).integers(-8, 9, size=(200, 2048)).astype(np.float32)
    w = wl.to_bf16_bits(vals)
    x = np.full((2, 2048), 0x3F80, np.uint16)
    x[1] = 0xBF80
    _, _, y = _gemv(s12, w, x)
    assert np.array_equal(y[0], vals.sum(1))
    assert np.array_equal(y[1], -vals.sum(1))


def test_gemv_escape_heavy(s12, oracle):
    """Every tile carries escapes (10 % rate) and some are all-escape."""
    w, _ = wl.escape_stress(0.10, 0, 64, 2048)
    # a row of random patterns with exponents 0..160: every window leaves
    # many escapes, and no product or FP32 partial sum can overflow
    g = wl.rng_for(4, 0)
    e = g.integers(0, 161, size=2048)
    w[5] = ((g.integers(0, 2, 2048) << 15) | (e << 7) | g.integers(0, 128, 2048)).astype(np.uint16)
    x = wl.activations(3, 2048, 3)
    flag = new_flag()
    _, _, y = _gemv(s12, w, x, flag)
    yr, sr = oracle.gemv_f64(oracle.encode(w), x)
    assert_within_tolerance(y, yr, sr)
    assert int(flag.item()) == 0


def test_gemv_workspace_reused_across_matrices(s12, oracle):
    """One workspace serves a sequence of calls on different shapes (the
    counters return to zero after every call), and a short one is refused."""
    shapes = [(1024, 4096), (16, 14336), (4096, 1024), (33, 256), (1024, 4096)]
    mats = [wl.student_t_scaled(r, c, i) for i, (r, c) in enumerate(shapes)]
    views = [s12.s12_open(s12.s12_encode(to_dev(w))) for w in mats]
    need = max(s12.s12_gemv_ws_bytes(v, 1) for v in views)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for i, (w, v) in enumerate(zip(mats, views)):
        x = wl.activations(2, w.shape[1], i)
        y = s12.s12_gemv(v, to_dev(x), ws=ws)
        torch.cuda.synchronize()
        yr, sr = oracle.matmul_f64(w, x)
        assert_within_tolerance(y.cpu().numpy(), yr, sr)
    small = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(s12.S12Error):
        s12.s12_gemv(views[0], to_dev(wl.activations(1, 4096, 0)), ws=small)


def test_gemv_deterministic(s12):
    w = wl.student_t_scaled(1000, 4096, 1)
    x = wl.activations(4, 4096, 1)
    blob = s12.s12_encode(to_dev(w))
    view = s12.s12_open(blob)
    xd = to_dev(x)
    a = s12.s12_gemv(view, xd)
    b = s12.s12_gemv(view, xd)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("name", list(wl.LLAMA8B_SHAPES))
@pytest.mark.parametrize("B", [1, 4, 8])
def test_gemv_llama8b_full_size_sampled(s12, oracle, name, B):
    """Full-size 8B-layer matrices in the launch configuration the benchmark
    times; 48 sampled rows checked one by one against the FP64 oracle."""
    mats, xs = wl.llama8b_layer(0, B, names=[name])
    w, x = mats[name], xs[name]
    blob, view, y = _gemv(s12, w, x)
    rows = np.unique(np.concatenate([[0, w.shape[0] - 1], wl.rng_for(7, 0).choice(w.shape[0], 46, replace=False)]))
    # the reference starts from W: the oracle encodes the sampled rows itself
    yr, sr = oracle.gemv_f64(oracle.encode(w[rows]), x)
    assert_within_tolerance(y[:, rows], yr, sr)


def test_gemv_single_tensor_full(s12, oracle):
    w, x = wl.single_tensor(0)
    blob, view, y = _gemv(s12, w, x)
    yr, sr = oracle.gemv_f64(oracle.encode(w), x)
    assert_within_tolerance(y, yr, sr)


@pytest.mark.parametrize("B", [1, 3, 8])
@pytest.mark.parametrize("shape", [(3, 384), (300, 1152), (1024, 4096)])
def test_bf16_baseline(s12, oracle, B, shape):
    r, c = shape
    w = wl.student_t_scaled(r, c, 2)
    x = wl.activations(B, c, 2)
    y = s12.s12_bf16_gemv(to_dev(w), to_dev(x))
    torch.cuda.synchronize()
    yr, sr = oracle.matmul_f64(w, x)
    assert_within_tolerance(y.cpu().numpy(), yr, sr)


@pytest.mark.parametrize("checked", [True, False])
@pytest.mark.parametrize("B", [1, 3, 8])
def test_gemv_multi_mixed_shapes(s12, oracle, B, checked):
    """One grouped launch over matrices of different shapes (ragged row
    groups, one-tile rows, long rows, escape-heavy rows) equals the oracle
    for every member."""
    shapes = [(77, 4096), (16, 14336), (300, 1152), (1, 128), (64, 2048), (33, 256)]
    mats = [wl.normal_with_outliers(r, c, 0.02, 0.002, 100 + i) for i, (r, c) in enumerate(shapes)]
    esc, _ = wl.escape_stress(0.10, 1, 64, 2048)
    mats[4] = esc
    xs = [wl.activations(B, c, 200 + i) for i, (_, c) in enumerate(shapes)]
    views = [s12.s12_open(s12.s12_encode(to_dev(w))) for w in mats]
    flag = new_flag() if checked else None
    ys = s12.s12_gemv_multi(views, [to_dev(x) for x in xs], err_flag=flag)
    torch.cuda.synchronize()
    for w, x, y in zip(mats, xs, ys):
        yr, sr = oracle.gemv_f64(oracle.encode(w), x)
        assert_within_tolerance(y.cpu().numpy(), yr, sr)
    if checked:
        assert int(flag.item()) == 0


def test_gemv_multi_llama_layer_matches_single_calls(s12):
    """The grouped launch over a full 8B-style layer gives, per matrix, the
    same y as separate s12_gemv calls up to the summation order (both are
    checked against the oracle elsewhere), and is repeatable bit for bit."""
    mats, xs = wl.llama8b_layer(0, 4)
    names = list(wl.LLAMA8B_SHAPES)
    views = [s12.s12_open(s12.s12_encode(to_dev(mats[n]))) for n in names]
    xd = [to_dev(xs[n]) for n in names]
    ws = torch.zeros(s12.s12_gemv_multi_ws_bytes(views, 4), dtype=torch.uint8, device="cuda")
    a = s12.s12_gemv_multi(views, xd, ws=ws)
    b = s12.s12_gemv_multi(views, xd, ws=ws)
    singles = [s12.s12_gemv(v, x) for v, x in zip(views, xd)]
    torch.cuda.synchronize()
    for ya, yb, ys in zip(a, b, singles):
        assert torch.equal(ya, yb)
        scale = ys.abs().max().item()
        assert torch.allclose(ya, ys, rtol=0, atol=1e-4 * scale)


def test_gemv_multi_rejects_bad_groups(s12):
    w = wl.student_t_scaled(64, 256, 0)
    v = s12.s12_open(s12.s12_encode(to_dev(w)))
    x = to_dev(wl.activations(1, 256, 0))
    with pytest.raises(s12.S12Error):
        s12.s12_gemv_multi([v] * 9, [x] * 9)


def test_gemv_top_of_range_bases(s12, oracle):
    """Tiles whose window sits at the top of the BF16 range (base 240 or 241,
    where base + 15 is an Inf/NaN exponent or carries out of the byte) with
    escapes below the window.  x is scaled down so that no product or sum
    leaves the FP32 range; the result matches the FP64 oracle."""
    g = wl.rng_for(21, 0)
    w = wl.normal_with_outliers(64, 1024, 0.02, 0.0, 21)
    for r in range(64):
        e = g.integers(241, 255, size=1024)                     # window [240, 254] or [241, 255]
        e[g.choice(1024, 6, replace=False)] = g.integers(100, 130, size=6)   # escapes
        w[r] = ((g.integers(0, 2, 1024) << 15) | (e << 7) | g.integers(0, 128, 1024)).astype(np.uint16)
    x = wl.to_bf16_bits(wl.rng_for(22, 0).standard_normal((2, 1024)).astype(np.float32) * np.float32(2.0 ** -120))
    flag = new_flag()
    _, _, y = _gemv(s12, w, x, flag)
    yr, sr = oracle.gemv_f64(oracle.encode(w), x)
    assert np.isfinite(y).all()
    assert_within_tolerance(y, yr, sr)
    assert int(flag.item()) == 0


@pytest.mark.parametrize("B", [1, 5, 8])
def test_gemv_huge_activations_at_escapes(s12, oracle, B):
    """Zero weights (always escapes, below every window) at six columns in
    40 of the rows, and x 2^40 times larger at exactly those columns.  The
    true sums of those rows are near 30 while any finite placeholder value
    at the escapes would give products near 1e12 (FP32 spacing 2^17 there),
    so a kernel must use the exact escaped values inside the product, not
    add a placeholder and cancel it later.  Checked against the FP64 oracle
    within the usual tolerance, and the error word stays clear."""
    R, K = 96, 2048
    w = wl.normal_with_outliers(R, K, 0.02, 0.0, 31)
    g = wl.rng_for(31, 1)
    hot = g.choice(K, 6, replace=False)
    rows = g.choice(R, 40, replace=False)
    w[np.ix_(rows, hot)] = 0          # +0.0 in bf16: exponent 0, an escape
    xf = g.standard_normal((B, K)).astype(np.float32)
    xf[:, hot] *= np.float32(2.0 ** 40)
    x = wl.to_bf16_bits(xf)
    flag = new_flag()
    _, _, y = _gemv(s12, w, x, flag)
    yr, sr = oracle.gemv_f64(oracle.encode(w), x)
    assert np.isfinite(y).all()
    assert_within_tolerance(y, yr, sr)
    assert int(flag.item()) == 0


def test_gemv_inf_activation_at_escape(s12, oracle):
    """x = +Inf at a column where one row has a zero weight (an escape) and
    the others ordinary weights: the zero row's exact result is NaN
    (0 * Inf), the rows with a nonzero weight there give +-Inf with the
    weight's sign (no escape may be replaced by a finite value there)."""
    R, K = 32, 512
    w = wl.normal_with_outliers(R, K, 0.02, 0.0, 41)
    col = 77
    w[5, col] = 0
    xf = wl.rng_for(41, 1).standard_normal((1, K)).astype(np.float32)
    xf[0, col] = np.inf
    x = wl.to_bf16_bits(xf)
    _, _, y = _gemv(s12, w, x, new_flag())
    wf = (w.astype(np.uint32) << 16).view(np.float32)
    for r in range(R):
        if r == 5:
            assert np.isnan(y[0, r])
        else:
            assert y[0, r] == (np.inf if wf[r, col] > 0 else -np.inf), r


# ---------------------------------------------------------------------------
# container version 2 (compact tile header) and the BF16 output

def _v2_blob(oracle, w):
    """A version 2 container built by the oracle from W, on the device."""
    from gpu_util import blob_to_dev
    return blob_to_dev(oracle.encode_v2(w))


@pytest.mark.parametrize("checked", [True, False])
@pytest.mark.parametrize("B", [1, 3, 8])
@pytest.mark.parametrize("shape", [(1, 128), (3, 384), (149, 640), (300, 1152), (77, 4096), (19, 14336)])
def test_gemv_v2_small_shapes(s12, oracle, shape, B, checked):
    """The fused GEMV reading a version 2 container (per tile one u16 of
    base | escape count, per row one u32 escape offset; [W] English
    edition, opening summary) matches the FP64 oracle; warps whose range
    starts in the middle of a row sum the earlier tiles' counts."""
    r, c = shape
    w = wl.normal_with_outliers(r, c, 0.02, 0.004, r + 7 * c)
    x = wl.activations(B, c, B + 1)
    blob = _v2_blob(oracle, w)
    view = s12.s12_open(blob)
    assert view.version == 2
    flag = new_flag() if checked else None
    y = s12.s12_gemv(view, to_dev(x), err_flag=flag)
    torch.cuda.synchronize()
    yr, sr = oracle.gemv_f64(oracle.encode(w), x)
    assert_within_tolerance(y.cpu().numpy(), yr, sr)
    if checked:
        assert int(flag.item()) == 0


def test_gemv_v2_escape_heavy_and_multi(s12, oracle):
    """Version 2 at 10 % escapes (every tile, some all-escape) in a grouped
    launch beside a second version 2 matrix; a call that mixes container
    versions is refused."""
    w0, _ = wl.escape_stress(0.10, 2, 64, 2048)
    w1 = wl.student_t_scaled(300, 1152, 3)
    x0, x1 = wl.activations(4, 2048, 5), wl.activations(4, 1152, 6)
    b0, b1 = _v2_blob(oracle, w0), _v2_blob(oracle, w1)
    v0, v1 = s12.s12_open(b0), s12.s12_open(b1)
    flag = new_flag()
    ys = s12.s12_gemv_multi([v0, v1], [to_dev(x0), to_dev(x1)], err_flag=flag)
    torch.cuda.synchronize()
    for w, x, y in ((w0, x0, ys[0]), (w1, x1, ys[1])):
        yr, sr = oracle.gemv_f64(oracle.encode(w), x)
        assert_within_tolerance(y.cpu().numpy(), yr, sr)
    assert int(flag.item()) == 0
    v_one = s12.s12_open(s12.s12_encode(to_dev(w1)))
    with pytest.raises(s12.S12Error):
        s12.s12_gemv_multi([v0, v_one], [to_dev(x0), to_dev(x1)])


@pytest.mark.parametrize("name", ["q", "down"])
def test_gemv_v2_llama8b_full_size_sampled(s12, oracle, name):
    """Full-size 8B-layer matrices as version 2 containers (the oracle's own
    encoding), sampled rows against the FP64 oracle."""
    mats, xs = wl.llama8b_layer(0, 1, names=[name])
    w, x = mats[name], xs[name]
    view = s12.s12_open(_v2_blob(oracle, w))
    y = s12.s12_gemv(view, to_dev(x))
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([[0, w.shape[0] - 1], wl.rng_for(7, 1).choice(w.shape[0], 46, replace=False)]))
    yr, sr = oracle.gemv_f64(oracle.encode(w[rows]), x)
    assert_within_tolerance(y.cpu().numpy()[:, rows], yr, sr)


@pytest.mark.parametrize("B", [1, 4, 8])
@pytest.mark.parametrize("shape", [(3, 384), (300, 1152), (1024, 4096)])
def test_gemv_bf16_output(s12, oracle, shape, B):
    """The BF16-output GEMV: each y is the FP32 sum rounded to BF16, so it is
    within 1e-3 * sum|W x| + 2^-9 |y_ref| of the FP64 oracle (the rounding of
    a BF16 result adds at most half an ulp, 2^-9 relative)."""
    r, c = shape
    w = wl.normal_with_outliers(r, c, 0.02, 0.002, r + c + B)
    x = wl.activations(B, c, 40 + B)
    view = s12.s12_open(s12.s12_encode(to_dev(w)))
    flag = new_flag()
    yb = s12.s12_gemv_bf16(view, to_dev(x), err_flag=flag)
    torch.cuda.synchronize()
    y = wl.bf16_bits_to_f32(yb.cpu().numpy().view(np.uint16)).astype(np.float64)
    yr, sr = oracle.gemv_f64(oracle.encode(w), x)
    err = np.abs(y - yr)
    bound = 1e-3 * sr + 2.0 ** -9 * np.abs(yr)
    assert (err <= bound).all(), float((err / np.maximum(bound, 1e-300)).max())
    assert int(flag.item()) == 0
