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


def _gemv(s12, w, x, flag=None):
    blob = s12.s12_encode(to_dev(w))
    view = s12.s12_open(blob)
    y = s12.s12_gemv(view, to_dev(x), err_flag=flag)
    torch.cuda.synchronize()
    return blob, view, y.cpu().numpy()


@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("shape", [(1, 128), (3, 384), (149, 640), (300, 1152), (77, 4096), (19, 14336)])
def test_gemv_small_shapes_all_batches(s12, oracle, B, shape):
    """Shapes that span several stages, a ragged row tail, partial 512-wide
    column slots and (for B*K*2 > 96 KB) the multi-phase column split."""
    r, c = shape
    w = wl.normal_with_outliers(r, c, 0.02, 0.002, r + c)
    x = wl.activations(B, c, B)
    flag = new_flag()
    blob, view, y = _gemv(s12, w, x, flag)
    yr, sr = oracle.gemv_f64(oracle.encode(w), x)
    assert_within_tolerance(y, yr, sr)
    assert int(flag.item()) == 0


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
    host = blob.cpu().numpy()
    rows = np.unique(np.concatenate([[0, w.shape[0] - 1], wl.rng_for(7, 0).choice(w.shape[0], 46, replace=False)]))
    yr, sr = oracle.gemv_rows_f64(host, x, rows)
    assert_within_tolerance(y[:, rows], yr, sr)


def test_gemv_single_tensor_full(s12, oracle):
    w, x = wl.single_tensor(0)
    blob, view, y = _gemv(s12, w, x)
    yr, sr = oracle.gemv_f64(blob.cpu().numpy(), x)
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
