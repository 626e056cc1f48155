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
    host = blob.cpu().numpy()
    rows = np.unique(np.concatenate([[0, w.shape[0] - 1], wl.rng_for(8, M).choice(w.shape[0], 46, replace=False)]))
    yr, sr = oracle.gemv_rows_f64(host, x, rows)
    assert_within_tolerance(y[:, rows], yr, sr)
