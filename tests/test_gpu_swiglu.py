"""GPU parity of the fused decode-GEMV with the SwiGLU epilogue
(s12_gemv_swiglu) against the FP64 oracle.

The kernel's gate and up sums each carry the GEMV bound |e| <= 1e-3 * s
(s = sum_k |W x|).  Through h = silu(g) * u, with |silu'| <= 1.1, that
becomes |dh| <= 1.1 |u| e_g + |silu(g)| e_u + 1.1 e_g e_u, and the BF16
rounding of h adds 2^-9 |h| (2^-8 is used, for the rounding of silu itself
in FP32)."""
import numpy as np
import pytest
import torch

from decode_split12_b200 import workloads as wl
from gpu_util import new_flag, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def s12(cuda_ok):
    from decode_split12_b200 import s12 as mod
    mod.device_check()
    return mod


def _assert_swiglu_close(h_bits, h, g, u, s_g, s_u, oracle):
    got = wl.bf16_bits_to_f32(np.asarray(h_bits, dtype=np.int16).view(np.uint16)).astype(np.float64)
    e_g, e_u = 1e-3 * s_g, 1e-3 * s_u
    silu_g = oracle.silu_mul_f64(g, np.ones_like(g))
    tol = 1.1 * np.abs(u) * e_g + np.abs(silu_g) * e_u + 1.1 * e_g * e_u + 2.0 ** -8 * np.abs(h) + 1e-30
    bad = np.abs(got - h) > tol
    assert not bad.any(), f"{int(bad.sum())} of {bad.size} outside; worst excess {float(np.max(np.abs(got - h) - tol)):.3e}"


@pytest.mark.parametrize("B", [1, 3, 8])
@pytest.mark.parametrize("F,K", [(8, 128), (64, 640), (512, 2048), (136, 4096)])
def test_swiglu_matches_oracle(s12, oracle, F, K, B):
    """Gate and up matrices encoded as one interleaved container: ragged
    counts of 16-row groups, groups split across warps (stream-K fix-up),
    every batch size class."""
    wg = wl.normal_with_outliers(F, K, 0.05, 0.002, F + K)
    wu = wl.normal_with_outliers(F, K, 0.05, 0.002, F + K + 1)
    x = wl.activations(B, K, B + 7)
    wi = s12.interleave_gate_up(to_dev(wg), to_dev(wu))
    view = s12.s12_open(s12.s12_encode(wi))
    flag = new_flag()
    hd = s12.s12_gemv_swiglu(view, to_dev(x), err_flag=flag)
    torch.cuda.synchronize()
    assert hd.shape == (B, F)
    assert int(flag.item()) == 0
    h, g, u, s_g, s_u = oracle.swiglu_f64(oracle.encode(wg), oracle.encode(wu), x)
    _assert_swiglu_close(hd.cpu().numpy(), h, g, u, s_g, s_u, oracle)


def test_swiglu_one_hot_is_activation_of_columns(s12, oracle):
    """x = e_j: the sums are single exact products, so h is silu(W_gate[f, j])
    * W_up[f, j] rounded once to BF16, for every f."""
    F, K = 128, 512
    wg = wl.normal_with_outliers(F, K, 1.0, 0.0, 3)
    wu = wl.normal_with_outliers(F, K, 1.0, 0.0, 4)
    view = s12.s12_open(s12.s12_encode(s12.interleave_gate_up(to_dev(wg), to_dev(wu))))
    for j in (0, 129, 511):
        x = np.zeros((1, K), np.uint16)
        x[0, j] = 0x3F80
        hd = s12.s12_gemv_swiglu(view, to_dev(x))
        torch.cuda.synchronize()
        cg = wl.bf16_bits_to_f32(wg[:, j]).astype(np.float64)
        cu = wl.bf16_bits_to_f32(wu[:, j]).astype(np.float64)
        h = oracle.silu_mul_f64(cg, cu)[None, :]
        _assert_swiglu_close(hd.cpu().numpy(), h, cg[None, :], cu[None, :], np.abs(cg)[None, :],
                             np.abs(cu)[None, :], oracle)


def test_swiglu_8b_mlp_full_size_sampled(s12, oracle):
    """The 8B-style MLP's gate and up (14336 x 4096 each) at full size, as
    the single interleaved 28672 x 4096 container; 64 sampled outputs per
    batch row checked against the oracle's GEMVs of the separate matrices."""
    F, K = 14336, 4096
    wg = wl.student_t_scaled(F, K, 0, 4)
    wu = wl.student_t_scaled(F, K, 0, 5)
    x = wl.activations(4, K, 11)
    view = s12.s12_open(s12.s12_encode(s12.interleave_gate_up(to_dev(wg), to_dev(wu))))
    hd = s12.s12_gemv_swiglu(view, to_dev(x)).cpu().numpy()
    rows = np.unique(np.concatenate([[0, 7, 8, F - 1], wl.rng_for(12, 0).choice(F, 60, replace=False)]))
    g, s_g = oracle.gemv_rows_f64(oracle.encode(wg[rows]), x, np.arange(rows.size))
    u, s_u = oracle.gemv_rows_f64(oracle.encode(wu[rows]), x, np.arange(rows.size))
    h = oracle.silu_mul_f64(g, u)
    _assert_swiglu_close(hd[:, rows], h, g, u, s_g, s_u, oracle)


def test_swiglu_rejects_rows_not_multiple_of_16(s12):
    w = wl.normal_with_outliers(24, 256, 0.02, 0.0, 1)
    view = s12.s12_open(s12.s12_encode(to_dev(w)))
    with pytest.raises(s12.S12Error):
        s12.s12_gemv_swiglu(view, to_dev(wl.activations(1, 256, 0)))
