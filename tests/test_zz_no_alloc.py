"""s12_gemv_noalloc: the fused decode-GEMV for callers that cannot allocate
device memory (a plugin whose host engine owns every device byte, code under
a fixed memory budget, or a path where cudaMalloc's implicit synchronisation
is not allowed).  It runs the s12_gemv kernel on a workspace that is a static
array inside the library, so its result must match s12_gemv's within the
GEMV tolerance, |y - y_ref| <= 1e-3 * sum_j |W_ij x_j|, call after call.

Kept in a file of its own, named so that pytest collects it last: the
static array outlives every other test in the process, and this test must
pass both alone in a fresh process and after all the others."""
import ctypes as C

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


def _call_noalloc(s12, view, x, y, flag):
    """Through the C ABI directly: view, x (B x cols bf16), B, y, err_flag,
    stream (the current torch stream)."""
    lib = s12.lib()
    B = x.shape[0]
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.s12_gemv_noalloc(C.byref(view), C.c_void_p(x.data_ptr()), B, C.c_void_p(y.data_ptr()),
                                C.c_void_p(flag.data_ptr()), stream)


@pytest.mark.parametrize("B", [1, 8])
def test_noalloc_matches_gemv_two_calls(s12, oracle, B):
    """Two different matrices, one after the other (the second call reuses
    the static workspace the first one left behind): each result matches
    s12_gemv on the same inputs within the tolerance, and the error word
    stays clear."""
    cases = [(wl.student_t_scaled(4096, 4096, 11), 4096), (wl.normal_with_outliers(1000, 14336, 0.02, 0.002, 12),
                                                          14336)]
    for i, (w, k) in enumerate(cases):
        x = wl.activations(B, k, 20 + i)
        blob = s12.s12_encode(to_dev(w))
        view = s12.s12_open(blob)
        xd = to_dev(x)
        y_ref = s12.s12_gemv(view, xd)
        y = torch.full((B, w.shape[0]), float("nan"), dtype=torch.float32, device="cuda")
        flag = new_flag()
        assert _call_noalloc(s12, view, xd, y, flag) == s12.S12_OK
        torch.cuda.synchronize()
        assert int(flag.item()) == 0
        _, s_ref = oracle.matmul_f64(w, x)
        assert_within_tolerance(y.cpu().numpy(), y_ref.cpu().numpy().astype(np.float64), s_ref)


def test_noalloc_repeated_same_call(s12, oracle):
    """The same call twice in a row gives results within the tolerance of
    s12_gemv both times (the counters are cleared at the start of each
    call)."""
    w = wl.student_t_scaled(1024, 4096, 13)
    x = wl.activations(4, 4096, 14)
    view = s12.s12_open(s12.s12_encode(to_dev(w)))
    xd = to_dev(x)
    y_ref = s12.s12_gemv(view, xd).cpu().numpy().astype(np.float64)
    _, s_ref = oracle.matmul_f64(w, x)
    for _ in range(2):
        y = torch.full((4, 1024), float("nan"), dtype=torch.float32, device="cuda")
        flag = new_flag()
        assert _call_noalloc(s12, view, xd, y, flag) == s12.S12_OK
        torch.cuda.synchronize()
        assert int(flag.item()) == 0
        assert_within_tolerance(y.cpu().numpy(), y_ref, s_ref)


def test_noalloc_rejects_oversized(s12):
    """A container above the static workspace's row limit is refused before
    any device work."""
    v = s12.View()
    v.rows, v.cols, v.n_tiles = (1 << 20) + 16, 128, (1 << 20) + 16
    for f in ("container", "raw", "code", "base", "esc_off", "esc"):
        setattr(v, f, 0x100000)
    v.version = 1
    x = torch.zeros((1, 128), dtype=torch.int16, device="cuda")
    y = torch.zeros((1, 16), dtype=torch.float32, device="cuda")
    rc = s12.lib().s12_gemv_noalloc(C.byref(v), C.c_void_p(x.data_ptr()), 1, C.c_void_p(y.data_ptr()), None, None)
    assert rc == s12.S12_ERR_CAPACITY
