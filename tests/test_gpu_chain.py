"""The decoder-stack loop with a real activation chain ([W] "What does
'lossless' mean for LLM weights?": decode and use the weights at once, layer
after layer): each layer runs its attention projections (q, k, v, o in one
grouped launch; attention itself is outside the path, so o reads the layer
input in place of the attention output), the fused gate/up GEMV with the
SwiGLU epilogue, and the down GEMV with a BF16 output, which is the next
layer's input.  Every step is checked against the FP64 oracle on the input
that step actually received, so the test shows that each layer's GEMVs read
the previous layer's output, without rounding differences piling up."""
import numpy as np
import pytest
import torch

from decode_split12_b200 import workloads as wl
from gpu_util import assert_within_tolerance, new_flag, to_dev

pytestmark = pytest.mark.gpu

D, KV, F, LAYERS = 256, 128, 512, 3


@pytest.fixture(scope="module")
def s12(cuda_ok):
    from decode_split12_b200 import s12 as mod
    mod.device_check()
    return mod


def _layer(s12, oracle, l):
    shapes = {"q": (D, D), "k": (KV, D), "v": (KV, D), "o": (D, D), "gate": (F, D), "up": (F, D), "down": (D, F)}
    w = {n: wl.normal_with_outliers(r, c, 1.0 / np.sqrt(c), 0.002, 100 * l + i)
         for i, (n, (r, c)) in enumerate(shapes.items())}
    views, blobs = {}, {}
    for n in ("q", "k", "v", "o", "down"):
        blobs[n] = s12.s12_encode(to_dev(w[n]))
        views[n] = s12.s12_open(blobs[n])
    blobs["gu"] = s12.s12_encode(s12.interleave_gate_up(to_dev(w["gate"]), to_dev(w["up"])))
    views["gu"] = s12.s12_open(blobs["gu"])
    ref = {n: oracle.encode(w[n]) for n in shapes}
    return views, blobs, ref


@pytest.mark.parametrize("B", [1, 4])
def test_activation_chain_three_layers(s12, oracle, B):
    layers = [_layer(s12, oracle, l) for l in range(LAYERS)]
    h0 = wl.activations(B, D, 77 + B)
    hs = [to_dev(h0)] + [torch.zeros((B, D), dtype=torch.int16, device="cuda") for _ in range(LAYERS)]
    hids = [torch.zeros((B, F), dtype=torch.int16, device="cuda") for _ in range(LAYERS)]
    proj = [[torch.zeros((B, r), dtype=torch.float32, device="cuda") for r in (D, KV, KV, D)] for _ in range(LAYERS)]
    v0 = layers[0][0]
    need = max(s12.s12_gemv_multi_ws_bytes([v0["q"], v0["k"], v0["v"], v0["o"]], B),
               s12.s12_gemv_ws_bytes(v0["gu"], B), s12.s12_gemv_ws_bytes(v0["down"], B))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    flag = new_flag()
    for l, (views, _, _) in enumerate(layers):
        h = hs[l]
        s12.s12_gemv_multi([views["q"], views["k"], views["v"], views["o"]], [h] * 4, proj[l], ws=ws,
                           err_flag=flag)
        s12.s12_gemv_swiglu(views["gu"], h, hids[l], ws=ws, err_flag=flag)
        s12.s12_gemv_bf16(views["down"], hids[l], hs[l + 1], ws=ws, err_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    for l, (_, _, ref) in enumerate(layers):
        h_in = hs[l].cpu().numpy().view(np.uint16)
        for n, y in zip(("q", "k", "v", "o"), proj[l]):
            yr, sr = oracle.gemv_f64(ref[n], h_in)
            assert_within_tolerance(y.cpu().numpy(), yr, sr)
        # the SwiGLU output from this layer's input (tolerance as in the SwiGLU tests)
        hh, g, u, s_g, s_u = oracle.swiglu_f64(ref["gate"], ref["up"], h_in)
        got = wl.bf16_bits_to_f32(hids[l].cpu().numpy().view(np.uint16)).astype(np.float64)
        e_g, e_u = 1e-3 * s_g, 1e-3 * s_u
        silu_g = oracle.silu_mul_f64(g, np.ones_like(g))
        tol = 1.1 * np.abs(u) * e_g + np.abs(silu_g) * e_u + 1.1 * e_g * e_u + 2.0 ** -8 * np.abs(hh) + 1e-30
        assert (np.abs(got - hh) <= tol).all()
        # the down projection of the hidden vector the GPU produced, rounded to BF16
        hid_in = hids[l].cpu().numpy().view(np.uint16)
        yr, sr = oracle.gemv_f64(ref["down"], hid_in)
        y = wl.bf16_bits_to_f32(hs[l + 1].cpu().numpy().view(np.uint16)).astype(np.float64)
        assert (np.abs(y - yr) <= 1e-3 * sr + 2.0 ** -9 * np.abs(yr)).all()
    # the chain carries signal: the last layer's input is not all zero
    assert np.abs(wl.bf16_bits_to_f32(hs[LAYERS].cpu().numpy().view(np.uint16))).max() > 0
