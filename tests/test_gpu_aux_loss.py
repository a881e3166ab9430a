"""The router's load-balancing auxiliary loss on the GPU against the fp64 oracle (pinned in
test_oracle_pins.py), on seeded gap-enforced inputs so that the top-k counts f agree exactly.

Tolerance, from the arithmetic: the logits carry fp32 accumulation error (relative ~1e-6 here),
which the softmax passes on to s and P; the loss is a sum of T*E such terms, and the gradients are
fp32 sums over T (dW_g) or E (dx) of s (f - c) products, where f - c can cancel to ~1e-2 of f.
So: |loss - L| <= 1e-5 |L|, and per gradient RMS(err) <= 1e-4 RMS(oracle), max|err| <=
1e-3 max|oracle|.
"""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
import sparse_mixture_experts_16_b200 as moe
from helpers import gap_redraw, to_torch_bf16

pytestmark = pytest.mark.gpu


def W(T, D, E, k, bias="none"):
    return mi.Workload(f"aux_T{T}D{D}E{E}k{k}", T=T, D=D, E=E, k=k, F=64, Fs=0, bias=bias)


CASES = [
    (W(300, 256, 8, 2), 0.01),
    (W(64, 512, 32, 4, "zipf:1.1"), 0.02),
    (W(1000, 128, 256, 8, "normal:0.5"), 0.001),
    (W(5, 64, 6, 6), 0.1),          # k = E: every expert gets every token, f uniform
    (W(2500, 192, 16, 1), 0.05),    # k = 1; more tokens than one reduction pass
]


def _run(w, alpha):
    import torch

    rd = gap_redraw(w)
    h = mi.host_inputs(w, redraw=rd)
    x, wg = to_torch_bf16(h["x"]), to_torch_bf16(h["wg"])
    bias = None if h["bias"] is None else torch.from_numpy(h["bias"]).cuda()
    loss, dwg, dx = moe.moe_router_aux_loss(x, wg, bias, w.k, alpha)
    torch.cuda.synchronize()
    return h, loss, dwg, dx


@pytest.mark.parametrize("w,alpha", CASES, ids=[c[0].name for c in CASES])
def test_aux_loss_matches_oracle(cuda_device, w, alpha):
    h, loss, dwg, dx = _run(w, alpha)
    L_ref, dwg_ref, dx_ref = oracle.router_aux_loss(h["x"], h["wg"], h["bias"], w.k, alpha)
    assert float(loss.item()) == pytest.approx(L_ref, rel=1e-5)
    xs = np.abs(oracle._f64(h["x"])).max()
    ws = np.abs(oracle._f64(h["wg"])).max()
    for got, ref, operand in ((dwg, dwg_ref, xs), (dx, dx_ref, ws)):
        g = got.double().cpu().numpy()
        if w.k == w.E:
            # every expert takes every token: f = 1/E = c_t, so the exact gradient is 0 and both
            # sides hold only the rounding of f - c (a few fp32 ulps of 1/E, times alpha E / T
            # per term, at most T terms of |operand|)
            assert np.abs(g).max() <= 1e-6 * alpha * operand
            continue
        err = g - ref
        assert np.sqrt(np.mean(err * err)) <= 1e-4 * np.sqrt(np.mean(ref * ref))
        assert np.abs(err).max() <= 1e-3 * np.abs(ref).max()


def test_aux_loss_single_expert_is_alpha_with_zero_gradient(cuda_device):
    """E = 1: f = P = 1, so L = alpha and every logit gradient s (f - c) is exactly 0."""
    h, loss, dwg, dx = _run(W(77, 128, 1, 1), 0.3)
    assert float(loss.item()) == pytest.approx(0.3, rel=1e-6)
    assert not dwg.any() and not dx.any()


def test_aux_loss_is_deterministic(cuda_device):
    w = W(700, 256, 64, 4, "normal:0.5")
    _, l1, g1, x1 = _run(w, 0.01)
    _, l2, g2, x2 = _run(w, 0.01)
    assert bool((l1 == l2).all()) and bool((g1 == g2).all()) and bool((x1 == x2).all())
