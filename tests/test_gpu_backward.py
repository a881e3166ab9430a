"""The layer backward pass on the GPU against the oracle's chain-rule gradients (fp64, pinned by
finite differences in test_oracle_pins.py), on seeded gap-enforced inputs.

Tolerance, derived from the arithmetic: every gradient is a sum of products whose factors carry at
most three bf16 roundings (unit roundoff u = 2^-8: the saved g|u, dO = p*dy or dGU, h or x),
accumulated in fp32, and dx is rounded once more to bf16.  Rounding is relative to each entry, and
gradient tensors are heavy-tailed (peak entries 10-20x the RMS: dx carries the router term
sum_j dl_j W_g[idx_j]), so the bound is normwise:
    RMS(err) <= 1e-2 * RMS(oracle)      (about 2.5u)
    max|err| <= 2e-2 * max|oracle|      (about 5u on the largest entries)
Experts that no token selects get exactly zero.  (A CPU emulation of these rounding points
reproduces the GPU's errors to several digits; the max|err|/RMS metric of the forward output would
charge the same arithmetic 4-5% here.)
"""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
import sparse_mixture_experts_16_b200 as moe
from helpers import bf16_np_to_f64, gap_redraw, to_np_bf16, to_torch_bf16

pytestmark = pytest.mark.gpu

GRAD_RMS_TOL = 1e-2   # RMS(err) / RMS(oracle)
GRAD_PEAK_TOL = 2e-2  # max|err| / max|oracle|


def W(T, D, E, k, F, Fs=0, bias="none"):
    return mi.Workload(f"bwd_T{T}D{D}E{E}k{k}F{F}Fs{Fs}", T=T, D=D, E=E, k=k, F=F, Fs=Fs, bias=bias)


def _dy(w, seed=7):
    return mi.rows_bf16(mi.STREAM_X, np.arange(w.T), w.D, 1.0, seed=1000 + seed)


def _run(w, flags=moe.MOE_FLAG_SAVE_FOR_BACKWARD):
    rd = gap_redraw(w)
    h = mi.host_inputs(w, redraw=rd)
    d = mi.device_inputs(w, redraw=rd)
    dy_h = _dy(w)
    L = moe.MoELayer(d["wg"], d["gate_up"], d["down"], w.k, bias=d["bias"], shared_gate_up=d["shared_gate_up"],
                     shared_down=d["shared_down"], flags=flags)
    y = L(d["x"])
    dx, g = L.backward(d["x"], to_torch_bf16(dy_h))
    assert L.device_error() == 0 and L.backward_error() == 0
    return h, d, dy_h, L, y, dx, g


def _check(w, h, dy_h, dx, g):
    ref = oracle.layer_backward(h["x"], h["wg"], h["bias"], h["gate_up"], h["down"], w.k, dy_h,
                                h["shared_gate_up"], h["shared_down"])
    got = dict(dx=bf16_np_to_f64(to_np_bf16(dx)), **{n: None if t is None else t.double().cpu().numpy()
                                                    for n, t in g.items()})
    for name in ("dx", "dw_gate", "dgate_up", "ddown", "dshared_gate_up", "dshared_down"):
        r, a = ref[name], got[name]
        if r is None:
            assert a is None, name
            continue
        assert a.shape == r.shape, name
        if not np.any(r):
            assert not np.any(a), name
            continue
        diff = a.reshape(r.shape) - r
        rms = float(np.sqrt(np.mean(diff * diff)) / np.sqrt(np.mean(r * r)))
        peak = float(np.abs(diff).max() / np.abs(r).max())
        assert rms <= GRAD_RMS_TOL and peak <= GRAD_PEAK_TOL, f"{name}: rms {rms:.3e} peak {peak:.3e}"
    return ref


CASES = [
    W(96, 128, 8, 2, 256),                                 # one m-tile per expert, ragged dW K
    W(200, 256, 16, 4, 192, Fs=128, bias="normal:0.5"),     # shared expert, bias, ragged N
    W(33, 192, 6, 6, 320),                                  # k = E: every expert, 2.5 column tiles
    W(300, 128, 4, 2, 128, Fs=64),                          # several m-tiles per expert
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_backward_matches_oracle(cuda_device, w):
    h, d, dy_h, L, y, dx, g = _run(w)
    _check(w, h, dy_h, dx, g)


TILINGS = {moe.MOE_FLAG_PREFILL_ROW_TILES: "row_tiles", moe.MOE_FLAG_PREFILL_WIDE_TILES: "wide_tiles",
           moe.MOE_FLAG_PREFILL_PAIR_TILES: "pair_tiles"}


@pytest.mark.parametrize("tiling", list(TILINGS), ids=list(TILINGS.values()))
def test_backward_after_every_forward_tiling(cuda_device, tiling):
    """Every prefill tiling saves the same g | u layout for the backward pass."""
    w = W(300, 256, 4, 2, 192, Fs=128, bias="normal:0.5")
    h, d, dy_h, L, y, dx, g = _run(w, flags=moe.MOE_FLAG_SAVE_FOR_BACKWARD | tiling)
    assert L.gemm_path(w.T) == TILINGS[tiling]
    _check(w, h, dy_h, dx, g)


def test_backward_single_expert_k1_has_no_router_gradient(cuda_device):
    """k = 1: the one softmax weight is 1, so dW_g is exactly zero (and the rest still matches)."""
    w = W(130, 128, 1, 1, 128)
    h, d, dy_h, L, y, dx, g = _run(w)
    _check(w, h, dy_h, dx, g)
    assert not g["dw_gate"].any()


def test_backward_unselected_experts_get_exact_zeros(cuda_device):
    """20 tokens, top-2 of 64 experts: most experts are never chosen and get zero gradients."""
    w = W(20, 128, 64, 2, 128)
    h, d, dy_h, L, y, dx, g = _run(w)
    ref = _check(w, h, dy_h, dx, g)
    unused = [e for e in range(64) if not np.any(ref["ddown"][e])]
    assert len(unused) > 20
    for e in unused:
        assert not g["ddown"][e].any() and not g["dgate_up"][e].any() and not g["dw_gate"][e].any()


def test_training_forward_equals_inference_forward_and_backward_is_deterministic(cuda_device):
    """Saving g|u does not change y (same tiled kernels), and two backward passes agree bit for bit."""
    w = W(64, 256, 8, 2, 256, Fs=128)
    h, d, dy_h, L, y, dx, g = _run(w)
    L2 = moe.MoELayer(d["wg"], d["gate_up"], d["down"], w.k, bias=d["bias"], shared_gate_up=d["shared_gate_up"],
                      shared_down=d["shared_down"], flags=moe.MOE_FLAG_FORCE_PREFILL)
    assert (to_np_bf16(L2(d["x"])) == to_np_bf16(y)).all()
    dx2, g2 = L.backward(d["x"], to_torch_bf16(dy_h))
    assert (to_np_bf16(dx2) == to_np_bf16(dx)).all()
    for n in g:
        if g[n] is not None:
            assert bool((g2[n] == g[n]).all()), n


@pytest.mark.slow
def test_backward_at_gpt_oss_dimensions(cuda_device):
    """D = F = 2880 (gpt-oss-shaped experts: 22.5 row tiles of 128 and 11.25 column tiles of 256, K not
    a multiple of 128), 256 tokens over 4 experts with a Zipf selection bias and a shared expert."""
    w = W(256, 2880, 4, 2, 2880, Fs=576, bias="zipf:1.1")
    h, d, dy_h, L, y, dx, g = _run(w)
    _check(w, h, dy_h, dx, g)
