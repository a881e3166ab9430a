"""Shared test helpers: workload preparation (gap-enforced inputs), host/device conversions and
the output tolerance."""
from __future__ import annotations

import numpy as np

import moe_inputs as mi
import oracle

from oracle import GAP, gap_redraw, gap_violations  # noqa: F401  (re-exported for the tests)

# Layer outputs: max |y_gpu - y_oracle| <= REL_RMS_TOL * RMS(y_oracle)  (bf16 weights and
# activations, fp32 accumulation).
REL_RMS_TOL = 2e-2

# Router weights: fp32 logits differ from the fp64 ones by ~u32 * sqrt(D) * |partial sums|
# (<= ~5e-5 for D = 7168, logits of std 8.5); a softmax weight moves by at most the largest
# logit error.  2e-4 keeps a 4x margin.
P_ATOL = 2e-4


def scores(w: mi.Workload, x_rows: np.ndarray, wg: np.ndarray, bias):
    return oracle.scores(x_rows, wg, bias, w.k)


def to_torch_bf16(a: np.ndarray, device="cuda"):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def to_np_bf16(t) -> np.ndarray:
    import torch

    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_np_to_f64(a: np.ndarray) -> np.ndarray:
    return mi.bf16_to_f64(a)


def rel_rms_err(got: np.ndarray, ref: np.ndarray) -> float:
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref))) / max(rms, 1e-30)
