"""Aux-loss-free balancing bias update on the GPU (gotburnout.io glossary "MoE", section 2
item 4): bit-exact against the oracle's rule, and a closed loop of layer forwards + updates
that lowers the load imbalance of a skewed router."""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
import sparse_mixture_experts_16_b200 as moe

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("E", [1, 7, 32, 256, 1024])
def test_bias_update_matches_oracle_bit_for_bit(cuda_device, E):
    import torch

    rng = np.random.default_rng(E)
    counts = rng.integers(0, 1000, E).astype(np.int32)
    counts[: E // 3] = counts[0]  # some equal loads, and (for E = 1) the mean itself
    bias = (rng.standard_normal(E) * 0.7).astype(np.float32)
    for gamma in (0.0, 1e-3, 0.0625):
        b = torch.from_numpy(bias).cuda()
        moe.moe_update_router_bias(torch.from_numpy(counts).cuda(), gamma, b)
        assert (b.cpu().numpy() == oracle.update_bias(counts, gamma, bias)).all()


def test_closed_loop_balancing_lowers_imbalance(cuda_device):
    import torch

    w = mi.Workload("balance", T=1024, D=256, E=32, k=4, F=128, bias="zipf:1.1")
    d = mi.device_inputs(w)
    bias = d["bias"].clone()
    layer = moe.MoELayer(d["wg"], d["gate_up"], d["down"], w.k, bias=bias)
    ratios = []
    for step in range(30):
        layer(d["x"])
        counts = layer.expert_counts(w.T)
        c = counts.cpu().numpy().copy()
        ratios.append(c.max() / c.mean())
        before = bias.cpu().numpy().copy()
        moe.moe_update_router_bias(counts, 0.05, bias)  # in place: the layer sees it next forward
        torch.cuda.synchronize()
        assert (bias.cpu().numpy() == oracle.update_bias(c, 0.05, before)).all()
        assert c.sum() == w.T * w.k
    assert layer.device_error() == 0
    assert ratios[-1] < 0.6 * ratios[0], ratios
