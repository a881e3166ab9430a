"""Device-side failure detection, without faulting the GPU.

A test-only environment flag makes the TMA producer of the grouped-GEMM kernels withhold its
first copies.  Nothing else is changed: the consumers' waits are bounded (1 s of wall time), so
each kernel records MOE_ERR_TIMEOUT in the workspace's error word, drains its own copies, frees
TMEM and returns.  The host reads the status, and the same context then runs a correct layer.
"""
import time

import numpy as np
import pytest

import moe_inputs as mi
import oracle
import sparse_mixture_experts_16_b200 as moe
from helpers import REL_RMS_TOL, gap_redraw, rel_rms_err, bf16_np_to_f64, to_np_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T", [100, 24], ids=["tiled", "streaming"])
def test_withheld_copy_times_out_and_the_context_stays_usable(cuda_device, monkeypatch, T):
    import torch

    w = mi.Workload(f"fault{T}", T=T, D=128, E=4, k=2, F=128)
    rd = gap_redraw(w)
    h = mi.host_inputs(w, redraw=rd)
    d = mi.device_inputs(w, redraw=rd)
    layer = moe.MoELayer(d["wg"], d["gate_up"], d["down"], w.k)
    layer(d["x"])
    torch.cuda.synchronize()
    assert layer.device_error() == 0

    monkeypatch.setenv("MOE_TEST_WITHHOLD_LOAD", "1")
    t0 = time.time()
    layer(d["x"])
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    monkeypatch.delenv("MOE_TEST_WITHHOLD_LOAD")
    assert layer.device_error() == 7  # MOE_ERR_TIMEOUT
    assert elapsed < 60

    y = layer(d["x"])
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    y_ref, _, _ = oracle.layer(h["x"], h["wg"], None, h["gate_up"], h["down"], w.k)
    assert rel_rms_err(bf16_np_to_f64(to_np_bf16(y)), y_ref) <= REL_RMS_TOL
