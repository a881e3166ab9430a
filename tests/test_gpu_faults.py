"""Device-side failure detection, without faulting the GPU.

A test-only environment variable, MOE_TEST_WITHHOLD_LOAD=n (read once per process), makes the
first n expert-GEMM launches of the process withhold the first stage's copies of every CTA.
Nothing else changes: the consumers' waits are bounded (1 s of wall time), so the kernel records
MOE_ERR_TIMEOUT in the workspace's error word, drains its own copies, frees TMEM and returns.
Each case runs in a child process started with n = 1: its first forward's gate_up launch times
out, the host reads the status, and the next forward on the same context must match the oracle.
The expert-GEMM kernels are covered: 128-row tiles, token-wide tiles (one CTA and CTA pairs) and
weight streaming.
"""
import json
import os
import subprocess
import sys

import pytest

import sparse_mixture_experts_16_b200 as moe

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import json, sys, time
sys.path[:0] = [{root!r}, {tests!r}]
import torch
import moe_inputs as mi
import oracle
import sparse_mixture_experts_16_b200 as moe
from helpers import bf16_np_to_f64, gap_redraw, rel_rms_err, to_np_bf16

T, flags = {T}, {flags}
w = mi.Workload("fault", T=T, D=128, E=4, k=2, F=128)
rd = gap_redraw(w)
h = mi.host_inputs(w, redraw=rd)
d = mi.device_inputs(w, redraw=rd)
torch.cuda.synchronize()
layer = moe.MoELayer(d["wg"], d["gate_up"], d["down"], w.k, flags=flags)
t0 = time.time()
layer(d["x"])                       # its gate_up launch withholds its first copies
torch.cuda.synchronize()
elapsed = time.time() - t0
first = layer.device_error()
y = layer(d["x"])                   # a normal forward on the same context
torch.cuda.synchronize()
second = layer.device_error()
y_ref, _, _ = oracle.layer(h["x"], h["wg"], None, h["gate_up"], h["down"], w.k)
err = rel_rms_err(bf16_np_to_f64(to_np_bf16(y)), y_ref)
print("RESULT " + json.dumps(dict(first=first, second=second, elapsed=elapsed, err=err,
                                  path=layer.gemm_path(T))))
"""

CASES = [(100, moe.MOE_FLAG_PREFILL_ROW_TILES, "row_tiles"), (100, moe.MOE_FLAG_PREFILL_WIDE_TILES, "wide_tiles"),
         (100, moe.MOE_FLAG_PREFILL_PAIR_TILES, "pair_tiles"), (24, 0, "streaming")]


@pytest.mark.parametrize("T,flags,path", CASES, ids=[c[2] for c in CASES])
def test_withheld_copy_times_out_and_the_context_stays_usable(cuda_device, T, flags, path):
    from sparse_mixture_experts_16_b200 import build

    build.build()
    env = dict(os.environ, MOE_TEST_WITHHOLD_LOAD="1")
    code = CHILD.format(root=ROOT, tests=os.path.join(ROOT, "tests"), T=T, flags=flags)
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    res = json.loads(line[len("RESULT "):])
    assert res["path"] == path
    assert res["first"] == 7  # MOE_ERR_TIMEOUT
    assert res["elapsed"] < 60
    assert res["second"] == 0
    assert res["err"] <= 2e-2
