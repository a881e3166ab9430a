"""FP8 (E4M3) expert weights on the GPU: the quantiser is bit-exact against the oracle's, and the
FP8-weight decode layer matches the oracle evaluated on the same dequantised weights (fp64) within
max|err| <= 2e-2 * RMS(y_oracle)."""
import numpy as np
import pytest

import moe_inputs as mi
import oracle
import sparse_mixture_experts_16_b200 as moe
from helpers import REL_RMS_TOL, bf16_np_to_f64, gap_redraw, rel_rms_err, to_np_bf16, to_torch_bf16

pytestmark = pytest.mark.gpu


def W(T, D, E, k, F, Fs=0, bias="none"):
    return mi.Workload(f"fp8_T{T}D{D}E{E}k{k}F{F}Fs{Fs}", T=T, D=D, E=E, k=k, F=F, Fs=Fs, bias=bias)


@pytest.mark.parametrize("rows,K", [(1, 64), (37, 256), (300, 2880)])
def test_quantizer_matches_oracle_bit_for_bit(cuda_device, rows, K):
    w = mi.rows_bf16(mi.STREAM_GATE_UP, np.arange(rows), K, 0.02, seed=rows)
    if rows > 2:
        w[1] = 0                                    # an all-zero row
        w[2, :5] = mi.rows_bf16(mi.STREAM_X, [0], 5, 30.0)[0]  # a row with a large outlier
    q_ref, s_ref = oracle.quantize_rows_fp8(w)
    q, s = moe.moe_quantize_rows_fp8(to_torch_bf16(w))
    assert (s.cpu().numpy() == s_ref).all()
    assert (q.cpu().numpy() == q_ref).all()


def _quantized_layer(w, rd):
    """Host inputs, the oracle's FP8 weights, and a device layer built from GPU-quantised weights."""
    import torch

    h = mi.host_inputs(w, redraw=rd)
    d = mi.device_inputs(w, redraw=rd)
    q_gu, s_gu = moe.moe_quantize_rows_fp8(d["gate_up"])
    q_dn, s_dn = moe.moe_quantize_rows_fp8(d["down"])
    scales = dict(gate_up=s_gu, down=s_dn)
    sh_q = sh_s = (None, None)
    if w.Fs:
        sh_q = moe.moe_quantize_rows_fp8(d["shared_gate_up"])
        sh_s = moe.moe_quantize_rows_fp8(d["shared_down"])
        scales.update(shared_gate_up=sh_q[1], shared_down=sh_s[1])
    layer = moe.MoELayer(d["wg"], q_gu, q_dn, w.k, bias=d["bias"], shared_gate_up=sh_q[0], shared_down=sh_s[0],
                         scales=scales)
    return h, d, layer


@pytest.mark.parametrize("w", [W(1, 256, 8, 2, 192), W(16, 512, 32, 4, 256, Fs=128, bias="normal:0.5"),
                               W(64, 256, 16, 8, 128, Fs=64), W(33, 192, 6, 6, 320), W(48, 2880, 32, 4, 2880,
                                                                                       bias="zipf:1.1")],
                         ids=lambda w: w.name)
def test_fp8_layer_parity(cuda_device, w):
    rd = gap_redraw(w)
    h, d, layer = _quantized_layer(w, rd)
    q = {}
    q["gu_q"], q["gu_s"] = oracle.quantize_rows_fp8(h["gate_up"])
    q["dn_q"], q["dn_s"] = oracle.quantize_rows_fp8(h["down"])
    assert (layer.gate_up.cpu().numpy() == q["gu_q"]).all() and (layer.scales["down"].cpu().numpy() == q["dn_s"]).all()
    shared = None
    if w.Fs:
        a, b = oracle.quantize_rows_fp8(h["shared_gate_up"])
        c, e = oracle.quantize_rows_fp8(h["shared_down"])
        shared = dict(gu_q=a, gu_s=b, dn_q=c, dn_s=e)
    y = layer(d["x"])
    assert layer.device_error() == 0
    y_ref, _, _ = oracle.layer_fp8(h["x"], h["wg"], h["bias"], w.k, q, shared)
    assert rel_rms_err(bf16_np_to_f64(to_np_bf16(y)), y_ref) <= REL_RMS_TOL
    # The quantisation itself: E4M3 keeps 3 mantissa bits, so against the bf16 layer the RMS error
    # is a few percent (max|err| / RMS reaches ~0.25 at these sizes); a wrong scale would be far off.
    y_bf16, _, _ = oracle.layer(h["x"], h["wg"], h["bias"], h["gate_up"], h["down"], w.k, h["shared_gate_up"],
                                h["shared_down"])
    diff = y_ref - y_bf16
    assert np.sqrt(np.mean(diff * diff)) < 0.1 * np.sqrt(np.mean(y_bf16 * y_bf16))


@pytest.mark.slow
@pytest.mark.parametrize("name,n_tok", [("deepseek_decode", 2), ("gptoss_decode_T64", 4), ("gptoss_decode_T1", 1)])
def test_fp8_full_size_sampled(cuda_device, name, n_tok):
    import torch

    w = mi.WORKLOADS[name]
    rd = gap_redraw(w)
    d = mi.device_inputs(w, redraw=rd)
    q_gu, s_gu = moe.moe_quantize_rows_fp8(d["gate_up"])
    q_dn, s_dn = moe.moe_quantize_rows_fp8(d["down"])
    scales = dict(gate_up=s_gu, down=s_dn)
    sq = (None, None), (None, None)
    if w.Fs:
        sq = moe.moe_quantize_rows_fp8(d["shared_gate_up"]), moe.moe_quantize_rows_fp8(d["shared_down"])
        scales.update(shared_gate_up=sq[0][1], shared_down=sq[1][1])
    del d["gate_up"], d["down"]
    layer = moe.MoELayer(d["wg"], q_gu, q_dn, w.k, bias=d["bias"], shared_gate_up=sq[0][0], shared_down=sq[1][0],
                         scales=scales)
    y = layer(d["x"])
    torch.cuda.synchronize()
    assert layer.device_error() == 0
    x_h = mi.host_x(w, redraw=rd)
    wg_h, bias_h = mi.host_wg(w), mi.bias_f32(w)
    rows = np.random.default_rng(2).choice(w.T, size=n_tok, replace=False)
    idx, _ = oracle.router(x_h[rows], wg_h, bias_h, w.k)
    used = sorted(set(idx.reshape(-1).tolist()))
    q = dict(gu_q={}, gu_s={}, dn_q={}, dn_s={})
    for e, gu, dn in zip(used, mi.host_gate_up(w, used), mi.host_down(w, used)):
        q["gu_q"][e], q["gu_s"][e] = oracle.quantize_rows_fp8(gu)
        q["dn_q"][e], q["dn_s"][e] = oracle.quantize_rows_fp8(dn)
    shared = None
    if w.Fs:
        sgu, sdn = mi.host_shared(w)
        a, b = oracle.quantize_rows_fp8(sgu)
        c, e = oracle.quantize_rows_fp8(sdn)
        shared = dict(gu_q=a, gu_s=b, dn_q=c, dn_s=e)
    y_ref, _, _ = oracle.layer_fp8(x_h[rows], wg_h, bias_h, w.k, q, shared)
    got = bf16_np_to_f64(to_np_bf16(y[torch.from_numpy(rows).cuda()]))
    assert rel_rms_err(got, y_ref) <= REL_RMS_TOL


def test_fp8_decode_split_k_deterministic_matches_oracle_and_leaves_counters_zero():
    """One token on 4 of 16 experts with F = 1024: 4 x 8 units of 128 rows (+ the shared expert),
    far fewer than SMs, so the FP8 GEMMs split K.  The last split of each unit sums the partials in
    a fixed order: repeated forwards are bit-identical and match the oracle, and the split
    counters (which follow the 256-byte error header of the workspace) are back to zero."""
    w = W(1, 512, 16, 4, 1024, Fs=256)
    rd = gap_redraw(w)
    h, d, layer = _quantized_layer(w, rd)
    ys = [to_np_bf16(layer(d["x"])) for _ in range(3)]
    assert all((y == ys[0]).all() for y in ys[1:])
    assert layer.device_error() == 0
    ws = layer.workspace(w.T)
    assert int(ws[256:256 + 4096].count_nonzero()) == 0
    q = {}
    q["gu_q"], q["gu_s"] = oracle.quantize_rows_fp8(h["gate_up"])
    q["dn_q"], q["dn_s"] = oracle.quantize_rows_fp8(h["down"])
    a, b = oracle.quantize_rows_fp8(h["shared_gate_up"])
    c, e = oracle.quantize_rows_fp8(h["shared_down"])
    y_ref, _, _ = oracle.layer_fp8(h["x"], h["wg"], h["bias"], w.k, q, dict(gu_q=a, gu_s=b, dn_q=c, dn_s=e))
    assert rel_rms_err(bf16_np_to_f64(ys[0]), y_ref) <= REL_RMS_TOL
