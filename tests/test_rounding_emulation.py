"""CPU checks of the rounding emulation the GPU tests compare with (tests/rounding_emulation.py)."""
import numpy as np

import moe_inputs as mi
import oracle
from rounding_emulation import bf16_round, emulate_layer


def test_bf16_round_is_round_to_nearest_even():
    one = 1.0
    ulp = 2.0 ** -7  # bf16 keeps 7 explicit mantissa bits
    vals = np.array([one, one + ulp / 2, one + 3 * ulp / 2, one + ulp / 4, -(one + ulp / 2), 3.0e38 * 1.1])
    got = bf16_round(vals[:5])
    np.testing.assert_array_equal(got, [one, one, one + 2 * ulp, one, -one])
    x = mi.normal_bf16(mi.STREAM_X, 1000, 1.0)
    np.testing.assert_array_equal(bf16_round(mi.bf16_to_f64(x)), mi.bf16_to_f64(x))  # bf16 values are fixed


def test_emulated_rounding_stays_within_the_bf16_error_budget_of_the_oracle():
    """On the tiny workload the emulated path is off the fp64 oracle by the roundings it applies:
    nonzero, and well inside 2e-2 x RMS(y)."""
    w = mi.WORKLOADS["tiny"]
    h = mi.host_inputs(w, redraw=oracle.gap_redraw(w))
    y_ref, _, _ = oracle.layer(h["x"], h["wg"], h["bias"], h["gate_up"], h["down"], w.k)
    y_emu = emulate_layer(h["x"], h["wg"], h["bias"], h["gate_up"], h["down"], w.k)
    rms = np.sqrt(np.mean(y_ref ** 2))
    err = np.abs(y_emu - y_ref).max() / rms
    assert 1e-3 < err < 2e-2
    # y is a bf16 value everywhere
    np.testing.assert_array_equal(bf16_round(y_emu), y_emu)


def test_emulation_with_shared_expert_bias_and_k3_stays_within_the_budget():
    """A p taken from the wrong slot, a shared expert weighted by p or left out, or a bias in the
    weights would put the emulation O(10%) off the oracle; the roundings alone keep it < 2e-2."""
    w = mi.Workload("emu", T=120, D=128, E=6, k=3, F=128, Fs=64, bias="normal:0.5")
    h = mi.host_inputs(w, redraw=oracle.gap_redraw(w))
    args = (h["x"], h["wg"], h["bias"], h["gate_up"], h["down"], w.k, h["shared_gate_up"], h["shared_down"])
    y_ref, _, _ = oracle.layer(*args)
    y_emu = emulate_layer(*args)
    rms = np.sqrt(np.mean(y_ref ** 2))
    assert 1e-3 < np.abs(y_emu - y_ref).max() / rms < 2e-2
    assert np.sqrt(np.mean((y_emu - y_ref) ** 2)) / rms < 5e-3
