"""The seeded input generator (CPU): published SplitMix64 values, the Irwin-Hall normal
transform, bf16 rounding, determinism and random access."""
import os

import numpy as np

import moe_inputs as mi

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
M64 = (1 << 64) - 1
GOLD = 0x9E3779B97F4A7C15


def _read_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def test_mix64_matches_published_splitmix64_outputs():
    rows = _read_golden("splitmix64_seed0.txt")
    for n, (val,) in enumerate(rows, start=1):
        assert mi.lib().mi_mix64_host((GOLD * n) & M64) == int(val, 16)


def test_normal_is_irwin_hall_of_twelve_16bit_uniforms():
    """Recompute a few variates from the raw words in Python: sum of 12 chunks, centred, / 2^16."""
    seed, stream = 5, mi.STREAM_X
    key = None
    # the stream key is mix64(mix64(seed) ^ mix64((stream << 32) | redraw))
    m = mi.lib().mi_mix64_host
    key = m(m(seed) ^ m((stream << 32) | 0))
    for i in [0, 1, 17, 123456]:
        s = 0
        for c in range(3):
            w = m((key + GOLD * (3 * i + c + 1)) & M64)
            s += sum((w >> (16 * q)) & 0xFFFF for q in range(4))
        assert mi.lib().mi_normal_host(seed, stream, 0, i) == (s - 393210) / 65536.0


def test_moments_and_bf16_rounding():
    a = mi.normal_bf16(mi.STREAM_GATE_UP, 400_000, 0.02)
    v = mi.bf16_to_f64(a)
    assert abs(v.mean()) < 3 * 0.02 / np.sqrt(v.size) * 2
    assert abs(v.std() / 0.02 - 1) < 0.01
    # every value is representable in bf16: round-tripping through float32 bits is exact
    assert (((v.astype(np.float32).view(np.uint32)) & 0xFFFF) == 0).all()
    # round to nearest even of z * sigma (recompute for a few variates)
    key_vals = [mi.lib().mi_normal_host(0, mi.STREAM_GATE_UP, 0, i) for i in range(64)]
    ref = np.array(key_vals, np.float32) * np.float32(0.02)
    u = ref.view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    assert (u == a[:64]).all()


def test_random_access_and_determinism():
    full = mi.normal_bf16(mi.STREAM_DOWN, 10_000, 0.02, seed=3)
    part = mi.normal_bf16(mi.STREAM_DOWN, 100, 0.02, seed=3, first=5000)
    assert (full[5000:5100] == part).all()
    assert (mi.normal_bf16(mi.STREAM_DOWN, 10_000, 0.02, seed=3) == full).all()
    assert not (mi.normal_bf16(mi.STREAM_DOWN, 10_000, 0.02, seed=4) == full).all()
    w = mi.WORKLOADS["tiny"]
    x = mi.host_x(w)
    rows = mi.host_x(w, rows=[7, 200])
    assert (rows == x[[7, 200]]).all()
    redrawn = mi.host_x(w, rows=[7], redraw=[1])
    assert not (redrawn[0] == x[7]).all()


def test_expert_slices_match_packed_tensor():
    w = mi.WORKLOADS["tiny"]
    gu = mi.host_gate_up(w)
    assert gu.shape == (w.E, 2 * w.F, w.D)
    assert (mi.host_gate_up(w, [5])[0] == gu[5]).all()
    dn = mi.host_down(w)
    assert (mi.host_down(w, [3])[0] == dn[3]).all()


def test_bias_recipes():
    z = mi.bias_f32(mi.WORKLOADS["gptoss"])
    ranks = np.rint(np.exp(-z.astype(np.float64) / 1.1)).astype(int)
    assert sorted(ranks.tolist()) == list(range(1, 33))
    b = mi.bias_f32(mi.WORKLOADS["deepseek"])
    assert b.dtype == np.float32 and b.shape == (256,) and 0.3 < b.std() < 0.7
    assert mi.bias_f32(mi.WORKLOADS["mixtral"]) is None
