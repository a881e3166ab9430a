"""Pins of the fp64 oracle to things other than itself (CPU only).

Each test ties one part of the oracle to a fact fixed by the pages' definition or by
mathematics -- an exhaustive search, a closed form, an invariance, a textbook reduction --
chosen so that a plausible slip in the oracle (dropped term, wrong sign, wrong index,
transposed operand, SiLU on the wrong half, bias in the weights) fails at least one of them.

Definition (gotburnout.io glossary "MoE", section 2; josueisai.com "Mixture of experts",
section "El router"): p = Softmax(TopK(W_g x)) normalised over the chosen k only,
y = sum_i p_i Expert_i(x) + shared experts, Expert(x) = (silu(x G^T) * (x U^T)) Down^T.
"""
import math

import numpy as np
import pytest

import moe_inputs as mi
import oracle

f64 = mi.bf16_to_f64


def _bf16(a):
    """float64 array -> bf16 bit patterns (round to nearest even)."""
    u = np.asarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def _rand_layer(rng, T, D, E, F, Fs=0, wscale=0.05):
    x = _bf16(rng.standard_normal((T, D)))
    wg = _bf16(rng.standard_normal((E, D)) * 0.3)
    gu = _bf16(rng.standard_normal((E, 2 * F, D)) * wscale)
    dn = _bf16(rng.standard_normal((E, D, F)) * wscale)
    sgu = _bf16(rng.standard_normal((2 * Fs, D)) * wscale) if Fs else None
    sdn = _bf16(rng.standard_normal((D, Fs)) * wscale) if Fs else None
    return x, wg, gu, dn, sgu, sdn


def _dense_swiglu(x, gu, dn):
    """Textbook dense SwiGLU FFN with numpy matmuls: (silu(x G^T) * (x U^T)) Down^T."""
    X, GU, DN = f64(x), f64(gu), f64(dn)
    F = DN.shape[1]
    g = X @ GU[:F].T
    u = X @ GU[F:].T
    a = g / (1.0 + np.exp(-g)) * u
    return a @ DN.T


# ----------------------------------------------------------------------------- router
@pytest.mark.parametrize("E,k", [(8, 1), (8, 2), (8, 3), (8, 8), (5, 3), (12, 4)])
def test_topk_equals_exhaustive_subset_search(E, k):
    rng = np.random.default_rng(E * 31 + k)
    x, wg, *_ = _rand_layer(rng, 64, 32, E, 8)
    bias = (rng.standard_normal(E) * 0.5).astype(np.float32)
    idx, p, lg = oracle.router(x, wg, bias, k, return_logits=True)
    s = lg + bias.astype(np.float64)
    assert (idx == oracle.topk_exhaustive(s, k)).all()


def test_logits_equal_library_matmul():
    rng = np.random.default_rng(1)
    x, wg, *_ = _rand_layer(rng, 40, 96, 7, 8)
    _, _, lg = oracle.router(x, wg, None, 2, return_logits=True)
    ref = f64(x) @ f64(wg).T
    np.testing.assert_allclose(lg, ref, rtol=1e-13, atol=1e-13)


def test_weights_sum_to_one_and_are_descending():
    rng = np.random.default_rng(2)
    x, wg, *_ = _rand_layer(rng, 200, 64, 16, 8)
    idx, p = oracle.router(x, wg, None, 4)
    assert np.abs(p.sum(1) - 1.0).max() <= 1e-12
    assert (np.diff(p, axis=1) <= 0).all()  # without bias, score order = weight order
    assert (p > 0).all()


def test_k1_weight_is_one():
    rng = np.random.default_rng(3)
    x, wg, *_ = _rand_layer(rng, 50, 32, 6, 8)
    _, p = oracle.router(x, wg, None, 1)
    assert (p == 1.0).all()


def test_k2_weights_are_logistic_of_logit_gap():
    """softmax over two chosen logits = logistic sigmoid of their difference (closed form)."""
    rng = np.random.default_rng(4)
    x, wg, *_ = _rand_layer(rng, 64, 48, 8, 8)
    idx, p, lg = oracle.router(x, wg, None, 2, return_logits=True)
    l0 = lg[np.arange(64), idx[:, 0]]
    l1 = lg[np.arange(64), idx[:, 1]]
    ref = np.array([1.0 / (1.0 + math.exp(b - a)) for a, b in zip(l0, l1)])
    np.testing.assert_allclose(p[:, 0], ref, rtol=0, atol=1e-14)
    np.testing.assert_allclose(p[:, 1], 1.0 - ref, rtol=0, atol=1e-14)


def test_shifting_every_logit_or_every_bias_changes_nothing():
    rng = np.random.default_rng(5)
    x, wg, *_ = _rand_layer(rng, 80, 32, 8, 8)
    bias = (rng.standard_normal(8) * 0.5).astype(np.float32)
    idx, p = oracle.router(x, wg, bias, 3)
    # append an all-ones feature whose router weight is 2.0 for every expert: logits + 2
    x2 = np.concatenate([x, np.full((80, 1), _bf16([1.0])[0], np.uint16)], axis=1)
    wg2 = np.concatenate([wg, np.full((8, 1), _bf16([2.0])[0], np.uint16)], axis=1)
    idx2, p2 = oracle.router(x2, wg2, bias, 3)
    assert (idx2 == idx).all()
    np.testing.assert_allclose(p2, p, rtol=0, atol=1e-13)
    idx3, p3 = oracle.router(x, wg, bias + np.float32(0.75), 3)
    assert (idx3 == idx).all()
    assert (p3 == p).all()


def test_bias_steers_selection_but_not_weights():
    rng = np.random.default_rng(6)
    x, wg, *_ = _rand_layer(rng, 30, 32, 8, 8)
    bias = np.zeros(8, np.float32)
    bias[5] = 1000.0
    idx, p, lg = oracle.router(x, wg, bias, 2, return_logits=True)
    assert (idx[:, 0] == 5).all()
    for t in range(30):
        l = lg[t, idx[t]]
        ref = np.exp(l - l.max()) / np.exp(l - l.max()).sum()
        np.testing.assert_allclose(p[t], ref, rtol=0, atol=1e-14)


# ----------------------------------------------------------------------------- dispatch
def test_permute_is_stable_sort_by_expert():
    rng = np.random.default_rng(7)
    T, E, k = 300, 13, 3
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, pt, ps, inv = oracle.permute(idx, E)
    flat = idx.reshape(-1)
    assert (counts == np.bincount(flat, minlength=E)).all()
    assert offsets[0] == 0 and (offsets[1:] == np.cumsum(counts)).all()
    order = np.argsort(flat, kind="stable")  # library stable sort of the (t, j) slots
    assert (pt == order // k).all() and (ps == order % k).all()
    assert (inv[order] == np.arange(T * k)).all()  # inv_perm o perm = identity
    assert sorted(inv.tolist()) == list(range(T * k))  # bijection
    for e in range(E):
        seg = pt[offsets[e]:offsets[e + 1]]
        assert (np.diff(seg) > 0).all()
        assert (flat[order[offsets[e]:offsets[e + 1]]] == e).all()


def test_permute_counts_equal_router_histogram():
    rng = np.random.default_rng(8)
    x, wg, *_ = _rand_layer(rng, 257, 64, 9, 8)
    idx, _ = oracle.router(x, wg, None, 2)
    counts, offsets, *_ = oracle.permute(idx, 9)
    for e in range(9):
        assert counts[e] == int((idx == e).sum())
    assert offsets[-1] == 257 * 2


def test_permute_rejects_out_of_range_ids():
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, 5]], np.int32), 4)


# ----------------------------------------------------------------------------- experts
def test_single_expert_reduces_to_dense_swiglu():
    rng = np.random.default_rng(9)
    x, wg, gu, dn, _, _ = _rand_layer(rng, 33, 64, 1, 48)
    y, idx, p = oracle.layer(x, wg, None, gu, dn, 1)
    assert (idx == 0).all() and (p == 1).all()
    np.testing.assert_allclose(y, _dense_swiglu(x, gu[0], dn[0]), rtol=1e-12, atol=1e-14)


def test_scalar_closed_form():
    """D = F = 1: y = c * silu(a x) * (b x), with a the gate (first-half) weight."""
    for (xv, a, b, c) in [(1.5, 0.75, -2.0, 0.5), (-3.0, 1.25, 0.5, -1.0), (0.25, -4.0, 3.0, 2.0)]:
        x = _bf16([[xv]])
        wg = _bf16([[1.0]])
        gu = _bf16([[[a], [b]]])
        dn = _bf16([[[c]]])
        y, _, _ = oracle.layer(x, wg, None, gu, dn, 1)
        g = a * xv
        ref = c * (g / (1.0 + math.exp(-g))) * (b * xv)
        assert abs(y[0, 0] - ref) <= 1e-15 * max(1.0, abs(ref))


def test_identical_experts_with_k_equal_E_give_dense_ffn():
    rng = np.random.default_rng(10)
    T, D, E, F = 20, 32, 4, 24
    x, wg, gu, dn, _, _ = _rand_layer(rng, T, D, E, F)
    gu[:] = gu[0]
    dn[:] = dn[0]
    y, _, _ = oracle.layer(x, wg, None, gu, dn, E)
    np.testing.assert_allclose(y, _dense_swiglu(x, gu[0], dn[0]), rtol=1e-12, atol=1e-14)


def test_scaling_down_proj_scales_output():
    rng = np.random.default_rng(11)
    x, wg, gu, dn, _, _ = _rand_layer(rng, 25, 32, 6, 16)
    y1, _, _ = oracle.layer(x, wg, None, gu, dn, 2)
    y2, _, _ = oracle.layer(x, wg, None, gu, _bf16(f64(dn) * 2.0), 2)
    np.testing.assert_array_equal(y2, 2.0 * y1)


def test_relabelling_experts_leaves_output_unchanged():
    rng = np.random.default_rng(12)
    E = 7
    x, wg, gu, dn, _, _ = _rand_layer(rng, 40, 32, E, 16)
    bias = (rng.standard_normal(E) * 0.3).astype(np.float32)
    y1, idx1, _ = oracle.layer(x, wg, bias, gu, dn, 3)
    perm = rng.permutation(E)
    y2, idx2, _ = oracle.layer(x, wg[perm], bias[perm], gu[perm], dn[perm], 3)
    assert (perm[idx2] == idx1).all()
    np.testing.assert_array_equal(y2, y1)


def test_permuting_tokens_permutes_output():
    rng = np.random.default_rng(13)
    x, wg, gu, dn, sgu, sdn = _rand_layer(rng, 37, 32, 5, 16, Fs=8)
    y1, _, _ = oracle.layer(x, wg, None, gu, dn, 2, sgu, sdn)
    perm = rng.permutation(37)
    y2, _, _ = oracle.layer(x[perm], wg, None, gu, dn, 2, sgu, sdn)
    np.testing.assert_array_equal(y2, y1[perm])


def test_shared_expert_adds_a_dense_ffn():
    rng = np.random.default_rng(14)
    x, wg, gu, dn, sgu, sdn = _rand_layer(rng, 30, 64, 6, 32, Fs=40)
    y0, _, _ = oracle.layer(x, wg, None, gu, dn, 2)
    y1, _, _ = oracle.layer(x, wg, None, gu, dn, 2, sgu, sdn)
    np.testing.assert_allclose(y1 - y0, _dense_swiglu(x, sgu, sdn), rtol=1e-10, atol=1e-13)


def test_routed_output_equals_weighted_sum_of_dense_experts():
    """y_t = sum_j p_tj * DenseFFN_{idx_tj}(x_t), each expert evaluated with numpy matmuls."""
    rng = np.random.default_rng(15)
    T, E, k = 50, 6, 3
    x, wg, gu, dn, _, _ = _rand_layer(rng, T, 48, E, 32)
    y, idx, p = oracle.layer(x, wg, None, gu, dn, k)
    dense = np.stack([_dense_swiglu(x, gu[e], dn[e]) for e in range(E)])  # [E, T, D]
    ref = np.zeros_like(y)
    for t in range(T):
        for j in range(k):
            ref[t] += p[t, j] * dense[idx[t, j], t]
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-14)


def test_eager_loop_equals_layer():
    rng = np.random.default_rng(16)
    x, wg, gu, dn, sgu, sdn = _rand_layer(rng, 45, 32, 8, 16, Fs=16)
    bias = (rng.standard_normal(8) * 0.4).astype(np.float32)
    y, _, _ = oracle.layer(x, wg, bias, gu, dn, 2, sgu, sdn)
    ye = oracle.layer_eager(x, wg, bias, gu, dn, 2, sgu, sdn)
    np.testing.assert_allclose(ye, y, rtol=1e-13, atol=1e-15)


def test_expert_ffn_matches_layer_for_single_assignment():
    rng = np.random.default_rng(17)
    x, wg, gu, dn, _, _ = _rand_layer(rng, 3, 64, 4, 32)
    y, idx, p = oracle.layer(x, wg, None, gu, dn, 1)
    for t in range(3):
        np.testing.assert_array_equal(oracle.expert_ffn(x[t], gu[idx[t, 0]], dn[idx[t, 0]]), y[t])


def test_sparse_expert_dict_matches_packed():
    w = mi.WORKLOADS["tiny"]
    inp = mi.host_inputs(w)
    x = inp["x"][:16]
    y1, idx, _ = oracle.layer(x, inp["wg"], None, inp["gate_up"], inp["down"], w.k)
    used = sorted(set(idx.reshape(-1).tolist()))
    y2, _, _ = oracle.layer(x, inp["wg"], None, {e: inp["gate_up"][e] for e in used},
                            {e: inp["down"][e] for e in used}, w.k)
    np.testing.assert_array_equal(y1, y2)


# ----------------------------------------------------------------------------- balancing bias
def test_bias_update_leaves_balanced_loads_alone():
    b = np.linspace(-1, 1, 8).astype(np.float32)
    assert (oracle.update_bias(np.full(8, 37, np.int32), 0.01, b) == b).all()


def test_bias_update_closed_form():
    """Loads 10, 30, 20 (mean 20): +gamma, -gamma, 0; the result is the fp32 sum."""
    b = np.array([0.5, 0.25, -1.0], np.float32)
    out = oracle.update_bias(np.array([10, 30, 20], np.int32), 0.125, b)
    assert out.tolist() == [0.625, 0.125, -1.0]
    # a step of half an ulp (on either side of 1024) rounds back to 1024 (ties to even)
    big = np.array([1024.0, 1024.0], np.float32)
    assert (oracle.update_bias(np.array([1, 3], np.int32), 2.0 ** -15, big) == big).all()


def test_bias_update_is_scale_free_and_follows_loads():
    rng = np.random.default_rng(18)
    c = rng.integers(0, 500, 64).astype(np.int32)
    b = (rng.standard_normal(64) * 0.3).astype(np.float32)
    out = oracle.update_bias(c, 0.01, b)
    assert (oracle.update_bias(c * 7, 0.01, b) == out).all()  # only relative loads matter
    mean = c.mean()
    assert (out[c > mean] < b[c > mean]).all() and (out[c < mean] > b[c < mean]).all()


def test_bias_update_moves_routing_towards_balance():
    """A few steps on a strongly skewed router lower the max/mean load (the rule's purpose)."""
    rng = np.random.default_rng(19)
    T, D, E, k = 512, 64, 16, 2
    x, wg, *_ = _rand_layer(rng, T, D, E, 8)
    bias = np.zeros(E, np.float32)
    bias[:3] = 3.0  # three favourite experts
    def imbalance(b):
        idx, _ = oracle.router(x, wg, b, k)
        c = np.bincount(idx.ravel(), minlength=E)
        return c.max() / c.mean(), c
    start, c = imbalance(bias)
    for _ in range(40):
        bias = oracle.update_bias(c.astype(np.int32), 0.1, bias)
        _, c = imbalance(bias)
    assert imbalance(bias)[0] < 0.6 * start


# ----------------------------------------------------------------------------- FP8 (E4M3) weights
def test_e4m3_code_values():
    """OCP FP8 E4M3: bias 7, 3 mantissa bits, no infinities, S.1111.111 is NaN."""
    assert oracle.e4m3_value(0x38) == 1.0
    assert oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0x08) == 2.0 ** -6          # smallest normal
    assert oracle.e4m3_value(0x01) == 2.0 ** -9          # smallest subnormal
    assert oracle.e4m3_value(0x07) == 7 * 2.0 ** -9
    assert oracle.e4m3_value(0xB8) == -1.0
    assert math.isnan(oracle.e4m3_value(0x7F)) and math.isnan(oracle.e4m3_value(0xFF))


def test_e4m3_encode_rounds_to_nearest_even_and_saturates():
    assert oracle.e4m3_encode(1.0) == 0x38
    assert oracle.e4m3_encode(1.0625) == 0x38            # halfway 1 .. 1.125 -> even
    assert oracle.e4m3_encode(1.1875) == 0x3A            # halfway 1.125 .. 1.25 -> even
    assert oracle.e4m3_encode(1.06) == 0x38 and oracle.e4m3_encode(1.07) == 0x39
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00        # halfway 0 .. 2^-9 -> even (zero)
    assert oracle.e4m3_encode(3 * 2.0 ** -10) == 0x02    # halfway 2^-9 .. 2^-8 -> even
    assert oracle.e4m3_encode(447.9) == 0x7E and oracle.e4m3_encode(1e6) == 0x7E
    assert oracle.e4m3_encode(-1e6) == 0xFE
    for c in list(range(0x00, 0x7F)) + list(range(0x81, 0xFF)):  # every finite non-zero code
        assert oracle.e4m3_encode(oracle.e4m3_value(c)) == c


def test_row_quantisation_scales_to_448():
    rng = np.random.default_rng(20)
    w = _bf16(rng.standard_normal((16, 256)) * 0.02)
    w[3] = 0  # an all-zero row
    q, s = oracle.quantize_rows_fp8(w)
    W = f64(w)
    assert s[3] == 1.0 and (q[3] == 0).all()
    for r in [0, 5, 15]:
        amax = np.abs(W[r]).max()
        assert s[r] == np.float32(np.float32(amax) / np.float32(448.0))
        vals = np.array([oracle.e4m3_value(c) for c in q[r]]) * s[r]
        assert np.abs(vals).max() == pytest.approx(amax, rel=1e-6)
        # within half an E4M3 step (relative 2^-4 for normals) of the original
        assert (np.abs(vals - W[r]) <= np.maximum(np.abs(W[r]) * 2.0 ** -4, 2.0 ** -10 * s[r]) + 1e-12).all()


def test_fp8_ffn_equals_bf16_ffn_on_exactly_representable_weights():
    """If every weight is an E4M3 value times a power-of-two scale, dequantisation is exact and the
    FP8-weight expert equals the bf16 expert bit for bit."""
    rng = np.random.default_rng(21)
    D, F = 32, 16
    codes = rng.integers(0, 0x7E, (2 * F + D, max(D, F))).astype(np.uint8)
    codes |= rng.integers(0, 2, codes.shape).astype(np.uint8) << 7
    codes[:, 0] = 0x7E  # every row reaches 448, so its scale is exactly the power of two below
    vals = np.vectorize(oracle.e4m3_value)(codes) * 2.0 ** -12
    gu = _bf16(vals[: 2 * F, :D])
    dn = _bf16(vals[2 * F:, :F])
    assert (f64(gu) == vals[: 2 * F, :D]).all()  # exactly representable in bf16 too
    x = _bf16(rng.standard_normal(D))
    gq, gs = oracle.quantize_rows_fp8(gu)
    dq, ds = oracle.quantize_rows_fp8(dn)
    np.testing.assert_array_equal(oracle.expert_ffn_fp8(x, gq, gs, dq, ds), oracle.expert_ffn(x, gu, dn))


def _e4m3_exact_bf16(rng, shape, exp):
    """bf16 weights that are E4M3 values times 2^exp, every row reaching 448 * 2^exp, so that the
    per-row quantiser reproduces them exactly (scale = 2^exp, codes = the drawn codes)."""
    codes = rng.integers(0, 0x7E, shape).astype(np.uint8)
    codes |= rng.integers(0, 2, shape).astype(np.uint8) << 7
    codes[..., 0] = 0x7E
    vals = np.vectorize(oracle.e4m3_value)(codes) * 2.0 ** exp
    w = _bf16(vals)
    assert (f64(w) == vals).all()
    return w


@pytest.mark.parametrize("k", [2, 3])
def test_fp8_layer_equals_bf16_layer_on_exactly_representable_weights(k):
    """The E4M3 layer (routing, FP8 experts weighted by p, shared expert at weight 1) on weights the
    quantiser reproduces exactly is the bf16 layer: a p taken from the wrong slot, a shared expert
    weighted by p, or a dropped term fails this (keryc.com, "Resultados practicos": per-expert
    quantisation leaves the layer's definition unchanged; gotburnout.io glossary "MoE", section 2)."""
    rng = np.random.default_rng(22 + k)
    T, D, E, F, Fs = 9, 32, 6, 16, 16
    gu = _e4m3_exact_bf16(rng, (E, 2 * F, D), -12)
    dn = _e4m3_exact_bf16(rng, (E, D, F), -11)
    sgu = _e4m3_exact_bf16(rng, (2 * Fs, D), -12)
    sdn = _e4m3_exact_bf16(rng, (D, Fs), -11)
    x = _bf16(rng.standard_normal((T, D)))
    wg = _bf16(rng.standard_normal((E, D)) * 0.3)
    bias = (rng.standard_normal(E) * 0.2).astype(np.float32)
    q = dict(gu_q={}, gu_s={}, dn_q={}, dn_s={})
    for e in range(E):
        q["gu_q"][e], q["gu_s"][e] = oracle.quantize_rows_fp8(gu[e])
        q["dn_q"][e], q["dn_s"][e] = oracle.quantize_rows_fp8(dn[e])
    a, b = oracle.quantize_rows_fp8(sgu)
    c, d = oracle.quantize_rows_fp8(sdn)
    shared_q = dict(gu_q=a, gu_s=b, dn_q=c, dn_s=d)
    y8, idx8, p8 = oracle.layer_fp8(x, wg, bias, k, q, shared_q)
    y, idx, p = oracle.layer(x, wg, bias, gu, dn, k, sgu, sdn)
    np.testing.assert_array_equal(idx8, idx)
    np.testing.assert_array_equal(p8, p)
    # the same terms in the same order up to the summation order of the C and numpy loops
    assert np.abs(y8 - y).max() <= 1e-13 * np.abs(y).max()
    # the weights in the p vector differ from one another, so a p from the wrong slot would show
    assert (np.abs(np.diff(p, axis=1)) > 1e-3).any()
    # and the shared expert's term is large enough that weighting it by p would show
    ys, _, _ = oracle.layer(x, wg, bias, gu, dn, k)
    assert np.abs(y - ys).max() > 1e-3 * np.abs(y).max()


# ----------------------------------------------------------------------------- backward pass
def _bwd_problem(seed=0, T=6, D=16, E=6, k=2, F=8, Fs=8, bias=True):
    """A small fp64 problem whose top-k choices are separated by at least 0.05 in score, so that the
    finite-difference steps below cannot change the selection."""
    rng = np.random.default_rng(seed)
    for _ in range(200):
        x = rng.normal(size=(T, D))
        wg = rng.normal(size=(E, D)) * 0.5
        b = (rng.normal(size=E) * 0.3).astype(np.float32) if bias else None
        s = x @ wg.T + (0.0 if b is None else b.astype(np.float64))
        top = -np.sort(-s, axis=1)[:, : min(k + 1, E)]
        if k == E or (np.diff(-top, axis=1) > 0.05).all():
            break
    gu = rng.normal(size=(E, 2 * F, D)) * 0.3
    dn = rng.normal(size=(E, D, F)) * 0.3
    sgu = rng.normal(size=(2 * Fs, D)) * 0.3 if Fs else None
    sdn = rng.normal(size=(D, Fs)) * 0.3 if Fs else None
    dy = rng.normal(size=(T, D))
    return dict(x=x, wg=wg, bias=b, gu=gu, dn=dn, sgu=sgu, sdn=sdn, dy=dy, k=k)


def _loss(P, **over):
    q = dict(P, **over)
    y = oracle.layer_f64(q["x"], q["wg"], q["bias"], q["gu"], q["dn"], q["k"], q["sgu"], q["sdn"])
    return float(np.sum(P["dy"] * y))


@pytest.mark.parametrize("k,Fs", [(2, 8), (3, 0), (1, 8)])
def test_backward_matches_finite_differences_of_the_forward(k, Fs):
    """<grad, V> equals the central difference of L = sum(dy * y) along a random V, for every
    input and parameter tensor (the fp64 forward is smooth while the selection stays fixed)."""
    P = _bwd_problem(seed=k + Fs, k=k, Fs=Fs)
    g = oracle.layer_backward(P["x"], P["wg"], P["bias"], P["gu"], P["dn"], k, P["dy"], P["sgu"], P["sdn"])
    rng = np.random.default_rng(99)
    eps = 1e-5
    pairs = [("x", "dx"), ("wg", "dw_gate"), ("gu", "dgate_up"), ("dn", "ddown")]
    if Fs:
        pairs += [("sgu", "dshared_gate_up"), ("sdn", "dshared_down")]
    for name, key in pairs:
        V = rng.normal(size=P[name].shape)
        fd = (_loss(P, **{name: P[name] + eps * V}) - _loss(P, **{name: P[name] - eps * V})) / (2 * eps)
        assert float(np.sum(g[key] * V)) == pytest.approx(fd, rel=1e-7, abs=1e-9), name


def test_backward_router_gradient_invariants():
    """The softmax over the chosen k is invariant to adding one constant to their logits, so for
    every token the logit gradients sum to zero and sum_e dW_g[e] = 0; with k = 1 the single weight
    is 1 and dW_g vanishes."""
    P = _bwd_problem(seed=3, E=8, k=3)
    g = oracle.layer_backward(P["x"], P["wg"], P["bias"], P["gu"], P["dn"], 3, P["dy"], P["sgu"], P["sdn"])
    assert np.abs(g["dw_gate"].sum(axis=0)).max() < 1e-12 * max(1.0, np.abs(g["dw_gate"]).max())
    assert np.abs(g["dw_gate"]).max() > 1e-3
    P1 = _bwd_problem(seed=4, E=8, k=1)
    g1 = oracle.layer_backward(P1["x"], P1["wg"], P1["bias"], P1["gu"], P1["dn"], 1, P1["dy"], P1["sgu"], P1["sdn"])
    assert (g1["dw_gate"] == 0).all()


def test_backward_leaves_unselected_experts_at_zero():
    """Weights of experts that no token selects get no gradient; selected ones do."""
    P = _bwd_problem(seed=5, T=3, E=12, k=2)
    g = oracle.layer_backward(P["x"], P["wg"], P["bias"], P["gu"], P["dn"], 2, P["dy"], P["sgu"], P["sdn"])
    s = P["x"] @ P["wg"].T + P["bias"].astype(np.float64)
    chosen = set(np.argsort(-s, axis=1)[:, :2].reshape(-1).tolist())
    for e in range(12):
        nz = np.abs(g["dgate_up"][e]).max() > 0 and np.abs(g["ddown"][e]).max() > 0
        assert nz == (e in chosen), e
        assert (np.abs(g["dw_gate"][e]).max() > 0) == (e in chosen), e


def test_f64_forward_is_the_bf16_forward():
    """oracle.layer_f64 on exact bf16 values is the same function as oracle.layer."""
    w = mi.Workload("t", T=9, D=64, E=8, k=2, F=32, Fs=32, bias="normal:0.5")
    h = mi.host_inputs(w)
    y16, _, _ = oracle.layer(h["x"], h["wg"], h["bias"], h["gate_up"], h["down"], 2, h["shared_gate_up"],
                             h["shared_down"])
    y64 = oracle.layer_f64(h["x"], h["wg"], h["bias"], h["gate_up"], h["down"], 2, h["shared_gate_up"],
                           h["shared_down"])
    np.testing.assert_allclose(y64, y16, rtol=1e-13, atol=1e-15)


# ----------------------------------------------------------------------------- auxiliary loss
def test_aux_loss_is_alpha_when_router_probabilities_are_uniform():
    """W_g = 0 makes every softmax uniform (P_e = 1/E), so L = alpha * E * sum_e f_e / E = alpha for
    any selection; the logit gradient is (alpha / T)(f_e - 1/E), so dW_g[e] = (alpha/T)(f_e - 1/E)
    sum_t x_t and dx = 0.  With zero logits the selection is the top-k of the bias alone."""
    rng = np.random.default_rng(11)
    T, D, E, k, alpha = 7, 12, 6, 2, 0.03
    x = rng.normal(size=(T, D))
    wg = np.zeros((E, D))
    bias = np.array([0.1, 0.5, -0.2, 0.4, 0.0, -0.3], np.float32)
    loss, dwg, dx = oracle.router_aux_loss(x, wg, bias, k, alpha)
    assert loss == pytest.approx(alpha, rel=1e-14)
    f = np.zeros(E)
    f[[1, 3]] = 1.0 / k  # the two largest biases
    np.testing.assert_allclose(dwg, np.outer(alpha / T * (f - 1.0 / E), x.sum(axis=0)), rtol=1e-12, atol=1e-15)
    assert not dx.any()


def test_aux_loss_two_expert_closed_form():
    """E = 2, k = 1, one token, D = 1 (x = [x0], W_g = [[a], [b]], a x0 > b x0): f = (1, 0) and
    P_0 = sigmoid(l_0 - l_1), so L = 2 alpha sigmoid(l_0 - l_1) and dL/dl_0 = -dL/dl_1 =
    2 alpha sig (1 - sig)."""
    alpha, x0, a, b = 0.5, 1.5, 0.8, -0.4
    loss, dwg, dx = oracle.router_aux_loss(np.array([[x0]]), np.array([[a], [b]]), None, 1, alpha)
    sig = 1.0 / (1.0 + np.exp(-(a - b) * x0))
    g = 2 * alpha * sig * (1 - sig)
    assert loss == pytest.approx(2 * alpha * sig, rel=1e-14)
    np.testing.assert_allclose(dwg[:, 0], [g * x0, -g * x0], rtol=1e-13)
    assert dx[0, 0] == pytest.approx(g * a - g * b, rel=1e-13)


def test_aux_loss_gradient_matches_finite_differences():
    """<grad, V> equals the central difference of L along a random V, for x and W_g (the fp64 loss
    is smooth while the selection stays fixed; top-k scores are 0.05 apart); and the logit gradient
    of each token sums to zero (softmax shift invariance), so sum_e dW_g[e] = 0."""
    for seed, k in ((1, 2), (2, 1), (3, 3)):
        P = _bwd_problem(seed=seed, T=5, D=10, E=6, k=k)
        loss, dwg, dx = oracle.router_aux_loss(P["x"], P["wg"], P["bias"], k, 0.1)
        rng = np.random.default_rng(seed + 50)
        eps = 1e-5
        for name, g in (("x", dx), ("wg", dwg)):
            V = rng.normal(size=P[name].shape)
            q = dict(P)
            q[name] = P[name] + eps * V
            lp = oracle.router_aux_loss(q["x"], q["wg"], P["bias"], k, 0.1)[0]
            q[name] = P[name] - eps * V
            lm = oracle.router_aux_loss(q["x"], q["wg"], P["bias"], k, 0.1)[0]
            assert float(np.sum(g * V)) == pytest.approx((lp - lm) / (2 * eps), rel=1e-6, abs=1e-11), (seed, name)
        assert np.abs(dwg.sum(axis=0)).max() < 1e-12 * max(1.0, np.abs(dwg).max())


# ----------------------------------------------------------------------------- full-size sampling helpers
def test_chunked_oracle_rows_equal_the_layer():
    """The sampled full-size check builds y from oracle expert FFNs, experts generated in chunks;
    on a small workload that must be the oracle's layer (up to summation order)."""
    from helpers import oracle_rows_chunked, segment_edge_tokens

    w = mi.Workload("chunk", T=40, D=64, E=6, k=3, F=64, Fs=64, bias="normal:0.5")
    h = mi.host_inputs(w)
    y, idx, p = oracle.layer(h["x"], h["wg"], h["bias"], h["gate_up"], h["down"], w.k, h["shared_gate_up"],
                             h["shared_down"])
    counts, offsets, pt, _, _ = oracle.permute(idx, w.E)
    rows = segment_edge_tokens(pt, offsets)
    for e in range(w.E):  # every non-empty segment's first and last token is among the rows
        if counts[e]:
            assert pt[offsets[e]] in rows and pt[offsets[e + 1] - 1] in rows
    got = oracle_rows_chunked(w, h["x"][rows], idx[rows], p[rows], chunk=4)
    assert np.abs(got - y[rows]).max() <= 1e-12 * np.abs(y).max()
