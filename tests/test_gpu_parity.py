"""Parity of the CUDA path (through the C ABI) with the fp64 oracle, on seeded inputs.

Bit-exact: top-k indices, counts, offsets, the permutation, x_perm, and the combine.  Router
weights within P_ATOL.  Layer outputs within max|err| <= 2e-2 * RMS(y_oracle).
"""
import ctypes
from dataclasses import replace

import numpy as np
import pytest

import moe_inputs as mi
import oracle
import sparse_mixture_experts_16_b200 as moe
from helpers import (GAP, P_ATOL, REL_RMS_TOL, bf16_np_to_f64, gap_redraw, gap_violations, oracle_rows_chunked,
                     rel_rms_err, scores, segment_edge_tokens, to_np_bf16, to_torch_bf16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _ready(cuda_device):
    from sparse_mixture_experts_16_b200 import build

    build.build()
    moe.lib()


def W(T, D, E, k, F, Fs=0, bias="none", seed=0):
    return mi.Workload(f"T{T}D{D}E{E}k{k}F{F}Fs{Fs}", T=T, D=D, E=E, k=k, F=F, Fs=Fs, bias=bias, seed=seed)


def host_case(w, delta=None):
    rd = gap_redraw(w) if delta is None else gap_redraw(w, delta)
    return mi.host_inputs(w, redraw=rd), rd


def device_from_host(inp):
    import torch

    out = {}
    for name, a in inp.items():
        if a is None:
            out[name] = None
        elif a.dtype == np.uint16:
            out[name] = to_torch_bf16(a)
        else:
            out[name] = torch.from_numpy(a).cuda()
    return out


def layer_from(d, k, flags=0):
    return moe.MoELayer(d["wg"], d["gate_up"], d["down"], k, bias=d["bias"], shared_gate_up=d["shared_gate_up"],
                        shared_down=d["shared_down"], flags=flags)


def oracle_layer(inp, k):
    return oracle.layer(inp["x"], inp["wg"], inp["bias"], inp["gate_up"], inp["down"], k, inp["shared_gate_up"],
                        inp["shared_down"])


# ----------------------------------------------------------------------------- generator
def test_device_generator_matches_host():
    w = W(70, 128, 5, 2, 64, Fs=64, bias="normal:0.5")
    rd = np.zeros(w.T, np.uint32)
    rd[[3, 11]] = [1, 4]
    h = mi.host_inputs(w, redraw=rd)
    d = mi.device_inputs(w, redraw=rd)
    for name in ("x", "wg", "gate_up", "down", "shared_gate_up", "shared_down"):
        assert (to_np_bf16(d[name]).reshape(h[name].shape) == h[name]).all(), name
    assert (d["bias"].cpu().numpy() == h["bias"]).all()


def test_device_generator_random_access_far_into_a_stream():
    import torch

    first = 3 * (1 << 33) + 12345  # past 2^32 elements
    t = torch.empty(4096, dtype=torch.bfloat16, device="cuda")
    mi.device_fill_bf16(t, mi.STREAM_GATE_UP, 0.02, seed=0, first=first)
    assert (to_np_bf16(t) == mi.normal_bf16(mi.STREAM_GATE_UP, 4096, 0.02, first=first)).all()


# ----------------------------------------------------------------------------- router
ROUTER_CASES = [
    W(1, 64, 1, 1, 64),
    W(7, 128, 2, 2, 64),
    W(129, 256, 8, 2, 64),
    W(300, 512, 33, 4, 64, bias="normal:0.5"),
    W(64, 1024, 256, 8, 64, bias="normal:0.5"),
    W(40, 256, 600, 16, 64, bias="zipf:1.1"),
    W(20, 128, 1024, 32, 64),
    W(33, 192, 6, 6, 64),
    W(48, 1088, 256, 8, 64, bias="normal:0.5"),           # decode T with W_g > 256 Ki: tensor-core router
]


@pytest.mark.parametrize("w", ROUTER_CASES, ids=lambda w: w.name)
def test_router_topk_parity(w):
    # with k = 32 of E = 1024 the 33 top scores are dense; at D = 128 the fp32 logit error is
    # ~1e-6, so a 2e-4 gap is still far above it
    inp, _ = host_case(w, delta=2e-4 if w.k >= 32 else None)
    d = device_from_host(inp)
    idx, wts = moe.moe_router_topk(d["x"], d["wg"], d["bias"], w.k)
    o_idx, o_p = oracle.router(inp["x"], inp["wg"], inp["bias"], w.k)
    assert (idx.cpu().numpy() == o_idx).all()
    np.testing.assert_allclose(wts.cpu().numpy(), o_p, rtol=0, atol=P_ATOL)
    assert np.abs(wts.cpu().numpy().sum(1) - 1).max() < 1e-5


# ----------------------------------------------------------------------------- dispatch
def _check_permute(idx, w_np, x_np, E, got):
    k = idx.shape[1]
    counts, offsets, pt, ps, inv = oracle.permute(idx, E)
    assert (got["counts"].cpu().numpy() == counts).all()
    assert (got["offsets"].cpu().numpy() == offsets).all()
    assert (got["perm_token"].cpu().numpy() == pt).all()
    assert (got["inv_perm"].cpu().numpy() == inv).all()
    assert (got["p_perm"].cpu().numpy() == w_np.reshape(-1)[pt * k + ps]).all()
    if x_np is not None:
        assert (to_np_bf16(got["x_perm"]) == x_np[pt]).all()


@pytest.mark.parametrize("T,E,k,D", [(1, 4, 2, 64), (255, 8, 2, 128), (256, 8, 2, 128), (1000, 33, 3, 64),
                                     (777, 256, 8, 192), (300, 1024, 4, 64), (513, 64, 32, 64),
                                     (8192, 256, 8, 64)])
def test_permute_parity_random_routing(T, E, k, D):
    import torch

    rng = np.random.default_rng(T * 7 + E)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    wts = rng.random((T, k)).astype(np.float32)
    x = mi.rows_bf16(mi.STREAM_X, np.arange(T), D, 1.0, seed=T)
    got = moe.moe_permute(torch.from_numpy(idx).cuda(), torch.from_numpy(wts).cuda(), to_torch_bf16(x), E)
    _check_permute(idx, wts, x, E, got)


def test_permute_edge_cases_empty_and_overfull_experts():
    import torch

    T, E, k, D = 700, 16, 2, 64
    idx = np.zeros((T, k), np.int32)
    idx[:, 0] = 5          # every token picks expert 5 first (700 rows: several 128-row tiles)
    idx[:, 1] = np.where(np.arange(T) % 3 == 0, 9, 12)  # experts 9 and 12 only; the rest stay empty
    wts = np.full((T, k), 0.5, np.float32)
    x = mi.rows_bf16(mi.STREAM_X, np.arange(T), D, 1.0)
    got = moe.moe_permute(torch.from_numpy(idx).cuda(), torch.from_numpy(wts).cuda(), to_torch_bf16(x), E)
    _check_permute(idx, wts, x, E, got)
    # metadata only (x = None)
    got2 = moe.moe_permute(torch.from_numpy(idx).cuda(), torch.from_numpy(wts).cuda(), None, E)
    assert (got2["perm_token"].cpu().numpy() == got["perm_token"].cpu().numpy()).all()


def test_multi_block_permute_drops_out_of_range_ids_and_keeps_the_rest_in_order():
    """Above 256 tokens the dispatch runs as histogram, scan and scatter kernels.  Slots whose
    expert id is outside [0, E) get inv_perm -1 and no row; every other slot keeps the order the
    oracle gives it, counted over the valid slots only."""
    import torch

    T, E, k = 600, 12, 3
    rng = np.random.default_rng(5)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    bad = rng.random((T, k)) < 0.05
    idx_bad = np.where(bad, np.where(rng.random((T, k)) < 0.5, -1, E + 3), idx).astype(np.int32)
    wts = rng.random((T, k)).astype(np.float32)
    got = moe.moe_permute(torch.from_numpy(idx_bad).cuda(), torch.from_numpy(wts).cuda(), None, E)
    assert moe.moe_get_device_error(got["ws"]) == 6  # MOE_ERR_DEVICE_INDEX
    inv = got["inv_perm"].cpu().numpy().reshape(T, k)
    assert (inv[bad] == -1).all()
    # the valid slots in (token, slot) order, stably sorted by expert, are the permutation
    slots = np.flatnonzero(~bad.reshape(-1))
    e_valid = idx.reshape(-1)[slots]
    order = slots[np.argsort(e_valid, kind="stable")]
    counts = np.bincount(e_valid, minlength=E)
    assert (got["counts"].cpu().numpy() == counts).all()
    assert (got["offsets"].cpu().numpy() == np.concatenate([[0], np.cumsum(counts)])).all()
    n = len(order)
    assert (got["perm_token"].cpu().numpy()[:n] == order // k).all()
    assert (inv.reshape(-1)[order] == np.arange(n)).all()
    assert (got["p_perm"].cpu().numpy()[:n] == wts.reshape(-1)[order]).all()


def test_permute_reports_out_of_range_ids_without_faulting():
    import torch

    idx = np.array([[0, 1], [2, 7], [1, -3]], np.int32)  # 7 and -3 are outside [0, 4)
    wts = np.ones((3, 2), np.float32)
    x = mi.rows_bf16(mi.STREAM_X, np.arange(3), 64, 1.0)
    got = moe.moe_permute(torch.from_numpy(idx).cuda(), torch.from_numpy(wts).cuda(), to_torch_bf16(x), 4)
    assert moe.moe_get_device_error(got["ws"]) == 6  # MOE_ERR_DEVICE_INDEX
    assert moe.moe_get_device_error(got["ws"]) == 0  # cleared
    assert got["offsets"].cpu().numpy()[-1] == 4
    inv = got["inv_perm"].cpu().numpy()
    assert inv[3] == -1 and inv[5] == -1


# ----------------------------------------------------------------------------- combine
@pytest.mark.parametrize("T,k,D,shared", [(1, 1, 64, False), (100, 2, 192, True), (513, 8, 128, True)])
def test_combine_bit_exact(T, k, D, shared):
    import torch

    rng = np.random.default_rng(T + k)
    M = T * k
    outp = rng.standard_normal((M, D)).astype(np.float32)
    inv = rng.permutation(M).astype(np.int32)
    sh = rng.standard_normal((T, D)).astype(np.float32) if shared else None
    y = moe.moe_combine(torch.from_numpy(outp).cuda(), torch.from_numpy(inv).cuda(),
                        torch.from_numpy(sh).cuda() if shared else None, T, k)
    # definition: fp32 sum over j = 0..k-1 in order, then the shared row, rounded to bf16
    acc = np.zeros((T, D), np.float32)
    for j in range(k):
        acc += outp[inv.reshape(T, k)[:, j]]
    if shared:
        acc += sh
    u = acc.view(np.uint32).astype(np.uint64)
    ref = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    assert (to_np_bf16(y) == ref).all()


# ----------------------------------------------------------------------------- grouped FFN
@pytest.mark.parametrize("max_seg_mode", ["tiled", "stream"])
def test_grouped_ffn_rows_match_oracle_expert_ffn(max_seg_mode):
    import torch

    T, D, E, k, F = (150, 192, 6, 2, 320) if max_seg_mode == "tiled" else (40, 192, 6, 2, 320)
    w = W(T, D, E, k, F, bias="normal:0.5")
    inp, _ = host_case(w)
    idx, p = oracle.router(inp["x"], inp["wg"], inp["bias"], k)
    counts, offsets, pt, ps, inv = oracle.permute(idx, E)
    xp = inp["x"][pt]
    scale = p.reshape(-1)[pt * k + ps].astype(np.float32)
    out, _ = moe.moe_grouped_swiglu_ffn(to_torch_bf16(xp), torch.from_numpy(offsets).cuda(),
                                        torch.from_numpy(scale).cuda(), to_torch_bf16(inp["gate_up"]),
                                        to_torch_bf16(inp["down"]),
                                        max_seg=int(counts.max()) if max_seg_mode == "stream" else None)
    got = out.cpu().numpy().astype(np.float64)
    ref = np.stack([scale[r] * oracle.expert_ffn(xp[r], inp["gate_up"][e], inp["down"][e])
                    for e in range(E) for r in range(offsets[e], offsets[e + 1])])
    assert rel_rms_err(got, ref) <= REL_RMS_TOL


# ----------------------------------------------------------------------------- whole layer
LAYER_CASES = [
    W(256, 256, 8, 2, 512),                                # tiny workload
    W(300, 192, 5, 2, 320),                                # ragged rows and columns
    W(77, 256, 16, 4, 192, Fs=128, bias="normal:0.5"),     # shared expert + bias, prefill path
    W(64, 512, 32, 4, 384, Fs=256, bias="zipf:1.1"),       # largest decode T
    W(33, 256, 8, 8, 128, Fs=64),                          # k = E
    W(1, 128, 4, 2, 64),                                   # a single token
    W(129, 128, 1, 1, 128),                                # one expert, two row tiles
]


@pytest.mark.parametrize("w", LAYER_CASES, ids=lambda w: w.name)
def test_layer_parity(w):
    inp, _ = host_case(w)
    d = device_from_host(inp)
    y_ref, _, _ = oracle_layer(inp, w.k)
    y = bf16_np_to_f64(to_np_bf16(layer_from(d, w.k)(d["x"])))
    assert rel_rms_err(y, y_ref) <= REL_RMS_TOL
    if w.T <= 64:  # the other path on the same inputs
        y2 = bf16_np_to_f64(to_np_bf16(layer_from(d, w.k, moe.MOE_FLAG_FORCE_PREFILL)(d["x"])))
        assert rel_rms_err(y2, y_ref) <= REL_RMS_TOL


def test_layer_all_tokens_to_one_expert_and_empty_experts():
    """A huge bias on expert 3 sends every token there (many 128-row tiles); with k=2 the second
    choice spreads over the rest, and with E=64, T=40 most experts stay empty."""
    w = W(40, 256, 64, 2, 192)
    inp = mi.host_inputs(w)
    inp["bias"] = np.zeros(64, np.float32)
    inp["bias"][3] = 1000.0
    d = device_from_host(inp)
    y_ref, idx, _ = oracle_layer(inp, w.k)
    assert (idx[:, 0] == 3).all()
    s = scores(w, inp["x"], inp["wg"], inp["bias"])
    if gap_violations(s, w.k).any():
        pytest.skip("seeded inputs violate the gap")
    for flags in (0, moe.MOE_FLAG_FORCE_PREFILL):
        y = bf16_np_to_f64(to_np_bf16(layer_from(d, w.k, flags)(d["x"])))
        assert rel_rms_err(y, y_ref) <= REL_RMS_TOL


def test_layer_is_deterministic_and_reports_no_device_error():
    w = W(200, 256, 8, 2, 256, Fs=128)
    inp, _ = host_case(w)
    d = device_from_host(inp)
    L = layer_from(d, w.k)
    y1 = to_np_bf16(L(d["x"]))
    y2 = to_np_bf16(L(d["x"]))
    assert (y1 == y2).all()
    assert L.device_error() == 0


def test_decode_path_is_deterministic_and_matches_oracle():
    """Two tokens on 16 experts: the weight-streaming (decode) GEMMs; repeated forwards are
    bit-identical and match the oracle."""
    w = W(2, 512, 16, 2, 1024, Fs=256, bias="normal:0.5")
    inp, _ = host_case(w)
    d = device_from_host(inp)
    y_ref, _, _ = oracle_layer(inp, w.k)
    L = layer_from(d, w.k)
    ys = [to_np_bf16(L(d["x"])) for _ in range(3)]
    assert all((y == ys[0]).all() for y in ys[1:])
    assert rel_rms_err(bf16_np_to_f64(ys[0]), y_ref) <= REL_RMS_TOL
    assert L.device_error() == 0


DECODE_STEP_CASES = [
    W(16, 256, 32, 4, 384, bias="normal:0.5"),
    W(1, 256, 32, 4, 384, bias="zipf:1.1"),
    W(2, 2880, 32, 4, 128, bias="zipf:1.1"),  # the gpt-oss-shaped router
    W(64, 256, 64, 8, 128, Fs=128, bias="normal:0.5"),
    W(3, 128, 256, 8, 64, Fs=64, bias="normal:0.5"),
]


@pytest.mark.parametrize("w", DECODE_STEP_CASES + [W(16, 128, 1024, 32, 64)], ids=lambda w: w.name)
def test_decode_layer_equals_the_step_by_step_path_bit_for_bit(w):
    """The decode layer forward and the step-by-step entry points (router, permute, grouped FFN
    with the same token tile, combine) are the same computation and must give the same bits; the
    layer's routing and counts equal the oracle's."""
    import torch

    # E = 1024, k = 32, T = 16: D = 128 logits are accurate to ~1e-6 in fp32, so a 2e-4 score gap
    # keeps the selection exact
    inp, _ = host_case(w, delta=2e-4 if w.E > 256 else None)
    d = device_from_host(inp)
    L = layer_from(d, w.k)
    assert L.kernel_count(w.T) == 6
    y_layer = to_np_bf16(L(d["x"]))
    assert L.device_error() == 0
    o_idx, _ = oracle.router(inp["x"], inp["wg"], inp["bias"], w.k)
    counts, _, _, _, _ = oracle.permute(o_idx, w.E)
    assert (L.expert_counts(w.T).cpu().numpy() == counts).all()
    idx, p = moe.moe_router_topk(d["x"], d["wg"], d["bias"], w.k)
    assert (idx.cpu().numpy() == o_idx).all()
    pm = moe.moe_permute(idx, p, d["x"], w.E)
    out_perm, _ = moe.moe_grouped_swiglu_ffn(pm["x_perm"], pm["offsets"], pm["p_perm"], d["gate_up"], d["down"],
                                             max_seg=w.T)
    shared = None
    if w.Fs:
        off = torch.tensor([0, w.T], dtype=torch.int32, device="cuda")
        shared, _ = moe.moe_grouped_swiglu_ffn(d["x"], off, None, d["shared_gate_up"][None], d["shared_down"][None],
                                               max_seg=w.T)
    y_steps = to_np_bf16(moe.moe_combine(out_perm, pm["inv_perm"], shared, w.T, w.k))
    assert (y_layer == y_steps).all()
    y_ref, _, _ = oracle_layer(inp, w.k)
    assert rel_rms_err(bf16_np_to_f64(y_layer), y_ref) <= REL_RMS_TOL


PREFILL_STEP_CASES = [
    W(300, 256, 8, 2, 128, bias="zipf:1.1"),               # ragged last tiles, one segment > 128 rows
    W(520, 512, 32, 4, 256, Fs=128, bias="normal:0.5"),    # with the shared expert (side stream)
    W(257, 128, 64, 8, 64, bias="zipf:1.1"),               # empty experts, multi-block dispatch
]


@pytest.mark.parametrize("w", PREFILL_STEP_CASES, ids=lambda w: w.name)
def test_prefill_layer_equals_the_step_by_step_path_bit_for_bit(w):
    """The prefill layer forward (the shared expert on its side stream) and the step-by-step entry
    points (router, permute, grouped FFN on x_perm with the same default tiling, the shared expert
    as a one-segment grouped FFN, combine) are the same computation and must give the same bits."""
    import torch

    inp, _ = host_case(w)
    d = device_from_host(inp)
    L = layer_from(d, w.k)
    assert L.kernel_count(w.T) == 2 + 4 + (4 if w.Fs else 2) + 1  # hist, scan, scatter, gather
    y_layer = to_np_bf16(L(d["x"]))
    assert L.device_error() == 0
    idx, p = moe.moe_router_topk(d["x"], d["wg"], d["bias"], w.k)
    pm = moe.moe_permute(idx, p, d["x"], w.E)
    out_perm, _ = moe.moe_grouped_swiglu_ffn(pm["x_perm"], pm["offsets"], pm["p_perm"], d["gate_up"], d["down"])
    shared = None
    if w.Fs:
        off = torch.tensor([0, w.T], dtype=torch.int32, device="cuda")
        shared, _ = moe.moe_grouped_swiglu_ffn(d["x"], off, None, d["shared_gate_up"][None], d["shared_down"][None])
    y_steps = to_np_bf16(moe.moe_combine(out_perm, pm["inv_perm"], shared, w.T, w.k))
    assert (y_layer == y_steps).all()
    y_ref, _, _ = oracle_layer(inp, w.k)
    assert rel_rms_err(bf16_np_to_f64(y_layer), y_ref) <= REL_RMS_TOL


def test_layer_host_buffers_match_device_buffers():
    import torch

    w = W(96, 256, 8, 2, 256)
    inp, _ = host_case(w)
    d = device_from_host(inp)
    L = layer_from(d, w.k)
    y_dev = to_np_bf16(L(d["x"]))
    xh = d["x"].cpu().pin_memory()
    yh = torch.empty_like(xh).pin_memory()
    L.forward_host(xh, yh)
    torch.cuda.current_stream().synchronize()
    assert (yh.view(torch.int16).numpy().view(np.uint16) == y_dev).all()


def test_overlapping_host_forwards_on_two_streams_give_the_same_bits():
    """Double-buffered use of the public API: forwards alternate between two streams, each with
    its own workspace and output buffer, so they overlap on the GPU (copies against compute, and
    compute against compute).  The library keeps no state shared between them: every output
    equals the single-stream forward bit for bit, including the shared expert's side streams."""
    import torch

    w = W(700, 256, 16, 4, 256, Fs=128, bias="normal:0.5")
    inp, _ = host_case(w)
    d = device_from_host(inp)
    L = layer_from(d, w.k)
    y_ref = to_np_bf16(L(d["x"]))
    xh = d["x"].cpu().pin_memory()
    streams = (torch.cuda.Stream(), torch.cuda.Stream())
    wss = (L.new_workspace(w.T), L.new_workspace(w.T))
    outs = [torch.empty_like(xh).pin_memory() for _ in range(6)]
    for i, yh in enumerate(outs):
        L.forward_host(xh, yh, stream=streams[i % 2], ws=wss[i % 2])
    torch.cuda.synchronize()
    for yh in outs:
        assert (yh.view(torch.int16).numpy().view(np.uint16) == y_ref).all()
    for ws in wss:
        assert moe.moe_get_device_error(ws) == 0


def test_layer_timed_records_six_events():
    import torch

    w = W(128, 256, 8, 2, 256)
    inp, _ = host_case(w)
    d = device_from_host(inp)
    L = layer_from(d, w.k)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    for e in evs:
        e.record()
    y = torch.empty_like(d["x"])
    L.forward_timed(d["x"], y, evs)
    torch.cuda.synchronize()
    times = [evs[i].elapsed_time(evs[i + 1]) for i in range(5)]
    assert all(t >= 0 for t in times)
    assert (to_np_bf16(y) == to_np_bf16(L(d["x"]))).all()


# ----------------------------------------------------------------------------- full-size workloads
FULL = ["mixtral", "gptoss", "gptoss_decode_T1", "gptoss_decode_T8", "gptoss_decode_T32", "gptoss_decode_T64",
        "deepseek", "deepseek_decode"]


# the prefill tilings other than the default mix, at full size
OTHER_TILING = [("mixtral", moe.MOE_FLAG_PREFILL_ROW_TILES), ("gptoss", moe.MOE_FLAG_PREFILL_WIDE_TILES),
                ("deepseek", moe.MOE_FLAG_PREFILL_ROW_TILES), ("deepseek", moe.MOE_FLAG_PREFILL_WIDE_TILES),
                ("mixtral", moe.MOE_FLAG_PREFILL_PAIR_TILES), ("gptoss", moe.MOE_FLAG_PREFILL_PAIR_TILES),
                ("deepseek", moe.MOE_FLAG_PREFILL_PAIR_TILES)]
_TILING_ID = {moe.MOE_FLAG_PREFILL_ROW_TILES: "row", moe.MOE_FLAG_PREFILL_WIDE_TILES: "wide",
              moe.MOE_FLAG_PREFILL_PAIR_TILES: "pair"}


@pytest.mark.slow
@pytest.mark.parametrize("name,flags", [(n, 0) for n in FULL] + OTHER_TILING,
                         ids=[n for n in FULL] + [f"{n}-{_TILING_ID[f]}" for n, f in OTHER_TILING])
def test_full_size_workload_parity(name, flags):
    """Routing of every token and the whole dispatch (counts, offsets, perm_token, inv_perm)
    bit-exact against the oracle; layer outputs within tolerance on every token that holds the
    first or the last row of an expert segment (so every segment's ragged last tile is checked).
    With flags = 0 the layer is launched exactly as the benchmark launches it."""
    import torch

    w = mi.WORKLOADS[name]
    rd = gap_redraw(w)
    d = mi.device_inputs(w, redraw=rd)
    L = moe.MoELayer(d["wg"], d["gate_up"], d["down"], w.k, bias=d["bias"], shared_gate_up=d["shared_gate_up"],
                     shared_down=d["shared_down"], flags=flags)
    y = L(d["x"])
    idx, topk_w = moe.moe_router_topk(d["x"], d["wg"], d["bias"], w.k)
    disp = moe.moe_permute(idx, topk_w, None, w.E)
    torch.cuda.synchronize()
    assert L.device_error() == 0
    x_h = mi.host_x(w, redraw=rd)
    wg_h = mi.host_wg(w)
    bias_h = mi.bias_f32(w)
    o_idx, o_p = oracle.router(x_h, wg_h, bias_h, w.k)
    assert (idx.cpu().numpy() == o_idx).all()
    assert np.abs(topk_w.cpu().numpy() - o_p).max() <= P_ATOL
    counts, offsets, pt, ps, inv = oracle.permute(o_idx, w.E)
    assert (disp["counts"].cpu().numpy() == counts).all()
    assert (disp["offsets"].cpu().numpy() == offsets).all()
    assert (disp["perm_token"].cpu().numpy() == pt).all()
    assert (disp["inv_perm"].cpu().numpy() == inv).all()
    rows = segment_edge_tokens(pt, offsets)
    y_ref = oracle_rows_chunked(w, x_h[rows], o_idx[rows], o_p[rows])
    got = bf16_np_to_f64(to_np_bf16(y[torch.from_numpy(rows).cuda()]))
    assert rel_rms_err(got, y_ref) <= REL_RMS_TOL
