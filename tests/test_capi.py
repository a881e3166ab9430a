"""The C-ABI library on the host (no GPU needed): it loads, exports every symbol the header
declares, and rejects bad arguments before touching the device.  The pointers here are made up,
so no call in this file may pass validation and launch when a GPU is present."""
import ctypes
import os
import re
import subprocess

import pytest

import sparse_mixture_experts_16_b200 as moe
from sparse_mixture_experts_16_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_b200.h")


@pytest.fixture(scope="module")
def L():
    moe_build.build()
    return moe.lib()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert sorted(_declared()) == sorted(moe.EXPORTS)


def test_library_exports_every_declared_symbol(L):
    out = subprocess.run(["nm", "-D", "--defined-only", moe.LIB_PATH], capture_output=True, text=True, check=True)
    exported = set(re.findall(r"\bT (moe_\w+)", out.stdout))
    missing = [s for s in _declared() if s not in exported]
    assert not missing, missing
    for s in _declared():
        assert getattr(L, s) is not None


def test_status_strings(L):
    for code, name in moe.STATUS.items():
        assert moe.moe_status_string(code) == name
    assert moe.moe_status_string(99) == "MOE_ERR_UNKNOWN"


def _desc(**kw):
    base = dict(T=16, D=128, E=8, k=2, F=128, Fs=0, w_gate=0x1000, bias=None, gate_up=0x2000, down=0x3000,
                shared_gate_up=None, shared_down=None, flags=0, weight_format=0, gate_up_fp8=None,
                gate_up_scale=None, down_fp8=None, down_scale=None, shared_gate_up_fp8=None,
                shared_gate_up_scale=None, shared_down_fp8=None, shared_down_scale=None)
    base.update(kw)
    return moe.LayerDesc(*[base[n] for n, _ in moe.LayerDesc._fields_])


@pytest.mark.parametrize("kw,status", [
    (dict(k=9), 1),               # k > E
    (dict(k=0), 1),
    (dict(T=-1), 1),
    (dict(D=96), 2),              # not a multiple of 64
    (dict(F=100), 2),
    (dict(E=1025, k=2), 2),
    (dict(E=64, k=33), 2),        # k > 32
    (dict(Fs=64), 1),             # shared size without shared weights
    (dict(w_gate=None), 1),
    (dict(w_gate=0x1008), 3),     # misaligned
    (dict(flags=3), 1),           # both force flags
    (dict(flags=2, T=65), 1),     # decode forced above the decode range
    (dict(flags=8 | 16), 1),      # both prefill tilings
    (dict(flags=2 | 16), 1),      # a prefill tiling with decode forced
    (dict(flags=16 | 32), 1),     # token-wide and pair tiles
    (dict(flags=2 | 32), 1),      # pair tiles with decode forced
    (dict(flags=64), 1),          # unknown flag
])
def test_layer_forward_rejects_bad_descriptors(L, kw, status):
    d = _desc(**kw)
    assert L.moe_layer_workspace_size(ctypes.byref(d)) == 0
    st = L.moe_layer_forward(ctypes.byref(d), 0x4000, 0x5000, 0x100000, 1 << 30, None)
    assert st == status, moe.STATUS.get(st)


def test_layer_workspace_size_and_small_workspace(L):
    d = _desc()
    need = L.moe_layer_workspace_size(ctypes.byref(d))
    assert need > 256 and need % 256 == 0
    assert L.moe_layer_forward(ctypes.byref(d), 0x4000, 0x5000, 0x100000, need - 1, None) == 4
    assert L.moe_layer_forward(ctypes.byref(d), 0x4000, 0x5000, 0x100010, need, None) == 3  # ws not 256-aligned
    assert L.moe_layer_forward(ctypes.byref(d), 0x4008, 0x5000, 0x100000, need, None) == 3
    # T=16: router GEMM, top-k, one kernel that sorts and gathers, 2 GEMMs, combine
    assert L.moe_layer_kernel_count(ctypes.byref(d)) == 6
    assert L.moe_layer_kernel_count(ctypes.byref(_desc(flags=1))) == 6  # forced prefill
    # prefill with a shared expert: its own gate_up and down on the side stream
    sh = dict(Fs=64, shared_gate_up=0x6000, shared_down=0x7000)
    assert L.moe_layer_kernel_count(ctypes.byref(_desc(T=300, **sh))) == 11
    assert L.moe_layer_kernel_count(ctypes.byref(_desc(T=16, **sh))) == 6  # decode: one launch for both sets
    # T=300 prefill: router GEMM, top-k, hist, scan, scatter, gather, 2 GEMMs, combine
    assert L.moe_layer_kernel_count(ctypes.byref(_desc(T=300))) == 9
    assert L.moe_layer_kernel_count(ctypes.byref(_desc(k=9))) == 0
    # shared expert grows the workspace
    d2 = _desc(Fs=256, shared_gate_up=0x6000, shared_down=0x7000)
    assert L.moe_layer_workspace_size(ctypes.byref(d2)) > need


def test_step_entry_points_validate_on_host(L):
    # router: k > E, D not multiple of 64, misaligned x
    rws = L.moe_router_topk_workspace_size(4, 128, 4)
    assert rws >= 256 + 4 * 32 * 4
    assert L.moe_router_topk(0x1000, 0x2000, None, 4, 128, 4, 5, 0x3000, 0x4000, 0x100000, rws, None) == 1
    assert L.moe_router_topk(0x1000, 0x2000, None, 4, 100, 4, 2, 0x3000, 0x4000, 0x100000, rws, None) == 2
    assert L.moe_router_topk(0x1001, 0x2000, None, 4, 128, 4, 2, 0x3000, 0x4000, 0x100000, rws, None) == 3
    assert L.moe_router_topk(None, 0x2000, None, 4, 128, 4, 2, 0x3000, 0x4000, 0x100000, rws, None) == 1
    assert L.moe_router_topk(0x1000, 0x2000, None, 4, 128, 4, 2, 0x3000, 0x4000, 0x100000, rws - 1, None) == 4
    # permute: workspace too small, x without x_perm
    need = L.moe_permute_workspace_size(300, 8, 2)
    assert need >= 256 + 2 * 8 * 4
    args = [0x1000, 0x2000, 0x3000, 300, 128, 8, 2, 0x4000, 0x5000, 0x6000, 0x7000, 0x8000, 0x9000]
    assert L.moe_permute(*args, 0x100000, need - 1, None) == 4
    args_bad = list(args)
    args_bad[-1] = None  # x given, x_perm missing
    assert L.moe_permute(*args_bad, 0x100000, need, None) == 1
    # grouped ffn: max_seg > M, F not multiple of 64, two tiling flags, an unknown flag
    assert L.moe_grouped_swiglu_ffn(0x1000, 0x2000, None, 10, 11, 0, 4, 128, 128, 0x3000, 0x4000, 0x5000, 0x100000,
                                    1 << 20, None) == 1
    assert L.moe_grouped_swiglu_ffn(0x1000, 0x2000, None, 10, 10, 0, 4, 128, 100, 0x3000, 0x4000, 0x5000, 0x100000,
                                    1 << 20, None) == 2
    assert L.moe_grouped_swiglu_ffn(0x1000, 0x2000, None, 10, 10, 8 | 32, 4, 128, 128, 0x3000, 0x4000, 0x5000,
                                    0x100000, 1 << 20, None) == 1
    assert L.moe_grouped_swiglu_ffn(0x1000, 0x2000, None, 10, 10, 2, 4, 128, 128, 0x3000, 0x4000, 0x5000,
                                    0x100000, 1 << 20, None) == 1
    assert L.moe_grouped_swiglu_ffn_workspace_size(10, 128) == 256 + 2560 + (256 - 2560 % 256) % 256
    # combine: k > 32, misaligned y
    assert L.moe_combine(0x1000, 0x2000, None, 4, 128, 33, 0x3000, None) == 2
    assert L.moe_combine(0x1000, 0x2000, None, 4, 128, 2, 0x3004, None) == 3
    # timed forward needs 6 events
    d = _desc()
    assert L.moe_layer_forward_timed(ctypes.byref(d), 0x4000, 0x5000, 0x100000, 1 << 30, None, None, 0) == 1


def test_valid_call_without_a_gpu_reports_no_device(L):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    d = _desc()
    need = L.moe_layer_workspace_size(ctypes.byref(d))
    assert L.moe_layer_forward(ctypes.byref(d), 0x4000, 0x5000, 0x100000, need, None) == 8
    assert L.moe_get_device_error(0x100000, None) == 8


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(moe, "_lib", None)
    monkeypatch.setattr(moe, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(ImportError):
        moe.lib()


def test_bias_update_and_counts_validate_on_host(L):
    assert L.moe_update_router_bias(None, 8, 0.01, 0x2000, None) == 1
    assert L.moe_update_router_bias(0x1000, 0, 0.01, 0x2000, None) == 1
    assert L.moe_update_router_bias(0x1000, 1025, 0.01, 0x2000, None) == 2
    assert L.moe_update_router_bias(0x1000, 8, -1.0, 0x2000, None) == 1
    assert L.moe_update_router_bias(0x1000, 8, float("nan"), 0x2000, None) == 1
    assert L.moe_update_router_bias(0x1002, 8, 0.01, 0x2000, None) == 3
    d = _desc()
    need = L.moe_layer_workspace_size(ctypes.byref(d))
    ptr = ctypes.c_void_p()
    assert L.moe_layer_expert_counts(ctypes.byref(d), 0x100000, need, ctypes.byref(ptr)) == 0
    assert 0x100000 < ptr.value < 0x100000 + need and ptr.value % 256 == 0
    assert L.moe_layer_expert_counts(ctypes.byref(d), 0x100000, need - 1, ctypes.byref(ptr)) == 4


FP8 = dict(weight_format=1, gate_up=None, down=None, gate_up_fp8=0x8000, gate_up_scale=0x9000, down_fp8=0xA000,
           down_scale=0xB000)


@pytest.mark.parametrize("kw,status", [
    (dict(), 0),                                   # valid (reaches the device check or the no-GPU status)
    (dict(weight_format=2), 1),
    (dict(gate_up_scale=None), 1),
    (dict(T=65), 2),                               # FP8 weights run the decode kernels only
    (dict(flags=1), 1),                            # ... so forcing the tiled kernels is invalid
    (dict(Fs=64, shared_gate_up_fp8=0xC000, shared_down_fp8=0xD000, shared_gate_up_scale=0xE000), 1),
    (dict(gate_up_fp8=0x8008), 3),
    (dict(down_scale=0xB002), 3),
])
def test_fp8_descriptor_validation(L, kw, status):
    import torch

    d = _desc(**{**FP8, **kw})
    if status == 0:
        assert L.moe_layer_workspace_size(ctypes.byref(d)) > 0
        if torch.cuda.is_available():
            return  # a valid descriptor would launch kernels on the made-up pointers: host checks only
        assert L.moe_layer_forward(ctypes.byref(d), 0x4000, 0x5000, 0x100000, 1 << 30, None) == 8
    else:
        st = L.moe_layer_forward(ctypes.byref(d), 0x4000, 0x5000, 0x100000, 1 << 30, None)
        assert st == status, moe.STATUS.get(st)


def test_fp8_kernel_count_and_quantizer_validation(L):
    d = _desc(**FP8, Fs=64, shared_gate_up_fp8=0xC000, shared_down_fp8=0xD000, shared_gate_up_scale=0xE000,
              shared_down_scale=0xF000)
    assert L.moe_layer_kernel_count(ctypes.byref(d)) == 6  # the f16 gather and cast of x ride in dispatch
    assert L.moe_quantize_rows_fp8(None, 4, 64, 0x2000, 0x3000, None) == 1
    assert L.moe_quantize_rows_fp8(0x1000, 4, 100, 0x2000, 0x3000, None) == 2
    assert L.moe_quantize_rows_fp8(0x1008, 4, 64, 0x2000, 0x3000, None) == 3


def test_backward_entry_validates_on_host(L):
    """The backward needs a training descriptor (MOE_FLAG_SAVE_FOR_BACKWARD, bf16 weights), aligned
    pointers, shared-expert gradients exactly when Fs > 0, and big enough workspaces; all checked
    before any launch."""
    SAVE = moe.MOE_FLAG_SAVE_FOR_BACKWARD
    plain = _desc()
    assert L.moe_layer_backward_workspace_size(ctypes.byref(plain)) == 0  # not a training descriptor
    d = _desc(flags=SAVE)
    need_b = L.moe_layer_backward_workspace_size(ctypes.byref(d))
    need_f = L.moe_layer_workspace_size(ctypes.byref(d))
    assert need_b > 256 and need_b % 256 == 0
    # the training forward keeps g | u: its workspace grows by T*k*2F bf16 over a (prefill) forward
    prefill = _desc(flags=moe.MOE_FLAG_FORCE_PREFILL)
    assert need_f >= L.moe_layer_workspace_size(ctypes.byref(prefill)) + 16 * 2 * 2 * 128 * 2
    assert L.moe_layer_kernel_count(ctypes.byref(d)) == 6  # tiled kernels at T = 16, separate combine
    g = moe.LayerGrads(0x10000, 0x20000, 0x30000, None, None)
    args = (0x4000, 0x5000, 0x6000, ctypes.byref(g), 0x100000, need_f, 0x200000, need_b, None)
    assert L.moe_layer_backward(ctypes.byref(plain), *args) == 1
    assert L.moe_layer_backward(ctypes.byref(d), 0x4000, 0x5000, 0x6000, ctypes.byref(g), 0x100000, need_f - 1,
                                0x200000, need_b, None) == 4
    assert L.moe_layer_backward(ctypes.byref(d), 0x4000, 0x5000, 0x6000, ctypes.byref(g), 0x100000, need_f,
                                0x200000, need_b - 1, None) == 4
    assert L.moe_layer_backward(ctypes.byref(d), 0x4008, 0x5000, 0x6000, ctypes.byref(g), 0x100000, need_f,
                                0x200000, need_b, None) == 3
    gs = moe.LayerGrads(0x10000, 0x20000, 0x30000, 0x40000, None)  # shared gradient without a shared expert
    assert L.moe_layer_backward(ctypes.byref(d), 0x4000, 0x5000, 0x6000, ctypes.byref(gs), 0x100000, need_f,
                                0x200000, need_b, None) == 1
    assert L.moe_layer_backward(ctypes.byref(d), 0x4000, 0x5000, 0x6000, None, 0x100000, need_f, 0x200000,
                                need_b, None) == 1
    # FP8 weights cannot be trained here; decode forcing conflicts with saving
    assert L.moe_layer_workspace_size(ctypes.byref(_desc(**FP8, flags=SAVE))) == 0
    assert L.moe_layer_workspace_size(ctypes.byref(_desc(flags=SAVE | moe.MOE_FLAG_FORCE_DECODE))) == 0


def test_gemm_path_query(L):
    """The host-only path query follows the flags and the default rule: T <= 64 streams the weights;
    larger T runs gate_up on 128-row tiles and down on token-wide tiles of CTA pairs unless one tiling is asked
    for; E4M3 weights always stream."""
    P = lambda **kw: L.moe_layer_gemm_path(ctypes.byref(_desc(**kw)))
    assert P() == moe.MOE_PATH_STREAMING                                     # T = 16
    assert P(T=16, flags=moe.MOE_FLAG_FORCE_PREFILL) == moe.MOE_PATH_MIXED_TILES
    assert P(T=16, flags=moe.MOE_FLAG_FORCE_PREFILL | moe.MOE_FLAG_PREFILL_WIDE_TILES) == moe.MOE_PATH_WIDE_TILES
    assert P(T=16, flags=moe.MOE_FLAG_FORCE_PREFILL | moe.MOE_FLAG_PREFILL_ROW_TILES) == moe.MOE_PATH_ROW_TILES
    assert P(T=65) == moe.MOE_PATH_MIXED_TILES
    assert P(T=4096, E=8, k=2, flags=moe.MOE_FLAG_PREFILL_ROW_TILES) == moe.MOE_PATH_ROW_TILES
    assert P(T=4096, E=8, k=2, flags=moe.MOE_FLAG_PREFILL_WIDE_TILES) == moe.MOE_PATH_WIDE_TILES
    assert P(T=4096, E=8, k=2, flags=moe.MOE_FLAG_PREFILL_PAIR_TILES) == moe.MOE_PATH_PAIR_TILES
    assert P(T=16, flags=moe.MOE_FLAG_PREFILL_WIDE_TILES) == moe.MOE_PATH_STREAMING  # tiling flags leave decode
    assert P(T=300, E=8, k=2, flags=moe.MOE_FLAG_PREFILL_ROW_TILES) == moe.MOE_PATH_ROW_TILES
    assert P(**FP8) == moe.MOE_PATH_FP8_STREAMING
    assert P(**FP8, flags=moe.MOE_FLAG_PREFILL_WIDE_TILES) == -1             # E4M3 has no prefill path
    assert P(k=9) == -1
    # the training forward runs a prefill tiling at any T
    assert P(flags=moe.MOE_FLAG_SAVE_FOR_BACKWARD) == moe.MOE_PATH_MIXED_TILES
    assert P(flags=moe.MOE_FLAG_SAVE_FOR_BACKWARD | moe.MOE_FLAG_PREFILL_ROW_TILES) == moe.MOE_PATH_ROW_TILES
    assert P(flags=moe.MOE_FLAG_SAVE_FOR_BACKWARD | moe.MOE_FLAG_PREFILL_WIDE_TILES) == moe.MOE_PATH_WIDE_TILES


def test_aux_loss_entry_validates_on_host(L):
    """The auxiliary-loss entry checks shapes, pointers, alignment and the workspace before any
    launch."""
    need = L.moe_router_aux_loss_workspace_size(16, 128, 8, 2)
    assert need > 256 and need % 256 == 0
    assert L.moe_router_aux_loss_workspace_size(16, 96, 8, 2) == 0   # D not a multiple of 64
    assert L.moe_router_aux_loss_workspace_size(16, 128, 8, 9) == 0  # k > E
    args = dict(x=0x1000, wg=0x2000, bias=None, loss=0x3000, dwg=0x4000, dx=0x5000, ws=0x100000, ws_bytes=need)

    def call(**kw):
        a = dict(args, **kw)
        return L.moe_router_aux_loss(a["x"], a["wg"], a["bias"], 16, 128, 8, 2, ctypes.c_float(0.01), a["loss"],
                                     a["dwg"], a["dx"], a["ws"], a["ws_bytes"], None)

    assert call(loss=None) == 1
    assert call(dx=None) == 1
    assert call(x=0x1008) == 3
    assert call(dwg=0x4002) == 3
    assert call(ws=0x100010) == 3
    assert call(ws_bytes=need - 1) == 4
