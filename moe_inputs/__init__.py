"""Seeded synthetic inputs for the sparse-MoE layer: the workload shapes and their recipe.

This module serves both the fp64 oracle (host arrays) and the GPU path (device
tensors).  It holds none of the layer's arithmetic; every value comes from the
counter-based generator in ``csrc/moe_inputs.h`` (SplitMix64 words, Irwin-Hall
normal variates, bf16 round-to-nearest-even), evaluated identically on host and
device.

Workloads (one per ``WORKLOADS`` entry) are the layer shapes named after the
model families the pages use as examples of coarse- and fine-grained MoE:
Mixtral-8x7B (8 experts, top-2), gpt-oss-20b (32 experts, top-4) and
DeepSeek-V3 (256 routed experts, top-8, one always-on shared expert).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, replace
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmoe_inputs.so")
_SRC = os.path.join(_HERE, "csrc", "moe_inputs.cu")
_lib = None

# stream ids (must match csrc/moe_inputs.h)
STREAM_X, STREAM_WG, STREAM_GATE_UP, STREAM_DOWN = 1, 2, 3, 4
STREAM_SH_GATE_UP, STREAM_SH_DOWN, STREAM_BIAS, STREAM_RANK = 5, 6, 7, 8

SIGMA_X = 1.0
SIGMA_EXPERT = 0.02
SIGMA_ROUTER = 0.1


@dataclass(frozen=True)
class Workload:
    """One synthetic layer: T tokens, model dim D, E routed experts, top-k, expert FFN
    width F, shared-expert width Fs (0 = none), and the selection-bias recipe."""

    name: str
    T: int
    D: int
    E: int
    k: int
    F: int
    Fs: int = 0
    bias: str = "none"  # "none" | "normal:<sigma>" | "zipf:<s>"
    seed: int = 0

    def with_T(self, T: int) -> "Workload":
        return replace(self, T=T, name=f"{self.name.split('@')[0]}@T{T}")

    @property
    def flops(self) -> float:
        """Algorithmic FLOPs: router 2DE, routed SwiGLU 6kDF, shared 6DFs, per token."""
        return float(self.T) * (2 * self.D * self.E + 6 * self.k * self.D * self.F + 6 * self.D * self.Fs)


WORKLOADS = {
    # tiny: the small case the oracle finishes in seconds
    "tiny": Workload("tiny", T=256, D=256, E=8, k=2, F=512),
    # coarse MoE, Mixtral-8x7B-shaped layer
    "mixtral": Workload("mixtral", T=4096, D=4096, E=8, k=2, F=14336),
    # gpt-oss-20b-shaped layer, prefill; Zipf(s=1.1) selection bias unbalances expert loads
    "gptoss": Workload("gptoss", T=8192, D=2880, E=32, k=4, F=2880, bias="zipf:1.1"),
    # fine-grained DeepSeek-V3-shaped layer with one always-on shared expert
    "deepseek": Workload("deepseek", T=8192, D=7168, E=256, k=8, F=2048, Fs=2048, bias="normal:0.5"),
    # decode-bound fine-grained layer
    "deepseek_decode": Workload("deepseek_decode", T=16, D=7168, E=256, k=8, F=2048, Fs=2048,
                                bias="normal:0.5"),
}
for _t in (1, 8, 32, 64):
    WORKLOADS[f"gptoss_decode_T{_t}"] = replace(WORKLOADS["gptoss"], name=f"gptoss_decode_T{_t}", T=_t)
# the DeepSeek-V3-shaped layer cut to 32 experts and 1024 tokens: the same per-expert GEMM shapes
# (~256 rows per expert segment, D = 7168, F = Fs = 2048) with 2.9 GB of weights instead of 22.6 GB,
# small enough for kernel profiling captures
WORKLOADS["deepseek_e32"] = replace(WORKLOADS["deepseek"], name="deepseek_e32", T=1024, E=32)


def build(force: bool = False) -> str:
    """Compile the generator (host + sm_100a device code) into libmoe_inputs.so."""
    if os.path.exists(_LIB_PATH) and not force and os.path.getmtime(_LIB_PATH) >= max(
        os.path.getmtime(_SRC), os.path.getmtime(os.path.join(_HERE, "csrc", "moe_inputs.h"))
    ):
        return _LIB_PATH
    cmd = [
        "nvcc", "-O2", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
        "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
        "-o", _LIB_PATH + ".tmp", _SRC,
    ]
    subprocess.run(cmd, check=True)
    os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        u16p, u32p, i64p, f32p = (ctypes.c_void_p,) * 4
        L.mi_fill_normal_bf16_host.argtypes = [u16p, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32,
                                               ctypes.c_uint32, ctypes.c_uint64, ctypes.c_float, ctypes.c_int]
        L.mi_fill_normal_f32_host.argtypes = [f32p, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32,
                                              ctypes.c_uint32, ctypes.c_uint64, ctypes.c_float]
        L.mi_fill_rows_bf16_host.argtypes = [u16p, ctypes.c_int64, ctypes.c_int64, i64p, u32p,
                                             ctypes.c_uint64, ctypes.c_uint32, ctypes.c_float, ctypes.c_int]
        L.mi_word_host.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64]
        L.mi_word_host.restype = ctypes.c_uint64
        L.mi_mix64_host.argtypes = [ctypes.c_uint64]
        L.mi_mix64_host.restype = ctypes.c_uint64
        L.mi_normal_host.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint64]
        L.mi_normal_host.restype = ctypes.c_float
        L.mi_fill_normal_bf16_device.argtypes = [u16p, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32,
                                                 ctypes.c_uint32, ctypes.c_uint64, ctypes.c_float,
                                                 ctypes.c_void_p]
        L.mi_fill_normal_bf16_device.restype = ctypes.c_int
        L.mi_fill_rows_bf16_device.argtypes = [u16p, ctypes.c_int64, ctypes.c_int64, u32p, ctypes.c_uint64,
                                               ctypes.c_uint32, ctypes.c_float, ctypes.c_void_p]
        L.mi_fill_rows_bf16_device.restype = ctypes.c_int
        _lib = L
    return _lib


def _nthreads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------- host side
def normal_bf16(stream: int, n: int, sigma: float, seed: int = 0, first: int = 0, redraw: int = 0) -> np.ndarray:
    """Variates [first, first+n) of a stream as bf16 bit patterns (uint16)."""
    out = np.empty(n, dtype=np.uint16)
    lib().mi_fill_normal_bf16_host(out.ctypes.data, n, seed, stream, redraw, first, sigma, _nthreads())
    return out


def rows_bf16(stream: int, rows, cols: int, sigma: float, seed: int = 0, redraw=None) -> np.ndarray:
    """Rows `rows` (int array) of a [*, cols] bf16 tensor, row i drawn from substream redraw[i]."""
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    out = np.empty((rows.size, cols), dtype=np.uint16)
    rd = None
    if redraw is not None:
        rd = np.ascontiguousarray(redraw, dtype=np.uint32)
        assert rd.size == rows.size
    lib().mi_fill_rows_bf16_host(out.ctypes.data, rows.size, cols, rows.ctypes.data,
                                 rd.ctypes.data if rd is not None else None, seed, stream, sigma, _nthreads())
    return out


def bias_f32(w: Workload) -> Optional[np.ndarray]:
    """Per-expert selection bias[E] (fp32) or None.

    normal:<s>  -> bias[e] ~ N(0, s^2) (same variates as the other tensors, kept in fp32)
    zipf:<s>    -> a seeded random rank r_e in {1..E} per expert, bias[e] = -s * ln(r_e)
    """
    if w.bias == "none":
        return None
    kind, val = w.bias.split(":")
    s = float(val)
    if kind == "normal":
        out = np.empty(w.E, dtype=np.float32)
        lib().mi_fill_normal_f32_host(out.ctypes.data, w.E, w.seed, STREAM_BIAS, 0, 0, s)
        return out
    if kind == "zipf":
        words = [lib().mi_word_host(w.seed, STREAM_RANK, 0, e) for e in range(w.E)]
        order = sorted(range(w.E), key=lambda e: (words[e], e))
        rank = [0] * w.E
        for pos, e in enumerate(order):
            rank[e] = pos + 1
        return np.array([-s * math.log(r) for r in rank], dtype=np.float32)
    raise ValueError(w.bias)


def host_x(w: Workload, rows=None, redraw=None) -> np.ndarray:
    rows = np.arange(w.T) if rows is None else rows
    return rows_bf16(STREAM_X, rows, w.D, SIGMA_X, w.seed, redraw)


def host_wg(w: Workload) -> np.ndarray:
    return normal_bf16(STREAM_WG, w.E * w.D, SIGMA_ROUTER, w.seed).reshape(w.E, w.D)


def host_gate_up(w: Workload, experts=None) -> np.ndarray:
    """gate_up_proj rows of the given experts: [len(experts), 2F, D] (rows [0,F) gate, [F,2F) up)."""
    experts = range(w.E) if experts is None else experts
    per = 2 * w.F * w.D
    return np.stack([normal_bf16(STREAM_GATE_UP, per, SIGMA_EXPERT, w.seed, first=e * per)
                     for e in experts]).reshape(-1, 2 * w.F, w.D)


def host_down(w: Workload, experts=None) -> np.ndarray:
    experts = range(w.E) if experts is None else experts
    per = w.D * w.F
    return np.stack([normal_bf16(STREAM_DOWN, per, SIGMA_EXPERT, w.seed, first=e * per)
                     for e in experts]).reshape(-1, w.D, w.F)


def host_shared(w: Workload):
    if w.Fs == 0:
        return None, None
    gu = normal_bf16(STREAM_SH_GATE_UP, 2 * w.Fs * w.D, SIGMA_EXPERT, w.seed).reshape(2 * w.Fs, w.D)
    dn = normal_bf16(STREAM_SH_DOWN, w.D * w.Fs, SIGMA_EXPERT, w.seed).reshape(w.D, w.Fs)
    return gu, dn


def host_inputs(w: Workload, redraw=None) -> dict:
    """Every input of a (small) workload as host arrays (bf16 as uint16 bit patterns)."""
    sgu, sdn = host_shared(w)
    return dict(x=host_x(w, redraw=redraw), wg=host_wg(w), bias=bias_f32(w), gate_up=host_gate_up(w),
                down=host_down(w), shared_gate_up=sgu, shared_down=sdn)


def bf16_to_f64(a: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact float64 values."""
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------- device side
def device_fill_bf16(t, stream_id: int, sigma: float, seed: int = 0, first: int = 0, redraw: int = 0):
    """Fill a contiguous torch bf16 CUDA tensor with variates [first, first+numel) of a stream."""
    import torch

    assert t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous()
    rc = lib().mi_fill_normal_bf16_device(t.data_ptr(), t.numel(), seed, stream_id, redraw, first, sigma,
                                          torch.cuda.current_stream().cuda_stream)
    if rc != 0:
        raise RuntimeError(f"device fill failed: cuda error {rc}")
    return t


def device_fill_rows_bf16(t, stream_id: int, sigma: float, seed: int = 0, redraw_dev=None):
    import torch

    assert t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and t.dim() == 2
    rc = lib().mi_fill_rows_bf16_device(t.data_ptr(), t.shape[0], t.shape[1],
                                        redraw_dev.data_ptr() if redraw_dev is not None else None,
                                        seed, stream_id, sigma, torch.cuda.current_stream().cuda_stream)
    if rc != 0:
        raise RuntimeError(f"device fill failed: cuda error {rc}")
    return t


def device_inputs(w: Workload, device="cuda", redraw=None) -> dict:
    """Every input of a workload generated directly in HBM (bit-identical to host_inputs)."""
    import torch

    bf = torch.bfloat16
    x = torch.empty(w.T, w.D, dtype=bf, device=device)
    rd = None
    if redraw is not None:
        rd = torch.as_tensor(np.ascontiguousarray(redraw, dtype=np.uint32).view(np.int32), device=device)
    device_fill_rows_bf16(x, STREAM_X, SIGMA_X, w.seed, rd)
    wg = device_fill_bf16(torch.empty(w.E, w.D, dtype=bf, device=device), STREAM_WG, SIGMA_ROUTER, w.seed)
    gu = device_fill_bf16(torch.empty(w.E, 2 * w.F, w.D, dtype=bf, device=device), STREAM_GATE_UP,
                          SIGMA_EXPERT, w.seed)
    dn = device_fill_bf16(torch.empty(w.E, w.D, w.F, dtype=bf, device=device), STREAM_DOWN, SIGMA_EXPERT,
                          w.seed)
    sgu = sdn = None
    if w.Fs:
        sgu = device_fill_bf16(torch.empty(2 * w.Fs, w.D, dtype=bf, device=device), STREAM_SH_GATE_UP,
                               SIGMA_EXPERT, w.seed)
        sdn = device_fill_bf16(torch.empty(w.D, w.Fs, dtype=bf, device=device), STREAM_SH_DOWN,
                               SIGMA_EXPERT, w.seed)
    b = bias_f32(w)
    bias = torch.from_numpy(b).to(device) if b is not None else None
    return dict(x=x, wg=wg, bias=bias, gate_up=gu, down=dn, shared_gate_up=sgu, shared_down=sdn)
