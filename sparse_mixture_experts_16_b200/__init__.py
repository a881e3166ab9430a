"""Sparse Mixture-of-Experts FFN layer forward on one B200 (sm_100a).

A thin ctypes binding over ``libmoe_b200.so`` (declared in ``include/moe_b200.h``).  The
functions below carry the C entry points' names and only marshal arguments: torch tensors
supply device pointers, torch's current CUDA stream supplies the stream, and every step of
the layer runs in the library's CUDA kernels.  There is no fallback: if the library is
missing or the device is not a B200, calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

MOE_FLAG_FORCE_PREFILL = 1
MOE_FLAG_FORCE_DECODE = 2
MOE_FLAG_SAVE_FOR_BACKWARD = 4
MOE_FLAG_PREFILL_ROW_TILES = 8
MOE_FLAG_PREFILL_WIDE_TILES = 16
MOE_FLAG_PREFILL_PAIR_TILES = 32
MOE_PATH_STREAMING, MOE_PATH_FP8_STREAMING, MOE_PATH_ROW_TILES, MOE_PATH_WIDE_TILES, MOE_PATH_MIXED_TILES = 0, 1, 2, 3, 4
MOE_PATH_PAIR_TILES = 5
MOE_WEIGHTS_BF16 = 0
MOE_WEIGHTS_FP8_E4M3 = 1

STATUS = {
    0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE", 3: "MOE_ERR_ALIGNMENT",
    4: "MOE_ERR_WORKSPACE_TOO_SMALL", 5: "MOE_ERR_CUDA", 6: "MOE_ERR_DEVICE_INDEX", 7: "MOE_ERR_TIMEOUT",
    8: "MOE_ERR_NO_DEVICE",
}

# every symbol include/moe_b200.h declares
EXPORTS = (
    "moe_quantize_rows_fp8", "moe_router_topk_workspace_size", "moe_router_topk", "moe_router_aux_loss_workspace_size",
    "moe_router_aux_loss", "moe_permute_workspace_size", "moe_permute", "moe_permute_noalloc",
    "moe_grouped_swiglu_ffn_workspace_size",
    "moe_grouped_swiglu_ffn", "moe_combine", "moe_layer_workspace_size", "moe_layer_forward",
    "moe_layer_forward_host", "moe_layer_forward_timed", "moe_layer_kernel_count", "moe_layer_gemm_path", "moe_update_router_bias",
    "moe_layer_expert_counts", "moe_get_device_error", "moe_layer_backward_workspace_size", "moe_layer_backward",
    "moe_status_string",
)


class LayerGrads(ctypes.Structure):
    """moe_layer_grads_t: fp32 gradient outputs (device pointers)."""
    _fields_ = [(n, ctypes.c_void_p) for n in ("dw_gate", "dgate_up", "ddown", "dshared_gate_up", "dshared_down")]


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class LayerDesc(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int32), ("D", ctypes.c_int32), ("E", ctypes.c_int32), ("k", ctypes.c_int32),
        ("F", ctypes.c_int32), ("Fs", ctypes.c_int32),
        ("w_gate", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("gate_up", ctypes.c_void_p),
        ("down", ctypes.c_void_p), ("shared_gate_up", ctypes.c_void_p), ("shared_down", ctypes.c_void_p),
        ("flags", ctypes.c_int32),
        ("weight_format", ctypes.c_int32),
        ("gate_up_fp8", ctypes.c_void_p), ("gate_up_scale", ctypes.c_void_p),
        ("down_fp8", ctypes.c_void_p), ("down_scale", ctypes.c_void_p),
        ("shared_gate_up_fp8", ctypes.c_void_p), ("shared_gate_up_scale", ctypes.c_void_p),
        ("shared_down_fp8", ctypes.c_void_p), ("shared_down_scale", ctypes.c_void_p),
    ]


_lib = None


def lib():
    """The loaded C library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m sparse_mixture_experts_16_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        sig = {
            "moe_quantize_rows_fp8": ([P, ctypes.c_int64, I, P, P, P], I),
            "moe_router_topk_workspace_size": ([I, I, I], Z),
            "moe_router_topk": ([P, P, P, I, I, I, I, P, P, P, Z, P], I),
            "moe_router_aux_loss_workspace_size": ([I, I, I, I], Z),
            "moe_router_aux_loss": ([P, P, P, I, I, I, I, ctypes.c_float, P, P, P, P, Z, P], I),
            "moe_permute_workspace_size": ([I, I, I], Z),
            "moe_permute": ([P, P, P, I, I, I, I, P, P, P, P, P, P, P, Z, P], I),
            "moe_permute_noalloc": ([P, P, P, I, I, I, I, P, P, P, P, P, P, P], I),
            "moe_grouped_swiglu_ffn_workspace_size": ([I, I], Z),
            "moe_grouped_swiglu_ffn": ([P, P, P, I, I, I, I, I, I, P, P, P, P, Z, P], I),
            "moe_combine": ([P, P, P, I, I, I, P, P], I),
            "moe_layer_workspace_size": ([ctypes.POINTER(LayerDesc)], Z),
            "moe_layer_forward": ([ctypes.POINTER(LayerDesc), P, P, P, Z, P], I),
            "moe_layer_forward_host": ([ctypes.POINTER(LayerDesc), P, P, P, Z, P], I),
            "moe_layer_forward_timed": ([ctypes.POINTER(LayerDesc), P, P, P, Z, P, ctypes.POINTER(P), I], I),
            "moe_layer_kernel_count": ([ctypes.POINTER(LayerDesc)], I),
            "moe_layer_gemm_path": ([ctypes.POINTER(LayerDesc)], I),
            "moe_update_router_bias": ([P, I, ctypes.c_float, P, P], I),
            "moe_layer_expert_counts": ([ctypes.POINTER(LayerDesc), P, Z, ctypes.POINTER(P)], I),
            "moe_get_device_error": ([P, P], I),
            "moe_layer_backward_workspace_size": ([ctypes.POINTER(LayerDesc)], Z),
            "moe_layer_backward": ([ctypes.POINTER(LayerDesc), P, P, P, ctypes.POINTER(LayerGrads), P, Z, P, Z, P], I),
            "moe_status_string": ([I], ctypes.c_char_p),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes, f.restype = args, res
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != 0:
        raise MoeError(status, where)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    import torch

    return (stream if stream is not None else torch.cuda.current_stream()).cuda_stream


def _need(t, dtype, shape, name):
    import torch

    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


# ------------------------------------------------------------------------------ steps
def moe_quantize_rows_fp8(w, stream=None):
    """Per-row E4M3 codes of a bf16 tensor [..., K]: (codes uint8 [..., K], scales fp32 [...])."""
    import torch

    _need(w, torch.bfloat16, None, "w")
    K = w.shape[-1]
    rows = w.numel() // K
    q = torch.empty(w.shape, dtype=torch.uint8, device=w.device)
    sc = torch.empty(w.shape[:-1], dtype=torch.float32, device=w.device)
    _check(lib().moe_quantize_rows_fp8(w.data_ptr(), rows, K, q.data_ptr(), sc.data_ptr(), _stream(stream)),
           "moe_quantize_rows_fp8")
    return q, sc


def moe_router_topk(x, w_gate, bias, k, topk_idx=None, topk_w=None, ws=None, stream=None):
    """Router projection + top-k + softmax over the chosen k -> (topk_idx[T,k] int32, topk_w[T,k] fp32)."""
    import torch

    T, D = x.shape
    E = w_gate.shape[0]
    _need(x, torch.bfloat16, None, "x")
    _need(w_gate, torch.bfloat16, (E, D), "w_gate")
    if bias is not None:
        _need(bias, torch.float32, (E,), "bias")
    if topk_idx is None:
        topk_idx = torch.empty(T, k, dtype=torch.int32, device=x.device)
    if topk_w is None:
        topk_w = torch.empty(T, k, dtype=torch.float32, device=x.device)
    need = lib().moe_router_topk_workspace_size(T, D, E)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=x.device)
    _check(lib().moe_router_topk(x.data_ptr(), w_gate.data_ptr(), _ptr(bias), T, D, E, k, topk_idx.data_ptr(),
                                 topk_w.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)), "moe_router_topk")
    return topk_idx, topk_w


def moe_router_aux_loss(x, w_gate, bias, k, alpha, ws=None, stream=None):
    """Router load-balancing auxiliary loss L = alpha * E * sum_e f_e P_e (training) and its
    gradients -> (loss [1], dw_gate [E, D], dx [T, D]), all fp32 on x's device; add the gradients
    to the layer backward's."""
    import torch

    T, D = x.shape
    E = w_gate.shape[0]
    _need(x, torch.bfloat16, None, "x")
    _need(w_gate, torch.bfloat16, (E, D), "w_gate")
    if bias is not None:
        _need(bias, torch.float32, (E,), "bias")
    loss = torch.empty(1, dtype=torch.float32, device=x.device)
    dwg = torch.empty(E, D, dtype=torch.float32, device=x.device)
    dx = torch.empty(T, D, dtype=torch.float32, device=x.device)
    need = lib().moe_router_aux_loss_workspace_size(T, D, E, k)
    if need == 0:
        raise MoeError(1, "moe_router_aux_loss_workspace_size")
    if ws is None or ws.numel() < need:
        ws = torch.zeros(need, dtype=torch.uint8, device=x.device)
    _check(lib().moe_router_aux_loss(x.data_ptr(), w_gate.data_ptr(), _ptr(bias), T, D, E, k, float(alpha),
                                     loss.data_ptr(), dwg.data_ptr(), dx.data_ptr(), ws.data_ptr(), ws.numel(),
                                     _stream(stream)), "moe_router_aux_loss")
    return loss, dwg, dx


def moe_permute(topk_idx, topk_w, x, E, stream=None, ws=None):
    """Dispatch metadata and the expert-contiguous copy of x.

    Returns dict(counts, offsets, perm_token, inv_perm, p_perm, x_perm (None if x is None), ws)."""
    import torch

    T, k = topk_idx.shape
    dev = topk_idx.device
    D = x.shape[1] if x is not None else 64
    M = T * k
    need = lib().moe_permute_workspace_size(T, E, k)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=dev)
    out = dict(
        counts=torch.empty(E, dtype=torch.int32, device=dev),
        offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
        perm_token=torch.empty(M, dtype=torch.int32, device=dev),
        inv_perm=torch.empty(M, dtype=torch.int32, device=dev),
        p_perm=torch.empty(M, dtype=torch.float32, device=dev),
        x_perm=torch.empty(M, D, dtype=torch.bfloat16, device=dev) if x is not None else None,
        ws=ws,
    )
    _check(lib().moe_permute(topk_idx.data_ptr(), topk_w.data_ptr(), _ptr(x), T, D, E, k,
                             out["counts"].data_ptr(), out["offsets"].data_ptr(), out["perm_token"].data_ptr(),
                             out["inv_perm"].data_ptr(), out["p_perm"].data_ptr(), _ptr(out["x_perm"]),
                             ws.data_ptr(), ws.numel(), _stream(stream)), "moe_permute")
    return out


def moe_permute_noalloc(topk_idx, topk_w, x, E, out=None, stream=None):
    """moe_permute for callers that cannot allocate device memory: the library keeps the
    scratch in a fixed internal array.  ``out`` (optional) holds caller-provided output tensors
    (keys as moe_permute's result); missing ones are created here by torch, not by the library."""
    import torch

    T, k = topk_idx.shape
    dev = topk_idx.device
    D = x.shape[1] if x is not None else 64
    M = T * k
    out = dict(out or {})
    out.setdefault("counts", torch.empty(E, dtype=torch.int32, device=dev))
    out.setdefault("offsets", torch.empty(E + 1, dtype=torch.int32, device=dev))
    out.setdefault("perm_token", torch.empty(M, dtype=torch.int32, device=dev))
    out.setdefault("inv_perm", torch.empty(M, dtype=torch.int32, device=dev))
    out.setdefault("p_perm", torch.empty(M, dtype=torch.float32, device=dev))
    if x is not None:
        out.setdefault("x_perm", torch.empty(M, D, dtype=torch.bfloat16, device=dev))
    _check(lib().moe_permute_noalloc(topk_idx.data_ptr(), topk_w.data_ptr(), _ptr(x), T, D, E, k,
                                     out["counts"].data_ptr(), out["offsets"].data_ptr(),
                                     out["perm_token"].data_ptr(), out["inv_perm"].data_ptr(),
                                     out["p_perm"].data_ptr(), _ptr(out.get("x_perm")), _stream(stream)),
           "moe_permute_noalloc")
    return out


def moe_grouped_swiglu_ffn(x_perm, offsets, row_scale, gate_up, down, max_seg=None, out_perm=None, ws=None,
                           stream=None, tiling=0):
    """out_perm[r] = row_scale[r] * Expert_e(x_perm[r]) for the rows r of each expert segment e.
    ``tiling``: 0 (the layer's default) or one MOE_FLAG_PREFILL_* flag."""
    import torch

    M, D = x_perm.shape
    E, twoF, D2 = gate_up.shape
    F = twoF // 2
    assert D2 == D and tuple(down.shape) == (E, D, F)
    if out_perm is None:
        out_perm = torch.empty(M, D, dtype=torch.float32, device=x_perm.device)
    need = lib().moe_grouped_swiglu_ffn_workspace_size(M, F)
    if ws is None or ws.numel() < need:
        ws = torch.zeros(max(need, 256), dtype=torch.uint8, device=x_perm.device)
    _check(lib().moe_grouped_swiglu_ffn(x_perm.data_ptr(), offsets.data_ptr(), _ptr(row_scale), M,
                                        M if max_seg is None else max_seg, tiling, E, D, F, gate_up.data_ptr(),
                                        down.data_ptr(), out_perm.data_ptr(), ws.data_ptr(), ws.numel(),
                                        _stream(stream)), "moe_grouped_swiglu_ffn")
    return out_perm, ws


def moe_combine(out_perm, inv_perm, shared_out, T, k, y=None, stream=None):
    import torch

    D = out_perm.shape[1]
    if y is None:
        y = torch.empty(T, D, dtype=torch.bfloat16, device=out_perm.device)
    _check(lib().moe_combine(out_perm.data_ptr(), inv_perm.data_ptr(), _ptr(shared_out), T, D, k, y.data_ptr(),
                             _stream(stream)), "moe_combine")
    return y


# ------------------------------------------------------------------------------ whole layer
class MoELayer:
    """Holds the layer's device weights and a workspace; ``forward(x)`` runs the whole layer.

    w_gate [E,D] bf16, bias [E] fp32 or None, gate_up [E,2F,D] bf16, down [E,D,F] bf16,
    shared_gate_up [2Fs,D] / shared_down [D,Fs] bf16 or None.  Tensors must stay alive.
    With ``scales`` = dict(gate_up=[E,2F], down=[E,D], shared_gate_up=[2Fs], shared_down=[D]) the
    weight tensors are E4M3 codes (uint8, from moe_quantize_rows_fp8) and the layer runs its
    FP8-weight decode kernels (T <= 64).
    """

    def __init__(self, w_gate, gate_up, down, k, bias=None, shared_gate_up=None, shared_down=None, flags=0,
                 scales=None):
        self.w_gate, self.gate_up, self.down, self.bias = w_gate, gate_up, down, bias
        self.shared_gate_up, self.shared_down = shared_gate_up, shared_down
        self.scales = scales
        self.E, self.D = w_gate.shape
        self.F = gate_up.shape[1] // 2
        self.Fs = 0 if shared_gate_up is None else shared_gate_up.shape[0] // 2
        self.k = k
        self.flags = flags
        self._ws = None

    def desc(self, T: int) -> LayerDesc:
        if self.scales is None:
            return LayerDesc(T, self.D, self.E, self.k, self.F, self.Fs, self.w_gate.data_ptr(), _ptr(self.bias),
                             self.gate_up.data_ptr(), self.down.data_ptr(), _ptr(self.shared_gate_up),
                             _ptr(self.shared_down), self.flags, MOE_WEIGHTS_BF16)
        sc = self.scales
        return LayerDesc(T, self.D, self.E, self.k, self.F, self.Fs, self.w_gate.data_ptr(), _ptr(self.bias),
                         None, None, None, None, self.flags, MOE_WEIGHTS_FP8_E4M3,
                         self.gate_up.data_ptr(), sc["gate_up"].data_ptr(), self.down.data_ptr(),
                         sc["down"].data_ptr(), _ptr(self.shared_gate_up), _ptr(sc.get("shared_gate_up")),
                         _ptr(self.shared_down), _ptr(sc.get("shared_down")))

    def workspace(self, T: int):
        import torch

        d = self.desc(T)
        need = lib().moe_layer_workspace_size(ctypes.byref(d))
        if need == 0:
            raise MoeError(1, "moe_layer_workspace_size")
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.zeros(need, dtype=torch.uint8, device=self.w_gate.device)
        return self._ws

    def new_workspace(self, T: int):
        """A workspace of its own for T tokens: forwards that may overlap (on different streams)
        each need one."""
        import torch

        d = self.desc(T)
        need = lib().moe_layer_workspace_size(ctypes.byref(d))
        if need == 0:
            raise MoeError(1, "moe_layer_workspace_size")
        return torch.zeros(need, dtype=torch.uint8, device=self.w_gate.device)

    def kernel_count(self, T: int) -> int:
        d = self.desc(T)
        return lib().moe_layer_kernel_count(ctypes.byref(d))

    def gemm_path(self, T: int) -> str:
        """The expert-GEMM kernels a forward over T tokens runs: "streaming", "fp8_streaming",
        "row_tiles", "wide_tiles", "mixed_tiles" (gate_up on row tiles, down on pair tiles) or
        "pair_tiles" (both on token-wide tiles of CTA pairs)."""
        d = self.desc(T)
        code = lib().moe_layer_gemm_path(ctypes.byref(d))
        if code < 0:
            raise MoeError(1, "moe_layer_gemm_path")
        return ("streaming", "fp8_streaming", "row_tiles", "wide_tiles", "mixed_tiles", "pair_tiles")[code]

    def forward(self, x, y=None, stream=None):
        import torch

        T = x.shape[0]
        _need(x, torch.bfloat16, (T, self.D), "x")
        if y is None:
            y = torch.empty_like(x)
        ws = self.workspace(T)
        d = self.desc(T)
        _check(lib().moe_layer_forward(ctypes.byref(d), x.data_ptr(), y.data_ptr(), ws.data_ptr(), ws.numel(),
                                       _stream(stream)), "moe_layer_forward")
        return y

    __call__ = forward

    def forward_host(self, x_host, y_host, stream=None, ws=None):
        """x_host / y_host: pinned CPU bf16 tensors [T, D]; asynchronous on the stream.  ``ws``:
        a workspace from new_workspace() (default: the layer's own)."""
        T = x_host.shape[0]
        ws = self.workspace(T) if ws is None else ws
        d = self.desc(T)
        _check(lib().moe_layer_forward_host(ctypes.byref(d), x_host.data_ptr(), y_host.data_ptr(), ws.data_ptr(),
                                            ws.numel(), _stream(stream)), "moe_layer_forward_host")
        return y_host

    def forward_timed(self, x, y, events, stream=None):
        """forward() recording 6 torch.cuda.Event objects around the stages (router, dispatch,
        gate_up GEMM, down GEMM, combine)."""
        T = x.shape[0]
        ws = self.workspace(T)
        d = self.desc(T)
        handles = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
        _check(lib().moe_layer_forward_timed(ctypes.byref(d), x.data_ptr(), y.data_ptr(), ws.data_ptr(), ws.numel(),
                                             _stream(stream), handles, len(events)), "moe_layer_forward_timed")
        return y

    def expert_counts(self, T: int):
        """counts[E] int32 left in the workspace by the last forward of T tokens (a view, not a copy)."""
        import torch

        ws = self.workspace(T)
        d = self.desc(T)
        ptr = ctypes.c_void_p()
        _check(lib().moe_layer_expert_counts(ctypes.byref(d), ws.data_ptr(), ws.numel(), ctypes.byref(ptr)),
               "moe_layer_expert_counts")
        off = ptr.value - ws.data_ptr()
        return ws[off:off + 4 * self.E].view(torch.int32)

    def backward(self, x, dy, stream=None):
        """Gradients of sum(dy * y) after forward(x) on a layer built with
        flags=MOE_FLAG_SAVE_FOR_BACKWARD: (dx [T, D] bf16, dict of fp32 weight gradients
        dw_gate, dgate_up, ddown, dshared_gate_up, dshared_down (None without a shared expert))."""
        import torch

        T = x.shape[0]
        _need(dy, torch.bfloat16, (T, self.D), "dy")
        d = self.desc(T)
        need = lib().moe_layer_backward_workspace_size(ctypes.byref(d))
        if need == 0:
            raise MoeError(1, "moe_layer_backward_workspace_size")
        if getattr(self, "_bws", None) is None or self._bws.numel() < need:
            self._bws = torch.zeros(need, dtype=torch.uint8, device=x.device)
        dev, f32 = x.device, torch.float32
        g = dict(dw_gate=torch.empty(self.E, self.D, dtype=f32, device=dev),
                 dgate_up=torch.empty(self.E, 2 * self.F, self.D, dtype=f32, device=dev),
                 ddown=torch.empty(self.E, self.D, self.F, dtype=f32, device=dev),
                 dshared_gate_up=torch.empty(2 * self.Fs, self.D, dtype=f32, device=dev) if self.Fs else None,
                 dshared_down=torch.empty(self.D, self.Fs, dtype=f32, device=dev) if self.Fs else None)
        grads = LayerGrads(*[_ptr(g[n]) for n in ("dw_gate", "dgate_up", "ddown", "dshared_gate_up", "dshared_down")])
        dx = torch.empty_like(x)
        ws = self.workspace(T)
        _check(lib().moe_layer_backward(ctypes.byref(d), x.data_ptr(), dy.data_ptr(), dx.data_ptr(), ctypes.byref(grads),
                                        ws.data_ptr(), ws.numel(), self._bws.data_ptr(), self._bws.numel(),
                                        _stream(stream)), "moe_layer_backward")
        return dx, g

    def backward_error(self, stream=None) -> int:
        """Synchronises and returns (and clears) the backward workspace's device error status."""
        if getattr(self, "_bws", None) is None:
            return 0
        return lib().moe_get_device_error(self._bws.data_ptr(), _stream(stream))

    def device_error(self, stream=None) -> int:
        """Synchronises and returns (and clears) the workspace's device error status."""
        if self._ws is None:
            return 0
        return lib().moe_get_device_error(self._ws.data_ptr(), _stream(stream))


def moe_update_router_bias(counts, gamma, bias, stream=None):
    """One aux-loss-free balancing step in place: bias += gamma * sign(mean(counts) - counts)."""
    import torch

    _need(counts, torch.int32, None, "counts")
    _need(bias, torch.float32, tuple(counts.shape), "bias")
    _check(lib().moe_update_router_bias(counts.data_ptr(), counts.numel(), float(gamma), bias.data_ptr(),
                                        _stream(stream)), "moe_update_router_bias")
    return bias


def moe_get_device_error(ws, stream=None) -> int:
    return lib().moe_get_device_error(ws.data_ptr(), _stream(stream))


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(status).decode()
