"""fp64 CPU oracle of the sparse-MoE FFN layer forward -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg of
``bench.py`` may import this package.  The product path (``sparse_mixture_experts_16_b200``)
never does, and shares no code with it.

The arithmetic lives in ``moe_oracle.cpp`` (plain C++ loops in fp64 over exact bf16 inputs);
this module only compiles it with g++ and marshals numpy arrays.  Pins that tie it to the
pages and to mathematics (not to itself) are in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.cpp")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    if os.path.exists(_LIB) and not force and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    subprocess.run(["g++", "-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
                    "-o", _LIB + ".tmp", _SRC], check=True)
    os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _L():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64, i32 = ctypes.c_int64, ctypes.c_int
        L.oracle_router.argtypes = [P, P, P, i64, i64, i32, i32, P, P, P, i32]
        L.oracle_topk_exhaustive.argtypes = [P, i64, i32, i32, P]
        L.oracle_permute.argtypes = [P, i64, i32, i32, P, P, P, P, P]
        L.oracle_expert_ffn.argtypes = [P, P, P, i64, i64, P]
        L.oracle_expert_ffn.restype = None
        L.oracle_layer.argtypes = [P, P, P, P, P, P, P, i64, i64, i32, i32, i64, i64, P, P, P, i32]
        L.oracle_layer_eager.argtypes = [P, P, P, P, P, P, P, i64, i64, i32, i32, i64, i64, P]
        L.oracle_update_bias.argtypes = [P, i32, ctypes.c_float, P, P]
        L.oracle_update_bias.restype = None
        L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e4m3_encode.argtypes = [ctypes.c_double]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_quantize_rows_fp8.argtypes = [P, i64, i64, P, P, i32]
        L.oracle_quantize_rows_fp8.restype = None
        L.oracle_expert_ffn_fp8.argtypes = [P, P, P, P, P, i64, i64, P]
        L.oracle_expert_ffn_fp8.restype = None
        L.oracle_layer_f64.argtypes = [P, P, P, P, P, P, P, i64, i64, i32, i32, i64, i64, P, i32]
        L.oracle_layer_backward_f64.argtypes = [P, P, P, P, P, P, P, P, i64, i64, i32, i32, i64, i64,
                                                P, P, P, P, P, P, i32]
        L.oracle_router_aux_loss_f64.argtypes = [P, P, P, i64, i64, i32, i32, ctypes.c_double, P, P, P, i32]
        _lib = L
    return _lib


def _nthreads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _u16(a):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


def _ptr(a):
    return None if a is None else a.ctypes.data


def router(x, wg, bias, k, return_logits=False, nthreads=None):
    """idx[T,k] int32 (score-descending), p[T,k] float64 (and logits[T,E] float64)."""
    x, wg = _u16(x), _u16(wg)
    T, D = x.shape
    E = wg.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    idx = np.empty((T, k), np.int32)
    p = np.empty((T, k), np.float64)
    lg = np.empty((T, E), np.float64) if return_logits else None
    rc = _L().oracle_router(x.ctypes.data, wg.ctypes.data, _ptr(b), T, D, E, k, _ptr(lg), idx.ctypes.data,
                            p.ctypes.data, nthreads or _nthreads())
    if rc != 0:
        raise ValueError(f"oracle_router rc={rc}")
    return (idx, p, lg) if return_logits else (idx, p)


def topk_exhaustive(scores, k):
    s = np.ascontiguousarray(scores, dtype=np.float64)
    T, E = s.shape
    idx = np.empty((T, k), np.int32)
    rc = _L().oracle_topk_exhaustive(s.ctypes.data, T, E, k, idx.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_topk_exhaustive rc={rc}")
    return idx


def permute(idx, E):
    """counts[E], offsets[E+1], perm_token[T*k], perm_slot[T*k], inv_perm[T*k] (all int32)."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, k = idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    pt = np.empty(T * k, np.int32)
    ps = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    rc = _L().oracle_permute(idx.ctypes.data, T, E, k, counts.ctypes.data, offsets.ctypes.data,
                             pt.ctypes.data, ps.ctypes.data, inv.ctypes.data)
    if rc != 0:
        raise ValueError("expert id out of range")
    return counts, offsets, pt, ps, inv


def expert_ffn(x_row, gate_up_e, down_e):
    x_row, gu, dn = _u16(x_row), _u16(gate_up_e), _u16(down_e)
    D = x_row.shape[-1]
    F = dn.shape[1]
    assert gu.shape == (2 * F, D) and dn.shape == (D, F)
    out = np.empty(D, np.float64)
    _L().oracle_expert_ffn(x_row.ctypes.data, gu.ctypes.data, dn.ctypes.data, D, F, out.ctypes.data)
    return out


def layer(x, wg, bias, gate_up, down, k, shared_gate_up=None, shared_down=None, nthreads=None,
          F=None):
    """y[T,D] float64 plus (idx, p).

    gate_up / down are either packed arrays [E,2F,D] / [E,D,F] or dicts {expert: array} holding
    only the experts that the tokens of ``x`` route to (for sampled checks at full size).
    """
    x, wg = _u16(x), _u16(wg)
    T, D = x.shape
    E = wg.shape[0]
    keep = []
    if isinstance(gate_up, dict):
        gu_ptrs = (ctypes.c_void_p * E)()
        dn_ptrs = (ctypes.c_void_p * E)()
        for e, a in gate_up.items():
            a = _u16(a)
            keep.append(a)
            gu_ptrs[e] = a.ctypes.data
            F = a.shape[0] // 2
        for e, a in down.items():
            a = _u16(a)
            keep.append(a)
            dn_ptrs[e] = a.ctypes.data
    else:
        gate_up, down = _u16(gate_up), _u16(down)
        keep += [gate_up, down]
        F = gate_up.shape[1] // 2
        gu_ptrs = (ctypes.c_void_p * E)(*[gate_up.ctypes.data + e * gate_up[0].nbytes for e in range(E)])
        dn_ptrs = (ctypes.c_void_p * E)(*[down.ctypes.data + e * down[0].nbytes for e in range(E)])
    sgu = None if shared_gate_up is None else _u16(shared_gate_up)
    sdn = None if shared_down is None else _u16(shared_down)
    Fs = 0 if sgu is None else sgu.shape[0] // 2
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    y = np.empty((T, D), np.float64)
    idx = np.empty((T, k), np.int32)
    p = np.empty((T, k), np.float64)
    rc = _L().oracle_layer(x.ctypes.data, wg.ctypes.data, _ptr(b), gu_ptrs, dn_ptrs, _ptr(sgu), _ptr(sdn),
                           T, D, E, k, F, Fs, y.ctypes.data, idx.ctypes.data, p.ctypes.data,
                           nthreads or _nthreads())
    if rc != 0:
        raise ValueError(f"oracle_layer rc={rc}")
    return y, idx, p


def layer_eager(x, wg, bias, gate_up, down, k, shared_gate_up=None, shared_down=None):
    x, wg, gate_up, down = _u16(x), _u16(wg), _u16(gate_up), _u16(down)
    T, D = x.shape
    E = wg.shape[0]
    F = gate_up.shape[1] // 2
    sgu = None if shared_gate_up is None else _u16(shared_gate_up)
    sdn = None if shared_down is None else _u16(shared_down)
    Fs = 0 if sgu is None else sgu.shape[0] // 2
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    y = np.empty((T, D), np.float64)
    rc = _L().oracle_layer_eager(x.ctypes.data, wg.ctypes.data, _ptr(b), gate_up.ctypes.data,
                                 down.ctypes.data, _ptr(sgu), _ptr(sdn), T, D, E, k, F, Fs, y.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_layer_eager rc={rc}")
    return y


def update_bias(counts, gamma, bias):
    """One aux-loss-free balancing step: bias + gamma * sign(mean(counts) - counts), fp32."""
    c = np.ascontiguousarray(counts, dtype=np.int32)
    b = np.ascontiguousarray(bias, dtype=np.float32)
    out = np.empty_like(b)
    _L().oracle_update_bias(c.ctypes.data, c.size, gamma, b.ctypes.data, out.ctypes.data)
    return out


def e4m3_value(code: int) -> float:
    return _L().oracle_e4m3_value(code)


def e4m3_encode(v: float) -> int:
    return _L().oracle_e4m3_encode(v)


def quantize_rows_fp8(w):
    """Per-row E4M3 quantisation of a bf16 [rows, K] array: (codes uint8 [rows, K], scales fp32 [rows])."""
    w = _u16(w)
    K = w.shape[-1]
    rows = w.size // K
    q = np.empty(w.shape, np.uint8)
    sc = np.empty(w.shape[:-1], np.float32)
    _L().oracle_quantize_rows_fp8(w.ctypes.data, rows, K, q.ctypes.data, sc.ctypes.data, _nthreads())
    return q, sc


def expert_ffn_fp8(x_row, gu_q, gu_s, dn_q, dn_s):
    x_row = _u16(x_row)
    gu_q, dn_q = np.ascontiguousarray(gu_q, np.uint8), np.ascontiguousarray(dn_q, np.uint8)
    gu_s, dn_s = np.ascontiguousarray(gu_s, np.float32), np.ascontiguousarray(dn_s, np.float32)
    D = x_row.shape[-1]
    F = dn_q.shape[1]
    assert gu_q.shape == (2 * F, D) and dn_q.shape == (D, F) and gu_s.shape == (2 * F,) and dn_s.shape == (D,)
    out = np.empty(D, np.float64)
    _L().oracle_expert_ffn_fp8(x_row.ctypes.data, gu_q.ctypes.data, gu_s.ctypes.data, dn_q.ctypes.data,
                               dn_s.ctypes.data, D, F, out.ctypes.data)
    return out


def layer_fp8(x, wg, bias, k, q, shared=None):
    """y[T, D] of the layer with E4M3 expert weights.  q: dict(gu_q [E,2F,D], gu_s [E,2F],
    dn_q [E,D,F], dn_s [E,D]) (or dicts {expert: array} for the experts used); shared: the same
    four arrays for the shared expert or None.  Returns (y, idx, p)."""
    from concurrent.futures import ThreadPoolExecutor

    idx, p = router(x, wg, bias, k)
    T, D = x.shape

    def token(t):  # tokens are independent; the C call releases the GIL
        yt = np.zeros(D, np.float64)
        for j in range(k):
            e = int(idx[t, j])
            yt += p[t, j] * expert_ffn_fp8(x[t], q["gu_q"][e], q["gu_s"][e], q["dn_q"][e], q["dn_s"][e])
        if shared is not None:
            yt += expert_ffn_fp8(x[t], shared["gu_q"], shared["gu_s"], shared["dn_q"], shared["dn_s"])
        return yt

    with ThreadPoolExecutor(max_workers=_nthreads()) as pool:
        y = np.stack(list(pool.map(token, range(T)))) if T else np.zeros((0, D), np.float64)
    return y, idx, p


# ----------------------------------------------------------------------------- backward (training)
def _f64(a):
    """bf16 bit patterns (uint16) -> exact float64 values; float arrays -> contiguous float64."""
    if a is None:
        return None
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return np.ascontiguousarray((a.astype(np.uint32) << 16).view(np.float32).astype(np.float64))
    return np.ascontiguousarray(a, dtype=np.float64)


def layer_f64(x, wg, bias, gate_up, down, k, shared_gate_up=None, shared_down=None):
    """The layer forward on fp64 parameters (bf16 bit patterns are read exactly): y [T, D]."""
    x, wg, gu, dn = _f64(x), _f64(wg), _f64(gate_up), _f64(down)
    sgu, sdn = _f64(shared_gate_up), _f64(shared_down)
    T, D = x.shape
    E = wg.shape[0]
    F = dn.shape[2]
    Fs = 0 if sgu is None else sgu.shape[0] // 2
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    y = np.empty((T, D), np.float64)
    rc = _L().oracle_layer_f64(x.ctypes.data, wg.ctypes.data, _ptr(b), gu.ctypes.data, dn.ctypes.data, _ptr(sgu),
                               _ptr(sdn), T, D, E, k, F, Fs, y.ctypes.data, _nthreads())
    if rc != 0:
        raise ValueError(f"oracle_layer_f64 rc={rc}")
    return y


def layer_backward(x, wg, bias, gate_up, down, k, dy, shared_gate_up=None, shared_down=None):
    """Gradients of L = sum(dy * y) for the layer forward: dict(dx, dw_gate, dgate_up, ddown,
    dshared_gate_up, dshared_down), all float64 (shared entries None without a shared expert)."""
    x, wg, gu, dn, dy = _f64(x), _f64(wg), _f64(gate_up), _f64(down), _f64(dy)
    sgu, sdn = _f64(shared_gate_up), _f64(shared_down)
    T, D = x.shape
    E = wg.shape[0]
    F = dn.shape[2]
    Fs = 0 if sgu is None else sgu.shape[0] // 2
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    out = dict(dx=np.empty((T, D)), dw_gate=np.empty((E, D)), dgate_up=np.empty((E, 2 * F, D)),
               ddown=np.empty((E, D, F)), dshared_gate_up=np.empty((2 * Fs, D)) if Fs else None,
               dshared_down=np.empty((D, Fs)) if Fs else None)
    rc = _L().oracle_layer_backward_f64(
        x.ctypes.data, wg.ctypes.data, _ptr(b), gu.ctypes.data, dn.ctypes.data, _ptr(sgu), _ptr(sdn), dy.ctypes.data,
        T, D, E, k, F, Fs, out["dx"].ctypes.data, out["dw_gate"].ctypes.data, out["dgate_up"].ctypes.data,
        out["ddown"].ctypes.data, _ptr(out["dshared_gate_up"]), _ptr(out["dshared_down"]), _nthreads())
    if rc != 0:
        raise ValueError(f"oracle_layer_backward_f64 rc={rc}")
    return out


def router_aux_loss(x, wg, bias, k, alpha):
    """Load-balancing auxiliary loss L = alpha * E * sum_e f_e P_e of the router (the reading and its
    gradient are stated at oracle_router_aux_loss_f64): (loss float, dw_gate [E, D], dx [T, D]),
    float64; f counts the top-k of l + bias and carries no gradient."""
    x, wg = _f64(x), _f64(wg)
    T, D = x.shape
    E = wg.shape[0]
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    loss = np.zeros(1)
    dwg = np.empty((E, D))
    dx = np.empty((T, D))
    rc = _L().oracle_router_aux_loss_f64(x.ctypes.data, wg.ctypes.data, _ptr(b), T, D, E, k, float(alpha),
                                         loss.ctypes.data, dwg.ctypes.data, dx.ctypes.data, _nthreads())
    if rc != 0:
        raise ValueError(f"oracle_router_aux_loss_f64 rc={rc}")
    return float(loss[0]), dwg, dx


# ----------------------------------------------------------------------------- gap-enforced inputs
# Router scores must be separated by at least GAP among each token's top k+1 experts (fp64
# scores on the bf16 inputs), so fp32 accumulation on a GPU (error ~1e-4 at D = 7168) cannot
# reorder them and top-k indices can be compared bit for bit.
GAP = 1e-2


def scores(x_rows, wg, bias, k):
    """Selection scores l + bias in fp64 for the given token rows."""
    _, _, lg = router(x_rows, wg, bias, k, return_logits=True)
    return lg + (0.0 if bias is None else np.asarray(bias, np.float64))


def gap_violations(s, k, delta=GAP):
    """Rows whose top-(k+1) scores have a consecutive gap below delta."""
    E = s.shape[1]
    m = min(k + 1, E)
    if m < 2:
        return np.zeros(s.shape[0], bool)
    top = -np.sort(-s, axis=1)[:, :m]
    return (np.diff(-top, axis=1) < delta).any(axis=1)


def gap_redraw(w, delta=GAP, max_rounds=200):
    """Per-token substream index for workload ``w`` (a moe_inputs.Workload) such that every
    token's router scores keep the minimum gap; a violating token row is redrawn from the next
    substream of x, deterministically."""
    import moe_inputs as mi

    wg = mi.host_wg(w)
    bias = mi.bias_f32(w)
    redraw = np.zeros(w.T, np.uint32)
    todo = np.arange(w.T)
    for _ in range(max_rounds):
        x = mi.host_x(w, rows=todo, redraw=redraw[todo])
        bad = gap_violations(scores(x, wg, bias, w.k), w.k, delta)
        if not bad.any():
            return redraw
        todo = todo[bad]
        redraw[todo] += 1
    raise RuntimeError("gap enforcement did not converge")
