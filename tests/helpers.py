"""Shared test helpers: workload preparation (gap-enforced inputs), host/device conversions and
the output tolerance."""
from __future__ import annotations

import numpy as np

import moe_inputs as mi
import oracle

from oracle import GAP, gap_redraw, gap_violations  # noqa: F401  (re-exported for the tests)

# Layer outputs: max |y_gpu - y_oracle| <= REL_RMS_TOL * RMS(y_oracle)  (bf16 weights and
# activations, fp32 accumulation).
REL_RMS_TOL = 2e-2

# Router weights: fp32 logits differ from the fp64 ones by ~u32 * sqrt(D) * |partial sums|
# (<= ~5e-5 for D = 7168, logits of std 8.5); a softmax weight moves by at most the largest
# logit error.  2e-4 keeps a 4x margin.
P_ATOL = 2e-4


def scores(w: mi.Workload, x_rows: np.ndarray, wg: np.ndarray, bias):
    return oracle.scores(x_rows, wg, bias, w.k)


def to_torch_bf16(a: np.ndarray, device="cuda"):
    import torch

    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def to_np_bf16(t) -> np.ndarray:
    import torch

    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_np_to_f64(a: np.ndarray) -> np.ndarray:
    return mi.bf16_to_f64(a)


def rel_rms_err(got: np.ndarray, ref: np.ndarray) -> float:
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref))) / max(rms, 1e-30)


def segment_edge_tokens(perm_token, offsets):
    """The tokens holding the first and the last row of every non-empty expert segment: the last
    row sits in the segment's ragged final tile, where a masking mistake would show."""
    toks = set()
    for e in range(len(offsets) - 1):
        if offsets[e + 1] > offsets[e]:
            toks.add(int(perm_token[offsets[e]]))
            toks.add(int(perm_token[offsets[e + 1] - 1]))
    return np.array(sorted(toks), dtype=np.int64)


def oracle_rows_chunked(w, x_rows, idx_rows, p_rows, chunk=16):
    """y of the given token rows by the layer's definition, sum_j p[t,j] Expert_{idx[t,j]}(x_t) +
    Shared(x_t), each term an oracle expert FFN in fp64; the experts' weights are generated
    ``chunk`` experts at a time (the DeepSeek-shaped layer's weights are 22.6 GB)."""
    from concurrent.futures import ThreadPoolExecutor

    T = len(x_rows)
    y = np.zeros((T, w.D), np.float64)
    used = sorted(set(idx_rows.reshape(-1).tolist()))
    jobs_of = {e: [(t, j) for t in range(T) for j in range(w.k) if idx_rows[t, j] == e] for e in used}
    with ThreadPoolExecutor(max_workers=oracle._nthreads()) as pool:
        for c0 in range(0, len(used), chunk):
            es = used[c0:c0 + chunk]
            gu = dict(zip(es, mi.host_gate_up(w, es)))
            dn = dict(zip(es, mi.host_down(w, es)))
            jobs = [(e, t, j) for e in es for (t, j) in jobs_of[e]]
            outs = pool.map(lambda a: oracle.expert_ffn(x_rows[a[1]], gu[a[0]], dn[a[0]]), jobs)
            for (e, t, j), o in zip(jobs, outs):
                y[t] += p_rows[t, j] * o
            del gu, dn
        if w.Fs:
            sgu, sdn = mi.host_shared(w)
            outs = pool.map(lambda t: oracle.expert_ffn(x_rows[t], sgu, sdn), range(T))
            for t, o in zip(range(T), outs):
                y[t] += o
    return y
