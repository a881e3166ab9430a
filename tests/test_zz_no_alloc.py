"""moe_permute_noalloc: the dispatch entry point for callers that cannot allocate device memory.

Such callers (whose device memory is owned by an engine's own pools, or a plugin without access
to its host program's allocator) cannot hand moe_permute a workspace; this entry point keeps its
scratch in a fixed array inside the library instead.  Its outputs must equal moe_permute's bit
for bit (integer and copy work), on two calls in a row -- the second call sees the array as the
first call left it -- and equal the oracle's stable counting sort, so that a mistake the two GPU
entry points share cannot pass.  This file runs last so that a stop-at-first-failure run has
already run every other test; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest

import moe_inputs as mi
import oracle
import sparse_mixture_experts_16_b200 as moe

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L(cuda_device):
    from sparse_mixture_experts_16_b200 import build

    build.build()
    return moe.lib()


def _inputs(T, E, k, D, seed):
    import torch

    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    wts = rng.random((T, k)).astype(np.float32)
    x = mi.rows_bf16(mi.STREAM_X, np.arange(T), D, 1.0, seed=seed)
    x_t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(idx).cuda(), torch.from_numpy(wts).cuda(), x_t


def _noalloc(L, idx, wts, x, E):
    import torch

    T, k = idx.shape
    D = x.shape[1]
    dev = idx.device
    out = dict(counts=torch.full((E,), -7, dtype=torch.int32, device=dev),
               offsets=torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
               perm_token=torch.full((T * k,), -7, dtype=torch.int32, device=dev),
               inv_perm=torch.full((T * k,), -7, dtype=torch.int32, device=dev),
               p_perm=torch.full((T * k,), -7.0, dtype=torch.float32, device=dev),
               x_perm=torch.zeros(T * k, D, dtype=torch.bfloat16, device=dev))
    st = L.moe_permute_noalloc(idx.data_ptr(), wts.data_ptr(), x.data_ptr(), T, D, E, k, out["counts"].data_ptr(),
                               out["offsets"].data_ptr(), out["perm_token"].data_ptr(), out["inv_perm"].data_ptr(),
                               out["p_perm"].data_ptr(), out["x_perm"].data_ptr(),
                               torch.cuda.current_stream().cuda_stream)
    assert st == 0, moe.STATUS.get(st)
    return out


def _check_against_oracle(got, idx, wts, x, E):
    """counts, offsets, perm_token, inv_perm bit-exact against the oracle's stable counting sort;
    p_perm and x_perm are the routed weight and token row of each permuted slot."""
    import torch

    idx_h, w_h = idx.cpu().numpy(), wts.cpu().numpy()
    counts, offsets, pt, ps, inv = oracle.permute(idx_h, E)
    assert (got["counts"].cpu().numpy() == counts).all()
    assert (got["offsets"].cpu().numpy() == offsets).all()
    assert (got["perm_token"].cpu().numpy() == pt).all()
    assert (got["inv_perm"].cpu().numpy() == inv).all()
    assert (got["p_perm"].cpu().numpy() == w_h[pt, ps]).all()
    x_h = x.view(torch.int16).cpu().numpy()
    assert (got["x_perm"].view(torch.int16).cpu().numpy() == x_h[pt]).all()


# (T, E, k, D, seed): multi-block counting (T > 256) first, filling more of the shared array than
# the calls after it read; then the one-kernel dispatch of T <= 256 and a single token
CASES = [(3000, 64, 4, 128, 1), (777, 33, 3, 192, 2), (200, 16, 4, 128, 3), (1, 8, 2, 64, 4)]


def test_noalloc_permute_matches_workspace_permute_on_two_calls_in_a_row(L):
    import torch

    for (T, E, k, D, seed) in CASES:
        idx, wts, x = _inputs(T, E, k, D, seed)
        ref = moe.moe_permute(idx, wts, x, E)
        got = _noalloc(L, idx, wts, x, E)
        torch.cuda.synchronize()
        for name in ("counts", "offsets", "perm_token", "inv_perm", "p_perm"):
            assert torch.equal(got[name], ref[name]), name
        assert torch.equal(got["x_perm"].view(torch.int16), ref["x_perm"].view(torch.int16))


def test_noalloc_permute_matches_the_oracle(L):
    import torch

    for (T, E, k, D, seed) in CASES:
        idx, wts, x = _inputs(T, E, k, D, seed)
        got = _noalloc(L, idx, wts, x, E)
        torch.cuda.synchronize()
        _check_against_oracle(got, idx, wts, x, E)


def test_noalloc_permute_rejects_sizes_beyond_its_fixed_scratch(L):
    # ceil(T/256) * E must fit in 131072 counts: E = 1024 allows T <= 32768
    args = (0x1000, 0x2000, None, 32769, 64, 1024, 2, 0x3000, 0x4000, 0x5000, 0x6000, 0x7000, None, None)
    assert L.moe_permute_noalloc(*args) == 4  # MOE_ERR_WORKSPACE_TOO_SMALL, nothing launched
