// Router load-balancing auxiliary loss (training): kernels in router_aux.cu.
#pragma once

#include "moe_common.cuh"

namespace moe {

// From the router's split-K partial logits [S_router][T][ld] (launch_router_gemm) and its top-k choices
// idx [T, k] (launch_router_select), with counts [E] zeroed beforehand:
//   counts[e] = routed slots of e;  c[t] = sum_e f_e s_{t,e};  dl [T, E] = the loss's logit gradient;
//   loss[0] = alpha E / T * sum_t c[t];  dw_gate [E, D] = dl^T x;  dx [T, D] = dl W_g  (all fp32,
//   overwritten).  Every sum runs in a fixed order, so results are deterministic.
// split_part: aux_token_splits(T, D, E) x E x D fp32 of scratch when that count is above 1 (dW_g
// is then summed over token splits, in split order), else unused.
int aux_token_splits(int T, int D, int E);
cudaError_t launch_router_aux(const float* partials, int S_router, int ld, const int32_t* idx, const uint16_t* x,
                              const uint16_t* w_gate, int T, int D, int E, int k, float alpha, int32_t* counts,
                              float* c, float* dl, float* split_part, float* loss, float* dw_gate, float* dx,
                              cudaStream_t s);

}  // namespace moe
