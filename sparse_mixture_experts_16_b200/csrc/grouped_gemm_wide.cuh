// Token-wide grouped GEMMs for prefill (sm_100a): the expert FFN's gate_up (+ SwiGLU) and down
// products with the weights as the MMA's M operand (128 weight rows) and up to 256 tokens of one
// expert segment as N.  The ragged end of a segment then costs an MMA of N = its rows rounded up
// to 16, where the 128-token tiles of grouped_gemm_sm100.cu pay a full 128-row tile.
#pragma once

#include "moe_common.cuh"

namespace moe {

// Same operands and outputs as launch_grouped_gemm(kind, sets, n_sets, 0, ...): kGateUp writes
// h = silu(g) * u (bf16) and, when a set's save_gu is set, g | u (bf16); kDown writes fp32 rows
// scaled by row_scale (or unscaled).  K must be a multiple of 64; gate_up's n_out (F) a multiple
// of 64, down's n_out (D) a multiple of 32.
cudaError_t launch_grouped_gemm_wide(GemmKind kind, const GemmSetHost* sets, int n_sets, int* err, cudaStream_t s);

// The same products on token-wide tiles computed by clusters of two CTAs (one M = 256 MMA per
// tile, each CTA loading half of each operand): grouped_gemm_pair_sm100.cu.  Same contract.
cudaError_t launch_grouped_gemm_pair(GemmKind kind, const GemmSetHost* sets, int n_sets, int* err, cudaStream_t s);

}  // namespace moe
