// router_topk.cu -- step 1 of the layer, second half: top-k and softmax over the chosen k.
//
// josueisai.com "Mixture of experts", section "El router": a linear projection gives one score
// per expert, the k best are kept and the softmax is normalised over those k only.
// gotburnout.io glossary "MoE", section 2 item 4: a per-expert bias (aux-loss-free balancing)
// steers the selection; it is added to the scores for choosing, not to the weights.
//
// The projection itself (logits = x W_g^T, bf16 products accumulated in fp32) runs on the
// tensor cores in grouped_gemm_sm100.cu and leaves k_splits partial sums [k_splits][T][ld].
// Here one warp owns one token: lane l sums the partials of experts [l*EJ, l*EJ + EJ) in split
// order (deterministic), then k rounds of a warp arg-max over (logit + bias) pick the experts
// (ties -> lower expert id), and the chosen unbiased logits are normalised with expf in fp32.
#include <cfloat>
#include <climits>

#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;  // 8 tokens per block

template <int EJ>
__global__ void __launch_bounds__(kThreads) router_select_kernel(const float* __restrict__ part, int S, int T, int ld,
                                                                 const float* __restrict__ bias, int E, int k,
                                                                 int32_t* __restrict__ idx_out,
                                                                 float* __restrict__ w_out) {
  const int lane = threadIdx.x & 31;
  const int e0 = lane * EJ;
  pdl_wait();
  float bj[EJ];
#pragma unroll
  for (int j = 0; j < EJ; ++j) bj[j] = (bias != nullptr && e0 + j < E) ? bias[e0 + j] : 0.f;

  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += (gridDim.x * blockDim.x) >> 5) {
    float l[EJ];
#pragma unroll
    for (int j = 0; j < EJ; ++j) l[j] = 0.f;
    // split partials in split order; loads of up to 4 splits are issued before their adds
    const size_t split_stride = (size_t)T * ld;
    const float* row0 = part + (size_t)t * ld + e0;
    for (int s0 = 0; s0 < S; s0 += 4) {
      float v[4][EJ];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int j = 0; j < EJ; ++j)
          v[u][j] = (s0 + u < S && e0 + j < E) ? __ldg(row0 + (size_t)(s0 + u) * split_stride + j) : 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int j = 0; j < EJ; ++j) l[j] += v[u][j];
    }
    uint32_t taken = 0;
    int my_idx = -1;
    float my_l = 0.f;
    for (int j = 0; j < k; ++j) {
      // best remaining expert of this lane: highest score, lowest id on ties
      float bv = -FLT_MAX, bl = 0.f;
      int be = INT_MAX;
#pragma unroll
      for (int jj = 0; jj < EJ; ++jj) {
        const int e = e0 + jj;
        const float sv = l[jj] + bj[jj];
        if (e < E && !((taken >> jj) & 1u) && (be == INT_MAX || sv > bv)) bv = sv, be = e, bl = l[jj];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oe = __shfl_xor_sync(0xffffffffu, be, off);
        const float ol = __shfl_xor_sync(0xffffffffu, bl, off);
        if (oe != INT_MAX && (be == INT_MAX || ov > bv || (ov == bv && oe < be))) bv = ov, be = oe, bl = ol;
      }
      if (be / EJ == lane) taken |= 1u << (be % EJ);
      if (lane == j) my_idx = be, my_l = bl;
    }
    float m = lane < k ? my_l : -FLT_MAX;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float ex = lane < k ? expf(my_l - m) : 0.f;
    float z = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    if (lane < k) {
      idx_out[(size_t)t * k + lane] = my_idx;
      w_out[(size_t)t * k + lane] = ex / z;
    }
  }
  pdl_trigger();
}

template <int EJ>
cudaError_t launch(const float* part, int S, int T, int ld, const float* bias, int E, int k, int32_t* idx, float* w,
                   cudaStream_t s) {
  long long blocks = ((long long)T + 7) / 8;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  return launch_pdl(router_select_kernel<EJ>, dim3((unsigned)blocks), dim3(kThreads), 0, s, part, S, T, ld, bias, E,
                    k, idx, w);
}

}  // namespace

cudaError_t launch_router_select(const float* partials, int k_splits, int T, int ld, const float* bias, int E, int k,
                                 int32_t* idx, float* w, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (E <= 32) return launch<1>(partials, k_splits, T, ld, bias, E, k, idx, w, s);
  if (E <= 64) return launch<2>(partials, k_splits, T, ld, bias, E, k, idx, w, s);
  if (E <= 128) return launch<4>(partials, k_splits, T, ld, bias, E, k, idx, w, s);
  if (E <= 256) return launch<8>(partials, k_splits, T, ld, bias, E, k, idx, w, s);
  if (E <= 512) return launch<16>(partials, k_splits, T, ld, bias, E, k, idx, w, s);
  return launch<32>(partials, k_splits, T, ld, bias, E, k, idx, w, s);
}

}  // namespace moe
