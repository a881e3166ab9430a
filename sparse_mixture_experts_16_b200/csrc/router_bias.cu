// router_bias.cu -- aux-loss-free balancing: move each expert's selection bias towards balance.
//
// gotburnout.io glossary "MoE", section 2 item 4: the router's biases are adjusted dynamically
// so that no expert (and no GPU holding it) is overloaded.  The pages give no rule; the one
// taken here is the sign rule on the loads of the last batch,
//     bias_e <- bias_e + gamma * sign(mean(load) - load_e),
// with load_e = counts[e] (slots routed to e, as produced by the dispatch step).  The comparison
// with the mean is exact in integers: sign(sum(load) - E * load_e).  One block of 1024 threads
// (E <= 1024): a block-wide 64-bit sum, then one fp32 add per expert.
#include "moe_common.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(1024) update_bias_kernel(const int32_t* __restrict__ counts, int E, float gamma,
                                                           float* __restrict__ bias) {
  __shared__ long long warp_sum[32];
  __shared__ long long total_s;
  pdl_wait();
  const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
  const long long c = e < E ? (long long)counts[e] : 0;
  long long v = c;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  if (lane == 0) warp_sum[warp] = v;
  __syncthreads();
  if (warp == 0) {
    long long w = warp_sum[lane];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) w += __shfl_xor_sync(0xffffffffu, w, off);
    if (lane == 0) total_s = w;
  }
  __syncthreads();
  if (e < E) {
    const long long diff = total_s - (long long)E * c;
    const float step = diff > 0 ? gamma : (diff < 0 ? -gamma : 0.0f);
    bias[e] = __fadd_rn(bias[e], step);
  }
  pdl_trigger();
}

}  // namespace

cudaError_t launch_update_bias(const int32_t* counts, int E, float gamma, float* bias, cudaStream_t s) {
  return launch_pdl(update_bias_kernel, dim3(1), dim3(1024), 0, s, counts, E, gamma, bias);
}

}  // namespace moe
