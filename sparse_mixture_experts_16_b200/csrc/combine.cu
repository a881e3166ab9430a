// combine.cu -- step 4 of the layer: weighted aggregation back to token order.
//
// gotburnout.io glossary "MoE", section 2 ("Weighted Aggregation: y = Sum(p_i * Expert_i(x))")
// and section 3 step 4: the selected experts' outputs, already multiplied by their normalised
// router weights in the down-projection epilogue, are summed per token; the always-on shared
// expert's output is added with weight 1.
//
// One warp per token row: the k row indices are loaded once and broadcast with shuffles, then
// every lane sums 8 bf16 columns at a time (16-byte loads) in fp32, in slot order j = 0..k-1.
#include "moe_common.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ out_perm,
                                                      const int32_t* __restrict__ inv_perm,
                                                      const uint16_t* __restrict__ shared_out, int T, int D, int k,
                                                      uint16_t* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int nv = D / 8;
  const long long M = (long long)T * k;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += (gridDim.x * blockDim.x) >> 5) {
    const int my_row = lane < k ? inv_perm[(size_t)t * k + lane] : -1;
    for (int v = lane; v < nv; v += 32) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int j = 0; j < k; ++j) {
        const int r = __shfl_sync(0xffffffffu, my_row, j);
        if (r < 0 || r >= M) continue;
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(out_perm + (size_t)r * D) + v);
        acc[0] += bf16_lo(q.x), acc[1] += bf16_hi(q.x), acc[2] += bf16_lo(q.y), acc[3] += bf16_hi(q.y);
        acc[4] += bf16_lo(q.z), acc[5] += bf16_hi(q.z), acc[6] += bf16_lo(q.w), acc[7] += bf16_hi(q.w);
      }
      if (shared_out != nullptr) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(shared_out + (size_t)t * D) + v);
        acc[0] += bf16_lo(q.x), acc[1] += bf16_hi(q.x), acc[2] += bf16_lo(q.y), acc[3] += bf16_hi(q.y);
        acc[4] += bf16_lo(q.z), acc[5] += bf16_hi(q.z), acc[6] += bf16_lo(q.w), acc[7] += bf16_hi(q.w);
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      reinterpret_cast<uint4*>(y + (size_t)t * D)[v] = o;
    }
  }
}

}  // namespace

cudaError_t launch_combine(const uint16_t* out_perm, const int32_t* inv_perm, const uint16_t* shared_out, int T,
                           int D, int k, uint16_t* y, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  long long blocks = ((long long)T + 7) / 8;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  combine_kernel<<<(unsigned)blocks, 256, 0, s>>>(out_perm, inv_perm, shared_out, T, D, k, y);
  return cudaGetLastError();
}

}  // namespace moe
