// combine.cu -- step 4 of the layer: weighted aggregation back to token order.
//
// gotburnout.io glossary "MoE", section 2 ("Weighted Aggregation: y = Sum(p_i * Expert_i(x))")
// and section 3 step 4: the selected experts' outputs, already multiplied by their normalised
// router weights in the down-projection epilogue (kept in fp32), are summed per token; the
// always-on shared expert's output is added with weight 1; y is rounded once to bf16.
//
// One warp per (token, 256-column chunk): the k row indices are loaded once and broadcast with
// shuffles; every lane sums its 8 fp32 columns (two 16-byte loads per row) in slot order.
#include "moe_common.cuh"

namespace moe {
namespace {

__device__ __forceinline__ void add8(float (&acc)[8], const float* src) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(src));
  const float4 b = __ldg(reinterpret_cast<const float4*>(src) + 1);
  acc[0] += a.x, acc[1] += a.y, acc[2] += a.z, acc[3] += a.w;
  acc[4] += b.x, acc[5] += b.y, acc[6] += b.z, acc[7] += b.w;
}

// One warp per (token, 256-column chunk): lane l sums columns [8l, 8l+8) of the chunk over the
// token's k rows (two 16-byte loads per row, all rows in flight at once), in slot order.
__global__ void __launch_bounds__(256) combine_kernel(const float* __restrict__ out_perm,
                                                      const int32_t* __restrict__ inv_perm,
                                                      const float* __restrict__ shared_out, int T, int D, int k,
                                                      uint16_t* __restrict__ y) {
  const int lane = threadIdx.x & 31;
  const int n_chunks = (D + 255) / 256;
  const long long M = (long long)T * k;
  const long long items = (long long)T * n_chunks;
  pdl_wait();
  for (long long it = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5; it < items;
       it += ((long long)gridDim.x * blockDim.x) >> 5) {
    const int t = (int)(it / n_chunks);
    const int col = (int)(it - (long long)t * n_chunks) * 256 + lane * 8;
    const int my_row = lane < k ? inv_perm[(size_t)t * k + lane] : -1;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
      const int r = __shfl_sync(0xffffffffu, my_row, j);
      if (col < D && r >= 0 && r < M) add8(acc, out_perm + (size_t)r * D + col);
    }
    if (col < D) {
      if (shared_out != nullptr) add8(acc, shared_out + (size_t)t * D + col);
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      *reinterpret_cast<uint4*>(y + (size_t)t * D + col) = o;
    }
  }
  pdl_trigger();
}

}  // namespace

cudaError_t launch_combine(const float* out_perm, const int32_t* inv_perm, const float* shared_out, int T, int D,
                           int k, uint16_t* y, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const long long warps = (long long)T * ((D + 255) / 256);
  long long blocks = (warps + 7) / 8;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  return launch_pdl(combine_kernel, dim3((unsigned)blocks), dim3(256), 0, s, out_perm, inv_perm, shared_out, T, D, k,
                    y);
}

}  // namespace moe
