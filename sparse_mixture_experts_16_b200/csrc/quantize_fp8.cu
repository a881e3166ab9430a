// quantize_fp8.cu -- per-row E4M3 quantisation of packed expert weights.
//
// keryc.com "Mixture of Experts optimiza Transformers y LLMs", section "Resultados practicos":
// once the experts are packed, the conversion pipeline can quantise them per expert.  Here each
// row of a packed weight tensor (one output feature of one expert) gets its own fp32 scale
//     s = amax(|row|) / 448        (1 for an all-zero row)
// and codes q = E4M3(w / s), round to nearest even, saturating at +-448 (448 is E4M3's largest
// finite value).  The weight-streaming GEMM kernels read the codes and apply s in their epilogue.
//
// One warp per row: 16-byte loads of 8 bf16, a warp max, then w / s in fp32 (IEEE division) and
// CUDA's saturating fp32 -> E4M3 pair conversion; 8-byte stores of 8 codes.
#include <cuda_fp8.h>

#include "moe_common.cuh"

namespace moe {
namespace {

__global__ void __launch_bounds__(256) quantize_rows_fp8_kernel(const uint16_t* __restrict__ w, long long rows,
                                                                int K, uint8_t* __restrict__ q,
                                                                float* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int nv = K / 8;
  pdl_wait();
  for (long long r = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5; r < rows;
       r += ((long long)gridDim.x * blockDim.x) >> 5) {
    const uint4* src = reinterpret_cast<const uint4*>(w + r * K);
    float amax = 0.0f;
    for (int v = lane; v < nv; v += 32) {
      const uint4 u = __ldg(src + v);
      const uint32_t p[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(p[i])), fabsf(bf16_hi(p[i]))));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    const float s = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    if (lane == 0) scales[r] = s;
    uint2* dst = reinterpret_cast<uint2*>(q + r * K);
    for (int v = lane; v < nv; v += 32) {
      const uint4 u = __ldg(src + v);
      const uint32_t p[4] = {u.x, u.y, u.z, u.w};
      uint32_t out[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = make_float2(__fdiv_rn(bf16_lo(p[i]), s), __fdiv_rn(bf16_hi(p[i]), s));
        const uint32_t pair = (uint32_t)__nv_cvt_float2_to_fp8x2(f, __NV_SATFINITE, __NV_E4M3);  // .x -> low byte
        out[i >> 1] |= pair << (16 * (i & 1));
      }
      dst[v] = make_uint2(out[0], out[1]);
    }
  }
  pdl_trigger();
}

}  // namespace

cudaError_t launch_quantize_rows_fp8(const uint16_t* w, long long rows, int K, uint8_t* q, float* scales,
                                     cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  long long blocks = (rows + 7) / 8;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  return launch_pdl(quantize_rows_fp8_kernel, dim3((unsigned)blocks), dim3(256), 0, s, w, rows, K, q, scales);
}

}  // namespace moe
