// router_topk.cu -- step 1 of the layer: router projection, top-k, softmax over the chosen k.
//
// josueisai.com "Mixture of experts", section "El router": a linear projection gives one score
// per expert, the k best are kept and the softmax is normalised over those k only.
// gotburnout.io glossary "MoE", section 2 item 4: a per-expert bias (aux-loss-free balancing)
// steers the selection; it is added to the scores for choosing, not to the weights.
//
// One fused kernel.  A block owns TT = 8*RT tokens and all E experts.  The D axis is walked in
// chunks of 32: the chunk of W_g (E x 32) and of x (TT x 32) is converted to fp32 in shared
// memory, W_g transposed so each lane reads its EJ consecutive experts with vector loads.  Each
// warp owns RT tokens; lane l accumulates experts [l*EJ, l*EJ + EJ) in fp32 registers.  Top-k is
// then a k-round warp arg-max over those registers (ties -> lower expert id), and the k chosen
// unbiased logits are normalised with expf in fp32.
#include <cfloat>
#include <climits>

#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kDC = 32;       // D chunk
constexpr int kThreads = 256; // 8 warps

template <int EJ>
__device__ __forceinline__ void load_row(const float* p, float (&w)[EJ]) {
  if constexpr (EJ % 4 == 0) {
#pragma unroll
    for (int q = 0; q < EJ / 4; ++q) {
      float4 v = reinterpret_cast<const float4*>(p)[q];
      w[4 * q] = v.x, w[4 * q + 1] = v.y, w[4 * q + 2] = v.z, w[4 * q + 3] = v.w;
    }
  } else if constexpr (EJ == 2) {
    float2 v = *reinterpret_cast<const float2*>(p);
    w[0] = v.x, w[1] = v.y;
  } else {
    w[0] = p[0];
  }
}

template <int EJ, int RT>
__global__ void __launch_bounds__(kThreads) router_topk_kernel(const uint16_t* __restrict__ x,
                                                               const uint16_t* __restrict__ wg,
                                                               const float* __restrict__ bias, int T, int D,
                                                               int E, int k, int32_t* __restrict__ idx_out,
                                                               float* __restrict__ w_out, int* err_clear) {
  constexpr int EP = 32 * EJ;  // padded expert count
  constexpr int TT = 8 * RT;   // tokens per block
  extern __shared__ __align__(16) float sm[];
  float* ws = sm;              // [kDC][EP]   (W_g chunk, transposed)
  float* xs = sm + kDC * EP;   // [TT][kDC]

  if (err_clear != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *err_clear = 0;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * TT;

  float acc[RT][EJ];
#pragma unroll
  for (int r = 0; r < RT; ++r)
#pragma unroll
    for (int j = 0; j < EJ; ++j) acc[r][j] = 0.f;

  for (int d0 = 0; d0 < D; d0 += kDC) {
    for (int v = threadIdx.x; v < EP * 4; v += kThreads) {
      const int e = v >> 2, c = (v & 3) * 8;
      uint4 q = make_uint4(0, 0, 0, 0);
      if (e < E) q = __ldg(reinterpret_cast<const uint4*>(wg + (size_t)e * D + d0 + c));
      const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        ws[(c + 2 * i) * EP + e] = bf16_lo(w4[i]);
        ws[(c + 2 * i + 1) * EP + e] = bf16_hi(w4[i]);
      }
    }
    for (int v = threadIdx.x; v < TT * 4; v += kThreads) {
      const int r = v >> 2, c = (v & 3) * 8, t = t0 + r;
      uint4 q = make_uint4(0, 0, 0, 0);
      if (t < T) q = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * D + d0 + c));
      float4* dst = reinterpret_cast<float4*>(xs + r * kDC + c);
      dst[0] = make_float4(bf16_lo(q.x), bf16_hi(q.x), bf16_lo(q.y), bf16_hi(q.y));
      dst[1] = make_float4(bf16_lo(q.z), bf16_hi(q.z), bf16_lo(q.w), bf16_hi(q.w));
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kDC; ++kk) {
      float xv[RT], wv[EJ];
#pragma unroll
      for (int r = 0; r < RT; ++r) xv[r] = xs[(warp * RT + r) * kDC + kk];
      load_row<EJ>(ws + kk * EP + lane * EJ, wv);
#pragma unroll
      for (int r = 0; r < RT; ++r)
#pragma unroll
        for (int j = 0; j < EJ; ++j) acc[r][j] = fmaf(xv[r], wv[j], acc[r][j]);
    }
    __syncthreads();
  }

  float bj[EJ];
#pragma unroll
  for (int j = 0; j < EJ; ++j) {
    const int e = lane * EJ + j;
    bj[j] = (bias != nullptr && e < E) ? bias[e] : 0.f;
  }

#pragma unroll
  for (int r = 0; r < RT; ++r) {
    const int t = t0 + warp * RT + r;
    if (t >= T) break;  // warp-uniform
    uint32_t taken = 0;
    int my_idx = -1;
    float my_l = 0.f;
    for (int j = 0; j < k; ++j) {
      // best remaining expert of this lane: highest score, lowest id on ties
      float bv = -FLT_MAX, bl = 0.f;
      int be = INT_MAX;
#pragma unroll
      for (int jj = 0; jj < EJ; ++jj) {
        const int e = lane * EJ + jj;
        const float sv = acc[r][jj] + bj[jj];
        if (e < E && !((taken >> jj) & 1u) && (be == INT_MAX || sv > bv)) bv = sv, be = e, bl = acc[r][jj];
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
}

template <int EJ, int RT>
cudaError_t launch(const uint16_t* x, const uint16_t* wg, const float* bias, int T, int D, int E, int k,
                   int32_t* idx, float* w, int* err_clear, cudaStream_t s) {
  constexpr int TT = 8 * RT;
  const size_t smem = (size_t)(kDC * 32 * EJ + TT * kDC) * sizeof(float);
  static bool configured = false;  // idempotent attribute set
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(router_topk_kernel<EJ, RT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int blocks = (T + TT - 1) / TT;
  router_topk_kernel<EJ, RT><<<blocks, kThreads, smem, s>>>(x, wg, bias, T, D, E, k, idx, w, err_clear);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_topk(const uint16_t* x, const uint16_t* wg, const float* bias, int T, int D, int E,
                               int k, int32_t* idx, float* w, int* err_clear, cudaStream_t s) {
  if (T == 0) {
    if (err_clear) return cudaMemsetAsync(err_clear, 0, sizeof(int), s);
    return cudaSuccess;
  }
  if (E <= 32) return launch<1, 4>(x, wg, bias, T, D, E, k, idx, w, err_clear, s);
  if (E <= 64) return launch<2, 4>(x, wg, bias, T, D, E, k, idx, w, err_clear, s);
  if (E <= 128) return launch<4, 4>(x, wg, bias, T, D, E, k, idx, w, err_clear, s);
  if (E <= 256) return launch<8, 4>(x, wg, bias, T, D, E, k, idx, w, err_clear, s);
  if (E <= 512) return launch<16, 2>(x, wg, bias, T, D, E, k, idx, w, err_clear, s);
  return launch<32, 1>(x, wg, bias, T, D, E, k, idx, w, err_clear, s);
}

}  // namespace moe
