// router_aux.cu -- the router's load-balancing auxiliary loss and its gradient (training).
//
// josueisai.com "Mixture of experts", section "El coste que la cifra bonita esconde": training a
// MoE adds an auxiliary loss that penalises uneven routing and pushes the router to use every
// expert alike (dev.smart-guide.co.kr, "Limitaciones y Cuidados": without it the router can
// collapse onto one expert).  No formula is printed; the reading taken is the product of each
// expert's load and its mean router probability,
//   L = alpha * E * sum_e f_e P_e,   f_e = (slots routed to e) / (T k),   P_e = mean_t softmax(l_t)_e,
// with the selection (top-k of l + bias) held fixed, so the gradient flows through P only:
//   dL/dl_{t,e} = (alpha E / T) s_{t,e} (f_e - c_t),   c_t = sum_j f_j s_{t,j},   s_t = softmax(l_t).
//
// Kernels (all fp32 on the CUDA cores, fixed summation orders):
//   aux_count_kernel    slot histogram of idx (integer atomics: exact);
//   aux_softmax_kernel  one warp per token: logits from the split partials in split order, the
//                       full softmax, c_t, and the row dl[t, :];
//   aux_loss_kernel     one block: sum_t c_t in a fixed tree, times alpha E / T;
//   aux_dwg_kernel      dW_g[e, d] = sum_t dl[t, e] x[t, d], 16 experts x 256 columns per block,
//                       tokens in order;
//   aux_dx_kernel       dx[t, d] = sum_e dl[t, e] W_g[e, d], 16 tokens x 256 columns per block,
//                       experts in order (dl staged in shared memory 256 experts at a time).
#include <cfloat>

#include "moe_common.cuh"
#include "router_aux.cuh"

namespace moe {
namespace {

constexpr int kAuxThreads = 256;
constexpr int kAuxRows = 16;   // experts (dW_g) or tokens (dx) per block
constexpr int kAuxCols = 256;  // columns of D per block

__global__ void aux_count_kernel(const int32_t* __restrict__ idx, long long n, int E, int32_t* __restrict__ counts) {
  pdl_wait();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int e = idx[i];
    if (e >= 0 && e < E) atomicAdd(&counts[e], 1);
  }
  pdl_trigger();
}

template <int EJ>
__global__ void __launch_bounds__(kAuxThreads) aux_softmax_kernel(const float* __restrict__ part, int S, int T, int ld,
                                                                  const int32_t* __restrict__ counts, int E, int k,
                                                                  float scale, float* __restrict__ c_out,
                                                                  float* __restrict__ dl) {
  const int lane = threadIdx.x & 31;
  const int e0 = lane * EJ;
  pdl_wait();
  float f[EJ];
  const float slots = (float)T * (float)k;
#pragma unroll
  for (int j = 0; j < EJ; ++j) f[j] = e0 + j < E ? (float)counts[e0 + j] / slots : 0.f;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += (gridDim.x * blockDim.x) >> 5) {
    float l[EJ];
#pragma unroll
    for (int j = 0; j < EJ; ++j) l[j] = 0.f;
    const size_t split_stride = (size_t)T * ld;
    const float* row0 = part + (size_t)t * ld + e0;
    for (int sp = 0; sp < S; ++sp)
#pragma unroll
      for (int j = 0; j < EJ; ++j)
        if (e0 + j < E) l[j] += __ldg(row0 + (size_t)sp * split_stride + j);
    float m = -FLT_MAX;
#pragma unroll
    for (int j = 0; j < EJ; ++j)
      if (e0 + j < E) m = fmaxf(m, l[j]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float ex[EJ], z = 0.f;
#pragma unroll
    for (int j = 0; j < EJ; ++j) {
      ex[j] = e0 + j < E ? expf(l[j] - m) : 0.f;
      z += ex[j];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    float c = 0.f;
#pragma unroll
    for (int j = 0; j < EJ; ++j) {
      ex[j] /= z;  // s_{t,e}
      c += f[j] * ex[j];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
    float* drow = dl + (size_t)t * E + e0;
#pragma unroll
    for (int j = 0; j < EJ; ++j)
      if (e0 + j < E) drow[j] = scale * ex[j] * (f[j] - c);
    if (lane == 0) c_out[t] = c;
  }
  pdl_trigger();
}

__global__ void __launch_bounds__(1024) aux_loss_kernel(const float* __restrict__ c, int T, float scale,
                                                        float* __restrict__ loss) {
  __shared__ float part[1024];
  pdl_wait();
  float acc = 0.f;
  for (int t = threadIdx.x; t < T; t += 1024) acc += c[t];
  part[threadIdx.x] = acc;
  __syncthreads();
  for (int h = 512; h > 0; h >>= 1) {
    if ((int)threadIdx.x < h) part[threadIdx.x] += part[threadIdx.x + h];
    __syncthreads();
  }
  if (threadIdx.x == 0) loss[0] = scale * part[0];
  pdl_trigger();
}

__global__ void __launch_bounds__(kAuxThreads) aux_dwg_kernel(const float* __restrict__ dl,
                                                              const uint16_t* __restrict__ x, int T, int D, int E,
                                                              float* __restrict__ dwg) {
  const int e0 = blockIdx.x * kAuxRows;
  const int d = blockIdx.y * kAuxCols + threadIdx.x;
  const int ne = min(kAuxRows, E - e0);
  pdl_wait();
  float acc[kAuxRows];
#pragma unroll
  for (int j = 0; j < kAuxRows; ++j) acc[j] = 0.f;
  if (d < D) {
    for (int t = 0; t < T; ++t) {
      const float xv = __uint_as_float((uint32_t)x[(size_t)t * D + d] << 16);
      const float* drow = dl + (size_t)t * E + e0;
#pragma unroll
      for (int j = 0; j < kAuxRows; ++j)
        if (j < ne) acc[j] = fmaf(__ldg(drow + j), xv, acc[j]);
    }
#pragma unroll
    for (int j = 0; j < kAuxRows; ++j)
      if (j < ne) dwg[(size_t)(e0 + j) * D + d] = acc[j];
  }
  pdl_trigger();
}

__global__ void __launch_bounds__(kAuxThreads) aux_dx_kernel(const float* __restrict__ dl,
                                                             const uint16_t* __restrict__ wg, int T, int D, int E,
                                                             float* __restrict__ dx) {
  __shared__ float sdl[kAuxRows][kAuxCols];  // dl[t0 + j][ec + i]
  const int t0 = blockIdx.x * kAuxRows;
  const int d = blockIdx.y * kAuxCols + threadIdx.x;
  const int nt = min(kAuxRows, T - t0);
  pdl_wait();
  float acc[kAuxRows];
#pragma unroll
  for (int j = 0; j < kAuxRows; ++j) acc[j] = 0.f;
  for (int ec = 0; ec < E; ec += kAuxCols) {
    const int ne = min(kAuxCols, E - ec);
    __syncthreads();  // the previous chunk's readers are done
    for (int i = threadIdx.x; i < kAuxRows * kAuxCols; i += kAuxThreads) {
      const int j = i / kAuxCols, e = i % kAuxCols;
      sdl[j][e] = (j < nt && e < ne) ? dl[(size_t)(t0 + j) * E + ec + e] : 0.f;
    }
    __syncthreads();
    if (d < D) {
      for (int e = 0; e < ne; ++e) {
        const float wv = __uint_as_float((uint32_t)wg[(size_t)(ec + e) * D + d] << 16);
#pragma unroll
        for (int j = 0; j < kAuxRows; ++j) acc[j] = fmaf(sdl[j][e], wv, acc[j]);
      }
    }
  }
  if (d < D) {
#pragma unroll
    for (int j = 0; j < kAuxRows; ++j)
      if (j < nt) dx[(size_t)(t0 + j) * D + d] = acc[j];
  }
  pdl_trigger();
}

template <int EJ>
cudaError_t launch_softmax(const float* part, int S, int T, int ld, const int32_t* counts, int E, int k, float scale,
                           float* c, float* dl, cudaStream_t s) {
  long long blocks = ((long long)T + 7) / 8;
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  return launch_pdl(aux_softmax_kernel<EJ>, dim3((unsigned)blocks), dim3(kAuxThreads), 0, s, part, S, T, ld, counts, E,
                    k, scale, c, dl);
}

}  // namespace

cudaError_t launch_router_aux(const float* partials, int S, int ld, const int32_t* idx, const uint16_t* x,
                              const uint16_t* w_gate, int T, int D, int E, int k, float alpha, int32_t* counts,
                              float* c, float* dl, float* loss, float* dw_gate, float* dx, cudaStream_t s) {
  if (T <= 0 || E <= 0 || E > 1024 || k <= 0) return cudaErrorInvalidValue;
  const long long slots = (long long)T * k;
  long long cb = (slots + 255) / 256;
  if (cb > 148LL * 8) cb = 148LL * 8;
  cudaError_t e = launch_pdl(aux_count_kernel, dim3((unsigned)cb), dim3(256), 0, s, idx, slots, E, counts);
  if (e != cudaSuccess) return e;
  const float scale = alpha * (float)E / (float)T;
  if (E <= 32) e = launch_softmax<1>(partials, S, T, ld, counts, E, k, scale, c, dl, s);
  else if (E <= 64) e = launch_softmax<2>(partials, S, T, ld, counts, E, k, scale, c, dl, s);
  else if (E <= 128) e = launch_softmax<4>(partials, S, T, ld, counts, E, k, scale, c, dl, s);
  else if (E <= 256) e = launch_softmax<8>(partials, S, T, ld, counts, E, k, scale, c, dl, s);
  else if (E <= 512) e = launch_softmax<16>(partials, S, T, ld, counts, E, k, scale, c, dl, s);
  else e = launch_softmax<32>(partials, S, T, ld, counts, E, k, scale, c, dl, s);
  if (e != cudaSuccess) return e;
  e = launch_pdl(aux_loss_kernel, dim3(1), dim3(1024), 0, s, (const float*)c, T, scale, loss);
  if (e != cudaSuccess) return e;
  const unsigned dcols = (unsigned)((D + kAuxCols - 1) / kAuxCols);
  e = launch_pdl(aux_dwg_kernel, dim3((unsigned)((E + kAuxRows - 1) / kAuxRows), dcols), dim3(kAuxThreads), 0, s,
                 (const float*)dl, x, T, D, E, dw_gate);
  if (e != cudaSuccess) return e;
  return launch_pdl(aux_dx_kernel, dim3((unsigned)((T + kAuxRows - 1) / kAuxRows), dcols), dim3(kAuxThreads), 0, s,
                    (const float*)dl, w_gate, T, D, E, dx);
}

}  // namespace moe
