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
//                       32-token chunks of x and dl staged in shared memory, tokens in order; when
//                       that gives too few blocks, the tokens are split and aux_sum_splits_kernel
//                       adds the partial sums in split order;
//   aux_dx_kernel       dx[t, d] = sum_e dl[t, e] W_g[e, d], 16 tokens x 256 columns per block,
//                       32-expert chunks of W_g and dl staged in shared memory, experts in order.
#include <cfloat>

#include "moe_common.cuh"
#include "router_aux.cuh"

namespace moe {
namespace {

constexpr int kAuxThreads = 256;
constexpr int kAuxRows = 16;   // experts (dW_g) or tokens (dx) per block
constexpr int kAuxCols = 256;  // columns of D per block
constexpr int kAuxChunk = 32;  // tokens (dW_g) or experts (dx) staged per step
constexpr int kAuxMaxSplits = 16;

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

// dW_g over the tokens of split blockIdx.z: x [32 tokens][256 columns] and dl [32 tokens][16
// experts] are staged in shared memory, then each thread adds 32 tokens x 16 experts for its
// column.  With one split the block writes dW_g; otherwise partials [split][E][D].
__global__ void __launch_bounds__(kAuxThreads) aux_dwg_kernel(const float* __restrict__ dl,
                                                              const uint16_t* __restrict__ x, int T, int D, int E,
                                                              int t_per, float* __restrict__ out) {
  __shared__ __align__(16) uint16_t sx[kAuxChunk][kAuxCols];
  __shared__ float sd[kAuxChunk][kAuxRows];
  const int e0 = blockIdx.x * kAuxRows, d0 = blockIdx.y * kAuxCols;
  const int d = d0 + threadIdx.x;
  const int ne = min(kAuxRows, E - e0);
  const int tb = blockIdx.z * t_per, te = min(T, tb + t_per);
  pdl_wait();
  float acc[kAuxRows];
#pragma unroll
  for (int j = 0; j < kAuxRows; ++j) acc[j] = 0.f;
  for (int tc = tb; tc < te; tc += kAuxChunk) {
    const int nt = min(kAuxChunk, te - tc);
    __syncthreads();  // the previous chunk's readers are done
    for (int i = threadIdx.x; i < kAuxChunk * (kAuxCols / 8); i += kAuxThreads) {
      const int r = i / (kAuxCols / 8), c = (i % (kAuxCols / 8)) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < nt && d0 + c < D) v = *reinterpret_cast<const uint4*>(x + (size_t)(tc + r) * D + d0 + c);
      *reinterpret_cast<uint4*>(&sx[r][c]) = v;
    }
    for (int i = threadIdx.x; i < kAuxChunk * kAuxRows; i += kAuxThreads) {
      const int r = i / kAuxRows, j = i % kAuxRows;
      sd[r][j] = (r < nt && j < ne) ? dl[(size_t)(tc + r) * E + e0 + j] : 0.f;
    }
    __syncthreads();
    for (int r = 0; r < nt; ++r) {
      const float xv = __uint_as_float((uint32_t)sx[r][threadIdx.x] << 16);
#pragma unroll
      for (int j = 0; j < kAuxRows; ++j) acc[j] = fmaf(sd[r][j], xv, acc[j]);
    }
  }
  if (d < D) {
    float* o = out + (size_t)blockIdx.z * E * D;
#pragma unroll
    for (int j = 0; j < kAuxRows; ++j)
      if (j < ne) o[(size_t)(e0 + j) * D + d] = acc[j];
  }
  pdl_trigger();
}

// out[i] = sum over splits s = 0, 1, ... of part[s][i], in that order
__global__ void aux_sum_splits_kernel(const float* __restrict__ part, int S, long long n, float* __restrict__ out) {
  pdl_wait();
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    float acc = 0.f;
    for (int sp = 0; sp < S; ++sp) acc += part[(size_t)sp * n + i];
    out[i] = acc;
  }
  pdl_trigger();
}

// dx for 16 tokens x 256 columns: W_g [32 experts][256 columns] and dl [16 tokens][32 experts] are
// staged in shared memory, experts in order.
__global__ void __launch_bounds__(kAuxThreads) aux_dx_kernel(const float* __restrict__ dl,
                                                             const uint16_t* __restrict__ wg, int T, int D, int E,
                                                             float* __restrict__ dx) {
  __shared__ __align__(16) uint16_t sw[kAuxChunk][kAuxCols];
  __shared__ float sdl[kAuxRows][kAuxChunk];
  const int t0 = blockIdx.x * kAuxRows, d0 = blockIdx.y * kAuxCols;
  const int d = d0 + threadIdx.x;
  const int nt = min(kAuxRows, T - t0);
  pdl_wait();
  float acc[kAuxRows];
#pragma unroll
  for (int j = 0; j < kAuxRows; ++j) acc[j] = 0.f;
  for (int ec = 0; ec < E; ec += kAuxChunk) {
    const int ne = min(kAuxChunk, E - ec);
    __syncthreads();  // the previous chunk's readers are done
    for (int i = threadIdx.x; i < kAuxChunk * (kAuxCols / 8); i += kAuxThreads) {
      const int r = i / (kAuxCols / 8), c = (i % (kAuxCols / 8)) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < ne && d0 + c < D) v = *reinterpret_cast<const uint4*>(wg + (size_t)(ec + r) * D + d0 + c);
      *reinterpret_cast<uint4*>(&sw[r][c]) = v;
    }
    for (int i = threadIdx.x; i < kAuxRows * kAuxChunk; i += kAuxThreads) {
      const int j = i / kAuxChunk, e = i % kAuxChunk;
      sdl[j][e] = (j < nt && e < ne) ? dl[(size_t)(t0 + j) * E + ec + e] : 0.f;
    }
    __syncthreads();
    for (int e = 0; e < ne; ++e) {
      const float wv = __uint_as_float((uint32_t)sw[e][threadIdx.x] << 16);
#pragma unroll
      for (int j = 0; j < kAuxRows; ++j) acc[j] = fmaf(sdl[j][e], wv, acc[j]);
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

int aux_token_splits(int T, int D, int E) {
  const long long tiles = (long long)((E + kAuxRows - 1) / kAuxRows) * ((D + kAuxCols - 1) / kAuxCols);
  long long S = (2 * 148 + tiles - 1) / tiles;  // about two blocks per SM
  const long long chunks = ((long long)T + kAuxChunk - 1) / kAuxChunk;
  if (S > kAuxMaxSplits) S = kAuxMaxSplits;
  if (S > chunks) S = chunks;
  return S < 1 ? 1 : (int)S;
}

cudaError_t launch_router_aux(const float* partials, int S_router, int ld, const int32_t* idx, const uint16_t* x,
                              const uint16_t* w_gate, int T, int D, int E, int k, float alpha, int32_t* counts,
                              float* c, float* dl, float* split_part, float* loss, float* dw_gate, float* dx,
                              cudaStream_t s) {
  if (T <= 0 || E <= 0 || E > 1024 || k <= 0) return cudaErrorInvalidValue;
  const long long slots = (long long)T * k;
  long long cb = (slots + 255) / 256;
  if (cb > 148LL * 8) cb = 148LL * 8;
  cudaError_t e = launch_pdl(aux_count_kernel, dim3((unsigned)cb), dim3(256), 0, s, idx, slots, E, counts);
  if (e != cudaSuccess) return e;
  const float scale = alpha * (float)E / (float)T;
  if (E <= 32) e = launch_softmax<1>(partials, S_router, T, ld, counts, E, k, scale, c, dl, s);
  else if (E <= 64) e = launch_softmax<2>(partials, S_router, T, ld, counts, E, k, scale, c, dl, s);
  else if (E <= 128) e = launch_softmax<4>(partials, S_router, T, ld, counts, E, k, scale, c, dl, s);
  else if (E <= 256) e = launch_softmax<8>(partials, S_router, T, ld, counts, E, k, scale, c, dl, s);
  else if (E <= 512) e = launch_softmax<16>(partials, S_router, T, ld, counts, E, k, scale, c, dl, s);
  else e = launch_softmax<32>(partials, S_router, T, ld, counts, E, k, scale, c, dl, s);
  if (e != cudaSuccess) return e;
  e = launch_pdl(aux_loss_kernel, dim3(1), dim3(1024), 0, s, (const float*)c, T, scale, loss);
  if (e != cudaSuccess) return e;
  const unsigned dcols = (unsigned)((D + kAuxCols - 1) / kAuxCols);
  const int S = aux_token_splits(T, D, E);
  const int t_per = (T + S - 1) / S;
  e = launch_pdl(aux_dwg_kernel, dim3((unsigned)((E + kAuxRows - 1) / kAuxRows), dcols, (unsigned)S),
                 dim3(kAuxThreads), 0, s, (const float*)dl, x, T, D, E, t_per, S > 1 ? split_part : dw_gate);
  if (e != cudaSuccess) return e;
  if (S > 1) {
    const long long n = (long long)E * D;
    long long blocks = (n + 255) / 256;
    if (blocks > 148LL * 8) blocks = 148LL * 8;
    e = launch_pdl(aux_sum_splits_kernel, dim3((unsigned)blocks), dim3(256), 0, s, (const float*)split_part, S, n,
                   dw_gate);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(aux_dx_kernel, dim3((unsigned)((T + kAuxRows - 1) / kAuxRows), dcols), dim3(kAuxThreads), 0, s,
                    (const float*)dl, w_gate, T, D, E, dx);
}

}  // namespace moe
