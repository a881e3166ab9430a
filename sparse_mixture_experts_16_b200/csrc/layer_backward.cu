// layer_backward.cu -- the CUDA-core steps of the layer's backward pass (the grouped GEMMs are in
// grouped_gemm_bwd_sm100.cu).
//
// keryc.com "Mixture of Experts optimiza...", section "Entrenamiento: todavia desafiante, pero con
// avances": MoE layers are trained.  The pages print no backward formulas; these are the chain rule
// of the forward (L = sum(dy * y)):
//   slot (t, j), expert e, row r of the expert-contiguous order, p = p_perm[r]:
//     dO_r = p * dy_t,                    dp_r = dy_t . o_r = sum_f (dy_t Down_e)_f h_rf
//     dl_r = p (dp_r - sum_i p_i dp_i)    (softmax over the token's chosen k)
//     dx_t = sum_j dX_{r_j} + dX_shared,t + sum_j dl_{r_j} W_g[idx_j]
//     dW_g[e] = sum_{r in e} dl_r x_perm_r
// The selection (top-k) and its bias carry no gradient.
//
// Layout: dy_perm, dO and dGU use a per-expert layout padded to multiples of 64 rows; the pad rows
// are zero, so the weight-gradient GEMMs (K = rows) may run over whole 64-row blocks.
#include "moe_common.cuh"

namespace moe {
namespace {

// pad_offsets[e] = sum over e' < e of round_up(rows(e'), 64); pad_offsets[E] = total.  One block.
__global__ void __launch_bounds__(1024) pad_offsets_kernel(const int32_t* __restrict__ offsets, int E,
                                                           int32_t* __restrict__ pad_offsets) {
  __shared__ int warp_tot[32];
  pdl_wait();
  const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
  const int v = e < E ? ((offsets[e + 1] - offsets[e] + 63) / 64) * 64 : 0;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tot[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += y;
    }
    warp_tot[lane] = w;
  }
  __syncthreads();
  if (warp > 0) incl += warp_tot[warp - 1];
  if (e < E) pad_offsets[e + 1] = incl;
  if (e == 0) pad_offsets[0] = 0;
  pdl_trigger();
}

__device__ __forceinline__ int group_of(const int32_t* pad_offsets, int E, int rp) {
  int lo = 0, hi = E - 1;  // largest e with pad_offsets[e] <= rp
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pad_offsets[mid] <= rp) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// One warp per padded row rp: dy_perm[rp] = dy[t], dO[rp] = bf16(p * dy[t]) for the rows of a
// segment; zeros (dy_perm, dO and dGU) for its pad rows.
__global__ void __launch_bounds__(256) gather_dy_kernel(const uint16_t* __restrict__ dy,
                                                        const int32_t* __restrict__ offsets,
                                                        const int32_t* __restrict__ pad_offsets, int E,
                                                        const int32_t* __restrict__ perm_token,
                                                        const float* __restrict__ p_perm, int D, int F2,
                                                        uint16_t* __restrict__ dyp, uint16_t* __restrict__ dO,
                                                        uint16_t* __restrict__ dgu) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int total = pad_offsets[E];
  for (int rp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; rp < total; rp += (gridDim.x * blockDim.x) >> 5) {
    const int e = group_of(pad_offsets, E, rp);
    const int i = rp - pad_offsets[e];
    uint4* a = reinterpret_cast<uint4*>(dyp + (size_t)rp * D);
    uint4* b = reinterpret_cast<uint4*>(dO + (size_t)rp * D);
    if (i < offsets[e + 1] - offsets[e]) {
      const int r = offsets[e] + i;
      const float pr = p_perm[r];
      const uint4* src = reinterpret_cast<const uint4*>(dy + (size_t)perm_token[r] * D);
      for (int v = lane; v < D / 8; v += 32) {
        const uint4 q = __ldg(src + v);
        a[v] = q;
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) o[k] = pack_bf16x2(pr * bf16_lo(w[k]), pr * bf16_hi(w[k]));
        b[v] = make_uint4(o[0], o[1], o[2], o[3]);
      }
    } else {
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      for (int v = lane; v < D / 8; v += 32) a[v] = z, b[v] = z;
      uint4* c = reinterpret_cast<uint4*>(dgu + (size_t)rp * F2);
      for (int v = lane; v < F2 / 8; v += 32) c[v] = z;
    }
  }
  pdl_trigger();
}

// One warp per token, lane j = slot j: dp = the fixed-order sum of the kDxDown partials, then the
// softmax backward over the chosen k; written per expert-contiguous row.
__global__ void __launch_bounds__(256) router_bwd_kernel(const int32_t* __restrict__ inv_perm,
                                                         const float* __restrict__ topk_w,
                                                         const float* __restrict__ dp_part, int n_tiles, int T,
                                                         int k, float* __restrict__ dl_row) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += (gridDim.x * blockDim.x) >> 5) {
    int r = -1;
    float pj = 0.f, dp = 0.f;
    if (lane < k) {
      r = inv_perm[(size_t)t * k + lane];
      pj = topk_w[(size_t)t * k + lane];
      if (r >= 0)
        for (int n = 0; n < n_tiles; ++n) dp += dp_part[(size_t)r * n_tiles + n];
    }
    float s = pj * dp;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (r >= 0) dl_row[r] = pj * (dp - s);
  }
  pdl_trigger();
}

// dW_g[e, d] = sum over the rows r of expert e, in order, of dl_row[r] * x_perm[r, d].
// Block (e, 256-column chunk); thread = column.
__global__ void __launch_bounds__(256) dwgate_kernel(const int32_t* __restrict__ offsets,
                                                     const float* __restrict__ dl_row,
                                                     const uint16_t* __restrict__ x_perm, int D,
                                                     float* __restrict__ dwg) {
  pdl_wait();
  const int e = blockIdx.x;
  const int d = blockIdx.y * 256 + threadIdx.x;
  if (d < D) {
    float acc = 0.f;
    for (int r = offsets[e]; r < offsets[e + 1]; ++r) {
      const uint16_t b = x_perm[(size_t)r * D + d];
      acc += dl_row[r] * __uint_as_float((uint32_t)b << 16);
    }
    dwg[(size_t)e * D + d] = acc;
  }
  pdl_trigger();
}

// dx[t] = bf16( sum_j dX[rp(t, j)] + dX_shared[t] + sum_j dl_j W_g[idx_j] ), one warp per (token,
// 256-column chunk); rp = the padded row of slot j.
__global__ void __launch_bounds__(256) unpermute_kernel(const float* __restrict__ dxp,
                                                        const float* __restrict__ dx_sh,
                                                        const int32_t* __restrict__ inv_perm,
                                                        const int32_t* __restrict__ topk_idx,
                                                        const int32_t* __restrict__ offsets,
                                                        const int32_t* __restrict__ pad_offsets,
                                                        const float* __restrict__ dl_row,
                                                        const uint16_t* __restrict__ wg, int T, int D, int k,
                                                        uint16_t* __restrict__ dx) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int n_chunks = (D + 255) / 256;
  const long long items = (long long)T * n_chunks;
  for (long long it = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5; it < items;
       it += ((long long)gridDim.x * blockDim.x) >> 5) {
    const int t = (int)(it / n_chunks);
    const int col = (int)(it - (long long)t * n_chunks) * 256 + lane * 8;
    int my_rp = -1, my_e = -1;
    float my_dl = 0.f;
    if (lane < k) {
      const int r = inv_perm[(size_t)t * k + lane];
      if (r >= 0) {
        my_e = topk_idx[(size_t)t * k + lane];
        my_rp = pad_offsets[my_e] + (r - offsets[my_e]);
        my_dl = dl_row[r];
      }
    }
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
      const int rp = __shfl_sync(0xffffffffu, my_rp, j);
      const int e = __shfl_sync(0xffffffffu, my_e, j);
      const float dl = __shfl_sync(0xffffffffu, my_dl, j);
      if (rp < 0 || col >= D) continue;
      const float4 a = *reinterpret_cast<const float4*>(dxp + (size_t)rp * D + col);
      const float4 b = *reinterpret_cast<const float4*>(dxp + (size_t)rp * D + col + 4);
      const uint4 w = *reinterpret_cast<const uint4*>(wg + (size_t)e * D + col);
      acc[0] += a.x + dl * bf16_lo(w.x), acc[1] += a.y + dl * bf16_hi(w.x);
      acc[2] += a.z + dl * bf16_lo(w.y), acc[3] += a.w + dl * bf16_hi(w.y);
      acc[4] += b.x + dl * bf16_lo(w.z), acc[5] += b.y + dl * bf16_hi(w.z);
      acc[6] += b.z + dl * bf16_lo(w.w), acc[7] += b.w + dl * bf16_hi(w.w);
    }
    if (col < D) {
      if (dx_sh != nullptr) {
        const float4 a = *reinterpret_cast<const float4*>(dx_sh + (size_t)t * D + col);
        const float4 b = *reinterpret_cast<const float4*>(dx_sh + (size_t)t * D + col + 4);
        acc[0] += a.x, acc[1] += a.y, acc[2] += a.z, acc[3] += a.w;
        acc[4] += b.x, acc[5] += b.y, acc[6] += b.z, acc[7] += b.w;
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      *reinterpret_cast<uint4*>(dx + (size_t)t * D + col) = o;
    }
  }
  pdl_trigger();
}

unsigned grid_for(long long warps) {
  long long b = (warps + 7) / 8;
  if (b < 1) b = 1;
  if (b > 148LL * 16) b = 148LL * 16;
  return (unsigned)b;
}

}  // namespace

cudaError_t launch_pad_offsets(const int32_t* offsets, int E, int32_t* pad_offsets, cudaStream_t s) {
  return launch_pdl(pad_offsets_kernel, dim3(1), dim3(1024), 0, s, offsets, E, pad_offsets);
}

cudaError_t launch_gather_dy(const uint16_t* dy, const int32_t* offsets, const int32_t* pad_offsets, int E,
                             const int32_t* perm_token, const float* p_perm, int D, int F2, long long rows_bound,
                             uint16_t* dyp, uint16_t* dO, uint16_t* dgu, cudaStream_t s) {
  return launch_pdl(gather_dy_kernel, dim3(grid_for(rows_bound)), dim3(256), 0, s, dy, offsets, pad_offsets, E,
                    perm_token, p_perm, D, F2, dyp, dO, dgu);
}

cudaError_t launch_router_bwd(const int32_t* inv_perm, const float* topk_w, const float* dp_part, int n_tiles, int T,
                              int k, float* dl_row, cudaStream_t s) {
  return launch_pdl(router_bwd_kernel, dim3(grid_for(T)), dim3(256), 0, s, inv_perm, topk_w, dp_part, n_tiles, T, k,
                    dl_row);
}

cudaError_t launch_dwgate(const int32_t* offsets, const float* dl_row, const uint16_t* x_perm, int E, int D,
                          float* dwg, cudaStream_t s) {
  return launch_pdl(dwgate_kernel, dim3(E, (D + 255) / 256), dim3(256), 0, s, offsets, dl_row, x_perm, D, dwg);
}

cudaError_t launch_unpermute(const float* dxp, const float* dx_sh, const int32_t* inv_perm, const int32_t* topk_idx,
                             const int32_t* offsets, const int32_t* pad_offsets, const float* dl_row, const uint16_t* wg,
                             int T, int D, int k, uint16_t* dx, cudaStream_t s) {
  return launch_pdl(unpermute_kernel, dim3(grid_for((long long)T * ((D + 255) / 256))), dim3(256), 0, s, dxp, dx_sh,
                    inv_perm, topk_idx, offsets, pad_offsets, dl_row, wg, T, D, k, dx);
}

}  // namespace moe
