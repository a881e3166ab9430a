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

// ------------------------------------------------------------------------------ small decode router
// For a few tokens and a router weight that fits in shared memory (the gpt-oss-shaped router is
// 32 x 2880 bf16 = 184 KB), one CTA does the whole routing step: bulk copies bring W_g and x into
// shared memory (issued before the wait on the previous kernel: neither is its output), CUDA-core
// dot products give the fp32 logits, then the top-k selection and, for the layer, the dispatch
// metadata -- no split-K partials, no second kernel, no inter-CTA counter.
//   logits : lane l of warp w accumulates x[t] . W_g[e] over the 16-byte chunks l, l + 32, ... of
//            expert e = w, w + 8, ... in fp32 (products in chunk order), then a butterfly sum;
//   select : k rounds of the highest l + bias, ties to the lower id; softmax of the chosen
//            unbiased logits (as router_select_kernel);
//   dispatch (counts != NULL): counts, offsets, and the stable order (experts ascending, tokens
//            ascending) as perm_token / inv_perm / p_perm.
constexpr int kSmallThreads = 256;
constexpr int kSmallWarps = kSmallThreads / 32;
constexpr int kSmallMaxT = 4;
constexpr int kSmallChunkBytes = 32 * 1024;
constexpr int kSmallMaxChunks = 8;
constexpr size_t kSmallSmemLimit = 220 * 1024;

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void sm_mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void sm_mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// bounded wait for phase 0 of a one-shot barrier
__device__ __forceinline__ bool sm_mbar_wait0(uint32_t bar) {
  uint64_t t0 = 0;
  for (;;) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar)
        : "memory");
    if (ok) return true;
    uint64_t now;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
    if (t0 == 0) t0 = now;
    else if (now - t0 > kWaitLimitNs) return false;
  }
}

struct SmallLayout {
  size_t w, x, logits, taken, idx, wts, cnt, run, wtot, bars, total;
};
__host__ __device__ inline SmallLayout small_layout(int T, int D, int E, int k) {
  SmallLayout L;
  size_t o = 0;
  auto take = [&](size_t bytes, size_t align) {
    o = (o + align - 1) / align * align;
    const size_t at = o;
    o += bytes;
    return at;
  };
  L.w = take((size_t)E * D * 2, 128);
  L.x = take((size_t)T * D * 2, 128);
  L.logits = take((size_t)T * E * 4, 16);
  L.taken = take((size_t)E, 16);
  L.idx = take((size_t)T * k * 4, 16);
  L.wts = take((size_t)T * k * 4, 16);
  L.cnt = take((size_t)E * 4, 16);
  L.run = take((size_t)E * 4, 16);
  L.wtot = take(kSmallWarps * 4, 16);
  L.bars = take((kSmallMaxChunks + 1) * 8, 8);
  L.total = o;
  return L;
}

__global__ void __launch_bounds__(kSmallThreads, 1) router_small_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ wg, const float* __restrict__ bias, int T, int D,
    int E, int k, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ perm_token, int32_t* __restrict__ inv_perm,
    float* __restrict__ p_perm, int* err) {
  extern __shared__ __align__(128) uint8_t sm[];
  const SmallLayout L = small_layout(T, D, E, k);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(sm);
  const uint32_t bars = base + (uint32_t)L.bars;
  const size_t row_bytes = (size_t)D * 2;
  const int rows_per_chunk = (int)(kSmallChunkBytes / row_bytes) > 0 ? (int)(kSmallChunkBytes / row_bytes) : 1;
  const int n_chunks = (E + rows_per_chunk - 1) / rows_per_chunk;
  if (tid == 0) {
    for (int c = 0; c <= n_chunks; ++c) sm_mbar_init(bars + 8 * c, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // the weights and the layer input are not outputs of the previous kernel: fetch them at once
  if (tid == 0) {
    for (int c = 0; c < n_chunks; ++c) {
      const int r0 = c * rows_per_chunk, r1 = min(E, r0 + rows_per_chunk);
      const uint32_t bytes = (uint32_t)((r1 - r0) * row_bytes);
      sm_mbar_expect_tx(bars + 8 * c, bytes);
      bulk_load(base + (uint32_t)(L.w + r0 * row_bytes), wg + (size_t)r0 * D, bytes, bars + 8 * c);
    }
    const uint32_t xb = (uint32_t)(T * row_bytes);
    sm_mbar_expect_tx(bars + 8 * n_chunks, xb);
    bulk_load(base + (uint32_t)L.x, x, xb, bars + 8 * n_chunks);
  }
  float* logits = reinterpret_cast<float*>(sm + L.logits);
  bool ok = sm_mbar_wait0(bars + 8 * n_chunks);
  // (1) logits: warp w owns experts w, w + 8, ...
  const int nv = D / 8;  // 16-byte chunks per row
  for (int e = warp; e < E && ok; e += kSmallWarps) {
    if (!sm_mbar_wait0(bars + 8 * (e / rows_per_chunk))) {
      ok = false;
      break;
    }
    const uint4* wrow = reinterpret_cast<const uint4*>(sm + L.w + (size_t)e * row_bytes);
    float acc[kSmallMaxT];
#pragma unroll
    for (int t = 0; t < kSmallMaxT; ++t) acc[t] = 0.f;
    for (int v = lane; v < nv; v += 32) {
      const uint4 w4 = wrow[v];
      const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
      for (int t = 0; t < kSmallMaxT; ++t) {
        if (t < T) {
          const uint4 x4 = reinterpret_cast<const uint4*>(sm + L.x + (size_t)t * row_bytes)[v];
          const uint32_t xv[4] = {x4.x, x4.y, x4.z, x4.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            acc[t] += bf16_lo(xv[i]) * bf16_lo(wv[i]);
            acc[t] += bf16_hi(xv[i]) * bf16_hi(wv[i]);
          }
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kSmallMaxT; ++t) {
      float a = acc[t];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
      if (lane == 0 && t < T) logits[t * E + e] = a;
    }
  }
  if (!ok) set_error(err, kErrTimeout);
  // everything below writes outputs the previous kernel may still read
  pdl_wait();
  __syncthreads();
  if (__syncthreads_or(!ok)) {
    pdl_trigger();
    return;
  }
  // (2) selection, one warp per token
  uint8_t* taken = sm + L.taken;
  int* idx_s = reinterpret_cast<int*>(sm + L.idx);
  float* w_s = reinterpret_cast<float*>(sm + L.wts);
  for (int t = warp; t < T; t += kSmallWarps) {
    const float* lrow = logits + t * E;
    for (int e = lane; e < E; e += 32) taken[e] = 0;
    __syncwarp();
    int my_idx = -1;
    float my_l = 0.f;
    for (int j = 0; j < k; ++j) {
      float bv = -FLT_MAX;
      int be = INT_MAX;
      for (int e = lane; e < E; e += 32) {
        const float sv = lrow[e] + (bias != nullptr ? bias[e] : 0.f);
        if (!taken[e] && (be == INT_MAX || sv > bv)) bv = sv, be = e;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oe = __shfl_xor_sync(0xffffffffu, be, off);
        if (oe != INT_MAX && (be == INT_MAX || ov > bv || (ov == bv && oe < be))) bv = ov, be = oe;
      }
      if (lane == 0) taken[be] = 1;
      if (lane == j) my_idx = be, my_l = lrow[be];
      __syncwarp();
    }
    float m = lane < k ? my_l : -FLT_MAX;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    const float ex = lane < k ? expf(my_l - m) : 0.f;
    float z = ex;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    if (lane < k) {
      const float wv = ex / z;
      topk_idx[(size_t)t * k + lane] = my_idx;
      topk_w[(size_t)t * k + lane] = wv;
      idx_s[t * k + lane] = my_idx;
      w_s[t * k + lane] = wv;
    }
    __syncwarp();
  }
  if (counts != nullptr) {
    // (3) dispatch: histogram, exclusive scan over experts, order-preserving scatter
    int* cnt = reinterpret_cast<int*>(sm + L.cnt);
    int* run = reinterpret_cast<int*>(sm + L.run);
    int* warp_tot = reinterpret_cast<int*>(sm + L.wtot);
    const int n_items = T * k;
    for (int e = tid; e < E; e += kSmallThreads) cnt[e] = 0;
    __syncthreads();
    for (int i = tid; i < n_items; i += kSmallThreads) atomicAdd(&cnt[idx_s[i]], 1);
    __syncthreads();
    const int per = (E + kSmallThreads - 1) / kSmallThreads;
    const int lo = min(E, tid * per), hi = min(E, lo + per);
    int sum = 0;
    for (int e = lo; e < hi; ++e) sum += cnt[e];
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0;
    for (int q = 0; q < warp; ++q) before += warp_tot[q];
    int r0 = before + incl - sum;
    for (int e = lo; e < hi; ++e) {
      counts[e] = cnt[e];
      offsets[e] = r0;
      run[e] = r0;
      r0 += cnt[e];
    }
    if (tid == kSmallThreads - 1) offsets[E] = before + incl;
    __syncthreads();
    if (warp == 0) {
      const unsigned lt_mask = (1u << lane) - 1u;
      for (int i0 = 0; i0 < n_items; i0 += 32) {
        const int i = i0 + lane;
        const int e = i < n_items ? idx_s[i] : -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0) {
          const int r = run[e] + __popc(peers & lt_mask);
          perm_token[r] = i / k;
          inv_perm[i] = r;
          p_perm[r] = w_s[i];
        }
        __syncwarp();
        if (e >= 0 && lane == 31 - __clz(peers)) run[e] += __popc(peers);
        __syncwarp();
      }
    }
  }
  pdl_trigger();
}

}  // namespace

bool router_small_fits(int T, int D, int E, int k) {
  if (T < 1 || T > kSmallMaxT || D % 64 != 0 || k < 1 || k > 32 || k > E) return false;
  const size_t row_bytes = (size_t)D * 2;
  if (row_bytes > kSmallChunkBytes) return false;
  const int rows_per_chunk = (int)(kSmallChunkBytes / row_bytes);
  if ((E + rows_per_chunk - 1) / rows_per_chunk > kSmallMaxChunks) return false;
  return small_layout(T, D, E, k).total <= kSmallSmemLimit;
}

cudaError_t launch_router_small(const uint16_t* x, const uint16_t* wg, const float* bias, int T, int D, int E, int k,
                                int32_t* topk_idx, float* topk_w, int32_t* counts, int32_t* offsets,
                                int32_t* perm_token, int32_t* inv_perm, float* p_perm, int* err, cudaStream_t s) {
  if (!router_small_fits(T, D, E, k)) return cudaErrorInvalidValue;
  const size_t smem = small_layout(T, D, E, k).total;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(router_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmallSmemLimit);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  return launch_pdl(router_small_kernel, dim3(1), dim3(kSmallThreads), smem, s, x, wg, bias, T, D, E, k, topk_idx,
                    topk_w, counts, offsets, perm_token, inv_perm, p_perm, err);
}

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
