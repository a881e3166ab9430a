// permute.cu -- step 2 of the layer: dispatch tokens into expert-contiguous order.
//
// keryc.com "Mixture of Experts optimiza Transformers y LLMs", section "Ejecucion eficiente:
// backends de expertos": the grouped backend sorts the tokens by expert id before the grouped
// GEMMs and puts the results back in the original order afterwards.
//
// A deterministic, stable counting sort of the T*k (token, slot) pairs by expert id:
//   1. hist    : per block of 256 tokens, per-expert counts with shared-memory atomics
//   2. scan    : per expert, exclusive scan over blocks; then exclusive scan over experts
//   3. scatter : per block, eight warps each walk 32 tokens' slots in (token, slot) order: a
//                first pass counts each warp's slots per expert, a warp-order prefix on the
//                block's offset gives each warp its start rows, and a second pass hands out rows
//                (ranks of equal experts inside each 32-slot step from __match_any_sync + popc)
//   4. gather  : x_perm[inv_perm[t*k + j]] = x[t], one warp per token: its row is read once and
//                written to each of its k rows, 16-byte vector moves
// For T <= 256 steps 1-4 run as one kernel (dispatch_small_kernel: every CTA sorts, all gather).
// Within an expert, rows are therefore ordered by token id (a token picks an expert at most once).
#include <cuda_fp16.h>

#include <algorithm>

#include "moe_common.cuh"

namespace moe {
namespace {

constexpr int kTokPerBlock = 256;

__global__ void __launch_bounds__(256) hist_kernel(const int32_t* __restrict__ idx, int T, int E, int k,
                                                   int32_t* __restrict__ block_counts, int* err) {
  extern __shared__ int cnt[];
  for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
  pdl_wait();
  __syncthreads();
  const int t0 = blockIdx.x * kTokPerBlock;
  const int n_items = min(T - t0, kTokPerBlock) * k;
  const int32_t* base = idx + (size_t)t0 * k;
  for (int i = threadIdx.x; i < n_items; i += blockDim.x) {
    const int e = base[i];
    if ((unsigned)e < (unsigned)E)
      atomicAdd(&cnt[e], 1);
    else
      set_error(err, kErrBadIndex);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) block_counts[(size_t)blockIdx.x * E + e] = cnt[e];
  pdl_trigger();
}

// One block of 1024 threads.  block_counts[b][e] becomes the exclusive prefix over blocks.
__global__ void __launch_bounds__(1024) scan_kernel(int32_t* __restrict__ block_counts, int nb, int E,
                                                    int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
  __shared__ int32_t warp_tot[32];
  const int e = threadIdx.x;  // E <= 1024
  int total = 0;
  pdl_wait();
  if (e < E) {
    for (int b = 0; b < nb; ++b) {
      const int v = block_counts[(size_t)b * E + e];
      block_counts[(size_t)b * E + e] = total;
      total += v;
    }
    counts[e] = total;
  }
  // block-wide inclusive scan of total over e
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = total;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_tot[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, w, off);
      if (lane >= off) w += v;
    }
    warp_tot[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  if (warp > 0) incl += warp_tot[warp - 1];
  if (e < E) offsets[e + 1] = incl;
  if (e == 0) offsets[0] = 0;
  pdl_trigger();
}

// One block of 8 warps per 256 tokens; warp w ranks the slots of tokens [32w, 32w + 32) of the
// block.  Order-preserving: a first pass counts each warp's slots per expert, the warps' counts
// are prefix-summed in warp order on top of the block's offset, and a second pass hands out rows
// in slot order (lanes in order within a 32-slot group via __match_any_sync, groups in order).
constexpr int kScatterWarps = kTokPerBlock / 32;

__global__ void __launch_bounds__(kScatterWarps * 32) scatter_kernel(const int32_t* __restrict__ idx,
                                                                     const float* __restrict__ w, int T, int E, int k,
                                                                     const int32_t* __restrict__ block_off,
                                                                     const int32_t* __restrict__ offsets,
                                                                     int32_t* __restrict__ perm_token,
                                                                     int32_t* __restrict__ inv_perm,
                                                                     float* __restrict__ p_perm) {
  extern __shared__ int run_all[];  // [warp][E]: the warp's count, then its next free row per expert
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int* run = run_all + warp * E;
  for (int e = lane; e < E; e += 32) run[e] = 0;
  pdl_wait();
  __syncwarp();
  const int t0 = blockIdx.x * kTokPerBlock;
  const int n_tok = min(T - t0, kTokPerBlock);
  const int i_lo = min(warp * 32, n_tok) * k, i_hi = min(warp * 32 + 32, n_tok) * k;
  const size_t base = (size_t)t0 * k;
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int i0 = i_lo; i0 < i_hi; i0 += 32) {  // pass 1: this warp's slots per expert
    const int i = i0 + lane;
    int e = i < i_hi ? idx[base + i] : -1;
    if ((unsigned)e >= (unsigned)E) e = -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0 && lane == 31 - __clz(peers)) run[e] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {  // warp-order prefix on the block's offset
    int r = offsets[e] + block_off[(size_t)blockIdx.x * E + e];
    for (int v = 0; v < kScatterWarps; ++v) {
      const int c = run_all[v * E + e];
      run_all[v * E + e] = r;
      r += c;
    }
  }
  __syncthreads();
  for (int i0 = i_lo; i0 < i_hi; i0 += 32) {  // pass 2: rows in slot order
    const int i = i0 + lane;
    int e = -1;
    if (i < i_hi) {
      e = idx[base + i];
      if ((unsigned)e >= (unsigned)E) {
        inv_perm[base + i] = -1;  // dropped slot (error already recorded by hist_kernel)
        e = -1;
      }
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    if (e >= 0) {
      const int r = run[e] + __popc(peers & lt_mask);
      const size_t slot = base + i;
      perm_token[r] = (int32_t)(slot / k);
      inv_perm[slot] = r;
      p_perm[r] = w[slot];
    }
    __syncwarp();
    if (e >= 0 && lane == 31 - __clz(peers)) run[e] += __popc(peers);
    __syncwarp();
  }
  pdl_trigger();
}

// bf16 -> f16 for 8 values (the FP8-weight GEMMs take f16 activations)
__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4 q) {
  const uint32_t in[4] = {q.x, q.y, q.z, q.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 h = __floats2half2_rn(bf16_lo(in[i]), bf16_hi(in[i]));
    o[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

constexpr int kGatherNone = 0, kGatherBf16 = 1, kGatherF16 = 2;
constexpr int kGatherChunk = 1024;  // columns per gather item

// T <= 256 (one counting block): histogram, scan and the order-preserving scatter of the T*k slots
// in one kernel -- the same three steps as above without two launches and the per-block scratch --
// fused with the gather.  Every CTA sorts the (at most 8192) slots in shared memory, which costs a
// few microseconds at most and needs no inter-CTA communication; CTA 0 alone writes the metadata.
// Then all CTAs copy (row, 1024-column chunk) items x[perm_token[r]] -> x_perm[r], as bf16 or
// converted to f16, followed (if x_cast is given) by x[t] -> x_cast[t] for every token.
template <int GATHER>
__global__ void __launch_bounds__(256) dispatch_small_kernel(const int32_t* __restrict__ idx,
                                                             const float* __restrict__ w, int T, int E, int k,
                                                             int32_t* __restrict__ counts,
                                                             int32_t* __restrict__ offsets,
                                                             int32_t* __restrict__ perm_token,
                                                             int32_t* __restrict__ inv_perm,
                                                             float* __restrict__ p_perm, int* err,
                                                             const uint16_t* __restrict__ x, int D,
                                                             uint16_t* __restrict__ x_perm,
                                                             uint16_t* __restrict__ x_cast) {
  extern __shared__ int sm[];
  int* cnt = sm;         // [E] counts
  int* run = sm + E;     // [E] next free row per expert
  int* perm_s = sm + 2 * E;  // [T*k] token of each row (gathering only)
  __shared__ int warp_tot[8];
  __shared__ int n_rows_s;
  const bool lead = blockIdx.x == 0;  // writes the metadata
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < E; e += 256) cnt[e] = 0;
  pdl_wait();
  __syncthreads();
  const int n_items = T * k;
  for (int i = tid; i < n_items; i += 256) {
    const int e = idx[i];
    if ((unsigned)e < (unsigned)E)
      atomicAdd(&cnt[e], 1);
    else if (lead)
      set_error(err, kErrBadIndex);
  }
  __syncthreads();
  // exclusive scan over experts: thread tid owns experts [tid*per, tid*per + per)
  const int per = (E + 255) / 256;
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
    if (lead) {
      counts[e] = cnt[e];
      offsets[e] = r0;
    }
    run[e] = r0;
    r0 += cnt[e];
  }
  if (tid == 255) {
    n_rows_s = before + incl;
    if (lead) offsets[E] = before + incl;
  }
  __syncthreads();
  if (warp == 0) {
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int i0 = 0; i0 < n_items; i0 += 32) {
      const int i = i0 + lane;
      int e = -1;
      if (i < n_items) {
        e = idx[i];
        if ((unsigned)e >= (unsigned)E) {
          if (lead) inv_perm[i] = -1;
          e = -1;
        }
      }
      const unsigned peers = __match_any_sync(0xffffffffu, e);
      if (e >= 0) {
        const int r = run[e] + __popc(peers & lt_mask);
        if (lead) {
          perm_token[r] = i / k;
          inv_perm[i] = r;
          p_perm[r] = w[i];
        }
        if (GATHER != kGatherNone) perm_s[r] = i / k;
      }
      __syncwarp();
      if (e >= 0 && lane == 31 - __clz(peers)) run[e] += __popc(peers);
      __syncwarp();
    }
  }
  if constexpr (GATHER != kGatherNone) {
    __syncthreads();
    const int n_chunks = (D + kGatherChunk - 1) / kGatherChunk;
    const int n_rows = n_rows_s;
    const int n_work = (n_rows + (x_cast != nullptr ? T : 0)) * n_chunks;
    for (int it = blockIdx.x * 8 + warp; it < n_work; it += gridDim.x * 8) {
      const int r = it / n_chunks, c0 = (it - r * n_chunks) * kGatherChunk;
      const int c1 = min(D, c0 + kGatherChunk);
      const bool cast_row = r >= n_rows;  // x_cast[t] = x[t], t = r - n_rows
      const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)(cast_row ? r - n_rows : perm_s[r]) * D);
      uint4* dst = reinterpret_cast<uint4*>(cast_row ? x_cast + (size_t)(r - n_rows) * D : x_perm + (size_t)r * D);
      for (int v = c0 / 8 + lane; v < c1 / 8; v += 32) {
        const uint4 q = __ldg(src + v);
        dst[v] = GATHER == kGatherF16 ? bf16x8_to_f16x8(q) : q;
      }
    }
  }
  pdl_trigger();
}

// x_perm[inv_perm[t*k + j]] = x[t] for every kept slot; one warp per token, 16-byte moves.  Each x
// row is read once and written to its k rows: read by permuted row instead, a token's row would
// come from DRAM up to k times, since x (T*D*2 bytes) does not stay in L2 between its k slots.
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint16_t* __restrict__ x,
                                                          const int32_t* __restrict__ inv_perm, int T, int k,
                                                          int D, int M, uint16_t* __restrict__ x_perm) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int nv = D / 8;
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += (gridDim.x * blockDim.x) >> 5) {
    int my_r = lane < k ? inv_perm[(size_t)t * k + lane] : -1;
    if ((unsigned)my_r >= (unsigned)M) my_r = -1;  // a dropped slot (expert id out of range)
    const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * D);
    for (int v0 = 0; v0 < nv; v0 += 32) {  // every lane runs every pass: the shuffles stay warp-uniform
      const int v = v0 + lane;
      uint4 a = make_uint4(0u, 0u, 0u, 0u);
      if (v < nv) a = __ldg(src + v);
      for (int j = 0; j < k; ++j) {
        const int r = __shfl_sync(0xffffffffu, my_r, j);
        if (v < nv && (unsigned)r < (unsigned)M) reinterpret_cast<uint4*>(x_perm + (size_t)r * D)[v] = a;
      }
    }
  }
  pdl_trigger();
}

}  // namespace

size_t permute_scratch_bytes(int T, int E) {
  const size_t nb = (size_t)(T + kTokPerBlock - 1) / kTokPerBlock;
  return align_up(nb * (size_t)E * sizeof(int32_t), 256);
}

cudaError_t launch_permute(const int32_t* idx, const float* topk_w, const uint16_t* x, int T, int D, int E, int k,
                           int32_t* counts, int32_t* offsets, int32_t* perm_token, int32_t* inv_perm, float* p_perm,
                           uint16_t* x_perm, bool x_perm_f16, uint16_t* x_cast, int32_t* scratch, int* err,
                           cudaStream_t s, int* n_launches) {
  const int nb = (T + kTokPerBlock - 1) / kTokPerBlock;
  const bool gather = x != nullptr && x_perm != nullptr && T > 0;
  if (!x_perm_f16) x_cast = nullptr;  // the cast copy exists for the f16 (FP8-weight) path only
  // f16 rows are for the E4M3-weight decode path (T <= 64), which the one-kernel dispatch serves
  if (x_perm_f16 && nb > 1) return cudaErrorInvalidValue;
  int launches = 0;
  cudaError_t e = cudaSuccess;
  if (nb == 1) {
    // one fused kernel: sort in every CTA, gather (row, column chunk) items across the grid
    const long long items =
        gather ? ((long long)T * k + (x_cast != nullptr ? T : 0)) * ((D + kGatherChunk - 1) / kGatherChunk) : 0;
    const unsigned blocks = gather ? (unsigned)std::min<long long>(148, (items + 7) / 8) : 1u;
    const size_t smem = (2 * (size_t)E + (gather ? (size_t)T * k : 0)) * sizeof(int);
    if (!gather)
      e = launch_pdl(dispatch_small_kernel<kGatherNone>, dim3(1), dim3(256), smem, s, idx, topk_w, T, E, k, counts,
                     offsets, perm_token, inv_perm, p_perm, err, x, D, x_perm, x_cast);
    else if (x_perm_f16)
      e = launch_pdl(dispatch_small_kernel<kGatherF16>, dim3(blocks), dim3(256), smem, s, idx, topk_w, T, E, k,
                     counts, offsets, perm_token, inv_perm, p_perm, err, x, D, x_perm, x_cast);
    else
      e = launch_pdl(dispatch_small_kernel<kGatherBf16>, dim3(blocks), dim3(256), smem, s, idx, topk_w, T, E, k,
                     counts, offsets, perm_token, inv_perm, p_perm, err, x, D, x_perm, x_cast);
    if (e != cudaSuccess) return e;
    if (n_launches) *n_launches = 1;
    return cudaGetLastError();
  }
  if (nb > 0) {
    e = launch_pdl(hist_kernel, dim3(nb), dim3(256), E * sizeof(int), s, idx, T, E, k, scratch, err);
    if (e != cudaSuccess) return e;
    ++launches;
  }
  e = launch_pdl(scan_kernel, dim3(1), dim3(1024), 0, s, scratch, nb, E, counts, offsets);
  if (e != cudaSuccess) return e;
  ++launches;
  if (nb > 0) {
    e = launch_pdl(scatter_kernel, dim3(nb), dim3(kScatterWarps * 32), kScatterWarps * E * sizeof(int), s, idx,
                   topk_w, T, E, k,
                   (const int32_t*)scratch, (const int32_t*)offsets, perm_token, inv_perm, p_perm);
    if (e != cudaSuccess) return e;
    ++launches;
  }
  if (gather) {  // one warp per token
    e = launch_pdl(gather_rows_kernel, dim3((unsigned)std::min<long long>(148LL * 16, ((long long)T + 7) / 8)),
                   dim3(256), 0, s, x, (const int32_t*)inv_perm, T, k, D, T * k, x_perm);
    if (e != cudaSuccess) return e;
    ++launches;
  }
  if (n_launches) *n_launches = launches;
  return cudaGetLastError();
}

}  // namespace moe
