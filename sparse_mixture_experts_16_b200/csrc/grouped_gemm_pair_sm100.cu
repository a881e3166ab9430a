// Token-wide grouped GEMMs on CTA pairs (sm_100a: tcgen05.mma.cta_group::2, TMEM, TMA) for the
// expert FFN of the MoE layer:
//   gate_up: h = silu(x_e G_e^T) * (x_e U_e^T)   (gotburnout.io glossary "MoE", section 3 step 3,
//            SwiGLU; the packed gate_up_proj [E, 2F, D] of dev.smart-guide.co.kr "La Solucion:
//            WeightConverter": rows [0, F) gate, [F, 2F) up)
//   down:    o = p * (h_e Down_e^T)              (section 3 step 4, weighted by the router's p)
// over the expert-contiguous segments of the permuted rows (keryc.com "Ejecucion eficiente:
// backends de expertos", the grouped backend), plus the always-on shared expert as a second
// operand set (gotburnout.io, section 2 item 3).
//
// Orientation as in the one-CTA token-wide kernel (weights as the MMA's M, up to 256 tokens of one
// segment as N; TMEM lane = output column, TMEM column = token), but one tile is computed by a
// cluster of two CTAs with one M = 256 MMA: each CTA loads its own 128 weight rows (A half) and
// its own N/2 token rows (B half) into its own shared memory, and receives the accumulator rows of
// its 128 weight rows for all N tokens.  Per SM and per 64-wide K block that is 32 KB of operands
// for a 128 x N x 64 product, against 48 KB in the one-CTA tile: a third less L2-to-SM traffic
// per FLOP.  No load is multicast: every CTA fetches its own operands.
//   gate_up: the pair's 256 weight rows are, per CTA, 64 gate rows stacked on the 64 up rows of the
//            same 64 output columns (CTA v: columns [128 n + 64 v, +64)), so the SwiGLU pairs stay
//            inside one CTA's TMEM.
//   down:    CTA v holds output columns [256 n + 128 v, +128).
// A segment of R rows becomes ceil(R / 256) token tiles, the last with N = rows rounded up to 16.
//
// Kernel layout (persistent clusters of two, 192 threads per CTA):
//   warp 0     TMA producer of each CTA: per K block, its weight half (16 KB) and its token half
//              (N/2 rows) into a 6-stage ring; completion is counted on the even CTA's barrier.
//   warp 1     TMEM allocation in both CTAs; in the even CTA one thread issues the pair MMAs and
//              commits to both CTAs' stage and accumulator barriers (commit multicast).
//   warps 2-5  epilogue of each CTA: per 32-token chunk, tcgen05.ld of the warp's 32 lanes, a
//              transpose through a padded shared-memory stage, row-contiguous stores (SwiGLU or the
//              p scale fused), then a release of the accumulator to the even CTA.
// Every wait is bounded (kWaitLimitNs); on expiry the kernel sets kErrTimeout and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>

#include "grouped_gemm_wide.cuh"
#include "moe_common.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kPT = 256;                       // token tile (MMA N at most)
constexpr int kPM = 128;                       // weight rows per CTA (the pair's MMA has M = 256)
constexpr int kPBK = 64;                       // K per stage
constexpr int kPThreads = 192;
constexpr int kPStages = 6;
constexpr int kPMaxGroups = 1025;              // E <= 1024 routed + 1 shared
constexpr int kPTileW = kPM * kPBK * 2;        // 16 KB of weights per CTA per stage
constexpr int kPBox = 64 * kPBK * 2;           // 8 KB: one 64-row box of tokens
constexpr int kPTileT = (kPT / 2) * kPBK * 2;  // 16 KB: up to 128 token rows per CTA per stage
constexpr int kPStageBytes = kPTileW + kPTileT;
constexpr int kPChunk = 32;                    // tokens per epilogue chunk
constexpr int kPPitch = 144;                   // fp32 words per staged token row (128 + 16)
constexpr int kPStagingBytes = kPChunk * kPPitch * 4;
constexpr int kPBarBytes = 256;
constexpr size_t kPSmemBytes = 1024 + (size_t)kPStages * kPStageBytes + kPStagingBytes + kPBarBytes +
                               4 * (kPMaxGroups + 1);
static_assert(kPSmemBytes <= 232448, "shared memory budget");
static_assert(kPStageBytes % 1024 == 0 && kPTileW % 1024 == 0, "alignment");

struct alignas(64) PairParams {
  CUtensorMap t_map[2];     // token operand per set (x_perm / x / h), box 64 K x 64 rows
  CUtensorMap t_map128[2];  // the same tensor, box 64 K x 128 rows (a full token half in one copy)
  CUtensorMap w_map[2];     // weights per set: down [rows, K], box 64 K x 128 rows; gate_up viewed as
                            // [groups][2 halves][F rows][K], box 64 K x 64 rows x 2 halves
  CUtensorMap o_map[2];     // down: fp32 output [rows, D], box 32 columns x 32 rows (TMA stores)
  const int32_t* offsets[2];
  void* out[2];             // gate_up: bf16 h [rows, F]; down: fp32 [rows, D]
  const float* row_scale[2];
  uint16_t* save_gu[2];     // gate_up in a training forward: g | u [rows, 2F] bf16, or NULL
  int n_groups[2];
  int m_rows[2];
  int n_out[2];
  int w_rows[2];            // weight rows per group: 2F (gate_up) or D (down)
  int k_blocks[2];          // K / 64
  int n_sets;
  int withhold_first_load;  // test only: the even CTA never issues its first stage's copies
  int* err;
};

struct PTile {
  int set, gl, row0, rows, m, n;
};

__device__ __forceinline__ void p_group_rows(const PairParams& p, int s, int gl, int& row0, int& rows) {
  if (p.offsets[s] != nullptr) {
    row0 = p.offsets[s][gl];
    rows = p.offsets[s][gl + 1] - row0;
  } else {
    row0 = 0;
    rows = p.m_rows[s];
  }
}

// output columns per pair tile: gate_up 128 (64 per CTA), down 256 (128 per CTA)
template <int KIND>
__host__ __device__ constexpr int p_cols_per_tile() {
  return KIND == kGateUp ? 128 : 256;
}

template <int KIND>
__device__ __forceinline__ int p_group_tiles(const PairParams& p, int s, int rows) {
  if (rows <= 0) return 0;
  const int nt = (p.n_out[s] + p_cols_per_tile<KIND>() - 1) / p_cols_per_tile<KIND>();
  return ((rows + kPT - 1) / kPT) * nt;
}

// tile t -> (group, token tile m, column tile n), token tiles fastest
template <int KIND>
__device__ __forceinline__ PTile p_decode(const PairParams& p, const int* tile_start, int G, int t) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= t) lo = mid; else hi = mid - 1;
  }
  PTile ti;
  ti.set = lo < p.n_groups[0] ? 0 : 1;
  ti.gl = ti.set == 0 ? lo : lo - p.n_groups[0];
  p_group_rows(p, ti.set, ti.gl, ti.row0, ti.rows);
  const int local = t - tile_start[lo];
  const int mt = (ti.rows + kPT - 1) / kPT;
  ti.n = local / mt;
  ti.m = local - ti.n * mt;
  return ti;
}

// tokens of tile ti (1..256); the MMA's N is this rounded up to 16, and each CTA holds half of N
__device__ __forceinline__ int p_tile_tokens(const PTile& ti) { return min(kPT, ti.rows - ti.m * kPT); }
__device__ __forceinline__ int p_half(int nr) { return ((nr + 15) / 16) * 8; }
// token bytes one CTA loads per stage: one 128-row box for a full half, else 64-row boxes
__device__ __forceinline__ int p_token_bytes(int half) { return half == 128 ? kPTileT : ((half + 63) / 64) * kPBox; }

__device__ __forceinline__ float p_silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }

__device__ __forceinline__ void p_epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ bool p_epi_any(bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %1, 0;\n\t"
      "bar.red.or.pred q, 1, 128, p;\n\t"
      "selp.b32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void p_st_shared_f32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// TMA bulk store of a box from shared memory, tracked in this thread's bulk group
__device__ __forceinline__ void p_tma_store_2d(const CUtensorMap* map, uint32_t src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void p_bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void p_bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void p_bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ float4 p_ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

template <int KIND>
__global__ void __launch_bounds__(kPThreads, 1) grouped_gemm_pair_kernel(const __grid_constant__ PairParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + kPStages * kPStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + kPStagingBytes);  // even CTA: both halves landed
  uint64_t* empty = full + kPStages;                                       // both CTAs: stage consumed
  uint64_t* acc_full = empty + kPStages;                                   // both CTAs: accumulator ready
  uint64_t* acc_empty = acc_full + 2;                                      // even CTA: both epilogues done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  int* tile_start = reinterpret_cast<int*>(staging + kPStagingBytes + kPBarBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs; 1: its partner
  const bool leader = rank == 0;
  const int G = p.n_groups[0] + (p.n_sets > 1 ? p.n_groups[1] : 0);
  const int cluster_id = blockIdx.x >> 1, n_clusters = gridDim.x >> 1;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kPStages; ++s) {
      mbar_init(&full[s], 1);   // the even CTA's arrive.expect_tx (bytes of both CTAs)
      mbar_init(&empty[s], 1);  // one commit of the pair's MMAs
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);   // one commit
      mbar_init(&acc_empty[b], 8);  // four epilogue warps of each CTA
    }
    fence_barrier_init();
    for (int s = 0; s < p.n_sets; ++s) {
      prefetch_tensormap(&p.t_map[s]);
      prefetch_tensormap(&p.t_map128[s]);
      prefetch_tensormap(&p.w_map[s]);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 2 * kPT);
    tmem_relinquish_pair();
  }
  // everything above overlaps the previous kernel; offsets and operands are its outputs
  pdl_wait();
  pdl_trigger();
  for (int g = threadIdx.x; g < G; g += kPThreads) {
    const int s = g < p.n_groups[0] ? 0 : 1;
    const int gl = s == 0 ? g : g - p.n_groups[0];
    int row0, rows;
    p_group_rows(p, s, gl, row0, rows);
    tile_start[g] = p_group_tiles<KIND>(p, s, rows);
  }
  __syncthreads();
  if (warp == 0) {  // exclusive scan of the per-group tile counts
    const int per = (G + 31) / 32;
    const int lo = lane * per, hi = min(G, lo + per);
    int sum = 0;
    for (int g = lo; g < hi; ++g) sum += tile_start[g];
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int run = incl - sum;
    for (int g = lo; g < hi; ++g) {
      const int c = tile_start[g];
      tile_start[g] = run;
      run += c;
    }
    if (lane == 31) tile_start[G] = incl;
  }
  tc_fence_before();
  // both CTAs' barriers are initialised and the TMEM allocation is visible before any remote use
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tile_start[G];

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = cluster_id; t < total && ok; t += n_clusters) {
        const PTile ti = p_decode<KIND>(p, tile_start, G, t);
        const int half = p_half(p_tile_tokens(ti));
        const int tbytes = p_token_bytes(half);
        const int trow = ti.row0 + ti.m * kPT + (int)rank * half;
        const int wrow = ti.gl * p.w_rows[ti.set] + ti.n * p_cols_per_tile<KIND>() + (int)rank * kPM;
        const int grow = ti.n * p_cols_per_tile<KIND>() + (int)rank * 64;  // gate_up: first output column
        for (int kb = 0; kb < p.k_blocks[ti.set]; ++kb, ++it) {
          const int stage = it % kPStages;
          if (!mbar_wait(&empty[stage], ((it / kPStages) & 1) ^ 1, kWaitLimitNs)) {
            ok = false;
            break;
          }
          uint8_t* sb = smem + stage * kPStageBytes;
          const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);  // the even CTA's barrier
          if (leader) mbar_arrive_expect_tx(&full[stage], 2u * (uint32_t)(kPTileW + tbytes));
          if (leader && p.withhold_first_load && it == 0) continue;  // these bytes never arrive
          const int kx = kb * kPBK;
          if constexpr (KIND == kGateUp) {
            tma_load_4d_pair(&p.w_map[ti.set], bar, sb, kx, grow, 0, ti.gl);  // 64 gate rows, then 64 up
          } else {
            tma_load_2d_pair(&p.w_map[ti.set], bar, sb, kx, wrow);
          }

          if (half == 128) {
            tma_load_2d_pair(&p.t_map128[ti.set], bar, sb + kPTileW, kx, trow);
          } else {
            for (int b = 0; b * 64 < half; ++b)
              tma_load_2d_pair(&p.t_map[ti.set], bar, sb + kPTileW + b * kPBox, kx, trow + b * 64);
          }
        }
      }
      if (!ok) set_error(p.err, kErrTimeout);
      // drain: every stage this CTA filled must be consumed (the even CTA: landed) before shared
      // memory is released.  After one expired wait the copies still in flight have long landed
      // (the limit is 1 s), so the remaining stages are not waited for again.
      const uint32_t issued = it;
      for (int s = 0; s < kPStages; ++s) {
        if ((uint32_t)s >= issued) break;
        const uint32_t last = issued - 1 - ((issued - 1 - s) % kPStages);
        const bool done = leader ? mbar_wait(&full[s], (last / kPStages) & 1, kWaitLimitNs)
                                 : mbar_wait(&empty[s], (last / kPStages) & 1, kWaitLimitNs);
        if (!done) {
          set_error(p.err, kErrTimeout);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (even CTA)
    if (leader && lane == 0) {
      uint32_t it = 0, tl = 0;
      bool ok = true;
      for (int t = cluster_id; t < total && ok; t += n_clusters, ++tl) {
        const uint32_t buf = tl & 1, use = tl >> 1;
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + buf * kPT;
        const PTile ti = p_decode<KIND>(p, tile_start, G, t);
        const uint32_t idesc = idesc_bf16_f32(2 * kPM, 2 * p_half(p_tile_tokens(ti)));
        for (int kb = 0; kb < p.k_blocks[ti.set]; ++kb, ++it) {
          const int stage = it % kPStages;
          if (!mbar_wait(&full[stage], (it / kPStages) & 1, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kPStageBytes);
#pragma unroll
          for (int kk = 0; kk < kPBK / 16; ++kk)
            umma_bf16_pair(d, sw128_kmajor_desc(sa + kk * 32), sw128_kmajor_desc(sa + kPTileW + kk * 32), idesc,
                           (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit_pair(&empty[stage], 0x3);  // frees the stage in both CTAs
        }
        if (!ok) break;
        umma_commit_pair(&acc_full[buf], 0x3);  // accumulator ready in both CTAs
      }
      if (!ok) set_error(p.err, kErrTimeout);
      if (it > 0) {  // the last commit covers every MMA issued before it
        const uint32_t last = it - 1;
        if (!mbar_wait(&empty[last % kPStages], (last / kPStages) & 1, kWaitLimitNs)) set_error(p.err, kErrTimeout);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5, both CTAs)
    const int q = warp & 3;
    const int e = threadIdx.x - 64;  // 0..127
    const int j_in = e >> 2, part = e & 3;
    const uint32_t stage_base = smem_u32(staging);
    const uint32_t st_col = stage_base + (uint32_t)(q * 32 + lane) * 4;
    const uint32_t ld_row = stage_base + (uint32_t)(j_in * kPPitch) * 4;
    uint32_t tl = 0;
    for (int t = cluster_id; t < total; t += n_clusters, ++tl) {
      const uint32_t buf = tl & 1, use = tl >> 1;
      const bool ok = mbar_wait(&acc_full[buf], use & 1, kWaitLimitNs);
      if (p_epi_any(!ok)) {  // all four warps leave together
        if (!ok) set_error(p.err, kErrTimeout);
        break;
      }
      tc_fence_after();
      const PTile ti = p_decode<KIND>(p, tile_start, G, t);
      const int nr = p_tile_tokens(ti);
      const int n_out = p.n_out[ti.set];
      const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + buf * kPT;
      const size_t trow = (size_t)ti.row0 + (size_t)ti.m * kPT;
      if constexpr (KIND == kDown) {
        // Each warp owns 32 output columns (its TMEM lanes) x 32 tokens per chunk: it scales them by
        // the tokens' router weights, stages them densely ([token][column], conflict-free) in its
        // own 4 KB of shared memory and writes them with one TMA bulk store.  A chunk that runs past
        // the segment (or a column block past the tensor) is stored directly instead: one coalesced
        // 128-byte row segment per instruction, never a box reaching into another segment's rows.
        const int c_warp = ti.n * 256 + (int)rank * 128 + q * 32;
        const float* rs = p.row_scale[ti.set];
        float* out = static_cast<float*>(p.out[ti.set]);
        const uint32_t wstg = stage_base + (uint32_t)q * 4096u;
#pragma unroll 1
        for (int j0 = 0; j0 < nr; j0 += kPChunk) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tacc + j0, v);
          tmem_ld_wait();
          const int nj = min(kPChunk, nr - j0);
          const float pv = (rs != nullptr && lane < nj) ? rs[trow + j0 + lane] : 1.0f;
          if (c_warp >= n_out) continue;  // this warp's columns lie past the tensor (D % 256 != 0)
          if (nj == kPChunk && c_warp + 32 <= n_out) {
            if (lane == 0) p_bulk_wait_read_all();  // the previous chunk's store has read the staging
            __syncwarp();
#pragma unroll
            for (int j = 0; j < 32; ++j)
              p_st_shared_f32(wstg + (uint32_t)(j * 128 + lane * 4),
                              __float_as_uint(__uint_as_float(v[j]) * __shfl_sync(0xffffffffu, pv, j)));
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic stores -> the TMA's reads
            __syncwarp();
            if (lane == 0) {
              p_tma_store_2d(&p.o_map[ti.set], wstg, c_warp, (int32_t)(trow + j0));
              p_bulk_commit();
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float sc = __shfl_sync(0xffffffffu, pv, j);
              if (j < nj && c_warp + lane < n_out)
                out[(trow + j0 + j) * n_out + c_warp + lane] = __uint_as_float(v[j]) * sc;
            }
          }
        }
      } else {
        // gate_up: the pair's 64 g and 64 u columns of each 32-token chunk go through a padded
        // [token][column] staging area so that each thread writes 4 h values of one token row
#pragma unroll 1
        for (int j0 = 0; j0 < nr; j0 += kPChunk) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tacc + j0, v);
          tmem_ld_wait();
          p_epi_sync();  // the previous chunk's readers are done with the stage
#pragma unroll
          for (int j = 0; j < 32; ++j) p_st_shared_f32(st_col + (uint32_t)(j * kPPitch) * 4, v[j]);
          p_epi_sync();
          const int c_base = ti.n * 128 + (int)rank * 64;
          if (j0 + j_in < nr && c_base < n_out) {
            const size_t grow = trow + j0 + j_in;
            uint16_t* hrow = static_cast<uint16_t*>(p.out[ti.set]) + grow * n_out + c_base;
            uint16_t* srow = p.save_gu[ti.set] != nullptr ? p.save_gu[ti.set] + grow * 2 * n_out + c_base : nullptr;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int c = part * 4 + i * 16;
              const float4 g = p_ld_shared_f4(ld_row + c * 4);
              const float4 u = p_ld_shared_f4(ld_row + (64 + c) * 4);
              *reinterpret_cast<uint2*>(hrow + c) =
                  make_uint2(pack_bf16x2(p_silu_mul(g.x, u.x), p_silu_mul(g.y, u.y)),
                             pack_bf16x2(p_silu_mul(g.z, u.z), p_silu_mul(g.w, u.w)));
              if (srow != nullptr) {  // the backward pass's SwiGLU inputs
                *reinterpret_cast<uint2*>(srow + c) = make_uint2(pack_bf16x2(g.x, g.y), pack_bf16x2(g.z, g.w));
                *reinterpret_cast<uint2*>(srow + n_out + c) = make_uint2(pack_bf16x2(u.x, u.y), pack_bf16x2(u.z, u.w));
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&acc_empty[buf]), 0));  // release to the MMA issuer
    }
    if constexpr (KIND == kDown) {
      if (lane == 0) p_bulk_wait_all();  // every output store of this warp has been performed
    }
  }

  tc_fence_before();
  __syncthreads();
  __syncwarp();
  // neither CTA leaves (or frees TMEM) while its partner may still signal its barriers or the
  // pair's MMAs may still write its tensor memory
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 2 * kPT);
  }
}

// ------------------------------------------------------------------------------ host side
typedef CUresult (*PEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

PEncodeFn p_encode_fn() {
  static PEncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PEncodeFn>(ptr);
  });
  return fn;
}

// 2-D bf16 row-major [rows, cols] map, box = 64 columns (128 bytes) x box_rows, 128-byte swizzle;
// rows past the end read as zero.
bool p_make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  PEncodeFn enc = p_encode_fn();
  if (enc == nullptr || rows == 0 || cols == 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// gate_up weights [groups, 2F, K] bf16 as a 4-D tensor (K, F rows, 2 halves, groups); the box of
// 64 K x 64 rows x 2 halves lands as 128 rows of 128 bytes: the 64 gate rows, then their 64 up rows.
bool p_make_gate_up_map(CUtensorMap* m, const void* base, int groups, int F, int K) {
  PEncodeFn enc = p_encode_fn();
  if (enc == nullptr || groups <= 0 || F <= 0 || K <= 0) return false;
  cuuint64_t dims[4] = {(cuuint64_t)K, (cuuint64_t)F, 2, (cuuint64_t)groups};
  cuuint64_t strides[3] = {(cuuint64_t)K * 2, (cuuint64_t)F * K * 2, (cuuint64_t)2 * F * K * 2};
  cuuint32_t box[4] = {64, 64, 2, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 row-major [rows, cols] output map for the down's TMA stores: box 32 columns x 32 rows
bool p_make_out_map(CUtensorMap* m, void* base, uint64_t rows, uint64_t cols) {
  PEncodeFn enc = p_encode_fn();
  if (enc == nullptr || rows == 0 || cols == 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// clusters of two that fit on the device at once (the persistent grid is twice this)
template <int KIND>
int pair_clusters() {
  static int n = 0;
  if (n == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = kPSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int c = 0;
    if (cudaOccupancyMaxActiveClusters(&c, grouped_gemm_pair_kernel<KIND>, &cfg) != cudaSuccess || c <= 0) {
      cudaGetLastError();
      c = 0;
    }
    n = c;
  }
  return n;
}

template <int KIND>
cudaError_t launch_pair(const GemmSetHost* sets, int n_sets, int* err, cudaStream_t s) {
  PairParams p;
  memset(&p, 0, sizeof(p));
  p.n_sets = n_sets;
  p.err = err;
  p.withhold_first_load = test_withhold_this_launch() ? 1 : 0;
  for (int i = 0; i < n_sets; ++i) {
    const GemmSetHost& st = sets[i];
    if (st.K <= 0 || st.K % kPBK != 0 || st.n_out <= 0) return cudaErrorInvalidValue;
    if (KIND == kGateUp ? (st.n_out % 64 != 0) : (st.n_out % 32 != 0)) return cudaErrorInvalidValue;
    if (st.ld_out != 0 && st.ld_out != st.n_out) return cudaErrorInvalidValue;
    p.k_blocks[i] = st.K / kPBK;
    p.w_rows[i] = KIND == kGateUp ? 2 * st.n_out : st.n_out;
    if (!p_make_map(&p.t_map[i], st.a, (uint64_t)st.a_rows, (uint64_t)st.K, 64) ||
        !p_make_map(&p.t_map128[i], st.a, (uint64_t)st.a_rows, (uint64_t)st.K, 128))
      return cudaErrorInvalidValue;
    if (KIND == kGateUp ? !p_make_gate_up_map(&p.w_map[i], st.w, st.n_groups, st.n_out, st.K)
                        : !p_make_map(&p.w_map[i], st.w, (uint64_t)st.n_groups * p.w_rows[i], (uint64_t)st.K, 128))
      return cudaErrorInvalidValue;
    if (KIND == kDown) {
      const uint64_t out_rows = st.offsets != nullptr ? (uint64_t)st.a_rows : (uint64_t)st.m_rows;
      if (!p_make_out_map(&p.o_map[i], st.out, out_rows, (uint64_t)st.n_out)) return cudaErrorInvalidValue;
    }
    p.offsets[i] = st.offsets;
    p.out[i] = st.out;
    p.row_scale[i] = KIND == kDown ? st.row_scale : nullptr;
    p.save_gu[i] = KIND == kGateUp ? st.save_gu : nullptr;
    p.n_groups[i] = st.n_groups;
    p.m_rows[i] = st.m_rows;
    p.n_out[i] = st.n_out;
  }
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_pair_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kPSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int clusters = pair_clusters<KIND>();
  if (clusters <= 0) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = kPSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, grouped_gemm_pair_kernel<KIND>, p);
}

}  // namespace

cudaError_t launch_grouped_gemm_pair(GemmKind kind, const GemmSetHost* sets, int n_sets, int* err, cudaStream_t s) {
  if (n_sets < 1 || n_sets > 2) return cudaErrorInvalidValue;
  int groups = 0;
  for (int i = 0; i < n_sets; ++i) groups += sets[i].n_groups;
  if (groups > kPMaxGroups) return cudaErrorInvalidValue;
  if (kind == kGateUp) return launch_pair<kGateUp>(sets, n_sets, err, s);
  if (kind == kDown) return launch_pair<kDown>(sets, n_sets, err, s);
  return cudaErrorInvalidValue;
}

}  // namespace moe
