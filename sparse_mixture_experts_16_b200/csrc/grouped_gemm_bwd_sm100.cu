// grouped_gemm_bwd_sm100.cu -- the backward pass's grouped GEMMs on the tcgen05 tensor cores.
//
// keryc.com "Mixture of Experts optimiza...", section "Entrenamiento: todavia desafiante, pero con
// avances", and dev.smart-guide.co.kr, section "Entrenamiento MoE: 12x Mas Rapido": MoE training
// runs the experts' grouped GEMMs backwards too.  The pages give no formulas; the gradients are the
// chain rule of the forward (layer_backward.cu lists them).  Per expert e, over its rows:
//   kDxDown    dHu  = dy_perm * Down_e            [rows, F], K = D;  epilogue: the SwiGLU backward
//                    dh = p * dHu, dg = dh * u * silu'(g), du = dh * silu(g)  -> dGU [rows, 2F]
//                    and the router's dp = sum_f dHu * h, kept as one partial per 256 columns
//   kDxGateUp  dX   = dGU * gate_up_e             [rows, D], K = 2F   (fp32)
//   kDwDown    dDown_e   = dO_e^T h_e              [D, F],  K = rows  (fp32; dO = p * dy_perm)
//   kDwGateUp  dGateUp_e = dGU_e^T x_perm_e        [2F, D], K = rows  (fp32)
// In every GEMM the contracted index is the row index of at least one operand's storage, so those
// operands are MN-major: TMA loads 64 x 64 boxes with the 128-byte swizzle (one 1024-byte atom per
// 8 rows of K), and the UMMA descriptor gives the stride between 64-element MN chunks (LBO, 8 KB)
// and between 8-row K groups (SBO, 1 KB).
// Rows of dy_perm, dO and dGU live in a per-expert layout padded to multiples of 64 rows with zero
// rows, so the weight-gradient K loops may end inside a k-block: the zero rows of A annul whatever
// rows of B follow the segment.  Experts with no rows get zero weight gradients.
// Same pipeline as the forward tiled kernel: one persistent 192-thread CTA per SM, a static
// round-robin tile list built on the device, warp 0 TMA, warp 1 MMA (+TMEM), warps 2-5 epilogue,
// two 128 x 256 fp32 accumulators in TMEM, bounded waits everywhere.
#include <cuda.h>

#include <cstdlib>
#include <cstring>
#include <mutex>

#include "moe_common.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kThreads = 192;
constexpr int kMaxGroups = 1025;
constexpr int kStageA = kBM * kBK * 2;   // 16 KB
constexpr int kStageB = kBN * kBK * 2;   // 32 KB
constexpr int kStageBytes = kStageA + kStageB;
constexpr int kStages = 4;
constexpr int kAccCols = kBN;
constexpr int kBarBytes = 256;
constexpr int kStageBytesOut = 32 * 128;  // one epilogue warp's 32 x 32 fp32 chunk, 128-byte swizzled rows
constexpr int kTileTableBytes = (4 * (kMaxGroups + 1) + 127) / 128 * 128;  // keeps the staging 128-byte aligned
constexpr int kStageOffset = (kStages * kStageBytes + kBarBytes + kTileTableBytes + 1023) / 1024 * 1024;
constexpr size_t kSmemBytes = 1024 + (size_t)kStageOffset + 4 * kStageBytesOut;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kStageOffset % 1024 == 0, "swizzle-atom aligned output staging");

__host__ __device__ constexpr bool is_dw(int kind) { return kind == kBwdDwDown || kind == kBwdDwGateUp; }

struct alignas(64) BwdParams {
  CUtensorMap a_map[2];  // dx kinds: K-major A [rows, K], box {64, 128}; dw kinds: MN-major [rows, M], box {64, 64}
  CUtensorMap b_map[2];  // MN-major B [K rows, N cols], box {64, 64}
  CUtensorMap o_map[2];  // fp32 outputs (dX, weight gradients) [rows, N], box {32, 32}, 128-byte swizzle
  const int32_t* offsets[2];      // per group: rows [offsets[g], offsets[g+1]) of the unpadded layout
  const int32_t* pad_offsets[2];  // the same groups in the 64-row padded layout (NULL: = offsets)
  int n_groups[2];
  int m_rows[2];        // rows of a set without offsets (the shared expert: T)
  int K[2];             // dx kinds: contracted size (D or 2F)
  int M_total[2];       // dw kinds: rows of each weight gradient (D or 2F)
  int N_total[2];       // output columns (F, D, F or D)
  // epilogue operands
  const float* p_perm[2];          // kDxDown: router weight per unpadded row (NULL: 1)
  const uint16_t* gu_saved[2];     // kDxDown: forward pre-activations [rows, 2F] bf16 (g | u)
  uint16_t* dgu[2];                // kDxDown: dGU out, padded rows [.., 2F] bf16
  float* dp_part[2];               // kDxDown: [unpadded rows][n tiles] partial dp (NULL: not needed)
  float* out[2];                   // kDxGateUp: dX fp32 [padded rows, D]; dw kinds: [groups][M_total][N_total]
  int n_sets;
  int* err;
};

struct Tile {
  int set, g, rows, row0, prow0, m, n, kb;  // kb: k-blocks of this tile
};

__device__ __forceinline__ void group_rows(const BwdParams& p, int s, int g, int& row0, int& prow0, int& rows) {
  if (p.offsets[s] != nullptr) {
    row0 = p.offsets[s][g];
    rows = p.offsets[s][g + 1] - row0;
    prow0 = p.pad_offsets[s] != nullptr ? p.pad_offsets[s][g] : row0;
  } else {
    row0 = 0, prow0 = 0, rows = p.m_rows[s];
  }
}

template <int KIND>
__device__ __forceinline__ int group_tiles(const BwdParams& p, int s, int rows) {
  const int nt = (p.N_total[s] + kBN - 1) / kBN;
  if constexpr (is_dw(KIND)) return ((p.M_total[s] + kBM - 1) / kBM) * nt;  // even for empty groups (zeros)
  return rows > 0 ? ((rows + kBM - 1) / kBM) * nt : 0;
}

template <int KIND>
__device__ __forceinline__ Tile decode_tile(const BwdParams& p, const int* tile_start, int G, int t) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= t) lo = mid; else hi = mid - 1;
  }
  Tile ti;
  ti.set = lo < p.n_groups[0] ? 0 : 1;
  ti.g = ti.set == 0 ? lo : lo - p.n_groups[0];
  group_rows(p, ti.set, ti.g, ti.row0, ti.prow0, ti.rows);
  const int local = t - tile_start[lo];
  if constexpr (is_dw(KIND)) {
    const int mt = (p.M_total[ti.set] + kBM - 1) / kBM;
    ti.n = local / mt;
    ti.m = local - ti.n * mt;
    ti.kb = (ti.rows + kBK - 1) / kBK;
  } else {
    const int mt = (ti.rows + kBM - 1) / kBM;
    ti.n = local / mt;
    ti.m = local - ti.n * mt;
    ti.kb = p.K[ti.set] / kBK;
  }
  return ti;
}

// UMMA shared-memory descriptor, 128-byte swizzle: start, LBO, SBO (bytes), version 1
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// kind::f16, bf16 A and B, fp32 accumulator, M = 128, N = 256; A K-major (dx) or MN-major (dw), B MN-major
template <int KIND>
__host__ __device__ constexpr uint32_t bwd_idesc() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((is_dw(KIND) ? 1u : 0u) << 15) | (1u << 16) |
         ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);
}

__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + __expf(-z)); }

// A warp's 32 x 32 fp32 chunk (lane i holds row i's 32 columns in a[]) written to rows
// out + r * ld, r < n_rows, columns [0, 32).  Staged through shared memory: each lane stores its row
// as 8 float4 (with a pitch of 36 floats every 8-lane phase covers the 32 banks once), then lane l
// writes columns 4(l % 8).. of rows l / 8 + 4i: one instruction stores 4 rows x 128 contiguous
// bytes, and the 8 loads of a chunk are independent.
__device__ __forceinline__ void st_shared_f4(uint32_t addr, float a, float b, float c, float d) {
  asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

// TMA bulk store of a box from shared memory (tracked in this thread's bulk group)
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, uint32_t src, int32_t x, int32_t y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// A warp's 32 x 32 fp32 chunk (lane i holds row i's 32 columns in a[]) written to the output
// tensor at (col x, row y) by one TMA bulk store.  The rows are staged with the 128-byte swizzle
// the output map uses (16-byte chunk j of row r at position j ^ (r & 7)): every 8-lane phase of the
// staging stores covers the 32 banks once.  Rows and columns past the tensor's extent are clipped
// by TMA; callers never pass a box that reaches into another group's rows.
__device__ __forceinline__ void store_chunk_tma(uint8_t* stg, const uint32_t (&a)[32], const CUtensorMap* map,
                                                int x, int y) {
  const int lane = threadIdx.x & 31;
  if (lane == 0) bulk_wait_read_all();  // the previous chunk's store has read the staging buffer
  __syncwarp();
  const uint32_t row = smem_u32(stg) + lane * 128;
#pragma unroll
  for (int v = 0; v < 8; ++v)
    st_shared_f4(row + ((v ^ (lane & 7)) << 4), __uint_as_float(a[4 * v]), __uint_as_float(a[4 * v + 1]),
                 __uint_as_float(a[4 * v + 2]), __uint_as_float(a[4 * v + 3]));
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // generic stores -> the TMA's reads
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(map, smem_u32(stg), x, y);
    bulk_commit();
  }
}

template <int KIND>
__global__ void __launch_bounds__(kThreads, 1) bwd_gemm_kernel(const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  int* tile_start = reinterpret_cast<int*>(smem + kStages * kStageBytes + kBarBytes);
  uint8_t* stage_o = smem + kStageOffset;  // [4 epilogue warps][32 rows][128 B], 128-byte swizzle

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.n_groups[0] + (p.n_sets > 1 ? p.n_groups[1] : 0);
  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    fence_barrier_init();
    prefetch_tensormap(&p.a_map[0]);
    prefetch_tensormap(&p.b_map[0]);
    if (p.n_sets > 1) {
      prefetch_tensormap(&p.a_map[1]);
      prefetch_tensormap(&p.b_map[1]);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * kAccCols);
    tmem_relinquish();
  }
  pdl_wait();
  pdl_trigger();
  for (int g = threadIdx.x; g < G; g += kThreads) {
    const int s = g < p.n_groups[0] ? 0 : 1;
    const int gl = s == 0 ? g : g - p.n_groups[0];
    int row0, prow0, rows;
    group_rows(p, s, gl, row0, prow0, rows);
    tile_start[g] = group_tiles<KIND>(p, s, rows);
  }
  __syncthreads();
  if (warp == 0) {
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
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = tile_start[G];

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Tile ti = decode_tile<KIND>(p, tile_start, G, t);
        const CUtensorMap* am = &p.a_map[ti.set];
        const CUtensorMap* bm = &p.b_map[ti.set];
        for (int kb = 0; kb < ti.kb; ++kb, ++it) {
          const int st = it % kStages;
          if (!mbar_wait(&empty[st], ((it / kStages) & 1) ^ 1, kWaitLimitNs)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + st * kStageBytes;
          uint8_t* sb = sa + kStageA;
          mbar_arrive_expect_tx(&full[st], kStageBytes);
          int brow;  // first K row of B for this k-block
          if constexpr (is_dw(KIND)) {
            const int krow = ti.prow0 + kb * kBK;  // padded rows of A (dO or dGU)
            tma_load_2d(am, &full[st], sa, ti.m * kBM, krow);
            tma_load_2d(am, &full[st], sa + kStageA / 2, ti.m * kBM + 64, krow);
            brow = ti.row0 + kb * kBK;  // unpadded rows of B (h or x_perm)
          } else {
            tma_load_2d(am, &full[st], sa, kb * kBK, ti.prow0 + ti.m * kBM);
            brow = ti.g * p.K[ti.set] + kb * kBK;  // expert g's weight rows
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) tma_load_2d(bm, &full[st], sb + c * (kStageB / 4), ti.n * kBN + c * 64, brow);
        }
      }
      if (!ok) set_error(p.err, kErrTimeout);
      const uint32_t issued = it;
      for (int s = 0; s < kStages; ++s) {
        if ((uint32_t)s >= issued) break;
        const uint32_t last = issued - 1 - ((issued - 1 - s) % kStages);
        if (!mbar_wait(&full[s], (last / kStages) & 1, kWaitLimitNs)) set_error(p.err, kErrTimeout);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tl = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++tl) {
        const uint32_t buf = tl & 1, use = tl >> 1;
        if (!mbar_wait(&acc_empty[buf], (use & 1) ^ 1, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + buf * kAccCols;
        const Tile ti = decode_tile<KIND>(p, tile_start, G, t);
        for (int kb = 0; kb < ti.kb; ++kb, ++it) {
          const int st = it % kStages;
          if (!mbar_wait(&full[st], (it / kStages) & 1, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + st * kStageBytes), sb = sa + kStageA;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t adesc = is_dw(KIND) ? sw128_desc(sa + kk * 2048, 8192, 1024) : sw128_kmajor_desc(sa + kk * 32);
            umma_bf16(d, adesc, sw128_desc(sb + kk * 2048, 8192, 1024), bwd_idesc<KIND>(), (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[st]);
        }
        if (!ok) break;
        umma_commit(&acc_full[buf]);  // also for an empty tile (no MMAs): the epilogue writes zeros
      }
      if (!ok) set_error(p.err, kErrTimeout);
      if (it > 0) {
        const uint32_t last = it - 1;
        if (!mbar_wait(&empty[last % kStages], (last / kStages) & 1, kWaitLimitNs)) set_error(p.err, kErrTimeout);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;
    uint32_t tl = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tl) {
      const uint32_t buf = tl & 1, use = tl >> 1;
      if (!mbar_wait(&acc_full[buf], use & 1, kWaitLimitNs)) {
        set_error(p.err, kErrTimeout);
        break;
      }
      tc_fence_after();
      const Tile ti = decode_tile<KIND>(p, tile_start, G, t);
      const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + buf * kAccCols;
      const int s = ti.set;
      const int N = p.N_total[s];
      const int lrow = ti.m * kBM + q * 32 + lane;  // row of the tile in its group
      uint8_t* stg = stage_o + (warp - 2) * kStageBytesOut;
      const int wrow0 = ti.m * kBM + q * 32;  // this warp's first tile row
      if constexpr (is_dw(KIND)) {
        const int n_rows = min(32, p.M_total[s] - wrow0);  // 32 or <= 0: M_total is a multiple of 64
        const int orow = ti.g * p.M_total[s] + wrow0;
#pragma unroll 1
        for (int c0 = 0; c0 < kBN; c0 += 32) {
          const int col = ti.n * kBN + c0;
          if (col >= N) break;
          uint32_t a[32];
          if (ti.kb > 0) {
            tmem_ld_32x32b_x32(tacc + c0, a);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) a[j] = 0u;  // an expert without rows: zero gradient
          }
          if (n_rows > 0) store_chunk_tma(stg, a, &p.o_map[s], col, orow);
        }
      } else {
        const bool row_ok = lrow < ti.rows;
        const size_t prow = (size_t)ti.prow0 + lrow;  // padded row (A, dGU, dX)
        const size_t urow = (size_t)ti.row0 + lrow;   // unpadded row (p, saved g/u, dp)
        if constexpr (KIND == kBwdDxGateUp) {
          // 32-row boxes stay inside the group's 64-row padded span (or the shared set's T rows, where
          // TMA clips): wrow0 < rows, both wrow0 and the span are multiples of 32
          const int n_rows = min(32, ti.rows - wrow0);
          const int orow = ti.prow0 + wrow0;
#pragma unroll 1
          for (int c0 = 0; c0 < kBN; c0 += 32) {
            const int col = ti.n * kBN + c0;
            if (col >= N) break;
            uint32_t a[32];
            tmem_ld_32x32b_x32(tacc + c0, a);
            tmem_ld_wait();
            if (n_rows > 0) store_chunk_tma(stg, a, &p.o_map[s], col, orow);
          }
        } else {
          // kDxDown: SwiGLU backward.  N = F; saved g in columns [0, F), u in [F, 2F)
          const float pr = (row_ok && p.p_perm[s] != nullptr) ? p.p_perm[s][urow] : 1.0f;
          const uint16_t* gsrc = p.gu_saved[s] + urow * 2 * (size_t)N;
          uint16_t* drow = p.dgu[s] + prow * 2 * (size_t)N;
          float dp = 0.0f;
#pragma unroll 1
          for (int c0 = 0; c0 < kBN; c0 += 32) {
            const int col = ti.n * kBN + c0;
            if (col >= N) break;
            uint32_t a[32];
            tmem_ld_32x32b_x32(tacc + c0, a);
            tmem_ld_wait();
            if (!row_ok) continue;
            uint32_t gp[16], up[16], dgp[16], dup[16];
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const uint4 gv = *reinterpret_cast<const uint4*>(gsrc + col + 8 * v);
              const uint4 uv = *reinterpret_cast<const uint4*>(gsrc + N + col + 8 * v);
              gp[4 * v] = gv.x, gp[4 * v + 1] = gv.y, gp[4 * v + 2] = gv.z, gp[4 * v + 3] = gv.w;
              up[4 * v] = uv.x, up[4 * v + 1] = uv.y, up[4 * v + 2] = uv.z, up[4 * v + 3] = uv.w;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float dg2[2], du2[2];
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
                const float g = h2 ? bf16_hi(gp[i]) : bf16_lo(gp[i]);
                const float u = h2 ? bf16_hi(up[i]) : bf16_lo(up[i]);
                const float acc = __uint_as_float(a[2 * i + h2]);
                const float sg = sigmoidf_(g);
                const float silu = g * sg;
                const float dh = pr * acc;
                dg2[h2] = dh * u * sg * (1.0f + g * (1.0f - sg));
                du2[h2] = dh * silu;
                dp += acc * (silu * u);
              }
              dgp[i] = pack_bf16x2(dg2[0], dg2[1]);
              dup[i] = pack_bf16x2(du2[0], du2[1]);
            }
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              *reinterpret_cast<uint4*>(drow + col + 8 * v) = make_uint4(dgp[4 * v], dgp[4 * v + 1], dgp[4 * v + 2], dgp[4 * v + 3]);
              *reinterpret_cast<uint4*>(drow + N + col + 8 * v) =
                  make_uint4(dup[4 * v], dup[4 * v + 1], dup[4 * v + 2], dup[4 * v + 3]);
            }
          }
          if (row_ok && p.dp_part[s] != nullptr) p.dp_part[s][urow * ((N + kBN - 1) / kBN) + ti.n] = dp;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
    if (lane == 0) bulk_wait_all();  // every output store issued by this warp has been performed
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kAccCols);
  }
}

// ------------------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// bf16 row-major [rows, cols], box = 64 columns x box_rows, 128-byte swizzle
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || rows == 0 || cols == 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 row-major [rows, cols] output map for TMA stores: box 32 x 32, 128-byte swizzle
bool make_out_map(CUtensorMap* m, void* base, uint64_t rows, uint64_t cols) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || rows == 0 || cols == 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

template <int KIND>
cudaError_t launch(const BwdSetHost* sets, int n_sets, int* err, cudaStream_t s) {
  BwdParams p;
  memset(&p, 0, sizeof(p));
  p.n_sets = n_sets;
  p.err = err;
  for (int i = 0; i < n_sets; ++i) {
    const BwdSetHost& st = sets[i];
    // A: dx kinds K-major [a_rows, K] (box 128 rows); dw kinds MN-major [a_rows, M_total] (box 64 rows)
    if (!make_map(&p.a_map[i], st.a, (uint64_t)st.a_rows, (uint64_t)st.a_cols, is_dw(KIND) ? 64 : 128))
      return cudaErrorInvalidValue;
    if (!make_map(&p.b_map[i], st.b, (uint64_t)st.b_rows, (uint64_t)st.b_cols, 64)) return cudaErrorInvalidValue;
    if (is_dw(KIND) || KIND == kBwdDxGateUp) {
      // weight gradients: [groups * M_total, N]; dX: [a_rows (padded rows, or T), N]
      const uint64_t orows = is_dw(KIND) ? (uint64_t)st.n_groups * st.M_total : (uint64_t)st.a_rows;
      if (st.out == nullptr || !make_out_map(&p.o_map[i], st.out, orows, (uint64_t)st.N_total))
        return cudaErrorInvalidValue;
    }
    p.offsets[i] = st.offsets;
    p.pad_offsets[i] = st.pad_offsets;
    p.n_groups[i] = st.n_groups;
    p.m_rows[i] = st.m_rows;
    p.K[i] = st.K;
    p.M_total[i] = st.M_total;
    p.N_total[i] = st.N_total;
    p.p_perm[i] = st.p_perm;
    p.gu_saved[i] = st.gu_saved;
    p.dgu[i] = st.dgu;
    p.dp_part[i] = st.dp_part;
    p.out[i] = st.out;
  }
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(bwd_gemm_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  return launch_pdl(bwd_gemm_kernel<KIND>, dim3(sm_count()), dim3(kThreads), kSmemBytes, s, p);
}

}  // namespace

cudaError_t launch_bwd_gemm(BwdKind kind, const BwdSetHost* sets, int n_sets, int* err, cudaStream_t s) {
  if (n_sets < 1 || n_sets > 2) return cudaErrorInvalidValue;
  int groups = 0;
  for (int i = 0; i < n_sets; ++i) {
    const BwdSetHost& st = sets[i];
    if (st.N_total <= 0 || st.N_total % 64 != 0) return cudaErrorInvalidValue;
    if (!is_dw(kind) && (st.K <= 0 || st.K % 64 != 0)) return cudaErrorInvalidValue;
    if (is_dw(kind) && (st.M_total <= 0 || st.M_total % 64 != 0)) return cudaErrorInvalidValue;
    groups += st.n_groups;
  }
  if (groups > kMaxGroups) return cudaErrorInvalidValue;
  switch (kind) {
    case kBwdDxDown: return launch<kBwdDxDown>(sets, n_sets, err, s);
    case kBwdDxGateUp: return launch<kBwdDxGateUp>(sets, n_sets, err, s);
    case kBwdDwDown: return launch<kBwdDwDown>(sets, n_sets, err, s);
    case kBwdDwGateUp: return launch<kBwdDwGateUp>(sets, n_sets, err, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
