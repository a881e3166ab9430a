// grouped_gemm_sm100.cu -- step 3 of the layer: the experts' SwiGLU FFNs as grouped GEMMs over
// expert-contiguous rows, on the 5th-generation tensor cores (tcgen05.mma, fp32 accumulators in
// TMEM, operands staged in shared memory by TMA).
//
// gotburnout.io glossary "MoE", section 3 step 3: each selected expert runs the SwiGLU FFN
//     FFN(x) = (silu(x G^T) * (x U^T)) Down^T
// (the page's formula prints SiLU on the other factor; the packed gate_up tensor of
// dev.smart-guide.co.kr, section "La Solucion: WeightConverter", concatenates w1 then w3 on dim
// 1, and SiLU is taken on the first half, rows [0, F) of gate_up[e]).
// keryc.com "Mixture of Experts optimiza...", section "Ejecucion eficiente": runtime kernels
// want the experts packed in one contiguous tensor so the per-expert GEMMs can run grouped.
//
// One kernel template, two GEMMs, two regimes:
//   kGateUp : h[r, :]   = silu(A[r] G_e^T) * (A[r] U_e^T)             (SwiGLU in the epilogue)
//   kDown   : out[r, :] = row_scale[r] * (h[r] Down_e^T)  in fp32       (router weight in epilogue)
//   kRouter : logits[r, :] = x[r] W_g^T in fp32 (one group; split-K partial sums, reduced by the
//             top-k kernel in a fixed order)
//   tiled (prefill, NT = 0): a tile is 128 activation rows of one expert segment x 256 MMA
//       columns (gate_up: 128 gate + 128 up weight rows, so both halves of a SwiGLU output land
//       in the same TMEM lane; down: 256 weight rows).  MMA M=128, N=256, K=16.  The last tile
//       of a segment computes up to 127 padding rows, which are never stored.
//   streaming (decode, NT > 0): swap-AB.  A unit is 128 weight rows of one active expert (two
//       accumulators for gate_up) x the <= NT tokens routed to it, MMA M=128, N=NT.  Each active
//       expert's weights are read exactly once.
// Grid: one persistent CTA per SM walks a static round-robin list of tiles built on the device
// from the segment offsets (no host synchronisation).  Tiles are uniform (128 rows x 256
// columns x K), so CTAs b, b+1, ... stay in step on the m-tiles of one weight tile and share it
// through L2; the two SMs of a TPC, which take consecutive CTAs, even merge their requests for
// it.  Warp roles per CTA:
//   warp 0 (one lane)  : TMA producer, multi-stage ring of shared-memory stages (mbarrier full/empty)
//   warp 1 (one lane)  : tcgen05.mma issuer; commits free a stage / publish an accumulator
//   warps 2-5          : epilogue; tcgen05.ld of their 32-lane quarter of TMEM, math, global stores
// Two TMEM accumulators alternate so the epilogue of tile i overlaps the MMAs of tile i+1.
// Every mbarrier wait is bounded (1 s); on expiry the kernel records kErrTimeout, drains its
// own in-flight copies and MMAs, frees TMEM and returns.
#include <cuda.h>

#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "moe_common.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;            // MMA M
constexpr int kBK = 64;             // K per stage (one 128-byte swizzle row of bf16)
constexpr int kThreads = 192;       // 6 warps
constexpr int kMaxGroups = 1025;    // E <= 1024 routed + 1 shared
constexpr int kTileBytesA = kBM * kBK * 2;  // 16 KB
constexpr int kBarBytes = 256;      // mbarriers and the TMEM address slot

struct alignas(64) GemmParams {
  CUtensorMap a_map[2];  // activations per set (box rows: 128 tiled / NT streaming)
  CUtensorMap w_map[2];  // weights per set (box rows: 128, or 256 for tiled kDown)
  const int32_t* offsets[2];
  void* out[2];  // kGateUp: bf16 h [rows, F]; kDown: fp32 [rows, D]
  const float* row_scale[2];
  int n_groups[2];
  int m_rows[2];
  int n_out[2];
  int w_rows[2];  // weight rows per group: 2F (gate_up) or D (down)
  int k_blocks[2];  // K / 64 per set (down: F routed, Fs shared)
  int ld_out[2];    // row stride of the output (elements)
  int k_splits;     // kRouter: K is split into this many contiguous k-block ranges
  uint16_t* save_gu[2];  // tiled kGateUp in a training forward: g | u [rows, 2F] bf16, or NULL
  int n_sets;
  int withhold_first_load;  // test only: never issue the first stage's copies (its wait then times out)
  int* err;
};

template <int KIND, int NT>
struct Cfg {
  static constexpr bool kTiled = (NT == 0);
  // shared-memory stage: [A (16 KB) | B ...]
  // (kRouter is laid out like kDown: one weight operand)
  static constexpr int kStageBytes = kTiled ? (kTileBytesA + 256 * kBK * 2)
                                            : (KIND == kGateUp ? 2 * kTileBytesA + NT * kBK * 2
                                                               : kTileBytesA + NT * kBK * 2);
  static constexpr int kStages = kTiled ? 4 : (KIND == kGateUp ? 5 : 8);
  static constexpr int kAccCols = kTiled ? 256 : (KIND == kGateUp ? 2 * NT : NT);
  static constexpr int kTmemCols = (2 * kAccCols <= 32) ? 32 : (2 * kAccCols <= 64) ? 64
                                 : (2 * kAccCols <= 128) ? 128 : (2 * kAccCols <= 256) ? 256 : 512;
  static constexpr int kOutPerTile = kTiled ? (KIND == kGateUp ? 128 : 256) : 128;
  static constexpr uint32_t kIdesc = kTiled ? idesc_bf16_f32(kBM, 256) : idesc_bf16_f32(kBM, NT);
  static constexpr size_t kSmemBytes =
      1024 /*alignment slack*/ + (size_t)kStages * kStageBytes + kBarBytes + 4 * (kMaxGroups + 1);
  static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte alignment");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct Tile {
  int set, gl, row0, rows, m, n;
  int ks, kb0, kb1;  // split index and k-block range [kb0, kb1)
};

__device__ __forceinline__ void group_rows(const GemmParams& p, int s, int gl, int& row0, int& rows) {
  if (p.offsets[s] != nullptr) {
    row0 = p.offsets[s][gl];
    rows = p.offsets[s][gl + 1] - row0;
  } else {
    row0 = 0;
    rows = p.m_rows[s];
  }
}

template <int KIND, int NT>
__device__ __forceinline__ int group_tiles(const GemmParams& p, int s, int rows) {
  using C = Cfg<KIND, NT>;
  const int nt = (p.n_out[s] + C::kOutPerTile - 1) / C::kOutPerTile;
  if (rows <= 0) return 0;
  const int splits = KIND == kRouter ? p.k_splits : 1;
  if constexpr (C::kTiled) return ((rows + kBM - 1) / kBM) * nt * splits;
  return nt * splits;
}

template <int KIND, int NT>
__device__ __forceinline__ Tile decode_tile(const GemmParams& p, const int* tile_start, int G, int t) {
  int lo = 0, hi = G - 1;  // largest g with tile_start[g] <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= t) lo = mid; else hi = mid - 1;
  }
  Tile ti;
  ti.set = lo < p.n_groups[0] ? 0 : 1;
  ti.gl = ti.set == 0 ? lo : lo - p.n_groups[0];
  group_rows(p, ti.set, ti.gl, ti.row0, ti.rows);
  int local = t - tile_start[lo];
  const int kbs = p.k_blocks[ti.set];
  ti.ks = 0, ti.kb0 = 0, ti.kb1 = kbs;
  if constexpr (KIND == kRouter) {
    const int per = (kbs + p.k_splits - 1) / p.k_splits;
    ti.ks = local % p.k_splits;
    local /= p.k_splits;
    ti.kb0 = ti.ks * per;
    ti.kb1 = min(kbs, ti.kb0 + per);
  }
  if constexpr (NT == 0) {
    const int mt = (ti.rows + kBM - 1) / kBM;
    ti.n = local / mt;
    ti.m = local - ti.n * mt;
  } else {
    ti.n = local;
    ti.m = 0;
  }
  return ti;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }

template <int KIND, int NT>
__global__ void __launch_bounds__(kThreads, 1) grouped_gemm_kernel(const __grid_constant__ GemmParams p) {
  using C = Cfg<KIND, NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* acc_full = empty + C::kStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  int* tile_start = reinterpret_cast<int*>(smem + C::kStages * C::kStageBytes + kBarBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.n_groups[0] + (p.n_sets > 1 ? p.n_groups[1] : 0);

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    fence_barrier_init();
    prefetch_tensormap(&p.a_map[0]);
    prefetch_tensormap(&p.w_map[0]);
    if (p.n_sets > 1) {
      prefetch_tensormap(&p.a_map[1]);
      prefetch_tensormap(&p.w_map[1]);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  // everything above overlaps the previous kernel; the offsets and operands are its outputs
  pdl_wait();
  pdl_trigger();
  // per-group tile counts, then an exclusive scan (warp 0) -> tile_start[0..G]
  for (int g = threadIdx.x; g < G; g += kThreads) {
    const int s = g < p.n_groups[0] ? 0 : 1;
    const int gl = s == 0 ? g : g - p.n_groups[0];
    int row0, rows;
    group_rows(p, s, gl, row0, rows);
    if (NT > 0 && rows > NT) set_error(p.err, kErrBadIndex);  // a segment longer than the token tile
    tile_start[g] = group_tiles<KIND, NT>(p, s, rows);
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
        const Tile ti = decode_tile<KIND, NT>(p, tile_start, G, t);
        const CUtensorMap* amap = &p.a_map[ti.set];
        const CUtensorMap* wmap = &p.w_map[ti.set];
        const int wbase = ti.gl * p.w_rows[ti.set];
        for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++it) {
          const int stage = it % C::kStages;
          if (!mbar_wait(&empty[stage], ((it / C::kStages) & 1) ^ 1, kWaitLimitNs)) {
            ok = false;
            break;
          }
          uint8_t* sb = smem + stage * C::kStageBytes;
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
          if (p.withhold_first_load && it == 0) continue;  // the bytes never arrive
          const int kx = kb * kBK;
          if constexpr (C::kTiled) {
            tma_load_2d(amap, &full[stage], sb, kx, ti.row0 + ti.m * kBM);
            if constexpr (KIND == kGateUp) {
              const int F = p.n_out[ti.set];
              tma_load_2d(wmap, &full[stage], sb + kTileBytesA, kx, wbase + ti.n * 128);
              tma_load_2d(wmap, &full[stage], sb + 2 * kTileBytesA, kx, wbase + F + ti.n * 128);
            } else {
              tma_load_2d(wmap, &full[stage], sb + kTileBytesA, kx, wbase + ti.n * 256);
            }
          } else {
            if constexpr (KIND == kGateUp) {
              const int F = p.n_out[ti.set];
              tma_load_2d(wmap, &full[stage], sb, kx, wbase + ti.n * 128);
              tma_load_2d(wmap, &full[stage], sb + kTileBytesA, kx, wbase + F + ti.n * 128);
              tma_load_2d(amap, &full[stage], sb + 2 * kTileBytesA, kx, ti.row0);
            } else {
              tma_load_2d(wmap, &full[stage], sb, kx, wbase + ti.n * 128);
              tma_load_2d(amap, &full[stage], sb + kTileBytesA, kx, ti.row0);
            }
          }
        }
      }
      if (!ok) set_error(p.err, kErrTimeout);
      // drain: every issued stage load must have landed before shared memory is released
      const uint32_t issued = it;
      for (int s = 0; s < C::kStages; ++s) {
        if ((uint32_t)s >= issued) break;
        const uint32_t last = issued - 1 - ((issued - 1 - s) % C::kStages);  // last index with it % S == s
        if (!mbar_wait(&full[s], (last / C::kStages) & 1, kWaitLimitNs)) set_error(p.err, kErrTimeout);
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
        const uint32_t d = tmem_base + buf * C::kAccCols;
        const Tile ti = decode_tile<KIND, NT>(p, tile_start, G, t);
        for (int kb = ti.kb0; kb < ti.kb1; ++kb, ++it) {
          const int stage = it % C::kStages;
          if (!mbar_wait(&full[stage], (it / C::kStages) & 1, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * C::kStageBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t acc = (kb > ti.kb0 || kk > 0) ? 1u : 0u;
            if constexpr (C::kTiled) {
              umma_bf16(d, sw128_kmajor_desc(sa + kk * 32), sw128_kmajor_desc(sa + kTileBytesA + kk * 32),
                        C::kIdesc, acc);
            } else if constexpr (KIND == kGateUp) {
              const uint64_t bdesc = sw128_kmajor_desc(sa + 2 * kTileBytesA + kk * 32);
              umma_bf16(d, sw128_kmajor_desc(sa + kk * 32), bdesc, C::kIdesc, acc);
              umma_bf16(d + NT, sw128_kmajor_desc(sa + kTileBytesA + kk * 32), bdesc, C::kIdesc, acc);
            } else {
              umma_bf16(d, sw128_kmajor_desc(sa + kk * 32), sw128_kmajor_desc(sa + kTileBytesA + kk * 32),
                        C::kIdesc, acc);
            }
          }
          umma_commit(&empty[stage]);  // frees the stage once these MMAs have read it
        }
        if (!ok) break;
        umma_commit(&acc_full[buf]);  // accumulator ready for the epilogue
      }
      if (!ok) set_error(p.err, kErrTimeout);
      if (it > 0) {  // the last commit covers every MMA issued before it
        const uint32_t last = it - 1;
        if (!mbar_wait(&empty[last % C::kStages], (last / C::kStages) & 1, kWaitLimitNs))
          set_error(p.err, kErrTimeout);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    uint32_t tl = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tl) {
      const uint32_t buf = tl & 1, use = tl >> 1;
      if (!mbar_wait(&acc_full[buf], use & 1, kWaitLimitNs)) {
        set_error(p.err, kErrTimeout);
        break;
      }
      tc_fence_after();
      const Tile ti = decode_tile<KIND, NT>(p, tile_start, G, t);
      const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + buf * C::kAccCols;
      const int n_out = p.n_out[ti.set];
      uint16_t* out_h = static_cast<uint16_t*>(p.out[ti.set]);
      float* out_f = static_cast<float*>(p.out[ti.set]);
      if constexpr (C::kTiled) {
        const int r_local = ti.m * kBM + q * 32 + lane;
        const bool row_ok = r_local < ti.rows;
        const size_t grow = (size_t)(ti.row0 + r_local);
        if constexpr (KIND == kGateUp) {
#pragma unroll 1
          for (int c0 = 0; c0 < 128; c0 += 32) {
            const int col = ti.n * 128 + c0;
            if (col >= n_out) break;
            uint32_t g[32], u[32];
            tmem_ld_32x32b_x32(tacc + c0, g);
            tmem_ld_32x32b_x32(tacc + 128 + c0, u);
            tmem_ld_wait();
            if (row_ok && p.save_gu[ti.set] != nullptr) {  // the backward pass's SwiGLU inputs
              uint16_t* srow = p.save_gu[ti.set] + grow * 2 * n_out;
              uint32_t gk[16], uk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                gk[i] = pack_bf16x2(__uint_as_float(g[2 * i]), __uint_as_float(g[2 * i + 1]));
                uk[i] = pack_bf16x2(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1]));
              }
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                reinterpret_cast<uint4*>(srow + col)[v] = make_uint4(gk[4 * v], gk[4 * v + 1], gk[4 * v + 2], gk[4 * v + 3]);
                reinterpret_cast<uint4*>(srow + n_out + col)[v] =
                    make_uint4(uk[4 * v], uk[4 * v + 1], uk[4 * v + 2], uk[4 * v + 3]);
              }
            }
            if (row_ok) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack_bf16x2(silu_mul(__uint_as_float(g[2 * i]), __uint_as_float(u[2 * i])),
                                    silu_mul(__uint_as_float(g[2 * i + 1]), __uint_as_float(u[2 * i + 1])));
              uint4* dst = reinterpret_cast<uint4*>(out_h + grow * n_out + col);
#pragma unroll
              for (int v = 0; v < 4; ++v) dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
            }
          }
        } else if constexpr (KIND == kRouter) {
          // partial logits of split ks: out[ks][row][col], row stride ld (a multiple of 32)
          const int ld = p.ld_out[ti.set];
          float* orow = out_f + ((size_t)ti.ks * p.m_rows[ti.set] + grow) * ld;
#pragma unroll 1
          for (int c0 = 0; c0 < 256; c0 += 32) {
            const int col = ti.n * 256 + c0;
            if (col >= n_out) break;
            uint32_t a[32];
            tmem_ld_32x32b_x32(tacc + c0, a);
            tmem_ld_wait();
            if (row_ok) {
              float4* dst = reinterpret_cast<float4*>(orow + col);
#pragma unroll
              for (int v = 0; v < 8; ++v)
                dst[v] = make_float4(__uint_as_float(a[4 * v]), __uint_as_float(a[4 * v + 1]),
                                     __uint_as_float(a[4 * v + 2]), __uint_as_float(a[4 * v + 3]));
            }
          }
        } else {
          const float sc = (row_ok && p.row_scale[ti.set] != nullptr) ? p.row_scale[ti.set][grow] : 1.0f;
#pragma unroll 1
          for (int c0 = 0; c0 < 256; c0 += 32) {
            const int col = ti.n * 256 + c0;
            if (col >= n_out) break;
            uint32_t a[32];
            tmem_ld_32x32b_x32(tacc + c0, a);
            tmem_ld_wait();
            if (row_ok) {
              float4* dst = reinterpret_cast<float4*>(out_f + grow * n_out + col);
#pragma unroll
              for (int v = 0; v < 8; ++v)
                dst[v] = make_float4(__uint_as_float(a[4 * v]) * sc, __uint_as_float(a[4 * v + 1]) * sc,
                                     __uint_as_float(a[4 * v + 2]) * sc, __uint_as_float(a[4 * v + 3]) * sc);
            }
          }
        }
      } else {
        // streaming: TMEM lane <-> output column (weight row), TMEM column <-> token
        const int col = ti.n * 128 + q * 32 + lane;
        const bool col_ok = col < n_out;
#pragma unroll 1
        for (int j0 = 0; j0 < NT; j0 += 16) {
          if (j0 >= ti.rows) break;
          if constexpr (KIND == kGateUp) {
            uint32_t g[16], u[16];
            tmem_ld_32x32b_x16(tacc + j0, g);
            tmem_ld_32x32b_x16(tacc + NT + j0, u);
            tmem_ld_wait();
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int j = j0 + jj;
              if (j < ti.rows && col_ok) {
                const float h = silu_mul(__uint_as_float(g[jj]), __uint_as_float(u[jj]));
                out_h[(size_t)(ti.row0 + j) * n_out + col] = (uint16_t)(pack_bf16x2(h, 0.f) & 0xFFFFu);
              }
            }
          } else if constexpr (KIND == kRouter) {
            uint32_t a[16];
            tmem_ld_32x32b_x16(tacc + j0, a);
            tmem_ld_wait();
            const int ld = p.ld_out[ti.set];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int j = j0 + jj;
              if (j < ti.rows && col_ok)
                out_f[((size_t)ti.ks * p.m_rows[ti.set] + ti.row0 + j) * ld + col] = __uint_as_float(a[jj]);
            }
          } else {
            uint32_t a[16];
            tmem_ld_32x32b_x16(tacc + j0, a);
            tmem_ld_wait();
            const float* rs = p.row_scale[ti.set];
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
              const int j = j0 + jj;
              if (j < ti.rows && col_ok) {
                const float sc = rs != nullptr ? rs[ti.row0 + j] : 1.0f;
                out_f[(size_t)(ti.row0 + j) * n_out + col] = __uint_as_float(a[jj]) * sc;
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ------------------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
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

// 2-D bf16 row-major [rows, cols] map, box = 64 columns (128 bytes) x box_rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr || rows == 0 || cols == 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

template <int KIND, int NT>
cudaError_t launch_kernel(const GemmSetHost* sets, int n_sets, int k_splits, int* err, cudaStream_t s) {
  using C = Cfg<KIND, NT>;
  GemmParams p;
  memset(&p, 0, sizeof(p));
  p.n_sets = n_sets;
  p.k_splits = k_splits;
  p.err = err;
  p.withhold_first_load = (KIND != kRouter && test_withhold_this_launch()) ? 1 : 0;
  const uint32_t a_box = C::kTiled ? kBM : NT;
  const uint32_t w_box = (C::kTiled && KIND != kGateUp) ? 256 : 128;
  for (int i = 0; i < n_sets; ++i) {
    const GemmSetHost& st = sets[i];
    const int K = st.K;
    p.k_blocks[i] = K / kBK;
    p.w_rows[i] = KIND == kGateUp ? 2 * st.n_out : st.n_out;
    if (!make_map(&p.a_map[i], st.a, (uint64_t)st.a_rows, (uint64_t)K, a_box)) return cudaErrorInvalidValue;
    if (!make_map(&p.w_map[i], st.w, (uint64_t)st.n_groups * p.w_rows[i], (uint64_t)K, w_box))
      return cudaErrorInvalidValue;
    p.offsets[i] = st.offsets;
    p.out[i] = st.out;
    p.row_scale[i] = st.row_scale;
    p.ld_out[i] = st.ld_out > 0 ? st.ld_out : st.n_out;
    p.save_gu[i] = (KIND == kGateUp && NT == 0) ? st.save_gu : nullptr;
    p.n_groups[i] = st.n_groups;
    p.m_rows[i] = st.m_rows;
    p.n_out[i] = st.n_out;
  }
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<KIND, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  return launch_pdl(grouped_gemm_kernel<KIND, NT>, dim3(num_sms()), dim3(kThreads), C::kSmemBytes, s, p);
}

}  // namespace

bool test_withhold_this_launch() {
  static std::atomic<int> remaining{0};
  static std::once_flag once;
  std::call_once(once, [] {
    const char* v = getenv("MOE_TEST_WITHHOLD_LOAD");
    remaining.store(v != nullptr ? atoi(v) : 0);
  });
  int r = remaining.load();
  while (r > 0 && !remaining.compare_exchange_weak(r, r - 1)) {
  }
  return r > 0;
}

cudaError_t launch_grouped_gemm(GemmKind kind, const GemmSetHost* sets, int n_sets, int decode_nt, int* err,
                                cudaStream_t s) {
  if (n_sets < 1 || n_sets > 2) return cudaErrorInvalidValue;
  int groups = 0;
  for (int i = 0; i < n_sets; ++i) {
    if (sets[i].K <= 0 || sets[i].K % kBK != 0) return cudaErrorInvalidValue;
    groups += sets[i].n_groups;
  }
  if (groups > kMaxGroups) return cudaErrorInvalidValue;
  if (kind == kGateUp) {
    switch (decode_nt) {
      case 0: return launch_kernel<kGateUp, 0>(sets, n_sets, 1, err, s);
      case 16: return launch_kernel<kGateUp, 16>(sets, n_sets, 1, err, s);
      case 32: return launch_kernel<kGateUp, 32>(sets, n_sets, 1, err, s);
      case 48: return launch_kernel<kGateUp, 48>(sets, n_sets, 1, err, s);
      case 64: return launch_kernel<kGateUp, 64>(sets, n_sets, 1, err, s);
    }
  } else {
    switch (decode_nt) {
      case 0: return launch_kernel<kDown, 0>(sets, n_sets, 1, err, s);
      case 16: return launch_kernel<kDown, 16>(sets, n_sets, 1, err, s);
      case 32: return launch_kernel<kDown, 32>(sets, n_sets, 1, err, s);
      case 48: return launch_kernel<kDown, 48>(sets, n_sets, 1, err, s);
      case 64: return launch_kernel<kDown, 64>(sets, n_sets, 1, err, s);
    }
  }
  return cudaErrorInvalidValue;
}

int router_k_splits(int T, int D, int E, int num_sm) {
  const int kbs = D / kBK;
  const long long base = T <= 64 ? (E + 127) / 128 : (long long)((T + kBM - 1) / kBM) * ((E + 255) / 256);
  long long want = (num_sm + base - 1) / base;  // enough tiles to give every SM one
  if (want > 16) want = 16;                      // bounds the partial sums the top-k kernel adds
  if (want < 1) want = 1;
  if (want > kbs) want = kbs;
  const int per = (int)((kbs + want - 1) / want);
  return (kbs + per - 1) / per;  // every split non-empty
}

int router_k_splits(int T, int D, int E) { return router_k_splits(T, D, E, num_sms()); }

cudaError_t launch_router_gemm(const uint16_t* x, const uint16_t* wg, int T, int D, int E, float* partials, int ld,
                               int k_splits, int* err, cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  GemmSetHost st;
  memset(&st, 0, sizeof(st));
  st.K = D, st.a = x, st.a_rows = T, st.w = wg, st.n_groups = 1, st.offsets = nullptr, st.m_rows = T;
  st.n_out = E, st.out = partials, st.row_scale = nullptr, st.ld_out = ld;
  if (T > 64) return launch_kernel<kRouter, 0>(&st, 1, k_splits, err, s);
  switch ((T + 15) / 16 * 16) {
    case 16: return launch_kernel<kRouter, 16>(&st, 1, k_splits, err, s);
    case 32: return launch_kernel<kRouter, 32>(&st, 1, k_splits, err, s);
    case 48: return launch_kernel<kRouter, 48>(&st, 1, k_splits, err, s);
    default: return launch_kernel<kRouter, 64>(&st, 1, k_splits, err, s);
  }
}

}  // namespace moe
