// Token-wide grouped GEMMs (sm_100a, tcgen05 + TMEM + TMA) for the expert FFN of the MoE layer:
//   gate_up: h = silu(x_e G_e^T) * (x_e U_e^T)   (gotburnout.io glossary "MoE", section 3 step 3,
//            SwiGLU; the packed gate_up_proj [E, 2F, D] of dev.smart-guide.co.kr "La Solucion:
//            WeightConverter": rows [0, F) gate, [F, 2F) up)
//   down:    o = p * (h_e Down_e^T)              (section 3 step 4, weighted by the router's p)
// over the expert-contiguous segments of the permuted rows (keryc.com "Ejecucion eficiente:
// backends de expertos", the grouped backend), plus the always-on shared expert as a second
// operand set (gotburnout.io, section 2 item 3).
//
// Orientation.  The MMA's M operand is 128 weight rows (gate_up: 64 gate rows stacked on the 64
// up rows of the same output columns; down: 128 output columns), and N is up to 256 tokens of one
// segment: TMEM lane = output column, TMEM column = token.  A segment of R rows becomes
// ceil(R / 256) token tiles, the last with N = its rows rounded up to 16.  Compared with
// 128-token x 256-output tiles this drops the padding of every segment's last tile to < 16 rows
// (at N >= 96, where an MMA's time follows N) and reads each weight tile once per 256 tokens.
//
// Kernel layout (persistent, one CTA per SM, 192 threads):
//   warp 0     TMA producer: per 64-wide K block, the weight tile (16 KB, one copy; gate_up's
//              through a 4-D view that stacks the gate and up rows) and the token rows
//              (one 256-row box for a full tile, else ceil(rows / 64) boxes of 64 rows, 8 KB
//              each) into a 4-stage ring;
//   warp 1     TMEM allocator and MMA issuer (one thread): 4 x tcgen05.mma M=128, N=round16(rows),
//              K=16 per stage into one of two 256-column accumulators;
//   warps 2-5  epilogue: per 32-token chunk, tcgen05.ld of the warp's 32 lanes, a transpose
//              through a padded shared-memory stage, then row-contiguous stores (SwiGLU or the p
//              scale fused).
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

constexpr int kWT = 256;          // token tile (MMA N at most)
constexpr int kWM = 128;          // weight rows per tile (MMA M)
constexpr int kWBK = 64;          // K per stage
constexpr int kWThreads = 192;
constexpr int kWStages = 4;
constexpr int kWMaxGroups = 1025;  // E <= 1024 routed + 1 shared
constexpr int kWTileA = kWM * kWBK * 2;         // 16 KB of weights per stage
constexpr int kWBox = 64 * kWBK * 2;            // 8 KB: one 64-row box of tokens
constexpr int kWStageBytes = kWTileA + kWT * kWBK * 2;  // 48 KB
constexpr int kWChunk = 32;                     // tokens per epilogue chunk
constexpr int kWPitch = 144;                    // fp32 words per staged token row (128 + 16)
constexpr int kWStagingBytes = kWChunk * kWPitch * 4;  // 18 KB
constexpr int kWBarBytes = 256;
constexpr size_t kWSmemBytes = 1024 + (size_t)kWStages * kWStageBytes + kWStagingBytes + kWBarBytes +
                               4 * (kWMaxGroups + 1);
static_assert(kWSmemBytes <= 232448, "shared memory budget");
static_assert(kWStageBytes % 1024 == 0 && kWStagingBytes % 16 == 0, "alignment");

struct alignas(64) WideParams {
  CUtensorMap t_map[2];     // token operand per set (x_perm / x / h), box 64 K x 64 rows
  CUtensorMap t_map256[2];  // the same tensor, box 64 K x 256 rows (full token tiles: one copy)
  CUtensorMap w_map[2];  // weights per set: down [rows, K], box 64 K x 128 rows; gate_up viewed as
                         // [groups][2 halves][F rows][K], box 64 K x 64 rows x 2 halves (the
                         // gate and up rows of 64 output columns in one copy)
  const int32_t* offsets[2];
  void* out[2];          // gate_up: bf16 h [rows, F]; down: fp32 [rows, D]
  const float* row_scale[2];
  uint16_t* save_gu[2];  // gate_up in a training forward: g | u [rows, 2F] bf16, or NULL
  int n_groups[2];
  int m_rows[2];
  int n_out[2];
  int w_rows[2];    // weight rows per group: 2F (gate_up) or D (down)
  int k_blocks[2];  // K / 64
  int n_sets;
  int withhold_first_load;  // test only: never issue the first stage's copies (its wait then times out)
  int* err;
};

struct WTile {
  int set, gl, row0, rows, m, n;
};

__device__ __forceinline__ void w_group_rows(const WideParams& p, int s, int gl, int& row0, int& rows) {
  if (p.offsets[s] != nullptr) {
    row0 = p.offsets[s][gl];
    rows = p.offsets[s][gl + 1] - row0;
  } else {
    row0 = 0;
    rows = p.m_rows[s];
  }
}

// output columns per tile: gate_up 64 (64 gate + 64 up weight rows), down 128
template <int KIND>
__host__ __device__ constexpr int w_cols_per_tile() {
  return KIND == kGateUp ? 64 : 128;
}

template <int KIND>
__device__ __forceinline__ int w_group_tiles(const WideParams& p, int s, int rows) {
  if (rows <= 0) return 0;
  const int nt = (p.n_out[s] + w_cols_per_tile<KIND>() - 1) / w_cols_per_tile<KIND>();
  return ((rows + kWT - 1) / kWT) * nt;
}

// tile t -> (group, token tile m, column tile n), token tiles fastest: the CTAs that read one
// weight tile run side by side and share it through L2, and the few token tiles of a segment stay
// in L2 while its column tiles pass.
template <int KIND>
__device__ __forceinline__ WTile w_decode(const WideParams& p, const int* tile_start, int G, int t) {
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= t) lo = mid; else hi = mid - 1;
  }
  WTile ti;
  ti.set = lo < p.n_groups[0] ? 0 : 1;
  ti.gl = ti.set == 0 ? lo : lo - p.n_groups[0];
  w_group_rows(p, ti.set, ti.gl, ti.row0, ti.rows);
  const int local = t - tile_start[lo];
  const int mt = (ti.rows + kWT - 1) / kWT;
  ti.n = local / mt;
  ti.m = local - ti.n * mt;
  return ti;
}

// tokens of tile ti (1..256)
__device__ __forceinline__ int w_tile_tokens(const WTile& ti) { return min(kWT, ti.rows - ti.m * kWT); }

__device__ __forceinline__ float w_silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }

// barrier 1 over the 128 epilogue threads (warps 2..5)
__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// the same barrier, returning whether any of the 128 threads passed pred = true
__device__ __forceinline__ bool epi_any(bool pred) {
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

__device__ __forceinline__ void st_shared_f32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

__device__ __forceinline__ void tma_load_4d(const CUtensorMap* map, uint64_t* bar, void* dst, int32_t x, int32_t y,
                                            int32_t z, int32_t w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}

template <int KIND>
__global__ void __launch_bounds__(kWThreads, 1) grouped_gemm_wide_kernel(const __grid_constant__ WideParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + kWStages * kWStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + kWStagingBytes);
  uint64_t* empty = full + kWStages;
  uint64_t* acc_full = empty + kWStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  int* tile_start = reinterpret_cast<int*>(staging + kWStagingBytes + kWBarBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.n_groups[0] + (p.n_sets > 1 ? p.n_groups[1] : 0);

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < kWStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    fence_barrier_init();
    for (int s = 0; s < p.n_sets; ++s) {
      prefetch_tensormap(&p.t_map[s]);
      prefetch_tensormap(&p.t_map256[s]);
      prefetch_tensormap(&p.w_map[s]);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * kWT);
    tmem_relinquish();
  }
  // everything above overlaps the previous kernel; offsets and operands are its outputs
  pdl_wait();
  pdl_trigger();
  for (int g = threadIdx.x; g < G; g += kWThreads) {
    const int s = g < p.n_groups[0] ? 0 : 1;
    const int gl = s == 0 ? g : g - p.n_groups[0];
    int row0, rows;
    w_group_rows(p, s, gl, row0, rows);
    tile_start[g] = w_group_tiles<KIND>(p, s, rows);
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
        const WTile ti = w_decode<KIND>(p, tile_start, G, t);
        const int nb = (w_tile_tokens(ti) + 63) / 64;  // 64-row token boxes this tile needs
        const int wbase = ti.gl * p.w_rows[ti.set];
        const int trow = ti.row0 + ti.m * kWT;
        for (int kb = 0; kb < p.k_blocks[ti.set]; ++kb, ++it) {
          const int stage = it % kWStages;
          if (!mbar_wait(&empty[stage], ((it / kWStages) & 1) ^ 1, kWaitLimitNs)) {
            ok = false;
            break;
          }
          uint8_t* sb = smem + stage * kWStageBytes;
          mbar_arrive_expect_tx(&full[stage], kWTileA + nb * kWBox);
          if (p.withhold_first_load && it == 0) continue;  // the bytes never arrive
          const int kx = kb * kWBK;
          if constexpr (KIND == kGateUp) {
            tma_load_4d(&p.w_map[ti.set], &full[stage], sb, kx, ti.n * 64, 0, ti.gl);  // 64 gate rows, then 64 up
          } else {
            tma_load_2d(&p.w_map[ti.set], &full[stage], sb, kx, wbase + ti.n * 128);
          }
          if (nb == kWT / 64)
            tma_load_2d(&p.t_map256[ti.set], &full[stage], sb + kWTileA, kx, trow);
          else
            for (int b = 0; b < nb; ++b)
              tma_load_2d(&p.t_map[ti.set], &full[stage], sb + kWTileA + b * kWBox, kx, trow + b * 64);
        }
      }
      if (!ok) set_error(p.err, kErrTimeout);
      // drain: every issued stage load must have landed before shared memory is released
      const uint32_t issued = it;
      for (int s = 0; s < kWStages; ++s) {
        if ((uint32_t)s >= issued) break;
        const uint32_t last = issued - 1 - ((issued - 1 - s) % kWStages);  // last index with it % S == s
        if (!mbar_wait(&full[s], (last / kWStages) & 1, kWaitLimitNs)) set_error(p.err, kErrTimeout);
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
        const uint32_t d = tmem_base + buf * kWT;
        const WTile ti = w_decode<KIND>(p, tile_start, G, t);
        const uint32_t idesc = idesc_bf16_f32(kWM, (w_tile_tokens(ti) + 15) / 16 * 16);
        for (int kb = 0; kb < p.k_blocks[ti.set]; ++kb, ++it) {
          const int stage = it % kWStages;
          if (!mbar_wait(&full[stage], (it / kWStages) & 1, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * kWStageBytes);
#pragma unroll
          for (int kk = 0; kk < kWBK / 16; ++kk)
            umma_bf16(d, sw128_kmajor_desc(sa + kk * 32), sw128_kmajor_desc(sa + kWTileA + kk * 32), idesc,
                      (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&empty[stage]);  // frees the stage once these MMAs have read it
        }
        if (!ok) break;
        umma_commit(&acc_full[buf]);  // accumulator ready for the epilogue
      }
      if (!ok) set_error(p.err, kErrTimeout);
      if (it > 0) {  // the last commit covers every MMA issued before it
        const uint32_t last = it - 1;
        if (!mbar_wait(&empty[last % kWStages], (last / kWStages) & 1, kWaitLimitNs)) set_error(p.err, kErrTimeout);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    // Chunk of 32 tokens: warp q reads TMEM lanes [32q, 32q + 32) (weight rows = output columns,
    // gate_up: lanes 0-63 gate, 64-127 up) x 32 token columns, writes them transposed into the
    // stage [token][column] (pitch 144 words), and the 128 threads then store token rows: thread
    // (token j = e / 4, part = e % 4) takes columns part*4 + 16 i.  With the pitch's 16-word
    // offset every 8-lane phase of the 16-byte reads hits 8 distinct bank groups.
    const int q = warp & 3;
    const int e = threadIdx.x - 64;  // 0..127
    const int j_in = e >> 2, part = e & 3;
    const uint32_t stage_base = smem_u32(staging);
    const uint32_t st_col = stage_base + (uint32_t)(q * 32 + lane) * 4;
    const uint32_t ld_row = stage_base + (uint32_t)(j_in * kWPitch) * 4;
    uint32_t tl = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tl) {
      const uint32_t buf = tl & 1, use = tl >> 1;
      const bool ok = mbar_wait(&acc_full[buf], use & 1, kWaitLimitNs);
      if (epi_any(!ok)) {  // all four warps leave together
        if (!ok) set_error(p.err, kErrTimeout);
        break;
      }
      tc_fence_after();
      const WTile ti = w_decode<KIND>(p, tile_start, G, t);
      const int nr = w_tile_tokens(ti);
      const int n_out = p.n_out[ti.set];
      const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + buf * kWT;
      const size_t trow = (size_t)ti.row0 + (size_t)ti.m * kWT;
#pragma unroll 1
      for (int j0 = 0; j0 < nr; j0 += kWChunk) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tacc + j0, v);
        tmem_ld_wait();
        epi_sync();  // the previous chunk's readers are done with the stage
#pragma unroll
        for (int j = 0; j < 32; ++j) st_shared_f32(st_col + (uint32_t)(j * kWPitch) * 4, v[j]);
        epi_sync();
        if (j0 + j_in < nr) {
          const size_t grow = trow + j0 + j_in;
          if constexpr (KIND == kGateUp) {
            uint16_t* hrow = static_cast<uint16_t*>(p.out[ti.set]) + grow * n_out + ti.n * 64;
            uint16_t* srow = p.save_gu[ti.set] != nullptr ? p.save_gu[ti.set] + grow * 2 * n_out + ti.n * 64 : nullptr;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int c = part * 4 + i * 16;
              const float4 g = ld_shared_f4(ld_row + c * 4);
              const float4 u = ld_shared_f4(ld_row + (64 + c) * 4);
              *reinterpret_cast<uint2*>(hrow + c) =
                  make_uint2(pack_bf16x2(w_silu_mul(g.x, u.x), w_silu_mul(g.y, u.y)),
                             pack_bf16x2(w_silu_mul(g.z, u.z), w_silu_mul(g.w, u.w)));
              if (srow != nullptr) {  // the backward pass's SwiGLU inputs
                *reinterpret_cast<uint2*>(srow + c) = make_uint2(pack_bf16x2(g.x, g.y), pack_bf16x2(g.z, g.w));
                *reinterpret_cast<uint2*>(srow + n_out + c) =
                    make_uint2(pack_bf16x2(u.x, u.y), pack_bf16x2(u.z, u.w));
              }
            }
          } else {
            float* orow = static_cast<float*>(p.out[ti.set]) + grow * n_out + ti.n * 128;
            const float sc = p.row_scale[ti.set] != nullptr ? p.row_scale[ti.set][grow] : 1.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int c = part * 4 + i * 16;
              if (ti.n * 128 + c < n_out) {
                const float4 a = ld_shared_f4(ld_row + c * 4);
                *reinterpret_cast<float4*>(orow + c) = make_float4(a.x * sc, a.y * sc, a.z * sc, a.w * sc);
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
    tmem_dealloc(tmem_base, 2 * kWT);
  }
}

// ------------------------------------------------------------------------------ host side
typedef CUresult (*WEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

WEncodeFn w_encode_fn() {
  static WEncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<WEncodeFn>(ptr);
  });
  return fn;
}

// 2-D bf16 row-major [rows, cols] map, box = 64 columns (128 bytes) x box_rows, 128-byte swizzle;
// rows past the end read as zero.
bool w_make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  WEncodeFn enc = w_encode_fn();
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
bool w_make_gate_up_map(CUtensorMap* m, const void* base, int groups, int F, int K) {
  WEncodeFn enc = w_encode_fn();
  if (enc == nullptr || groups <= 0 || F <= 0 || K <= 0) return false;
  cuuint64_t dims[4] = {(cuuint64_t)K, (cuuint64_t)F, 2, (cuuint64_t)groups};
  cuuint64_t strides[3] = {(cuuint64_t)K * 2, (cuuint64_t)F * K * 2, (cuuint64_t)2 * F * K * 2};
  cuuint32_t box[4] = {64, 64, 2, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int w_num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  }
  return n;
}

template <int KIND>
cudaError_t launch_wide(const GemmSetHost* sets, int n_sets, int* err, cudaStream_t s) {
  WideParams p;
  memset(&p, 0, sizeof(p));
  p.n_sets = n_sets;
  p.err = err;
  p.withhold_first_load = test_withhold_this_launch() ? 1 : 0;
  for (int i = 0; i < n_sets; ++i) {
    const GemmSetHost& st = sets[i];
    if (st.K <= 0 || st.K % kWBK != 0 || st.n_out <= 0) return cudaErrorInvalidValue;
    if (KIND == kGateUp ? (st.n_out % 64 != 0) : (st.n_out % 32 != 0)) return cudaErrorInvalidValue;
    if (st.ld_out != 0 && st.ld_out != st.n_out) return cudaErrorInvalidValue;
    p.k_blocks[i] = st.K / kWBK;
    p.w_rows[i] = KIND == kGateUp ? 2 * st.n_out : st.n_out;
    if (!w_make_map(&p.t_map[i], st.a, (uint64_t)st.a_rows, (uint64_t)st.K, 64) ||
        !w_make_map(&p.t_map256[i], st.a, (uint64_t)st.a_rows, (uint64_t)st.K, kWT))
      return cudaErrorInvalidValue;
    if (KIND == kGateUp ? !w_make_gate_up_map(&p.w_map[i], st.w, st.n_groups, st.n_out, st.K)
                        : !w_make_map(&p.w_map[i], st.w, (uint64_t)st.n_groups * p.w_rows[i], (uint64_t)st.K, 128))
      return cudaErrorInvalidValue;
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
    cudaError_t e = cudaFuncSetAttribute(grouped_gemm_wide_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kWSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  return launch_pdl(grouped_gemm_wide_kernel<KIND>, dim3(w_num_sms()), dim3(kWThreads), kWSmemBytes, s, p);
}

}  // namespace

cudaError_t launch_grouped_gemm_wide(GemmKind kind, const GemmSetHost* sets, int n_sets, int* err, cudaStream_t s) {
  if (n_sets < 1 || n_sets > 2) return cudaErrorInvalidValue;
  int groups = 0;
  for (int i = 0; i < n_sets; ++i) groups += sets[i].n_groups;
  if (groups > kWMaxGroups) return cudaErrorInvalidValue;
  if (kind == kGateUp) return launch_wide<kGateUp>(sets, n_sets, err, s);
  if (kind == kDown) return launch_wide<kDown>(sets, n_sets, err, s);
  return cudaErrorInvalidValue;
}

}  // namespace moe
