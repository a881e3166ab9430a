// stream_fp8w_sm100.cu -- weight-streaming (decode) grouped GEMMs with E4M3 expert weights.
//
// The decode path of the layer reads every active expert's weights once, so its time is the
// weight bytes over HBM bandwidth (keryc.com "Mixture of Experts optimiza...", section "Por que
// MoEs importan": decode speed = bandwidth / active bytes).  Storing the weights as E4M3 codes
// with one fp32 scale per row (quantize_fp8.cu; the pages' per-expert quantisation, section
// "Resultados practicos") halves those bytes.
//
// Same maths as the bf16 weight-streaming kernels in grouped_gemm_sm100.cu (swap-AB: 128 weight
// rows of one active expert are the MMA M operand, the <= NT tokens routed to it the N operand),
// built around where the converted weights live:
//   * TMA brings each stage's codes as 128 rows x 128 bytes (K = 128) with the 128-byte swizzle,
//     and the f16 activations as two 64-column swizzled atoms;
//   * eight converter warps read their weight rows from shared memory (conflict-free under the
//     swizzle), turn the codes into f16 (exact) and store them with tcgen05.st straight into
//     tensor memory, where the MMA takes its A operand.  Shared memory then carries 2 bytes per
//     code (TMA write + converter read) instead of 6 with an f16 copy in shared memory, which is
//     what bounded the first design well below HBM bandwidth;
//   * the tensor cores run kind::f16 (f16 A from TMEM, f16 B from shared memory);
//   * the epilogue multiplies each accumulator row by its weight row's scale (TMEM lane = weight
//     row), before the SwiGLU (gate_up) or together with the router weight (down).
// K need only be a multiple of 64: the last stage's columns past K are zero-filled by TMA.
// Warp roles: 0 TMA producer, 1 MMA issuer (+TMEM owner), 2-5 epilogue, 6-13 converters (warp w
// owns TMEM lanes 32*(w%4).. and K half (w-6)/4).  All waits are bounded as in the bf16 kernels.
#include <cuda.h>
#include <cuda_fp16.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "moe_common.cuh"
#include "sm100_ptx.cuh"

namespace moe {
namespace {

constexpr int kBM = 128;             // MMA M: weight rows per unit
constexpr int kBK = 128;             // K per stage (codes: one 128-byte swizzle row)
constexpr int kThreads = 448;        // 14 warps
constexpr int kConvWarps = 8;        // warps 6..13
constexpr int kMaxGroups = 1025;
constexpr int kRawW = kBM * kBK;     // one E4M3 weight tile: 128 rows x 128 bytes = 16 KB
constexpr int kBarBytes = 512;

struct alignas(64) Fp8Params {
  CUtensorMap a_map[2];  // f16 activations [rows, K], 128-byte swizzle, box {64, NT}
  CUtensorMap w_map[2];  // E4M3 weights [groups * w_rows, K], 128-byte swizzle, box {128 bytes, 128}
  const float* w_scale[2];  // per weight row
  const int32_t* offsets[2];
  void* out[2];             // gate_up: f16 h [rows, F]; down: fp32 [rows, D]
  const float* row_scale[2];
  int n_groups[2];
  int m_rows[2];
  int n_out[2];
  int w_rows[2];
  int k_blocks[2];          // ceil(K / 128)
  float* partial;           // split-K partial accumulators [items][kAccCols][128] or null (no split)
  int* counters;            // per unit: splits finished (zero on entry, left zero on exit)
  int max_items;            // capacity of `partial` in items
  int n_sets;
  int withhold_first_load;
  int* err;
};

// f16 MMA inputs (A and B formats 0 = F16), fp32 accumulator
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

constexpr int pow2_cols(int c) { return c <= 32 ? 32 : c <= 64 ? 64 : c <= 128 ? 128 : c <= 256 ? 256 : 512; }

template <int KIND, int NT>
struct Fp8Cfg {
  static constexpr int kW = KIND == kGateUp ? 2 : 1;      // weight tiles per stage
  static constexpr int kAtom = NT * 128;                   // one f16 activation atom: NT rows x 64 K
  static constexpr int kStage = 2 * kAtom + kW * kRawW;    // [act k0-63 | act k64-127 | w0 | w1]
  static constexpr int kAccCols = kW * NT;                 // one accumulator buffer
  static constexpr int kACol = 2 * kAccCols;               // A stages follow the two buffers
  static constexpr int kAStageCols = kW * 64;              // 128 K of f16 per tile = 64 columns
  static constexpr int kAStages = (512 - kACol) / kAStageCols >= 4 ? 4 : (512 - kACol) / kAStageCols;
  static constexpr int kTmemCols = pow2_cols(kACol + kAStages * kAStageCols);
  static constexpr int kRawBudget = 232448 - 1024 - kBarBytes - 4 * (kMaxGroups + 1);
  static constexpr int kStages = kRawBudget / kStage >= 8 ? 8 : kRawBudget / kStage;
  static constexpr uint32_t kIdesc = idesc_f16_f32(kBM, NT);
  static constexpr size_t kSmemBytes = 1024 + (size_t)kStages * kStage + kBarBytes + 4 * (kMaxGroups + 1);
  static_assert(kStage % 1024 == 0, "1024-byte aligned stages");
  static_assert(kAStages >= 2 && kStages >= 3, "pipeline depth");
  static_assert(kACol + kAStages * kAStageCols <= 512, "tensor memory");
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

struct Unit {
  int set, gl, row0, rows, n;
};

__device__ __forceinline__ void unit_rows(const Fp8Params& p, int s, int gl, int& row0, int& rows) {
  if (p.offsets[s] != nullptr) {
    row0 = p.offsets[s][gl];
    rows = p.offsets[s][gl + 1] - row0;
  } else {
    row0 = 0;
    rows = p.m_rows[s];
  }
}

__device__ __forceinline__ Unit decode_unit(const Fp8Params& p, const int* unit_start, int G, int t) {
  int lo = 0, hi = G - 1;  // largest g with unit_start[g] <= t
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (unit_start[mid] <= t) lo = mid; else hi = mid - 1;
  }
  Unit u;
  u.set = lo < p.n_groups[0] ? 0 : 1;
  u.gl = u.set == 0 ? lo : lo - p.n_groups[0];
  unit_rows(p, u.set, u.gl, u.row0, u.rows);
  u.n = t - unit_start[lo];
  return u;
}

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + __expf(-g)) * u; }

// split-K for small unit counts (moe_common.cuh): an item is (unit, split)
__device__ __forceinline__ int choose_splits(const Fp8Params& p, int units, int grid) {
  if (p.partial == nullptr) return 1;
  int kb_min = p.k_blocks[0];
  if (p.n_sets > 1) kb_min = min(kb_min, p.k_blocks[1]);
  return split_count(units, grid, kb_min, p.max_items);
}

template <int KIND, int NT>
__global__ void __launch_bounds__(kThreads, 1) stream_fp8w_kernel(const __grid_constant__ Fp8Params p) {
  using C = Fp8Cfg<KIND, NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStage);
  uint64_t* empty = full + C::kStages;
  uint64_t* afull = empty + C::kStages;  // converted A stage in TMEM ready (8 converter warps)
  uint64_t* aempty = afull + C::kAStages;  // A stage consumed by the MMAs (tcgen05.commit)
  uint64_t* acc_full = aempty + C::kAStages;
  uint64_t* acc_empty = acc_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  int* unit_start = reinterpret_cast<int*>(smem + C::kStages * C::kStage + kBarBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.n_groups[0] + (p.n_sets > 1 ? p.n_groups[1] : 0);

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < C::kAStages; ++s) {
      mbar_init(&afull[s], kConvWarps);
      mbar_init(&aempty[s], 1);
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
  pdl_wait();
  pdl_trigger();
  // units (one per active group and 128-row weight block), then an exclusive scan
  for (int g = threadIdx.x; g < G; g += kThreads) {
    const int s = g < p.n_groups[0] ? 0 : 1;
    const int gl = s == 0 ? g : g - p.n_groups[0];
    int row0, rows;
    unit_rows(p, s, gl, row0, rows);
    if (rows > NT) set_error(p.err, kErrBadIndex);  // a segment longer than the token tile
    unit_start[g] = rows > 0 ? (p.n_out[s] + kBM - 1) / kBM : 0;
  }
  __syncthreads();
  if (warp == 0) {
    const int per = (G + 31) / 32;
    const int lo = lane * per, hi = min(G, lo + per);
    int sum = 0;
    for (int g = lo; g < hi; ++g) sum += unit_start[g];
    int incl = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int run = incl - sum;
    for (int g = lo; g < hi; ++g) {
      const int c = unit_start[g];
      unit_start[g] = run;
      run += c;
    }
    if (lane == 31) unit_start[G] = incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int n_units = unit_start[G];
  const int S = choose_splits(p, n_units, gridDim.x);  // identical in every CTA
  const int total = n_units * S;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Unit u = decode_unit(p, unit_start, G, t / S);
        const int wrow = u.gl * p.w_rows[u.set] + u.n * kBM;
        const int kb_end = split_end(p.k_blocks[u.set], t % S, S);
        for (int kb = split_begin(p.k_blocks[u.set], t % S, S); kb < kb_end; ++kb, ++it) {
          const int st = it % C::kStages;
          if (!mbar_wait(&empty[st], ((it / C::kStages) & 1) ^ 1, kWaitLimitNs)) {
            ok = false;
            break;
          }
          uint8_t* sb = smem + st * C::kStage;
          mbar_arrive_expect_tx(&full[st], C::kStage);
          if (p.withhold_first_load && it == 0) continue;  // test only: the bytes never arrive
          const int kx = kb * kBK;
          tma_load_2d(&p.a_map[u.set], &full[st], sb, kx, u.row0);
          tma_load_2d(&p.a_map[u.set], &full[st], sb + C::kAtom, kx + 64, u.row0);
          tma_load_2d(&p.w_map[u.set], &full[st], sb + 2 * C::kAtom, kx, wrow);
          if constexpr (KIND == kGateUp)
            tma_load_2d(&p.w_map[u.set], &full[st], sb + 2 * C::kAtom + kRawW, kx, wrow + p.n_out[u.set]);
        }
      }
      if (!ok) set_error(p.err, kErrTimeout);
      const uint32_t issued = it;
      for (int s = 0; s < C::kStages; ++s) {
        if ((uint32_t)s >= issued) break;
        const uint32_t last = issued - 1 - ((issued - 1 - s) % C::kStages);
        if (!mbar_wait(&full[s], (last / C::kStages) & 1, kWaitLimitNs)) set_error(p.err, kErrTimeout);
      }
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------------------ E4M3 -> f16 into TMEM
    // Thread = weight row r of its quadrant; it converts the 64 codes of K half h of row r (four
    // 16-byte chunks, placed by the 128-byte swizzle at chunk ^ (r & 7)) and stores them as 32
    // f16x2 columns of TMEM lane r.
    const int q = warp & 3, h = (warp - 6) >> 2;
    const int r = 32 * q + lane;
    const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
    uint32_t it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const Unit u = decode_unit(p, unit_start, G, t / S);
      const int kb_end = split_end(p.k_blocks[u.set], t % S, S);
      for (int kb = split_begin(p.k_blocks[u.set], t % S, S); kb < kb_end; ++kb, ++it) {
        const int st = it % C::kStages, as = it % C::kAStages;
        if (!mbar_wait(&full[st], (it / C::kStages) & 1, kWaitLimitNs) ||
            !mbar_wait(&aempty[as], ((it / C::kAStages) & 1) ^ 1, kWaitLimitNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t src = smem_u32(smem + st * C::kStage + 2 * C::kAtom) + r * kBK;
#pragma unroll
        for (int w = 0; w < C::kW; ++w) {
          uint4 in[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) in[c] = ld_shared_v4(src + w * kRawW + (((4 * h + c) ^ (r & 7)) << 4));
          uint32_t o[32];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            e4m3x4_to_f16x4(in[c].x, o[8 * c + 0], o[8 * c + 1]);
            e4m3x4_to_f16x4(in[c].y, o[8 * c + 2], o[8 * c + 3]);
            e4m3x4_to_f16x4(in[c].z, o[8 * c + 4], o[8 * c + 5]);
            e4m3x4_to_f16x4(in[c].w, o[8 * c + 6], o[8 * c + 7]);
          }
          tmem_st_32x32b_x32(tmem_base + lane_addr + C::kACol + as * C::kAStageCols + w * 64 + h * 32, o);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[as]);
      }
    }
    if (!ok) set_error(p.err, kErrTimeout);
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
        const Unit u = decode_unit(p, unit_start, G, t / S);
        const int kb0 = split_begin(p.k_blocks[u.set], t % S, S), kb_end = split_end(p.k_blocks[u.set], t % S, S);
        for (int kb = kb0; kb < kb_end; ++kb, ++it) {
          const int st = it % C::kStages, as = it % C::kAStages;
          if (!mbar_wait(&full[st], (it / C::kStages) & 1, kWaitLimitNs) ||
              !mbar_wait(&afull[as], (it / C::kAStages) & 1, kWaitLimitNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + st * C::kStage);  // activation atoms (B)
          const uint32_t acol = tmem_base + C::kACol + as * C::kAStageCols;  // converted weights (A)
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint32_t acc = (kb != kb0 || kk != 0) ? 1u : 0u;
            const uint64_t bdesc = sw128_kmajor_desc(sa + (kk >> 2) * C::kAtom + (kk & 3) * 32);
            umma_f16_tmem_a(d, acol + kk * 8, bdesc, C::kIdesc, acc);
            if constexpr (KIND == kGateUp) umma_f16_tmem_a(d + NT, acol + 64 + kk * 8, bdesc, C::kIdesc, acc);
          }
          umma_commit(&empty[st]);   // the stage's codes and activations are free
          umma_commit(&aempty[as]);  // the converted A stage is free
        }
        if (!ok) break;
        umma_commit(&acc_full[buf]);
      }
      if (!ok) set_error(p.err, kErrTimeout);
      if (it > 0) {
        const uint32_t last = it - 1;
        if (!mbar_wait(&aempty[last % C::kAStages], (last / C::kAStages) & 1, kWaitLimitNs))
          set_error(p.err, kErrTimeout);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    // Thread = accumulator row r (TMEM lane) = output column n*128 + r of its unit.
    const int q = warp & 3;
    const int r = q * 32 + lane;
    uint32_t tl = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++tl) {
      const uint32_t buf = tl & 1, use = tl >> 1;
      if (!mbar_wait(&acc_full[buf], use & 1, kWaitLimitNs)) {
        set_error(p.err, kErrTimeout);
        break;
      }
      tc_fence_after();
      const Unit u = decode_unit(p, unit_start, G, t / S);
      const uint32_t tacc = tmem_base + ((uint32_t)(q * 32) << 16) + buf * C::kAccCols;
      const int n_out = p.n_out[u.set];
      const int wbase = u.gl * p.w_rows[u.set];
      const int col = u.n * kBM + r;  // output column = weight row within the group
      const bool col_ok = col < n_out;
      const float* ws = p.w_scale[u.set];
      const float s0 = col_ok ? ws[wbase + col] : 0.f;                                    // gate / down row
      const float s1 = (KIND == kGateUp && col_ok) ? ws[wbase + n_out + col] : 0.f;      // up row
      const float* rs = p.row_scale[u.set];
      // final value of token j (accumulators a = gate or down, b = up), written to the output
      auto store = [&](int j, float a, float b) {
        if (!col_ok) return;
        if constexpr (KIND == kGateUp) {
          static_cast<__half*>(p.out[u.set])[(size_t)(u.row0 + j) * n_out + col] = __float2half_rn(silu_mul(a * s0, b * s1));
        } else {
          static_cast<float*>(p.out[u.set])[(size_t)(u.row0 + j) * n_out + col] =
              a * s0 * (rs != nullptr ? rs[u.row0 + j] : 1.0f);
        }
      };
      float* part = S > 1 ? p.partial + (size_t)t * C::kAccCols * kBM : nullptr;
#pragma unroll 1
      for (int j0 = 0; j0 < NT; j0 += 16) {
        if (j0 >= u.rows) break;
        uint32_t a[16], b[16];
        tmem_ld_32x32b_x16(tacc + j0, a);
        if constexpr (KIND == kGateUp) tmem_ld_32x32b_x16(tacc + NT + j0, b);
        tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
          const int j = j0 + jj;
          if (j >= u.rows) continue;
          const float av = __uint_as_float(a[jj]), bv = KIND == kGateUp ? __uint_as_float(b[jj]) : 0.f;
          if (part == nullptr) {
            store(j, av, bv);
          } else {
            part[(size_t)j * kBM + r] = av;
            if constexpr (KIND == kGateUp) part[(size_t)(NT + j) * kBM + r] = bv;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[buf]);
      if (part != nullptr) {
        // publish this split's rows; the last of the S splits of this quadrant sums them in split
        // order (deterministic) and finishes the epilogue
        __threadfence();
        __syncwarp();
        int* counter = p.counters + (size_t)(t / S) * 4 + q;
        int done = 0;
        if (lane == 0) done = atomicAdd(counter, 1);
        done = __shfl_sync(0xffffffffu, done, 0);
        if (done == S - 1) {
          __threadfence();
          const float* base = p.partial + (size_t)(t / S) * S * C::kAccCols * kBM + r;
          for (int j = 0; j < u.rows; ++j) {
            float av = 0.f, bv = 0.f;
            for (int sp = 0; sp < S; ++sp) {
              av += __ldcg(base + ((size_t)sp * C::kAccCols + j) * kBM);
              if constexpr (KIND == kGateUp) bv += __ldcg(base + ((size_t)sp * C::kAccCols + NT + j) * kBM);
            }
            store(j, av, bv);
          }
          if (lane == 0) *counter = 0;  // ready for the next launch
        }
      }
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

// 2-D row-major [rows, cols] map with the 128-byte swizzle; box = box_cols x box_rows elements
bool make_map(CUtensorMap* m, CUtensorMapDataType type, int elem_bytes, const void* base, uint64_t rows,
              uint64_t cols, uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr || rows == 0 || cols == 0) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (uint64_t)elem_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, type, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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

template <int KIND, int NT>
cudaError_t launch_fp8(const GemmSetHost* sets, const float* const* scales, int n_sets, float* partial,
                       size_t partial_bytes, int* counters, int* err, cudaStream_t s) {
  using C = Fp8Cfg<KIND, NT>;
  Fp8Params p;
  memset(&p, 0, sizeof(p));
  p.n_sets = n_sets;
  p.err = err;
  const size_t item_bytes = (size_t)C::kAccCols * kBM * sizeof(float);
  if (partial != nullptr && counters != nullptr && partial_bytes >= 2 * item_bytes) {
    p.partial = partial;
    p.counters = counters;
    p.max_items = (int)std::min<size_t>(partial_bytes / item_bytes, (size_t)kMaxSplitItems);
  }
  p.withhold_first_load = test_withhold_this_launch() ? 1 : 0;
  for (int i = 0; i < n_sets; ++i) {
    const GemmSetHost& st = sets[i];
    const int K = st.K;
    p.k_blocks[i] = (K + kBK - 1) / kBK;
    p.w_rows[i] = KIND == kGateUp ? 2 * st.n_out : st.n_out;
    if (!make_map(&p.a_map[i], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, st.a, (uint64_t)st.a_rows, (uint64_t)K, 64, NT))
      return cudaErrorInvalidValue;
    if (!make_map(&p.w_map[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, st.w, (uint64_t)st.n_groups * p.w_rows[i],
                  (uint64_t)K, kBK, kBM))
      return cudaErrorInvalidValue;
    p.w_scale[i] = scales[i];
    p.offsets[i] = st.offsets;
    p.out[i] = st.out;
    p.row_scale[i] = st.row_scale;
    p.n_groups[i] = st.n_groups;
    p.m_rows[i] = st.m_rows;
    p.n_out[i] = st.n_out;
  }
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(stream_fp8w_kernel<KIND, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)C::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  return launch_pdl(stream_fp8w_kernel<KIND, NT>, dim3(sm_count()), dim3(kThreads), C::kSmemBytes, s, p);
}

template <int KIND>
cudaError_t launch_kind(const GemmSetHost* sets, const float* const* scales, int n_sets, int nt, float* partial,
                        size_t partial_bytes, int* counters, int* err, cudaStream_t s) {
  switch (nt) {
    case 16: return launch_fp8<KIND, 16>(sets, scales, n_sets, partial, partial_bytes, counters, err, s);
    case 32: return launch_fp8<KIND, 32>(sets, scales, n_sets, partial, partial_bytes, counters, err, s);
    case 48: return launch_fp8<KIND, 48>(sets, scales, n_sets, partial, partial_bytes, counters, err, s);
    case 64: return launch_fp8<KIND, 64>(sets, scales, n_sets, partial, partial_bytes, counters, err, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_stream_fp8w(GemmKind kind, const GemmSetHost* sets, const float* const* w_scales, int n_sets,
                               int decode_nt, SplitBuf split, int* err, cudaStream_t s) {
  if (n_sets < 1 || n_sets > 2) return cudaErrorInvalidValue;
  int groups = 0;
  for (int i = 0; i < n_sets; ++i) {
    if (sets[i].K <= 0 || sets[i].K % 64 != 0 || w_scales[i] == nullptr) return cudaErrorInvalidValue;
    groups += sets[i].n_groups;
  }
  if (groups > kMaxGroups) return cudaErrorInvalidValue;
  if (kind == kGateUp)
    return launch_kind<kGateUp>(sets, w_scales, n_sets, decode_nt, split.partial, split.partial_bytes, split.counters,
                                err, s);
  if (kind == kDown)
    return launch_kind<kDown>(sets, w_scales, n_sets, decode_nt, split.partial, split.partial_bytes, split.counters,
                              err, s);
  return cudaErrorInvalidValue;
}

}  // namespace moe
