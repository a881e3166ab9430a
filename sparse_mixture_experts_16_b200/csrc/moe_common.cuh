// moe_common.cuh -- shared definitions of the CUDA path (kernels and host launchers).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe_b200.h"

namespace moe {

// ---- device error word (first 256 bytes of every workspace) -------------------------------
constexpr int kErrBadIndex = 1;  // an expert id outside [0, E)
constexpr int kErrTimeout = 2;   // a bounded device-side wait gave up
constexpr size_t kWsHeader = 256;

// Wall-time limit of every spin-wait inside a kernel, measured on %globaltimer.  A context that
// is descheduled for longer than this while a kernel waits (time-slicing with another process,
// a debugger) can therefore report a spurious MOE_ERR_TIMEOUT.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s

// Fault-path test hook of the expert-GEMM launches (not of the router GEMM): the environment
// variable MOE_TEST_WITHHOLD_LOAD=n, read once per process, makes the first n such launches
// withhold the first stage's copies of every CTA.  The barriers are armed but the bytes never
// arrive, so the bounded waits expire and the kernel reports MOE_ERR_TIMEOUT and returns.
// Returns whether the launch being prepared is one of those n.
bool test_withhold_this_launch();

// ---- split-K of the weight-streaming (decode) GEMMs ---------------------------------------------
// A decode step with fewer 128-row units than SMs splits each unit's K range.  Partial fp32
// accumulators go to a workspace buffer; four counters per unit (one per TMEM lane quadrant) let
// the last split finish the epilogue.  The counters must be zero when a launch starts; every
// launch leaves them zero.
constexpr int kMaxSplitUnits = 256;                                      // no split above this
constexpr size_t kSplitCounterBytes = (size_t)kMaxSplitUnits * 4 * sizeof(int);
constexpr int kMaxSplitItems = 4 * 148;                                  // partial capacity (items)
constexpr int kMaxSplits = 16;

// workspace the host hands to a weight-streaming launch for split-K (all null: never split)
struct SplitBuf {
  float* partial = nullptr;  // partial accumulators, fp32
  size_t partial_bytes = 0;
  int* counters = nullptr;   // kSplitCounterBytes, zero when the launch starts
};

// K range [begin, end) of split s of S over kb k-blocks (balanced, non-empty when S <= kb)
__device__ __forceinline__ int split_begin(int kb, int s, int S) { return (int)((long long)kb * s / S); }
__device__ __forceinline__ int split_end(int kb, int s, int S) { return (int)((long long)kb * (s + 1) / S); }

// Number of K splits for `units` units on `grid` CTAs: S minimises waves / S + 0.02 * S, capped by
// the smallest k-block count and the partial buffer's capacity.  Every CTA gets the same answer.
__device__ __forceinline__ int split_count(int units, int grid, int kb_min, int max_items) {
  if (max_items <= 0 || units <= 0 || units >= grid || units > kMaxSplitUnits) return 1;
  const int s_max = min(kMaxSplits, min(kb_min, max_items / units));
  int best_s = 1;
  float best = 1e30f;
  for (int s = 1; s <= s_max; ++s) {
    const int waves = (units * s + grid - 1) / grid;
    const float cost = (float)waves / (float)s + 0.02f * (float)s;
    if (cost < best) {
      best = cost;
      best_s = s;
    }
  }
  return best_s;
}

__device__ __forceinline__ void set_error(int* err, int bits) {
  if (err) atomicOr(err, bits);
}

// ---- bf16 helpers -----------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// two fp32 -> packed bf16x2 (round to nearest even), low half = a
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// ---- programmatic dependent launch --------------------------------------------------------------
// Every kernel of the layer is launched with programmatic stream serialisation: it may start (and
// run its prologue) while the previous kernel drains.  Each kernel executes pdl_wait() before it
// reads anything an earlier kernel (or the caller) wrote, and pdl_trigger() once its own
// dependents may be scheduled.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ---- host launchers (defined in the .cu files) ---------------------------------------------
// Router: logits on the tensor cores (split-K partial sums, [k_splits][T][ld] fp32, ld = E rounded
// up to 32), then a warp-level top-k + softmax kernel that reduces the splits in a fixed order.
int router_k_splits(int T, int D, int E);
inline int router_ld(int E) { return (E + 31) / 32 * 32; }
inline size_t router_scratch_bytes(int T, int D, int E) {
  return align_up((size_t)router_k_splits(T, D, E) * (size_t)T * router_ld(E) * sizeof(float), 256);
}
cudaError_t launch_router_gemm(const uint16_t* x, const uint16_t* wg, int T, int D, int E, float* partials, int ld,
                               int k_splits, int* err, cudaStream_t s);
cudaError_t launch_router_select(const float* partials, int k_splits, int T, int ld, const float* bias, int E, int k,
                                 int32_t* idx, float* w, cudaStream_t s);

cudaError_t launch_update_bias(const int32_t* counts, int E, float gamma, float* bias, cudaStream_t s);

size_t permute_scratch_bytes(int T, int E);
cudaError_t launch_permute(const int32_t* idx, const float* topk_w, const uint16_t* x, int T, int D, int E,
                           int k, int32_t* counts, int32_t* offsets, int32_t* perm_token, int32_t* inv_perm,
                           float* p_perm, uint16_t* x_perm, bool x_perm_f16, uint16_t* x_cast, int32_t* scratch,
                           int* err, cudaStream_t s, int* n_launches);

cudaError_t launch_combine(const float* out_perm, const int32_t* inv_perm, const float* shared_out, int T, int D,
                           int k, uint16_t* y, cudaStream_t s);

// One "set" of a grouped GEMM launch: either the routed experts (groups = segments of the
// expert-contiguous rows given by offsets) or the shared expert (one group of m_rows rows).
struct GemmSetHost {
  int K;                    // reduction length (multiple of 64)
  const uint16_t* a;        // activations [a_rows, K]
  int64_t a_rows;           // rows of the activation tensor (tensor-map extent)
  const uint16_t* w;        // weights [n_groups * w_rows_per_group, K]
  int n_groups;             // E (routed) or 1 (shared)
  const int32_t* offsets;   // routed: device offsets[E+1]; shared: NULL
  int m_rows;               // shared: rows of its single group
  int n_out;                // output columns (F for gate_up -> h, D for down)
  void* out;                // [rows, n_out]: bf16 (gate_up -> h) or fp32 (down)
  const float* row_scale;   // per-row factor (down) or NULL
  int ld_out;               // output row stride in elements (0: n_out)
  uint16_t* save_gu = nullptr;  // tiled gate_up, training: also store g | u [rows, 2 * n_out] bf16
};

enum GemmKind { kGateUp = 0, kDown = 1, kRouter = 2 };

// ---- backward pass (grouped_gemm_bwd_sm100.cu, layer_backward.cu) ----------------------------
enum BwdKind { kBwdDxDown = 0, kBwdDxGateUp = 1, kBwdDwDown = 2, kBwdDwGateUp = 3 };

// One operand set of a backward GEMM launch (set 0: the routed experts, set 1: the shared expert).
struct BwdSetHost {
  const void* a = nullptr;  // bf16 A storage [a_rows, a_cols]
  int64_t a_rows = 0;
  int a_cols = 0;
  const void* b = nullptr;  // bf16 B storage [b_rows, b_cols] (contracted index = row)
  int64_t b_rows = 0;
  int b_cols = 0;
  const int32_t* offsets = nullptr;      // groups' unpadded rows (NULL: one group of m_rows rows)
  const int32_t* pad_offsets = nullptr;  // groups' rows in the 64-row padded layout
  int n_groups = 1, m_rows = 0;
  int K = 0, M_total = 0, N_total = 0;
  const float* p_perm = nullptr;
  const uint16_t* gu_saved = nullptr;
  uint16_t* dgu = nullptr;
  float* dp_part = nullptr;
  float* out = nullptr;
};
cudaError_t launch_bwd_gemm(BwdKind kind, const BwdSetHost* sets, int n_sets, int* err, cudaStream_t s);
cudaError_t launch_pad_offsets(const int32_t* offsets, int E, int32_t* pad_offsets, cudaStream_t s);
cudaError_t launch_gather_dy(const uint16_t* dy, const int32_t* offsets, const int32_t* pad_offsets, int E,
                             const int32_t* perm_token, const float* p_perm, int D, int F2, long long rows_bound,
                             uint16_t* dyp, uint16_t* dO, uint16_t* dgu, cudaStream_t s);
cudaError_t launch_router_bwd(const int32_t* inv_perm, const float* topk_w, const float* dp_part, int n_tiles, int T,
                              int k, float* dl_row, cudaStream_t s);
cudaError_t launch_dwgate(const int32_t* offsets, const float* dl_row, const uint16_t* x_perm, int E, int D,
                          float* dwg, cudaStream_t s);
cudaError_t launch_unpermute(const float* dxp, const float* dx_sh, const int32_t* inv_perm, const int32_t* topk_idx,
                             const int32_t* offsets, const int32_t* pad_offsets, const float* dl_row, const uint16_t* wg,
                             int T, int D, int k, uint16_t* dx, cudaStream_t s);

// Launch one grouped GEMM (gate_up + SwiGLU, or down + row scale) over up to two sets.
// decode_nt > 0 selects the weight-streaming
// kernels with a token tile of decode_nt (16/32/48/64); 0 selects the tiled kernels.
cudaError_t launch_grouped_gemm(GemmKind kind, const GemmSetHost* sets, int n_sets, int decode_nt, int* err,
                                cudaStream_t s);

// Weight-streaming grouped GEMMs with E4M3 expert weights (one fp32 scale per weight row,
// w_scales[set]) and f16 activations (sets[i].a); gate_up writes f16 h.  decode_nt: 16..64.
cudaError_t launch_stream_fp8w(GemmKind kind, const GemmSetHost* sets, const float* const* w_scales, int n_sets,
                               int decode_nt, SplitBuf split, int* err, cudaStream_t s);

// Per-row E4M3 quantisation: scales[r] = amax(row) / 448, q = E4M3(w / scale).  K % 8 == 0.
cudaError_t launch_quantize_rows_fp8(const uint16_t* w, long long rows, int K, uint8_t* q, float* scales,
                                     cudaStream_t s);


}  // namespace moe
