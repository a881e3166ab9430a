// moe_layer.cu -- the C ABI (include/moe_b200.h): argument validation, workspace layout and the
// chaining of the layer's kernels on one stream.  Host code only; the kernels live in
// router_topk.cu, permute.cu, grouped_gemm_sm100.cu and combine.cu.
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>

#include "grouped_gemm_wide.cuh"
#include "router_aux.cuh"
#include "moe_common.cuh"

using namespace moe;

namespace {

constexpr int kDecodeTMax = 64;  // T <= this runs the weight-streaming kernels

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

moe_status_t check_device() {
  static int arch_state[64];  // per device: 0 unchecked, 1 sm_100, 2 other
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  if (dev < 64 && arch_state[dev] == 1) return MOE_OK;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  if (dev < 64) arch_state[dev] = major == 10 ? 1 : 2;
  return major == 10 ? MOE_OK : MOE_ERR_NO_DEVICE;
}

moe_status_t shape_status(long long T, long long D, long long E, long long k) {
  if (T < 0 || D <= 0 || E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (D % 64 != 0 || E > 1024 || k > 32) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (T * k >= (1LL << 31) || T * D >= (1LL << 40)) return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

bool use_decode(const moe_layer_desc_t& d) {
  if (d.flags & MOE_FLAG_SAVE_FOR_BACKWARD) return false;  // the tiled kernels save g | u
  if (d.flags & MOE_FLAG_FORCE_DECODE) return true;
  if (d.flags & MOE_FLAG_FORCE_PREFILL) return false;
  return d.T <= kDecodeTMax;
}

int decode_tile(int max_seg) { return ((max_seg + 15) / 16) * 16; }

// Prefill tiling: which kernel runs each expert GEMM.  Row tiles: 128 permuted rows x 256 output
// columns (tokens are the MMA's M).  Wide tiles: 128 weight rows x up to 256 rows of one expert
// segment (tokens are N, so a segment's last tile pads to 16 rows instead of 128).  Pair tiles: the
// wide orientation on a cluster of two CTAs, 256 weight rows x up to 256 tokens per MMA (each SM
// loads a third fewer operand bytes per FLOP).  The default mixes the measured best per GEMM.
enum TileKind { kRowT = 0, kWideT = 1, kPairT = 2 };
struct Tiling {
  int gu, dn;
};
Tiling prefill_tiling(int flags) {
  if (flags & MOE_FLAG_PREFILL_WIDE_TILES) return {kWideT, kWideT};
  if (flags & MOE_FLAG_PREFILL_ROW_TILES) return {kRowT, kRowT};
  if (flags & MOE_FLAG_PREFILL_PAIR_TILES) return {kPairT, kPairT};
  return {kRowT, kPairT};
}

cudaError_t launch_tiled(TileKind t, GemmKind kind, const GemmSetHost* sets, int n_sets, int* err, cudaStream_t s) {
  if (t == kPairT) return launch_grouped_gemm_pair(kind, sets, n_sets, err, s);
  if (t == kWideT) return launch_grouped_gemm_wide(kind, sets, n_sets, err, s);
  return launch_grouped_gemm(kind, sets, n_sets, 0, err, s);
}

struct LayerWs {
  size_t split_counters, split_partial, split_partial_bytes, gu_saved, gu_saved_sh, router, topk_idx, topk_w, scratch, counts, offsets, perm_token, inv_perm, p_perm, x_perm, h, h_sh, out_perm,
      out_sh, x16, x_stage, y_stage, total;
};

LayerWs layer_ws(const moe_layer_desc_t& d) {
  LayerWs w;
  size_t o = kWsHeader;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  const size_t T = d.T, D = d.D, E = d.E, k = d.k, F = d.F, Fs = d.Fs, M = T * k;
  // split-K counters directly after the error word, so one memset clears both
  w.split_counters = take(kSplitCounterBytes);
  // split-K partials of the FP8 weight-streaming GEMMs: gate_up items are the larger, 2 * NT
  // accumulator columns x 128 rows x fp32
  w.split_partial_bytes = d.weight_format == MOE_WEIGHTS_FP8_E4M3
                              ? (size_t)kMaxSplitItems * 2 * decode_tile(d.T) * 128 * sizeof(float)
                              : 0;
  w.split_partial = take(w.split_partial_bytes);
  // training forward: the SwiGLU inputs g | u of the routed rows and of the shared expert (bf16)
  const bool save = (d.flags & MOE_FLAG_SAVE_FOR_BACKWARD) != 0;
  w.gu_saved = take(save ? M * 2 * F * 2 : 0);
  w.gu_saved_sh = take(save ? T * 2 * Fs * 2 : 0);
  w.router = take(router_scratch_bytes(d.T, d.D, d.E));
  w.topk_idx = take(M * 4);
  w.topk_w = take(M * 4);
  w.scratch = take(permute_scratch_bytes(d.T, d.E));
  w.counts = take(E * 4);
  w.offsets = take((E + 1) * 4);
  w.perm_token = take(M * 4);
  w.inv_perm = take(M * 4);
  w.p_perm = take(M * 4);
  w.x_perm = take(M * D * 2);
  w.h = take(M * F * 2);
  w.h_sh = take(T * Fs * 2);
  w.out_perm = take(M * D * 4);
  w.out_sh = take(T * D * 4);
  w.x16 = take(T * D * 2);
  w.x_stage = take(T * D * 2);
  w.y_stage = take(T * D * 2);
  w.total = o;
  return w;
}

moe_status_t validate_desc(const moe_layer_desc_t* d) {
  if (d == nullptr) return MOE_ERR_INVALID_ARG;
  moe_status_t st = shape_status(d->T, d->D, d->E, d->k);
  if (st != MOE_OK) return st;
  if (d->F <= 0 || d->Fs < 0) return MOE_ERR_INVALID_ARG;
  if (d->F % 64 != 0 || d->Fs % 64 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if ((long long)d->E * 2 * d->F >= (1LL << 31) || (long long)d->T * d->k * d->F >= (1LL << 40))
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!d->w_gate) return MOE_ERR_INVALID_ARG;
  if (d->weight_format == MOE_WEIGHTS_BF16) {
    if (!d->gate_up || !d->down) return MOE_ERR_INVALID_ARG;
    if ((d->Fs > 0) != (d->shared_gate_up != nullptr) || (d->Fs > 0) != (d->shared_down != nullptr))
      return MOE_ERR_INVALID_ARG;
  } else if (d->weight_format == MOE_WEIGHTS_FP8_E4M3) {
    if (!d->gate_up_fp8 || !d->down_fp8 || !d->gate_up_scale || !d->down_scale) return MOE_ERR_INVALID_ARG;
    const bool sh = d->Fs > 0;
    if (sh != (d->shared_gate_up_fp8 != nullptr) || sh != (d->shared_down_fp8 != nullptr) ||
        sh != (d->shared_gate_up_scale != nullptr) || sh != (d->shared_down_scale != nullptr))
      return MOE_ERR_INVALID_ARG;
    if (d->flags & (MOE_FLAG_FORCE_PREFILL | MOE_FLAG_SAVE_FOR_BACKWARD)) return MOE_ERR_INVALID_ARG;
    if (d->T > kDecodeTMax) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(d->gate_up_fp8, 16) || !aligned(d->down_fp8, 16) || !aligned(d->shared_gate_up_fp8, 16) ||
        !aligned(d->shared_down_fp8, 16) || !aligned(d->gate_up_scale, 4) || !aligned(d->down_scale, 4) ||
        !aligned(d->shared_gate_up_scale, 4) || !aligned(d->shared_down_scale, 4))
      return MOE_ERR_ALIGNMENT;
  } else {
    return MOE_ERR_INVALID_ARG;
  }
  if ((d->flags & ~(MOE_FLAG_FORCE_PREFILL | MOE_FLAG_FORCE_DECODE | MOE_FLAG_SAVE_FOR_BACKWARD |
                    MOE_FLAG_PREFILL_ROW_TILES | MOE_FLAG_PREFILL_WIDE_TILES | MOE_FLAG_PREFILL_PAIR_TILES)) != 0)
    return MOE_ERR_INVALID_ARG;
  const int tiling = d->flags & (MOE_FLAG_PREFILL_ROW_TILES | MOE_FLAG_PREFILL_WIDE_TILES | MOE_FLAG_PREFILL_PAIR_TILES);
  if (tiling & (tiling - 1)) return MOE_ERR_INVALID_ARG;  // at most one tiling flag
  if (tiling && ((d->flags & MOE_FLAG_FORCE_DECODE) || d->weight_format != MOE_WEIGHTS_BF16)) return MOE_ERR_INVALID_ARG;
  if ((d->flags & MOE_FLAG_SAVE_FOR_BACKWARD) && (d->flags & MOE_FLAG_FORCE_DECODE)) return MOE_ERR_INVALID_ARG;
  if ((d->flags & MOE_FLAG_FORCE_PREFILL) && (d->flags & MOE_FLAG_FORCE_DECODE)) return MOE_ERR_INVALID_ARG;
  if ((d->flags & MOE_FLAG_FORCE_DECODE) && d->T > kDecodeTMax) return MOE_ERR_INVALID_ARG;
  if (!aligned(d->w_gate, 16) || !aligned(d->gate_up, 16) || !aligned(d->down, 16) ||
      !aligned(d->shared_gate_up, 16) || !aligned(d->shared_down, 16) || !aligned(d->bias, 4))
    return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}


#define MOE_CUDA_TRY(expr)                 \
  do {                                     \
    if ((expr) != cudaSuccess) {           \
      cudaGetLastError();                  \
      return MOE_ERR_CUDA;                 \
    }                                      \
  } while (0)

moe_status_t run_ffn(const uint16_t* x_perm, const int32_t* offsets, const float* row_scale, int M, int E, int D,
                     int F, const uint16_t* gate_up, const uint16_t* down, uint16_t* h, float* out_perm,
                     // optional shared expert over x[T, D]
                     const uint16_t* x, int T, int Fs, const uint16_t* sgu, const uint16_t* sdn, uint16_t* h_sh,
                     float* out_sh, int decode_nt, Tiling tiling, int* err, cudaStream_t s, cudaEvent_t ev_mid,
                     unsigned ev_flags, uint16_t* save_gu = nullptr, uint16_t* save_gu_sh = nullptr) {
  GemmSetHost g[2] = {};
  g[0].K = D, g[0].a = x_perm, g[0].a_rows = M, g[0].w = gate_up, g[0].n_groups = E, g[0].offsets = offsets;
  g[0].n_out = F, g[0].out = h, g[0].save_gu = save_gu;
  int n_sets = 1;
  if (Fs > 0) {
    g[1].K = D, g[1].a = x, g[1].a_rows = T, g[1].w = sgu, g[1].n_groups = 1, g[1].m_rows = T;
    g[1].n_out = Fs, g[1].out = h_sh, g[1].save_gu = save_gu_sh;
    n_sets = 2;
  }
  if (decode_nt == 0)
    MOE_CUDA_TRY(launch_tiled((TileKind)tiling.gu, kGateUp, g, n_sets, err, s));
  else
    MOE_CUDA_TRY(launch_grouped_gemm(kGateUp, g, n_sets, decode_nt, err, s));
  if (ev_mid) MOE_CUDA_TRY(cudaEventRecordWithFlags(ev_mid, s, ev_flags));
  GemmSetHost dn[2] = {};
  dn[0].K = F, dn[0].a = h, dn[0].a_rows = M, dn[0].w = down, dn[0].n_groups = E, dn[0].offsets = offsets;
  dn[0].n_out = D, dn[0].out = out_perm, dn[0].row_scale = row_scale;
  if (Fs > 0) {
    dn[1].K = Fs, dn[1].a = h_sh, dn[1].a_rows = T, dn[1].w = sdn, dn[1].n_groups = 1, dn[1].m_rows = T;
    dn[1].n_out = D, dn[1].out = out_sh;
  }
  if (decode_nt == 0)
    MOE_CUDA_TRY(launch_tiled((TileKind)tiling.dn, kDown, dn, n_sets, err, s));
  else
    MOE_CUDA_TRY(launch_grouped_gemm(kDown, dn, n_sets, decode_nt, err, s));
  return MOE_OK;
}

// The shared expert of a prefill forward depends only on x, so it runs on a side stream while the
// caller's stream routes and dispatches: a fork after the router GEMM and a join before the
// combine (captured into a CUDA graph as two parallel branches like any cross-stream dependency).
// One side stream and its two events per (device, caller stream), created on first use and kept
// until the process exits.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

moe_status_t side_stream_for(cudaStream_t main, SideStream* out) {
  static std::mutex mu;
  static std::map<std::pair<int, cudaStream_t>, SideStream> table;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(mu);
  auto it = table.find({dev, main});
  if (it == table.end()) {
    SideStream ss;
    if (cudaStreamCreateWithFlags(&ss.stream, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    it = table.emplace(std::make_pair(dev, main), ss).first;
  }
  *out = it->second;
  return MOE_OK;
}

// prefill forwards with a shared expert fork it onto the side stream (bf16 weights)
bool fork_shared_expert(const moe_layer_desc_t& d) {
  return d.Fs > 0 && !use_decode(d) && d.weight_format == MOE_WEIGHTS_BF16;
}

// The shared expert alone: gate_up (+ SwiGLU) then down over the T rows of x, one group each.
moe_status_t run_shared_ffn(const uint16_t* x, int T, int D, int Fs, const uint16_t* sgu, const uint16_t* sdn,
                            uint16_t* h_sh, float* out_sh, Tiling tiling, uint16_t* save_gu_sh, int* err,
                            cudaStream_t s) {
  GemmSetHost g = {};
  g.K = D, g.a = x, g.a_rows = T, g.w = sgu, g.n_groups = 1, g.m_rows = T, g.n_out = Fs, g.out = h_sh;
  g.save_gu = save_gu_sh;
  MOE_CUDA_TRY(launch_tiled((TileKind)tiling.gu, kGateUp, &g, 1, err, s));
  GemmSetHost dn = {};
  dn.K = Fs, dn.a = h_sh, dn.a_rows = T, dn.w = sdn, dn.n_groups = 1, dn.m_rows = T, dn.n_out = D, dn.out = out_sh;
  MOE_CUDA_TRY(launch_tiled((TileKind)tiling.dn, kDown, &dn, 1, err, s));
  return MOE_OK;
}

moe_status_t layer_forward(const moe_layer_desc_t* d, const uint16_t* x, uint16_t* y, void* ws, size_t ws_bytes,
                           cudaStream_t s, cudaEvent_t const* ev) {
  moe_status_t st = validate_desc(d);
  if (st != MOE_OK) return st;
  if (!x || !y || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(ws, 256)) return MOE_ERR_ALIGNMENT;
  const LayerWs w = layer_ws(*d);
  if (ws_bytes < w.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if ((st = check_device()) != MOE_OK) return st;
  if (d->T == 0) return MOE_OK;

  uint8_t* b = static_cast<uint8_t*>(ws);
  int* err = reinterpret_cast<int*>(b);
  auto I = [&](size_t off) { return reinterpret_cast<int32_t*>(b + off); };
  auto Fp = [&](size_t off) { return reinterpret_cast<float*>(b + off); };
  auto H = [&](size_t off) { return reinterpret_cast<uint16_t*>(b + off); };
  const int T = d->T, D = d->D, E = d->E, k = d->k, F = d->F, Fs = d->Fs, M = T * k;

  // Under stream capture, stage events become event-record nodes of the graph (so they can
  // time each replay); otherwise they are plain records on the stream.
  unsigned rec_flags = cudaEventRecordDefault;
  if (ev) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    MOE_CUDA_TRY(cudaStreamIsCapturing(s, &cs));
    if (cs == cudaStreamCaptureStatusActive) rec_flags = cudaEventRecordExternal;
  }
  auto record = [&](cudaEvent_t e) { return cudaEventRecordWithFlags(e, s, rec_flags); };

  if (ev) MOE_CUDA_TRY(record(ev[0]));
  // a fresh error word and zeroed split-K counters (they follow the header) for this forward
  MOE_CUDA_TRY(cudaMemsetAsync(err, 0, w.split_counters + kSplitCounterBytes, s));
  const int splits = router_k_splits(T, D, E);
  const bool fp8 = d->weight_format == MOE_WEIGHTS_FP8_E4M3;
  const int nt = use_decode(*d) ? decode_tile(T) : 0;
  // prefill with a shared expert: it runs on a side stream (forked after the router GEMM) and the
  // routed GEMMs below leave it out
  const bool fork = fork_shared_expert(*d);
  SideStream side;
  if (fork && (st = side_stream_for(s, &side)) != MOE_OK) return st;
  // joins the side stream's branch back into `s` when armed: before the combine, or on an early
  // error return (a capture of `s` must not end with an unjoined branch)
  struct Join {
    cudaStream_t s;
    cudaEvent_t e;
    bool armed = false;
    bool wait() {
      armed = false;
      if (cudaStreamWaitEvent(s, e, 0) == cudaSuccess) return true;
      cudaGetLastError();
      return false;
    }
    ~Join() {
      if (armed) wait();
    }
  } join{s, side.join};
  MOE_CUDA_TRY(launch_router_gemm(x, d->w_gate, T, D, E, Fp(w.router), router_ld(E), splits, err, s));
  if (fork) {
    // the shared expert's branch: it needs only x, and the GEMMs it runs take the SMs the
    // latency-bound top-k and dispatch kernels leave idle
    if (cudaEventRecord(side.fork, s) != cudaSuccess || cudaStreamWaitEvent(side.stream, side.fork, 0) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    const moe_status_t sst =
        run_shared_ffn(x, T, D, Fs, d->shared_gate_up, d->shared_down, H(w.h_sh), Fp(w.out_sh),
                       prefill_tiling(d->flags), (d->flags & MOE_FLAG_SAVE_FOR_BACKWARD) ? H(w.gu_saved_sh) : nullptr,
                       err, side.stream);
    if (cudaEventRecord(side.join, side.stream) != cudaSuccess) {
      cudaGetLastError();
      return MOE_ERR_CUDA;
    }
    join.armed = true;  // `s` waits for the branch before the combine, or on any early return
    if (sst != MOE_OK) return sst;
  }
  MOE_CUDA_TRY(launch_router_select(Fp(w.router), splits, T, router_ld(E), d->bias, E, k, I(w.topk_idx),
                                    Fp(w.topk_w), s));
  if (ev) MOE_CUDA_TRY(record(ev[1]));
  // dispatch + gather (one kernel for T <= 256); the FP8 path gathers f16 rows and, for the
  // shared expert, an f16 copy of x
  MOE_CUDA_TRY(launch_permute(I(w.topk_idx), Fp(w.topk_w), x, T, D, E, k, I(w.counts), I(w.offsets), I(w.perm_token),
                              I(w.inv_perm), Fp(w.p_perm), H(w.x_perm), fp8, (fp8 && Fs > 0) ? H(w.x16) : nullptr,
                              I(w.scratch), err, s, nullptr));
  if (ev) MOE_CUDA_TRY(record(ev[2]));
  SplitBuf split;  // split-K buffers of the FP8 weight-streaming GEMMs
  if (w.split_partial_bytes > 0) {
    split.partial = Fp(w.split_partial);
    split.partial_bytes = w.split_partial_bytes;
    split.counters = I(w.split_counters);
  }
  if (fp8) {
    GemmSetHost g[2];
    memset(g, 0, sizeof(g));
    const float* gs[2] = {d->gate_up_scale, d->shared_gate_up_scale};
    g[0].K = D, g[0].a = H(w.x_perm), g[0].a_rows = M, g[0].w = reinterpret_cast<const uint16_t*>(d->gate_up_fp8);
    g[0].n_groups = E, g[0].offsets = I(w.offsets), g[0].n_out = F, g[0].out = H(w.h);
    if (Fs > 0) {
      g[1].K = D, g[1].a = H(w.x16), g[1].a_rows = T, g[1].w = reinterpret_cast<const uint16_t*>(d->shared_gate_up_fp8);
      g[1].n_groups = 1, g[1].m_rows = T, g[1].n_out = Fs, g[1].out = H(w.h_sh);
    }
    MOE_CUDA_TRY(launch_stream_fp8w(kGateUp, g, gs, Fs > 0 ? 2 : 1, nt, split, err, s));
    if (ev) MOE_CUDA_TRY(record(ev[3]));
    GemmSetHost dn[2];
    memset(dn, 0, sizeof(dn));
    const float* ds[2] = {d->down_scale, d->shared_down_scale};
    dn[0].K = F, dn[0].a = H(w.h), dn[0].a_rows = M, dn[0].w = reinterpret_cast<const uint16_t*>(d->down_fp8);
    dn[0].n_groups = E, dn[0].offsets = I(w.offsets), dn[0].n_out = D, dn[0].out = Fp(w.out_perm);
    dn[0].row_scale = Fp(w.p_perm);
    if (Fs > 0) {
      dn[1].K = Fs, dn[1].a = H(w.h_sh), dn[1].a_rows = T, dn[1].w = reinterpret_cast<const uint16_t*>(d->shared_down_fp8);
      dn[1].n_groups = 1, dn[1].m_rows = T, dn[1].n_out = D, dn[1].out = Fp(w.out_sh);
    }
    MOE_CUDA_TRY(launch_stream_fp8w(kDown, dn, ds, Fs > 0 ? 2 : 1, nt, split, err, s));
  } else {
  st = run_ffn(H(w.x_perm), I(w.offsets), Fp(w.p_perm), M, E, D, F, d->gate_up, d->down, H(w.h), Fp(w.out_perm), x,
               T, fork ? 0 : Fs, d->shared_gate_up, d->shared_down, H(w.h_sh), Fp(w.out_sh), nt, prefill_tiling(d->flags), err,
               s, ev ? ev[3] : nullptr,
               rec_flags, (d->flags & MOE_FLAG_SAVE_FOR_BACKWARD) ? H(w.gu_saved) : nullptr,
               (d->flags & MOE_FLAG_SAVE_FOR_BACKWARD) && Fs > 0 ? H(w.gu_saved_sh) : nullptr);
  if (st != MOE_OK) return st;
  }
  if (ev) MOE_CUDA_TRY(record(ev[4]));
  if (join.armed && !join.wait()) return MOE_ERR_CUDA;
  MOE_CUDA_TRY(launch_combine(Fp(w.out_perm), I(w.inv_perm), Fs > 0 ? Fp(w.out_sh) : nullptr, T, D, k, y, s));
  if (ev) MOE_CUDA_TRY(record(ev[5]));
  return MOE_OK;
}

// Backward workspace: per-row gradients in the 64-row padded per-expert layout (rows_pad rows at
// most: every expert pads fewer than 64 rows).
struct BwdWs {
  size_t pad_offsets, dyp, d_o, dgu, dxp, dp_part, dl_row, dgu_sh, dx_sh, total;
  int64_t rows_pad;
  int n_tiles;  // 256-column tiles of F: the partial dp per row
};

BwdWs bwd_ws(const moe_layer_desc_t& d) {
  BwdWs b;
  size_t o = kWsHeader;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  const size_t T = d.T, D = d.D, E = d.E, k = d.k, F = d.F, Fs = d.Fs, M = T * k;
  b.rows_pad = (int64_t)M + 64 * (int64_t)E;
  b.n_tiles = (d.F + 255) / 256;
  const size_t R = (size_t)b.rows_pad;
  b.pad_offsets = take((E + 1) * 4);
  b.dyp = take(R * D * 2);
  b.d_o = take(R * D * 2);
  b.dgu = take(R * 2 * F * 2);
  b.dxp = take(R * D * 4);
  b.dp_part = take(M * b.n_tiles * 4);
  b.dl_row = take(M * 4);
  b.dgu_sh = take(T * 2 * Fs * 2);
  b.dx_sh = take(T * D * 4);
  b.total = o;
  return b;
}

moe_status_t validate_backward(const moe_layer_desc_t* d) {
  moe_status_t st = validate_desc(d);
  if (st != MOE_OK) return st;
  if (!(d->flags & MOE_FLAG_SAVE_FOR_BACKWARD) || d->weight_format != MOE_WEIGHTS_BF16) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status_t status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE";
    case MOE_ERR_ALIGNMENT: return "MOE_ERR_ALIGNMENT";
    case MOE_ERR_WORKSPACE_TOO_SMALL: return "MOE_ERR_WORKSPACE_TOO_SMALL";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_INDEX: return "MOE_ERR_DEVICE_INDEX";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT";
    case MOE_ERR_NO_DEVICE: return "MOE_ERR_NO_DEVICE";
  }
  return "MOE_ERR_UNKNOWN";
}

size_t moe_router_topk_workspace_size(int T, int D, int E) {
  if (shape_status(T, D, E, 1) != MOE_OK) return 0;
  return kWsHeader + router_scratch_bytes(T, D, E);
}

moe_status_t moe_router_topk(const moe_bf16_t* x, const moe_bf16_t* w_gate, const float* bias, int T, int D, int E,
                             int k, int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                             moe_stream_t stream) {
  moe_status_t st = shape_status(T, D, E, k);
  if (st != MOE_OK) return st;
  if (!x || !w_gate || !topk_idx || !topk_w || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w_gate, 16) || !aligned(bias, 4) || !aligned(topk_idx, 4) ||
      !aligned(topk_w, 4) || !aligned(ws, 256))
    return MOE_ERR_ALIGNMENT;
  if (ws_bytes < moe_router_topk_workspace_size(T, D, E)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if ((st = check_device()) != MOE_OK) return st;
  if (T == 0) return MOE_OK;
  uint8_t* b = static_cast<uint8_t*>(ws);
  float* part = reinterpret_cast<float*>(b + kWsHeader);
  const int splits = router_k_splits(T, D, E);
  cudaStream_t s = (cudaStream_t)stream;
  MOE_CUDA_TRY(launch_router_gemm(x, w_gate, T, D, E, part, router_ld(E), splits, reinterpret_cast<int*>(b), s));
  MOE_CUDA_TRY(launch_router_select(part, splits, T, router_ld(E), bias, E, k, topk_idx, topk_w, s));
  return MOE_OK;
}

namespace {
struct AuxWs {
  size_t part, idx, w, counts, c, dl, split, total;
};
AuxWs aux_ws(int T, int D, int E, int k) {
  AuxWs a;
  size_t o = kWsHeader;
  auto take = [&](size_t bytes) {
    const size_t at = o;
    o = align_up(o + bytes, 256);
    return at;
  };
  a.part = take(router_scratch_bytes(T, D, E));
  a.idx = take((size_t)T * k * 4);
  a.w = take((size_t)T * k * 4);
  a.counts = take((size_t)E * 4);
  a.c = take((size_t)T * 4);
  a.dl = take((size_t)T * E * 4);
  const int S = T > 0 ? aux_token_splits(T, D, E) : 1;
  a.split = take(S > 1 ? (size_t)S * E * D * 4 : 0);
  a.total = o;
  return a;
}
}  // namespace

size_t moe_router_aux_loss_workspace_size(int T, int D, int E, int k) {
  if (shape_status(T, D, E, k) != MOE_OK) return 0;
  return aux_ws(T, D, E, k).total;
}

moe_status_t moe_router_aux_loss(const moe_bf16_t* x, const moe_bf16_t* w_gate, const float* bias, int T, int D,
                                 int E, int k, float alpha, float* loss, float* dw_gate, float* dx, void* ws,
                                 size_t ws_bytes, moe_stream_t stream) {
  moe_status_t st = shape_status(T, D, E, k);
  if (st != MOE_OK) return st;
  if (!x || !w_gate || !loss || !dw_gate || !dx || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w_gate, 16) || !aligned(bias, 4) || !aligned(loss, 4) || !aligned(dw_gate, 4) ||
      !aligned(dx, 4) || !aligned(ws, 256))
    return MOE_ERR_ALIGNMENT;
  const AuxWs a = aux_ws(T, D, E, k);
  if (ws_bytes < a.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if ((st = check_device()) != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if (T == 0) {
    MOE_CUDA_TRY(cudaMemsetAsync(loss, 0, sizeof(float), s));
    MOE_CUDA_TRY(cudaMemsetAsync(dw_gate, 0, (size_t)E * D * sizeof(float), s));
    return MOE_OK;
  }
  uint8_t* b = static_cast<uint8_t*>(ws);
  auto Fp = [&](size_t off) { return reinterpret_cast<float*>(b + off); };
  auto I = [&](size_t off) { return reinterpret_cast<int32_t*>(b + off); };
  MOE_CUDA_TRY(cudaMemsetAsync(b, 0, kWsHeader, s));
  MOE_CUDA_TRY(cudaMemsetAsync(b + a.counts, 0, (size_t)E * 4, s));
  const int splits = router_k_splits(T, D, E);
  MOE_CUDA_TRY(launch_router_gemm(x, w_gate, T, D, E, Fp(a.part), router_ld(E), splits, reinterpret_cast<int*>(b), s));
  MOE_CUDA_TRY(launch_router_select(Fp(a.part), splits, T, router_ld(E), bias, E, k, I(a.idx), Fp(a.w), s));
  MOE_CUDA_TRY(launch_router_aux(Fp(a.part), splits, router_ld(E), I(a.idx), x, w_gate, T, D, E, k, alpha, I(a.counts),
                                 Fp(a.c), Fp(a.dl), Fp(a.split), loss, dw_gate, dx, s));
  return MOE_OK;
}

moe_status_t moe_quantize_rows_fp8(const moe_bf16_t* w, int64_t rows, int K, uint8_t* q, float* scales,
                                   moe_stream_t stream) {
  if (!w || !q || !scales || rows < 0 || K <= 0) return MOE_ERR_INVALID_ARG;
  if (K % 64 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(w, 16) || !aligned(q, 16) || !aligned(scales, 4)) return MOE_ERR_ALIGNMENT;
  moe_status_t st = check_device();
  if (st != MOE_OK) return st;
  MOE_CUDA_TRY(launch_quantize_rows_fp8(w, rows, K, q, scales, (cudaStream_t)stream));
  return MOE_OK;
}

size_t moe_permute_workspace_size(int T, int E, int k) {
  if (shape_status(T, 64, E, k) != MOE_OK) return 0;
  return kWsHeader + permute_scratch_bytes(T, E);
}

moe_status_t moe_permute(const int32_t* topk_idx, const float* topk_w, const moe_bf16_t* x, int T, int D, int E, int k,
                         int32_t* counts, int32_t* offsets, int32_t* perm_token, int32_t* inv_perm, float* p_perm,
                         moe_bf16_t* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status_t st = shape_status(T, D, E, k);
  if (st != MOE_OK) return st;
  if (!topk_idx || !topk_w || !counts || !offsets || !perm_token || !inv_perm || !p_perm || !ws)
    return MOE_ERR_INVALID_ARG;
  if ((x == nullptr) != (x_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(x_perm, 16) || !aligned(ws, 256) || !aligned(topk_idx, 4) ||
      !aligned(topk_w, 4) || !aligned(counts, 4) || !aligned(offsets, 4) || !aligned(perm_token, 4) ||
      !aligned(inv_perm, 4) || !aligned(p_perm, 4))
    return MOE_ERR_ALIGNMENT;
  if (ws_bytes < moe_permute_workspace_size(T, E, k)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if ((st = check_device()) != MOE_OK) return st;
  uint8_t* b = static_cast<uint8_t*>(ws);
  MOE_CUDA_TRY(launch_permute(topk_idx, topk_w, x, T, D, E, k, counts, offsets, perm_token, inv_perm, p_perm, x_perm,
                              false, nullptr, reinterpret_cast<int32_t*>(b + kWsHeader), reinterpret_cast<int*>(b),
                              (cudaStream_t)stream, nullptr));
  return MOE_OK;
}

size_t moe_grouped_swiglu_ffn_workspace_size(int M, int F) {
  if (M < 0 || F <= 0 || F % 64 != 0) return 0;
  return kWsHeader + align_up((size_t)M * F * 2, 256);
}

moe_status_t moe_grouped_swiglu_ffn(const moe_bf16_t* x_perm, const int32_t* offsets, const float* row_scale, int M,
                                    int max_seg, int flags, int E, int D, int F, const moe_bf16_t* gate_up,
                                    const moe_bf16_t* down, float* out_perm, void* ws, size_t ws_bytes,
                                    moe_stream_t stream) {
  if (M < 0 || E <= 0 || D <= 0 || F <= 0 || max_seg < 0 || max_seg > M) return MOE_ERR_INVALID_ARG;
  const int tiling_flags = MOE_FLAG_PREFILL_ROW_TILES | MOE_FLAG_PREFILL_WIDE_TILES | MOE_FLAG_PREFILL_PAIR_TILES;
  if ((flags & ~tiling_flags) != 0 || (flags & (flags - 1)) != 0) return MOE_ERR_INVALID_ARG;
  if (D % 64 != 0 || F % 64 != 0 || E > 1024) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!x_perm || !offsets || !gate_up || !down || !out_perm || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned(x_perm, 16) || !aligned(gate_up, 16) || !aligned(down, 16) || !aligned(out_perm, 16) ||
      !aligned(ws, 256) || !aligned(offsets, 4) || !aligned(row_scale, 4))
    return MOE_ERR_ALIGNMENT;
  if (ws_bytes < moe_grouped_swiglu_ffn_workspace_size(M, F)) return MOE_ERR_WORKSPACE_TOO_SMALL;
  moe_status_t st = check_device();
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  uint8_t* b = static_cast<uint8_t*>(ws);
  const int nt = max_seg <= kDecodeTMax ? decode_tile(max_seg < 1 ? 1 : max_seg) : 0;
  return run_ffn(x_perm, offsets, row_scale, M, E, D, F, gate_up, down, reinterpret_cast<uint16_t*>(b + kWsHeader),
                 out_perm, nullptr, 0, 0, nullptr, nullptr, nullptr, nullptr, nt, prefill_tiling(flags),
                 reinterpret_cast<int*>(b),
                 (cudaStream_t)stream, nullptr, cudaEventRecordDefault);
}

moe_status_t moe_combine(const float* out_perm, const int32_t* inv_perm, const float* shared_out, int T, int D,
                         int k, moe_bf16_t* y, moe_stream_t stream) {
  if (T < 0 || D <= 0 || k <= 0) return MOE_ERR_INVALID_ARG;
  if (D % 64 != 0 || k > 32 || (long long)T * k >= (1LL << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!out_perm || !inv_perm || !y) return MOE_ERR_INVALID_ARG;
  if (!aligned(out_perm, 16) || !aligned(shared_out, 16) || !aligned(y, 16) || !aligned(inv_perm, 4))
    return MOE_ERR_ALIGNMENT;
  moe_status_t st = check_device();
  if (st != MOE_OK) return st;
  MOE_CUDA_TRY(launch_combine(out_perm, inv_perm, shared_out, T, D, k, y, (cudaStream_t)stream));
  return MOE_OK;
}

size_t moe_layer_workspace_size(const moe_layer_desc_t* desc) {
  if (validate_desc(desc) != MOE_OK) return 0;
  return layer_ws(*desc).total;
}

moe_status_t moe_layer_forward(const moe_layer_desc_t* desc, const moe_bf16_t* x, moe_bf16_t* y, void* ws,
                               size_t ws_bytes, moe_stream_t stream) {
  return layer_forward(desc, x, y, ws, ws_bytes, (cudaStream_t)stream, nullptr);
}

moe_status_t moe_layer_forward_timed(const moe_layer_desc_t* desc, const moe_bf16_t* x, moe_bf16_t* y, void* ws,
                                     size_t ws_bytes, moe_stream_t stream, void* const* events, int n_events) {
  if (events == nullptr || n_events < 6) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i)
    if (events[i] == nullptr) return MOE_ERR_INVALID_ARG;
  return layer_forward(desc, x, y, ws, ws_bytes, (cudaStream_t)stream,
                       reinterpret_cast<cudaEvent_t const*>(events));
}

moe_status_t moe_layer_forward_host(const moe_layer_desc_t* desc, const moe_bf16_t* x_host, moe_bf16_t* y_host,
                                    void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status_t st = validate_desc(desc);
  if (st != MOE_OK) return st;
  if (!x_host || !y_host || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_ALIGNMENT;
  const LayerWs w = layer_ws(*desc);
  if (ws_bytes < w.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if ((st = check_device()) != MOE_OK) return st;
  if (desc->T == 0) return MOE_OK;
  uint8_t* b = static_cast<uint8_t*>(ws);
  const size_t bytes = (size_t)desc->T * desc->D * 2;
  cudaStream_t s = (cudaStream_t)stream;
  MOE_CUDA_TRY(cudaMemcpyAsync(b + w.x_stage, x_host, bytes, cudaMemcpyHostToDevice, s));
  st = layer_forward(desc, reinterpret_cast<uint16_t*>(b + w.x_stage), reinterpret_cast<uint16_t*>(b + w.y_stage),
                     ws, ws_bytes, s, nullptr);
  if (st != MOE_OK) return st;
  MOE_CUDA_TRY(cudaMemcpyAsync(y_host, b + w.y_stage, bytes, cudaMemcpyDeviceToHost, s));
  return MOE_OK;
}

int moe_layer_kernel_count(const moe_layer_desc_t* desc) {
  if (validate_desc(desc) != MOE_OK || desc->T == 0) return 0;
  // T <= 256: one kernel sorts and gathers (and casts x for the FP8 path's shared expert, T <= 64);
  // above: hist, scan, scatter, gather
  const int dispatch = desc->T <= 256 ? 1 : 4;
  const int gemms = fork_shared_expert(*desc) ? 4 : 2;  // the shared expert's own two on the side stream
  return 2 /*router GEMM, top-k*/ + dispatch + gemms + 1 /*combine*/;
}

int moe_layer_gemm_path(const moe_layer_desc_t* desc) {
  if (validate_desc(desc) != MOE_OK) return -1;
  if (desc->weight_format == MOE_WEIGHTS_FP8_E4M3) return MOE_PATH_FP8_STREAMING;
  if (use_decode(*desc)) return MOE_PATH_STREAMING;
  const Tiling t = prefill_tiling(desc->flags);
  if (t.gu == kRowT && t.dn == kRowT) return MOE_PATH_ROW_TILES;
  if (t.gu == kWideT && t.dn == kWideT) return MOE_PATH_WIDE_TILES;
  if (t.gu == kPairT && t.dn == kPairT) return MOE_PATH_PAIR_TILES;
  if (t.gu == kRowT && t.dn == kPairT) return MOE_PATH_MIXED_TILES;
  return -1;
}

moe_status_t moe_update_router_bias(const int32_t* counts, int E, float gamma, float* bias, moe_stream_t stream) {
  if (!counts || !bias || E <= 0) return MOE_ERR_INVALID_ARG;
  if (E > 1024) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!(gamma >= 0.0f) || gamma > 1e30f) return MOE_ERR_INVALID_ARG;  // also rejects NaN
  if (!aligned(counts, 4) || !aligned(bias, 4)) return MOE_ERR_ALIGNMENT;
  moe_status_t st = check_device();
  if (st != MOE_OK) return st;
  MOE_CUDA_TRY(launch_update_bias(counts, E, gamma, bias, (cudaStream_t)stream));
  return MOE_OK;
}

moe_status_t moe_layer_expert_counts(const moe_layer_desc_t* desc, void* ws, size_t ws_bytes,
                                     const int32_t** counts) {
  moe_status_t st = validate_desc(desc);
  if (st != MOE_OK) return st;
  if (!ws || !counts) return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_ALIGNMENT;
  const LayerWs w = layer_ws(*desc);
  if (ws_bytes < w.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  *counts = reinterpret_cast<const int32_t*>(static_cast<const uint8_t*>(ws) + w.counts);
  return MOE_OK;
}

size_t moe_layer_backward_workspace_size(const moe_layer_desc_t* desc) {
  if (validate_backward(desc) != MOE_OK) return 0;
  return bwd_ws(*desc).total;
}

moe_status_t moe_layer_backward(const moe_layer_desc_t* desc, const moe_bf16_t* x, const moe_bf16_t* dy,
                                moe_bf16_t* dx, const moe_layer_grads_t* grads, const void* fwd_ws,
                                size_t fwd_ws_bytes, void* bwd_ws_ptr, size_t bwd_ws_bytes, moe_stream_t stream) {
  moe_status_t st = validate_backward(desc);
  if (st != MOE_OK) return st;
  const moe_layer_desc_t& d = *desc;
  if (!x || !dy || !dx || !grads || !fwd_ws || !bwd_ws_ptr || !grads->dw_gate || !grads->dgate_up || !grads->ddown)
    return MOE_ERR_INVALID_ARG;
  if ((d.Fs > 0) != (grads->dshared_gate_up != nullptr) || (d.Fs > 0) != (grads->dshared_down != nullptr))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(dy, 16) || !aligned(dx, 16) || !aligned(grads->dw_gate, 16) ||
      !aligned(grads->dgate_up, 16) || !aligned(grads->ddown, 16) || !aligned(grads->dshared_gate_up, 16) ||
      !aligned(grads->dshared_down, 16) || !aligned(fwd_ws, 256) || !aligned(bwd_ws_ptr, 256))
    return MOE_ERR_ALIGNMENT;
  const LayerWs w = layer_ws(d);
  const BwdWs b = bwd_ws(d);
  if (fwd_ws_bytes < w.total || bwd_ws_bytes < b.total) return MOE_ERR_WORKSPACE_TOO_SMALL;
  if ((st = check_device()) != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const int T = d.T, D = d.D, E = d.E, k = d.k, F = d.F, Fs = d.Fs, M = T * k;
  const size_t nd = (size_t)E * D, ngu = (size_t)E * 2 * F * D, ndn = (size_t)E * D * F;
  if (T == 0) {  // no tokens: every gradient is zero
    MOE_CUDA_TRY(cudaMemsetAsync(grads->dw_gate, 0, nd * 4, s));
    MOE_CUDA_TRY(cudaMemsetAsync(grads->dgate_up, 0, ngu * 4, s));
    MOE_CUDA_TRY(cudaMemsetAsync(grads->ddown, 0, ndn * 4, s));
    if (Fs > 0) {
      MOE_CUDA_TRY(cudaMemsetAsync(grads->dshared_gate_up, 0, (size_t)2 * Fs * D * 4, s));
      MOE_CUDA_TRY(cudaMemsetAsync(grads->dshared_down, 0, (size_t)D * Fs * 4, s));
    }
    return MOE_OK;
  }
  const uint8_t* f = static_cast<const uint8_t*>(fwd_ws);
  uint8_t* bb = static_cast<uint8_t*>(bwd_ws_ptr);
  auto FI = [&](size_t off) { return reinterpret_cast<const int32_t*>(f + off); };
  auto FF = [&](size_t off) { return reinterpret_cast<const float*>(f + off); };
  auto FH = [&](size_t off) { return reinterpret_cast<const uint16_t*>(f + off); };
  auto BI = [&](size_t off) { return reinterpret_cast<int32_t*>(bb + off); };
  auto BF = [&](size_t off) { return reinterpret_cast<float*>(bb + off); };
  auto BH = [&](size_t off) { return reinterpret_cast<uint16_t*>(bb + off); };
  int* err = reinterpret_cast<int*>(bb);
  const int32_t* offsets = FI(w.offsets);
  int32_t* pad = BI(b.pad_offsets);
  const int n_sets = Fs > 0 ? 2 : 1;

  MOE_CUDA_TRY(cudaMemsetAsync(err, 0, sizeof(int), s));
  MOE_CUDA_TRY(launch_pad_offsets(offsets, E, pad, s));
  MOE_CUDA_TRY(launch_gather_dy(dy, offsets, pad, E, FI(w.perm_token), FF(w.p_perm), D, 2 * F, b.rows_pad,
                                BH(b.dyp), BH(b.d_o), BH(b.dgu), s));
  // dHu = dy_perm Down_e, fused SwiGLU backward -> dGU, partial dp
  BwdSetHost st2[2];
  st2[0].a = BH(b.dyp), st2[0].a_rows = b.rows_pad, st2[0].a_cols = D;
  st2[0].b = d.down, st2[0].b_rows = (int64_t)E * D, st2[0].b_cols = F;
  st2[0].offsets = offsets, st2[0].pad_offsets = pad, st2[0].n_groups = E;
  st2[0].K = D, st2[0].N_total = F, st2[0].p_perm = FF(w.p_perm), st2[0].gu_saved = FH(w.gu_saved);
  st2[0].dgu = BH(b.dgu), st2[0].dp_part = BF(b.dp_part);
  if (Fs > 0) {
    st2[1].a = dy, st2[1].a_rows = T, st2[1].a_cols = D;
    st2[1].b = d.shared_down, st2[1].b_rows = D, st2[1].b_cols = Fs;
    st2[1].m_rows = T, st2[1].K = D, st2[1].N_total = Fs, st2[1].gu_saved = FH(w.gu_saved_sh);
    st2[1].dgu = BH(b.dgu_sh);
  }
  MOE_CUDA_TRY(launch_bwd_gemm(kBwdDxDown, st2, n_sets, err, s));
  // dX = dGU gate_up_e
  BwdSetHost sx[2];
  sx[0].a = BH(b.dgu), sx[0].a_rows = b.rows_pad, sx[0].a_cols = 2 * F;
  sx[0].b = d.gate_up, sx[0].b_rows = (int64_t)E * 2 * F, sx[0].b_cols = D;
  sx[0].offsets = offsets, sx[0].pad_offsets = pad, sx[0].n_groups = E;
  sx[0].K = 2 * F, sx[0].N_total = D, sx[0].out = BF(b.dxp);
  if (Fs > 0) {
    sx[1].a = BH(b.dgu_sh), sx[1].a_rows = T, sx[1].a_cols = 2 * Fs;
    sx[1].b = d.shared_gate_up, sx[1].b_rows = 2 * Fs, sx[1].b_cols = D;
    sx[1].m_rows = T, sx[1].K = 2 * Fs, sx[1].N_total = D, sx[1].out = BF(b.dx_sh);
  }
  MOE_CUDA_TRY(launch_bwd_gemm(kBwdDxGateUp, sx, n_sets, err, s));
  // dDown_e = dO_e^T h_e
  BwdSetHost sd[2];
  sd[0].a = BH(b.d_o), sd[0].a_rows = b.rows_pad, sd[0].a_cols = D;
  sd[0].b = FH(w.h), sd[0].b_rows = M, sd[0].b_cols = F;
  sd[0].offsets = offsets, sd[0].pad_offsets = pad, sd[0].n_groups = E;
  sd[0].M_total = D, sd[0].N_total = F, sd[0].out = grads->ddown;
  if (Fs > 0) {
    sd[1].a = dy, sd[1].a_rows = T, sd[1].a_cols = D;
    sd[1].b = FH(w.h_sh), sd[1].b_rows = T, sd[1].b_cols = Fs;
    sd[1].m_rows = T, sd[1].M_total = D, sd[1].N_total = Fs, sd[1].out = grads->dshared_down;
  }
  MOE_CUDA_TRY(launch_bwd_gemm(kBwdDwDown, sd, n_sets, err, s));
  // dGateUp_e = dGU_e^T x_perm_e
  BwdSetHost su[2];
  su[0].a = BH(b.dgu), su[0].a_rows = b.rows_pad, su[0].a_cols = 2 * F;
  su[0].b = FH(w.x_perm), su[0].b_rows = M, su[0].b_cols = D;
  su[0].offsets = offsets, su[0].pad_offsets = pad, su[0].n_groups = E;
  su[0].M_total = 2 * F, su[0].N_total = D, su[0].out = grads->dgate_up;
  if (Fs > 0) {
    su[1].a = BH(b.dgu_sh), su[1].a_rows = T, su[1].a_cols = 2 * Fs;
    su[1].b = x, su[1].b_rows = T, su[1].b_cols = D;
    su[1].m_rows = T, su[1].M_total = 2 * Fs, su[1].N_total = D, su[1].out = grads->dshared_gate_up;
  }
  MOE_CUDA_TRY(launch_bwd_gemm(kBwdDwGateUp, su, n_sets, err, s));
  // router: dp -> dl (softmax over the chosen k), dW_g, and dx
  MOE_CUDA_TRY(launch_router_bwd(FI(w.inv_perm), FF(w.topk_w), BF(b.dp_part), b.n_tiles, T, k, BF(b.dl_row), s));
  MOE_CUDA_TRY(launch_dwgate(offsets, BF(b.dl_row), FH(w.x_perm), E, D, grads->dw_gate, s));
  MOE_CUDA_TRY(launch_unpermute(BF(b.dxp), Fs > 0 ? BF(b.dx_sh) : nullptr, FI(w.inv_perm), FI(w.topk_idx), offsets,
                                pad, BF(b.dl_row), d.w_gate, T, D, k, dx, s));
  return MOE_OK;
}

moe_status_t moe_get_device_error(void* ws, moe_stream_t stream) {
  if (!ws) return MOE_ERR_INVALID_ARG;
  if (!aligned(ws, 256)) return MOE_ERR_ALIGNMENT;
  moe_status_t st = check_device();
  if (st != MOE_OK) return st;
  int h = 0;
  cudaStream_t s = (cudaStream_t)stream;
  MOE_CUDA_TRY(cudaMemcpyAsync(&h, ws, sizeof(int), cudaMemcpyDeviceToHost, s));
  MOE_CUDA_TRY(cudaStreamSynchronize(s));
  if (h != 0) {
    MOE_CUDA_TRY(cudaMemsetAsync(ws, 0, sizeof(int), s));
    MOE_CUDA_TRY(cudaStreamSynchronize(s));
  }
  if (h & kErrTimeout) return MOE_ERR_TIMEOUT;
  if (h & kErrBadIndex) return MOE_ERR_DEVICE_INDEX;
  return MOE_OK;
}

}  // extern "C"
