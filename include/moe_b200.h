/*
 * moe_b200.h -- C ABI of the sparse Mixture-of-Experts FFN layer forward on one B200 (sm_100a).
 *
 * The layer (gotburnout.io glossary "MoE (Mixture of Experts)", section 2, layer diagram and
 * section 3, token pipeline; josueisai.com "Mixture of experts", section "El router"):
 *
 *     logits = W_g x                       router projection, fp32 accumulation
 *     S      = the k experts with the largest (logits + bias)   (bias: optional, selection only)
 *     p_j    = softmax over the chosen k of the unbiased logits
 *     y      = sum_j p_j * Expert_{S_j}(x) + SharedExpert(x)
 *     Expert_e(x) = down[e] (silu(G_e x) * (U_e x)),   G_e = gate_up[e][0:F], U_e = gate_up[e][F:2F]
 *
 * The residual add of the diagram is the caller's: y excludes it.
 *
 * Packed weights (dev.smart-guide.co.kr deep-dive, section "La Solucion: WeightConverter": the
 * per-expert w1 / w3 matrices merged on a new expert dim 0 and concatenated on dim 1):
 *     gate_up [E, 2F, D]  row-major, rows [0,F) = w1 ("gate", through SiLU), [F,2F) = w3 ("up")
 *     down    [E, D, F]   row-major
 *
 * Conventions for every entry point:
 *   - bf16 tensors are passed as moe_bf16_t (the raw bf16 bit pattern), row-major, contiguous.
 *   - All tensor pointers are DEVICE pointers owned by the caller, except the two host
 *     buffers of moe_layer_forward_host.  The library never allocates, frees or keeps them.
 *   - Tensor pointers must be 16-byte aligned; workspaces 256-byte aligned.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  No entry point synchronises except moe_get_device_error.
 *   - Arguments are validated on the host before anything is launched; on an error status
 *     nothing has been enqueued.  A failed launch returns MOE_ERR_CUDA.
 *   - Errors found by kernels (an expert id outside [0,E) reaching moe_permute, a device-side
 *     wait that gave up) are OR-ed into a sticky error word in the first 256 bytes of the
 *     workspace; read it with moe_get_device_error.
 *   - Shapes: D, F, Fs multiples of 64; 1 <= E <= 1024; 1 <= k <= min(E, 32); T >= 0 (T = 0 is a
 *     no-op); T*k < 2^31.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t moe_bf16_t; /* bf16 bit pattern */
typedef void* moe_stream_t;  /* cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,         /* null pointer, k > E, negative size, ...          */
  MOE_ERR_UNSUPPORTED_SHAPE = 2,   /* D/F/Fs not a multiple of 64, E > 1024, k > 32     */
  MOE_ERR_ALIGNMENT = 3,           /* a pointer is not 16-byte (workspace: 256-byte) aligned */
  MOE_ERR_WORKSPACE_TOO_SMALL = 4, /* ws_bytes below the matching *_workspace_size()     */
  MOE_ERR_CUDA = 5,                /* a CUDA runtime call or kernel launch failed         */
  MOE_ERR_DEVICE_INDEX = 6,        /* (device) an expert id outside [0, E) was seen       */
  MOE_ERR_TIMEOUT = 7,             /* (device) a bounded wait inside a kernel gave up     */
  MOE_ERR_NO_DEVICE = 8            /* no current CUDA device of compute capability 10.x   */
} moe_status_t;

/* ----------------------------------------------------------------------------------------
 * Step 1: router projection + top-k + renormalised softmax.
 * josueisai.com "Mixture of experts", section "El router"; gotburnout.io glossary, section 2
 * (p = Softmax(TopK(W_g x))) and section 2 item 4 (aux-loss-free balancing bias).
 *
 *   x        [T, D]  bf16      w_gate [E, D] bf16      bias [E] fp32 or NULL
 *   topk_idx [T, k]  int32     out: expert ids, by (logit + bias) descending, ties -> lower id
 *   topk_w   [T, k]  fp32      out: exp(l_j - m) / sum_i exp(l_i - m) over the chosen k, with
 *                              the UNBIASED logits l (the bias only steers the selection)
 * The logits are bf16 x bf16 products accumulated in fp32 on the tensor cores (split over K in
 * a fixed number of partial sums that the top-k kernel adds in a fixed order).
 *   ws: >= moe_router_topk_workspace_size(T, D, E) bytes of device memory (first 256 bytes:
 *       the device error word; the rest holds the partial logits).
 * ---------------------------------------------------------------------------------------- */
size_t moe_router_topk_workspace_size(int T, int D, int E);
moe_status_t moe_router_topk(const moe_bf16_t* x, const moe_bf16_t* w_gate, const float* bias, int T,
                             int D, int E, int k, int32_t* topk_idx, float* topk_w, void* ws,
                             size_t ws_bytes, moe_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * Router load-balancing auxiliary loss (training).  josueisai.com "Mixture of experts", section
 * "El coste que la cifra bonita esconde": MoE training adds a loss that penalises the router for
 * spreading tokens unevenly (dev.smart-guide.co.kr, "Limitaciones y Cuidados": without it the
 * router collapses onto few experts).  The pages print no formula; the one computed here is the
 * product of each expert's load and mean router probability:
 *   L = alpha * E * sum_e f_e * P_e,
 *   f_e = (slots of the top-k of l + bias that chose e) / (T * k)      -- a count, no gradient,
 *   P_e = mean over tokens of softmax(l_t)_e over all E unbiased logits,
 * so L = alpha when both are uniform.  Outputs (device, fp32, overwritten):
 *   loss    [1]      L
 *   dw_gate [E, D]   dL/dW_g      (add it to the layer backward's dw_gate)
 *   dx      [T, D]   dL/dx        (add it to the layer backward's dx)
 * Logits are computed as in moe_router_topk; every sum runs in a fixed order (deterministic).
 * T = 0 writes loss = 0 and zeros dw_gate.  x, w_gate 16-byte aligned; bias, loss, dw_gate, dx
 * 4-byte aligned.
 *   ws: >= moe_router_aux_loss_workspace_size(T, D, E, k) bytes of device memory.
 * ---------------------------------------------------------------------------------------- */
size_t moe_router_aux_loss_workspace_size(int T, int D, int E, int k);
moe_status_t moe_router_aux_loss(const moe_bf16_t* x, const moe_bf16_t* w_gate, const float* bias, int T,
                                 int D, int E, int k, float alpha, float* loss, float* dw_gate, float* dx,
                                 void* ws, size_t ws_bytes, moe_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * Step 2: dispatch -- histogram, exclusive prefix sum and permutation into expert-contiguous
 * order (keryc.com "Mixture of Experts optimiza Transformers y LLMs", section "Ejecucion
 * eficiente: backends de expertos": the grouped backend sorts tokens by expert id).
 * Order: experts ascending, tokens ascending within an expert (a stable counting sort of the
 * T*k slots by expert id).  M = T*k rows.
 *
 *   topk_idx [T, k] int32, topk_w [T, k] fp32, x [T, D] bf16 (NULL: metadata only)
 *   counts   [E]    int32  out: slots routed to each expert
 *   offsets  [E+1]  int32  out: offsets[0] = 0, offsets[e+1] = offsets[e] + counts[e]
 *   perm_token [M]  int32  out: token of row r
 *   inv_perm [T*k]  int32  out: row of slot t*k + j
 *   p_perm   [M]    fp32   out: topk_w of row r
 *   x_perm   [M, D] bf16   out (if x != NULL): x_perm[r] = x[perm_token[r]]
 *   ws: >= moe_permute_workspace_size(T, E, k) bytes of device memory (contents need not be
 *       initialised); its first 256 bytes are the device error word.
 * An id outside [0, E) sets MOE_ERR_DEVICE_INDEX in the error word; that slot is dropped.
 * ---------------------------------------------------------------------------------------- */
size_t moe_permute_workspace_size(int T, int E, int k);
moe_status_t moe_permute(const int32_t* topk_idx, const float* topk_w, const moe_bf16_t* x, int T,
                         int D, int E, int k, int32_t* counts, int32_t* offsets, int32_t* perm_token,
                         int32_t* inv_perm, float* p_perm, moe_bf16_t* x_perm, void* ws,
                         size_t ws_bytes, moe_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * moe_permute without a workspace.  The pages have no counterpart to this entry point: it
 * exists for callers that cannot allocate device memory -- their GPU memory is owned by
 * someone else (an inference engine that reserves the device's memory for its own pools up
 * front, a plugin whose host program does not share its allocator) -- and so cannot hand
 * moe_permute a workspace.  It allocates nothing.
 *
 * Arguments, results and row order are those of moe_permute, without ws / ws_bytes.  The
 * scratch (per-block expert counts) is a fixed 512 KiB array inside the library, held by every
 * GPU that loads the library until the process exits; it fits ceil(T/256) * E <= 131072
 * (e.g. T <= 32768 with E = 1024).  Larger sizes return MOE_ERR_WORKSPACE_TOO_SMALL and
 * launch nothing.
 * The array has one copy per CUDA context: each call looks up its address in the calling
 * thread's current context (cudaGetSymbolAddress, a host-side lookup), so a caller that works
 * in its own driver-API context, or after cudaDeviceReset, gets that context's copy.  The first
 * call in a context loads the library's device code into it; make that first call before any
 * stream capture.
 * All calls share the one array: calls whose kernels overlap on the GPU (e.g. on two streams
 * with no ordering between them) race and give wrong results.  Each call writes every scratch
 * entry it reads, so contents left by an earlier call do no harm.
 * Out-of-range expert ids are dropped as in moe_permute (inv_perm entry -1) but, with no
 * workspace, there is no error word that reports them.
 * ---------------------------------------------------------------------------------------- */
moe_status_t moe_permute_noalloc(const int32_t* topk_idx, const float* topk_w, const moe_bf16_t* x,
                                 int T, int D, int E, int k, int32_t* counts, int32_t* offsets,
                                 int32_t* perm_token, int32_t* inv_perm, float* p_perm,
                                 moe_bf16_t* x_perm, moe_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * Step 3: the routed experts as grouped GEMMs over expert-contiguous rows (tcgen05 / TMEM /
 * TMA).  gotburnout.io glossary, section 3 step 3 (the SwiGLU expert) and step 4 (outputs
 * multiplied by the router weights).
 *
 *   x_perm   [M, D] bf16       rows of segment e are [offsets[e], offsets[e+1])
 *   offsets  [E+1]  int32      device; offsets[E] <= M
 *   row_scale [M]   fp32 or NULL (1.0): multiplies output row r (pass p_perm)
 *   max_seg:  an upper bound on any segment length (pass M if unknown).  max_seg <= 64
 *             selects the weight-streaming (decode) kernels, otherwise the tiled kernels.
 *   flags:    0 for the layer's default prefill tiling, or one of MOE_FLAG_PREFILL_ROW_TILES /
 *             _WIDE_TILES / _PAIR_TILES (defined with moe_layer_desc_t below); ignored when the
 *             streaming kernels run.  Any other bit is MOE_ERR_INVALID_ARG.
 *   gate_up  [E, 2F, D] bf16, down [E, D, F] bf16
 *   out_perm [M, D] fp32 out:   out_perm[r] = row_scale[r] * Expert_e(x_perm[r])
 *            (kept in fp32 so that y is rounded to bf16 once, in the combine)
 *   ws: >= moe_grouped_swiglu_ffn_workspace_size(M, F) bytes (holds h = silu(G x) * (U x),
 *       [M, F] bf16); first 256 bytes: the device error word.
 * ---------------------------------------------------------------------------------------- */
size_t moe_grouped_swiglu_ffn_workspace_size(int M, int F);
moe_status_t moe_grouped_swiglu_ffn(const moe_bf16_t* x_perm, const int32_t* offsets,
                                    const float* row_scale, int M, int max_seg, int flags, int E, int D, int F,
                                    const moe_bf16_t* gate_up, const moe_bf16_t* down,
                                    float* out_perm, void* ws, size_t ws_bytes, moe_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * Step 4: weighted combine back to token order (gotburnout.io glossary, section 2 "Weighted
 * Aggregation", section 3 step 4).  out_perm rows are already scaled by their router weight.
 *
 *   y[t] = bf16( sum_{j=0..k-1} out_perm[inv_perm[t*k + j]] + shared_out[t] )  (fp32 sum, j order)
 *   out_perm [T*k, D] fp32, inv_perm [T*k] int32 (entries < 0 are skipped), shared_out [T, D]
 *   fp32 or NULL, y [T, D] bf16
 * ---------------------------------------------------------------------------------------- */
moe_status_t moe_combine(const float* out_perm, const int32_t* inv_perm, const float* shared_out,
                         int T, int D, int k, moe_bf16_t* y, moe_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * The whole layer (steps 1-4, plus the always-on shared expert of gotburnout.io glossary,
 * section 2 item 3 "Shared Experts", added with weight 1).
 * T <= 64 runs the weight-streaming (decode) kernels, larger T the tiled (prefill) kernels;
 * `flags` can force either for testing.
 * ---------------------------------------------------------------------------------------- */
#define MOE_FLAG_FORCE_PREFILL 1
#define MOE_FLAG_FORCE_DECODE 2 /* only valid for T <= 64 */
/* Training forward: keep in the workspace what moe_layer_backward needs (the routing, x_perm, h
 * and the SwiGLU inputs g | u of the gate_up GEMMs, bf16).  Uses the tiled kernels at any T;
 * bf16 weights only. */
#define MOE_FLAG_SAVE_FOR_BACKWARD 4
/* Prefill tiling of the expert GEMMs (at most one of the three; none with FORCE_DECODE):
 *  ROW_TILES  both GEMMs on 128 permuted rows x 256 output columns per tile (tokens are the
 *             MMA's M);
 *  WIDE_TILES both on 128 weight rows x up to 256 rows of one expert segment (tokens are N, so a
 *             segment's last tile is padded to a multiple of 16 rows instead of 128);
 *  PAIR_TILES both on the WIDE orientation computed by a cluster of two CTAs: 256 weight rows x
 *             up to 256 tokens per tcgen05.mma.cta_group::2, each CTA loading its own half of both
 *             operands (no multicast).
 * Without any, gate_up runs ROW_TILES and down PAIR_TILES (the measured best per GEMM).  All
 * give the same routing; outputs agree within fp32 rounding order. */
#define MOE_FLAG_PREFILL_ROW_TILES 8
#define MOE_FLAG_PREFILL_WIDE_TILES 16
#define MOE_FLAG_PREFILL_PAIR_TILES 32

#define MOE_WEIGHTS_BF16 0     /* gate_up / down (and shared_*) hold bf16 weights            */
#define MOE_WEIGHTS_FP8_E4M3 1 /* *_fp8 hold E4M3 codes with one fp32 scale per weight row  */

typedef struct {
  int32_t T, D, E, k, F, Fs;       /* Fs = 0: no shared expert                              */
  const moe_bf16_t* w_gate;        /* [E, D]                                                */
  const float* bias;               /* [E] selection bias or NULL                            */
  const moe_bf16_t* gate_up;       /* [E, 2F, D]                                            */
  const moe_bf16_t* down;          /* [E, D, F]                                             */
  const moe_bf16_t* shared_gate_up;/* [2Fs, D] or NULL                                      */
  const moe_bf16_t* shared_down;   /* [D, Fs] or NULL                                       */
  int32_t flags;                   /* 0 or MOE_FLAG_*                                       */
  /* Expert weights as E4M3 codes (the pages' per-expert quantisation, keryc.com "Mixture of
   * Experts optimiza...", section "Resultados practicos"; codes from moe_quantize_rows_fp8):
   * used when weight_format == MOE_WEIGHTS_FP8_E4M3, where the bf16 gate_up / down / shared_*
   * pointers are ignored.  Row r of a tensor dequantises to code * scale[r].  Decode only
   * (T <= 64; larger T returns MOE_ERR_UNSUPPORTED_SHAPE).  Activations (x and h) run in f16:
   * x converts exactly for 2^-14 <= |x| <= 65504 (smaller values lose low bits, larger ones
   * overflow).  Code pointers must be 16-byte aligned, scales 4-byte aligned.  Steps with fewer
   * 128-row units than SMs split K; the partial sums are added in a fixed order, so results are
   * deterministic. */
  int32_t weight_format;                /* MOE_WEIGHTS_BF16 or MOE_WEIGHTS_FP8_E4M3          */
  const uint8_t* gate_up_fp8;           /* [E, 2F, D] codes                                  */
  const float* gate_up_scale;           /* [E, 2F]                                           */
  const uint8_t* down_fp8;              /* [E, D, F] codes                                   */
  const float* down_scale;              /* [E, D]                                            */
  const uint8_t* shared_gate_up_fp8;    /* [2Fs, D] codes or NULL                            */
  const float* shared_gate_up_scale;    /* [2Fs] or NULL                                     */
  const uint8_t* shared_down_fp8;       /* [D, Fs] codes or NULL                             */
  const float* shared_down_scale;       /* [D] or NULL                                       */
} moe_layer_desc_t;

/* Per-row E4M3 quantisation of a packed bf16 weight tensor w [rows, K] (device; K a multiple of
 * 64): scales[r] = amax(|w[r]|) / 448 (1 for an all-zero row) and q[r][k] = E4M3(w[r][k] /
 * scales[r]), round to nearest even, saturating at +-448.  q [rows, K] uint8, scales [rows] fp32
 * (device).  Asynchronous on `stream`. */
moe_status_t moe_quantize_rows_fp8(const moe_bf16_t* w, int64_t rows, int K, uint8_t* q, float* scales,
                                   moe_stream_t stream);

/* Device workspace bytes for moe_layer_forward / moe_layer_forward_host (0 if desc invalid). */
size_t moe_layer_workspace_size(const moe_layer_desc_t* desc);

/* x [T, D] bf16 (device) -> y [T, D] bf16 (device).  Clears the workspace's error word (and the
 * split-K counters that follow it) first, with one memset on `stream`.
 * Prefill (T > 64, bf16 weights) with a shared expert runs the shared expert's two GEMMs on a side
 * stream owned by the library -- one per (device, caller stream), with two events, created on the
 * first such call and kept until the process exits -- forked from `stream` after the router GEMM
 * and joined back before the combine.  All work still completes in `stream` order; under stream
 * capture the graph gets two parallel branches.  Make the first such call on each stream before
 * capturing it. */
moe_status_t moe_layer_forward(const moe_layer_desc_t* desc, const moe_bf16_t* x, moe_bf16_t* y,
                               void* ws, size_t ws_bytes, moe_stream_t stream);

/* Same with HOST buffers (pinned memory for asynchronous copies): copies x_host into the
 * workspace, runs the layer, copies y back to y_host, all on `stream`.  The caller
 * synchronises the stream before reading y_host. */
moe_status_t moe_layer_forward_host(const moe_layer_desc_t* desc, const moe_bf16_t* x_host,
                                    moe_bf16_t* y_host, void* ws, size_t ws_bytes,
                                    moe_stream_t stream);

/* moe_layer_forward that also records events[0..n_events) (cudaEvent_t handles created by the
 * caller) on `stream` around its stages: events[0] before the router, then one event after
 * each of: router, dispatch, gate_up GEMM (+SwiGLU), down GEMM, combine (6 events in all;
 * n_events must be >= 6).  Used to time each stage on the launching stream. */
moe_status_t moe_layer_forward_timed(const moe_layer_desc_t* desc, const moe_bf16_t* x,
                                     moe_bf16_t* y, void* ws, size_t ws_bytes, moe_stream_t stream,
                                     void* const* events, int n_events);

/* Number of kernels one moe_layer_forward launches for this descriptor (0 if invalid). */
int moe_layer_kernel_count(const moe_layer_desc_t* desc);

/* Which expert-GEMM kernels moe_layer_forward runs for this descriptor (host-only query; -1 if
 * the descriptor is invalid): the weight-streaming decode kernels (bf16 or E4M3 weights), or the
 * prefill tilings of MOE_FLAG_PREFILL_ROW_TILES / _WIDE_TILES / _PAIR_TILES. */
#define MOE_PATH_STREAMING 0
#define MOE_PATH_FP8_STREAMING 1
#define MOE_PATH_ROW_TILES 2
#define MOE_PATH_WIDE_TILES 3
#define MOE_PATH_MIXED_TILES 4 /* gate_up on 128-row tiles, down on token-wide tiles of CTA pairs */
#define MOE_PATH_PAIR_TILES 5  /* both on token-wide tiles of CTA pairs */
int moe_layer_gemm_path(const moe_layer_desc_t* desc);

/* ----------------------------------------------------------------------------------------
 * Backward pass (training; keryc.com "Mixture of Experts optimiza...", section "Entrenamiento:
 * todavia desafiante, pero con avances", dev.smart-guide.co.kr, section "Entrenamiento MoE: 12x
 * Mas Rapido").  The pages give no formulas: the gradients are the chain rule of the forward, with
 * L = sum(dy * y), no gradient through the top-k selection or the selection bias:
 *   dx [T, D] bf16; dw_gate [E, D], dgate_up [E, 2F, D], ddown [E, D, F], dshared_gate_up [2Fs, D],
 *   dshared_down [D, Fs] fp32 (overwritten, not accumulated; experts no token chose get zeros).
 * Inputs: the descriptor of a forward run with MOE_FLAG_SAVE_FOR_BACKWARD on the same x, and that
 * forward's workspace (fwd_ws, read only; the saved state), dy [T, D] bf16.  bwd_ws:
 * >= moe_layer_backward_workspace_size(desc) bytes, 256-byte aligned, its first 256 bytes the
 * device error word (moe_get_device_error).  Device pointers; asynchronous on `stream`.
 * ---------------------------------------------------------------------------------------- */
typedef struct {
  float* dw_gate;          /* [E, D]                  */
  float* dgate_up;         /* [E, 2F, D]              */
  float* ddown;            /* [E, D, F]               */
  float* dshared_gate_up;  /* [2Fs, D] or NULL (Fs=0) */
  float* dshared_down;     /* [D, Fs] or NULL (Fs=0)  */
} moe_layer_grads_t;

size_t moe_layer_backward_workspace_size(const moe_layer_desc_t* desc);
moe_status_t moe_layer_backward(const moe_layer_desc_t* desc, const moe_bf16_t* x, const moe_bf16_t* dy,
                                moe_bf16_t* dx, const moe_layer_grads_t* grads, const void* fwd_ws,
                                size_t fwd_ws_bytes, void* bwd_ws, size_t bwd_ws_bytes, moe_stream_t stream);

/* ----------------------------------------------------------------------------------------
 * Aux-loss-free balancing (gotburnout.io glossary "MoE", section 2 item 4: router biases are
 * adjusted dynamically so that no expert is overloaded).  The pages give no update rule; this
 * library applies the sign rule on the loads of the last batch:
 *     bias[e] += gamma * sign(mean(counts) - counts[e])        (fp32 add, round to nearest)
 * with the comparison done exactly in integers.  counts [E] int32 (device; e.g. from
 * moe_permute or moe_layer_expert_counts), bias [E] fp32 (device, updated in place),
 * 1 <= E <= 1024, gamma >= 0.  One kernel; asynchronous on `stream`.
 * ---------------------------------------------------------------------------------------- */
moe_status_t moe_update_router_bias(const int32_t* counts, int E, float gamma, float* bias,
                                    moe_stream_t stream);

/* Device address of the per-expert loads counts[E] (int32) that moe_layer_forward leaves in
 * its workspace (valid once the forward has run on the stream, until the next forward).  Host
 * call only: nothing is launched. */
moe_status_t moe_layer_expert_counts(const moe_layer_desc_t* desc, void* ws, size_t ws_bytes,
                                     const int32_t** counts);

/* Synchronises `stream`, returns the status held in the workspace's error word (MOE_OK,
 * MOE_ERR_DEVICE_INDEX or MOE_ERR_TIMEOUT) and clears it.  MOE_ERR_TIMEOUT: a pipeline wait
 * inside a GEMM kernel gave up after 1 s of wall-clock time (the GPU's global timer); the kernel
 * then drained its own copies, freed its tensor memory and returned, and that launch's outputs
 * are invalid.  A context kept off the GPU for longer than that (time slicing, preemption) can
 * report it spuriously. */
moe_status_t moe_get_device_error(void* ws, moe_stream_t stream);

/* Static, human-readable name of a status. */
const char* moe_status_string(moe_status_t status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
