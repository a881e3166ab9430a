// permute_noalloc.cu -- moe_permute_noalloc: the dispatch step for callers that cannot allocate
// device memory (their GPU memory belongs to someone else, e.g. an inference engine that
// reserves the device's memory for its own pools up front, or a plugin whose host program does
// not share its allocator), so they cannot provide moe_permute's workspace either.
//
// The only scratch the dispatch kernels need -- the per-block expert counts -- lives here in a
// fixed file-scope device array instead of a caller workspace.  The kernels and their launcher
// are the ones moe_permute uses; only where the scratch lives differs.
#include "moe_common.cuh"

namespace {

constexpr size_t kScratchBytes = 512 * 1024;                        // held by every GPU that loads the library
constexpr long long kScratchInts = (long long)(kScratchBytes / 4);  // room for ceil(T/256) * E counts
constexpr int kTokPerBlock = 256;                                    // tokens per counting block (permute.cu)

// The array's name is only a host-side stand-in in host code; its device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_permute_scratch[kScratchBytes];

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Device address of the scratch array in the calling thread's current context.  A __device__
// array's address belongs to a CUDA context, not to a device ordinal: after cudaDeviceReset, or
// when the caller runs in its own driver-API context on the same device, the array lives at
// another address.  So the address is looked up on every call -- a host-side lookup in the
// module's symbol table, with no allocation and no stream operation.  The first call in a
// context loads the library's module into it (lazy loading), which is why that first call
// should come before any stream capture.
moe_status_t scratch_for_current_context(int32_t** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10) {
    cudaGetLastError();
    return MOE_ERR_NO_DEVICE;
  }
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  *out = static_cast<int32_t*>(p);
  return MOE_OK;
}

}  // namespace

extern "C" moe_status_t moe_permute_noalloc(const int32_t* topk_idx, const float* topk_w, const moe_bf16_t* x, int T,
                                            int D, int E, int k, int32_t* counts, int32_t* offsets,
                                            int32_t* perm_token, int32_t* inv_perm, float* p_perm,
                                            moe_bf16_t* x_perm, moe_stream_t stream) {
  if (T < 0 || D <= 0 || E <= 0 || k <= 0 || k > E) return MOE_ERR_INVALID_ARG;
  if (D % 64 != 0 || E > 1024 || k > 32 || (long long)T * k >= (1LL << 31)) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!topk_idx || !topk_w || !counts || !offsets || !perm_token || !inv_perm || !p_perm) return MOE_ERR_INVALID_ARG;
  if ((x == nullptr) != (x_perm == nullptr)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(x_perm, 16) || !aligned(topk_idx, 4) || !aligned(topk_w, 4) ||
      !aligned(counts, 4) || !aligned(offsets, 4) || !aligned(perm_token, 4) || !aligned(inv_perm, 4) ||
      !aligned(p_perm, 4))
    return MOE_ERR_ALIGNMENT;
  const long long blocks = ((long long)T + kTokPerBlock - 1) / kTokPerBlock;
  if (blocks * E > kScratchInts) return MOE_ERR_WORKSPACE_TOO_SMALL;  // beyond the fixed scratch
  int32_t* scratch = nullptr;
  moe_status_t st = scratch_for_current_context(&scratch);
  if (st != MOE_OK) return st;
  // Every entry the kernels read is written earlier in the same call, so the previous call's
  // contents need no clearing.  No error word: out-of-range ids are dropped but not reported.
  if (moe::launch_permute(topk_idx, topk_w, x, T, D, E, k, counts, offsets, perm_token, inv_perm, p_perm, x_perm,
                          false, nullptr, scratch, nullptr, (cudaStream_t)stream, nullptr) != cudaSuccess) {
    cudaGetLastError();
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
