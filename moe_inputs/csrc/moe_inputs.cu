// moe_inputs.cu -- host and device fill routines for the seeded input generator.
//
// Both sides evaluate the same functions from moe_inputs.h element by element,
// so a tensor filled on the device equals the one filled on the host bit for
// bit.  Host fills may use several threads; the result does not depend on the
// thread count because each element is a pure function of its index.

#include <cuda_runtime.h>
#include <stdint.h>
#include <thread>
#include <vector>

#include "moe_inputs.h"

namespace {

template <class F>
void parallel_for(int64_t n, int nthreads, F f) {
  if (nthreads <= 1 || n < (1 << 16)) {
    f(int64_t(0), n);
    return;
  }
  std::vector<std::thread> pool;
  int64_t chunk = (n + nthreads - 1) / nthreads;
  for (int t = 0; t < nthreads; ++t) {
    int64_t lo = t * chunk, hi = lo + chunk < n ? lo + chunk : n;
    if (lo >= hi) break;
    pool.emplace_back([=] { f(lo, hi); });
  }
  for (auto& th : pool) th.join();
}

__global__ void fill_normal_bf16_kernel(uint16_t* __restrict__ out, uint64_t n, uint64_t key,
                                        uint64_t first, float sigma) {
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = mi_normal_bf16(key, first + i, sigma);
}

__global__ void fill_rows_bf16_kernel(uint16_t* __restrict__ out, int64_t rows, int64_t cols,
                                      const uint32_t* __restrict__ redraw, uint64_t seed,
                                      uint32_t stream, float sigma) {
  // one block-row per grid-y step; columns across threads
  for (int64_t r = blockIdx.y; r < rows; r += gridDim.y) {
    uint64_t key = mi_stream_key(seed, stream, redraw ? redraw[r] : 0u);
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < cols;
         c += (int64_t)gridDim.x * blockDim.x)
      out[r * cols + c] = mi_normal_bf16(key, (uint64_t)(r * cols + c), sigma);
  }
}

}  // namespace

extern "C" {

// Elements [first, first + n) of stream (seed, stream, redraw), N(0, sigma^2), as bf16 bits.
void mi_fill_normal_bf16_host(uint16_t* out, uint64_t n, uint64_t seed, uint32_t stream,
                              uint32_t redraw, uint64_t first, float sigma, int nthreads) {
  uint64_t key = mi_stream_key(seed, stream, redraw);
  parallel_for((int64_t)n, nthreads, [=](int64_t lo, int64_t hi) {
    for (int64_t i = lo; i < hi; ++i) out[i] = mi_normal_bf16(key, first + (uint64_t)i, sigma);
  });
}

// Same draw kept in fp32 (used for the per-expert selection bias).
void mi_fill_normal_f32_host(float* out, uint64_t n, uint64_t seed, uint32_t stream,
                             uint32_t redraw, uint64_t first, float sigma) {
  uint64_t key = mi_stream_key(seed, stream, redraw);
  for (uint64_t i = 0; i < n; ++i) out[i] = mi_scale(mi_normal(key, first + i), sigma);
}

// Rows row_ids[i] (i < nrows) of a [*, cols] tensor whose row r is drawn from substream
// redraw[i] (NULL: 0).  Element (r, c) is variate r*cols + c of that substream.
void mi_fill_rows_bf16_host(uint16_t* out, int64_t nrows, int64_t cols, const int64_t* row_ids,
                            const uint32_t* redraw, uint64_t seed, uint32_t stream, float sigma,
                            int nthreads) {
  parallel_for(nrows, nthreads > 1 && nrows >= nthreads ? nthreads : 1, [=](int64_t lo, int64_t hi) {
    for (int64_t i = lo; i < hi; ++i) {
      int64_t r = row_ids ? row_ids[i] : i;
      uint64_t key = mi_stream_key(seed, stream, redraw ? redraw[i] : 0u);
      for (int64_t c = 0; c < cols; ++c)
        out[i * cols + c] = mi_normal_bf16(key, (uint64_t)(r * cols + c), sigma);
    }
  });
}

// The raw SplitMix64 output function (exported so tests can pin it to published values).
uint64_t mi_mix64_host(uint64_t z) { return mi_mix64(z); }

// The float variate before scaling (exported for tests of the normal transform).
float mi_normal_host(uint64_t seed, uint32_t stream, uint32_t redraw, uint64_t i) {
  return mi_normal(mi_stream_key(seed, stream, redraw), i);
}

uint64_t mi_word_host(uint64_t seed, uint32_t stream, uint32_t redraw, uint64_t i) {
  return mi_word(mi_stream_key(seed, stream, redraw), i);
}

// Device fill of a contiguous bf16 tensor: elements [first, first + n) of the stream.
int mi_fill_normal_bf16_device(uint16_t* out, uint64_t n, uint64_t seed, uint32_t stream,
                               uint32_t redraw, uint64_t first, float sigma, void* cuda_stream) {
  if (n == 0) return 0;
  uint64_t key = mi_stream_key(seed, stream, redraw);
  uint64_t blocks = (n + 255) / 256;
  if (blocks > 148ull * 64ull) blocks = 148ull * 64ull;
  fill_normal_bf16_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)cuda_stream>>>(out, n, key,
                                                                                   first, sigma);
  return (int)cudaGetLastError();
}

// Device fill of all rows [0, rows) of a [rows, cols] tensor; redraw is a device array or NULL.
int mi_fill_rows_bf16_device(uint16_t* out, int64_t rows, int64_t cols, const uint32_t* redraw,
                             uint64_t seed, uint32_t stream, float sigma, void* cuda_stream) {
  if (rows == 0 || cols == 0) return 0;
  unsigned gx = (unsigned)((cols + 255) / 256);
  if (gx > 64) gx = 64;
  unsigned gy = rows < 65535 ? (unsigned)rows : 65535u;
  fill_rows_bf16_kernel<<<dim3(gx, gy), 256, 0, (cudaStream_t)cuda_stream>>>(out, rows, cols, redraw,
                                                                            seed, stream, sigma);
  return (int)cudaGetLastError();
}

}  // extern "C"
