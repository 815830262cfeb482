/*
 * Device side of the seeded input generator (see gen_core.h).  Writes the
 * same values as gen_host.c, bit for bit, straight into device buffers, so
 * that multi-GB inputs need no host copy.  Test and benchmark plumbing only:
 * it shares no code with the attention kernels.
 */
#include <cuda_runtime.h>
#include <stdint.h>

#include "gen_core.h"

__global__ void gen_fill_kernel(uint64_t state, uint64_t start, uint64_t count, int kind, double a,
                                double b, int as_bf16, void* out) {
  uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (; i < count; i += stride) {
    float v = gen_value_f32(kind, state, start + i, a, b);
    if (as_bf16)
      ((uint16_t*)out)[i] = gen_f32_to_bf16(v);
    else
      ((float*)out)[i] = v;
  }
}

/* Cache tensor [B, H, n_cap, d] of bf16: row r of head (b, h) holds counter
   values ((b*H + h)*n_cap + r)*d + c when r < lens[b], and a quiet NaN otherwise. */
__global__ void gen_fill_cache_kernel(uint64_t state, int64_t H, int64_t n_cap, int64_t d,
                                      const int* lens, int kind, double a, double b, uint64_t total,
                                      uint16_t* out) {
  uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (; i < total; i += stride) {
    uint64_t row = i / (uint64_t)d;
    uint64_t r = row % (uint64_t)n_cap;
    uint64_t bh = row / (uint64_t)n_cap;
    uint64_t bb = bh / (uint64_t)H;
    if ((int64_t)r < (int64_t)lens[bb])
      out[i] = gen_f32_to_bf16(gen_value_f32(kind, state, i, a, b));
    else
      out[i] = 0x7FC0u;
  }
}

static int gen_grid(uint64_t n) {
  uint64_t blocks = (n + 255) / 256;
  if (blocks > 148ull * 64ull) blocks = 148ull * 64ull;
  if (blocks < 1) blocks = 1;
  return (int)blocks;
}

extern "C" int gen_cuda_fill(uint64_t seed, uint64_t stream, uint64_t start, uint64_t count, int kind,
                             double a, double b, int as_bf16, void* dev_out, void* cuda_stream) {
  if (count == 0) return 0;
  if (!dev_out || (kind != GEN_NORMAL && kind != GEN_UNIFORM)) return -1;
  gen_fill_kernel<<<gen_grid(count), 256, 0, (cudaStream_t)cuda_stream>>>(
      gen_stream_state(seed, stream), start, count, kind, a, b, as_bf16, dev_out);
  return cudaGetLastError() == cudaSuccess ? 0 : -2;
}

extern "C" int gen_cuda_fill_cache(uint64_t seed, uint64_t stream, int64_t B, int64_t H, int64_t n_cap,
                                   int64_t d, const int* dev_lens, int kind, double a, double b,
                                   void* dev_out, void* cuda_stream) {
  if (B <= 0 || H <= 0 || n_cap <= 0 || d <= 0) return 0;
  if (!dev_out || !dev_lens || (kind != GEN_NORMAL && kind != GEN_UNIFORM)) return -1;
  uint64_t total = (uint64_t)B * (uint64_t)H * (uint64_t)n_cap * (uint64_t)d;
  gen_fill_cache_kernel<<<gen_grid(total), 256, 0, (cudaStream_t)cuda_stream>>>(
      gen_stream_state(seed, stream), H, n_cap, d, dev_lens, kind, a, b, total, (uint16_t*)dev_out);
  return cudaGetLastError() == cudaSuccess ? 0 : -2;
}
