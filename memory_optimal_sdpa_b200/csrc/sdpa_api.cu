// sdpa_api.cu -- the C ABI (include/sdpa.h): argument checks, TMA tensor-map
// encoding and kernel launches.  One translation unit holds every kernel so the
// device error word is a single symbol without relocatable device code.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cfloat>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "sdpa.h"
#include "prefill_bf16.cuh"
#include "prefill_f32.cuh"
#include "decode.cuh"
#include "decode_gqa.cuh"
#include "backward.cuh"
#include "backward_d64.cuh"

namespace {

// SDPA_DEBUG=1 in the environment: report the failing CUDA call on stderr.
bool debug_on() {
  static const bool on = [] {
    const char* e = std::getenv("SDPA_DEBUG");
    return e && e[0] && e[0] != '0';
  }();
  return on;
}
int cuda_fail(const char* what, cudaError_t e) {
  if (debug_on()) std::fprintf(stderr, "sdpa: %s failed: %s\n", what, cudaGetErrorString(e));
  return SDPA_ERR_CUDA;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (e == cudaSuccess && q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else if (debug_on())
      std::fprintf(stderr, "sdpa: cuTensorMapEncodeTiled entry point not found (%s, query %d)\n",
                   cudaGetErrorString(e), (int)q);
  });
  return fn;
}

// [bh][n][d] bf16 tensor, 64-column x box_rows-row boxes, 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* map, const void* ptr, int d, int n, int bh, int box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n, (cuuint64_t)bh};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)n * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && debug_on())
    std::fprintf(stderr, "sdpa: cuTensorMapEncodeTiled failed (CUresult %d) d=%d n=%d bh=%d\n", (int)r, d, n, bh);
  return r == CUDA_SUCCESS;
}

// [bh][n][d] fp32 tensor, 32-column x 128-row boxes, 128-byte swizzle (the fused dQ accumulator).
bool make_map_f32(CUtensorMap* map, const float* ptr, int d, int n, int bh) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n, (cuuint64_t)bh};
  cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)n * d * 4};
  cuuint32_t box[3] = {32, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(ptr), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && debug_on())
    std::fprintf(stderr, "sdpa: cuTensorMapEncodeTiled (fp32) failed (CUresult %d) d=%d n=%d bh=%d\n", (int)r, d, n, bh);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

// Multiprocessors of the current device (the persistent prefill grid).
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      n <= 0)
    return 148;
  return n;
}
bool aligned4(const void* p) { return ((uintptr_t)p & 3u) == 0; }

// The current device must be an sm_100 part (B200 class).
int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SDPA_ERR_CUDA;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return SDPA_ERR_CUDA;
  if (major != 10 || minor != 0) return SDPA_ERR_UNSUPPORTED;
  return SDPA_OK;
}

template <int D, int MASK>
int launch_prefill(const void* Q, const void* K, const void* V, void* O, float* LSE, int bh, int n_q,
                   int n_kv, float scale, int win_left, int win_right, cudaStream_t stream) {
  using Cfg = sdpa::PrefillCfg<D>;
  auto kern = sdpa::sdpa_fwd_bf16_kernel<D, MASK>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(max dynamic smem)", attr_err);
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, Q, D, n_q, bh) || !make_map(&mk, K, D, n_kv, bh) || !make_map(&mv, V, D, n_kv, bh))
    return SDPA_ERR_CUDA;
  sdpa::PrefillParams p;
  p.O = (__nv_bfloat16*)O;
  p.LSE = LSE;
  p.n_q = n_q;
  p.n_kv = n_kv;
  p.bh_count = bh;
  p.n_pairs = (n_q + 255) / 256;
  // scale = 0 runs with the smallest normal float as the factor: every finite score s then gets
  // 2^(s * 2^-126 - m) = 1 exactly in fp32 (|s| < 2^100), the weights are uniform as the definition
  // says, and masked entries (-inf) still give 0, where a factor of exactly 0 would give -inf * 0 = NaN.
  p.scale_log2 = scale == 0.f ? FLT_MIN : std::fabs(scale) * 1.4426950408889634f;
  p.negate_s = scale < 0.f ? 1 : 0;
  p.win_left = win_left;
  p.win_right = win_right;
  // persistent: one CTA per SM (at most one per work unit), each striding over the units
  long long grid = (long long)bh * p.n_pairs;
  if (grid > sm_count()) grid = sm_count();
  p.heads_per_group = sdpa::prefill_heads_per_group(MASK, bh);
  kern<<<(unsigned)grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(mq, mk, mv, p);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess && debug_on()) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, kern) == cudaSuccess)
      std::fprintf(stderr,
                   "sdpa: prefill<%d,%d> regs %d maxThreads %d static smem %zu max dyn smem %d local %zu; "
                   "launch %lld x %d threads, %d B dynamic smem\n",
                   D, MASK, fa.numRegs, fa.maxThreadsPerBlock, fa.sharedSizeBytes,
                   fa.maxDynamicSharedSizeBytes, fa.localSizeBytes, grid, Cfg::THREADS, Cfg::SMEM_BYTES);
  }
  return e == cudaSuccess ? SDPA_OK : cuda_fail("prefill launch", e);
}

size_t decode_ws_bytes(long long batch, long long heads, long long n_cap, long long d_v) {
  const long long chunk = sdpa::decode_chunk(batch, heads, n_cap);
  const long long ns = (n_cap + chunk - 1) / chunk;
  return (size_t)(batch * heads * ns) * (size_t)(d_v + 1) * sizeof(float);
}

}  // namespace

extern "C" int sdpa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int batch,
                        int heads, int n_q, int n_kv, int d_k, int d_v, float scale, int causal,
                        void* stream) {
  if (batch < 0 || heads < 0 || n_q < 0 || n_kv < 1 || (causal != 0 && causal != 1) || !std::isfinite(scale))
    return SDPA_ERR_INVALID_ARG;
  if (d_k != d_v || (d_k != 64 && d_k != 128)) return SDPA_ERR_UNSUPPORTED;
  if (batch == 0 || heads == 0 || n_q == 0) return SDPA_OK;
  if (!Q || !K || !V || !O) return SDPA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || (LSE && !aligned4(LSE)))
    return SDPA_ERR_MISALIGNED;
  const long long bh = (long long)batch * heads;
  if (bh * (long long)(n_q > n_kv ? n_q : n_kv) >= (1LL << 31) || bh * ((n_q + 255) / 256) >= (1LL << 31))
    return SDPA_ERR_UNSUPPORTED;
  if (int e = check_device()) return e;
  cudaStream_t s = (cudaStream_t)stream;
  if (d_k == 64)
    return causal ? launch_prefill<64, 1>(Q, K, V, O, LSE, (int)bh, n_q, n_kv, scale, -1, 0, s)
                  : launch_prefill<64, 0>(Q, K, V, O, LSE, (int)bh, n_q, n_kv, scale, -1, -1, s);
  return causal ? launch_prefill<128, 1>(Q, K, V, O, LSE, (int)bh, n_q, n_kv, scale, -1, 0, s)
                : launch_prefill<128, 0>(Q, K, V, O, LSE, (int)bh, n_q, n_kv, scale, -1, -1, s);
}

extern "C" int sdpa_fwd_window(const void* Q, const void* K, const void* V, void* O, float* LSE, int batch,
                               int heads, int n_q, int n_kv, int d_k, int d_v, float scale, int window_left,
                               int window_right, void* stream) {
  if (batch < 0 || heads < 0 || n_q < 0 || n_kv < 1 || window_left < -1 || window_right < -1 || !std::isfinite(scale))
    return SDPA_ERR_INVALID_ARG;
  if (d_k != d_v || (d_k != 64 && d_k != 128)) return SDPA_ERR_UNSUPPORTED;
  if (batch == 0 || heads == 0 || n_q == 0) return SDPA_OK;
  if (!Q || !K || !V || !O) return SDPA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || (LSE && !aligned4(LSE)))
    return SDPA_ERR_MISALIGNED;
  const long long bh = (long long)batch * heads;
  if (bh * (long long)(n_q > n_kv ? n_q : n_kv) >= (1LL << 31) || bh * ((n_q + 255) / 256) >= (1LL << 31))
    return SDPA_ERR_UNSUPPORTED;
  if (int e = check_device()) return e;
  cudaStream_t s = (cudaStream_t)stream;
  // Open windows are the plain kernels; everything else takes the windowed instantiation.
  const int mode = window_left == -1 ? (window_right == -1 ? 0 : (window_right == 0 ? 1 : 2)) : 2;
  if (d_k == 64) {
    if (mode == 0) return launch_prefill<64, 0>(Q, K, V, O, LSE, (int)bh, n_q, n_kv, scale, -1, -1, s);
    if (mode == 1) return launch_prefill<64, 1>(Q, K, V, O, LSE, (int)bh, n_q, n_kv, scale, -1, 0, s);
    return launch_prefill<64, 2>(Q, K, V, O, LSE, (int)bh, n_q, n_kv, scale, window_left, window_right, s);
  }
  if (mode == 0) return launch_prefill<128, 0>(Q, K, V, O, LSE, (int)bh, n_q, n_kv, scale, -1, -1, s);
  if (mode == 1) return launch_prefill<128, 1>(Q, K, V, O, LSE, (int)bh, n_q, n_kv, scale, -1, 0, s);
  return launch_prefill<128, 2>(Q, K, V, O, LSE, (int)bh, n_q, n_kv, scale, window_left, window_right, s);
}

extern "C" int sdpa_fwd_f32(const float* Q, const float* K, const float* V, float* O, float* LSE, int batch,
                            int heads, int n_q, int n_kv, int d_k, int d_v, float scale, int causal,
                            void* stream) {
  if (batch < 0 || heads < 0 || n_q < 0 || n_kv < 1 || d_k < 1 || d_v < 1 || (causal != 0 && causal != 1) ||
      !std::isfinite(scale))
    return SDPA_ERR_INVALID_ARG;
  if (d_k > sdpa::F32_DMAX || d_v > sdpa::F32_DMAX) return SDPA_ERR_UNSUPPORTED;
  if (batch == 0 || heads == 0 || n_q == 0) return SDPA_OK;
  if (!Q || !K || !V || !O) return SDPA_ERR_INVALID_ARG;
  if (!aligned4(Q) || !aligned4(K) || !aligned4(V) || !aligned4(O) || (LSE && !aligned4(LSE)))
    return SDPA_ERR_MISALIGNED;
  const long long bh = (long long)batch * heads;
  if (bh > 65535 || bh * (long long)(n_q > n_kv ? n_q : n_kv) * 128 >= (1LL << 40)) return SDPA_ERR_UNSUPPORTED;
  if (int e = check_device()) return e;
  sdpa::F32Params p{Q, K, V, O, LSE, n_q, n_kv, d_k, d_v, scale, causal};
  dim3 grid((unsigned)((n_q + sdpa::F32_ROWS - 1) / sdpa::F32_ROWS), (unsigned)bh);
  sdpa::sdpa_fwd_f32_kernel<<<grid, 128, 0, (cudaStream_t)stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

extern "C" size_t sdpa_decode_workspace_size(int batch, int heads, int n_kv_cap, int d_v) {
  if (batch <= 0 || heads <= 0 || n_kv_cap <= 0 || d_v <= 0) return 0;
  return decode_ws_bytes(batch, heads, n_kv_cap, d_v);
}

extern "C" int sdpa_decode(const void* Q, const void* K, const void* V, const int* kv_lens, void* O,
                           float* LSE, int batch, int heads, int n_kv_cap, int d_k, int d_v, float scale,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (batch < 0 || heads < 0 || n_kv_cap < 1 || !std::isfinite(scale)) return SDPA_ERR_INVALID_ARG;
  if (d_k != d_v || (d_k != 64 && d_k != 128)) return SDPA_ERR_UNSUPPORTED;
  if (batch == 0 || heads == 0) return SDPA_OK;
  if (!Q || !K || !V || !kv_lens || !O) return SDPA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned4(kv_lens) ||
      (LSE && !aligned4(LSE)))
    return SDPA_ERR_MISALIGNED;
  if (batch > 65535 || heads > 65535) return SDPA_ERR_UNSUPPORTED;
  const size_t need = decode_ws_bytes(batch, heads, n_kv_cap, d_v);
  if (!workspace || workspace_bytes < need) return SDPA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SDPA_ERR_MISALIGNED;
  if (int e = check_device()) return e;
  sdpa::DecodeParams p;
  p.Q = (const __nv_bfloat16*)Q;
  p.K = (const __nv_bfloat16*)K;
  p.V = (const __nv_bfloat16*)V;
  p.kv_lens = kv_lens;
  p.H = heads;
  p.H_kv = heads;
  p.group = 1;
  p.n_cap = n_kv_cap;
  p.chunk = sdpa::decode_chunk(batch, heads, n_kv_cap);
  p.n_split = (n_kv_cap + p.chunk - 1) / p.chunk;
  p.part_o = (float*)workspace;
  p.part_lse = p.part_o + (size_t)batch * heads * p.n_split * d_v;
  p.O = (__nv_bfloat16*)O;
  p.LSE = LSE;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t s = (cudaStream_t)stream;
  dim3 grid((unsigned)p.n_split, (unsigned)heads, (unsigned)batch);
  if (d_k == 64) {
    sdpa::sdpa_decode_split_kernel<64><<<grid, sdpa::DECODE_THREADS, 0, s>>>(p);
    sdpa::sdpa_decode_combine_kernel<64><<<(unsigned)(batch * heads), 64, 0, s>>>(p);
  } else {
    sdpa::sdpa_decode_split_kernel<128><<<grid, sdpa::DECODE_THREADS, 0, s>>>(p);
    sdpa::sdpa_decode_combine_kernel<128><<<(unsigned)(batch * heads), 128, 0, s>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? SDPA_OK : SDPA_ERR_CUDA;
}

// ------------------------------------------------------------------ sdpa_decode_noalloc
// Scratch for callers that cannot allocate: one fixed array per device that loads
// this library.  Host code must never pass `g_decode_static_scratch` itself to a
// kernel (on the host it names a stand-in, not device memory); it passes the
// address cudaGetSymbolAddress returns for the current device.
namespace {
constexpr size_t kStaticScratchFloats = SDPA_DECODE_STATIC_SCRATCH_BYTES / sizeof(float);
__device__ __align__(256) float g_decode_static_scratch[kStaticScratchFloats];

constexpr int kMaxDevices = 64;
std::mutex g_static_scratch_mutex;
float* g_static_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device.  Looked up on the first call on
// each device, and again on every call whose stream is not capturing (so a device reset that
// reloads this module cannot leave a stale address); a capturing stream reuses the last one.
float* static_scratch_for_current_device(cudaStream_t stream, int* status) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    *status = cuda_fail("cudaGetDevice", e);
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    *status = SDPA_ERR_UNSUPPORTED;
    return nullptr;
  }
  cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &capture) != cudaSuccess) {
    (void)cudaGetLastError();  // e.g. the legacy stream while another stream captures: treat as capturing
    capture = cudaStreamCaptureStatusActive;
  }
  std::lock_guard<std::mutex> lock(g_static_scratch_mutex);
  if (!g_static_scratch_ptr[dev] || capture == cudaStreamCaptureStatusNone) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_static_scratch);
    if (e != cudaSuccess || !p) {
      *status = cuda_fail("cudaGetSymbolAddress(static decode scratch)", e);
      return nullptr;
    }
    g_static_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *status = SDPA_OK;
  return g_static_scratch_ptr[dev];
}
}  // namespace

extern "C" int sdpa_decode_noalloc(const void* Q, const void* K, const void* V, const int* kv_lens, void* O,
                                   float* LSE, int batch, int heads, int n_kv_cap, int d_k, int d_v, float scale,
                                   void* stream) {
  if (batch < 0 || heads < 0 || n_kv_cap < 1 || !std::isfinite(scale)) return SDPA_ERR_INVALID_ARG;
  if (d_k != d_v || (d_k != 64 && d_k != 128)) return SDPA_ERR_UNSUPPORTED;
  if (batch == 0 || heads == 0) return SDPA_OK;
  if (!Q || !K || !V || !kv_lens || !O) return SDPA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned4(kv_lens) ||
      (LSE && !aligned4(LSE)))
    return SDPA_ERR_MISALIGNED;
  if (batch > 65535 || heads > 65535) return SDPA_ERR_UNSUPPORTED;
  // Smallest split length (from the one sdpa_decode uses, doubling) whose partials fit the array.
  const long long bh = (long long)batch * heads;
  long long chunk = sdpa::decode_chunk(batch, heads, n_kv_cap);
  while (bh * ((n_kv_cap + chunk - 1) / chunk) * (d_v + 1) > (long long)kStaticScratchFloats) {
    if (chunk >= n_kv_cap) return SDPA_ERR_WORKSPACE;  // one split per (batch, head) is already too big
    chunk *= 2;
  }
  if (int e = check_device()) return e;
  int status = SDPA_OK;
  float* scratch = static_scratch_for_current_device((cudaStream_t)stream, &status);
  if (!scratch) return status;
  sdpa::DecodeParams p;
  p.Q = (const __nv_bfloat16*)Q;
  p.K = (const __nv_bfloat16*)K;
  p.V = (const __nv_bfloat16*)V;
  p.kv_lens = kv_lens;
  p.H = heads;
  p.H_kv = heads;
  p.group = 1;
  p.n_cap = n_kv_cap;
  p.chunk = (int)chunk;
  p.n_split = (int)((n_kv_cap + chunk - 1) / chunk);
  p.part_o = scratch;
  p.part_lse = scratch + (size_t)bh * p.n_split * d_v;
  p.O = (__nv_bfloat16*)O;
  p.LSE = LSE;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t s = (cudaStream_t)stream;
  dim3 grid((unsigned)p.n_split, (unsigned)heads, (unsigned)batch);
  if (d_k == 64) {
    sdpa::sdpa_decode_split_kernel<64><<<grid, sdpa::DECODE_THREADS, 0, s>>>(p);
    sdpa::sdpa_decode_combine_kernel<64><<<(unsigned)bh, 64, 0, s>>>(p);
  } else {
    sdpa::sdpa_decode_split_kernel<128><<<grid, sdpa::DECODE_THREADS, 0, s>>>(p);
    sdpa::sdpa_decode_combine_kernel<128><<<(unsigned)bh, 128, 0, s>>>(p);
  }
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SDPA_OK : cuda_fail("decode launch (static scratch)", e);
}

// ------------------------------------------------------------------ sdpa_decode_gqa
namespace {
// The tensor-core kernel takes d = 128 and groups of 2 .. 32 query heads; every other shape
// runs the CUDA-core split kernel with its group mapping.
bool gqa_tensor_path(int group, int d) { return d == 128 && group >= 2 && group <= 32; }

long long gqa_chunk_for(long long batch, long long heads_q, long long heads_kv, long long n_cap, int d) {
  return gqa_tensor_path((int)(heads_q / heads_kv), d) ? sdpa::gqa_chunk(batch, heads_kv, n_cap)
                                                        : sdpa::decode_chunk(batch, heads_q, n_cap);
}

size_t gqa_ws_bytes(long long batch, long long heads_q, long long heads_kv, long long n_cap, long long d_v) {
  const long long chunk = gqa_chunk_for(batch, heads_q, heads_kv, n_cap, (int)d_v);
  const long long n_split = (n_cap + chunk - 1) / chunk;
  return (size_t)(batch * heads_q * n_split * (d_v + 1)) * sizeof(float);
}

template <int NQ>
int launch_decode_gqa(const void* Q, const void* K, const void* V, const int* kv_lens, float* part_o,
                      float* part_lse, int batch, int heads_q, int heads_kv, int n_cap, int chunk, int n_split,
                      float scale, cudaStream_t stream) {
  using Cfg = sdpa::GqaCfg<NQ>;
  auto kern = sdpa::sdpa_decode_gqa_kernel<NQ>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(max dynamic smem, gqa)", attr_err);
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, Q, 128, batch * heads_q, 1, NQ) || !make_map(&mk, K, 128, n_cap, batch * heads_kv) ||
      !make_map(&mv, V, 128, n_cap, batch * heads_kv))
    return SDPA_ERR_CUDA;
  sdpa::GqaParams p;
  p.part_o = part_o;
  p.part_lse = part_lse;
  p.kv_lens = kv_lens;
  p.H_q = heads_q;
  p.H_kv = heads_kv;
  p.group = heads_q / heads_kv;
  p.n_cap = n_cap;
  p.chunk = chunk;
  p.n_split = n_split;
  p.scale_log2 = scale * 1.4426950408889634f;
  dim3 grid((unsigned)n_split, (unsigned)heads_kv, (unsigned)batch);
  kern<<<grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(mq, mk, mv, p);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SDPA_OK : cuda_fail("gqa decode launch", e);
}
}  // namespace

extern "C" size_t sdpa_decode_gqa_workspace_size(int batch, int heads_q, int heads_kv, int n_kv_cap, int d_v) {
  if (batch <= 0 || heads_q <= 0 || heads_kv <= 0 || heads_q % heads_kv != 0 || n_kv_cap <= 0 || d_v <= 0)
    return 0;
  return gqa_ws_bytes(batch, heads_q, heads_kv, n_kv_cap, d_v);
}

extern "C" int sdpa_decode_gqa(const void* Q, const void* K, const void* V, const int* kv_lens, void* O,
                               float* LSE, int batch, int heads_q, int heads_kv, int n_kv_cap, int d_k, int d_v,
                               float scale, void* workspace, size_t workspace_bytes, void* stream) {
  if (batch < 0 || heads_q < 0 || heads_kv < 1 || n_kv_cap < 1 || !std::isfinite(scale))
    return SDPA_ERR_INVALID_ARG;
  if (heads_q % heads_kv != 0) return SDPA_ERR_INVALID_ARG;
  if (d_k != d_v || (d_k != 64 && d_k != 128)) return SDPA_ERR_UNSUPPORTED;
  if (batch == 0 || heads_q == 0) return SDPA_OK;
  if (!Q || !K || !V || !kv_lens || !O) return SDPA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned4(kv_lens) ||
      (LSE && !aligned4(LSE)))
    return SDPA_ERR_MISALIGNED;
  if (batch > 65535 || heads_q > 65535) return SDPA_ERR_UNSUPPORTED;
  if ((long long)batch * heads_q >= (1LL << 31) || (long long)batch * heads_kv * n_kv_cap >= (1LL << 31))
    return SDPA_ERR_UNSUPPORTED;
  const size_t need = gqa_ws_bytes(batch, heads_q, heads_kv, n_kv_cap, d_v);
  if (!workspace || workspace_bytes < need) return SDPA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SDPA_ERR_MISALIGNED;
  if (int e = check_device()) return e;
  const int group = heads_q / heads_kv;
  const int chunk = (int)gqa_chunk_for(batch, heads_q, heads_kv, n_kv_cap, d_k);
  sdpa::DecodeParams p;  // the combine (and the CUDA-core split) parameters
  p.Q = (const __nv_bfloat16*)Q;
  p.K = (const __nv_bfloat16*)K;
  p.V = (const __nv_bfloat16*)V;
  p.kv_lens = kv_lens;
  p.H = heads_q;
  p.H_kv = heads_kv;
  p.group = group;
  p.n_cap = n_kv_cap;
  p.chunk = chunk;
  p.n_split = (n_kv_cap + chunk - 1) / chunk;
  p.part_o = (float*)workspace;
  p.part_lse = p.part_o + (size_t)batch * heads_q * p.n_split * d_v;
  p.O = (__nv_bfloat16*)O;
  p.LSE = LSE;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t s = (cudaStream_t)stream;
  if (gqa_tensor_path(group, d_k)) {
    const int rc = group <= 16
                       ? launch_decode_gqa<16>(Q, K, V, kv_lens, p.part_o, p.part_lse, batch, heads_q, heads_kv,
                                               n_kv_cap, chunk, p.n_split, scale, s)
                       : launch_decode_gqa<32>(Q, K, V, kv_lens, p.part_o, p.part_lse, batch, heads_q, heads_kv,
                                               n_kv_cap, chunk, p.n_split, scale, s);
    if (rc != SDPA_OK) return rc;
    sdpa::sdpa_decode_combine_kernel<128><<<(unsigned)(batch * heads_q), 128, 0, s>>>(p);
  } else {
    dim3 grid((unsigned)p.n_split, (unsigned)heads_q, (unsigned)batch);
    if (d_k == 64) {
      sdpa::sdpa_decode_split_kernel<64><<<grid, sdpa::DECODE_THREADS, 0, s>>>(p);
      sdpa::sdpa_decode_combine_kernel<64><<<(unsigned)(batch * heads_q), 64, 0, s>>>(p);
    } else {
      sdpa::sdpa_decode_split_kernel<128><<<grid, sdpa::DECODE_THREADS, 0, s>>>(p);
      sdpa::sdpa_decode_combine_kernel<128><<<(unsigned)(batch * heads_q), 128, 0, s>>>(p);
    }
  }
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SDPA_OK : cuda_fail("gqa decode launch", e);
}

// ------------------------------------------------------------------ sdpa_bwd
namespace {
long long bwd_rows_padded(long long n_q) { return (n_q + 127) / 128 * 128; }

template <int D, bool CAUSAL>
int launch_bwd(const void* Q, const void* K, const void* V, const sdpa::BwdParams& p, cudaStream_t stream) {
  using Cfg = sdpa::BwdCfg<D>;
  auto kdkdv = sdpa::sdpa_bwd_dkdv_kernel<D, CAUSAL>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kdkdv, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
    if constexpr (!Cfg::FUSED_DQ)
      if (attr_err == cudaSuccess)
        attr_err = cudaFuncSetAttribute(sdpa::sdpa_bwd_dq_kernel<D, CAUSAL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        Cfg::SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(max dynamic smem, backward)", attr_err);
  CUtensorMap mq, mk, mv, mdo, mdqa;
  if (!make_map(&mq, Q, D, p.n_q, p.bh_count) || !make_map(&mk, K, D, p.n_kv, p.bh_count) ||
      !make_map(&mv, V, D, p.n_kv, p.bh_count) || !make_map(&mdo, p.dO, D, p.n_q, p.bh_count))
    return SDPA_ERR_CUDA;
  if (Cfg::FUSED_DQ) {
    if (!make_map_f32(&mdqa, p.dQacc, D, p.n_q_pad, p.bh_count)) return SDPA_ERR_CUDA;
  } else {
    mdqa = mq;  // not read
  }
  sdpa::sdpa_bwd_pre_kernel<D><<<dim3((unsigned)(p.n_q_pad / 128), (unsigned)p.bh_count), 128, 0, stream>>>(p);
  const long long n_kt = (p.n_kv + 127) / 128, n_qt = (p.n_q + 127) / 128;
  kdkdv<<<(unsigned)(p.bh_count * n_kt), Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(mq, mk, mv, mdo, mdqa, p);
  if constexpr (Cfg::FUSED_DQ) {
    // dQ = scale * the accumulator, in bf16 (eight elements per thread and pass)
    const long long n8 = (long long)p.bh_count * p.n_q * (D / 8);
    long long blocks = (n8 + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    sdpa::sdpa_bwd_dq_out_kernel<D><<<(unsigned)blocks, 256, 0, stream>>>(p);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SDPA_OK : cuda_fail("backward launch", e);
  } else {
    // dq reads only what the pre kernel wrote (complete before dkdv started), so it is launched as a
    // programmatic dependent: its CTAs start on the SMs dkdv's last wave leaves, and it waits for
    // dkdv itself before it completes.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.bh_count * n_qt));
    cfg.blockDim = dim3(Cfg::THREADS);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, sdpa::sdpa_bwd_dq_kernel<D, CAUSAL>, mq, mk, mv, mdo, p);
    return e == cudaSuccess ? SDPA_OK : cuda_fail("backward launch", e);
  }
}
}  // namespace

// Per padded query row: D and LSE log2(e), then (used at d = 64) 64 fp32 dQ accumulator columns and
// 32 bytes of the d = 64 kernel's per-query terms.
constexpr long long kBwdFloatsPerRow = 2 + 64 + 8;

// d = 64: the one-kernel backward (sdpa_bwd_d64_kernel), then dQ = scale * the fp32 accumulator.
#ifndef SDPA_BWD_D64_KERNEL
#define SDPA_BWD_D64_KERNEL 1
#endif
namespace {
template <bool CAUSAL>
int launch_bwd_d64(const void* Q, const void* K, const void* V, const sdpa::BwdParams& p, cudaStream_t stream) {
  using Cfg = sdpa::BwdD64Cfg;
  auto kern = sdpa::sdpa_bwd_d64_kernel<CAUSAL>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [&] {
    attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(max dynamic smem, backward d64)", attr_err);
  CUtensorMap mq, mk, mv, mdo, mdqa;
  if (!make_map(&mq, Q, 64, p.n_q, p.bh_count) || !make_map(&mk, K, 64, p.n_kv, p.bh_count) ||
      !make_map(&mv, V, 64, p.n_kv, p.bh_count) || !make_map(&mdo, p.dO, 64, p.n_q, p.bh_count) ||
      !make_map_f32(&mdqa, p.dQacc, 64, p.n_q_pad, p.bh_count))
    return SDPA_ERR_CUDA;
  sdpa::sdpa_bwd_pre_kernel<64><<<dim3((unsigned)(p.n_q_pad / 128), (unsigned)p.bh_count), 128, 0, stream>>>(p);
  // persistent: one CTA per SM (at most one per unit), each walking (batch-head, key tile) units
  long long grid = (long long)p.bh_count * ((p.n_kv + 127) / 128);
  if (grid > sm_count()) grid = sm_count();
  kern<<<(unsigned)grid, Cfg::THREADS, Cfg::SMEM_BYTES, stream>>>(mq, mk, mv, mdo, mdqa, p);
  const long long n8 = (long long)p.bh_count * p.n_q * (64 / 8);
  long long blocks = (n8 + 255) / 256;
  if (blocks > 148 * 8) blocks = 148 * 8;
  sdpa::sdpa_bwd_dq_out_kernel<64><<<(unsigned)blocks, 256, 0, stream>>>(p);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SDPA_OK : cuda_fail("backward launch", e);
}
}  // namespace

extern "C" size_t sdpa_bwd_workspace_size(int batch, int heads, int n_q) {
  if (batch <= 0 || heads <= 0 || n_q <= 0) return 0;
  return (size_t)(kBwdFloatsPerRow * batch * heads * bwd_rows_padded(n_q)) * sizeof(float);
}

extern "C" int sdpa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                        void* dQ, void* dK, void* dV, int batch, int heads, int n_q, int n_kv, int d_k, int d_v,
                        float scale, int causal, void* workspace, size_t workspace_bytes, void* stream) {
  if (batch < 0 || heads < 0 || n_q < 0 || n_kv < 1 || !std::isfinite(scale)) return SDPA_ERR_INVALID_ARG;
  if (d_k != d_v || (d_k != 64 && d_k != 128)) return SDPA_ERR_UNSUPPORTED;
  if (batch == 0 || heads == 0 || n_q == 0) return SDPA_OK;
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV) return SDPA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) || !aligned4(LSE) ||
      !aligned16(dQ) || !aligned16(dK) || !aligned16(dV))
    return SDPA_ERR_MISALIGNED;
  const long long bh = (long long)batch * heads;
  if (bh * (long long)(n_q > n_kv ? n_q : n_kv) >= (1LL << 31) || bh * ((n_kv + 127) / 128) >= (1LL << 31) ||
      bh * bwd_rows_padded(n_q) >= (1LL << 31))
    return SDPA_ERR_UNSUPPORTED;
  const size_t need = sdpa_bwd_workspace_size(batch, heads, n_q);
  if (!workspace || workspace_bytes < need) return SDPA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SDPA_ERR_MISALIGNED;
  if (int e = check_device()) return e;
  sdpa::BwdParams p;
  p.O = (const __nv_bfloat16*)O;
  p.dO = (const __nv_bfloat16*)dO;
  p.LSE = LSE;
  p.n_q = n_q;
  p.n_kv = n_kv;
  p.n_q_pad = (int)bwd_rows_padded(n_q);
  p.bh_count = (int)bh;
  p.Dvec = (float*)workspace;
  p.L2 = p.Dvec + (size_t)bh * p.n_q_pad;
  // d = 64 accumulates dQ in fp32 here (16-byte aligned: n_q_pad is a multiple of 128); its
  // one-kernel form needs scale != 0 (it adds -LSE log2(e) / (scale log2(e)) to S)
  p.dQacc = d_k == 64 ? p.L2 + (size_t)bh * p.n_q_pad : nullptr;
  const bool one_kernel = d_k == 64 && SDPA_BWD_D64_KERNEL && std::fabs(scale * 1.4426950408889634f) >= 1e-30f;
  // the per-query term images (d = 64 one-kernel form; d = 128 dK/dV kernel), both need scale != 0
  const bool terms = std::fabs(scale * 1.4426950408889634f) >= 1e-30f &&
                     (d_k == 64 ? one_kernel : sdpa::BwdCfg<128>::AUG);
  p.aug = terms ? reinterpret_cast<uint8_t*>(p.L2 + (size_t)bh * p.n_q_pad * 65) : nullptr;
  p.dQ = (__nv_bfloat16*)dQ;
  p.dK = (__nv_bfloat16*)dK;
  p.dV = (__nv_bfloat16*)dV;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  cudaStream_t s = (cudaStream_t)stream;
  if (d_k == 64) {
    if (one_kernel) return causal ? launch_bwd_d64<true>(Q, K, V, p, s) : launch_bwd_d64<false>(Q, K, V, p, s);
    return causal ? launch_bwd<64, true>(Q, K, V, p, s) : launch_bwd<64, false>(Q, K, V, p, s);
  }
  return causal ? launch_bwd<128, true>(Q, K, V, p, s) : launch_bwd<128, false>(Q, K, V, p, s);
}

extern "C" int sdpa_get_last_device_error(void* stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return SDPA_ERR_CUDA;
  int v = 0;
  const int zero = 0;
  if (cudaMemcpyFromSymbol(&v, sdpa::g_sdpa_error, sizeof v) != cudaSuccess) return SDPA_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(sdpa::g_sdpa_error, &zero, sizeof zero) != cudaSuccess) return SDPA_ERR_CUDA;
  return v;
}

extern "C" const char* sdpa_status_string(int status) {
  switch (status) {
    case SDPA_OK: return "SDPA_OK";
    case SDPA_ERR_INVALID_ARG: return "SDPA_ERR_INVALID_ARG";
    case SDPA_ERR_UNSUPPORTED: return "SDPA_ERR_UNSUPPORTED";
    case SDPA_ERR_MISALIGNED: return "SDPA_ERR_MISALIGNED";
    case SDPA_ERR_WORKSPACE: return "SDPA_ERR_WORKSPACE";
    case SDPA_ERR_CUDA: return "SDPA_ERR_CUDA";
    case SDPA_ERR_DEVICE_TIMEOUT: return "SDPA_ERR_DEVICE_TIMEOUT";
    case SDPA_ERR_DEVICE_BAD_LENGTH: return "SDPA_ERR_DEVICE_BAD_LENGTH";
    case SDPA_ERR_DEVICE_CHECK: return "SDPA_ERR_DEVICE_CHECK";
    default: return "SDPA_UNKNOWN_STATUS";
  }
}
