/*
 * sdpa.h -- C ABI of the B200 (sm_100a) exact scaled dot-product attention library.
 *
 * What every entry point computes, for each (batch b, head h) slice:
 *
 *     O = softmax(Q K^T * scale) V          (row-wise, numerically stable softmax)
 *     LSE_i = ln sum_j exp(scale * q_i . k_j)   over the keys row i may see
 *
 * This is the attention definition of the Mathematics-of-Arrays article
 * (agents-report.net, "DNF derivation": Attention(Q,K,V) = softmax(QK^T/sqrt(d_k))V,
 * here with the scale passed in) and of the MoA paper's abstract ("Attention at
 * the Theoretical Minimum", paperdance.org): no intermediate array -- no n x n
 * score or probability buffer and no transposed-key copy -- is ever written to
 * memory, so global-memory traffic is O(n*d_k + n*d_v): Q, K and V are read and
 * O (and LSE) written, once.
 *
 * Conventions shared by all entry points
 *  - Layout: row-major and contiguous.  Q [batch, heads, n_q, d_k],
 *    K [batch, heads, n_kv, d_k], V [batch, heads, n_kv, d_v],
 *    O [batch, heads, n_q, d_v], LSE [batch, heads, n_q] (float).
 *  - Ownership: every pointer is caller-owned DEVICE memory, valid until the work
 *    queued on `stream` has finished.  The library allocates no memory.
 *  - Execution: asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 *    stream) on the current device.  No call synchronises except
 *    sdpa_get_last_device_error.
 *  - Causal masking is bottom-right aligned: query row i sees key j iff
 *    j <= i + (n_kv - n_q).  A row that sees no key (only when n_q > n_kv) gets
 *    O = 0 and LSE = -inf.
 *  - LSE may be NULL (not written).  It is the natural log of the SCALED logits.
 *  - Errors: argument checks run on the host before any launch and return a
 *    status without touching memory.  A failed launch returns SDPA_ERR_CUDA.
 *    Problems found on the device (a pipeline wait that ran out of time, a decode
 *    length outside [1, n_kv_cap]) set a device error word that
 *    sdpa_get_last_device_error reads; kernels never trap.
 *  - Degenerate shapes: batch == 0, heads == 0 or n_q == 0 -> SDPA_OK, nothing written.
 */
#ifndef SDPA_B200_H
#define SDPA_B200_H

#include <stddef.h>

#if defined(__GNUC__)
#define SDPA_API __attribute__((visibility("default")))
#else
#define SDPA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SDPA_OK = 0,
  SDPA_ERR_INVALID_ARG = 1,     /* null pointer, negative size, n_kv == 0, bad flag */
  SDPA_ERR_UNSUPPORTED = 2,     /* valid but not implemented (e.g. head dim) */
  SDPA_ERR_MISALIGNED = 3,      /* a pointer is not 16-byte aligned */
  SDPA_ERR_WORKSPACE = 4,       /* workspace missing or too small */
  SDPA_ERR_CUDA = 5,            /* a CUDA runtime/driver call failed */
  SDPA_ERR_DEVICE_TIMEOUT = 6,  /* a kernel pipeline wait gave up (device error word) */
  SDPA_ERR_DEVICE_BAD_LENGTH = 7, /* a decode length was outside [1, n_kv_cap] (device error word) */
  SDPA_ERR_DEVICE_CHECK = 8     /* debug builds (-DSDPA_DEBUG=1) only: a device-side consistency check
                                   failed -- a pipeline barrier ended a kernel with a phase count its
                                   users did not account for, or TMEM was not allocated at column 0 */
} sdpa_status;

/*
 * sdpa_fwd -- bf16 prefill on the 5th-generation tensor cores (tcgen05/TMEM, TMA).
 *
 * Q, K, V, O: __nv_bfloat16, layout above.  LSE: float or NULL.
 * d_k == d_v, and both in {64, 128} (else SDPA_ERR_UNSUPPORTED).
 * n_q >= 0, n_kv >= 1.  batch*heads*max(n_q, n_kv) < 2^31.
 * causal: 0 or 1.  scale: any finite value (else SDPA_ERR_INVALID_ARG).  A negative
 * scale is applied by negating Q inside the S = Q K^T product (the instruction's
 * negate-A bit), so the online softmax always works with |scale|; scale == 0 gives every
 * visible key weight 1 / (number of visible keys) and LSE = ln(number of visible keys)
 * (computed with the factor 2^-126 in place of 0, which leaves every weight exactly 1 in
 * fp32 for scores below 2^100 in magnitude and keeps masked entries at weight 0).
 * Every pointer 16-byte aligned (TMA), else SDPA_ERR_MISALIGNED.
 * Arithmetic: S = Q K^T and O += P V on the tensor cores with fp32
 * accumulation; softmax in fp32 with P rounded to bf16; O rounded to bf16
 * (round to nearest even); LSE in fp32.
 */
SDPA_API int sdpa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int batch, int heads,
             int n_q, int n_kv, int d_k, int d_v, float scale, int causal, void* stream);

/*
 * sdpa_fwd_window -- sdpa_fwd with a local (sliding) window instead of the causal flag.
 *
 * Query row i sits at key position p = i + (n_kv - n_q) (bottom-right alignment, as for
 * causal masking) and sees keys j with p - window_left <= j <= p + window_right.  -1 leaves
 * that side open: (-1, 0) is causal, (-1, -1) full attention, (w, 0) a causal window of
 * w + 1 keys.  Key tiles wholly outside every row's window are skipped, so the work is
 * proportional to the window, not to n_kv.  Rows whose window holds no key get O = 0 and
 * LSE = -inf.  Windowed attention as the way to bound the cost of long sequences follows the
 * 2-simplicial article (szyisi.cn, "model design": sliding windows w1, w2 over the sequence);
 * here the window is the one-dimensional one of ordinary attention.
 * Other arguments, layouts, alignment and errors as sdpa_fwd; window_left and window_right
 * must be >= -1 (else SDPA_ERR_INVALID_ARG).
 */
SDPA_API int sdpa_fwd_window(const void* Q, const void* K, const void* V, void* O, float* LSE, int batch,
                             int heads, int n_q, int n_kv, int d_k, int d_v, float scale, int window_left,
                             int window_right, void* stream);

/*
 * sdpa_fwd_f32 -- fp32 prefill on the CUDA cores (FMA pipes); same semantics as
 * sdpa_fwd with float tensors.  1 <= d_k, d_v <= 128.  Scores, softmax
 * weights and the output sum are all fp32 (no tensor cores: TF32 would lose
 * about three decimal digits).  Pointers must be 4-byte aligned.
 */
SDPA_API int sdpa_fwd_f32(const float* Q, const float* K, const float* V, float* O, float* LSE, int batch,
                 int heads, int n_q, int n_kv, int d_k, int d_v, float scale, int causal, void* stream);

/*
 * sdpa_decode_workspace_size -- bytes of device workspace sdpa_decode needs
 * for this shape (partial outputs and log-sum-exps of the KV splits).
 * Returns 0 for a degenerate or invalid shape.
 */
SDPA_API size_t sdpa_decode_workspace_size(int batch, int heads, int n_kv_cap, int d_v);

/*
 * sdpa_decode -- one query row per (batch, head) against a KV cache (split-KV).
 *
 * Q [batch, heads, d_k]; K [batch, heads, n_kv_cap, d_k]; V [batch, heads, n_kv_cap, d_v],
 * all __nv_bfloat16.  kv_lens: int32 [batch] in DEVICE memory, each in
 * [1, n_kv_cap]: sequence b attends to cache rows 0 .. kv_lens[b]-1, and rows
 * at or past kv_lens[b] are never read (they may hold anything, NaN included).
 * O [batch, heads, d_v] bf16; LSE [batch, heads] float or NULL.
 * d_k == d_v in {64, 128}.  All pointers 16-byte aligned.
 * workspace: caller-owned device memory of at least
 * sdpa_decode_workspace_size(batch, heads, n_kv_cap, d_v) bytes, else
 * SDPA_ERR_WORKSPACE; its contents need no initialisation and are scratch
 * afterwards.  A length outside [1, n_kv_cap] is clamped on the device and
 * reported as SDPA_ERR_DEVICE_BAD_LENGTH by sdpa_get_last_device_error.
 * (A single query row sees every cached key, so causal masking does not apply.)
 */
SDPA_API int sdpa_decode(const void* Q, const void* K, const void* V, const int* kv_lens, void* O, float* LSE,
                int batch, int heads, int n_kv_cap, int d_k, int d_v, float scale, void* workspace,
                size_t workspace_bytes, void* stream);

/*
 * sdpa_decode_noalloc -- sdpa_decode for callers that cannot allocate device memory.
 *
 * The attention pages have no counterpart to this entry point; it exists for
 * callers that are not allowed to call cudaMalloc or to hold a workspace
 * buffer -- for example a plug-in whose host application owns every device
 * allocation, or code running under a fixed memory budget where a framework's
 * allocator is the only one permitted.  It computes exactly what sdpa_decode
 * computes, with the same arguments minus the workspace, and allocates nothing:
 * its scratch (the per-split partial outputs and log-sum-exps) lives in one
 * library-owned device array of SDPA_DECODE_STATIC_SCRATCH_BYTES, which every
 * GPU that loads this library holds until the process exits.
 *
 *  - Size limit: batch * heads * splits * (d_v + 1) * 4 bytes must fit in the array.
 *    The call picks the smallest key-split length (a power of two, at least the
 *    one sdpa_decode uses) that fits; if even one split per (batch, head) does not
 *    fit (batch * heads * (d_v + 1) * 4 > SDPA_DECODE_STATIC_SCRATCH_BYTES) it
 *    returns SDPA_ERR_WORKSPACE before launching anything.
 *  - Set-up: the first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current.  Make that first call on
 *    every device before any stream capture begins.  Later calls on a stream that
 *    is not capturing look the address up again (it allocates nothing), so a device
 *    reset that reloads the library's module never leaves a stale address behind;
 *    calls on a capturing stream use the address of the last call outside capture,
 *    so after a device reset make one call outside capture before capturing again.
 *  - Sharing: every call uses the same array and it keeps the last call's
 *    contents.  Nothing in it needs to start at zero (each call writes every
 *    partial it reads).  Calls whose work overlaps on the GPU (other streams,
 *    other host threads on the same device) race on the array: serialise them.
 *  - Results may differ from sdpa_decode in the last bits, because the key
 *    splits can be longer.
 */
#define SDPA_DECODE_STATIC_SCRATCH_BYTES (16u << 20)
SDPA_API int sdpa_decode_noalloc(const void* Q, const void* K, const void* V, const int* kv_lens, void* O,
                                 float* LSE, int batch, int heads, int n_kv_cap, int d_k, int d_v, float scale,
                                 void* stream);

/*
 * sdpa_bwd_workspace_size -- bytes of device workspace sdpa_bwd needs:
 * 74 * batch * heads * round_up(n_q, 128) floats: the per-row vectors D and LSE log2(e), then
 * for the d = 64 backward 64 fp32 columns per row in which it accumulates dQ before rounding it
 * to bf16, and 32 bytes per row of per-query terms it adds inside its tensor-core products
 * (both unused at d = 128).  0 for a degenerate shape.
 */
SDPA_API size_t sdpa_bwd_workspace_size(int batch, int heads, int n_q);

/*
 * sdpa_bwd -- gradients of sdpa_fwd: dQ, dK, dV for the loss gradient dO, from the forward's
 * inputs, its output O and its LSE (the MoA roadmap's last stage, a backward pass in the same
 * memory-optimal form: agents-report.net MoA article, "implementation roadmap").
 *
 * With P = softmax(Q K^T scale) recomputed from LSE, D_i = dO_i . O_i and dS = P (dO V^T - D):
 *   dV = P^T dO,   dK = scale dS^T Q,   dQ = scale dS K.
 * Nothing of size n_q x n_kv is written; each gradient is written once.  At d = 64 (scale != 0)
 * dQ is first summed over the key tiles in fp32 in the workspace by reduce-adds whose order is not
 * fixed, so dQ can differ in its last bits from one call to the next (dK and dV, and everything
 * at d = 128, are reproducible).
 * Q, O, dO, dQ [batch, heads, n_q, d]; K, V, dK, dV [batch, heads, n_kv, d]; all
 * __nv_bfloat16, contiguous, 16-byte aligned.  LSE [batch, heads, n_q] float as sdpa_fwd wrote
 * it (required).  d_k == d_v in {64, 128}; scale (any finite value) and causal as in the forward call.
 * workspace: caller-owned device memory of sdpa_bwd_workspace_size bytes (scratch, rewritten
 * by every call: calls that may run at the same time need separate workspaces).
 * Rows whose window held no key (causal, n_q > n_kv) contribute nothing and get dQ = 0.
 * Errors as sdpa_fwd, plus SDPA_ERR_WORKSPACE.
 */
SDPA_API int sdpa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                      void* dQ, void* dK, void* dV, int batch, int heads, int n_q, int n_kv, int d_k, int d_v,
                      float scale, int causal, void* workspace, size_t workspace_bytes, void* stream);

/*
 * sdpa_decode_gqa_workspace_size -- bytes of device workspace sdpa_decode_gqa needs for
 * this shape; 0 for a degenerate or invalid one (heads_q not a multiple of heads_kv).
 */
SDPA_API size_t sdpa_decode_gqa_workspace_size(int batch, int heads_q, int heads_kv, int n_kv_cap, int d_v);

/*
 * sdpa_decode_gqa -- grouped-query decode: heads_q query heads share heads_kv key/value
 * heads, query head h reading key/value head h / (heads_q / heads_kv) (consecutive query
 * heads form a group).  Grouped-query layouts are what let the 2-simplicial article
 * (szyisi.cn, "model design") tile along query heads into dense products; here each
 * group's keys and values are read from HBM once for all of its query heads.
 *
 * Q [batch, heads_q, d_k]; K [batch, heads_kv, n_kv_cap, d_k]; V [batch, heads_kv,
 * n_kv_cap, d_v]; O [batch, heads_q, d_v], all __nv_bfloat16; LSE [batch, heads_q] float
 * or NULL.  kv_lens, alignment, workspace ownership and errors as sdpa_decode, with the
 * workspace sized by sdpa_decode_gqa_workspace_size.  heads_q % heads_kv != 0 is
 * SDPA_ERR_INVALID_ARG.  d_k == d_v == 128 with 2 to 32 query heads per group runs on
 * the tensor cores (tcgen05); other groups and d = 64 run the CUDA-core split kernel
 * with the same head mapping.  heads_q == heads_kv is sdpa_decode.
 */
SDPA_API int sdpa_decode_gqa(const void* Q, const void* K, const void* V, const int* kv_lens, void* O, float* LSE,
                             int batch, int heads_q, int heads_kv, int n_kv_cap, int d_k, int d_v, float scale,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * sdpa_get_last_device_error -- synchronise `stream`, then read and clear the
 * device error word of the current device.  Returns SDPA_OK, the first device
 * error recorded since the last call, or SDPA_ERR_CUDA if the synchronisation
 * itself failed.
 */
SDPA_API int sdpa_get_last_device_error(void* stream);

/* sdpa_status_string -- a static, human-readable name for a status code. */
SDPA_API const char* sdpa_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* SDPA_B200_H */
