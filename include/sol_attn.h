/*
 * sol_attn.h -- C ABI of the B200 (sm_100a) Sol-Attn sparse attention forward.
 *
 * The operation (Sol-Attn visual explainer, mxino.github.io, "The complete idea
 * in one pass", Eqs. 4, 5, 9, 10, 11): for every (batch, head)
 *   1. pool:   Qbar_i = mean of the query rows of block i, Kbar_j = mean of the
 *              key rows of block j, Vhat_j = sum of the value rows of block j
 *              (blocks are contiguous runs of Bq query / Bk key tokens; the
 *              last may be partial, key block j holding n_j tokens);
 *   2. score:  s_ij = Qbar_i . Kbar_j / sqrt(d)                      (Eq. 4 legend)
 *   3. route:  mu_i, sigma_i = mean and population std of row s_i    (Eq. 5)
 *              (or sigma_i from the diagonal estimator, see the flags);
 *              tau_i = mu_i + beta * sigma_i; S_i = { j : s_ij > tau_i } (Eq. 4)
 *   4. attend: for every query token q of block i
 *                D = sum_{j in U_i} n_j exp(q.Kbar_j/sqrt d) + sum_{j in S_i} sum_{k in j} exp(q.k/sqrt d)  (Eq. 9)
 *                N = sum_{j in U_i} exp(q.Kbar_j/sqrt d) Vhat_j + sum_{j in S_i} sum_{k in j} exp(q.k/sqrt d) v_k (Eq. 10)
 *              out = N / D, accumulated in one online-softmax pass.
 * beta = -INFINITY selects every block (dense attention); beta = +INFINITY
 * selects none (every block through its pooled key).  The 1/sqrt(d) logit
 * scale is applied inside.  Rows are not masked (bidirectional attention).
 *
 * Conventions for every entry point
 *   - Tensors are dense row-major [batch, heads, L, d] (d fastest), on the
 *     current CUDA device, 16-byte aligned.  The caller owns them.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *     enqueued on it; no call synchronises the host, except
 *     sol_attn_device_status().
 *   - Scratch memory (pooled tensors, the 1-bit selection mask, the work list;
 *     about 4% of one input tensor) is taken stream-ordered on `stream` from a
 *     memory pool the library creates per device (it keeps freed memory for
 *     the next call) and released with cudaFreeAsync on the same stream.
 *   - Return value: SOL_OK or a negative sol_status.  Arguments are checked on
 *     the host before anything is enqueued; on an argument error nothing is
 *     enqueued.  Errors of kernels already enqueued surface at the caller's
 *     next synchronisation, as usual in CUDA.
 *   - Results are deterministic for a given input, shape and GPU.
 */
#ifndef SOL_ATTN_H
#define SOL_ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SOL_OK = 0,
  SOL_ERR_INVALID_ARG = -1,     /* null/misaligned pointer, bad size, NaN beta */
  SOL_ERR_UNSUPPORTED = -2,     /* valid but not built: see the support list below */
  SOL_ERR_CUDA = -3,            /* a CUDA runtime call failed */
  SOL_ERR_NO_MEMORY = -4,       /* scratch allocation failed */
  SOL_ERR_DEVICE_TIMEOUT = -5   /* a kernel gave up on a bounded wait (see sol_attn_device_status) */
} sol_status;

/* Flags of sol_attn_forward_ex and sol_attn_stats_ex. */
#define SOL_FLAG_KEEP_OR_DROP 1u  /* correction off: unselected blocks contribute nothing (the
                                     "ordinary block sparse" baseline the method is contrasted
                                     with; a query block with no selected block outputs zeros) */
#define SOL_FLAG_DIAGONAL_SIGMA 2u /* sigma_i of Eq. 4 from the cheaper diagonal estimator the
                                     explainer names beside Eq. 5 (formula not printed; read as
                                     sigma_i^2 = sum_c Qbar_ic^2 Var_j(Kbar_jc) / d, the population
                                     variance of each pooled-key channel over the key blocks,
                                     i.e. Eq. 5 with the off-diagonal covariance dropped).
                                     mu_i is unchanged. */
#define SOL_FLAG_ROUTE_IN_KERNEL 4u /* Eq. 4 decided inside the tensor-core attention kernel
                                     (two of its warps score each key block from the fp32
                                     pooled vectors with the router's arithmetic and compare
                                     with the router's tau_i; Eq. 11's "proxy reuse"): no
                                     selection mask is written or read.  Same results as
                                     without the flag.  Tensor-core calls only (bf16, Bq = 128)
                                     with ceil(L / Bk) <= 2048, else SOL_ERR_UNSUPPORTED. */

typedef enum {
  SOL_DTYPE_BF16 = 0,           /* bfloat16 inputs and output; fp32 accumulation */
  SOL_DTYPE_F32 = 1             /* float32 inputs and output; fp32 arithmetic */
} sol_dtype;

/*
 * Supported shapes: d in {64, 128}; Bq in {64, 128} and Bk in {64, 128}
 * (independently: query blocks of Bq tokens, key blocks of Bk tokens, the
 * Eq. 9 weight of a key block is its token count); L >= 1;
 * 1 <= batch * heads <= 65535; batch * heads * L * d < 2^40;
 * ceil(L / Bk) <= 6144; beta not NaN.
 * Other values return SOL_ERR_UNSUPPORTED.  bf16 (any supported d, Bq and
 * Bk) runs the tensor-core (tcgen05/TMEM/TMA) kernel; with Bq == 64 each
 * 128-row tile holds two consecutive query blocks, which walk the union of
 * their selections, each masking the key blocks it did not select (the
 * results are those of one block at a time).  fp32 runs the CUDA-core
 * kernel.
 */

/*
 * Sparse attention forward, bf16.
 *   q, k, v : const bf16*  [batch, heads, L, d], device
 *   out     : bf16*        [batch, heads, L, d], device, written fully
 *   Bq, Bk  : query / key block size in tokens
 *   beta    : Eq. 4 knob; -INFINITY = dense, +INFINITY = all approximate
 *   stream  : cudaStream_t
 */
int sol_attn_forward(const void* q, const void* k, const void* v, void* out,
                     int batch, int heads, int L, int d, int Bq, int Bk,
                     float beta, void* stream);

/* Same operation on float32 tensors (fp32 arithmetic throughout). */
int sol_attn_forward_f32(const float* q, const float* k, const float* v, float* out,
                         int batch, int heads, int L, int d, int Bq, int Bk,
                         float beta, void* stream);

/*
 * Selection statistics, computed by the same pooling and routing kernels as
 * the forward (Eqs. 4-5).  No V is needed.
 *   counts      : int32* [batch, heads, Nq] device; counts[.] = |S_i|
 *   mask_or_null: uint32* [batch, heads, Nq, ceil(Nk/32)] device, or NULL;
 *                 bit (j % 32) of word (j / 32) is 1 iff key block j is in S_i
 *   dtype       : sol_dtype of q and k
 * Nq = ceil(L/Bq), Nk = ceil(L/Bk).
 */
int sol_attn_stats(const void* q, const void* k, int32_t* counts, uint32_t* mask_or_null,
                   int batch, int heads, int L, int d, int Bq, int Bk,
                   float beta, int dtype, void* stream);

/* sol_attn_stats with flags: 0 or SOL_FLAG_DIAGONAL_SIGMA (any other bit:
 * SOL_ERR_INVALID_ARG).  sol_attn_stats(...) is sol_attn_stats_ex(..., 0, stream). */
int sol_attn_stats_ex(const void* q, const void* k, int32_t* counts, uint32_t* mask_or_null,
                      int batch, int heads, int L, int d, int Bq, int Bk,
                      float beta, int dtype, unsigned int flags, void* stream);

/*
 * Routing diagnostic: how many of each query block's decisions are near ties.
 * Runs the forward's pooling and routing kernels (Eqs. 4-5) and writes, for
 * every query block i,
 *   near_ties[i] = #{ j : |s_ij - tau_i| < margin }      (s, tau as in Eq. 4)
 * -- the pairs whose selection fp32 rounding may decide either way (an exact
 * fp64 evaluation can land on the other side of tau_i).  With beta = +-INFINITY
 * every count is 0.
 *   near_ties: int32* [batch, heads, Nq] device
 *   margin   : >= 0 and finite, in the units of s (logits scaled by 1/sqrt(d))
 *   dtype, flags: as sol_attn_stats_ex (flags 0 or SOL_FLAG_DIAGONAL_SIGMA)
 * The paper has no counterpart; it is a measurement aid.  Errors as
 * sol_attn_stats (null near_ties or a negative, NaN or infinite margin:
 * SOL_ERR_INVALID_ARG).
 */
int sol_attn_near_ties(const void* q, const void* k, int32_t* near_ties, float margin,
                       int batch, int heads, int L, int d, int Bq, int Bk,
                       float beta, int dtype, unsigned int flags, void* stream);

/*
 * Extended forward.  Arguments as sol_attn_forward plus:
 *   dtype  : sol_dtype of q, k, v, out
 *   flags  : 0 or an OR of SOL_FLAG_KEEP_OR_DROP, SOL_FLAG_DIAGONAL_SIGMA,
 *            SOL_FLAG_ROUTE_IN_KERNEL (unknown bits: SOL_ERR_INVALID_ARG)
 *   events : NULL, or 4 cudaEvent_t the library records on `stream`
 *            before pooling, after pooling, after routing and after the
 *            attention kernel (time each stage with cudaEventElapsedTime)
 */
int sol_attn_forward_ex(const void* q, const void* k, const void* v, void* out, int dtype,
                        int batch, int heads, int L, int d, int Bq, int Bk,
                        float beta, unsigned int flags, void* const* events, void* stream);

/*
 * Reads and clears this device's status word, which a kernel sets when one of
 * its bounded waits runs out (it then abandons its work and exits cleanly).
 * Synchronises `stream` first.  Returns SOL_OK or SOL_ERR_DEVICE_TIMEOUT; if
 * detail is not NULL it receives the raw word (0 = no error; else 0x1000 | the
 * id of the first wait that ran out).
 * There is ONE such word per device, shared by every call on every stream of
 * the process: the first expiry since the last read is kept, later ones are
 * dropped.  With calls in flight on several streams, the word cannot say
 * which call's wait ran out; a caller that needs to know must read it after
 * each call, with no other call of this library running on the device.
 */
int sol_attn_device_status(void* stream, int32_t* detail);

/*
 * Load-balance record of the most recent tensor-core attention launch made by
 * this process (on the current device): for each CTA of its grid (one per SM
 * at most) one row of four uint64 -- start and end time of the CTA's work in
 * ns of the GPU's global timer, the work items (query blocks) it took and the
 * tiles it processed.  Synchronises `stream` first.  Writes min(grid,
 * max_rows) rows to the host array `rows` and returns that count (0 if no
 * such launch has been made), or a negative sol_status.  The record is one
 * per device and the next tensor-core launch overwrites it; with launches in
 * flight on several streams, read it with no other call running.  The paper
 * has no counterpart: it is a measurement aid.
 */
int sol_attn_cta_times(void* stream, uint64_t* rows, int max_rows);

/*
 * Forward without any memory allocation, for callers that may not allocate
 * device memory (plugin hosts that own all device memory, serving loops that
 * reserve everything up front and treat an allocation as a failure).  The
 * paper has no counterpart; the computation is that of sol_attn_forward, with
 * the same arguments, kernels and results.
 *   - Scratch comes from a fixed 48 MiB device array inside the library,
 *     present on every GPU that loads it until the process exits.  A call
 *     whose scratch would not fit returns SOL_ERR_NO_MEMORY before enqueueing
 *     anything.  With Bk = 128 the Wan2.1 720p call (40 heads, L = 75600)
 *     needs about 37 MiB and the HunyuanVideo 720p call (24 heads,
 *     L = 119056) about 36 MiB, so both fit; the same calls with Bk = 64 need
 *     about 61 and 60 MiB and return SOL_ERR_NO_MEMORY.
 *   - The first call on a device looks up the array's device address (a
 *     cudaGetSymbolAddress); make that first call before any stream capture.
 *   - All calls on a device share the array, and it keeps the previous call's
 *     contents (the call resets what must start at zero).  Calls that overlap
 *     on the GPU -- e.g. on two streams without ordering between them -- race
 *     on it: keep them ordered.
 */
int sol_attn_forward_noalloc(const void* q, const void* k, const void* v, void* out,
                             int batch, int heads, int L, int d, int Bq, int Bk,
                             float beta, void* stream);

/*
 * Forward with the tensors in HOST memory: q, k, v are read from and out is
 * written to host buffers (page-locked memory, e.g. from cudaHostAlloc, lets
 * the copies run asynchronously; pageable memory works, with copies that
 * block the host).  The paper has no counterpart: this is for callers that
 * keep activations in host memory.  The (batch, head) slices are independent,
 * so the call cuts them into groups of `slices_per_step` and pipelines the
 * groups through two device staging buffers: group c + 1's inputs are copied
 * in and group c - 1's output copied back (on two streams the library owns
 * per device) while group c is computed on `stream`.  Same kernels and, slice
 * for slice, the same results as sol_attn_forward_ex on device copies.
 *   q, k, v        : const host pointers [batch, heads, L, d] of `dtype`, 16-byte aligned
 *   out            : host pointer, same layout; complete once `stream` reaches
 *                    the point where this call was enqueued
 *   dtype, flags   : as sol_attn_forward_ex
 *   slices_per_step: (batch, head) slices per group; 0 lets the library choose
 *                    (about 16 groups, at most 1 GiB of staging); < 0 is
 *                    SOL_ERR_INVALID_ARG
 * The host buffers must stay valid and unmodified until then.  Staging (two
 * groups of q, k, v and out) and scratch come stream-ordered from the
 * library's pool, as for sol_attn_forward.  Errors as sol_attn_forward_ex.
 */
int sol_attn_forward_host(const void* q, const void* k, const void* v, void* out, int dtype,
                          int batch, int heads, int L, int d, int Bq, int Bk,
                          float beta, unsigned int flags, int slices_per_step, void* stream);

/* Human-readable name of a sol_status value. */
const char* sol_attn_status_string(int status);

/* Library ABI version (major * 100 + minor): 105. */
int sol_attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SOL_ATTN_H */
