/*
 * diffattn.h — C ABI of libdiffattn.so: differential attention on B200.
 *
 * The operator (both forms) is
 *     DiffAttn = (softmax(Q1 K1^T / sqrt(d)) - lambda * softmax(Q2 K2^T / sqrt(d))) V
 * as defined on the "Differential Transformer" glossary page (Ultralytics),
 * section "Cómo funciona la atención diferencial", and in the lesson
 * "Atención Diferencial (V2)" (ai-engineering.academy), section
 * "La idea diferencial".  d is the width of ONE branch's query/key.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Pointers marked "device" are caller-owned CUDA device memory; the
 *    library never allocates, frees or keeps a pointer after returning.
 *  - Tensors are dense, row-major (last index fastest), with the shapes
 *    given per argument; element type is `dtype` (bf16 or fp32) for Q/K/V
 *    and the output, fp32 for lambda and norm weights.  Q/K/V/out base
 *    addresses must be 16-byte aligned (DA_ERR_ALIGNMENT otherwise).
 *  - `out` must not overlap any input.
 *  - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL is
 *    the legacy default stream) and returns before it completes.
 *  - Argument errors are detected on the host before anything is enqueued
 *    and return a negative da_status.  A launch failure returns DA_ERR_CUDA.
 *    No C++ exception crosses this interface.
 *  - `dev_status` (optional, device int, may be NULL): kernels that wait on
 *    asynchronous copies bound every wait; if one ever times out the kernel
 *    stores DA_ERR_DEVICE_TIMEOUT there (first error wins; the caller zeroes
 *    it beforehand) and returns early, leaving the output undefined.
 *  - Thread safety: concurrent calls on different streams are independent,
 *    with two exceptions: diffattn_v2_decode_noalloc's shared scratch array
 *    (see that entry point) and the prefill's tile counters (next).  The
 *    library calls no other library that keeps state.  Global state: for
 *    the bf16 tensor-core prefill (diffattn_v1_fwd / diffattn_v2_prefill
 *    and their window, training and projection variants), 64 tile counters
 *    per device in a statically allocated array.  The host gives each such
 *    launch the next counter in turn, fixed when the launch is enqueued (or
 *    captured into a CUDA graph, whose every replay then uses that
 *    counter).  On the device
 *    a launch claims its counter when it is free, hands out one tile per
 *    ticket and frees it when its last tile is taken.  A launch that finds
 *    its counter held by another launch still in flight (two graph
 *    executions made from one capture that overlap, or more than 64 launches
 *    in flight on one device) waits until that launch has taken its last
 *    tile, then proceeds: overlapping launches stay correct.  That wait is
 *    bounded: after 2 s the waiting CTAs compute nothing and store
 *    DA_ERR_SCHEDULE in dev_status, so an incomplete output never comes with
 *    status 0 (pass a status word to see it).  A counter whose holder has
 *    stopped taking tickets for 250 ms (a launch that ended with
 *    DA_ERR_DEVICE_TIMEOUT) is taken over; diffattn_reset_tile_counters
 *    frees every counter at once.
 */
#ifndef DIFFATTN_H_
#define DIFFATTN_H_

#include <stddef.h>

#if defined(__GNUC__)
#define DA_API __attribute__((visibility("default")))
#else
#define DA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DA_OK = 0,
  DA_ERR_INVALID_ARG = -1,   /* null pointer, non-positive size, bad combination */
  DA_ERR_UNSUPPORTED = -2,   /* valid arguments this library does not implement */
  DA_ERR_ALIGNMENT = -3,     /* a base address is not 16-byte aligned */
  DA_ERR_WORKSPACE = -4,     /* workspace missing or smaller than required */
  DA_ERR_CUDA = -5,          /* a CUDA runtime/driver call or launch failed */
  DA_ERR_DEVICE_TIMEOUT = -6, /* written to dev_status by a kernel whose wait timed out */
  DA_ERR_SCHEDULE = -7        /* written to dev_status by a prefill launch whose tile
                                 counter another launch held for longer than 2 s */
} da_status;

typedef enum { DA_BF16 = 0, DA_FP32 = 1 } da_dtype;

/* Human-readable name of a da_status value (static string, never NULL). */
DA_API const char* diffattn_status_string(int status);

/* lambda_init(l) = 0.8 - 0.6 * exp(-0.3 * (l - 1)) for 1-based layer l
 * (glossary page, "Cómo funciona": the per-layer starting value of lambda).
 * Host only.  Returns NaN if layer < 1. */
DA_API double diffattn_lambda_init(int layer);

/* Per-head lambda from its four learned vectors (lesson "La idea
 * diferencial"; glossary page: four small vectors, per-layer initial value):
 *     lambda_h = exp(lq1_h . lk1_h) - exp(lq2_h . lk2_h) + lambda_init(layer)
 * lq1, lk1, lq2, lk2 : device fp32 [n_heads, dim]
 * lambda_out         : device fp32 [n_heads]
 * Any real result is kept (lambda may be negative); no clamping.
 * Errors: DA_ERR_INVALID_ARG for null pointers, n_heads < 1, dim < 1 or
 * layer < 1. */
DA_API int lambda_from_params(const float* lq1, const float* lk1, const float* lq2,
                       const float* lk2, int n_heads, int dim, int layer,
                       float* lambda_out, void* stream);

/* V1 prefill (glossary page "Cómo funciona"; lesson "V1 vs V2").
 * Each head's 2*d_qk-wide query/key row is split into two halves: branch 1
 * uses columns [0, d_qk), branch 2 columns [d_qk, 2*d_qk).  V is d_v wide and
 * shared by both branches.  Optional per-head normalisation of each output
 * row (the page's "GroupNorm", an RMS norm over the d_v features):
 *     y_c = o_c / sqrt(mean_c(o_c^2) + norm_eps) * g_c * (1 - lambda_init)
 * q, k  : device [batch, seqlen, n_heads, 2*d_qk]
 * v     : device [batch, seqlen, n_heads, d_v]
 * out   : device [batch, seqlen, n_heads, d_v]
 * lambda: device fp32 [n_heads]
 * causal: nonzero -> query i sees keys j <= i (same for both branches)
 * apply_norm: nonzero -> apply the normalisation above; norm_weight is a
 *         device fp32 [d_v] gain or NULL for all-ones.  lambda_init is the
 *         value that sets the post-norm scale (1 - lambda_init).
 * Supported: fp32 with any d_qk <= 128, d_v <= 256 (CUDA-core kernel); bf16
 * with d_qk = 64, d_v = 128 on the tcgen05 tensor-core kernel, other bf16
 * widths up to the same limits on the CUDA-core kernel. */
DA_API int diffattn_v1_fwd(const void* q, const void* k, const void* v, void* out,
                    da_dtype dtype, int batch, int seqlen, int n_heads, int d_qk,
                    int d_v, const float* lambda, int causal, int apply_norm,
                    const float* norm_weight, float norm_eps, float lambda_init,
                    int* dev_status, void* stream);

/* V2 prefill (lesson "V1 vs V2": query heads doubled, KV heads kept, head
 * width kept, no per-head norm; "Ejercicios" 5: GQA).
 * Query heads come in subtracted pairs p = (2p, 2p+1), head 2p positive;
 * query head h reads KV head h / (n_q_heads / n_kv_heads), so both heads of a
 * pair share one KV head (n_q_heads / n_kv_heads must be even).
 * q     : device [batch, seqlen, n_q_heads, head_dim]
 * k, v  : device [batch, seqlen, n_kv_heads, head_dim]
 * out   : device [batch, seqlen, n_q_heads / 2, head_dim]
 * lambda: device fp32 [n_q_heads / 2]
 * Supported: bf16 head_dim = 128 on the tcgen05 kernel; fp32 (and other bf16
 * widths) with head_dim <= 128 on the CUDA-core kernel. */
DA_API int diffattn_v2_prefill(const void* q, const void* k, const void* v, void* out,
                        da_dtype dtype, int batch, int seqlen, int n_q_heads,
                        int n_kv_heads, int head_dim, const float* lambda,
                        int causal, int* dev_status, void* stream);

/* Bytes of device workspace diffattn_v2_decode needs for these sizes
 * (0 if it needs none).  Host only; never fails (returns 0 for bad sizes,
 * which the decode call then rejects). */
DA_API size_t diffattn_v2_decode_workspace_size(int batch, int n_q_heads, int n_kv_heads,
                                         int head_dim, int max_cache_len);

/* V2 single-token decode against a KV cache (lesson "V1 vs V2": the cache is
 * read once per step for both heads of every pair).  The new token's K/V
 * must already be in the cache: batch entry b attends cache rows
 * 0 .. cache_lens[b]-1.
 * q        : device [batch, n_q_heads, head_dim]
 * k_cache, v_cache : device [batch, max_len, n_kv_heads, head_dim]
 * cache_lens: device int32 [batch] with 1 <= cache_lens[b] <= max_len, or
 *            NULL (every entry uses max_len).  Values are not checked on the
 *            host; an out-of-range length is clamped on the device.
 * out      : device [batch, n_q_heads / 2, head_dim]
 * lambda   : device fp32 [n_q_heads / 2]
 * workspace: device, at least diffattn_v2_decode_workspace_size(...) bytes,
 *            16-byte aligned, caller-owned scratch (contents undefined
 *            after the call); NULL allowed only when that size is 0.
 * Supported: bf16 head_dim = 128 with (n_q_heads / n_kv_heads) in {2, 4, 6, 8}
 * on the split-KV tensor-core kernel; other shapes (and fp32) with
 * head_dim <= 128 on the CUDA-core kernel. */
DA_API int diffattn_v2_decode(const void* q, const void* k_cache, const void* v_cache,
                       const int* cache_lens, int max_len, void* out, da_dtype dtype,
                       int batch, int n_q_heads, int n_kv_heads, int head_dim,
                       const float* lambda, void* workspace, size_t workspace_bytes,
                       int* dev_status, void* stream);

/* Size of the fixed device scratch array behind diffattn_v2_decode_noalloc:
 * 8 MiB.  Every GPU on which that entry point runs keeps this array until the
 * process exits. */
#define DA_NOALLOC_SCRATCH_BYTES (8u << 20)

/* diffattn_v2_decode for callers that cannot allocate device memory.
 * The source pages have no counterpart to this entry point; it exists for
 * callers that are not able to hand over a workspace, e.g. code that must
 * never call cudaMalloc (an allocation can synchronise the device and stall
 * a serving loop), a plug-in whose host framework owns every device buffer,
 * or a runtime whose device-memory budget is fixed at start-up.
 * Same operator, arguments and layouts as diffattn_v2_decode with
 * dtype = DA_BF16 and head_dim = 128, minus the workspace: the split-KV
 * partial results go to a statically allocated device array of
 * DA_NOALLOC_SCRATCH_BYTES, and the call allocates nothing (no cudaMalloc,
 * no cudaFree, no allocating library routine).
 *  - Supported: n_q_heads / n_kv_heads in {2, 4, 6, 8}; otherwise
 *    DA_ERR_UNSUPPORTED.  Sizes whose partial results cannot fit in the
 *    scratch (batch * n_kv_heads above 2016) return DA_ERR_UNSUPPORTED
 *    before anything is enqueued.
 *  - Set-up: the first call on a device, with that device current, looks up
 *    the array's device address (cudaGetSymbolAddress) and caches it with
 *    the device's current CUDA context; make that first call before any
 *    stream capture.  A call under another context of that device (after
 *    cudaDeviceReset, or under a context made with the driver API) looks the
 *    address up again first, so make such a call outside capture too.
 *  - Every call on a device shares the one array, which keeps the last
 *    call's contents; nothing in it needs to start at zero.  Calls whose
 *    execution overlaps on the GPU (other streams, other host threads) race
 *    on the array: the caller must serialise them. */
DA_API int diffattn_v2_decode_noalloc(const void* q, const void* k_cache,
                                      const void* v_cache, const int* cache_lens,
                                      int max_len, void* out, int batch, int n_q_heads,
                                      int n_kv_heads, const float* lambda,
                                      int* dev_status, void* stream);

/* Bytes of device workspace diffattn_v1_decode needs (0 if none). */
DA_API size_t diffattn_v1_decode_workspace_size(int batch, int n_heads, int d_qk, int d_v,
                                         int max_cache_len);

/* V1 single-token decode against a multi-head cache (lesson "V1 vs V2").
 * Both branches read each cached value row once here.
 * q       : device [batch, n_heads, 2*d_qk]
 * k_cache : device [batch, max_len, n_heads, 2*d_qk]
 * v_cache : device [batch, max_len, n_heads, d_v]
 * out     : device [batch, n_heads, d_v]
 * Other arguments as for diffattn_v1_fwd and diffattn_v2_decode.
 * Supported: bf16 d_qk = 64, d_v = 128 on the TMA-fed split-KV kernel of
 * diffattn_v2_decode, where a head's two branches are a pair of query heads
 * (branch 1 scores on features 0..d_qk-1, branch 2 on the rest); other
 * widths (and fp32) with d_qk <= 128, d_v <= 256 on the CUDA-core kernel. */
DA_API int diffattn_v1_decode(const void* q, const void* k_cache, const void* v_cache,
                       const int* cache_lens, int max_len, void* out, da_dtype dtype,
                       int batch, int n_heads, int d_qk, int d_v, const float* lambda,
                       int apply_norm, const float* norm_weight, float norm_eps,
                       float lambda_init, void* workspace, size_t workspace_bytes,
                       int* dev_status, void* stream);

/* ---- Sliding-window variants ---------------------------------------------
 * The lesson "Atención Diferencial (V2)", section "Úselo", names models that
 * combine differential attention with sliding-window attention.  Reading:
 * with window W >= 1, query i sees only keys j with i - W < j <= i, in both
 * branches (prefill requires causal = 1), and a decode query sees the last
 * W of its len_b cache entries.  window = 0 is the unwindowed operator (the
 * functions above are these with window 0).  Every other argument, layout,
 * kernel choice and error is as for the function without "_window"; a
 * negative window, or window > 0 with causal = 0, is DA_ERR_INVALID_ARG.
 * The decode variants plan their cache splits over min(window, max_len)
 * entries, so their workspace is diffattn_v2_decode_workspace_size (or
 * diffattn_v1_decode_workspace_size) evaluated at that length. */
DA_API int diffattn_v1_fwd_window(const void* q, const void* k, const void* v, void* out,
                                  da_dtype dtype, int batch, int seqlen, int n_heads, int d_qk,
                                  int d_v, const float* lambda, int causal, int window,
                                  int apply_norm, const float* norm_weight, float norm_eps,
                                  float lambda_init, int* dev_status, void* stream);

DA_API int diffattn_v2_prefill_window(const void* q, const void* k, const void* v, void* out,
                                      da_dtype dtype, int batch, int seqlen, int n_q_heads,
                                      int n_kv_heads, int head_dim, const float* lambda,
                                      int causal, int window, int* dev_status, void* stream);

DA_API int diffattn_v2_decode_window(const void* q, const void* k_cache, const void* v_cache,
                                     const int* cache_lens, int max_len, int window, void* out,
                                     da_dtype dtype, int batch, int n_q_heads, int n_kv_heads,
                                     int head_dim, const float* lambda, void* workspace,
                                     size_t workspace_bytes, int* dev_status, void* stream);

DA_API int diffattn_v1_decode_window(const void* q, const void* k_cache, const void* v_cache,
                                     const int* cache_lens, int max_len, int window, void* out,
                                     da_dtype dtype, int batch, int n_heads, int d_qk, int d_v,
                                     const float* lambda, int apply_norm,
                                     const float* norm_weight, float norm_eps, float lambda_init,
                                     void* workspace, size_t workspace_bytes, int* dev_status,
                                     void* stream);

/* ---- Backward pass ---------------------------------------------------------
 * Gradients of a scalar loss L with respect to the inputs of the forward
 * above, given dout = dL/d(out).  The pages define the forward only (the
 * glossary page calls lambda learned, from four re-parameterised vectors);
 * these are the chain-rule gradients of that forward.  With causal masking
 * and an optional sliding window (window = 0: none; > 0 needs causal) as in
 * the forward.  bf16 inputs only (else DA_ERR_UNSUPPORTED); gradients are
 * fp32, written (not accumulated) in the layout of the matching input.
 * Outputs must not overlap inputs or each other.
 *
 * For widths outside the tensor-core forward the implementation
 * materialises the two attention maps of one head (V1) or head pair (V2)
 * for a chunk of batch entries at a time in `workspace` (size from the
 * *_workspace_size query; about 10 N^2 bytes per batch entry of a chunk)
 * and runs its six matrix products per branch as strided-batched GEMMs on
 * a CUDA-core kernel of this library (bf16 operands, fp32 accumulation).
 * Errors: as for the forward, plus DA_ERR_WORKSPACE for a missing or short
 * workspace.
 *
 * The shapes of the tensor-core forward (V1 d_qk 64 / d_v 128, V2 head_dim
 * 128) take a fused path instead: the forward kernel re-runs with saves
 * (per-row log-sum-exp and normalised branch outputs), then one kernel
 * accumulates dQ per query tile and one accumulates dK and dV per key tile
 * in tensor memory, recomputing the maps tile by tile; no N x N buffer
 * exists and the workspace is about 1.8 KB per token and head (V1) or head
 * pair (V2).  `dev_status` (optional) receives DA_ERR_DEVICE_TIMEOUT if
 * one of its bounded waits ever times out. */

/* V1.  q, k: device [batch, seqlen, n_heads, 2*d_qk]; v, dout: device
 * [batch, seqlen, n_heads, d_v] (bf16); lambda [n_heads] fp32; norm as in
 * diffattn_v1_fwd.  Outputs (device fp32): dq, dk like q; dv like v;
 * dlambda [n_heads] (summed over batch and rows); dnorm_weight [d_v]
 * (gradient of the norm gain, used only with apply_norm; may be NULL).
 * Supported: d_qk <= 256, d_v <= 128, seqlen^2 <= 2^31. */
DA_API size_t diffattn_v1_bwd_workspace_size(int batch, int seqlen, int n_heads, int d_qk,
                                             int d_v);
DA_API int diffattn_v1_bwd(const void* q, const void* k, const void* v, const void* dout,
                           const float* lambda, da_dtype dtype, int batch, int seqlen,
                           int n_heads, int d_qk, int d_v, int causal, int window,
                           int apply_norm, const float* norm_weight, float norm_eps,
                           float lambda_init, float* dq, float* dk, float* dv, float* dlambda,
                           float* dnorm_weight, void* workspace, size_t workspace_bytes,
                           int* dev_status, void* stream);

/* V2.  q: device [batch, seqlen, n_q_heads, head_dim]; k, v: device
 * [batch, seqlen, n_kv_heads, head_dim]; dout: device [batch, seqlen,
 * n_q_heads/2, head_dim] (bf16); lambda [n_q_heads/2] fp32.  Outputs
 * (device fp32): dq like q; dk, dv like k (summed over the pairs that share
 * a KV head); dlambda [n_q_heads/2].  Supported: head_dim <= 128. */
DA_API size_t diffattn_v2_bwd_workspace_size(int batch, int seqlen, int n_q_heads,
                                             int n_kv_heads, int head_dim);
DA_API int diffattn_v2_bwd(const void* q, const void* k, const void* v, const void* dout,
                           const float* lambda, da_dtype dtype, int batch, int seqlen,
                           int n_q_heads, int n_kv_heads, int head_dim, int causal, int window,
                           float* dq, float* dk, float* dv, float* dlambda, void* workspace,
                           size_t workspace_bytes, int* dev_status, void* stream);

/* ---- Training forward with saves, and the backward from the saves --------
 * A training step runs the forward once for its output and then the
 * backward.  diffattn_v1_bwd / diffattn_v2_bwd above take no forward state
 * and so run the training forward again internally.  These calls split that
 * work: the *_train forward writes the output exactly as diffattn_v1_fwd /
 * diffattn_v2_prefill_window do, plus the saves the backward reads; the
 * *_bwd_saved backward takes those saves and computes the same gradients as
 * diffattn_v1_bwd / diffattn_v2_bwd.  (The pages give the forward only; the
 * gradients are its chain rule, as above.)
 *  - Supported: bf16 with the tensor-core widths (V1 d_qk 64, d_v 128; V2
 *    head_dim 128); else DA_ERR_UNSUPPORTED.
 *  - saves: caller-owned device memory of at least the *_saves_size bytes
 *    (contents: per-row log2-sum-exp of each branch and each branch's
 *    normalised output O_r / l_r, both fp32; any alignment).  The backward must
 *    get the same q, k, v, lambda, causal, window and norm arguments as the
 *    forward that wrote the saves; the saves are only read by it.
 *  - workspace of the backward: at least the *_bwd_saved_workspace_size
 *    bytes, scratch (contents undefined after the call).
 *  - Errors as for the forward and backward above, plus DA_ERR_WORKSPACE for
 *    short saves or workspace. */
DA_API size_t diffattn_v1_fwd_train_saves_size(int batch, int seqlen, int n_heads);
DA_API int diffattn_v1_fwd_train(const void* q, const void* k, const void* v, void* out,
                                 da_dtype dtype, int batch, int seqlen, int n_heads, int d_qk,
                                 int d_v, const float* lambda, int causal, int window,
                                 int apply_norm, const float* norm_weight, float norm_eps,
                                 float lambda_init, void* saves, size_t saves_bytes,
                                 int* dev_status, void* stream);
DA_API size_t diffattn_v1_bwd_saved_workspace_size(int batch, int seqlen, int n_heads);
DA_API int diffattn_v1_bwd_saved(const void* q, const void* k, const void* v, const void* dout,
                                 const float* lambda, da_dtype dtype, int batch, int seqlen,
                                 int n_heads, int d_qk, int d_v, int causal, int window,
                                 int apply_norm, const float* norm_weight, float norm_eps,
                                 float lambda_init, const void* saves, size_t saves_bytes,
                                 float* dq, float* dk, float* dv, float* dlambda,
                                 float* dnorm_weight, void* workspace, size_t workspace_bytes,
                                 int* dev_status, void* stream);
DA_API size_t diffattn_v2_prefill_train_saves_size(int batch, int seqlen, int n_q_heads);
DA_API int diffattn_v2_prefill_train(const void* q, const void* k, const void* v, void* out,
                                     da_dtype dtype, int batch, int seqlen, int n_q_heads,
                                     int n_kv_heads, int head_dim, const float* lambda,
                                     int causal, int window, void* saves, size_t saves_bytes,
                                     int* dev_status, void* stream);
DA_API size_t diffattn_v2_bwd_saved_workspace_size(int batch, int seqlen, int n_q_heads);
DA_API int diffattn_v2_bwd_saved(const void* q, const void* k, const void* v, const void* dout,
                                 const float* lambda, da_dtype dtype, int batch, int seqlen,
                                 int n_q_heads, int n_kv_heads, int head_dim, int causal,
                                 int window, const void* saves, size_t saves_bytes, float* dq,
                                 float* dk, float* dv, float* dlambda, void* workspace,
                                 size_t workspace_bytes, int* dev_status, void* stream);

/* Gradients of the four lambda vectors (device fp32 [n_heads, dim]) of
 * lambda_from_params, from dlambda [n_heads]:
 *   dlq1 = dlambda e^{lq1.lk1} lk1,  dlk1 = dlambda e^{lq1.lk1} lq1,
 *   dlq2 = -dlambda e^{lq2.lk2} lk2, dlk2 = -dlambda e^{lq2.lk2} lq2. */
DA_API int lambda_from_params_bwd(const float* lq1, const float* lk1, const float* lq2,
                                  const float* lk2, const float* dlambda, int n_heads, int dim,
                                  float* dlq1, float* dlk1, float* dlq2, float* dlk2,
                                  void* stream);

/* ---- V2 prefill + output projection ---------------------------------------
 * Lesson "Atención Diferencial (V2)", "V1 vs V2: la diferencia" and step 5:
 * the paired subtraction brings V2's doubled query heads back to Hq/2 heads
 * of width head_dim, which then go through the output projection O_W.
 * out[b, i, :] = o[b, i, :, :].flatten() . w_o, with o the output of
 * diffattn_v2_prefill_window (same arguments) and
 *   w_o : device [n_q_heads/2 * head_dim, d_model] bf16 (row-major)
 *   out : device [batch, seqlen, d_model] bf16
 * The attention output goes to `workspace` (size from the query), then one
 * GEMM on the tcgen05 tensor cores (bf16 operands, fp32 accumulation, bf16
 * result) writes `out`.  bf16 only; d_model and n_q_heads/2 * head_dim must
 * be multiples of 8 (DA_ERR_UNSUPPORTED otherwise).  Errors as for
 * diffattn_v2_prefill_window, plus DA_ERR_WORKSPACE.  `dev_status` also
 * receives DA_ERR_DEVICE_TIMEOUT from the GEMM's bounded waits. */
DA_API size_t diffattn_v2_prefill_oproj_workspace_size(int batch, int seqlen, int n_q_heads,
                                                       int head_dim);
DA_API int diffattn_v2_prefill_oproj(const void* q, const void* k, const void* v,
                                     const float* lambda, const void* w_o, void* out,
                                     da_dtype dtype, int batch, int seqlen, int n_q_heads,
                                     int n_kv_heads, int head_dim, int d_model, int causal,
                                     int window, void* workspace, size_t workspace_bytes,
                                     int* dev_status, void* stream);

/* ---- Tile counters of the tensor-core prefill ------------------------------
 * No counterpart on the pages (they are this library's scheduling state).
 * diffattn_reset_tile_counters frees all 64 counters of the current device
 * by a one-thread kernel enqueued on `stream`.  It is meant for recovery
 * after a prefill launch reported DA_ERR_DEVICE_TIMEOUT (which can leave its
 * counter held); no tensor-core prefill launch may be in flight on the
 * device while it runs.  Returns DA_ERR_CUDA if the launch fails.
 *
 * diffattn_selftest_hold_tile_counter is a test hook: it enqueues a write of
 * (tag, count) into counter `slot` (0 .. 63) and makes the next tensor-core
 * prefill launch of this process take that counter.  With count > 0 and a
 * tag no launch has, the counter looks held by a launch that stopped: the
 * next launch takes it over after 250 ms.  With count = 0 it is free.
 * Returns DA_ERR_INVALID_ARG for a slot out of range. */
DA_API int diffattn_reset_tile_counters(void* stream);
DA_API int diffattn_selftest_hold_tile_counter(int slot, unsigned int tag, unsigned int count,
                                               void* stream);

/* Test hook: enqueues a one-thread kernel that keeps counter `slot` held by
 * `tag` with a count that changes every ~20 us (as a launch in flight would)
 * for `duration_ms` (1 .. 10000), then frees it; the next tensor-core
 * prefill launch of this process takes that counter.  A prefill launch that
 * runs meanwhile on another stream waits for it and, if it is still held
 * after 2 s, reports DA_ERR_SCHEDULE.  Returns DA_ERR_INVALID_ARG for a slot
 * or duration out of range. */
DA_API int diffattn_selftest_keep_tile_counter(int slot, unsigned int tag,
                                               unsigned int duration_ms, void* stream);

/* ---- Self-test of the failure report ----------------------------------------
 * No counterpart on the pages.  Launches one CTA whose thread waits on an
 * mbarrier that nothing arrives on, using the pipelines' own bounded wait
 * with a limit of `timeout_us` microseconds (1 .. 1000000).  The wait gives
 * up, stores DA_ERR_DEVICE_TIMEOUT in *dev_status (device int, required;
 * first error wins, zero it beforehand) and the kernel returns, leaving the
 * context usable.  `waited_ns` (optional, device) receives the time waited.
 * Returns DA_ERR_INVALID_ARG for a null status word or a limit out of range. */
DA_API int diffattn_selftest_wait_timeout(unsigned int timeout_us, int* dev_status,
                                          unsigned long long* waited_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DIFFATTN_H_ */
