// api.cu — the C ABI of libdiffattn.so (declared in include/diffattn.h).
//
// Host-side only: argument validation (before anything is enqueued),
// kernel selection by dtype and shape, TMA descriptor encoding and launches
// on the caller's stream.  Allocates nothing and keeps no mutable state
// beyond the lazily resolved driver entry point.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "diffattn.h"
#include "kernels.h"

namespace {

using da::GenericProblem;

// Split planning assumes a full B200 (148 SMs) so that the workspace size a
// caller queries does not depend on which device is current; the launch
// grid still uses the real SM count.
constexpr int kPlanSMs = 148;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 4-D bf16 tensor map over a dense [d3][d2][d1][d0] array (d0 fastest) with a
// 128-byte swizzle and zero fill outside the array.
int make_tmap_4d(CUtensorMap* tm, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                 uint64_t d3, uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return DA_ERR_CUDA;
  cuuint64_t dims[4] = {d0, d1, d2, d3};
  cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};
  cuuint32_t box[4] = {b0, b1, b2, b3};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DA_OK : DA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return n;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? DA_OK : DA_ERR_CUDA; }

bool dtype_ok(da_dtype t) { return t == DA_BF16 || t == DA_FP32; }

bool v2_decode_fast(int n_q_heads, int n_kv_heads, int head_dim) {
  const int group = n_q_heads / n_kv_heads;
  return head_dim == 128 && group >= 2 && group <= 8 && group % 2 == 0;
}

bool v1_decode_fast(int d_qk, int d_v) { return d_qk == 64 && d_v == 128; }

// Sizes of every tensor must fit the 32-bit token/row indices the kernels use.
bool fits_int(long long x) { return x > 0 && x < (1LL << 31); }

}  // namespace

namespace da {
int make_tmap_bf16_4d(CUtensorMap* tm, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                      uint64_t d3, uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  return make_tmap_4d(tm, base, d0, d1, d2, d3, b0, b1, b2, b3);
}
int make_tmap_f32_4d(CUtensorMap* tm, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                     uint64_t d3, uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return DA_ERR_CUDA;
  cuuint64_t dims[4] = {d0, d1, d2, d3};
  cuuint64_t strides[3] = {d0 * 4, d0 * d1 * 4, d0 * d1 * d2 * 4};
  cuuint32_t box[4] = {b0, b1, b2, b3};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(tm, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DA_OK : DA_ERR_CUDA;
}
}  // namespace da

extern "C" {

const char* diffattn_status_string(int status) {
  switch (status) {
    case DA_OK: return "DA_OK";
    case DA_ERR_INVALID_ARG: return "DA_ERR_INVALID_ARG";
    case DA_ERR_UNSUPPORTED: return "DA_ERR_UNSUPPORTED";
    case DA_ERR_ALIGNMENT: return "DA_ERR_ALIGNMENT";
    case DA_ERR_WORKSPACE: return "DA_ERR_WORKSPACE";
    case DA_ERR_CUDA: return "DA_ERR_CUDA";
    case DA_ERR_DEVICE_TIMEOUT: return "DA_ERR_DEVICE_TIMEOUT";
    case DA_ERR_SCHEDULE: return "DA_ERR_SCHEDULE";
    default: return "DA_ERR_UNKNOWN";
  }
}

int diffattn_reset_tile_counters(void* stream) {
  return cuda_status(da::reset_tile_counters(static_cast<cudaStream_t>(stream)));
}

int diffattn_selftest_hold_tile_counter(int slot, unsigned int tag, unsigned int count,
                                        void* stream) {
  if (slot < 0 || slot >= 64) return DA_ERR_INVALID_ARG;
  return cuda_status(da::hold_tile_counter(slot, tag, count, static_cast<cudaStream_t>(stream)));
}

int diffattn_selftest_keep_tile_counter(int slot, unsigned int tag, unsigned int duration_ms,
                                        void* stream) {
  if (slot < 0 || slot >= 64 || duration_ms < 1 || duration_ms > 10000) return DA_ERR_INVALID_ARG;
  return cuda_status(
      da::keep_tile_counter(slot, tag, duration_ms, static_cast<cudaStream_t>(stream)));
}

double diffattn_lambda_init(int layer) {
  if (layer < 1) return NAN;
  return 0.8 - 0.6 * std::exp(-0.3 * (double)(layer - 1));
}

int lambda_from_params(const float* lq1, const float* lk1, const float* lq2, const float* lk2,
                       int n_heads, int dim, int layer, float* lambda_out, void* stream) {
  if (!lq1 || !lk1 || !lq2 || !lk2 || !lambda_out) return DA_ERR_INVALID_ARG;
  if (n_heads < 1 || dim < 1 || layer < 1) return DA_ERR_INVALID_ARG;
  const float linit = (float)diffattn_lambda_init(layer);
  return cuda_status(da::launch_lambda(lq1, lk1, lq2, lk2, n_heads, dim, linit, lambda_out,
                                       static_cast<cudaStream_t>(stream)));
}

int diffattn_v1_fwd(const void* q, const void* k, const void* v, void* out, da_dtype dtype,
                    int batch, int seqlen, int n_heads, int d_qk, int d_v, const float* lambda,
                    int causal, int apply_norm, const float* norm_weight, float norm_eps,
                    float lambda_init, int* dev_status, void* stream) {
  return diffattn_v1_fwd_window(q, k, v, out, dtype, batch, seqlen, n_heads, d_qk, d_v, lambda,
                                causal, 0, apply_norm, norm_weight, norm_eps, lambda_init,
                                dev_status, stream);
}

int diffattn_v1_fwd_window(const void* q, const void* k, const void* v, void* out,
                           da_dtype dtype, int batch, int seqlen, int n_heads, int d_qk, int d_v,
                           const float* lambda, int causal, int window, int apply_norm,
                           const float* norm_weight, float norm_eps, float lambda_init,
                           int* dev_status, void* stream) {
  if (!q || !k || !v || !out || !lambda) return DA_ERR_INVALID_ARG;
  if (window < 0 || (window > 0 && !causal)) return DA_ERR_INVALID_ARG;
  if (!dtype_ok(dtype)) return DA_ERR_INVALID_ARG;
  if (batch < 1 || seqlen < 1 || n_heads < 1 || d_qk < 1 || d_v < 1) return DA_ERR_INVALID_ARG;
  if (apply_norm && !(norm_eps >= 0.f)) return DA_ERR_INVALID_ARG;
  if (!fits_int((long long)batch * seqlen) || !fits_int((long long)seqlen * n_heads * 2 * d_qk))
    return DA_ERR_UNSUPPORTED;
  if (d_qk > 128 || d_v > 256) return DA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return DA_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float post_scale = 1.0f - lambda_init;

  if (dtype == DA_BF16 && d_qk == 64 && d_v == 128) {
    const int sms = num_sms();
    if (sms < 1) return DA_ERR_CUDA;
    CUtensorMap tq, tk, tv;
    // [B][N][H][128] viewed as 4-D (c, h, n, b); 64-column boxes of 128 rows
    // Q: 128-row boxes (one query tile); K, V: 64-row boxes (one key tile)
    if (make_tmap_4d(&tq, q, 128, n_heads, seqlen, batch, 64, 1, 128, 1) ||
        make_tmap_4d(&tk, k, 128, n_heads, seqlen, batch, 64, 1, 64, 1) ||
        make_tmap_4d(&tv, v, 128, n_heads, seqlen, batch, 64, 1, 64, 1))
      return DA_ERR_CUDA;
    da::PrefillArgs a{};
    a.form = 1;
    a.batch = batch;
    a.seqlen = seqlen;
    a.heads = n_heads;
    a.kv_heads = n_heads;
    a.pairs_per_kv = 1;
    a.causal = causal ? 1 : 0;
    a.window = window;
    a.lambda = lambda;
    a.apply_norm = apply_norm ? 1 : 0;
    a.norm_weight = norm_weight;
    a.eps = norm_eps;
    a.post_scale = post_scale;
    a.out = out;
    a.dev_status = dev_status;
    return cuda_status(da::launch_prefill_tc(tq, tk, tv, a, sms, st));
  }

  GenericProblem P{};
  P.q = q;
  P.k = k;
  P.v = v;
  P.out = out;
  P.batch = batch;
  P.n_q = seqlen;
  P.heads = n_heads;
  P.d = d_qk;
  P.dv = d_v;
  P.q_tok = (int64_t)n_heads * 2 * d_qk;
  P.q_batch = P.q_tok * seqlen;
  P.k_tok = P.q_tok;
  P.k_batch = P.q_batch;
  P.k_head_stride = 2 * d_qk;
  P.k2_off = d_qk;
  P.v_tok = (int64_t)n_heads * d_v;
  P.v_batch = P.v_tok * seqlen;
  P.v_head_stride = d_v;
  P.kv_div = 1;
  P.o_tok = P.v_tok;
  P.o_batch = P.v_batch;
  P.n_keys = seqlen;
  P.causal = causal ? 1 : 0;
  P.window = window;
  P.lens = nullptr;
  P.lambda = lambda;
  P.apply_norm = apply_norm ? 1 : 0;
  P.norm_weight = norm_weight;
  P.eps = norm_eps;
  P.post_scale = post_scale;
  return cuda_status(da::launch_generic(P, dtype == DA_BF16, st));
}

int diffattn_v2_prefill(const void* q, const void* k, const void* v, void* out, da_dtype dtype,
                        int batch, int seqlen, int n_q_heads, int n_kv_heads, int head_dim,
                        const float* lambda, int causal, int* dev_status, void* stream) {
  return diffattn_v2_prefill_window(q, k, v, out, dtype, batch, seqlen, n_q_heads, n_kv_heads,
                                    head_dim, lambda, causal, 0, dev_status, stream);
}

int diffattn_v2_prefill_window(const void* q, const void* k, const void* v, void* out,
                               da_dtype dtype, int batch, int seqlen, int n_q_heads,
                               int n_kv_heads, int head_dim, const float* lambda, int causal,
                               int window, int* dev_status, void* stream) {
  if (!q || !k || !v || !out || !lambda) return DA_ERR_INVALID_ARG;
  if (window < 0 || (window > 0 && !causal)) return DA_ERR_INVALID_ARG;
  if (!dtype_ok(dtype)) return DA_ERR_INVALID_ARG;
  if (batch < 1 || seqlen < 1 || n_q_heads < 2 || n_kv_heads < 1 || head_dim < 1)
    return DA_ERR_INVALID_ARG;
  if (n_q_heads % n_kv_heads != 0 || (n_q_heads / n_kv_heads) % 2 != 0)
    return DA_ERR_INVALID_ARG;
  if (!fits_int((long long)batch * seqlen) || !fits_int((long long)seqlen * n_q_heads * head_dim))
    return DA_ERR_UNSUPPORTED;
  if (head_dim > 128) return DA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return DA_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int group = n_q_heads / n_kv_heads;

  if (dtype == DA_BF16 && head_dim == 128) {
    const int sms = num_sms();
    if (sms < 1) return DA_ERR_CUDA;
    CUtensorMap tq, tk, tv;
    if (make_tmap_4d(&tq, q, 128, n_q_heads, seqlen, batch, 64, 1, 128, 1) ||
        make_tmap_4d(&tk, k, 128, n_kv_heads, seqlen, batch, 64, 1, 64, 1) ||
        make_tmap_4d(&tv, v, 128, n_kv_heads, seqlen, batch, 64, 1, 64, 1))
      return DA_ERR_CUDA;
    da::PrefillArgs a{};
    a.form = 2;
    a.batch = batch;
    a.seqlen = seqlen;
    a.heads = n_q_heads / 2;
    a.kv_heads = n_kv_heads;
    a.pairs_per_kv = group / 2;
    a.causal = causal ? 1 : 0;
    a.window = window;
    a.lambda = lambda;
    a.apply_norm = 0;
    a.norm_weight = nullptr;
    a.eps = 0.f;
    a.post_scale = 1.f;
    a.out = out;
    a.dev_status = dev_status;
    return cuda_status(da::launch_prefill_tc(tq, tk, tv, a, sms, st));
  }

  GenericProblem P{};
  P.q = q;
  P.k = k;
  P.v = v;
  P.out = out;
  P.batch = batch;
  P.n_q = seqlen;
  P.heads = n_q_heads / 2;
  P.d = head_dim;
  P.dv = head_dim;
  P.q_tok = (int64_t)n_q_heads * head_dim;
  P.q_batch = P.q_tok * seqlen;
  P.k_tok = (int64_t)n_kv_heads * head_dim;
  P.k_batch = P.k_tok * seqlen;
  P.k_head_stride = head_dim;
  P.k2_off = 0;
  P.v_tok = P.k_tok;
  P.v_batch = P.k_batch;
  P.v_head_stride = head_dim;
  P.kv_div = group / 2;
  P.o_tok = (int64_t)(n_q_heads / 2) * head_dim;
  P.o_batch = P.o_tok * seqlen;
  P.n_keys = seqlen;
  P.causal = causal ? 1 : 0;
  P.window = window;
  P.lens = nullptr;
  P.lambda = lambda;
  P.apply_norm = 0;
  P.norm_weight = nullptr;
  P.eps = 0.f;
  P.post_scale = 1.f;
  return cuda_status(da::launch_generic(P, dtype == DA_BF16, st));
}

size_t diffattn_v2_decode_workspace_size(int batch, int n_q_heads, int n_kv_heads, int head_dim,
                                         int max_cache_len) {
  if (batch < 1 || n_q_heads < 2 || n_kv_heads < 1 || head_dim < 1 || max_cache_len < 1)
    return 0;
  if (n_q_heads % n_kv_heads != 0) return 0;
  if (!v2_decode_fast(n_q_heads, n_kv_heads, head_dim)) return 0;
  da::V2DecodePlan plan = da::plan_v2_decode(batch, n_kv_heads, max_cache_len, kPlanSMs);
  return da::v2_decode_workspace_bytes(plan);
}

int diffattn_v2_decode(const void* q, const void* k_cache, const void* v_cache,
                       const int* cache_lens, int max_len, void* out, da_dtype dtype, int batch,
                       int n_q_heads, int n_kv_heads, int head_dim, const float* lambda,
                       void* workspace, size_t workspace_bytes, int* dev_status, void* stream) {
  return diffattn_v2_decode_window(q, k_cache, v_cache, cache_lens, max_len, 0, out, dtype,
                                   batch, n_q_heads, n_kv_heads, head_dim, lambda, workspace,
                                   workspace_bytes, dev_status, stream);
}

int diffattn_v2_decode_window(const void* q, const void* k_cache, const void* v_cache,
                              const int* cache_lens, int max_len, int window, void* out,
                              da_dtype dtype, int batch, int n_q_heads, int n_kv_heads,
                              int head_dim, const float* lambda, void* workspace,
                              size_t workspace_bytes, int* dev_status, void* stream) {
  if (!q || !k_cache || !v_cache || !out || !lambda) return DA_ERR_INVALID_ARG;
  if (window < 0) return DA_ERR_INVALID_ARG;
  if (!dtype_ok(dtype)) return DA_ERR_INVALID_ARG;
  if (batch < 1 || max_len < 1 || n_q_heads < 2 || n_kv_heads < 1 || head_dim < 1)
    return DA_ERR_INVALID_ARG;
  if (n_q_heads % n_kv_heads != 0 || (n_q_heads / n_kv_heads) % 2 != 0)
    return DA_ERR_INVALID_ARG;
  if (!fits_int((long long)batch * max_len) ||
      !fits_int((long long)max_len * n_kv_heads * head_dim))
    return DA_ERR_UNSUPPORTED;
  if (head_dim > 128) return DA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return DA_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // a window bounds the entries one query reads: plan the splits over that many
  const int span = (window > 0 && window < max_len) ? window : max_len;

  if (dtype == DA_BF16 && v2_decode_fast(n_q_heads, n_kv_heads, head_dim)) {
    da::V2DecodePlan plan = da::plan_v2_decode(batch, n_kv_heads, span, kPlanSMs);
    const size_t need = da::v2_decode_workspace_bytes(plan);
    if (!workspace || workspace_bytes < need) return DA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return DA_ERR_ALIGNMENT;
    const int sms = num_sms();
    if (sms < 1) return DA_ERR_CUDA;
    plan.grid = plan.n_items < sms ? plan.n_items : sms;
    CUtensorMap tk, tv;
    if (make_tmap_4d(&tk, k_cache, 128, n_kv_heads, max_len, batch, 64, 1, 64, 1) ||
        make_tmap_4d(&tv, v_cache, 128, n_kv_heads, max_len, batch, 64, 1, 64, 1))
      return DA_ERR_CUDA;
    return cuda_status(da::launch_v2_decode(tk, tv, q, cache_lens, max_len, window, out, batch,
                                            n_q_heads, n_kv_heads, lambda, plan, workspace,
                                            dev_status, st));
  }

  GenericProblem P{};
  P.q = q;
  P.k = k_cache;
  P.v = v_cache;
  P.out = out;
  P.batch = batch;
  P.n_q = 1;
  P.heads = n_q_heads / 2;
  P.d = head_dim;
  P.dv = head_dim;
  P.q_tok = 0;
  P.q_batch = (int64_t)n_q_heads * head_dim;
  P.k_tok = (int64_t)n_kv_heads * head_dim;
  P.k_batch = P.k_tok * max_len;
  P.k_head_stride = head_dim;
  P.k2_off = 0;
  P.v_tok = P.k_tok;
  P.v_batch = P.k_batch;
  P.v_head_stride = head_dim;
  P.kv_div = (n_q_heads / n_kv_heads) / 2;
  P.o_tok = 0;
  P.o_batch = (int64_t)(n_q_heads / 2) * head_dim;
  P.n_keys = max_len;
  P.causal = 0;
  P.window = window;
  P.lens = cache_lens;
  P.lambda = lambda;
  P.apply_norm = 0;
  P.norm_weight = nullptr;
  P.eps = 0.f;
  P.post_scale = 1.f;
  return cuda_status(da::launch_generic(P, dtype == DA_BF16, st));
}

size_t diffattn_v1_decode_workspace_size(int batch, int n_heads, int d_qk, int d_v,
                                         int max_cache_len) {
  if (batch < 1 || n_heads < 1 || d_qk < 1 || d_v < 1 || max_cache_len < 1) return 0;
  if (!v1_decode_fast(d_qk, d_v)) return 0;
  // the V1 fast path runs on the split-KV tensor-core kernel, one KV head per head
  da::V2DecodePlan plan = da::plan_v2_decode(batch, n_heads, max_cache_len, kPlanSMs);
  return da::v2_decode_workspace_bytes(plan);
}

int diffattn_v1_decode(const void* q, const void* k_cache, const void* v_cache,
                       const int* cache_lens, int max_len, void* out, da_dtype dtype, int batch,
                       int n_heads, int d_qk, int d_v, const float* lambda, int apply_norm,
                       const float* norm_weight, float norm_eps, float lambda_init,
                       void* workspace, size_t workspace_bytes, int* dev_status, void* stream) {
  return diffattn_v1_decode_window(q, k_cache, v_cache, cache_lens, max_len, 0, out, dtype,
                                   batch, n_heads, d_qk, d_v, lambda, apply_norm, norm_weight,
                                   norm_eps, lambda_init, workspace, workspace_bytes, dev_status,
                                   stream);
}

int diffattn_v1_decode_window(const void* q, const void* k_cache, const void* v_cache,
                              const int* cache_lens, int max_len, int window, void* out,
                              da_dtype dtype, int batch, int n_heads, int d_qk, int d_v,
                              const float* lambda, int apply_norm, const float* norm_weight,
                              float norm_eps, float lambda_init, void* workspace,
                              size_t workspace_bytes, int* dev_status, void* stream) {
  if (!q || !k_cache || !v_cache || !out || !lambda) return DA_ERR_INVALID_ARG;
  if (window < 0) return DA_ERR_INVALID_ARG;
  if (!dtype_ok(dtype)) return DA_ERR_INVALID_ARG;
  if (batch < 1 || max_len < 1 || n_heads < 1 || d_qk < 1 || d_v < 1) return DA_ERR_INVALID_ARG;
  if (apply_norm && !(norm_eps >= 0.f)) return DA_ERR_INVALID_ARG;
  if (!fits_int((long long)batch * max_len) || !fits_int((long long)max_len * n_heads * 2 * d_qk))
    return DA_ERR_UNSUPPORTED;
  if (d_qk > 128 || d_v > 256) return DA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
    return DA_ERR_ALIGNMENT;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float post_scale = 1.0f - lambda_init;

  const int span = (window > 0 && window < max_len) ? window : max_len;

  if (dtype == DA_BF16 && v1_decode_fast(d_qk, d_v)) {
    // Each head's K row is [branch 1 | branch 2] (64 + 64) and its V row is
    // 128 wide, so the split-KV tensor-core kernel of V2 serves it with the
    // head as a KV head and its two branches as a pair of query heads.
    da::V2DecodePlan plan = da::plan_v2_decode(batch, n_heads, span, kPlanSMs);
    const size_t need = da::v2_decode_workspace_bytes(plan);
    if (!workspace || workspace_bytes < need) return DA_ERR_WORKSPACE;
    if (!aligned16(workspace)) return DA_ERR_ALIGNMENT;
    const int sms = num_sms();
    if (sms < 1) return DA_ERR_CUDA;
    plan.grid = plan.n_items < sms ? plan.n_items : sms;
    CUtensorMap tk, tv;
    if (make_tmap_4d(&tk, k_cache, 128, n_heads, max_len, batch, 64, 1, 64, 1) ||
        make_tmap_4d(&tv, v_cache, 128, n_heads, max_len, batch, 64, 1, 64, 1))
      return DA_ERR_CUDA;
    return cuda_status(da::launch_v1_decode_tc(tk, tv, q, cache_lens, max_len, window, out,
                                               batch, n_heads, lambda, apply_norm ? 1 : 0,
                                               norm_weight, norm_eps, post_scale, plan, workspace,
                                               dev_status, st));
  }

  GenericProblem P{};
  P.q = q;
  P.k = k_cache;
  P.v = v_cache;
  P.out = out;
  P.batch = batch;
  P.n_q = 1;
  P.heads = n_heads;
  P.d = d_qk;
  P.dv = d_v;
  P.q_tok = 0;
  P.q_batch = (int64_t)n_heads * 2 * d_qk;
  P.k_tok = (int64_t)n_heads * 2 * d_qk;
  P.k_batch = P.k_tok * max_len;
  P.k_head_stride = 2 * d_qk;
  P.k2_off = d_qk;
  P.v_tok = (int64_t)n_heads * d_v;
  P.v_batch = P.v_tok * max_len;
  P.v_head_stride = d_v;
  P.kv_div = 1;
  P.o_tok = 0;
  P.o_batch = (int64_t)n_heads * d_v;
  P.n_keys = max_len;
  P.causal = 0;
  P.window = window;
  P.lens = cache_lens;
  P.lambda = lambda;
  P.apply_norm = apply_norm ? 1 : 0;
  P.norm_weight = norm_weight;
  P.eps = norm_eps;
  P.post_scale = post_scale;
  return cuda_status(da::launch_generic(P, dtype == DA_BF16, st));
}

}  // extern "C"
