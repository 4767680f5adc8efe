// oproj.cu — V2 prefill followed by the output projection.
//
// Lesson "Atención Diferencial (V2)", section "V1 vs V2: la diferencia" /
// step 5: V2 doubles the query heads, the paired subtraction brings the
// width back to Hq/2 heads x d, and the result then goes through O_W.
// This entry point runs the differential-attention prefill into a
// workspace and multiplies the [B*N, Hq/2*d] result by O_W [Hq/2*d, d_model]
// with the library's tcgen05 GEMM (gemm_tc.cu: bf16 operands, fp32
// accumulation, bf16 output).  A fused epilogue would need every one of a
// row's Hq/2 head pairs in one CTA, or cross-CTA reductions of Hq/2 partial
// products per output element; the separate GEMM reads the
// 2 x B x N x Hq/2 x d bytes of the finished attention output once, which
// on this part costs far less.
#include <cuda_runtime.h>

#include <cstdint>

#include "diffattn.h"
#include "kernels.h"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

size_t diffattn_v2_prefill_oproj_workspace_size(int batch, int seqlen, int n_q_heads,
                                                int head_dim) {
  if (batch < 1 || seqlen < 1 || n_q_heads < 2 || head_dim < 1) return 0;
  return (size_t)batch * seqlen * (n_q_heads / 2) * head_dim * 2 + 256;
}

int diffattn_v2_prefill_oproj(const void* q, const void* k, const void* v, const float* lambda,
                              const void* w_o, void* out, da_dtype dtype, int batch, int seqlen,
                              int n_q_heads, int n_kv_heads, int head_dim, int d_model,
                              int causal, int window, void* workspace, size_t workspace_bytes,
                              int* dev_status, void* stream) {
  if (!q || !k || !v || !lambda || !w_o || !out) return DA_ERR_INVALID_ARG;
  if (d_model < 1 || batch < 1 || seqlen < 1 || n_q_heads < 2 || head_dim < 1)
    return DA_ERR_INVALID_ARG;
  if (dtype != DA_BF16) return DA_ERR_UNSUPPORTED;
  const long long rows = (long long)batch * seqlen;
  const long long kdim = (long long)(n_q_heads / 2) * head_dim;
  // the GEMM's TMA row pitches must be multiples of 16 bytes
  if (d_model % 8 != 0 || kdim % 8 != 0) return DA_ERR_UNSUPPORTED;
  if (rows > 0x7fffffffLL || kdim > 0x7fffffffLL) return DA_ERR_UNSUPPORTED;
  if (!aligned16(w_o) || !aligned16(out)) return DA_ERR_ALIGNMENT;
  const size_t need = diffattn_v2_prefill_oproj_workspace_size(batch, seqlen, n_q_heads, head_dim);
  if (!workspace || workspace_bytes < need) return DA_ERR_WORKSPACE;
  void* o = reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(workspace) + 255) &
                                    ~uintptr_t(255));
  int st = diffattn_v2_prefill_window(q, k, v, o, dtype, batch, seqlen, n_q_heads, n_kv_heads,
                                      head_dim, lambda, causal, window, dev_status, stream);
  if (st != DA_OK) return st;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return DA_ERR_CUDA;
  // row-major out[rows x d_model] = o[rows x kdim] . W_o[kdim x d_model]
  cudaError_t e = da::launch_gemm_bf16_tc(o, w_o, out, (int)rows, d_model, (int)kdim, sms,
                                          dev_status, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? DA_OK : DA_ERR_CUDA;
}

}  // extern "C"
