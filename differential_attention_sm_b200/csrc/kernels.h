// kernels.h — internal launch interfaces between the C-ABI layer (api.cu)
// and the kernels.  Not installed; the public interface is diffattn.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace da {

// Addressing of the generic (CUDA-core) kernel; all strides in elements.
struct GenericProblem {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  int batch, n_q, heads;  // output rows = batch * n_q * heads
  int d, dv;
  int64_t q_batch, q_tok;
  int64_t k_batch, k_tok;
  int k_head_stride, k2_off;
  int64_t v_batch, v_tok;
  int v_head_stride;
  int kv_div;  // key/value head = output head / kv_div
  int64_t o_batch, o_tok;
  int n_keys;       // keys per sequence (prefill N, decode max_len)
  int causal;       // prefill: query i sees keys <= i
  int window;       // > 0: only the last `window` of those keys (prefill and decode)
  const int* lens;  // decode: per-batch valid cache rows, or nullptr
  const float* lambda;
  int apply_norm;
  const float* norm_weight;
  float eps, post_scale;
};

cudaError_t launch_lambda(const float* lq1, const float* lk1, const float* lq2, const float* lk2,
                          int n_heads, int dim, float lambda_init, float* out,
                          cudaStream_t stream);

cudaError_t launch_generic(const GenericProblem& P, bool bf16, cudaStream_t stream);

// ---- V2 split-KV decode (bf16, head_dim 128, group <= 8) ------------------
struct V2DecodePlan {
  int n_split;    // splits per (batch, kv head)
  int split_len;  // tokens per split (multiple of 64)
  int n_items;    // batch * n_kv_heads * n_split
  int grid;       // persistent CTAs
};
V2DecodePlan plan_v2_decode(int batch, int n_kv_heads, int max_len, int num_sms);
// Same search restricted to plans whose workspace fits in max_bytes; returns
// a plan with n_items == 0 if none does.
V2DecodePlan plan_v2_decode_capped(int batch, int n_kv_heads, int max_len, int num_sms,
                                   size_t max_bytes);
size_t v2_decode_workspace_bytes(const V2DecodePlan& plan);
cudaError_t launch_v2_decode(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const void* q,
                             const int* lens, int max_len, int window, void* out, int batch,
                             int n_q_heads, int n_kv_heads, const float* lambda,
                             const V2DecodePlan& plan,
                             void* workspace, int* dev_status, cudaStream_t stream);

// V1 decode (bf16, d_qk 64, d_v 128) on the same split kernel: each head is a
// KV head whose two branches are a pair (query features split by halves);
// the combine applies -lambda, the per-head norm and the post scale.  The
// workspace is v2_decode_workspace_bytes of plan_v2_decode(batch, n_heads, ...).
cudaError_t launch_v1_decode_tc(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const void* q,
                                const int* lens, int max_len, int window, void* out, int batch,
                                int n_heads, const float* lambda, int apply_norm,
                                const float* norm_weight, float eps, float post_scale,
                                const V2DecodePlan& plan, void* workspace, int* dev_status,
                                cudaStream_t stream);

// 4-D bf16 tensor map (128-byte swizzle, zero fill) over a dense
// [d3][d2][d1][d0] array; returns a da_status.  Implemented in api.cu.
int make_tmap_bf16_4d(CUtensorMap* tm, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                      uint64_t d3, uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3);
// The same over fp32 elements, without swizzle (boxes of 32-byte rows).
int make_tmap_f32_4d(CUtensorMap* tm, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                     uint64_t d3, uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3);

// ---- tcgen05 prefill (bf16) -----------------------------------------------
// Form 1 (V1): Q/K rows are 128 wide (two 64-wide branches), V 128 wide,
//              one KV head per head, optional RMS norm.
// Form 2 (V2): query heads 2p, 2p+1 (128 wide each) against KV head
//              2p / group, no norm.
struct PrefillArgs {
  int form;  // 1 or 2
  int batch, seqlen;
  int heads;     // V1: heads; V2: pairs (n_q_heads / 2)
  int kv_heads;  // V1: heads; V2: n_kv_heads
  int pairs_per_kv;  // V2: group / 2; V1: 1
  int causal;
  int window;  // > 0 (causal only): row i sees keys (i - window, i]
  const float* lambda;
  int apply_norm;
  const float* norm_weight;
  float eps, post_scale;
  void* out;
  float* lse;  // optional training saves (see the kernel's Params)
  int lse_stride;
  void* obr;
  int* dev_status;
};
cudaError_t launch_prefill_tc(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                              const CUtensorMap& tm_v, const PrefillArgs& a, int num_sms,
                              cudaStream_t stream);
// Tile counters of the tensor-core prefill (64 per device): free them all, or
// set one to (tag, count) and make the next launch of this process take it.
cudaError_t reset_tile_counters(cudaStream_t stream);
cudaError_t hold_tile_counter(int slot, unsigned tag, unsigned count, cudaStream_t stream);
cudaError_t keep_tile_counter(int slot, unsigned tag, unsigned duration_ms, cudaStream_t stream);

// ---- tcgen05 bf16 GEMM (row-major C[M][N] = A[M][K] . B[K][N]) -------------
// K and N multiples of 8, base addresses 16-byte aligned (TMA).
int gemm_bf16_tc_smem_bytes();
cudaError_t launch_gemm_bf16_tc(const void* a, const void* b, void* c, int M, int N, int K,
                                int num_sms, int* dev_status, cudaStream_t stream);

// ---- fused tcgen05 backward (bf16; V1 d_qk 64 / d_v 128, V2 head_dim 128) --
struct FusedBwdArgs {
  PrefillArgs fwd;  // the forward's problem (out/lse/obr are set internally)
  const void* q;
  const void* k;
  const void* v;
  const void* dout;  // [B][N][units][128] bf16
  float* dq;
  float* dk;
  float* dv;
  float* dlambda;    // [units]
  float* dg;         // [128] or nullptr
  void* workspace;   // fused_bwd_workspace_bytes
  int num_sms;
};
size_t fused_bwd_workspace_bytes(int batch, int seqlen, int units);
cudaError_t launch_fused_bwd(const FusedBwdArgs& a, cudaStream_t stream);
// The same split in two: the training forward (the prefill kernel writing
// `out` and the saves) and the backward from those saves (a.workspace holds
// saved_bwd_workspace_bytes).  units = heads (V1) or pairs (V2).
size_t train_saves_bytes(int batch, int seqlen, int units);
size_t saved_bwd_workspace_bytes(int batch, int seqlen, int units);
cudaError_t launch_fwd_train(const PrefillArgs& fwd, const void* q, const void* k,
                             const void* v, void* out, void* saves, int num_sms,
                             cudaStream_t stream);
cudaError_t launch_bwd_from_saves(const FusedBwdArgs& a, const void* saves,
                                  cudaStream_t stream);

}  // namespace da
