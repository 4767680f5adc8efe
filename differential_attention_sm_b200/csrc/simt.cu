// simt.cu — CUDA-core kernels: lambda re-parameterisation and the generic
// differential-attention kernel (one warp per output row) that serves fp32
// inputs and every shape the tensor-core kernels do not cover.
//
// Operator: "Differential Transformer" (Ultralytics glossary), section
// "Cómo funciona la atención diferencial"; lesson "Atención Diferencial (V2)"
// (ai-engineering.academy), sections "La idea diferencial" and
// "Implementación" steps 1-3.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "kernels.h"

namespace da {

// ---------------------------------------------------------------------------
// lambda_h = exp(lq1_h . lk1_h) - exp(lq2_h . lk2_h) + lambda_init
// (lesson, "La idea diferencial"; glossary: four small vectors per head).
// One warp per head.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) lambda_kernel(const float* __restrict__ lq1,
                                                     const float* __restrict__ lk1,
                                                     const float* __restrict__ lq2,
                                                     const float* __restrict__ lk2, int n_heads,
                                                     int dim, float lambda_init,
                                                     float* __restrict__ out) {
  const int h = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (h >= n_heads) return;
  float d1 = 0.f, d2 = 0.f;
  for (int c = lane; c < dim; c += 32) {
    const size_t o = (size_t)h * dim + c;
    d1 = fmaf(lq1[o], lk1[o], d1);
    d2 = fmaf(lq2[o], lk2[o], d2);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    d1 += __shfl_xor_sync(0xffffffffu, d1, off);
    d2 += __shfl_xor_sync(0xffffffffu, d2, off);
  }
  if (lane == 0) out[h] = expf(d1) - expf(d2) + lambda_init;
}

cudaError_t launch_lambda(const float* lq1, const float* lk1, const float* lq2, const float* lk2,
                          int n_heads, int dim, float lambda_init, float* out,
                          cudaStream_t stream) {
  const int warps = 4;
  dim3 grid((n_heads + warps - 1) / warps);
  lambda_kernel<<<grid, 32 * warps, 0, stream>>>(lq1, lk1, lq2, lk2, n_heads, dim, lambda_init,
                                                out);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Generic kernel.  Output row (b, i, h): branch-1 query at q + h*2d, branch-2
// query at q + h*2d + d (for V2 the pair's two heads are adjacent, so the same
// addressing holds), key/value head kvh = h / kv_div, branch-2 keys at
// k + kvh*k_head_stride + k2_off.  Three passes over the keys (row maxima,
// row sums, weighted value sum) keep every quantity exact in fp32 without
// staging a score row.
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ float ld(const T* p);
template <>
__device__ __forceinline__ float ld<float>(const float* p) {
  return __ldg(p);
}
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}
template <typename T>
__device__ __forceinline__ void st(T* p, float v);
template <>
__device__ __forceinline__ void st<float>(float* p, float v) {
  *p = v;
}
template <>
__device__ __forceinline__ void st<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

constexpr int GEN_WARPS = 4;
constexpr int GEN_MAX_D = 128;
constexpr int GEN_MAX_DV = 256;

template <typename T>
__global__ void __launch_bounds__(32 * GEN_WARPS) generic_kernel(GenericProblem P) {
  __shared__ float qs[GEN_WARPS][2][GEN_MAX_D];
  const int wib = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * GEN_WARPS + wib;
  const int64_t total = (int64_t)P.batch * P.n_q * P.heads;
  if (row >= total) return;
  const int h = (int)(row % P.heads);
  const int64_t bi = row / P.heads;
  const int i = (int)(bi % P.n_q);
  const int b = (int)(bi / P.n_q);

  const T* q = static_cast<const T*>(P.q) + b * P.q_batch + i * P.q_tok + (int64_t)h * 2 * P.d;
  const int kvh = h / P.kv_div;
  const T* k1 = static_cast<const T*>(P.k) + b * P.k_batch + (int64_t)kvh * P.k_head_stride;
  const T* k2 = k1 + P.k2_off;
  const T* vb = static_cast<const T*>(P.v) + b * P.v_batch + (int64_t)kvh * P.v_head_stride;

  int n_keys;
  if (P.lens) {
    n_keys = P.lens[b];
    n_keys = n_keys < 1 ? 1 : (n_keys > P.n_keys ? P.n_keys : n_keys);
  } else {
    n_keys = P.causal ? i + 1 : P.n_keys;
  }
  // sliding window: only the last `window` of the visible keys
  const int key0 = (P.window > 0 && n_keys > P.window) ? n_keys - P.window : 0;

  for (int c = lane; c < P.d; c += 32) {
    qs[wib][0][c] = ld(q + c);
    qs[wib][1][c] = ld(q + P.d + c);
  }
  __syncwarp();
  const float scale = 1.0f / sqrtf((float)P.d);
  const float lam = P.lambda[h];

  auto scores = [&](int j, float& s1, float& s2) {
    const T* a = k1 + (int64_t)j * P.k_tok;
    const T* c2 = k2 + (int64_t)j * P.k_tok;
    float x1 = 0.f, x2 = 0.f;
    for (int c = 0; c < P.d; ++c) {
      x1 = fmaf(qs[wib][0][c], ld(a + c), x1);
      x2 = fmaf(qs[wib][1][c], ld(c2 + c), x2);
    }
    s1 = x1 * scale;
    s2 = x2 * scale;
  };

  // pass 1: row maxima of both score rows
  float m1 = -INFINITY, m2 = -INFINITY;
  for (int j = key0 + lane; j < n_keys; j += 32) {
    float s1, s2;
    scores(j, s1, s2);
    m1 = fmaxf(m1, s1);
    m2 = fmaxf(m2, s2);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, off));
    m2 = fmaxf(m2, __shfl_xor_sync(0xffffffffu, m2, off));
  }
  // pass 2: softmax denominators
  float l1 = 0.f, l2 = 0.f;
  for (int j = key0 + lane; j < n_keys; j += 32) {
    float s1, s2;
    scores(j, s1, s2);
    l1 += expf(s1 - m1);
    l2 += expf(s2 - m2);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    l2 += __shfl_xor_sync(0xffffffffu, l2, off);
  }
  const float inv1 = 1.0f / l1, inv2 = lam / l2;
  // pass 3: o_c = sum_j (a1_j - lambda a2_j) v_j[c]; lane owns c = lane + 32t
  float acc[GEN_MAX_DV / 32];
#pragma unroll
  for (int t = 0; t < GEN_MAX_DV / 32; ++t) acc[t] = 0.f;
  for (int j0 = key0; j0 < n_keys; j0 += 32) {
    const int j = j0 + lane;
    float w = 0.f;
    if (j < n_keys) {
      float s1, s2;
      scores(j, s1, s2);
      w = expf(s1 - m1) * inv1 - expf(s2 - m2) * inv2;
    }
    const int cnt = min(32, n_keys - j0);
    for (int jj = 0; jj < cnt; ++jj) {
      const float wj = __shfl_sync(0xffffffffu, w, jj);
      const T* vr = vb + (int64_t)(j0 + jj) * P.v_tok;
#pragma unroll
      for (int t = 0; t < GEN_MAX_DV / 32; ++t) {
        const int c = lane + 32 * t;
        if (c < P.dv) acc[t] = fmaf(wj, ld(vr + c), acc[t]);
      }
    }
  }
  // optional per-head RMS normalisation, then the (1 - lambda_init) scale
  float mul = 1.0f;
  if (P.apply_norm) {
    float ss = 0.f;
#pragma unroll
    for (int t = 0; t < GEN_MAX_DV / 32; ++t) ss = fmaf(acc[t], acc[t], ss);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    mul = P.post_scale / sqrtf(ss / (float)P.dv + P.eps);
  }
  T* o = static_cast<T*>(P.out) + b * P.o_batch + i * P.o_tok + (int64_t)h * P.dv;
#pragma unroll
  for (int t = 0; t < GEN_MAX_DV / 32; ++t) {
    const int c = lane + 32 * t;
    if (c < P.dv) {
      const float g = (P.apply_norm && P.norm_weight) ? P.norm_weight[c] : 1.0f;
      st(o + c, acc[t] * mul * g);
    }
  }
}

cudaError_t launch_generic(const GenericProblem& P, bool bf16, cudaStream_t stream) {
  const int64_t total = (int64_t)P.batch * P.n_q * P.heads;
  if (total <= 0) return cudaSuccess;
  dim3 grid((unsigned)((total + GEN_WARPS - 1) / GEN_WARPS));
  if (bf16)
    generic_kernel<__nv_bfloat16><<<grid, 32 * GEN_WARPS, 0, stream>>>(P);
  else
    generic_kernel<float><<<grid, 32 * GEN_WARPS, 0, stream>>>(P);
  return cudaGetLastError();
}

}  // namespace da
