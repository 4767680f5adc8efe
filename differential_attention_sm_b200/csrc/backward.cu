// backward.cu — gradients of differential attention (both forms).
//
// Forward: glossary page "Differential Transformer", section "Cómo funciona
// la atención diferencial"; lesson "Atención Diferencial (V2)", sections "La
// idea diferencial" and "V1 vs V2: la diferencia".  lambda is learned (the
// glossary page re-parameterises it by four vectors), so its gradient and,
// in V1, that of the per-head norm gain are produced too.
//
// The general implementation materialises the two attention maps of one head
// (V1) or head pair (V2) for a chunk of batch entries at a time:
//   for each branch r:  S_r = Q_r K_r^T / sqrt(d)           (GEMM)
//                       P_r = masked softmax(S_r)            (kernel, bf16)
//                       O_r = P_r V                          (GEMM)
//   o = O_1 - lambda O_2;  V1: y = RMSNorm(o) g (1 - lambda_init)
//   do (through the norm), dlambda = -sum do . O_2,  D_r = do_r . O_r   (kernel)
//   for each branch r, with do_1 = do and do_2 = -lambda do:
//                       dP_r = do_r V^T                      (GEMM)
//                       dS_r = P_r (dP_r - D_r)              (kernel, bf16)
//                       dQ_r = dS_r K_r / sqrt(d)            (GEMM)
//                       dK_r += dS_r^T Q_r / sqrt(d)         (GEMM)
//                       dV  += P_r^T do_r                    (GEMM)
// The six products are strided-batched GEMMs (bf16 operands, fp32
// accumulation) on a CUDA-core kernel of this file; every other step is a
// kernel here too.  This path only serves the widths the fused tensor-core
// backward (backward_tc.cu) does not cover.  The masked-out part of each map
// is zero, so the GEMMs run over the full N x N square (twice the causal
// work).  Gradients are written in fp32.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <initializer_list>

#include "diffattn.h"
#include "kernels.h"

namespace da {
namespace {

constexpr size_t kChunkCap = size_t(4) << 30;  // workspace bound per chunk of batch entries
constexpr int kMaxDv = 128;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
  return x;
}

// Visible keys of query row i: [first, last] (causal, optional window) or all.
__device__ __forceinline__ void visible(int i, int N, int causal, int window, int& first,
                                        int& last) {
  last = causal ? i : N - 1;
  first = (window > 0 && last + 1 > window) ? last + 1 - window : 0;
}

// P = softmax over the visible keys of each row of S (fp32, already scaled);
// zero elsewhere.  One warp per row; rows of `units` N x N blocks.
__global__ void bwd_softmax_kernel(const float* __restrict__ S, __nv_bfloat16* __restrict__ P,
                                   int N, int units, int causal, int window) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= (long long)units * N) return;
  const int i = (int)(row % N);
  const float* s = S + row * N;
  __nv_bfloat16* p = P + row * N;
  int first, last;
  visible(i, N, causal, window, first, last);
  float m = -INFINITY;
  for (int j = first + lane; j <= last; j += 32) m = fmaxf(m, s[j]);
  m = warp_max(m);
  float l = 0.f;
  for (int j = first + lane; j <= last; j += 32) l += __expf(s[j] - m);
  l = warp_sum(l);
  const float inv = 1.0f / l;
  for (int j = lane; j < N; j += 32) {
    const float v = (j >= first && j <= last) ? __expf(s[j] - m) * inv : 0.f;
    p[j] = __float2bfloat16_rn(v);
  }
}

// dS = P (dP - D_row), bf16.  One warp per row.
__global__ void bwd_ds_kernel(const __nv_bfloat16* __restrict__ P, const float* __restrict__ dP,
                              const float* __restrict__ D, __nv_bfloat16* __restrict__ dS, int N,
                              int units) {
  const long long row = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (row >= (long long)units * N) return;
  const float dr = D[row];
  const __nv_bfloat16* p = P + row * N;
  const float* dp = dP + row * N;
  __nv_bfloat16* ds = dS + row * N;
  for (int j = lane; j < N; j += 32)
    ds[j] = __float2bfloat16_rn(__bfloat162float(p[j]) * (dp[j] - dr));
}

// Per row: o = O1 - lambda O2, the norm backward (V1), do_1 = do and
// do_2 = -lambda do (bf16), D_r = do_r . O_r, and the block's share of
// dlambda = -sum do . O2 and of the norm gain's gradient.  Block: 8 warps,
// kRowsPerBlock rows; grid (row blocks, units).
constexpr int kPreWarps = 8;
constexpr int kRowsPerBlock = 64;

struct PreArgs {
  const float* O1;  // [units][N][dv]
  const float* O2;
  const __nv_bfloat16* dout;  // row i of unit u at dout + u * dout_unit + i * dout_row
  long long dout_unit, dout_row;
  __nv_bfloat16* do1;  // [units][N][dv]
  __nv_bfloat16* do2;
  float* D1;  // [units][N]
  float* D2;
  int N, dv;
  float lambda_host;  // unused when lambda_dev is given
  const float* lambda_dev;
  int apply_norm;
  const float* g;
  float eps, post;
  float* dlambda;  // one value (this head / pair)
  float* dg;       // [dv] or nullptr
};

__global__ void __launch_bounds__(32 * kPreWarps) bwd_pre_kernel(PreArgs a) {
  __shared__ float sh_dg[kPreWarps][kMaxDv];
  __shared__ float sh_dl[kPreWarps];
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int u = blockIdx.y;
  const float lam = *a.lambda_dev;
  constexpr int kT = kMaxDv / 32;
  float dg[kT] = {0.f, 0.f, 0.f, 0.f};
  float dl = 0.f;
  const int r0 = blockIdx.x * kRowsPerBlock;
  for (int i = r0 + warp; i < min(r0 + kRowsPerBlock, a.N); i += kPreWarps) {
    const size_t rb = ((size_t)u * a.N + i) * a.dv;
    float o1[kT], o2[kT], o[kT], dy[kT];
#pragma unroll
    for (int t = 0; t < kT; ++t) {
      const int c = lane + 32 * t;
      const bool in = c < a.dv;
      o1[t] = in ? a.O1[rb + c] : 0.f;
      o2[t] = in ? a.O2[rb + c] : 0.f;
      o[t] = o1[t] - lam * o2[t];
      dy[t] = in ? __bfloat162float(a.dout[u * a.dout_unit + i * a.dout_row + c]) : 0.f;
    }
    float d_o[kT];
    if (a.apply_norm) {
      float ss = 0.f, gdo = 0.f;
#pragma unroll
      for (int t = 0; t < kT; ++t) {
        const int c = lane + 32 * t;
        const float gc = (c < a.dv && a.g) ? a.g[c] : 1.f;
        ss = fmaf(o[t], o[t], ss);
        gdo = fmaf(gc * dy[t], o[t], gdo);
      }
      ss = warp_sum(ss);
      gdo = warp_sum(gdo);
      const float rr = sqrtf(ss / (float)a.dv + a.eps);
      const float cr = a.post / rr;
      const float k2 = gdo / ((float)a.dv * rr * rr);
#pragma unroll
      for (int t = 0; t < kT; ++t) {
        const int c = lane + 32 * t;
        const float gc = (c < a.dv && a.g) ? a.g[c] : 1.f;
        d_o[t] = cr * (gc * dy[t] - o[t] * k2);
        dg[t] = fmaf(dy[t] * o[t], cr, dg[t]);
      }
    } else {
#pragma unroll
      for (int t = 0; t < kT; ++t) d_o[t] = dy[t];
    }
    // bf16 upstream gradients (the GEMM inputs) and D from the same values
    float s1 = 0.f, s2 = 0.f, sl = 0.f;
#pragma unroll
    for (int t = 0; t < kT; ++t) {
      const int c = lane + 32 * t;
      if (c < a.dv) {
        const __nv_bfloat16 b1 = __float2bfloat16_rn(d_o[t]);
        const __nv_bfloat16 b2 = __float2bfloat16_rn(-lam * d_o[t]);
        a.do1[rb + c] = b1;
        a.do2[rb + c] = b2;
        s1 = fmaf(__bfloat162float(b1), o1[t], s1);
        s2 = fmaf(__bfloat162float(b2), o2[t], s2);
        sl = fmaf(d_o[t], o2[t], sl);
      }
    }
    s1 = warp_sum(s1);
    s2 = warp_sum(s2);
    sl = warp_sum(sl);
    if (lane == 0) {
      a.D1[(size_t)u * a.N + i] = s1;
      a.D2[(size_t)u * a.N + i] = s2;
    }
    dl -= sl;
  }
  // block reductions, then one atomic per value
#pragma unroll
  for (int t = 0; t < kT; ++t) sh_dg[warp][lane + 32 * t] = dg[t];
  if (lane == 0) sh_dl[warp] = dl;
  __syncthreads();
  if (threadIdx.x < kMaxDv && a.dg && threadIdx.x < a.dv) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kPreWarps; ++w) s += sh_dg[w][threadIdx.x];
    atomicAdd(a.dg + threadIdx.x, s);
  }
  if (threadIdx.x == 0) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kPreWarps; ++w) s += sh_dl[w];
    atomicAdd(a.dlambda, s);
  }
}

// dlq1 = dl e^{lq1.lk1} lk1, dlk1 = dl e^{lq1.lk1} lq1, and the same with a
// minus sign for the second pair.  One warp per head.
__global__ void lambda_params_bwd_kernel(const float* lq1, const float* lk1, const float* lq2,
                                         const float* lk2, const float* dlambda, int H, int dim,
                                         float* dlq1, float* dlk1, float* dlq2, float* dlk2) {
  const int h = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (h >= H) return;
  const size_t b = (size_t)h * dim;
  float d1 = 0.f, d2 = 0.f;
  for (int c = lane; c < dim; c += 32) {
    d1 = fmaf(lq1[b + c], lk1[b + c], d1);
    d2 = fmaf(lq2[b + c], lk2[b + c], d2);
  }
  d1 = warp_sum(d1);
  d2 = warp_sum(d2);
  const float e1 = expf(d1) * dlambda[h], e2 = expf(d2) * dlambda[h];
  for (int c = lane; c < dim; c += 32) {
    dlq1[b + c] = e1 * lk1[b + c];
    dlk1[b + c] = e1 * lq1[b + c];
    dlq2[b + c] = -e2 * lk2[b + c];
    dlk2[b + c] = -e2 * lq2[b + c];
  }
}

// Row-major C[M x N] (ldc) = alpha op(A) op(B) + beta C, batched with strides.
// A is row-major [M x K] (lda), or [K x M] read transposed when ta; B is
// [K x N] (ldb), or [N x K] read transposed when tb.  bf16 operands, fp32 C.
// A plain CUDA-core kernel: this path serves only the widths the fused
// tensor-core backward does not cover.  64 x 64 output tiles, K in steps of
// 16 staged in shared memory as fp32, a 4 x 4 block of outputs per thread;
// out-of-range operand elements read as zero.
constexpr int kGT = 64, kGK = 16;

template <bool kTA, bool kTB>
__global__ void __launch_bounds__(256) gemm_bf16_simt_kernel(
    int M, int N, int K, float alpha, const __nv_bfloat16* A, int lda, long long sA,
    const __nv_bfloat16* Bm, int ldb, long long sB, float beta, float* C, int ldc, long long sC) {
  __shared__ float As[kGK][kGT + 4];
  __shared__ float Bs[kGK][kGT + 4];
  const int z = blockIdx.z;
  A += z * sA;
  Bm += z * sB;
  C += z * sC;
  const int m0 = blockIdx.y * kGT, n0 = blockIdx.x * kGT;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += kGK) {
    for (int e = threadIdx.x; e < kGT * kGK; e += 256) {
      // element (row i of the tile, column kk of the K step), both operands
      const int i = kTA ? e % kGT : e / kGK, kk = kTA ? e / kGT : e % kGK;
      const int m = m0 + i, k = k0 + kk;
      float va = 0.f;
      if (m < M && k < K)
        va = __bfloat162float(kTA ? A[(long long)k * lda + m] : A[(long long)m * lda + k]);
      As[kk][i] = va;
      const int j = kTB ? e / kGK : e % kGT, kb = kTB ? e % kGK : e / kGT;
      const int n = n0 + j, kn = k0 + kb;
      float vb = 0.f;
      if (n < N && kn < K)
        vb = __bfloat162float(kTB ? Bm[(long long)n * ldb + kn] : Bm[(long long)kn * ldb + n]);
      Bs[kb][j] = vb;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kGK; ++kk) {
      float a4[4], b4[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        a4[t] = As[kk][ty * 4 + t];
        b4[t] = Bs[kk][tx * 4 + t];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a4[i], b4[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= N) continue;
      float* c = C + (long long)m * ldc + n;
      *c = alpha * acc[i][j] + (beta != 0.f ? beta * *c : 0.f);
    }
  }
}

cudaError_t gemm_rm(cudaStream_t st, bool ta, bool tb, int M, int N, int K, float alpha,
                    const void* A, int lda, long long sA, const void* B, int ldb, long long sB,
                    float beta, float* C, int ldc, long long sC, int batch) {
  const dim3 grid((unsigned)((N + kGT - 1) / kGT), (unsigned)((M + kGT - 1) / kGT),
                  (unsigned)batch);
  const auto* a = static_cast<const __nv_bfloat16*>(A);
  const auto* b = static_cast<const __nv_bfloat16*>(B);
  if (ta && tb)
    gemm_bf16_simt_kernel<true, true><<<grid, 256, 0, st>>>(M, N, K, alpha, a, lda, sA, b, ldb, sB,
                                                          beta, C, ldc, sC);
  else if (ta)
    gemm_bf16_simt_kernel<true, false><<<grid, 256, 0, st>>>(M, N, K, alpha, a, lda, sA, b, ldb,
                                                           sB, beta, C, ldc, sC);
  else if (tb)
    gemm_bf16_simt_kernel<false, true><<<grid, 256, 0, st>>>(M, N, K, alpha, a, lda, sA, b, ldb,
                                                           sB, beta, C, ldc, sC);
  else
    gemm_bf16_simt_kernel<false, false><<<grid, 256, 0, st>>>(M, N, K, alpha, a, lda, sA, b, ldb,
                                                            sB, beta, C, ldc, sC);
  return cudaGetLastError();
}

// Geometry of one backward problem, in elements.  A "unit" is one head (V1)
// or head pair (V2) of one batch entry; row i of branch r of unit (b, h):
//   Q_r at q + b*q_b + i*q_row + h*q_unit + r*q_br, K_r likewise with k_*
//   (k_unit is per KV head: kv(h) = h / kv_div), V at v + b*v_b + i*v_row +
//   kv(h)*v_unit, dout at dout + b*o_b + i*o_row + h*o_unit.
// dq/dk/dv use the q/k/v geometry.
struct Geo {
  int B, N, H, d, dv, kv_div;
  long long q_b, q_row, q_unit, q_br;
  long long k_b, k_row, k_unit, k_br;
  long long v_b, v_row, v_unit;
  long long o_b, o_row, o_unit;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

size_t unit_bytes(int N, int dv) {
  const size_t n2 = (size_t)N * N;
  return align256(n2 * 4) + 3 * align256(n2 * 2) + 2 * align256((size_t)N * dv * 4) +
         2 * align256((size_t)N * dv * 2) + 2 * align256((size_t)N * 4);
}

int chunk_units(int B, int N, int dv) {
  const size_t per = unit_bytes(N, dv);
  size_t c = kChunkCap / per;
  if (c < 1) c = 1;
  return (int)(c < (size_t)B ? c : (size_t)B);
}

size_t bwd_workspace_bytes(int B, int N, int dv) {
  return (size_t)chunk_units(B, N, dv) * unit_bytes(N, dv) + 256;
}

// The whole backward for one problem (device pointers; fp32 gradients).
int run_bwd(const Geo& G, const __nv_bfloat16* q, const __nv_bfloat16* k,
            const __nv_bfloat16* v, const __nv_bfloat16* dout, const float* lambda, int causal,
            int window, int apply_norm, const float* g, float eps, float post, float* dq,
            float* dk, float* dv, float* dlambda, float* dg, void* ws, size_t ws_bytes,
            cudaStream_t st) {
  const int N = G.N, dvw = G.dv;
  const int cu = chunk_units(G.B, N, dvw);
  if (!ws || ws_bytes < bwd_workspace_bytes(G.B, N, dvw)) return DA_ERR_WORKSPACE;

  // carve the workspace
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(ws) + 255) & ~uintptr_t(255));
  const size_t n2 = (size_t)N * N;
  auto take = [&](size_t bytes) {
    uint8_t* p = base;
    base += align256(bytes);
    return p;
  };
  float* X = reinterpret_cast<float*>(take((size_t)cu * n2 * 4));
  __nv_bfloat16* P[2];
  P[0] = reinterpret_cast<__nv_bfloat16*>(take((size_t)cu * n2 * 2));
  P[1] = reinterpret_cast<__nv_bfloat16*>(take((size_t)cu * n2 * 2));
  __nv_bfloat16* dS = reinterpret_cast<__nv_bfloat16*>(take((size_t)cu * n2 * 2));
  float* O[2];
  O[0] = reinterpret_cast<float*>(take((size_t)cu * N * dvw * 4));
  O[1] = reinterpret_cast<float*>(take((size_t)cu * N * dvw * 4));
  __nv_bfloat16* dO[2];
  dO[0] = reinterpret_cast<__nv_bfloat16*>(take((size_t)cu * N * dvw * 2));
  dO[1] = reinterpret_cast<__nv_bfloat16*>(take((size_t)cu * N * dvw * 2));
  float* D[2];
  D[0] = reinterpret_cast<float*>(take((size_t)cu * N * 4));
  D[1] = reinterpret_cast<float*>(take((size_t)cu * N * 4));

  // gradients that accumulate start at zero (dq is written, not accumulated)
  const size_t n_k = (size_t)G.B * G.k_b, n_v = (size_t)G.B * G.v_b;
  if (cudaMemsetAsync(dk, 0, n_k * 4, st) != cudaSuccess ||
      cudaMemsetAsync(dv, 0, n_v * 4, st) != cudaSuccess ||
      cudaMemsetAsync(dlambda, 0, (size_t)G.H * 4, st) != cudaSuccess ||
      (dg && cudaMemsetAsync(dg, 0, (size_t)dvw * 4, st) != cudaSuccess))
    return DA_ERR_CUDA;

  const float scale = 1.0f / std::sqrt((float)G.d);
  const int rows_per_blk = 4;  // warps per block of the row kernels
  for (int hh = 0; hh < G.H; ++hh) {
    const int kvh = hh / G.kv_div;
    for (int b0 = 0; b0 < G.B; b0 += cu) {
      const int nb = (G.B - b0) < cu ? (G.B - b0) : cu;
      const long long rows = (long long)nb * N;
      const unsigned grid_rows = (unsigned)((rows + rows_per_blk - 1) / rows_per_blk);
      const __nv_bfloat16* vb = v + b0 * G.v_b + kvh * G.v_unit;
      for (int r = 0; r < 2; ++r) {
        const __nv_bfloat16* qr = q + b0 * G.q_b + hh * G.q_unit + r * G.q_br;
        const __nv_bfloat16* kr = k + b0 * G.k_b + kvh * G.k_unit + r * G.k_br;
        if (gemm_rm(st, false, true, N, N, G.d, scale, qr, (int)G.q_row, G.q_b, kr,
                    (int)G.k_row, G.k_b, 0.f, X, N, (long long)n2, nb) != cudaSuccess)
          return DA_ERR_CUDA;
        bwd_softmax_kernel<<<grid_rows, 32 * rows_per_blk, 0, st>>>(X, P[r], N, nb, causal,
                                                                    window);
        if (gemm_rm(st, false, false, N, dvw, N, 1.f, P[r], N, (long long)n2, vb, (int)G.v_row,
                    G.v_b, 0.f, O[r], dvw, (long long)N * dvw, nb) != cudaSuccess)
          return DA_ERR_CUDA;
      }
      PreArgs pa;
      pa.O1 = O[0];
      pa.O2 = O[1];
      pa.dout = dout + b0 * G.o_b + hh * G.o_unit;
      pa.dout_unit = G.o_b;
      pa.dout_row = G.o_row;
      pa.do1 = dO[0];
      pa.do2 = dO[1];
      pa.D1 = D[0];
      pa.D2 = D[1];
      pa.N = N;
      pa.dv = dvw;
      pa.lambda_host = 0.f;
      pa.lambda_dev = lambda + hh;
      pa.apply_norm = apply_norm;
      pa.g = g;
      pa.eps = eps;
      pa.post = post;
      pa.dlambda = dlambda + hh;
      pa.dg = apply_norm ? dg : nullptr;
      dim3 pgrid((unsigned)((N + kRowsPerBlock - 1) / kRowsPerBlock), (unsigned)nb);
      bwd_pre_kernel<<<pgrid, 32 * kPreWarps, 0, st>>>(pa);
      for (int r = 0; r < 2; ++r) {
        const __nv_bfloat16* qr = q + b0 * G.q_b + hh * G.q_unit + r * G.q_br;
        const __nv_bfloat16* kr = k + b0 * G.k_b + kvh * G.k_unit + r * G.k_br;
        float* dqr = dq + b0 * G.q_b + hh * G.q_unit + r * G.q_br;
        float* dkr = dk + b0 * G.k_b + kvh * G.k_unit + r * G.k_br;
        float* dvb = dv + b0 * G.v_b + kvh * G.v_unit;
        if (gemm_rm(st, false, true, N, N, dvw, 1.f, dO[r], dvw, (long long)N * dvw, vb,
                    (int)G.v_row, G.v_b, 0.f, X, N, (long long)n2, nb) != cudaSuccess)
          return DA_ERR_CUDA;
        bwd_ds_kernel<<<grid_rows, 32 * rows_per_blk, 0, st>>>(P[r], X, D[r], dS, N, nb);
        if (gemm_rm(st, false, false, N, G.d, N, scale, dS, N, (long long)n2, kr, (int)G.k_row,
                    G.k_b, 0.f, dqr, (int)G.q_row, G.q_b, nb) != cudaSuccess ||
            gemm_rm(st, true, false, N, G.d, N, scale, dS, N, (long long)n2, qr, (int)G.q_row,
                    G.q_b, 1.f, dkr, (int)G.k_row, G.k_b, nb) != cudaSuccess ||
            gemm_rm(st, true, false, N, dvw, N, 1.f, P[r], N, (long long)n2, dO[r], dvw,
                    (long long)N * dvw, 1.f, dvb, (int)G.v_row, G.v_b, nb) != cudaSuccess)
          return DA_ERR_CUDA;
      }
    }
  }
  return cudaGetLastError() == cudaSuccess ? DA_OK : DA_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool fits_int(long long x) { return x >= 0 && x <= 0x7fffffffLL; }
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

}  // namespace
}  // namespace da

extern "C" {

size_t diffattn_v1_bwd_workspace_size(int batch, int seqlen, int n_heads, int d_qk, int d_v) {
  if (batch < 1 || seqlen < 1 || n_heads < 1 || d_qk < 1 || d_v < 1) return 0;
  if (d_qk == 64 && d_v == 128) return da::fused_bwd_workspace_bytes(batch, seqlen, n_heads);
  return da::bwd_workspace_bytes(batch, seqlen, d_v);
}

int diffattn_v1_bwd(const void* q, const void* k, const void* v, const void* dout,
                    const float* lambda, da_dtype dtype, int batch, int seqlen, int n_heads,
                    int d_qk, int d_v, int causal, int window, int apply_norm,
                    const float* norm_weight, float norm_eps, float lambda_init, float* dq,
                    float* dk, float* dv, float* dlambda, float* dnorm_weight, void* workspace,
                    size_t workspace_bytes, int* dev_status, void* stream) {
  if (!q || !k || !v || !dout || !lambda || !dq || !dk || !dv || !dlambda)
    return DA_ERR_INVALID_ARG;
  if (batch < 1 || seqlen < 1 || n_heads < 1 || d_qk < 1 || d_v < 1) return DA_ERR_INVALID_ARG;
  if (window < 0 || (window > 0 && !causal)) return DA_ERR_INVALID_ARG;
  if (apply_norm && !(norm_eps >= 0.f)) return DA_ERR_INVALID_ARG;
  if (dtype != DA_BF16) return DA_ERR_UNSUPPORTED;
  if (d_v > da::kMaxDv || d_qk > 256) return DA_ERR_UNSUPPORTED;
  if ((long long)seqlen * seqlen > (1LL << 31)) return DA_ERR_UNSUPPORTED;
  if (!da::aligned16(q) || !da::aligned16(k) || !da::aligned16(v) || !da::aligned16(dout))
    return DA_ERR_ALIGNMENT;
  da::Geo G;
  G.B = batch;
  G.N = seqlen;
  G.H = n_heads;
  G.d = d_qk;
  G.dv = d_v;
  G.kv_div = 1;
  G.q_row = (long long)n_heads * 2 * d_qk;
  G.q_b = G.q_row * seqlen;
  G.q_unit = 2 * d_qk;
  G.q_br = d_qk;
  G.k_row = G.q_row;
  G.k_b = G.q_b;
  G.k_unit = G.q_unit;
  G.k_br = d_qk;
  G.v_row = (long long)n_heads * d_v;
  G.v_b = G.v_row * seqlen;
  G.v_unit = d_v;
  G.o_row = G.v_row;
  G.o_b = G.v_b;
  G.o_unit = d_v;
  if (d_qk == 64 && d_v == 128) {  // fused tcgen05 path
    if (!workspace || workspace_bytes < da::fused_bwd_workspace_bytes(batch, seqlen, n_heads))
      return DA_ERR_WORKSPACE;
    if (!da::fits_int((long long)batch * seqlen)) return DA_ERR_UNSUPPORTED;
    da::FusedBwdArgs a{};
    a.fwd.form = 1;
    a.fwd.batch = batch;
    a.fwd.seqlen = seqlen;
    a.fwd.heads = n_heads;
    a.fwd.kv_heads = n_heads;
    a.fwd.pairs_per_kv = 1;
    a.fwd.causal = causal ? 1 : 0;
    a.fwd.window = window;
    a.fwd.lambda = lambda;
    a.fwd.apply_norm = apply_norm ? 1 : 0;
    a.fwd.norm_weight = norm_weight;
    a.fwd.eps = norm_eps;
    a.fwd.post_scale = 1.0f - lambda_init;
    a.fwd.dev_status = dev_status;
    a.q = q;
    a.k = k;
    a.v = v;
    a.dout = dout;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.dlambda = dlambda;
    a.dg = apply_norm ? dnorm_weight : nullptr;
    a.workspace = workspace;
    a.num_sms = da::sm_count();
    if (a.num_sms < 1) return DA_ERR_CUDA;
    return da::launch_fused_bwd(a, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? DA_OK
               : DA_ERR_CUDA;
  }
  return da::run_bwd(G, static_cast<const __nv_bfloat16*>(q),
                     static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
                     static_cast<const __nv_bfloat16*>(dout), lambda, causal ? 1 : 0, window,
                     apply_norm ? 1 : 0, norm_weight, norm_eps, 1.0f - lambda_init, dq, dk, dv,
                     dlambda, apply_norm ? dnorm_weight : nullptr, workspace, workspace_bytes,
                     static_cast<cudaStream_t>(stream));
}

size_t diffattn_v2_bwd_workspace_size(int batch, int seqlen, int n_q_heads, int n_kv_heads,
                                      int head_dim) {
  if (batch < 1 || seqlen < 1 || n_q_heads < 2 || n_kv_heads < 1 || head_dim < 1) return 0;
  if (head_dim == 128) return da::fused_bwd_workspace_bytes(batch, seqlen, n_q_heads / 2);
  return da::bwd_workspace_bytes(batch, seqlen, head_dim);
}

int diffattn_v2_bwd(const void* q, const void* k, const void* v, const void* dout,
                    const float* lambda, da_dtype dtype, int batch, int seqlen, int n_q_heads,
                    int n_kv_heads, int head_dim, int causal, int window, float* dq, float* dk,
                    float* dv, float* dlambda, void* workspace, size_t workspace_bytes,
                    int* dev_status, void* stream) {
  if (!q || !k || !v || !dout || !lambda || !dq || !dk || !dv || !dlambda)
    return DA_ERR_INVALID_ARG;
  if (batch < 1 || seqlen < 1 || n_q_heads < 2 || n_kv_heads < 1 || head_dim < 1)
    return DA_ERR_INVALID_ARG;
  if (n_q_heads % n_kv_heads != 0 || (n_q_heads / n_kv_heads) % 2 != 0)
    return DA_ERR_INVALID_ARG;
  if (window < 0 || (window > 0 && !causal)) return DA_ERR_INVALID_ARG;
  if (dtype != DA_BF16) return DA_ERR_UNSUPPORTED;
  if (head_dim > da::kMaxDv) return DA_ERR_UNSUPPORTED;
  if ((long long)seqlen * seqlen > (1LL << 31)) return DA_ERR_UNSUPPORTED;
  if (!da::aligned16(q) || !da::aligned16(k) || !da::aligned16(v) || !da::aligned16(dout))
    return DA_ERR_ALIGNMENT;
  const int group = n_q_heads / n_kv_heads;
  da::Geo G;
  G.B = batch;
  G.N = seqlen;
  G.H = n_q_heads / 2;
  G.d = head_dim;
  G.dv = head_dim;
  G.kv_div = group / 2;
  G.q_row = (long long)n_q_heads * head_dim;
  G.q_b = G.q_row * seqlen;
  G.q_unit = 2 * head_dim;
  G.q_br = head_dim;
  G.k_row = (long long)n_kv_heads * head_dim;
  G.k_b = G.k_row * seqlen;
  G.k_unit = head_dim;
  G.k_br = 0;
  G.v_row = G.k_row;
  G.v_b = G.k_b;
  G.v_unit = head_dim;
  G.o_row = (long long)(n_q_heads / 2) * head_dim;
  G.o_b = G.o_row * seqlen;
  G.o_unit = head_dim;
  if (head_dim == 128) {  // fused tcgen05 path
    if (!workspace ||
        workspace_bytes < da::fused_bwd_workspace_bytes(batch, seqlen, n_q_heads / 2))
      return DA_ERR_WORKSPACE;
    if (!da::fits_int((long long)batch * seqlen)) return DA_ERR_UNSUPPORTED;
    da::FusedBwdArgs a{};
    a.fwd.form = 2;
    a.fwd.batch = batch;
    a.fwd.seqlen = seqlen;
    a.fwd.heads = n_q_heads / 2;
    a.fwd.kv_heads = n_kv_heads;
    a.fwd.pairs_per_kv = group / 2;
    a.fwd.causal = causal ? 1 : 0;
    a.fwd.window = window;
    a.fwd.lambda = lambda;
    a.fwd.apply_norm = 0;
    a.fwd.post_scale = 1.f;
    a.fwd.dev_status = dev_status;
    a.q = q;
    a.k = k;
    a.v = v;
    a.dout = dout;
    a.dq = dq;
    a.dk = dk;
    a.dv = dv;
    a.dlambda = dlambda;
    a.workspace = workspace;
    a.num_sms = da::sm_count();
    if (a.num_sms < 1) return DA_ERR_CUDA;
    return da::launch_fused_bwd(a, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? DA_OK
               : DA_ERR_CUDA;
  }
  return da::run_bwd(G, static_cast<const __nv_bfloat16*>(q),
                     static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
                     static_cast<const __nv_bfloat16*>(dout), lambda, causal ? 1 : 0, window, 0,
                     nullptr, 0.f, 1.f, dq, dk, dv, dlambda, nullptr, workspace,
                     workspace_bytes, static_cast<cudaStream_t>(stream));
}

// ---- training forward with saves, and the backward from those saves -------
namespace {

da::PrefillArgs v1_fwd_args(int batch, int seqlen, int n_heads, int causal, int window,
                            const float* lambda, int apply_norm, const float* norm_weight,
                            float norm_eps, float lambda_init, int* dev_status) {
  da::PrefillArgs f{};
  f.form = 1;
  f.batch = batch;
  f.seqlen = seqlen;
  f.heads = n_heads;
  f.kv_heads = n_heads;
  f.pairs_per_kv = 1;
  f.causal = causal ? 1 : 0;
  f.window = window;
  f.lambda = lambda;
  f.apply_norm = apply_norm ? 1 : 0;
  f.norm_weight = norm_weight;
  f.eps = norm_eps;
  f.post_scale = 1.0f - lambda_init;
  f.dev_status = dev_status;
  return f;
}

da::PrefillArgs v2_fwd_args(int batch, int seqlen, int n_q_heads, int n_kv_heads, int causal,
                            int window, const float* lambda, int* dev_status) {
  da::PrefillArgs f{};
  f.form = 2;
  f.batch = batch;
  f.seqlen = seqlen;
  f.heads = n_q_heads / 2;
  f.kv_heads = n_kv_heads;
  f.pairs_per_kv = (n_q_heads / n_kv_heads) / 2;
  f.causal = causal ? 1 : 0;
  f.window = window;
  f.lambda = lambda;
  f.apply_norm = 0;
  f.post_scale = 1.f;
  f.dev_status = dev_status;
  return f;
}

// Shared checks of the saved-state calls: sizes, masks, the tensor-core
// widths, alignment.  Returns DA_OK or the status to return.
int check_train(int batch, int seqlen, int units, int causal, int window, bool widths_ok,
                std::initializer_list<const void*> ptrs) {
  for (const void* q : ptrs)
    if (!q) return DA_ERR_INVALID_ARG;
  if (batch < 1 || seqlen < 1 || units < 1) return DA_ERR_INVALID_ARG;
  if (window < 0 || (window > 0 && !causal)) return DA_ERR_INVALID_ARG;
  if (!widths_ok) return DA_ERR_UNSUPPORTED;
  if (!da::fits_int((long long)batch * seqlen) || (long long)seqlen * seqlen > (1LL << 31))
    return DA_ERR_UNSUPPORTED;
  for (const void* q : ptrs)
    if (!da::aligned16(q)) return DA_ERR_ALIGNMENT;
  return DA_OK;
}

}  // namespace

size_t diffattn_v1_fwd_train_saves_size(int batch, int seqlen, int n_heads) {
  if (batch < 1 || seqlen < 1 || n_heads < 1) return 0;
  return da::train_saves_bytes(batch, seqlen, n_heads);
}

int diffattn_v1_fwd_train(const void* q, const void* k, const void* v, void* out,
                          da_dtype dtype, int batch, int seqlen, int n_heads, int d_qk, int d_v,
                          const float* lambda, int causal, int window, int apply_norm,
                          const float* norm_weight, float norm_eps, float lambda_init,
                          void* saves, size_t saves_bytes, int* dev_status, void* stream) {
  if (apply_norm && !(norm_eps >= 0.f)) return DA_ERR_INVALID_ARG;
  if (dtype != DA_BF16) return DA_ERR_UNSUPPORTED;
  int rc = check_train(batch, seqlen, n_heads, causal, window, d_qk == 64 && d_v == 128,
                       {q, k, v, out, lambda, saves});
  if (rc != DA_OK) return rc;
  if (saves_bytes < da::train_saves_bytes(batch, seqlen, n_heads)) return DA_ERR_WORKSPACE;
  const int sms = da::sm_count();
  if (sms < 1) return DA_ERR_CUDA;
  return da::launch_fwd_train(v1_fwd_args(batch, seqlen, n_heads, causal, window, lambda,
                                          apply_norm, norm_weight, norm_eps, lambda_init,
                                          dev_status),
                              q, k, v, out, saves, sms, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? DA_OK
             : DA_ERR_CUDA;
}

size_t diffattn_v1_bwd_saved_workspace_size(int batch, int seqlen, int n_heads) {
  if (batch < 1 || seqlen < 1 || n_heads < 1) return 0;
  return da::saved_bwd_workspace_bytes(batch, seqlen, n_heads);
}

int diffattn_v1_bwd_saved(const void* q, const void* k, const void* v, const void* dout,
                          const float* lambda, da_dtype dtype, int batch, int seqlen,
                          int n_heads, int d_qk, int d_v, int causal, int window, int apply_norm,
                          const float* norm_weight, float norm_eps, float lambda_init,
                          const void* saves, size_t saves_bytes, float* dq, float* dk,
                          float* dv, float* dlambda, float* dnorm_weight, void* workspace,
                          size_t workspace_bytes, int* dev_status, void* stream) {
  if (!dq || !dk || !dv || !dlambda) return DA_ERR_INVALID_ARG;
  if (apply_norm && !(norm_eps >= 0.f)) return DA_ERR_INVALID_ARG;
  if (dtype != DA_BF16) return DA_ERR_UNSUPPORTED;
  int rc = check_train(batch, seqlen, n_heads, causal, window, d_qk == 64 && d_v == 128,
                       {q, k, v, dout, lambda, saves, workspace});
  if (rc != DA_OK) return rc;
  if (saves_bytes < da::train_saves_bytes(batch, seqlen, n_heads) ||
      workspace_bytes < da::saved_bwd_workspace_bytes(batch, seqlen, n_heads))
    return DA_ERR_WORKSPACE;
  da::FusedBwdArgs a{};
  a.fwd = v1_fwd_args(batch, seqlen, n_heads, causal, window, lambda, apply_norm, norm_weight,
                      norm_eps, lambda_init, dev_status);
  a.q = q;
  a.k = k;
  a.v = v;
  a.dout = dout;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dlambda = dlambda;
  a.dg = apply_norm ? dnorm_weight : nullptr;
  a.workspace = workspace;
  a.num_sms = da::sm_count();
  if (a.num_sms < 1) return DA_ERR_CUDA;
  return da::launch_bwd_from_saves(a, saves, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? DA_OK
             : DA_ERR_CUDA;
}

size_t diffattn_v2_prefill_train_saves_size(int batch, int seqlen, int n_q_heads) {
  if (batch < 1 || seqlen < 1 || n_q_heads < 2) return 0;
  return da::train_saves_bytes(batch, seqlen, n_q_heads / 2);
}

int diffattn_v2_prefill_train(const void* q, const void* k, const void* v, void* out,
                              da_dtype dtype, int batch, int seqlen, int n_q_heads,
                              int n_kv_heads, int head_dim, const float* lambda, int causal,
                              int window, void* saves, size_t saves_bytes, int* dev_status,
                              void* stream) {
  if (n_q_heads < 2 || n_kv_heads < 1 || n_q_heads % n_kv_heads != 0 ||
      (n_q_heads / n_kv_heads) % 2 != 0)
    return DA_ERR_INVALID_ARG;
  if (dtype != DA_BF16) return DA_ERR_UNSUPPORTED;
  int rc = check_train(batch, seqlen, n_q_heads / 2, causal, window, head_dim == 128,
                       {q, k, v, out, lambda, saves});
  if (rc != DA_OK) return rc;
  if (saves_bytes < da::train_saves_bytes(batch, seqlen, n_q_heads / 2)) return DA_ERR_WORKSPACE;
  const int sms = da::sm_count();
  if (sms < 1) return DA_ERR_CUDA;
  return da::launch_fwd_train(
             v2_fwd_args(batch, seqlen, n_q_heads, n_kv_heads, causal, window, lambda,
                         dev_status),
             q, k, v, out, saves, sms, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? DA_OK
             : DA_ERR_CUDA;
}

size_t diffattn_v2_bwd_saved_workspace_size(int batch, int seqlen, int n_q_heads) {
  if (batch < 1 || seqlen < 1 || n_q_heads < 2) return 0;
  return da::saved_bwd_workspace_bytes(batch, seqlen, n_q_heads / 2);
}

int diffattn_v2_bwd_saved(const void* q, const void* k, const void* v, const void* dout,
                          const float* lambda, da_dtype dtype, int batch, int seqlen,
                          int n_q_heads, int n_kv_heads, int head_dim, int causal, int window,
                          const void* saves, size_t saves_bytes, float* dq, float* dk,
                          float* dv, float* dlambda, void* workspace, size_t workspace_bytes,
                          int* dev_status, void* stream) {
  if (!dq || !dk || !dv || !dlambda) return DA_ERR_INVALID_ARG;
  if (n_q_heads < 2 || n_kv_heads < 1 || n_q_heads % n_kv_heads != 0 ||
      (n_q_heads / n_kv_heads) % 2 != 0)
    return DA_ERR_INVALID_ARG;
  if (dtype != DA_BF16) return DA_ERR_UNSUPPORTED;
  int rc = check_train(batch, seqlen, n_q_heads / 2, causal, window, head_dim == 128,
                       {q, k, v, dout, lambda, saves, workspace});
  if (rc != DA_OK) return rc;
  if (saves_bytes < da::train_saves_bytes(batch, seqlen, n_q_heads / 2) ||
      workspace_bytes < da::saved_bwd_workspace_bytes(batch, seqlen, n_q_heads / 2))
    return DA_ERR_WORKSPACE;
  da::FusedBwdArgs a{};
  a.fwd = v2_fwd_args(batch, seqlen, n_q_heads, n_kv_heads, causal, window, lambda, dev_status);
  a.q = q;
  a.k = k;
  a.v = v;
  a.dout = dout;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dlambda = dlambda;
  a.workspace = workspace;
  a.num_sms = da::sm_count();
  if (a.num_sms < 1) return DA_ERR_CUDA;
  return da::launch_bwd_from_saves(a, saves, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? DA_OK
             : DA_ERR_CUDA;
}

int lambda_from_params_bwd(const float* lq1, const float* lk1, const float* lq2,
                           const float* lk2, const float* dlambda, int n_heads, int dim,
                           float* dlq1, float* dlk1, float* dlq2, float* dlk2, void* stream) {
  if (!lq1 || !lk1 || !lq2 || !lk2 || !dlambda || !dlq1 || !dlk1 || !dlq2 || !dlk2)
    return DA_ERR_INVALID_ARG;
  if (n_heads < 1 || dim < 1) return DA_ERR_INVALID_ARG;
  const int warps = 4;
  da::lambda_params_bwd_kernel<<<(n_heads + warps - 1) / warps, 32 * warps, 0,
                                 static_cast<cudaStream_t>(stream)>>>(
      lq1, lk1, lq2, lk2, dlambda, n_heads, dim, dlq1, dlk1, dlq2, dlk2);
  return cudaGetLastError() == cudaSuccess ? DA_OK : DA_ERR_CUDA;
}

}  // extern "C"
