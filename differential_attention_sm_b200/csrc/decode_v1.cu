// decode_v1.cu — V1 single-token decode against a multi-head cache.
//
// Lesson "Atención Diferencial (V2)", section "V1 vs V2: la diferencia": a
// V1 head splits its query/key into two 64-wide halves and shares one value
// row between both softmax branches.  This kernel reads each cached K row
// (both halves) and each V row once for both branches.
//
// The contraction is 1.5 flop per cached byte, so CUDA cores keep up with
// HBM.  Work item = (batch b, head h, split s).  Inside a CTA, four lanes
// share one cache row: lane j of the group loads 16-byte pieces
// {32 i + 8 j .. +7 : i = 0..3} of the 128-wide K and V rows (64 contiguous
// bytes per group per load, fully used sectors).  Each 4-lane group keeps
// its own online-softmax state for both branches; groups are merged with
// shuffles, warps through shared memory, splits by a combine kernel that
// also applies -lambda, the per-head RMS norm and the (1 - lambda_init)
// scale.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace da {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = 32 * kWarps;
constexpr int kRowsPerSweep = kWarps * 8;  // rows one pass of the CTA covers
constexpr int kW = 128;                    // K row width (2 x 64) = V row width

struct Params {
  const __nv_bfloat16* q;   // [B, H, 128]
  const __nv_bfloat16* kc;  // [B, L, H, 128]
  const __nv_bfloat16* vc;  // [B, L, H, 128]
  const int* lens;
  int max_len, H;
  int window;  // > 0: the query sees only the last `window` valid entries
  int split_len, n_split, n_items;
  float scale_log2;
  float* part_o;   // [n_items][2][128]
  float* part_ml;  // [n_items][2][2]
};

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  f[0] = bf16lo(u.x);
  f[1] = bf16hi(u.x);
  f[2] = bf16lo(u.y);
  f[3] = bf16hi(u.y);
  f[4] = bf16lo(u.z);
  f[5] = bf16hi(u.z);
  f[6] = bf16lo(u.w);
  f[7] = bf16hi(u.w);
}

__device__ __forceinline__ uint4 ldg_stream(const __nv_bfloat16* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Online-softmax update of one branch with two new logits (log2 units).
__device__ __forceinline__ void branch_update(float& m, float& l, float (&o)[4][8], float sA,
                                              float sB, float& pA, float& pB) {
  const float mn = fmaxf(m, fmaxf(sA, sB));
  if (mn > m) {  // new running max: rescale (rare after the first rows)
    const float a = ex2(m - mn);
    l *= a;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) o[i][e] *= a;
    m = mn;
  }
  const float u = m == -INFINITY ? 0.f : m;
  pA = ex2(sA - u);
  pB = ex2(sB - u);
  l += pA + pB;
}

// Merge the running state held by the lane `off` away (same lane-in-group).
__device__ __forceinline__ void merge_xor(float& m, float& l, float (&o)[4][8], int off) {
  const float mo = __shfl_xor_sync(0xffffffffu, m, off);
  const float lo = __shfl_xor_sync(0xffffffffu, l, off);
  const float mn = fmaxf(m, mo);
  const float as = m == -INFINITY ? 0.f : ex2(m - mn);
  const float ao = mo == -INFINITY ? 0.f : ex2(mo - mn);
  l = l * as + lo * ao;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x = __shfl_xor_sync(0xffffffffu, o[i][e], off);
      o[i][e] = o[i][e] * as + x * ao;
    }
  m = mn;
}

__global__ void __launch_bounds__(kThreads, 1) v1_decode_split_kernel(const Params p) {
  __shared__ float sm_o[kWarps][2][kW];
  __shared__ float sm_ml[kWarps][2][2];
  const int item = blockIdx.x;
  const int s = item % p.n_split;
  const int bh = item / p.n_split;
  const int h = bh % p.H, b = bh / p.H;
  int len = p.lens ? p.lens[b] : p.max_len;
  len = len < 1 ? 1 : (len > p.max_len ? p.max_len : len);
  const int first = (p.window > 0 && len > p.window) ? len - p.window : 0;
  const int t0 = first + s * p.split_len;
  const int t1 = min(t0 + p.split_len, len);

  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int grp = lane >> 2, j = lane & 3;

  float qf[4][8];
  {
    const __nv_bfloat16* qrow = p.q + ((size_t)b * p.H + h) * kW;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      unpack8(*reinterpret_cast<const uint4*>(qrow + 32 * i + 8 * j), qf[i]);
#pragma unroll
      for (int e = 0; e < 8; ++e) qf[i][e] *= p.scale_log2;
    }
  }
  float o1[4][8], o2[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) o1[i][e] = o2[i][e] = 0.f;
  float m1 = -INFINITY, m2 = -INFINITY, l1 = 0.f, l2 = 0.f;

  const size_t row_stride = (size_t)p.H * kW;
  const __nv_bfloat16* kb = p.kc + ((size_t)b * p.max_len * p.H + h) * kW + 8 * j;
  const __nv_bfloat16* vb = p.vc + ((size_t)b * p.max_len * p.H + h) * kW + 8 * j;

  for (int base = t0 + warp * 8; base < t1; base += 2 * kRowsPerSweep) {
    const int tA = base + grp;
    const int tB = tA + kRowsPerSweep;
    const bool okA = tA < t1, okB = tB < t1;
    uint4 ka[4], kbv[4], va[4], vbv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      ka[i] = okA ? ldg_stream(kb + tA * row_stride + 32 * i) : make_uint4(0, 0, 0, 0);
      kbv[i] = okB ? ldg_stream(kb + tB * row_stride + 32 * i) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      va[i] = okA ? ldg_stream(vb + tA * row_stride + 32 * i) : make_uint4(0, 0, 0, 0);
      vbv[i] = okB ? ldg_stream(vb + tB * row_stride + 32 * i) : make_uint4(0, 0, 0, 0);
    }
    // logits: branch 1 = K columns 0..63 (i = 0, 1), branch 2 = 64..127 (i = 2, 3)
    float sA1 = 0.f, sA2 = 0.f, sB1 = 0.f, sB2 = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float fa[8], fb[8];
      unpack8(ka[i], fa);
      unpack8(kbv[i], fb);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (i < 2) {
          sA1 = fmaf(qf[i][e], fa[e], sA1);
          sB1 = fmaf(qf[i][e], fb[e], sB1);
        } else {
          sA2 = fmaf(qf[i][e], fa[e], sA2);
          sB2 = fmaf(qf[i][e], fb[e], sB2);
        }
      }
    }
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
      sA1 += __shfl_xor_sync(0xffffffffu, sA1, off);
      sA2 += __shfl_xor_sync(0xffffffffu, sA2, off);
      sB1 += __shfl_xor_sync(0xffffffffu, sB1, off);
      sB2 += __shfl_xor_sync(0xffffffffu, sB2, off);
    }
    if (!okA) sA1 = sA2 = -INFINITY;
    if (!okB) sB1 = sB2 = -INFINITY;
    float pA1, pB1, pA2, pB2;
    branch_update(m1, l1, o1, sA1, sB1, pA1, pB1);
    branch_update(m2, l2, o2, sA2, sB2, pA2, pB2);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float fa[8], fb[8];
      unpack8(va[i], fa);
      unpack8(vbv[i], fb);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        o1[i][e] = fmaf(pA1, fa[e], fmaf(pB1, fb[e], o1[i][e]));
        o2[i][e] = fmaf(pA2, fa[e], fmaf(pB2, fb[e], o2[i][e]));
      }
    }
  }
  // merge the 8 lane groups of the warp
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    merge_xor(m1, l1, o1, off);
    merge_xor(m2, l2, o2, off);
  }
  if (grp == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        sm_o[warp][0][32 * i + 8 * j + e] = o1[i][e];
        sm_o[warp][1][32 * i + 8 * j + e] = o2[i][e];
      }
    if (j == 0) {
      sm_ml[warp][0][0] = m1;
      sm_ml[warp][0][1] = l1;
      sm_ml[warp][1][0] = m2;
      sm_ml[warp][1][1] = l2;
    }
  }
  __syncthreads();
  {
    const int br = threadIdx.x / kW, c = threadIdx.x % kW;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm_ml[w][br][0]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float mw = sm_ml[w][br][0];
        if (mw == -INFINITY) continue;
        const float f = ex2(mw - M);
        L = fmaf(sm_ml[w][br][1], f, L);
        O = fmaf(sm_o[w][br][c], f, O);
      }
    }
    p.part_o[((size_t)item * 2 + br) * kW + c] = O;
    if (c == 0) {
      p.part_ml[((size_t)item * 2 + br) * 2 + 0] = M;
      p.part_ml[((size_t)item * 2 + br) * 2 + 1] = L;
    }
  }
}

// One block (128 threads, one per channel) per (batch, head).
__global__ void __launch_bounds__(kW) v1_decode_combine_kernel(
    const float* __restrict__ part_o, const float* __restrict__ part_ml,
    const float* __restrict__ lambda, __nv_bfloat16* __restrict__ out, int H, int n_split,
    int apply_norm, const float* __restrict__ g, float eps, float post_scale) {
  __shared__ float red[kW / 32];
  const int bh = blockIdx.x, h = bh % H;
  const int c = threadIdx.x;
  float M[2] = {-INFINITY, -INFINITY};
  for (int s = 0; s < n_split; ++s)
#pragma unroll
    for (int br = 0; br < 2; ++br)
      M[br] = fmaxf(M[br], part_ml[(((size_t)bh * n_split + s) * 2 + br) * 2]);
  float L[2] = {0.f, 0.f}, O[2] = {0.f, 0.f};
  for (int s = 0; s < n_split; ++s) {
#pragma unroll
    for (int br = 0; br < 2; ++br) {
      const size_t it = ((size_t)bh * n_split + s) * 2 + br;
      const float m = part_ml[it * 2];
      if (m == -INFINITY) continue;
      const float f = ex2(m - M[br]);
      L[br] = fmaf(part_ml[it * 2 + 1], f, L[br]);
      O[br] = fmaf(part_o[it * kW + c], f, O[br]);
    }
  }
  float r = O[0] / L[0] - lambda[h] * (O[1] / L[1]);
  if (apply_norm) {
    float ss = r * r;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((c & 31) == 0) red[c / 32] = ss;
    __syncthreads();
    ss = 0.f;
#pragma unroll
    for (int w = 0; w < kW / 32; ++w) ss += red[w];
    r = r * (post_scale / sqrtf(ss / (float)kW + eps)) * (g ? g[c] : 1.0f);
  }
  out[(size_t)bh * kW + c] = __float2bfloat16_rn(r);
}

}  // namespace

V1DecodePlan plan_v1_decode(int batch, int n_heads, int max_len, int num_sms) {
  // Non-persistent grid, one CTA per SM at a time: minimise
  // waves x rows-per-item (plus one sweep of overhead per item).
  const long units = (long)batch * n_heads;
  const int max_split = (max_len + kRowsPerSweep - 1) / kRowsPerSweep;
  V1DecodePlan best{1, max_len, (int)units};
  double best_cost = 1e300;
  for (int ns = 1; ns <= max_split && ns <= 256; ++ns) {
    int sl = (max_len + ns - 1) / ns;
    sl = (sl + kRowsPerSweep - 1) / kRowsPerSweep * kRowsPerSweep;
    const int ns_eff = (max_len + sl - 1) / sl;
    const long items = units * ns_eff;
    const long waves = (items + num_sms - 1) / num_sms;
    const double cost = (double)waves * (sl + 2 * kRowsPerSweep);
    if (cost < best_cost * 0.999) {
      best_cost = cost;
      best = {ns_eff, sl, (int)items};
    }
  }
  return best;
}

size_t v1_decode_workspace_bytes(const V1DecodePlan& plan) {
  return (size_t)plan.n_items * 2 * (kW + 2) * sizeof(float);
}

cudaError_t launch_v1_decode(const void* q, const void* k_cache, const void* v_cache,
                             const int* lens, int max_len, int window, void* out, int batch,
                             int n_heads, const float* lambda, int apply_norm,
                             const float* norm_weight, float eps, float post_scale,
                             const V1DecodePlan& plan, void* workspace, cudaStream_t stream) {
  Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.kc = static_cast<const __nv_bfloat16*>(k_cache);
  p.vc = static_cast<const __nv_bfloat16*>(v_cache);
  p.lens = lens;
  p.max_len = max_len;
  p.window = window;
  p.H = n_heads;
  p.split_len = plan.split_len;
  p.n_split = plan.n_split;
  p.n_items = plan.n_items;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt(64.0));
  p.part_o = static_cast<float*>(workspace);
  p.part_ml = p.part_o + (size_t)plan.n_items * 2 * kW;
  v1_decode_split_kernel<<<plan.n_items, kThreads, 0, stream>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  v1_decode_combine_kernel<<<batch * n_heads, kW, 0, stream>>>(
      p.part_o, p.part_ml, lambda, static_cast<__nv_bfloat16*>(out), n_heads, plan.n_split,
      apply_norm, norm_weight, eps, post_scale);
  return cudaGetLastError();
}

}  // namespace da
