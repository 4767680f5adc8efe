// decode_v2.cu — V2 single-token decode, split over the KV cache.
//
// Lesson "Atención Diferencial (V2)", section "V1 vs V2: la diferencia":
// V2 doubles the query heads and keeps the KV heads, so one decode step
// reads every cached K/V row once for all paired query heads of its GQA
// group ("Ejercicios" 5: 32 query heads on 8 KV heads).
//
// Work item = (batch b, KV head g, split s) covering cache rows
// [s*split_len, min((s+1)*split_len, len_b)).  A persistent CTA walks items
// with a static stride.  One producer warp streams 64-row K and V chunks
// into a 4-stage ring with TMA (128-byte swizzle, no multicast); four
// consumer warps each take 16 rows of a chunk.  Per consumer warp:
//   S^T[16 rows x 8 heads] = K_chunk . Q^T         (mma.sync m16n8k16, tokens
//                                                    as M, the group's heads as N)
//   online softmax per head (running max / sum; the pair's two heads are the
//   two columns a thread holds, so both branches stay in one thread)
//   O^T[128 x 8 heads] += V_chunk^T . P^T           (P to the B operand with
//                                                    movmatrix, V^T via ldmatrix.trans)
// The four warps' partial (m, l, O) are merged through shared memory and
// written to the workspace; a combine kernel merges the splits and forms
// o = O1 / l1 - lambda * O2 / l2 per pair.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace da {
namespace {

constexpr int kChunk = 64;                          // cache rows per stage
constexpr int kStages = 4;
constexpr int kConsumers = 4;                       // consumer warps
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kHalfBytes = kChunk * 64 * 2;         // 64 rows x 64 bf16 (one swizzle atom wide)
constexpr int kStageBytes = 4 * kHalfBytes;         // K[0:64], K[64:128], V[0:64], V[64:128]
constexpr int kHeads = 8;                           // MMA N: heads of one GQA group (padded)
constexpr int kD = 128;
constexpr int kRedOBytes = kConsumers * kHeads * kD * 4;
constexpr int kRedMLBytes = kConsumers * kHeads * 2 * 4;
constexpr int kSmemBytes =
    1024 + kStages * kStageBytes + kRedOBytes + kRedMLBytes + 2 * kStages * 8 + 16;

struct Params {
  const __nv_bfloat16* q;  // V2: [B, Hq, 128]; V1 form: [B, Hkv, 128] (branch halves)
  int v1;                  // V1 form: each KV head is one V1 head, seen as a pair of heads
  const int* lens;
  int max_len;
  int window;  // > 0: the query sees only the last `window` valid entries
  int Hq, Hkv, group;
  int split_len, n_split, n_items;
  float scale_log2;
  float* part_o;   // [n_items][8][128]
  float* part_ml;  // [n_items][8][2]  (max in log2 units, sum)
  int* dev_status;
};

__device__ __forceinline__ void item_coords(const Params& p, int item, int& b, int& g, int& t0,
                                            int& t1) {
  const int s = item % p.n_split;
  const int bg = item / p.n_split;
  g = bg % p.Hkv;
  b = bg / p.Hkv;
  int len = p.lens ? p.lens[b] : p.max_len;
  len = len < 1 ? 1 : (len > p.max_len ? p.max_len : len);
  const int first = (p.window > 0 && len > p.window) ? len - p.window : 0;
  t0 = first + s * p.split_len;
  t1 = min(t0 + p.split_len, len);
}

__global__ void __launch_bounds__(kThreads, 1)
    v2_decode_split_kernel(const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  float* red_o = reinterpret_cast<float*>(smem + kStages * kStageBytes);
  float* red_ml = red_o + kConsumers * kHeads * kD;
  uint64_t* full = reinterpret_cast<uint64_t*>(red_ml + kConsumers * kHeads * 2);
  uint64_t* empty = full + kStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumers);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  bool failed = false;

  if (warp == kConsumers) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int stage = 0;
      uint32_t phase = 0;
      for (int item = blockIdx.x; item < p.n_items && !failed; item += gridDim.x) {
        int b, g, t0, t1;
        item_coords(p, item, b, g, t0, t1);
        for (int t = t0; t < t1; t += kChunk) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, p.dev_status, &failed)) break;
          mbar_arrive_expect_tx(&full[stage], kStageBytes);
          uint8_t* dst = stages + stage * kStageBytes;
          tma_load_4d(dst, &tm_k, &full[stage], 0, g, t, b);
          tma_load_4d(dst + kHalfBytes, &tm_k, &full[stage], 64, g, t, b);
          tma_load_4d(dst + 2 * kHalfBytes, &tm_v, &full[stage], 0, g, t, b);
          tma_load_4d(dst + 3 * kHalfBytes, &tm_v, &full[stage], 64, g, t, b);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
    }
    return;
  }

  // ------------------------------ consumers -------------------------------
  const int cw = warp;           // 0..3: rows [16 cw, 16 cw + 16) of each chunk
  const int gq = lane >> 2;      // MMA group id: row (token) / column (head) index
  const int qq = lane & 3;       // thread in group: owns heads 2qq, 2qq+1 = pair qq
  const int mi = lane >> 3;      // ldmatrix: matrix this lane addresses
  const int mr = lane & 7;       // ldmatrix: row within that matrix
  int stage = 0;
  uint32_t phase = 0;

  for (int item = blockIdx.x; item < p.n_items; item += gridDim.x) {
    int b, g, t0, t1;
    item_coords(p, item, b, g, t0, t1);

    // Q^T fragments (B operand, k = feature, n = head), 8 k-steps of 16.
    // V1 form: head 0 of the pair is the query's first 64 features with zeros
    // above, head 1 zeros below and the last 64, so that one K row of 128
    // gives both branches' logits.
    uint32_t qf[8][2];
    {
      const bool valid = gq < p.group;
      const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
          p.v1 ? p.q + ((size_t)b * p.Hkv + g) * kD
               : p.q + ((size_t)b * p.Hq + (size_t)g * p.group + (valid ? gq : 0)) * kD);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const bool use = valid && (!p.v1 || (gq == (ks >> 2)));
        qf[ks][0] = use ? __ldg(qrow + ks * 8 + qq) : 0u;
        qf[ks][1] = use ? __ldg(qrow + ks * 8 + 4 + qq) : 0u;
      }
    }
    float o[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.f;
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;

    for (int t = t0; t < t1; t += kChunk) {
      if (!mbar_wait(&full[stage], phase, p.dev_status, &failed)) break;
      const uint32_t base = smem_u32(stages + stage * kStageBytes);
      const int row0 = cw * 16;

      // ---- S^T = K . Q^T for this warp's 16 rows ----
      float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int half = ks >> 2;
        const int row = row0 + mr + 8 * (mi & 1);
        const int c16 = (ks & 3) * 2 + (mi >> 1);  // 16-byte column chunk within the row
        const uint32_t addr =
            base + half * kHalfBytes + row * 128 + ((c16 ^ (row & 7)) << 4);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4(addr, a0, a1, a2, a3);
        mma_bf16_16816(s, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
      }
      // s[0]: (row gq, head 2qq)   s[1]: (row gq, head 2qq+1)
      // s[2]: (row gq+8, head 2qq) s[3]: (row gq+8, head 2qq+1)
      const int tok_a = t + row0 + gq;
      float sa0 = tok_a < t1 ? s[0] * p.scale_log2 : -INFINITY;
      float sb0 = tok_a < t1 ? s[1] * p.scale_log2 : -INFINITY;
      float sa1 = tok_a + 8 < t1 ? s[2] * p.scale_log2 : -INFINITY;
      float sb1 = tok_a + 8 < t1 ? s[3] * p.scale_log2 : -INFINITY;

      // ---- online softmax, one running state per head ----
      float cma = fmaxf(sa0, sa1), cmb = fmaxf(sb0, sb1);
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        cma = fmaxf(cma, __shfl_xor_sync(0xffffffffu, cma, off));
        cmb = fmaxf(cmb, __shfl_xor_sync(0xffffffffu, cmb, off));
      }
      const float na = fmaxf(m_a, cma), nb = fmaxf(m_b, cmb);
      const float ua = na == -INFINITY ? 0.f : na;  // all-masked guard
      const float ub = nb == -INFINITY ? 0.f : nb;
      const float alpha_a = ex2(m_a - ua), alpha_b = ex2(m_b - ub);
      const float pa0 = ex2(sa0 - ua), pa1 = ex2(sa1 - ua);
      const float pb0 = ex2(sb0 - ub), pb1 = ex2(sb1 - ub);
      l_a = l_a * alpha_a + pa0 + pa1;
      l_b = l_b * alpha_b + pb0 + pb1;
      m_a = na;
      m_b = nb;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        o[mt][0] *= alpha_a;
        o[mt][1] *= alpha_b;
        o[mt][2] *= alpha_a;
        o[mt][3] *= alpha_b;
      }
      // P[row][head] as bf16 8x8 tiles -> transposed into the B operand
      const uint32_t b0 = movmatrix_trans(pack_bf16(pa0, pb0));
      const uint32_t b1 = movmatrix_trans(pack_bf16(pa1, pb1));

      // ---- O^T += V^T . P^T over 8 tiles of 16 channels ----
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const int half = mt >> 2;
        const int row = row0 + mr + 8 * (mi >> 1);
        const int c16 = (mt & 3) * 2 + (mi & 1);
        const uint32_t addr =
            base + (2 + half) * kHalfBytes + row * 128 + ((c16 ^ (row & 7)) << 4);
        uint32_t a0, a1, a2, a3;
        ldmatrix_x4_trans(addr, a0, a1, a2, a3);
        mma_bf16_16816(o[mt], a0, a1, a2, a3, b0, b1);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (++stage == kStages) {
        stage = 0;
        phase ^= 1u;
      }
    }
    // A warp whose wait timed out still takes part in both barriers below,
    // so that the other consumer warps never block; all leave together.
    if (failed) *abort_flag = 1;

    // ---- merge the four warps' partial states ----
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l_a += __shfl_xor_sync(0xffffffffu, l_a, off);
      l_b += __shfl_xor_sync(0xffffffffu, l_b, off);
    }
    float* ro = red_o + cw * kHeads * kD;
    if (gq == 0) {
      red_ml[(cw * kHeads + 2 * qq) * 2 + 0] = m_a;
      red_ml[(cw * kHeads + 2 * qq) * 2 + 1] = l_a;
      red_ml[(cw * kHeads + 2 * qq + 1) * 2 + 0] = m_b;
      red_ml[(cw * kHeads + 2 * qq + 1) * 2 + 1] = l_b;
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      const int c = mt * 16 + gq;
      ro[(2 * qq) * kD + c] = o[mt][0];
      ro[(2 * qq + 1) * kD + c] = o[mt][1];
      ro[(2 * qq) * kD + c + 8] = o[mt][2];
      ro[(2 * qq + 1) * kD + c + 8] = o[mt][3];
    }
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumers) : "memory");
    {
      const int c = threadIdx.x;  // 0..127: one channel, all heads
      float* po = p.part_o + (size_t)item * kHeads * kD;
      float* pml = p.part_ml + (size_t)item * kHeads * 2;
#pragma unroll
      for (int hh = 0; hh < kHeads; ++hh) {
        float mw[kConsumers], M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumers; ++w) {
          mw[w] = red_ml[(w * kHeads + hh) * 2];
          M = fmaxf(M, mw[w]);
        }
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < kConsumers; ++w) {
            const float f = ex2(mw[w] - M);
            L = fmaf(red_ml[(w * kHeads + hh) * 2 + 1], f, L);
            O = fmaf(red_o[(w * kHeads + hh) * kD + c], f, O);
          }
        }
        po[hh * kD + c] = O;
        if (c == 0) {
          pml[hh * 2 + 0] = M;
          pml[hh * 2 + 1] = L;
        }
      }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumers) : "memory");
    if (*abort_flag) break;
  }
}

// One block per (batch, KV head): merge the splits of both heads of every
// pair and write o = O1/l1 - lambda * O2/l2 (bf16).
__global__ void v2_decode_combine_kernel(const float* __restrict__ part_o,
                                         const float* __restrict__ part_ml,
                                         const float* __restrict__ lambda,
                                         __nv_bfloat16* __restrict__ out, int Hkv, int group,
                                         int n_split) {
  const int bg = blockIdx.x;
  const int g = bg % Hkv, b = bg / Hkv;
  const int pl = threadIdx.x / kD;  // pair within the group
  const int c = threadIdx.x % kD;
  if (pl >= group / 2) return;
  const int ha = 2 * pl, hb = 2 * pl + 1;
  float Ma = -INFINITY, Mb = -INFINITY;
  for (int s = 0; s < n_split; ++s) {
    const float* ml = part_ml + ((size_t)bg * n_split + s) * kHeads * 2;
    Ma = fmaxf(Ma, ml[ha * 2]);
    Mb = fmaxf(Mb, ml[hb * 2]);
  }
  float La = 0.f, Lb = 0.f, Oa = 0.f, Ob = 0.f;
  for (int s = 0; s < n_split; ++s) {
    const size_t it = (size_t)bg * n_split + s;
    const float* ml = part_ml + it * kHeads * 2;
    const float* po = part_o + it * kHeads * kD;
    if (ml[ha * 2] != -INFINITY) {
      const float f = ex2(ml[ha * 2] - Ma);
      La = fmaf(ml[ha * 2 + 1], f, La);
      Oa = fmaf(po[ha * kD + c], f, Oa);
    }
    if (ml[hb * 2] != -INFINITY) {
      const float f = ex2(ml[hb * 2] - Mb);
      Lb = fmaf(ml[hb * 2 + 1], f, Lb);
      Ob = fmaf(po[hb * kD + c], f, Ob);
    }
  }
  const int Hp = Hkv * group / 2;
  const int pair = g * (group / 2) + pl;
  const float r = Oa / La - lambda[pair] * (Ob / Lb);
  out[((size_t)b * Hp + pair) * kD + c] = __float2bfloat16_rn(r);
}

// V1 form: one block per (batch, head), 128 threads = channels.  Merges the
// splits of the head's two branches, forms o = O1/l1 - lambda * O2/l2 and,
// with the norm, y = o / sqrt(mean(o^2) + eps) * g * (1 - lambda_init).
__global__ void v1_decode_combine_tc_kernel(const float* __restrict__ part_o,
                                            const float* __restrict__ part_ml,
                                            const float* __restrict__ lambda,
                                            __nv_bfloat16* __restrict__ out, int H, int n_split,
                                            int apply_norm, const float* __restrict__ gain,
                                            float eps, float post_scale) {
  __shared__ float red[kD / 32];
  const int bh = blockIdx.x;
  const int h = bh % H;
  const int c = threadIdx.x;
  float Ma = -INFINITY, Mb = -INFINITY;
  for (int s = 0; s < n_split; ++s) {
    const float* ml = part_ml + ((size_t)bh * n_split + s) * kHeads * 2;
    Ma = fmaxf(Ma, ml[0]);
    Mb = fmaxf(Mb, ml[2]);
  }
  float La = 0.f, Lb = 0.f, Oa = 0.f, Ob = 0.f;
  for (int s = 0; s < n_split; ++s) {
    const size_t it = (size_t)bh * n_split + s;
    const float* ml = part_ml + it * kHeads * 2;
    const float* po = part_o + it * kHeads * kD;
    if (ml[0] != -INFINITY) {
      const float f = ex2(ml[0] - Ma);
      La = fmaf(ml[1], f, La);
      Oa = fmaf(po[c], f, Oa);
    }
    if (ml[2] != -INFINITY) {
      const float f = ex2(ml[2] - Mb);
      Lb = fmaf(ml[3], f, Lb);
      Ob = fmaf(po[kD + c], f, Ob);
    }
  }
  float o = Oa / La - lambda[h] * (Ob / Lb);
  if (apply_norm) {
    float ss = o * o;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if ((c & 31) == 0) red[c >> 5] = ss;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < kD / 32; ++w) tot += red[w];
    o = o * (post_scale / sqrtf(tot * (1.0f / kD) + eps)) * (gain ? gain[c] : 1.f);
  }
  out[(size_t)bh * kD + c] = __float2bfloat16_rn(o);
}

}  // namespace

V2DecodePlan plan_v2_decode(int batch, int n_kv_heads, int max_len, int num_sms) {
  // Pick the split count that minimises the rows the busiest persistent CTA
  // streams (static round-robin over equal items), counting a fixed
  // per-item overhead of one chunk.
  const long units = (long)batch * n_kv_heads;
  const int max_split = (max_len + kChunk - 1) / kChunk;
  V2DecodePlan best{1, 0, 0, 0};
  double best_cost = 1e300;
  for (int ns = 1; ns <= max_split && ns <= 256; ++ns) {
    int sl = (max_len + ns - 1) / ns;
    sl = (sl + kChunk - 1) / kChunk * kChunk;
    const int ns_eff = (max_len + sl - 1) / sl;
    const long items = units * ns_eff;
    const long grid = items < num_sms ? items : num_sms;
    const long per_cta = (items + grid - 1) / grid;
    const double cost = (double)per_cta * (sl + kChunk);
    if (cost < best_cost * 0.999) {
      best_cost = cost;
      best = {ns_eff, sl, (int)items, (int)grid};
    }
  }
  return best;
}

V2DecodePlan plan_v2_decode_capped(int batch, int n_kv_heads, int max_len, int num_sms,
                                   size_t max_bytes) {
  const long units = (long)batch * n_kv_heads;
  const int max_split = (max_len + kChunk - 1) / kChunk;
  const size_t per_item = (size_t)kHeads * (kD + 2) * sizeof(float);
  V2DecodePlan best{0, 0, 0, 0};
  double best_cost = 1e300;
  for (int ns = 1; ns <= max_split && ns <= 256; ++ns) {
    int sl = (max_len + ns - 1) / ns;
    sl = (sl + kChunk - 1) / kChunk * kChunk;
    const int ns_eff = (max_len + sl - 1) / sl;
    const long items = units * ns_eff;
    if ((size_t)items * per_item > max_bytes) break;  // more splits only grow the workspace
    const long grid = items < num_sms ? items : num_sms;
    const long per_cta = (items + grid - 1) / grid;
    const double cost = (double)per_cta * (sl + kChunk);
    if (cost < best_cost * 0.999) {
      best_cost = cost;
      best = {ns_eff, sl, (int)items, (int)grid};
    }
  }
  return best;
}

size_t v2_decode_workspace_bytes(const V2DecodePlan& plan) {
  return (size_t)plan.n_items * kHeads * (kD + 2) * sizeof(float);
}

cudaError_t launch_v2_decode(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const void* q,
                             const int* lens, int max_len, int window, void* out, int batch,
                             int n_q_heads, int n_kv_heads, const float* lambda,
                             const V2DecodePlan& plan, void* workspace, int* dev_status,
                             cudaStream_t stream) {
  Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.v1 = 0;
  p.lens = lens;
  p.max_len = max_len;
  p.window = window;
  p.Hq = n_q_heads;
  p.Hkv = n_kv_heads;
  p.group = n_q_heads / n_kv_heads;
  p.split_len = plan.split_len;
  p.n_split = plan.n_split;
  p.n_items = plan.n_items;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt(128.0));
  p.part_o = static_cast<float*>(workspace);
  p.part_ml = p.part_o + (size_t)plan.n_items * kHeads * kD;
  p.dev_status = dev_status;
  cudaError_t e = cudaFuncSetAttribute(v2_decode_split_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  v2_decode_split_kernel<<<plan.grid, kThreads, kSmemBytes, stream>>>(tm_k, tm_v, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  v2_decode_combine_kernel<<<batch * n_kv_heads, (p.group / 2) * kD, 0, stream>>>(
      p.part_o, p.part_ml, lambda, static_cast<__nv_bfloat16*>(out), n_kv_heads, p.group,
      plan.n_split);
  return cudaGetLastError();
}

cudaError_t launch_v1_decode_tc(const CUtensorMap& tm_k, const CUtensorMap& tm_v, const void* q,
                                const int* lens, int max_len, int window, void* out, int batch,
                                int n_heads, const float* lambda, int apply_norm,
                                const float* norm_weight, float eps, float post_scale,
                                const V2DecodePlan& plan, void* workspace, int* dev_status,
                                cudaStream_t stream) {
  Params p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.v1 = 1;
  p.lens = lens;
  p.max_len = max_len;
  p.window = window;
  p.Hq = 2 * n_heads;
  p.Hkv = n_heads;
  p.group = 2;
  p.split_len = plan.split_len;
  p.n_split = plan.n_split;
  p.n_items = plan.n_items;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt(64.0));  // one branch is 64 wide
  p.part_o = static_cast<float*>(workspace);
  p.part_ml = p.part_o + (size_t)plan.n_items * kHeads * kD;
  p.dev_status = dev_status;
  cudaError_t e = cudaFuncSetAttribute(v2_decode_split_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  v2_decode_split_kernel<<<plan.grid, kThreads, kSmemBytes, stream>>>(tm_k, tm_v, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  v1_decode_combine_tc_kernel<<<batch * n_heads, kD, 0, stream>>>(
      p.part_o, p.part_ml, lambda, static_cast<__nv_bfloat16*>(out), n_heads, plan.n_split,
      apply_norm, norm_weight, eps, post_scale);
  return cudaGetLastError();
}

}  // namespace da
