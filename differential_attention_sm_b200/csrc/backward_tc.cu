// backward_tc.cu — fused backward of differential attention on the 5th-
// generation tensor cores (tcgen05 + tensor memory + TMA), both forms.
//
// Forward: glossary page "Differential Transformer", section "Cómo funciona
// la atención diferencial"; lesson "Atención Diferencial (V2)", sections "La
// idea diferencial" and "V1 vs V2: la diferencia".  With P_r the two softmax
// maps, o = P_1 V - lambda P_2 V, do the gradient of the pre-norm output,
// do_1 = do, do_2 = -lambda do and D_r = do_r . (P_r V) per row, the
// gradients of each branch are the usual ones of softmax attention:
//     dP_r = do_r V^T,  dS_r = P_r (dP_r - D_r),
//     dQ_r = dS_r K_r / sqrt(d),  dK_r += dS_r^T Q_r / sqrt(d),  dV += P_r^T do_r.
// The training forward (prefill kernel with saves) provides the per-row
// log2-sum-exp of each branch, so P_r = 2^(s sc - lse_r) is recomputed
// tile by tile and nothing of size N x N ever reaches memory.
//
// Two kernels:
//   * dq kernel, one CTA per 128 query rows of a head (V1) or head pair
//     (V2), walking 64-key tiles like the forward: per branch, S_r into
//     tensor memory (SS MMA); one dP = do_1 V^T for both branches, since
//     do_2 = -lambda do_1 makes dP_2 = -lambda dP_1; dS_r written as bf16 by
//     the softmax-backward warps, then dQ_r += dS_r K_r in tensor memory.  V1
//     writes dS_r back over S_r (TS MMA); V2, whose tensor memory has no
//     second S buffer, writes it to swizzled shared memory (SS MMA) so that
//     S_r(j+1) only waits for S_r(j) to be loaded.  The softmax-backward
//     warps form P as soon as S_r has landed and wait for dP only after
//     that.  Warps: 0-15 softmax backward (thread = query row; two
//     warpgroups per branch, one per half of the tile's 64 key columns),
//     16 TMA producer, 17 / 19 the S_1 / S_2 issuers and 18 the dP issuer
//     (one thread per product stream, as in the forward), 20 / 21 dQ issuers.
//   * dkdv kernel, one CTA per 128 keys of a head (V1) or KV head (V2),
//     walking 64-query tiles (and, for V2, every pair that reads the KV
//     head): S^T = K_r Q_r^T and dP^T = V do_r^T (SS), P^T and dS^T written
//     back as bf16 by the softmax-backward warps (thread = key row), then
//     dV += P^T do_r and dK_r += dS^T Q_r (TS) in tensor memory.  Each
//     accumulator has one issuing thread, so its order is fixed.  The two
//     halves of each step's handshake are separate: P^T is written (and the
//     dV product released) as soon as S^T lands, dS^T once dP^T has; the
//     next S^T into a buffer waits only for dV, the next dP^T only for dK.
//     Warps: 0-15 softmax backward (two warpgroups per step parity, one per
//     half of the step's 64 query columns), 16 producer, 17 S^T issuer,
//     18 dP^T issuer, 19 dV issuer, 20 dK issuer.
// Every wait is bounded (DA_ERR_DEVICE_TIMEOUT in the status word).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace da {
namespace {

constexpr int kBox128 = 128 * 64 * 2;  // TMA box: 128 rows x 64 bf16 = 16 KB
constexpr int kBox64 = 64 * 64 * 2;    // TMA box: 64 rows x 64 bf16 = 8 KB
constexpr int kTile128 = 2 * kBox128;  // 128 x 128 bf16
constexpr int kTile64 = 2 * kBox64;    // 64 x 128 bf16

struct BwdParams {
  int batch, seqlen, units, pairs_per_kv, causal, window;
  int npad;          // row stride of lse and D (seqlen rounded up to 64)
  float scale_log2;  // log2(e) / sqrt(d)
  float scale;       // 1 / sqrt(d)
  const float* lse;  // [B][units][2][npad]: p = 2^(s * scale_log2 - lse)
  const float* Dv;   // [B][units][2][npad]: D_r = do_r . O_r
  const float* lambda;  // [units]: do_2 = -lambda do_1, so dP_2 = -lambda dP_1
  float* dq;         // like q
  float* dk;         // like k
  float* dv;         // like v
  int q_heads, kv_heads;
  int n_qtiles;      // dq grid: ceil(N / 128) per unit
  int n_ktiles;      // dkdv grid: ceil(N / 128) per KV unit
  int group_q;       // dq: units whose tiles are interleaved, heaviest first
  int group_kv;      // dkdv: KV units whose tiles are interleaved, heaviest first
  int* dev_status;
};

// Block index -> (tile index, unit): blocks are numbered by groups of `group`
// units, and within a group by tile index first, so the tiles with the same
// index (the same amount of causal work) of the group's units run together,
// heaviest first, and each group ends with light tiles.
__device__ __forceinline__ void grouped_tile(int bid, int n_tiles, int n_units, int group,
                                             int* tile, int* unit) {
  const int per_group = group * n_tiles;
  const int g = bid / per_group, rr = bid % per_group;
  const int g_size = min(group, n_units - g * group);
  *tile = rr / g_size;
  *unit = g * group + rr % g_size;
}

// ===================================================================== dQ
// warps 0-15: softmax backward (branch r = (warp >> 2) & 1, key-column half
// h = warp >> 3); 16 producer; 17 / 19 the S_1 / S_2 issuers and 18 the dP
// issuer (17 owns tensor memory); 20 / 21 the dQ_1 / dQ_2 issuers
constexpr int kDqThreads = 704;
constexpr int kDqProducer = 16;
constexpr int kDqStages = 2;

struct DqBarriers {
  uint64_t q_full;
  uint64_t k_full[kDqStages], k_empty[kDqStages];
  uint64_t v_full[kDqStages], v_empty[kDqStages];
  uint64_t s_full[2][2];   // [branch][S buffer]: S_r landed
  uint64_t dp_full[2];     // [0]: dP_1 landed (dP_2 = -lambda dP_1; [1] unused)
  uint64_t ds_full[2][2];  // [branch][column half]: dS_r written back (and dP_r read)
  uint64_t dq_done[2][2];  // [branch][S buffer]: the dQ product of a tile has read its dS
  uint64_t s_free[2];      // [branch], V2: the softmax backward has loaded S_r
  uint32_t tmem_base;
  int abort_flag;
};

template <int kForm, bool kWindow>
__global__ void __launch_bounds__(kDqThreads, 1)
    diffattn_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_do,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const BwdParams p) {
  constexpr int D = kForm == 1 ? 64 : 128;  // one branch's query width
  constexpr uint32_t kQBytes = kForm == 1 ? kTile128 : 2 * kTile128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sdO = sQ + kQBytes;                     // do_1: 128 x 128
  uint8_t* sK = sdO + kTile128;                    // stages x 64 x 128
  uint8_t* sV = sK + kDqStages * kTile64;
  // V2: dS_r (128 queries x 64 keys bf16, 128-byte swizzle, K-major) per branch
  uint8_t* sDS = sV + kDqStages * kTile64;
  DqBarriers* bars = reinterpret_cast<DqBarriers*>(sDS + (kForm == 2 ? 2 * kBox128 : 0));

  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  int mt, bu;  // heavy tiles first within each group of units
  grouped_tile((int)blockIdx.x, p.n_qtiles, p.batch * p.units, p.group_q, &mt, &bu);
  mt = p.n_qtiles - 1 - mt;
  const int hh = bu % p.units, b = bu / p.units;
  const int kvh = kForm == 1 ? hh : hh / p.pairs_per_kv;
  const int q0 = mt * 128;
  const int key_end = p.causal ? min(q0 + 128, p.seqlen) : p.seqlen;
  const int kv0 = kWindow ? max(0, q0 - p.window + 1) / 64 : 0;
  const int n_kv = (key_end + 63) / 64 - kv0;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kDqStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 4);  // both branches' S and dQ products read K
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);  // the one dP product reads V
    }
    for (int r = 0; r < 2; ++r) {
      mbar_init(&bars->s_full[r][0], 1);
      mbar_init(&bars->s_full[r][1], 1);
      mbar_init(&bars->dp_full[r], 1);
      mbar_init(&bars->ds_full[r][0], 128);
      mbar_init(&bars->ds_full[r][1], 128);
      mbar_init(&bars->dq_done[r][0], 1);
      mbar_init(&bars->dq_done[r][1], 1);
      mbar_init(&bars->s_free[r], 256);
    }
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kDqProducer + 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // tensor-memory columns: S_r, dP_r (64 each), dQ_r (D each).  V1 leaves room
  // for a second S buffer per branch at [384, 512), so S_r(j+1) can be computed
  // while dS_r(j), written back over S_r(j), still waits for its dQ product.  V2
  // has no room for one; its dS_r goes to shared memory instead, so S_r(j+1)
  // only waits for the softmax backward to have loaded S_r(j).
  constexpr int kSBufs = kForm == 1 ? 2 : 1;
  auto colS = [](int r, int j) {
    return (uint32_t)((kSBufs == 2 && (j & 1)) ? 384 + 64 * r : 128 * r);
  };
  auto colP = [](int r) { return (uint32_t)(128 * r + 64); };
  auto colQ = [](int r) { return (uint32_t)(256 + D * r); };
  bool failed = false;

  if (warp == kDqProducer) {
    if (lane == 0) {  // ---------------------------------------------- producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&bars->q_full, kQBytes + kTile128);
      if (kForm == 1) {
        tma_load_4d(sQ, &tm_q, &bars->q_full, 0, hh, q0, b);
        tma_load_4d(sQ + kBox128, &tm_q, &bars->q_full, 64, hh, q0, b);
      } else {
        for (int r = 0; r < 2; ++r) {
          tma_load_4d(sQ + r * kTile128, &tm_q, &bars->q_full, 0, 2 * hh + r, q0, b);
          tma_load_4d(sQ + r * kTile128 + kBox128, &tm_q, &bars->q_full, 64, 2 * hh + r, q0, b);
        }
      }
      tma_load_4d(sdO, &tm_do, &bars->q_full, 0, 2 * hh, q0, b);
      tma_load_4d(sdO + kBox128, &tm_do, &bars->q_full, 64, 2 * hh, q0, b);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % kDqStages;
        const uint32_t ph = (uint32_t)(j / kDqStages) & 1u;
        const int row = (kv0 + j) * 64;
        if (!mbar_wait(&bars->k_empty[s], ph ^ 1u, p.dev_status, &failed)) break;
        mbar_arrive_expect_tx(&bars->k_full[s], kTile64);
        tma_load_4d(sK + s * kTile64, &tm_k, &bars->k_full[s], 0, kvh, row, b);
        tma_load_4d(sK + s * kTile64 + kBox64, &tm_k, &bars->k_full[s], 64, kvh, row, b);
        if (!mbar_wait(&bars->v_empty[s], ph ^ 1u, p.dev_status, &failed)) break;
        mbar_arrive_expect_tx(&bars->v_full[s], kTile64);
        tma_load_4d(sV + s * kTile64, &tm_v, &bars->v_full[s], 0, kvh, row, b);
        tma_load_4d(sV + s * kTile64 + kBox64, &tm_v, &bars->v_full[s], 64, kvh, row, b);
      }
    }
  } else if (warp >= kDqProducer + 1 && warp <= kDqProducer + 3) {
    // ---- S_r issuer (kind 0, warp 17 + 2r) or the dP issuer (kind 1, warp 18):
    // dP_2 = -lambda dP_1, so only branch 1's dP product is computed
    const int r = (warp - kDqProducer - 1) >> 1, kind = (warp - kDqProducer - 1) & 1;
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(sQ), do_addr = smem_u32(sdO);
      constexpr uint32_t idS = idesc_bf16_f32(128, 64, false, false);
      if (mbar_wait(&bars->q_full, 0, p.dev_status, &failed)) {
        for (int j = 0; j < n_kv; ++j) {
          const int s = j % kDqStages;
          const uint32_t ph = (uint32_t)(j / kDqStages) & 1u;
          if (!mbar_wait(kind == 0 ? &bars->k_full[s] : &bars->v_full[s], ph, p.dev_status,
                         &failed))
            break;
          // S_r's buffer last held dS_r(j - kSBufs): its dQ product must have
          // read it; dP_r's buffer is free once the softmax backward has read
          // dP_r(j-1)
          if (kForm == 1 && kind == 0 && j >= kSBufs &&
              !mbar_wait(&bars->dq_done[r][(j - kSBufs) & 1], (uint32_t)((j - kSBufs) >> 1) & 1u,
                         p.dev_status, &failed))
            break;
          if (kForm == 2 && kind == 0 && j >= 1 &&
              !mbar_wait(&bars->s_free[r], (uint32_t)(j - 1) & 1u, p.dev_status, &failed))
            break;
          // dP's buffer is free once both branches' softmax backward has read dP(j-1)
          if (kind == 1 && j > 0 &&
              !(mbar_wait(&bars->ds_full[0][0], (uint32_t)(j - 1) & 1u, p.dev_status, &failed) &&
                mbar_wait(&bars->ds_full[0][1], (uint32_t)(j - 1) & 1u, p.dev_status, &failed) &&
                mbar_wait(&bars->ds_full[1][0], (uint32_t)(j - 1) & 1u, p.dev_status, &failed) &&
                mbar_wait(&bars->ds_full[1][1], (uint32_t)(j - 1) & 1u, p.dev_status, &failed)))
            break;
          tc_fence_after();
          if (kind == 0) {
            const uint32_t kt = smem_u32(sK) + s * kTile64;
            for (int kk = 0; kk < D / 16; ++kk) {
              uint32_t a, bb;
              if (kForm == 1) {
                a = q_addr + r * kBox128 + kk * 32;
                bb = kt + r * kBox64 + kk * 32;
              } else {
                a = q_addr + r * kTile128 + (kk >> 2) * kBox128 + (kk & 3) * 32;
                bb = kt + (kk >> 2) * kBox64 + (kk & 3) * 32;
              }
              tc_mma_ss(tmem + colS(r, j), smem_desc_sw128(a, 16, 1024),
                        smem_desc_sw128(bb, 16, 1024), idS, kk > 0 ? 1u : 0u);
            }
            tc_commit(&bars->s_full[r][j % kSBufs]);
            tc_commit(&bars->k_empty[s]);
          } else {
            const uint32_t vt = smem_u32(sV) + s * kTile64;
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t a = do_addr + (kk >> 2) * kBox128 + (kk & 3) * 32;
              const uint32_t bb = vt + (kk >> 2) * kBox64 + (kk & 3) * 32;
              tc_mma_ss(tmem + colP(0), smem_desc_sw128(a, 16, 1024),
                        smem_desc_sw128(bb, 16, 1024), idS, kk > 0 ? 1u : 0u);
            }
            tc_commit(&bars->dp_full[0]);
            tc_commit(&bars->v_empty[s]);
          }
        }
      }
    }
  } else if (warp == kDqProducer + 4 || warp == kDqProducer + 5) {
    if (lane == 0) {  // ------------------------------------ dQ_r issuer, r = warp - 20
      const int r = warp - kDqProducer - 4;
      constexpr uint32_t idQ = idesc_bf16_f32(128, D, false, true);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % kDqStages;
        if (!mbar_wait(&bars->k_full[s], (uint32_t)(j / kDqStages) & 1u, p.dev_status, &failed))
          break;
        const uint32_t kt = smem_u32(sK) + s * kTile64 + (kForm == 1 ? r * kBox64 : 0);
        // each column half's products go out as soon as that half's dS_r is written
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait(&bars->ds_full[r][h], (uint32_t)j & 1u, p.dev_status, &failed)) break;
          tc_fence_after();
          for (int kk = 2 * h; kk < 2 * h + 2; ++kk) {  // 16 keys each; B = K_r, MN-major
            // keys [32h, 32h + 32) of a tile are packed into columns [32h, 32h + 16)
            // of the S buffer (each column half writes inside the columns it read)
            if (kForm == 1)  // A = dS_r in tensor memory
              tc_mma_ts(tmem + colQ(r), tmem + colS(r, j) + 32 * h + 8 * (kk & 1),
                        smem_desc_sw128(kt + kk * 2048, kBox64, 1024), idQ,
                        (j > 0 || kk > 0) ? 1u : 0u);
            else  // A = dS_r in shared memory, K-major
              tc_mma_ss(tmem + colQ(r),
                        smem_desc_sw128(smem_u32(sDS) + r * kBox128 + kk * 32, 16, 1024),
                        smem_desc_sw128(kt + kk * 2048, kBox64, 1024), idQ,
                        (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        if (failed) break;
        tc_commit(&bars->dq_done[r][j & 1]);
        tc_commit(&bars->k_empty[s]);
      }
    }
  } else {
    // ------------------------- softmax backward, branch r, key columns of half h
    // Each tile's 64 key columns are split between two warpgroups per branch,
    // which halves every thread's serial chain and gives each sub-partition
    // four softmax warps to interleave.
    const int r = (warp >> 2) & 1;
    const int h = warp >> 3;
    const int row = (warp & 3) * 32 + lane;
    const int qrow = q0 + row;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const int lim = p.causal ? min(qrow + 1, p.seqlen) : p.seqlen;
    const int lo = kWindow ? max(0, qrow - p.window + 1) : 0;
    const size_t vrow = (((size_t)b * p.units + hh) * 2 + r) * p.npad + qrow;
    const float lse = qrow < p.seqlen ? p.lse[vrow] : 0.f;
    const float Dr = qrow < p.seqlen ? p.Dv[vrow] : 0.f;
    const float sc = p.scale_log2;
    const uint64_t sc2 = f2pack(sc, sc), nl2 = f2pack(-lse, -lse), nd2 = f2pack(-Dr, -Dr);
    const float mr = r == 0 ? 1.f : -p.lambda[hh];  // dP_r = mr dP_1
    const uint64_t mr2 = f2pack(mr, mr);
    // Two passes per tile: P = 2^(s sc - lse) as soon as S_r has landed (the
    // dP_r product may still be in flight), then dS = P (dP - D) from the same
    // P, kept in registers as bf16 pairs, written back over S_r.
    for (int j = 0; j < n_kv; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[r][j % kSBufs],
                                             (uint32_t)(j / kSBufs) & 1u, p.dev_status,
                                             &failed))) {
        failed = true;
        break;
      }
      tc_fence_after();
      const int k0 = (kv0 + j) * 64 + 32 * h;  // first key of this half
      // halves fully inside every row's visible range skip the masks
      const bool full = __all_sync(0xffffffffu, k0 + 32 <= lim && (!kWindow || k0 >= lo));
      uint32_t pp[16];
      {
        uint32_t sv[32];
        tmem_ld32(tmem + lane_off + colS(r, j) + 32 * h, sv);
        tc_wait_ld();
        if (kForm == 2) {  // S_r fully loaded: its buffer may take S_r(j+1)
          tc_fence_before();
          mbar_arrive(&bars->s_free[r]);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float x0, x1;
          f2unpack(fma2(f2pack(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])),
                        sc2, nl2),
                   x0, x1);
          float p0 = ex2(x0), p1 = ex2(x1);
          if (!full) {
            const int key = k0 + 2 * e;
            p0 = (key < lim && (!kWindow || key >= lo)) ? p0 : 0.f;
            p1 = (key + 1 < lim && (!kWindow || key + 1 >= lo)) ? p1 : 0.f;
          }
          pp[e] = pack_bf16(p0, p1);
        }
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->dp_full[0], (uint32_t)j & 1u, p.dev_status,
                                             &failed))) {
        failed = true;
        break;
      }
      // V2: the dQ product of the previous tile must have read dS_r out of
      // shared memory before it is overwritten
      if (kForm == 2 && j >= 1 &&
          !__all_sync(0xffffffffu, mbar_wait(&bars->dq_done[r][(j - 1) & 1],
                                             (uint32_t)((j - 1) >> 1) & 1u, p.dev_status,
                                             &failed))) {
        failed = true;
        break;
      }
      tc_fence_after();
      {
        uint32_t dp[32], pk[16];
        tmem_ld32(tmem + lane_off + colP(0) + 32 * h, dp);
        tc_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const uint32_t pb = pp[e];
          float ds0, ds1;
          f2unpack(fma2(f2pack(bf16lo(pb), bf16hi(pb)),
                        fma2(f2pack(__uint_as_float(dp[2 * e]), __uint_as_float(dp[2 * e + 1])),
                             mr2, nd2),
                        0ull),
                   ds0, ds1);
          pk[e] = pack_bf16(ds0, ds1);
        }
        if (kForm == 1) {
          tmem_st16(tmem + lane_off + colS(r, j) + 32 * h, pk);
        } else {
          // row `row` of the 128-byte-swizzled tile: 16-byte chunk c (8 keys)
          // sits at chunk position c ^ (row & 7)
          uint8_t* drow = sDS + r * kBox128 + row * 128;
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const int ch = 4 * h + c4;
            *reinterpret_cast<uint4*>(drow + ((ch ^ (row & 7)) << 4)) =
                make_uint4(pk[4 * c4], pk[4 * c4 + 1], pk[4 * c4 + 2], pk[4 * c4 + 3]);
          }
        }
      }
      if (kForm == 2) fence_proxy_async_smem();  // visible to the tensor core
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->ds_full[r][h]);
    }
    __syncwarp();
    if (failed) bars->abort_flag = 1;
    if (n_kv > 0)
      mbar_wait(&bars->dq_done[r][(n_kv - 1) & 1], (uint32_t)((n_kv - 1) >> 1) & 1u,
                p.dev_status, &failed);
    tc_fence_after();
    const bool store = qrow < p.seqlen;
    // each half writes half of this branch's dQ_r columns
    float* dst = (kForm == 1
                      ? p.dq + (((size_t)b * p.seqlen + qrow) * p.q_heads + hh) * 128 + 64 * r
                      : p.dq + (((size_t)b * p.seqlen + qrow) * p.q_heads + 2 * hh + r) * 128) +
                 (D / 2) * h;
#pragma unroll 1
    for (int c = 0; c < D / 64; ++c) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_off + colQ(r) + (D / 2) * h + 32 * c, v);
      tc_wait_ld();
      if (store && !bars->abort_flag) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          float4 f;
          f.x = __uint_as_float(v[e]) * p.scale;
          f.y = __uint_as_float(v[e + 1]) * p.scale;
          f.z = __uint_as_float(v[e + 2]) * p.scale;
          f.w = __uint_as_float(v[e + 3]) * p.scale;
          *reinterpret_cast<float4*>(dst + 32 * c + e) = f;
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kDqProducer + 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// =================================================================== dK, dV
// warps 0-15: softmax backward (step parity w = (warp >> 2) & 1, query-column
// half h = warp >> 3); 16 producer; 17 S^T issuer (owns tensor memory);
// 18 dP^T issuer; 19 dV issuer; 20 dK issuer
constexpr int kKvThreads = 672;
constexpr int kKvProducer = 16;
constexpr int kKvStages = 4;  // 4 ran 2.7 % faster than 3 on the V2 backward; 5 do not fit
constexpr int kStageQ = kTile64;                       // Q_r tile (V1 uses one box)
// + dO_r tile + lse/D vectors; a multiple of 1 KB keeps every stage's
// 128-byte-swizzled tiles on the 1 KB alignment their descriptors assume
constexpr int kStageBytes = kStageQ + kTile64 + 1024;
static_assert(kStageBytes % 1024 == 0, "stage alignment");

struct KvBarriers {
  uint64_t kv_full;
  uint64_t qd_full[kKvStages], qd_empty[kKvStages];
  uint64_t s_full[2], dp_full[2];        // S^T, dP^T landed [buffer]
  uint64_t p_full[2][2], ds_full[2][2];  // P^T, dS^T written back [buffer][column half]
  uint64_t pt_free[2], dst_free[2];      // dV, dK products done with them [buffer]
  uint64_t acc_done;
  uint32_t tmem_base;
  int abort_flag;
};

template <int kForm, bool kWindow>
__global__ void __launch_bounds__(kKvThreads, 1)
    diffattn_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                             const __grid_constant__ CUtensorMap tm_do,
                             const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ CUtensorMap tm_v, const BwdParams p) {
  constexpr int D = kForm == 1 ? 64 : 128;
  constexpr uint32_t kQStepBytes = kForm == 1 ? kBox64 : kTile64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;                  // 128 keys x 128
  uint8_t* sV = sK + kTile128;
  uint8_t* sStage = sV + kTile128;     // stages x (Q, dO, lse[64], D[64])
  KvBarriers* bars = reinterpret_cast<KvBarriers*>(sStage + kKvStages * kStageBytes);

  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  int kt_idx, bg;  // causal: key tile 0 sees the most queries, so it goes first
  grouped_tile((int)blockIdx.x, p.n_ktiles, p.batch * p.kv_heads, p.group_kv, &kt_idx, &bg);
  const int g = bg % p.kv_heads, b = bg / p.kv_heads;  // V1: g is the head
  const int k0 = kt_idx * 128;
  const int members = kForm == 1 ? 1 : p.pairs_per_kv;
  const int n_qt = (p.seqlen + 63) / 64;
  const int i0 = p.causal ? k0 / 64 : 0;
  int i1 = n_qt;
  if (kWindow) i1 = min(i1, (k0 + 127 + p.window - 1) / 64 + 1);
  const int n_steps = (i1 - i0) * members * 2;

  if (threadIdx.x == 0) {
    mbar_init(&bars->kv_full, 1);
    for (int s = 0; s < kKvStages; ++s) {
      mbar_init(&bars->qd_full[s], 1);
      mbar_init(&bars->qd_empty[s], 4);  // all four products read Q_r or dO_r
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bars->s_full[w], 1);
      mbar_init(&bars->dp_full[w], 1);
      for (int h = 0; h < 2; ++h) {
        mbar_init(&bars->p_full[w][h], 128);
        mbar_init(&bars->ds_full[w][h], 128);
      }
      mbar_init(&bars->pt_free[w], 1);
      mbar_init(&bars->dst_free[w], 1);
    }
    mbar_init(&bars->acc_done, 2);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kKvProducer + 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  // columns: S^T_w [128w, +64), dP^T_w [128w+64, +64), dV [256, 384), dK [384, 512)
  constexpr uint32_t kColDV = 256, kColDK = 384;
  bool failed = false;
  // step s -> (query tile, member, branch): branch innermost
  auto step_q0 = [&](int s) { return (i0 + (s >> 1) / members) * 64; };
  auto step_unit = [&](int s) {
    return kForm == 1 ? g : g * p.pairs_per_kv + (s >> 1) % members;
  };

  if (warp == kKvProducer) {
    if (lane == 0) {  // ---------------------------------------------- producer
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_do);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&bars->kv_full, 2 * kTile128);
      tma_load_4d(sK, &tm_k, &bars->kv_full, 0, g, k0, b);
      tma_load_4d(sK + kBox128, &tm_k, &bars->kv_full, 64, g, k0, b);
      tma_load_4d(sV, &tm_v, &bars->kv_full, 0, g, k0, b);
      tma_load_4d(sV + kBox128, &tm_v, &bars->kv_full, 64, g, k0, b);
      for (int s = 0; s < n_steps; ++s) {
        const int st = s % kKvStages;
        const uint32_t ph = (uint32_t)(s / kKvStages) & 1u;
        const int r = s & 1, q0 = step_q0(s), u = step_unit(s);
        if (!mbar_wait(&bars->qd_empty[st], ph ^ 1u, p.dev_status, &failed)) break;
        uint8_t* sq = sStage + st * kStageBytes;
        uint8_t* sdo = sq + kStageQ;
        float* svec = reinterpret_cast<float*>(sdo + kTile64);
        mbar_arrive_expect_tx(&bars->qd_full[st], kQStepBytes + kTile64 + 512);
        if (kForm == 1) {
          tma_load_4d(sq, &tm_q, &bars->qd_full[st], 64 * r, u, q0, b);
        } else {
          tma_load_4d(sq, &tm_q, &bars->qd_full[st], 0, 2 * u + r, q0, b);
          tma_load_4d(sq + kBox64, &tm_q, &bars->qd_full[st], 64, 2 * u + r, q0, b);
        }
        tma_load_4d(sdo, &tm_do, &bars->qd_full[st], 0, 2 * u + r, q0, b);
        tma_load_4d(sdo + kBox64, &tm_do, &bars->qd_full[st], 64, 2 * u + r, q0, b);
        const size_t vrow = (((size_t)b * p.units + u) * 2 + r) * p.npad + q0;
        bulk_load(svec, p.lse + vrow, 256, &bars->qd_full[st]);
        bulk_load(svec + 64, p.Dv + vrow, 256, &bars->qd_full[st]);
      }
    }
  } else if (warp == kKvProducer + 1 || warp == kKvProducer + 2) {
    if (lane == 0) {  // -------------------------------------- S^T issuer and dP^T issuer
      const bool is_s = warp == kKvProducer + 1;
      constexpr uint32_t idS = idesc_bf16_f32(128, 64, false, false);
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      if (mbar_wait(&bars->kv_full, 0, p.dev_status, &failed)) {
        for (int s = 0; s < n_steps; ++s) {
          const int st = s % kKvStages, w = s & 1, r = s & 1;
          if (!mbar_wait(&bars->qd_full[st], (uint32_t)(s / kKvStages) & 1u, p.dev_status,
                         &failed))
            break;
          // the buffer last held step s-2's P^T (read by the dV product) or
          // dS^T (read by the dK product)
          if (s >= 2 && !mbar_wait(is_s ? &bars->pt_free[w] : &bars->dst_free[w],
                                   (uint32_t)((s - 2) >> 1) & 1u, p.dev_status, &failed))
            break;
          tc_fence_after();
          const uint32_t sq = smem_u32(sStage) + st * kStageBytes, sdo = sq + kStageQ;
          if (is_s) {
            for (int kk = 0; kk < D / 16; ++kk) {
              uint32_t a, bb;
              if (kForm == 1) {
                a = k_addr + r * kBox128 + kk * 32;
                bb = sq + kk * 32;
              } else {
                a = k_addr + (kk >> 2) * kBox128 + (kk & 3) * 32;
                bb = sq + (kk >> 2) * kBox64 + (kk & 3) * 32;
              }
              tc_mma_ss(tmem + 128 * w, smem_desc_sw128(a, 16, 1024),
                        smem_desc_sw128(bb, 16, 1024), idS, kk > 0 ? 1u : 0u);
            }
          } else {
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t a = v_addr + (kk >> 2) * kBox128 + (kk & 3) * 32;
              const uint32_t bb = sdo + (kk >> 2) * kBox64 + (kk & 3) * 32;
              tc_mma_ss(tmem + 128 * w + 64, smem_desc_sw128(a, 16, 1024),
                        smem_desc_sw128(bb, 16, 1024), idS, kk > 0 ? 1u : 0u);
            }
          }
          tc_commit(is_s ? &bars->s_full[w] : &bars->dp_full[w]);
          tc_commit(&bars->qd_empty[st]);
        }
      }
    }
  } else if (warp == kKvProducer + 3 || warp == kKvProducer + 4) {
    if (lane == 0) {  // ---------------------------------------- dV issuer and dK issuer
      // each accumulator has one issuing thread, so its order is fixed
      const bool is_v = warp == kKvProducer + 3;
      constexpr uint32_t idV = idesc_bf16_f32(128, 128, false, true);
      constexpr uint32_t idK = idesc_bf16_f32(128, D, false, true);
      bool first[2] = {true, true};
      for (int s = 0; s < n_steps; ++s) {
        const int st = s % kKvStages, w = s & 1, r = s & 1;
        const uint32_t sq = smem_u32(sStage) + st * kStageBytes, sdo = sq + kStageQ;
        const int fb = (is_v || kForm == 2) ? 0 : r;  // accumulator of this step
        // each column half's products go out as soon as that half's P^T / dS^T is written
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait(is_v ? &bars->p_full[w][h] : &bars->ds_full[w][h],
                         (uint32_t)(s >> 1) & 1u, p.dev_status, &failed))
            break;
          tc_fence_after();
          for (int kk = 2 * h; kk < 2 * h + 2; ++kk) {  // 16 queries each; B operands MN-major
            const uint32_t acc = (first[fb] && kk == 0) ? 0u : 1u;
            // queries [32h, 32h + 32) of a step are packed into columns [32h, 32h + 16)
            // of their buffer (each column half writes inside the columns it read)
            const uint32_t pc = 32u * (uint32_t)h + 8u * (uint32_t)(kk & 1);
            if (is_v)
              tc_mma_ts(tmem + kColDV, tmem + 128 * w + pc,
                        smem_desc_sw128(sdo + kk * 2048, kBox64, 1024), idV, acc);
            else
              tc_mma_ts(tmem + kColDK + (kForm == 1 ? 64 * r : 0), tmem + 128 * w + 64 + pc,
                        smem_desc_sw128(sq + kk * 2048, kBox64, 1024), idK, acc);
          }
        }
        if (failed) break;
        first[fb] = false;
        tc_commit(is_v ? &bars->pt_free[w] : &bars->dst_free[w]);
        tc_commit(&bars->qd_empty[st]);
      }
      tc_commit(&bars->acc_done);
    }
  } else {
    // ------------------ softmax backward, steps of parity w, query columns of half h
    // Two passes per step.  P = 2^(s sc - lse) goes out as soon as S^T has
    // landed, so the dV product starts (and frees the S^T buffer for step
    // s + 2) while dP^T may still be in flight; dS = P (dP - D) follows from
    // the same bf16 P, kept in registers.  Each step's 64 query columns are
    // split between two warpgroups, which halves every thread's serial chain
    // and gives each sub-partition four softmax warps to interleave.
    const int w = (warp >> 2) & 1;
    const int h = warp >> 3;
    const int krow = (warp & 3) * 32 + lane;
    const int key = k0 + krow;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t t_s = tmem + lane_off + 128 * w + 32 * h, t_dp = t_s + 64;
    const float sc = p.scale_log2;
    for (int s = w; s < n_steps; s += 2) {
      const int st = s % kKvStages;
      const uint32_t ph = (uint32_t)(s >> 1) & 1u;
      const bool ok = mbar_wait(&bars->qd_full[st], (uint32_t)(s / kKvStages) & 1u,
                                p.dev_status, &failed) &&
                      mbar_wait(&bars->s_full[w], ph, p.dev_status, &failed);
      if (!__all_sync(0xffffffffu, ok)) {
        failed = true;
        break;
      }
      tc_fence_after();
      const int q0 = step_q0(s);
      const float* svec =
          reinterpret_cast<const float*>(sStage + st * kStageBytes + kStageQ + kTile64) + 32 * h;
      // query columns this key row sees in the step: [c_lo, c_hi), relative
      // to this half's first column
      int c_lo = 0, c_hi = min(64, p.seqlen - q0);
      if (key >= p.seqlen) c_hi = 0;
      if (p.causal) c_lo = max(0, key - q0);
      if (kWindow) c_hi = min(c_hi, key + p.window - q0);
      c_lo -= 32 * h;
      c_hi -= 32 * h;
      const bool full = __all_sync(0xffffffffu, c_lo <= 0 && c_hi >= 32);
      const uint64_t sc2 = f2pack(sc, sc);
      uint32_t pp[16];  // P row (32 queries) as packed bf16 pairs
      {
        uint32_t sv[32];
        tmem_ld32(t_s, sv);
        tc_wait_ld();
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {  // 4 query columns: lse by a broadcast load
          const int c = 4 * e4;
          const float4 L = *reinterpret_cast<const float4*>(svec + c);
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int e = 2 * e4 + h2;
            const float l0 = h2 ? L.z : L.x, l1 = h2 ? L.w : L.y;
            float x0, x1;
            f2unpack(fma2(f2pack(__uint_as_float(sv[2 * e]), __uint_as_float(sv[2 * e + 1])),
                          sc2, f2pack(-l0, -l1)),
                     x0, x1);
            float p0 = ex2(x0), p1 = ex2(x1);
            if (!full) {
              const int cc = c + 2 * h2;
              p0 = (cc >= c_lo && cc < c_hi) ? p0 : 0.f;
              p1 = (cc + 1 >= c_lo && cc + 1 < c_hi) ? p1 : 0.f;
            }
            pp[e] = pack_bf16(p0, p1);
          }
        }
        // P^T over the first 16 of the 32 columns this half has read
        tmem_st16(t_s, pp);
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->p_full[w][h]);

      if (!__all_sync(0xffffffffu, mbar_wait(&bars->dp_full[w], ph, p.dev_status, &failed))) {
        failed = true;
        break;
      }
      tc_fence_after();
      {
        uint32_t dp[32], pd[16];
        tmem_ld32(t_dp, dp);
        tc_wait_ld();
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {  // D by a broadcast load
          const int c = 4 * e4;
          const float4 Dd = *reinterpret_cast<const float4*>(svec + 64 + c);
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int e = 2 * e4 + h2;
            const float d0 = h2 ? Dd.z : Dd.x, d1 = h2 ? Dd.w : Dd.y;
            const uint32_t pb = pp[e];
            const uint64_t pr = f2pack(bf16lo(pb), bf16hi(pb));
            const uint64_t dd = add2(
                f2pack(__uint_as_float(dp[2 * e]), __uint_as_float(dp[2 * e + 1])),
                f2pack(-d0, -d1));
            float ds0, ds1;
            f2unpack(fma2(pr, dd, 0ull), ds0, ds1);
            pd[e] = pack_bf16(ds0, ds1);
          }
        }
        tmem_st16(t_dp, pd);
      }
      tc_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->ds_full[w][h]);
    }
    __syncwarp();
    if (failed) bars->abort_flag = 1;
    mbar_wait(&bars->acc_done, 0, p.dev_status, &failed);
    tc_fence_after();
    asm volatile("bar.sync 2, 512;" ::: "memory");
    const bool store = key < p.seqlen && !bars->abort_flag;
    // warpgroups of w = 0 write dV, of w = 1 dK (scaled by 1/sqrt(d)), columns [64h, 64h + 64)
    float* dst = (w == 0 ? p.dv : p.dk) + (((size_t)b * p.seqlen + key) * p.kv_heads + g) * 128 +
                 64 * h;
    const uint32_t col = (w == 0 ? kColDV : kColDK) + 64u * (uint32_t)h;
    const float mul = w == 0 ? 1.f : p.scale;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_off + col + 32 * c, v);
      tc_wait_ld();
      if (store) {
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          float4 f;
          f.x = __uint_as_float(v[e]) * mul;
          f.y = __uint_as_float(v[e + 1]) * mul;
          f.z = __uint_as_float(v[e + 2]) * mul;
          f.w = __uint_as_float(v[e + 3]) * mul;
          *reinterpret_cast<float4*>(dst + 32 * c + e) = f;
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kKvProducer + 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Per row: the pre-norm output o = O_1 - lambda O_2 from the saved
// normalised branch outputs, the norm backward (V1), do_1 = do and
// do_2 = -lambda do (bf16, [B][N][units][2][128]), D_r = do_r . O_r and the
// block's shares of dlambda and of the norm gain's gradient.
constexpr int kPreWarps = 8;
constexpr int kPreRows = 64;

struct Pre2Args {
  const float* obr;          // [B][N][units][2][128]
  const __nv_bfloat16* dout; // [B][N][units][128]
  __nv_bfloat16* dob;        // [B][N][units][2][128]
  float* Dv;                 // [B][units][2][npad]
  int B, N, units, npad;
  const float* lambda;
  int apply_norm;
  const float* g;
  float eps, post;
  float* dlambda;
  float* dg;
};

__global__ void __launch_bounds__(32 * kPreWarps) bwd_pre2_kernel(Pre2Args a) {
  __shared__ float sh_dg[kPreWarps][128];
  __shared__ float sh_dl[kPreWarps];
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int u = blockIdx.y % a.units, b = blockIdx.y / a.units;
  const float lam = a.lambda[u];
  // lane l owns channels 4l .. 4l + 3: every row moves as 8-byte vectors
  const int c0 = 4 * lane;
  float gc[4] = {1.f, 1.f, 1.f, 1.f};
  if (a.apply_norm && a.g) {  // the gain has no alignment guarantee: scalar loads
#pragma unroll
    for (int t = 0; t < 4; ++t) gc[t] = a.g[c0 + t];
  }
  float dg[4] = {0.f, 0.f, 0.f, 0.f};
  float dl = 0.f;
  const int r0 = blockIdx.x * kPreRows;
  for (int i = r0 + warp; i < min(r0 + kPreRows, a.N); i += kPreWarps) {
    const size_t tok = ((size_t)b * a.N + i) * a.units + u;
    const float4 w1 = *reinterpret_cast<const float4*>(a.obr + tok * 256 + c0);
    const float4 w2 = *reinterpret_cast<const float4*>(a.obr + tok * 256 + 128 + c0);
    const uint2 wy = *reinterpret_cast<const uint2*>(a.dout + tok * 128 + c0);
    const float o1[4] = {w1.x, w1.y, w1.z, w1.w};
    const float o2[4] = {w2.x, w2.y, w2.z, w2.w};
    const float dy[4] = {bf16lo(wy.x), bf16hi(wy.x), bf16lo(wy.y), bf16hi(wy.y)};
    float o[4], d_o[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) o[t] = o1[t] - lam * o2[t];
    if (a.apply_norm) {
      float ss = 0.f, gdo = 0.f;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        ss = fmaf(o[t], o[t], ss);
        gdo = fmaf(gc[t] * dy[t], o[t], gdo);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        ss += __shfl_xor_sync(0xffffffffu, ss, off);
        gdo += __shfl_xor_sync(0xffffffffu, gdo, off);
      }
      const float rr = sqrtf(ss / 128.f + a.eps);
      const float cr = a.post / rr, k2 = gdo / (128.f * rr * rr);
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        d_o[t] = cr * (gc[t] * dy[t] - o[t] * k2);
        dg[t] = fmaf(dy[t] * o[t], cr, dg[t]);
      }
    } else {
#pragma unroll
      for (int t = 0; t < 4; ++t) d_o[t] = dy[t];
    }
    // bf16 upstream gradients of each branch; D_r from the same rounded values
    uint2 b1, b2;
    b1.x = pack_bf16(d_o[0], d_o[1]);
    b1.y = pack_bf16(d_o[2], d_o[3]);
    b2.x = pack_bf16(-lam * d_o[0], -lam * d_o[1]);
    b2.y = pack_bf16(-lam * d_o[2], -lam * d_o[3]);
    *reinterpret_cast<uint2*>(a.dob + tok * 256 + c0) = b1;
    *reinterpret_cast<uint2*>(a.dob + tok * 256 + 128 + c0) = b2;
    const float r1[4] = {bf16lo(b1.x), bf16hi(b1.x), bf16lo(b1.y), bf16hi(b1.y)};
    const float r2[4] = {bf16lo(b2.x), bf16hi(b2.x), bf16lo(b2.y), bf16hi(b2.y)};
    float s1 = 0.f, s2 = 0.f, sl = 0.f;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      s1 = fmaf(r1[t], o1[t], s1);
      s2 = fmaf(r2[t], o2[t], s2);
      sl = fmaf(d_o[t], o2[t], sl);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      s1 += __shfl_xor_sync(0xffffffffu, s1, off);
      s2 += __shfl_xor_sync(0xffffffffu, s2, off);
      sl += __shfl_xor_sync(0xffffffffu, sl, off);
    }
    if (lane == 0) {
      const size_t vr = ((size_t)b * a.units + u) * 2 * a.npad + i;
      a.Dv[vr] = s1;
      a.Dv[vr + a.npad] = s2;
    }
    dl -= sl;
  }
#pragma unroll
  for (int t = 0; t < 4; ++t) sh_dg[warp][c0 + t] = dg[t];
  if (lane == 0) sh_dl[warp] = dl;
  __syncthreads();
  if (threadIdx.x < 128 && a.dg) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kPreWarps; ++w) s += sh_dg[w][threadIdx.x];
    atomicAdd(a.dg + threadIdx.x, s);
  }
  if (threadIdx.x == 0) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kPreWarps; ++w) s += sh_dl[w];
    atomicAdd(a.dlambda + u, s);
  }
}

}  // namespace

// Saves of the training forward: per-row log2-sum-exp of each branch
// (fp32 [B][units][2][npad], padding zero) and each branch's normalised output
// O_r / l_r (fp32 [B][N][units][2][128]: dlambda and the gain gradient are
// sums of N x 128 products of them with heavy cancellation, which bf16 saves
// would leave a few percent off).  The backward's workspace holds D_r (as lse)
// and the per-branch upstream gradients (bf16, the MMA operands).
struct SavesLayout {
  size_t lse_bytes, obr_bytes, dob_bytes;
};

SavesLayout saves_layout(int batch, int seqlen, int units) {
  const size_t npad = (size_t)((seqlen + 63) / 64) * 64;
  SavesLayout L;
  L.lse_bytes = ((size_t)batch * units * 2 * npad * 4 + 255) & ~size_t(255);
  L.obr_bytes = ((size_t)batch * seqlen * units * 256 * 4 + 255) & ~size_t(255);
  L.dob_bytes = ((size_t)batch * seqlen * units * 256 * 2 + 255) & ~size_t(255);
  return L;
}

size_t train_saves_bytes(int batch, int seqlen, int units) {
  const SavesLayout L = saves_layout(batch, seqlen, units);
  return L.lse_bytes + L.obr_bytes + 256;
}

size_t saved_bwd_workspace_bytes(int batch, int seqlen, int units) {
  const SavesLayout L = saves_layout(batch, seqlen, units);
  return L.lse_bytes + L.dob_bytes + 256;
}

size_t fused_bwd_workspace_bytes(int batch, int seqlen, int units) {
  const size_t out = (size_t)batch * seqlen * units * 128 * 2;
  // + 256: the workspace's own start is rounded up to 256 bytes
  return train_saves_bytes(batch, seqlen, units) + saved_bwd_workspace_bytes(batch, seqlen, units) +
         ((out + 255) & ~size_t(255)) + 256;
}

namespace {
uint8_t* align256(void* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 255) & ~uintptr_t(255));
}
}  // namespace

cudaError_t launch_fwd_train(const PrefillArgs& fwd, const void* q, const void* k,
                             const void* v, void* out, void* saves, int num_sms,
                             cudaStream_t st) {
  const int B = fwd.batch, N = fwd.seqlen, U = fwd.heads;
  const int npad = (N + 63) / 64 * 64;
  const SavesLayout L = saves_layout(B, N, U);
  uint8_t* base = align256(saves);
  float* lse = reinterpret_cast<float*>(base);
  void* obr = base + L.lse_bytes;
  const int qh = fwd.form == 1 ? U : 2 * U, kvh = fwd.kv_heads;
  CUtensorMap tq128, tk64, tv64;
  if (make_tmap_bf16_4d(&tq128, q, 128, qh, N, B, 64, 1, 128, 1) ||
      make_tmap_bf16_4d(&tk64, k, 128, kvh, N, B, 64, 1, 64, 1) ||
      make_tmap_bf16_4d(&tv64, v, 128, kvh, N, B, 64, 1, 64, 1))
    return cudaErrorInvalidValue;
  // lse rows are read in 64-entry blocks, so the padding is zeroed first
  cudaError_t e = cudaMemsetAsync(lse, 0, (size_t)B * U * 2 * npad * 4, st);
  if (e != cudaSuccess) return e;
  PrefillArgs fa = fwd;
  fa.out = out;
  fa.lse = lse;
  fa.lse_stride = npad;
  fa.obr = obr;
  return launch_prefill_tc(tq128, tk64, tv64, fa, num_sms, st);
}

cudaError_t launch_bwd_from_saves(const FusedBwdArgs& a, const void* saves, cudaStream_t st) {
  const int B = a.fwd.batch, N = a.fwd.seqlen, U = a.fwd.heads;
  const int npad = (N + 63) / 64 * 64;
  const SavesLayout L = saves_layout(B, N, U);
  const uint8_t* sv = align256(const_cast<void*>(saves));
  const float* lse = reinterpret_cast<const float*>(sv);
  const float* obr = reinterpret_cast<const float*>(sv + L.lse_bytes);
  uint8_t* wb = align256(a.workspace);
  float* Dv = reinterpret_cast<float*>(wb);
  __nv_bfloat16* dob = reinterpret_cast<__nv_bfloat16*>(wb + L.lse_bytes);

  // tensor maps: inputs as [B][N][heads][128] with 64-column boxes of 128
  // or 64 rows, and the per-branch upstream gradients [B][N][2U][128]
  const int qh = a.fwd.form == 1 ? U : 2 * U, kvh = a.fwd.kv_heads;
  CUtensorMap tq128, tq64, tk64, tk128, tv64, tv128, tdo128, tdo64;
  if (make_tmap_bf16_4d(&tq128, a.q, 128, qh, N, B, 64, 1, 128, 1) ||
      make_tmap_bf16_4d(&tq64, a.q, 128, qh, N, B, 64, 1, 64, 1) ||
      make_tmap_bf16_4d(&tk64, a.k, 128, kvh, N, B, 64, 1, 64, 1) ||
      make_tmap_bf16_4d(&tk128, a.k, 128, kvh, N, B, 64, 1, 128, 1) ||
      make_tmap_bf16_4d(&tv64, a.v, 128, kvh, N, B, 64, 1, 64, 1) ||
      make_tmap_bf16_4d(&tv128, a.v, 128, kvh, N, B, 64, 1, 128, 1) ||
      make_tmap_bf16_4d(&tdo128, dob, 128, 2 * U, N, B, 64, 1, 128, 1) ||
      make_tmap_bf16_4d(&tdo64, dob, 128, 2 * U, N, B, 64, 1, 64, 1))
    return cudaErrorInvalidValue;
  // upstream gradients per branch, D, dlambda, gain gradient
  cudaError_t e;
  if ((e = cudaMemsetAsync(Dv, 0, (size_t)B * U * 2 * npad * 4, st)) != cudaSuccess ||
      (e = cudaMemsetAsync(a.dlambda, 0, (size_t)U * 4, st)) != cudaSuccess ||
      (a.dg && (e = cudaMemsetAsync(a.dg, 0, 128 * 4, st)) != cudaSuccess))
    return e;
  Pre2Args pa;
  pa.obr = obr;
  pa.dout = static_cast<const __nv_bfloat16*>(a.dout);
  pa.dob = dob;
  pa.Dv = Dv;
  pa.B = B;
  pa.N = N;
  pa.units = U;
  pa.npad = npad;
  pa.lambda = a.fwd.lambda;
  pa.apply_norm = a.fwd.apply_norm;
  pa.g = a.fwd.norm_weight;
  pa.eps = a.fwd.eps;
  pa.post = a.fwd.post_scale;
  pa.dlambda = a.dlambda;
  pa.dg = a.fwd.apply_norm ? a.dg : nullptr;
  bwd_pre2_kernel<<<dim3((N + kPreRows - 1) / kPreRows, B * U), 32 * kPreWarps, 0, st>>>(pa);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  BwdParams p;
  p.batch = B;
  p.seqlen = N;
  p.units = U;
  p.pairs_per_kv = a.fwd.pairs_per_kv;
  p.causal = a.fwd.causal;
  p.window = a.fwd.window;
  p.npad = npad;
  const double d = a.fwd.form == 1 ? 64.0 : 128.0;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt(d));
  p.scale = (float)(1.0 / std::sqrt(d));
  p.lse = lse;
  p.Dv = Dv;
  p.lambda = a.fwd.lambda;
  p.dq = a.dq;
  p.dk = a.dk;
  p.dv = a.dv;
  p.q_heads = qh;
  p.kv_heads = a.fwd.kv_heads;
  p.n_qtiles = (N + 127) / 128;
  p.n_ktiles = (N + 127) / 128;
  // Tile order: groups of 8 units, heaviest tiles first within a group.  In a
  // sweep of the group size on the V1 (B4 H16 N4096) and V2 (B2 Hq32 N8192)
  // backward, 4 to 16 units all ran 4-6 % faster than one unit (unit-major
  // order) and 32 or more slower again.
  p.group_q = std::min(8, B * U);
  p.group_kv = std::min(8, B * a.fwd.kv_heads);
  p.dev_status = a.fwd.dev_status;
  const bool win = a.fwd.window > 0;
  // dQ
  {
    const int qbytes = a.fwd.form == 1 ? kTile128 : 2 * kTile128;
    const int smem = 1024 + qbytes + kTile128 + 2 * kDqStages * kTile64 +
                     (a.fwd.form == 2 ? 2 * kBox128 : 0) + (int)sizeof(DqBarriers) + 64;
    decltype(&diffattn_bwd_dq_kernel<1, false>) k =
        a.fwd.form == 1 ? (win ? diffattn_bwd_dq_kernel<1, true> : diffattn_bwd_dq_kernel<1, false>)
                        : (win ? diffattn_bwd_dq_kernel<2, true> : diffattn_bwd_dq_kernel<2, false>);
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
      return e;
    k<<<p.n_qtiles * B * U, kDqThreads, smem, st>>>(tq128, tdo128, tk64, tv64, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // dK, dV
  {
    const int smem = 1024 + 2 * kTile128 + kKvStages * kStageBytes + (int)sizeof(KvBarriers) + 64;
    decltype(&diffattn_bwd_dkdv_kernel<1, false>) k =
        a.fwd.form == 1
            ? (win ? diffattn_bwd_dkdv_kernel<1, true> : diffattn_bwd_dkdv_kernel<1, false>)
            : (win ? diffattn_bwd_dkdv_kernel<2, true> : diffattn_bwd_dkdv_kernel<2, false>);
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
      return e;
    k<<<p.n_ktiles * B * a.fwd.kv_heads, kKvThreads, smem, st>>>(tq64, tdo64, tk128, tv128, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_fused_bwd(const FusedBwdArgs& a, cudaStream_t st) {
  // workspace: [saves of the training forward][backward workspace][forward output]
  const int B = a.fwd.batch, N = a.fwd.seqlen, U = a.fwd.heads;
  uint8_t* base = align256(a.workspace);
  const size_t saves = train_saves_bytes(B, N, U), bwd = saved_bwd_workspace_bytes(B, N, U);
  void* fwd_out = base + saves + bwd;
  cudaError_t e = launch_fwd_train(a.fwd, a.q, a.k, a.v, fwd_out, base, a.num_sms, st);
  if (e != cudaSuccess) return e;
  FusedBwdArgs b = a;
  b.workspace = base + saves;
  return launch_bwd_from_saves(b, base, st);
}

}  // namespace da
