// gemm_tc.cu — bf16 matrix product on the 5th-generation tensor cores
// (tcgen05 + tensor memory + TMA) for the V2 output projection:
//     C[M][N] = A[M][K] . B[K][N]      (row-major bf16, fp32 accumulation)
// with A the differential-attention output flattened to [tokens, Hq/2 * d]
// and B the projection O_W [Hq/2 * d, d_model] (lesson "Atención
// Diferencial (V2)", section "V1 vs V2: la diferencia" and step 5 of
// "Implementación": the paired heads are brought back down and projected).
//
// Tiles of 128 rows x 256 columns, K in steps of 64 (one 128-byte swizzle
// row of bf16).  A is K-major (one 128-row x 64 box per step), B is read in
// its row-major layout as an MN-major operand (four 64-column x 64-row boxes
// per step).  One CTA per SM walks the tiles persistently (tile t, t + grid,
// ...; column tiles of a row block are adjacent, so CTAs working at the same
// time share A rows in L2, and B stays in L2 whole).
//
// Warp roles (192 threads):
//   warp 0     TMA producer: A and B boxes through a 4-stage ring (48 KB per stage)
//   warp 1     allocates tensor memory; one thread issues the MMAs
//              (M128 N256 K16, four per K step) into one of two accumulators
//   warps 2-5  epilogue: each thread reads one accumulator row (its warp's
//              tensor-memory lane quarter) and stores it as bf16
// The two accumulators (2 x 256 columns = all 512) let the epilogue of one
// tile run while the MMAs of the next tile fill the other.  Every wait is
// bounded; a timed-out wait records DA_ERR_DEVICE_TIMEOUT and the CTA
// unwinds, still freeing its tensor memory.  No TMA multicast is used.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace da {
namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kABytes = kBM * kBK * 2;   // 16 KB
constexpr int kBBox = 64 * kBK * 2;      // 8 KB: 64 columns x 64 K rows
constexpr int kBBytes = 4 * kBBox;       // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kThreads = 192;
constexpr uint32_t kIdesc = idesc_bf16_f32(kBM, kBN, false, true);

struct GemmBars {
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint32_t tmem_base;
};

struct GemmParams {
  int M, N, K;
  int tiles_n, n_tiles, k_blocks;
  __nv_bfloat16* C;
  int* dev_status;
};

__global__ void __launch_bounds__(kThreads, 1)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tm_a,
                        const __grid_constant__ CUtensorMap tm_b, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                       // kStages x 16 KB
  uint8_t* sB = smem + kStages * kABytes;   // kStages x 32 KB
  GemmBars* bars = reinterpret_cast<GemmBars*>(sB + kStages * kBBytes);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->acc_full[b], 1);
      mbar_init(&bars->acc_empty[b], 128);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  bool failed = false;

  if (warp == 0) {
    // ------------------------------ TMA producer ---------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      uint32_t it = 0;
      for (int tile = blockIdx.x; tile < p.n_tiles && !failed; tile += gridDim.x) {
        const int m0 = (tile / p.tiles_n) * kBM;
        const int n0 = (tile % p.tiles_n) * kBN;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int s = it % kStages;
          const uint32_t ph = (it / kStages) & 1u;
          if (!mbar_wait(&bars->empty[s], ph ^ 1u, p.dev_status, &failed)) break;
          mbar_arrive_expect_tx(&bars->full[s], kStageBytes);
          tma_load_4d(sA + s * kABytes, &tm_a, &bars->full[s], kb * kBK, m0, 0, 0);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tma_load_4d(sB + s * kBBytes + c * kBBox, &tm_b, &bars->full[s], n0 + 64 * c,
                        kb * kBK, 0, 0);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    if (lane == 0) {
      const uint32_t a0 = smem_u32(sA);
      const uint32_t b0 = smem_u32(sB);
      uint32_t it = 0;
      int lt = 0;
      for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++lt) {
        const int buf = lt & 1;
        // the epilogue must have read this accumulator's previous tile out
        if (!mbar_wait(&bars->acc_empty[buf], ((uint32_t)(lt >> 1) & 1u) ^ 1u, p.dev_status,
                       &failed))
          break;
        tc_fence_after();
        const uint32_t acc = tmem + 256u * (uint32_t)buf;
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&bars->full[s], (it / kStages) & 1u, p.dev_status, &failed)) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            // A: K-major rows of 128 bytes, 8-row groups 1 KB apart
            // B: MN-major, 64-column boxes kBBox apart, 8-row (K) groups 1 KB apart
            tc_mma_ss(acc, smem_desc_sw128(a0 + s * kABytes + kk * 32, 16, 1024),
                      smem_desc_sw128(b0 + s * kBBytes + kk * 2048, kBBox, 1024), kIdesc,
                      (kb > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(&bars->empty[s]);
        }
        if (failed) break;
        tc_commit(&bars->acc_full[buf]);
      }
    }
  } else {
    // ------------------------------ epilogue --------------------------------
    const int quarter = warp & 3;                  // tensor-memory lane quarter of this warp
    const int row = quarter * 32 + lane;           // accumulator row = tile row
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    int lt = 0;
    for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++lt) {
      const int buf = lt & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->acc_full[buf], (uint32_t)(lt >> 1) & 1u,
                                              p.dev_status, &failed))) {
        failed = true;
        break;
      }
      tc_fence_after();
      const int m = (tile / p.tiles_n) * kBM + row;
      const int n0 = (tile % p.tiles_n) * kBN;
      __nv_bfloat16* dst = p.C + (size_t)m * p.N;
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + 256u * (uint32_t)buf + 32u * (uint32_t)c, r);
        tc_wait_ld();
        if (c == kBN / 32 - 1) {  // accumulator read out: the next tile may overwrite it
          tc_fence_before();
          mbar_arrive(&bars->acc_empty[buf]);
        }
        const int n = n0 + 32 * c;
        if (m < p.M && n < p.N) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {  // N is a multiple of 8: whole 16-byte groups
            if (n + 8 * v < p.N) {
              uint4 w;
              w.x = pack_bf16(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
              w.y = pack_bf16(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
              w.z = pack_bf16(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
              w.w = pack_bf16(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
              *reinterpret_cast<uint4*>(dst + n + 8 * v) = w;
            }
          }
        }
      }
    }
  }

  // ---- teardown: every role reaches this point, then TMEM is released ----
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

int gemm_bf16_tc_smem_bytes() {
  return 1024 + kStages * kStageBytes + (int)sizeof(GemmBars) + 64;
}

cudaError_t launch_gemm_bf16_tc(const void* a, const void* b, void* c, int M, int N, int K,
                                int num_sms, int* dev_status, cudaStream_t stream) {
  CUtensorMap ta, tb;
  // A [M][K]: boxes of 64 K-columns x 128 rows; B [K][N]: boxes of 64 columns x 64 K-rows
  if (make_tmap_bf16_4d(&ta, a, (uint64_t)K, (uint64_t)M, 1, 1, 64, kBM, 1, 1) != 0 ||
      make_tmap_bf16_4d(&tb, b, (uint64_t)N, (uint64_t)K, 1, 1, 64, kBK, 1, 1) != 0)
    return cudaErrorInvalidValue;
  GemmParams p;
  p.M = M;
  p.N = N;
  p.K = K;
  p.tiles_n = (N + kBN - 1) / kBN;
  const long long tiles = (long long)((M + kBM - 1) / kBM) * p.tiles_n;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  p.n_tiles = (int)tiles;
  p.k_blocks = (K + kBK - 1) / kBK;
  p.C = static_cast<__nv_bfloat16*>(c);
  p.dev_status = dev_status;
  const int smem = gemm_bf16_tc_smem_bytes();
  cudaError_t e =
      cudaFuncSetAttribute(gemm_bf16_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = p.n_tiles < num_sms ? p.n_tiles : num_sms;
  gemm_bf16_tc_kernel<<<grid, kThreads, smem, stream>>>(ta, tb, p);
  return cudaGetLastError();
}

}  // namespace da
