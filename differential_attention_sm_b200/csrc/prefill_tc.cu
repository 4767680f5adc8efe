// prefill_tc.cu — differential-attention prefill on the 5th-generation
// tensor cores (tcgen05 + tensor memory + TMA), both forms.
//
// Operator: glossary page "Differential Transformer", section "Cómo funciona
// la atención diferencial" (two softmax maps from the two halves of each
// head's query/key, combined as (map1 - lambda map2) V, then a per-head
// normalisation and a (1 - lambda_init) scale); lesson "Atención
// Diferencial (V2)", section "V1 vs V2: la diferencia" (V2: paired query
// heads on shared GQA KV heads, full head width, no per-head norm).
//
// A query tile is 128 query rows of one head (V1) or one head pair (V2).
// Both branches see the same K and V tiles, so each 64-key tile is loaded
// once by TMA for the pair.  Tensor memory (512 columns x 128 lanes fp32):
//     S1 [0,64) [64,128)   S2 [128,192) [192,256)   O1 [256,384)   O2 [384,512)
// Each branch's score tile is double-buffered: while the softmax warps of
// branch r turn S_r(j) into P_r(j) (bf16, written in place over the first
// 32 columns of that buffer and fed to the P.V MMA straight from tensor
// memory), the tensor core already computes S_r(j+1) into the other buffer.
// The two branches need separate O accumulators because their running
// maxima and normalisers differ; the subtraction happens in the epilogue:
//     o = O1 / l1 - lambda * O2 / l2   (then, V1 only, RMS norm * g * (1 - lambda_init)).
//
// Warp roles (V2: 13 warps; V1: 12, with one score issuer for both branches):
//   warps 0-3  softmax for branch 1 (thread = one query row = one TMEM lane)
//   warps 4-7  softmax for branch 2
//   warp  8    TMA producer (Q per tile; K and V tiles through 4-stage rings;
//              requests the next tile)
//   warp  9    issues branch 1's score MMAs (Q1.K^T); owns the tensor memory
//   warp 10    issues branch 2's score MMAs (Q2.K^T)           (V2 only)
//   then       one warp per branch issuing its P_r.V MMAs
// V1 gives both branches' score MMAs (64-wide, 4 k-steps each) to warp 9:
// with 12 warps no sub-partition holds more than three, so the softmax
// threads get 168 registers instead of the 128 that four warps leave, and
// the V1 softmax runs without the spills and re-loads the cap forced.  V2's
// score products are twice as long and keep an issuer per branch.
// tcgen05.mma issue runs at the tensor pipe's pace and every commit and
// barrier poll costs the issuing thread time, so the P.V streams have a
// thread each: P_r(j).V goes out as soon as P_r(j) is ready, and S_r(j+2)
// as soon as that P.V has freed its buffer, without waiting behind the
// other stream's bookkeeping.
// The V1 epilogue writes each softmax warp's 32 output rows (and in the
// training forward its saved fp32 branch outputs, 8 columns at a time)
// through a 4 KB shared-memory block and TMA tensor stores; so does the V2
// training forward (with three K/V ring slots to make room), while V2
// inference stores from registers.
// Softmax keeps a per-row reference maximum and only rescales O (in tensor
// memory) when a new row maximum exceeds it by more than 2^8, so P <= 256.
// Causal masking is applied only on the tiles that cross the diagonal (and
// the ragged tail).
//
// Scheduling.  The grid has one CTA per query tile; tiles are numbered by
// groups of heads whose K/V fit in L2, heaviest query tiles first within a
// group.  Only one CTA fits on an SM, and a resident CTA does not exit
// after its tile: near the end of each tile the producer asks the hardware
// scheduler (cluster launch control) to cancel a CTA that has not started
// and takes over its share of the work.  Which tile a unit of work (a CTA
// that starts, or one it cancels) computes comes from a ticket counter, so
// the SMs pull tiles strictly in the order above, whatever order the
// hardware starts or cancels CTAs in.  The rings, the score buffers and
// their barrier phases run on counters that continue across tiles: the
// next tile's Q load and first Q.K^T proceed during the current tile's
// last P.V and epilogue, with no barrier set-up or tensor-memory
// allocation between tiles.  The first P.V of a tile overwrites O, so it
// waits for the previous epilogue to have read O out of tensor memory.
// Every wait is bounded (the softmax warps exchange their normalisers
// through mbarriers, not named barriers); a timed-out wait records
// DA_ERR_DEVICE_TIMEOUT in the caller's status word and the CTA unwinds,
// still freeing its tensor memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace da {
namespace {

constexpr int kBM = 128;                   // query rows per CTA
constexpr int kBN = 64;                    // keys per KV tile
// Output (and, for the training forward, the saved branch outputs) staged
// through shared memory and written by TMA stores: V1, and the V2 training
// forward, which makes room for the 32 KB with a three-slot K/V ring (V2
// inference keeps four slots and stores from registers)
__host__ __device__ constexpr bool stage_out(int form, bool save) { return form == 1 || save; }
// score-MMA issuer warps and threads per CTA, by form
__host__ __device__ constexpr int score_issuers(int form) { return form == 1 ? 1 : 2; }
__host__ __device__ constexpr int cta_threads(int form) { return (11 + score_issuers(form)) * 32; }
constexpr int kQBox = kBM * 64 * 2;        // TMA box of Q: 128 rows x 64 bf16 = 16 KB
constexpr int kQTile = 2 * kQBox;          // one 128 x 128 query tile
constexpr int kKVBox = kBN * 64 * 2;       // TMA box of K/V: 64 rows x 64 bf16 = 8 KB
constexpr int kKVTile = 2 * kKVBox;        // one 64 x 128 key or value tile
constexpr int kStages = 4;  // K/V ring slots (barriers are sized for this many)
__host__ __device__ constexpr int kv_stages(int form, bool save) { return form == 2 && save ? 3 : 4; }
constexpr uint32_t kColS1 = 0, kColS2 = 128, kColO1 = 256, kColO2 = 384;
constexpr float kLazyTau = 8.0f;           // log2 units: rescale only when max grows by > 2^8

constexpr uint32_t kIdescQK = idesc_bf16_f32(128, kBN, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(128, 128, false, true);

struct Barriers {
  uint64_t q_full, q_empty;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t s_full[2][2];                  // [branch][buffer]
  uint64_t p_full[2][2][2];               // [branch][buffer][key half]
  uint64_t o_done[2][2];                  // [branch][buffer]: P_r(j).V complete
  uint64_t o_free;                        // the epilogue has read O out of tensor memory
  uint64_t t_full[2], t_empty[2];         // tile numbers handed to the roles [buffer]
  uint64_t xchg[2], nchg[2];              // softmax threads' exchanges [tile parity]
  uint64_t clc_full;                      // response of a cancellation request
  alignas(16) uint32_t clc_resp[4];
  int t_id[2];
  uint32_t tmem_base;
  int abort_flag;
};

// Arrivals that release a tile-number buffer: the score issuer(s), the two
// P.V issuers and the eight softmax warps.
__host__ __device__ constexpr uint32_t tile_readers(int form) {
  return 10u + (uint32_t)score_issuers(form);
}

struct Params {
  int form;
  int batch, seqlen, heads, pairs_per_kv;
  int n_qtiles;
  int n_tiles;      // query tiles in the grid (= CTAs launched)
  int ticket_slot;  // tile counter of this launch (see take_ticket)
  int group;        // heads (V1) / pairs (V2) scheduled together for L2 reuse
  int causal;
  int window;       // > 0: row i sees keys (i - window, i]
  float scale_log2;
  const float* lambda;
  int apply_norm;
  const float* norm_weight;
  float eps, post_scale;
  __nv_bfloat16* out;
  // training saves (nullptr when not wanted): per-row log2-sum-exp of each
  // branch [B][units][2][lse_stride], and each branch's normalised output
  // O_r / l_r as fp32 [B][N][units][2][128]
  float* lse;
  int lse_stride;  // row stride of lse (>= seqlen)
  float* obr;
  int* dev_status;
};

__device__ __forceinline__ uint32_t s_col(int r, int buf) {
  return (r == 0 ? kColS1 : kColS2) + 64u * (uint32_t)buf;
}

// One query tile: 128 rows of one head (V1) or head pair (V2).
struct Tile {
  int b, hh, kvh, q0, kv0, n_kv;
};

// Tile number -> coordinates.  Tiles are numbered by groups of heads whose
// K/V fit in L2, heaviest query tiles first within a group, and handed out
// in that order.
__device__ __forceinline__ Tile tile_at(const Params& p, int id, int form, bool window) {
  const int bh_count = p.batch * p.heads;
  const int per_group = p.group * p.n_qtiles;
  const int g = id / per_group;
  const int rr = id % per_group;
  const int g_size = min(p.group, bh_count - g * p.group);
  const int mt = p.n_qtiles - 1 - rr / g_size;
  const int bh = g * p.group + rr % g_size;
  Tile t;
  t.hh = bh % p.heads;
  t.b = bh / p.heads;
  t.kvh = form == 1 ? t.hh : t.hh / p.pairs_per_kv;
  t.q0 = mt * kBM;
  const int key_end = p.causal ? min(t.q0 + kBM, p.seqlen) : p.seqlen;  // keys this tile needs
  // Sliding window: row i sees keys (i - window, i], so the tile's first row
  // sets the first key tile it needs.  n_kv counts the tiles processed.
  t.kv0 = window ? max(0, t.q0 - p.window + 1) / kBN : 0;
  t.n_kv = (key_end + kBN - 1) / kBN - t.kv0;
  return t;
}

// Tile counters.  The host hands each launch one of these slots in turn, so
// launches that run at the same time on different streams normally count on
// different slots.  A slot is one 64-bit word: the tag of the launch that
// holds it in the high half and the tickets taken so far in the low half.
//   * A launch claims a slot whose count is zero (free) with one
//     compare-and-swap that writes its tag and count 1 (ticket 0); every later
//     unit of work of the same launch takes the next ticket with a plain
//     atomic add, so the CTAs that start together do not contend on a CAS.
//   * A launch takes exactly one ticket per tile; the unit that takes the last
//     one clears the count, so a finished launch leaves the slot free.
//   * The first unit of a CTA that finds the slot held by another launch
//     (two executions of one captured launch that overlap, or more launches
//     in flight than slots) waits for that launch to hand out its last tile,
//     then claims the slot.  The holder has a resident CTA that never waits
//     on this one, so the wait ends; it is still bounded: after
//     kScheduleWaitNs it gives up and DA_ERR_SCHEDULE is reported, so an
//     incomplete output never comes with status 0.  A holder whose word has
//     not changed for kStaleNs has stopped taking tickets (a launch that
//     ended with DA_ERR_DEVICE_TIMEOUT); its slot is taken over.
//   * Every later unit of a CTA finds its own launch's tag (the launch holds
//     the slot until its last ticket); anything else is reported at once.
// The tag is the grid's %gridid, which differs between launches that are in
// flight at the same time (graph replays included).
constexpr int kTicketSlots = 64;
constexpr uint64_t kScheduleWaitNs = 2000000000ull;  // below the 4 s pipeline waits
constexpr uint64_t kStaleNs = 250000000ull;
__device__ unsigned long long g_tickets[kTicketSlots];
__device__ unsigned g_gave_up[kTicketSlots];  // tag of the last launch that gave up waiting

__device__ __forceinline__ uint32_t launch_tag() {
  uint64_t g;
  asm volatile("mov.u64 %0, %%gridid;" : "=l"(g));
  const uint32_t t = (uint32_t)(g ^ (g >> 32));
  return t ? t : 1u;  // 0 marks a slot that no launch has used
}

// One ticket per unit of work (a CTA that starts, or a CTA it cancels):
// returns the tile number, or -1 (the caller reports DA_ERR_SCHEDULE).
// `first`: the CTA's own unit, the only one that may wait for or claim a slot.
__device__ __noinline__ int take_ticket(int slot, int n_tiles, uint32_t tag, bool first) {
  unsigned long long* ctr = g_tickets + slot;
  volatile unsigned long long* vctr = ctr;
  const unsigned long long claim =
      ((unsigned long long)tag << 32) | (n_tiles == 1 ? 0ull : 1ull);
  unsigned long long cur = *vctr, seen = 0ull;
  uint64_t t0 = 0, t_seen = 0;
  unsigned sleep_ns = 64;
  for (uint32_t iter = 0; iter < (1u << 26); ++iter) {
    if ((uint32_t)(cur >> 32) == tag) {
      const unsigned long long old = atomicAdd(ctr, 1ull);
      const uint32_t t = (uint32_t)old;
      if ((uint32_t)(old >> 32) != tag || t >= (uint32_t)n_tiles) return -1;
      if (t == (uint32_t)n_tiles - 1u) atomicAnd(ctr, 0xffffffff00000000ull);  // last: free
      return (int)t;
    }
    if (!first) return -1;
    // a CTA of this launch has already given up on the slot: so does this one
    if (*reinterpret_cast<volatile unsigned*>(g_gave_up + slot) == tag) return -1;
    if ((uint32_t)cur == 0u) {  // free: claim it
      const unsigned long long prev = atomicCAS(ctr, cur, claim);
      if (prev == cur) return 0;
      cur = prev;  // lost the race (normally to a CTA of this launch): look again
      continue;
    }
    // held by another launch: wait for it to hand out its last tile
    const uint64_t now = global_ns();
    if (t0 == 0) {
      t0 = t_seen = now;
      seen = cur;
    } else if (cur != seen) {
      seen = cur;
      t_seen = now;
    } else if (now - t_seen > kStaleNs) {  // the holder has stopped: take over
      const unsigned long long prev = atomicCAS(ctr, cur, claim);
      if (prev == cur) return 0;
      cur = prev;
      continue;
    }
    if (now - t0 > kScheduleWaitNs) {
      g_gave_up[slot] = tag;
      return -1;
    }
    __nanosleep(sleep_ns);
    if (sleep_ns < 8192) sleep_ns *= 2;
    cur = *vctr;
  }
  return -1;
}

// Tile number of this role's tile tc, published by the producer (-1: no
// tile left, or the wait failed and *failed is set).
__device__ __forceinline__ int read_tile(Barriers* bars, int tc, int* dev_status, bool* failed) {
  if (!mbar_wait(&bars->t_full[tc & 1], (uint32_t)(tc >> 1) & 1u, dev_status, failed)) return -1;
  return *(volatile int*)&bars->t_id[tc & 1];
}

// kForm: 1 = V1 (d_qk 64 per branch, one head), 2 = V2 (d 128 per branch, a head pair).
// kWindow: sliding-window masking compiled in (p.window > 0) or out.
// kSave: also write the training saves p.lse and p.obr.
template <int kForm, bool kWindow, bool kSave>
__global__ void __launch_bounds__(cta_threads(kForm), 1)
    diffattn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                               const __grid_constant__ CUtensorMap tm_k,
                               const __grid_constant__ CUtensorMap tm_v,
                               const __grid_constant__ CUtensorMap tm_o,
                               const __grid_constant__ CUtensorMap tm_obr, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t qbytes = kForm == 1 ? kQTile : 2 * kQTile;
  uint8_t* sQ = smem;
  constexpr int kSt = kv_stages(kForm, kSave);
  uint8_t* sK = smem + qbytes;
  uint8_t* sV = sK + kSt * kKVTile;
  Barriers* bars = reinterpret_cast<Barriers*>(sV + kSt * kKVTile);
  float* x_inv_l = reinterpret_cast<float*>(bars + 1);  // [tile parity][2][128]
  float* x_ss = x_inv_l + 4 * kBM;                       // [tile parity][2][128]
  // output staging (V1; V2 training forward): per softmax warp, its 32 rows x 64 bf16
  // (128-byte rows, the 16-byte chunks of row t at positions c ^ (t & 7));
  // 1024-byte aligned, as the 128-byte swizzle of the TMA box requires
  uint8_t* x_out = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(x_ss + 4 * kBM) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 2);        // released by both branches' score MMAs
    for (int s = 0; s < kSt; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 2);   // released by both branches' MMAs
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 2);
    }
    for (int r = 0; r < 2; ++r) {
      for (int u = 0; u < 2; ++u) {
        mbar_init(&bars->s_full[r][u], 1);
        mbar_init(&bars->p_full[r][u][0], 128);
        mbar_init(&bars->p_full[r][u][1], 128);
        mbar_init(&bars->o_done[r][u], 1);
      }
    }
    mbar_init(&bars->o_free, 256);
    for (int u = 0; u < 2; ++u) {
      mbar_init(&bars->xchg[u], 256);
      mbar_init(&bars->nchg[u], 256);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init(&bars->t_full[u], 1);
      mbar_init(&bars->t_empty[u], tile_readers(kForm));
    }
    mbar_init(&bars->clc_full, 1);
    bars->abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  bool failed = false;

  // Every role walks the same tile sequence, one tile per unit of work (this
  // CTA, then each CTA it cancels), as published by the producer.  Ring
  // slots and buffer phases run on counters (tc tiles, J key tiles) that
  // continue across tiles.
  if (warp == 8) {
    // ------------------------------ TMA producer ---------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      uint32_t J = 0;
      const uint32_t tag = launch_tag();
      int id = take_ticket(p.ticket_slot, p.n_tiles, tag, true);
      if (id < 0) report(p.dev_status, DA_ERR_SCHEDULE);
      for (int tc = 0;; ++tc) {
        // publish the tile number once every role has read the one before last
        const uint32_t u = (uint32_t)tc >> 1;
        if (u > 0 && !mbar_wait(&bars->t_empty[tc & 1], (u - 1) & 1u, p.dev_status, &failed))
          break;
        bars->t_id[tc & 1] = id;
        mbar_arrive(&bars->t_full[tc & 1]);
        if (id < 0) break;
        // Q of the previous tile must be consumed by both branches' score MMAs
        if (tc > 0 && !mbar_wait(&bars->q_empty, (uint32_t)(tc - 1) & 1u, p.dev_status, &failed))
          break;
        const Tile T = tile_at(p, id, kForm, kWindow);
        mbar_arrive_expect_tx(&bars->q_full, qbytes);
        if (kForm == 1) {
          tma_load_4d(sQ, &tm_q, &bars->q_full, 0, T.hh, T.q0, T.b);
          tma_load_4d(sQ + kQBox, &tm_q, &bars->q_full, 64, T.hh, T.q0, T.b);
        } else {
          tma_load_4d(sQ, &tm_q, &bars->q_full, 0, 2 * T.hh, T.q0, T.b);
          tma_load_4d(sQ + kQBox, &tm_q, &bars->q_full, 64, 2 * T.hh, T.q0, T.b);
          tma_load_4d(sQ + 2 * kQBox, &tm_q, &bars->q_full, 0, 2 * T.hh + 1, T.q0, T.b);
          tma_load_4d(sQ + 3 * kQBox, &tm_q, &bars->q_full, 64, 2 * T.hh + 1, T.q0, T.b);
        }
        for (int j = 0; j < T.n_kv; ++j, ++J) {
          const int s = J % kSt;
          const uint32_t ph = (J / kSt) & 1u;
          const int key = (T.kv0 + j) * kBN;
          if (!mbar_wait(&bars->k_empty[s], ph ^ 1u, p.dev_status, &failed)) break;
          mbar_arrive_expect_tx(&bars->k_full[s], kKVTile);
          tma_load_4d(sK + s * kKVTile, &tm_k, &bars->k_full[s], 0, T.kvh, key, T.b);
          tma_load_4d(sK + s * kKVTile + kKVBox, &tm_k, &bars->k_full[s], 64, T.kvh, key, T.b);
          if (!mbar_wait(&bars->v_empty[s], ph ^ 1u, p.dev_status, &failed)) break;
          mbar_arrive_expect_tx(&bars->v_full[s], kKVTile);
          tma_load_4d(sV + s * kKVTile, &tm_v, &bars->v_full[s], 0, T.kvh, key, T.b);
          tma_load_4d(sV + s * kKVTile + kKVBox, &tm_v, &bars->v_full[s], 64, T.kvh, key, T.b);
        }
        if (failed || *(volatile int*)&bars->abort_flag) break;
        // Next unit of work: cancel a CTA that has not started, and take a
        // ticket for it.  Once a request finds none, no request follows.
        mbar_arrive_expect_tx(&bars->clc_full, 16);
        clc_try_cancel(bars->clc_resp, &bars->clc_full);
        if (!mbar_wait(&bars->clc_full, (uint32_t)tc & 1u, p.dev_status, &failed)) break;
        if (clc_response(bars->clc_resp) < 0) {
          id = -1;
        } else {
          id = take_ticket(p.ticket_slot, p.n_tiles, tag, false);
          if (id < 0) report(p.dev_status, DA_ERR_SCHEDULE);
        }
      }
    }
  } else if (warp >= 9 && warp < 9 + score_issuers(kForm)) {
    // ------ score MMA issuer: S_r(j) = Q_r . K(j)^T for branch r = warp - 9 (V2),
    // ------ or for both branches (V1)
    if (lane == 0) {
      const int r0 = score_issuers(kForm) == 1 ? 0 : warp - 9;
      const int r1 = score_issuers(kForm) == 1 ? 2 : r0 + 1;
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t k_addr = smem_u32(sK);
      const int nk = kForm == 1 ? 4 : 8;  // 16-wide k-steps of Q.K^T
      uint32_t J = 0;
      for (int tc = 0;; ++tc) {
        const int id = read_tile(bars, tc, p.dev_status, &failed);
        mbar_arrive(&bars->t_empty[tc & 1]);
        if (id < 0) break;
        const Tile T = tile_at(p, id, kForm, kWindow);
        if (!mbar_wait(&bars->q_full, (uint32_t)tc & 1u, p.dev_status, &failed)) break;
        for (int j = 0; j < T.n_kv; ++j, ++J) {
          const int s = J % kSt;
          if (!mbar_wait(&bars->k_full[s], (J / kSt) & 1u, p.dev_status, &failed)) break;
          const uint32_t kt = k_addr + s * kKVTile;
          for (int r = r0; r < r1; ++r) {
            // buffer J % 2 last held P_r(J-2): its P.V must have completed
            if (J >= 2 && !mbar_wait(&bars->o_done[r][J & 1], ((J - 2) >> 1) & 1u,
                                     p.dev_status, &failed))
              break;
            tc_fence_after();
            for (int kk = 0; kk < nk; ++kk) {
              uint32_t a, bb;
              if (kForm == 1) {  // branch r = columns [64 r, 64 r + 64)
                a = q_addr + r * kQBox + kk * 32;
                bb = kt + r * kKVBox + kk * 32;
              } else {            // branch r = query head 2p + r, full 128 columns
                a = q_addr + r * kQTile + (kk >> 2) * kQBox + (kk & 3) * 32;
                bb = kt + (kk >> 2) * kKVBox + (kk & 3) * 32;
              }
              tc_mma_ss(tmem + s_col(r, J & 1), smem_desc_sw128(a, 16, 1024),
                        smem_desc_sw128(bb, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
            }
            tc_commit(&bars->s_full[r][J & 1]);
            tc_commit(&bars->k_empty[s]);  // one of the two releases of this K stage
          }
          if (failed) break;
        }
        if (failed) break;
        // Q free once both branches' score MMAs are done (one release each)
        for (int r = r0; r < r1; ++r) tc_commit(&bars->q_empty);
      }
    }
  } else if (warp == 9 + score_issuers(kForm) || warp == 10 + score_issuers(kForm)) {
    // ------- P.V MMA issuer of branch r: O_r += P_r(j) . V(j) -------
    if (lane == 0) {
      const int r = warp - 9 - score_issuers(kForm);
      const uint32_t v_addr = smem_u32(sV);
      const uint32_t pcol0 = tmem + s_col(r, 0);
      const uint32_t ocol = tmem + (r == 0 ? kColO1 : kColO2);
      uint32_t J = 0;
      for (int tc = 0;; ++tc) {
        const int id = read_tile(bars, tc, p.dev_status, &failed);
        mbar_arrive(&bars->t_empty[tc & 1]);
        if (id < 0) break;
        const Tile T = tile_at(p, id, kForm, kWindow);
        for (int j = 0; j < T.n_kv; ++j, ++J) {
          const int s = J % kSt;
          if (!mbar_wait(&bars->v_full[s], (J / kSt) & 1u, p.dev_status, &failed)) break;
          // the first P.V of a tile overwrites O: the previous tile's
          // epilogue must have read it out
          if (j == 0 && tc > 0 &&
              !mbar_wait(&bars->o_free, (uint32_t)(tc - 1) & 1u, p.dev_status, &failed))
            break;
          const uint32_t vt = v_addr + s * kKVTile;
          const uint32_t pcol = pcol0 + 64u * (J & 1u);
          // each half of the keys goes out once its P is in tensor memory (V2
          // releases the halves one after the other, V1 both at the end)
          for (int h = 0; h < 2; ++h) {
            if (!mbar_wait(&bars->p_full[r][J & 1][h], (J >> 1) & 1u, p.dev_status, &failed))
              break;
            tc_fence_after();
            for (int kk = 2 * h; kk < 2 * h + 2; ++kk) {
              // B = V tile, MN-major: 64-column halves kKVBox apart, 8-key groups 1 KB apart
              tc_mma_ts(ocol, pcol + kk * 8, smem_desc_sw128(vt + kk * 2048, kKVBox, 1024),
                        kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
            }
          }
          if (failed) break;
          tc_commit(&bars->o_done[r][J & 1]);
          tc_commit(&bars->v_empty[s]);
        }
        if (failed) break;
      }
    }
  } else {
    // ------------------------------ softmax warpgroups ---------------------
    const int r = warp / 4;                  // branch
    const int sub = warp & 3;                // TMEM lane quarter
    const int row = sub * 32 + lane;         // query row within the tile
    const uint32_t lane_off = (uint32_t)(sub * 32) << 16;
    const uint32_t t_o = tmem + lane_off + (r == 0 ? kColO1 : kColO2);
    const float sc = p.scale_log2;
    uint32_t J = 0;
    for (int tc = 0;; ++tc) {
      // tensor-memory accesses below are warp-collective: the tile decision
      // is taken by the whole warp
      int id = read_tile(bars, tc, p.dev_status, &failed);
      id = __shfl_sync(0xffffffffu, __all_sync(0xffffffffu, !failed) ? id : -1, 0);
      __syncwarp();
      if (lane == 0) mbar_arrive(&bars->t_empty[tc & 1]);
      if (id < 0) break;
      const Tile T = tile_at(p, id, kForm, kWindow);
      const int qrow = T.q0 + row;             // query row within the sequence
      const int lim = p.causal ? min(qrow + 1, p.seqlen) : p.seqlen;  // keys < lim visible
      const int lo = kWindow ? max(0, qrow - p.window + 1) : 0;         // and keys >= lo
      float m_ref = -INFINITY, l_run = 0.f;

      for (int j = 0; j < T.n_kv; ++j, ++J) {
        const int buf = J & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[r][buf], (J >> 1) & 1u,
                                                p.dev_status, &failed))) {
          failed = true;
          break;
        }
        tc_fence_after();
        const uint32_t t_s = tmem + lane_off + s_col(r, buf);
        uint32_t sr[64];  // raw S row of this tile (masked entries set to -inf)
        tmem_ld32(t_s, *reinterpret_cast<uint32_t(*)[32]>(sr));
        tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
        tc_wait_ld();
        const int k0 = (T.kv0 + j) * kBN;
        if (k0 + kBN > lim) {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (k0 + c >= lim) sr[c] = __float_as_uint(-INFINITY);
        }
        if (kWindow && k0 < lo) {  // window start (a row may see none of this tile)
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (k0 + c < lo) sr[c] = __float_as_uint(-INFINITY);
        }
        // row maximum: 3-input max over 8 independent chains
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float m = max3(__uint_as_float(sr[i]), __uint_as_float(sr[8 + i]),
                         __uint_as_float(sr[16 + i]));
          m = max3(m, __uint_as_float(sr[24 + i]), __uint_as_float(sr[32 + i]));
          m = max3(m, __uint_as_float(sr[40 + i]), __uint_as_float(sr[48 + i]));
          m8[i] = fmaxf(m, __uint_as_float(sr[56 + i]));
        }
        const float mx = max3(max3(m8[0], m8[1], m8[2]), max3(m8[3], m8[4], m8[5]),
                              fmaxf(m8[6], m8[7])) * sc;  // sc > 0 commutes with max
        float alpha = 1.f;
        bool resc = false;
        if (j == 0) {
          m_ref = mx;
        } else {
          const float m_new = fmaxf(m_ref, mx);
          resc = m_new > m_ref + kLazyTau;
          if (resc) {
            alpha = ex2(m_ref - m_new);
            m_ref = m_new;
          }
        }
        const float u = m_ref == -INFINITY ? 0.f : m_ref;
        // O_r rescaled in place when a row's reference moved: O_r must be
        // quiescent first (the previous tile's P.V into O_r done); rows that
        // keep their reference use alpha 1.  V2 does it before any P of this
        // tile is released to its P.V, V1 after computing P (both orders put
        // the rescale before this tile's P.V).
        auto rescale_o = [&]() -> bool {
          if (!__all_sync(0xffffffffu, mbar_wait(&bars->o_done[r][(J - 1) & 1],
                                                  ((J - 1) >> 1) & 1u, p.dev_status,
                                                  &failed)))
            return false;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t ov[16];
            tmem_ld16(t_o + 16 * c, ov);
            tc_wait_ld();
#pragma unroll
            for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st16(t_o + 16 * c, ov);
          }
          return true;
        };
        if (kForm == 2 && __any_sync(0xffffffffu, resc) && !rescale_o()) {
          failed = true;
          break;
        }
        // p = 2^(s*sc - u): pairs on the f32x2 pipe; some pairs take the
        // polynomial 2^x on the FMA pipe, the rest the multi-function unit.
        const uint64_t sc2 = f2pack(sc, sc), nu2 = f2pack(-u, -u);
        uint64_t ps2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int qt = 0; qt < 2; ++qt) {  // 32 logits -> 16 packed bf16 pairs per store
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = qt * 32 + 2 * e;
            const uint64_t x2 = fma2(f2pack(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])),
                                     sc2, nu2);
            float x0, x1, p0, p1;
            f2unpack(x2, x0, x1);
            // Share of exponentials on the polynomial (both shares and positions
            // measured): one pair in sixteen for V1, whose softmax has 168
            // registers at 12 warps, one in eight for V2 at 13 warps.
            if (kForm == 1 ? e == 3 : (e & 7) == 7) {
              exp2_poly2(x0, x1, p0, p1);
            } else {
              p0 = ex2(x0);
              p1 = ex2(x1);
            }
            ps2[e & 3] = add2(ps2[e & 3], f2pack(p0, p1));
            pk[e] = pack_bf16(p0, p1);
          }
          tmem_st16(t_s + 16 * qt, pk);
          if (kForm == 2) {  // this half of P is ready for its P.V
            tc_wait_st();
            tc_fence_before();
            mbar_arrive(&bars->p_full[r][buf][qt]);
          }
        }
        float psum, psum_hi;
        f2unpack(add2(add2(ps2[0], ps2[1]), add2(ps2[2], ps2[3])), psum, psum_hi);
        psum += psum_hi;
        if (kForm == 1 && __any_sync(0xffffffffu, resc) && !rescale_o()) {
          failed = true;
          break;
        }
        l_run = l_run * alpha + psum;
        if (kForm == 1) {
          tc_wait_st();
          tc_fence_before();
          mbar_arrive(&bars->p_full[r][buf][0]);
          mbar_arrive(&bars->p_full[r][buf][1]);
        }
      }

      // ---- epilogue: o = O1/l1 - lambda O2/l2 (+ V1 norm), channels [64 r, 64 r + 64) ----
      __syncwarp();
      if (failed) bars->abort_flag = 1;
      // own branch's last P.V done; the named barrier then orders both branches
      const uint32_t Jl = J - 1;
      mbar_wait(&bars->o_done[r][Jl & 1], (Jl >> 1) & 1u, p.dev_status, &failed);
      tc_fence_after();
      float* inv_l = x_inv_l + (tc & 1) * 2 * kBM;
      inv_l[r * kBM + row] = 1.0f / l_run;
      if (kSave && qrow < p.seqlen)  // p_ij = 2^(s_ij * sc - lse) for the backward
        p.lse[(((size_t)T.b * p.heads + T.hh) * 2 + r) * p.lse_stride + qrow] =
            (m_ref == -INFINITY ? 0.f : m_ref) + log2f(l_run);
      // both branches' normalisers (bounded wait, unlike a named barrier)
      mbar_arrive(&bars->xchg[tc & 1]);
      mbar_wait(&bars->xchg[tc & 1], (uint32_t)(tc >> 1) & 1u, p.dev_status, &failed);
      const bool stop = *(volatile int*)&bars->abort_flag != 0;
      tc_fence_after();
      const float inv1 = inv_l[row];
      const float inv2_raw = inv_l[kBM + row];
      const float inv2 = inv2_raw * p.lambda[T.hh];
      float o[64];
      {
        // accumulator columns read at a time: the training saves keep fewer in
        // flight, so that O1, O2 and the 64 outputs fit in registers together
        constexpr int kEC = kSave ? 8 : 32;
        uint32_t a[kEC], c2[kEC];
#pragma unroll
        for (int ch = 0; ch < 64 / kEC; ++ch) {
          if constexpr (kEC == 32) {
            tmem_ld32(tmem + lane_off + kColO1 + 64 * r + kEC * ch, a);
            tmem_ld32(tmem + lane_off + kColO2 + 64 * r + kEC * ch, c2);
          } else {
            tmem_ld8(tmem + lane_off + kColO1 + 64 * r + kEC * ch, a);
            tmem_ld8(tmem + lane_off + kColO2 + 64 * r + kEC * ch, c2);
          }
          tc_wait_ld();
          if (ch == 64 / kEC - 1) {  // O fully read: the next tile's first P.V may overwrite it
            tc_fence_before();
            mbar_arrive(&bars->o_free);
          }
#pragma unroll
          for (int e = 0; e < kEC; ++e)
            o[ch * kEC + e] = __uint_as_float(a[e]) * inv1 - __uint_as_float(c2[e]) * inv2;
          if constexpr (kSave && stage_out(kForm, kSave)) {
            // normalised branch outputs, fp32, by TMA stores: this chunk's 8
            // columns of O_1/l_1 and of O_2/l_2 for the warp's 32 rows (1 KB
            // each) go through one half of the warp's staging block, the
            // halves alternating; a half is reused once the store of two
            // chunks ago has read it
            uint8_t* half = x_out + warp * 4096 + (ch & 1) * 2048;
            if (lane == 0) {
              if (ch == 0) bulk_wait_read(); else bulk_wait_read_1();
            }
            __syncwarp();
            float* s1 = reinterpret_cast<float*>(half) + lane * kEC;
            float* s2 = reinterpret_cast<float*>(half + 1024) + lane * kEC;
#pragma unroll
            for (int v4 = 0; v4 < kEC / 4; ++v4) {
              *reinterpret_cast<float4*>(s1 + 4 * v4) =
                  make_float4(__uint_as_float(a[4 * v4]) * inv1, __uint_as_float(a[4 * v4 + 1]) * inv1,
                              __uint_as_float(a[4 * v4 + 2]) * inv1,
                              __uint_as_float(a[4 * v4 + 3]) * inv1);
              *reinterpret_cast<float4*>(s2 + 4 * v4) = make_float4(
                  __uint_as_float(c2[4 * v4]) * inv2_raw, __uint_as_float(c2[4 * v4 + 1]) * inv2_raw,
                  __uint_as_float(c2[4 * v4 + 2]) * inv2_raw,
                  __uint_as_float(c2[4 * v4 + 3]) * inv2_raw);
            }
            fence_proxy_async_smem();
            __syncwarp();
            const bool wr = __all_sync(0xffffffffu, !failed) && !stop;
            if (lane == 0 && wr) {
              tma_store_4d(&tm_obr, half, 64 * r + kEC * ch, T.hh, T.q0 + sub * 32, T.b);
              tma_store_4d(&tm_obr, half + 1024, 128 + 64 * r + kEC * ch, T.hh, T.q0 + sub * 32,
                           T.b);
              bulk_commit();
            }
          } else if (kSave && qrow < p.seqlen) {  // normalised branch outputs, fp32
            float* ob = p.obr + (((size_t)T.b * p.seqlen + qrow) * p.heads + T.hh) * 256 +
                        64 * r + kEC * ch;
#pragma unroll
            for (int v4 = 0; v4 < kEC / 4; ++v4) {
              *reinterpret_cast<float4*>(ob + 4 * v4) =
                  make_float4(__uint_as_float(a[4 * v4]) * inv1, __uint_as_float(a[4 * v4 + 1]) * inv1,
                              __uint_as_float(a[4 * v4 + 2]) * inv1,
                              __uint_as_float(a[4 * v4 + 3]) * inv1);
              *reinterpret_cast<float4*>(ob + 128 + 4 * v4) = make_float4(
                  __uint_as_float(c2[4 * v4]) * inv2_raw, __uint_as_float(c2[4 * v4 + 1]) * inv2_raw,
                  __uint_as_float(c2[4 * v4 + 2]) * inv2_raw,
                  __uint_as_float(c2[4 * v4 + 3]) * inv2_raw);
            }
          }
        }
      }
      float mul = 1.f;
      if (p.apply_norm) {
        float* ssq = x_ss + (tc & 1) * 2 * kBM;
        float ss4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int e = 0; e < 64; ++e) ss4[e & 3] = fmaf(o[e], o[e], ss4[e & 3]);
        ssq[r * kBM + row] = (ss4[0] + ss4[1]) + (ss4[2] + ss4[3]);
        mbar_arrive(&bars->nchg[tc & 1]);
        mbar_wait(&bars->nchg[tc & 1], (uint32_t)(tc >> 1) & 1u, p.dev_status, &failed);
        const float tot = ssq[row] + ssq[kBM + row];
        mul = p.post_scale / sqrtf(tot * (1.0f / 128.0f) + p.eps);
      }
      if constexpr (stage_out(kForm, kSave)) {
        // V1, and the V2 training forward: the warp's 32 rows leave by one
        // TMA tensor store from its staging block (128-byte swizzled, the
        // layout of the output map's box).  Stored directly, each thread's 16-byte stores (rows 4 KB
        // apart) would still be draining when the next tile's first P is
        // released, and that release waits for them; the bulk store is
        // outside that ordering.  Rows past the sequence end are clipped by
        // the map.
        uint8_t* wst = x_out + warp * 4096;
        if (lane == 0) bulk_wait_read();  // the previous tile's store has read the block
        __syncwarp();
#pragma unroll
        for (int v8 = 0; v8 < 8; ++v8) {
          float y[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int c = v8 * 8 + e;
            const float gm = (p.apply_norm && p.norm_weight) ? __ldg(p.norm_weight + 64 * r + c)
                                                             : 1.f;
            y[e] = o[c] * mul * gm;
          }
          uint4 w;
          w.x = pack_bf16(y[0], y[1]);
          w.y = pack_bf16(y[2], y[3]);
          w.z = pack_bf16(y[4], y[5]);
          w.w = pack_bf16(y[6], y[7]);
          *reinterpret_cast<uint4*>(wst + lane * 128 + ((v8 ^ (lane & 7)) << 4)) = w;
        }
        fence_proxy_async_smem();  // visible to the tensor-memory-access unit
        __syncwarp();
        const bool write = __all_sync(0xffffffffu, !failed) && !stop;
        if (lane == 0 && write) {
          tma_store_4d(&tm_o, wst, 64 * r, T.hh, T.q0 + sub * 32, T.b);
          bulk_commit();
        }
      } else if (qrow < p.seqlen && !stop && !failed) {
        __nv_bfloat16* dst =
            p.out + (((size_t)T.b * p.seqlen + qrow) * p.heads + T.hh) * 128 + 64 * r;
#pragma unroll
        for (int v8 = 0; v8 < 8; ++v8) {
          float y[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int c = v8 * 8 + e;
            const float gm = (p.apply_norm && p.norm_weight) ? __ldg(p.norm_weight + 64 * r + c)
                                                             : 1.f;
            y[e] = o[c] * mul * gm;
          }
          uint4 w;
          w.x = pack_bf16(y[0], y[1]);
          w.y = pack_bf16(y[2], y[3]);
          w.z = pack_bf16(y[4], y[5]);
          w.w = pack_bf16(y[6], y[7]);
          *reinterpret_cast<uint4*>(dst + v8 * 8) = w;
        }
      }
      if (__any_sync(0xffffffffu, failed) || stop) break;
    }
  }

  // ---- teardown: every role reaches this point, then TMEM is released ----
  if (stage_out(kForm, kSave) && warp < 8 && lane == 0) bulk_wait_all();
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}
// Host side of the tile counters: the slot the next launch takes.
std::atomic<unsigned> g_next_slot{0};

// Self-test: keeps counter `slot` held by `tag` with a count that changes
// every ~20 us (a launch in flight, as another launch sees it) for
// `duration_ns`, then frees it.
__global__ void keep_ticket_word_kernel(int slot, unsigned tag, unsigned long long duration_ns) {
  const uint64_t t0 = global_ns();
  unsigned k = 1;
  while (global_ns() - t0 < duration_ns) {
    g_tickets[slot] = ((unsigned long long)tag << 32) | (unsigned long long)k;
    k = k % 1000000u + 1u;
    __nanosleep(20000);
  }
  g_tickets[slot] = (unsigned long long)tag << 32;
}

__global__ void set_ticket_word_kernel(int slot, unsigned long long value) {
  if (slot < 0) {
    for (int i = 0; i < kTicketSlots; ++i) {
      g_tickets[i] = 0ull;
      g_gave_up[i] = 0u;
    }
  } else {
    g_tickets[slot] = value;
  }
}
}  // namespace

cudaError_t reset_tile_counters(cudaStream_t stream) {
  set_ticket_word_kernel<<<1, 1, 0, stream>>>(-1, 0ull);
  return cudaGetLastError();
}

cudaError_t hold_tile_counter(int slot, unsigned tag, unsigned count, cudaStream_t stream) {
  if (slot < 0 || slot >= kTicketSlots) return cudaErrorInvalidValue;
  set_ticket_word_kernel<<<1, 1, 0, stream>>>(
      slot, ((unsigned long long)tag << 32) | (unsigned long long)count);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) g_next_slot.store((unsigned)slot, std::memory_order_relaxed);
  return e;
}

cudaError_t keep_tile_counter(int slot, unsigned tag, unsigned duration_ms,
                              cudaStream_t stream) {
  if (slot < 0 || slot >= kTicketSlots || duration_ms == 0 || duration_ms > 10000)
    return cudaErrorInvalidValue;
  keep_ticket_word_kernel<<<1, 1, 0, stream>>>(slot, tag, 1000000ull * duration_ms);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) g_next_slot.store((unsigned)slot, std::memory_order_relaxed);
  return e;
}

cudaError_t launch_prefill_tc(const CUtensorMap& tm_q, const CUtensorMap& tm_k,
                              const CUtensorMap& tm_v, const PrefillArgs& a, int num_sms,
                              cudaStream_t stream) {
  (void)num_sms;
  Params p;
  p.form = a.form;
  p.batch = a.batch;
  p.seqlen = a.seqlen;
  p.heads = a.heads;
  p.pairs_per_kv = a.pairs_per_kv;
  p.n_qtiles = (a.seqlen + kBM - 1) / kBM;
  p.ticket_slot = (int)(g_next_slot.fetch_add(1u, std::memory_order_relaxed) % kTicketSlots);
  // Heads (V1) or pairs (V2) scheduled together: the KV heads of a group
  // keep their K and V (2 x seqlen x 128 bf16 each) within about half of the
  // L2, and a group has at most 8 KV heads (8 ran 1 % faster than 32 at 4k
  // and 8k tokens, where the L2 would hold 32 and 16).
  const double kv_bytes = 2.0 * a.seqlen * 128 * 2;
  const int bh_count = a.batch * a.heads;
  const int kv_group = std::min(8, (int)((64.0 * 1024 * 1024) / kv_bytes));
  int grp = kv_group * a.pairs_per_kv;
  grp = grp < a.pairs_per_kv ? a.pairs_per_kv : grp;
  p.group = grp > bh_count ? bh_count : grp;
  p.causal = a.causal;
  p.window = a.window;
  const double d = a.form == 1 ? 64.0 : 128.0;  // width of one branch's query
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt(d));
  p.lambda = a.lambda;
  p.apply_norm = a.apply_norm;
  p.norm_weight = a.norm_weight;
  p.eps = a.eps;
  p.post_scale = a.post_scale;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.lse_stride = a.lse_stride;
  p.obr = static_cast<float*>(a.obr);
  p.dev_status = a.dev_status;
  const int qbytes = a.form == 1 ? kQTile : 2 * kQTile;
  const int smem = 1024 + qbytes + 2 * kv_stages(a.form, a.lse && a.obr) * kKVTile +
                   (int)sizeof(Barriers) +
                   8 * kBM * (int)sizeof(float) +
                   (stage_out(a.form, a.lse && a.obr) ? 8 * 4096 + 1024 : 0) + 64;
  const bool win = a.window > 0;
  decltype(&diffattn_prefill_tc_kernel<1, false, false>) kern;
  if (a.lse && a.obr)  // training forward
    kern = a.form == 1 ? (win ? diffattn_prefill_tc_kernel<1, true, true>
                              : diffattn_prefill_tc_kernel<1, false, true>)
                       : (win ? diffattn_prefill_tc_kernel<2, true, true>
                              : diffattn_prefill_tc_kernel<2, false, true>);
  else
    kern = a.form == 1 ? (win ? diffattn_prefill_tc_kernel<1, true, false>
                              : diffattn_prefill_tc_kernel<1, false, false>)
                       : (win ? diffattn_prefill_tc_kernel<2, true, false>
                              : diffattn_prefill_tc_kernel<2, false, false>);
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const long long grid = (long long)p.n_qtiles * bh_count;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidValue;
  p.n_tiles = (int)grid;
  // output [B][N][heads][128] in boxes of 64 columns x 32 rows, for the
  // instantiations that store through shared memory (unused by the others)
  CUtensorMap tm_o = tm_q;
  if (stage_out(a.form, a.lse && a.obr) &&
      make_tmap_bf16_4d(&tm_o, a.out, 128, (uint64_t)a.heads, (uint64_t)a.seqlen,
                        (uint64_t)a.batch, 64, 1, 32, 1) != 0)
    return cudaErrorInvalidValue;
  // training saves O_r / l_r [B][N][heads][256] fp32 in boxes of 8 columns x 32 rows
  CUtensorMap tm_obr = tm_q;
  if (a.lse && a.obr && stage_out(a.form, true) &&
      make_tmap_f32_4d(&tm_obr, a.obr, 256, (uint64_t)a.heads, (uint64_t)a.seqlen,
                       (uint64_t)a.batch, 8, 1, 32, 1) != 0)
    return cudaErrorInvalidValue;
  kern<<<(unsigned)grid, cta_threads(a.form), smem, stream>>>(tm_q, tm_k, tm_v, tm_o, tm_obr, p);
  return cudaGetLastError();
}

}  // namespace da
