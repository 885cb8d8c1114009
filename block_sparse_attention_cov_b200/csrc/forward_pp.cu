// forward_pp.cu -- fused Sol-Attn forward for sm_100a whose softmax warps
// "ping-pong" between alternate key tiles: the kernel behind solattn_forward
// (threshold rule, block-level correction) and solattn_dense.
//
// Method: "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly
// Attention Sparsification" (pages: hotpaper.ai abstract; paithon.it sections
// "Una soglia per ogni riga" and "Scegliere mentre si calcola"). For every
// query block i the proxy scores s_hat_ij = qbar_i . kbar_j / sqrt(d) are
// produced one key block at a time and compared with tau_i = mu_i + beta sigma_i
// on the fly; blocks above tau_i are attended exactly, the others are folded in
// through the zeroth-order Taylor term n_j e^{s_hat_ij} (vbar_j in the
// numerator) in the same online-softmax state. The proxy row never leaves the
// SM.
//
// Work unit: two adjacent 64-token query blocks of one head (128 rows, the
// full-rate tcgen05 tile height). Its key tiles are the union of the two
// blocks' kept sets, two kept blocks per 128-key tile; a row masks the blocks
// its own query block did not keep (P = 0, state untouched), so each block's
// result is exactly its own.
//
// One persistent CTA per SM, one unit at a time. TMEM holds three S slots
// (128 fp32 columns each; the bf16 P of a tile is written over its own S) and
// one O accumulator: the QKs of the next two tiles run while a tile's softmax
// is computed. The softmax is split over two warp groups that take alternate
// tiles (group 0 the even tiles, group 1 the odd ones), one thread per row and
// a whole 128-key row per thread; each SM sub-partition hosts one warp of each
// group, so the serial steps of one tile (S wait, TMEM loads, row max, P
// store) overlap the exponentials of the next.
//
// Both groups feed the one O, so all P of a row share one reference max m.
// It only moves up, and lazily (when a tile's max exceeds it by more than 16 in
// log2 units), and it is kept integral, so every rescale is an exact power of
// two. A group computes a tile's P with the reference it last knew, then
// receives the reference the other group settled for the previous tile (a
// one-way handshake per row group), reconciles (rescales P or O by a power of
// two, rarely), and passes its own on.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cmath>
#include <cstdint>

#include "fwd_common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace solattn {

namespace {

constexpr int kThreadsPP = 512;  // 16 warps, 128 registers per thread at launch
constexpr int kSSlots = 3;       // S slots in TMEM
constexpr uint32_t kColO = kSSlots * 128;

template <int D>
struct __align__(1024) SmemPP {
#ifndef SOLATTN_PP_KSTAGES
#define SOLATTN_PP_KSTAGES 3
#define SOLATTN_PP_VSTAGES 4
#endif
  static constexpr int kKStages = D == 128 ? SOLATTN_PP_KSTAGES : 4;  // 128-key K tiles
  static constexpr int kVStages = D == 128 ? SOLATTN_PP_VSTAGES : 8;  // 64-key V blocks
  uint8_t qt[kBM * D * 2];               // Q tile of the unit, SW128 K-major panels of 128 rows
  uint8_t kt[kKStages][kBM * D * 2];     // K tiles: two blocks stacked in every 64-column panel
  uint8_t vt[kVStages][kBN * D * 2];     // V blocks, SW128 panels of 64 rows
  // ---- routing (names as route_unit expects; route slot = unit number % 2)
  float rchunk[2][kChunk][D];
  float cnum[2][2][D];
  float cden[2][2];
  float cmax[2][2];
  int unit[2];
  int count[2];
  float rq[2][D];
  float rstat[4][4];
  float rscore[2][kChunk];
  float rweight[2][kChunk];
  float rscale[2];
  float rmax[2];
  float rden[2];
  int rkept[2];
  uint32_t bits[2][2][kNbMax / 32];
  float score[1][1];  // top-k / top-p only (not instantiated here)
  uint32_t cut[2];
  int keep_none[2];
  // ---- barriers
  uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[kSSlots], p_full[kSSlots], pv_done[kSSlots];
  uint64_t o_free[2];  // per route slot: both groups' epilogues have read O
  uint64_t q_full, q_free;
  uint64_t route_full[2], route_empty[2];
  uint64_t rfull[2];
  uint64_t mma_done[2];
  uint64_t e_full[8];
  uint64_t hand[4];          // per row group: the one-way handshake between the two softmax groups
  uint32_t kentry[8][2];     // key-list entries of the key tiles, published by the K producer
  float xm[kBM];             // per row: the reference max passed with the handshake
  float xl[kBM];             // per row: row sums exchanged at the end of a unit
  uint32_t tmem_base;
  int bcast;
  int abort_flag;
};

static_assert(sizeof(SmemPP<128>) + 1024 <= 232448, "shared memory layout too large");
static_assert(sizeof(SmemPP<64>) + 1024 <= 232448, "shared memory layout too large");

// One softmax half-tile: P = 2^(S sl2 - m) for 64 keys into 32 packed bf16x2
// words, their fp32 sum into l. Masked keys (-inf) give P = 0.
__device__ __forceinline__ void softmax_half(const uint32_t (&sv)[64], float sl2, float m, float& l,
                                             uint32_t (&pw)[32]) {
  const uint64_t sc2 = f2_dup(sl2);
  const uint64_t nm2 = f2_dup(-m);
  uint64_t lsum = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    softmax_slice(&sv[16 * q], sc2, nm2, lsum, *reinterpret_cast<uint32_t(*)[8]>(&pw[8 * q]));
  float l0, l1;
  f2_split(lsum, l0, l1);
  l = l0 + l1;
}

// 2^k for an integral k <= 0 (k = -inf allowed) as an fp32; 0 below the
// normal range.
__device__ __forceinline__ float pow2_f32(float k) {
  return k < -126.f ? 0.f : __int_as_float((127 + static_cast<int>(k)) << 23);
}

// The same power of two as a bf16 pair (bf16 has fp32's exponent range).
__device__ __forceinline__ uint32_t pow2_bf16x2(float k) {
  const uint32_t h = __float_as_uint(pow2_f32(k)) >> 16;
  return h | (h << 16);
}

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Rare paths of the softmax, out of line to keep its hot loop small (the
// softmax warps share each SM sub-partition's instruction cache with the
// routing, producer and issuer warps). Warp-collective: every lane calls them;
// a lane with k = 0 leaves its row unchanged.
// 32 TMEM columns of packed bf16 P (one 64-key half) times 2^k.
static __device__ __noinline__ void rescale_p_half(uint32_t taddr, float k) {
  const uint32_t f2 = pow2_bf16x2(k);
  uint32_t pw[32];
  tmem_ld32_wait(taddr, pw);
#pragma unroll
  for (int i = 0; i < 32; ++i) pw[i] = mul_bf16x2(pw[i], f2);
  tmem_st32_wait(taddr, pw);
}

// The thread's row of O (D fp32 columns) times 2^k.
template <int D>
static __device__ __noinline__ void rescale_o_row(uint32_t colO, float k) {
  const float f = pow2_f32(k);
#pragma unroll 1
  for (int ch = 0; ch < D / 16; ++ch) {
    uint32_t ov[16];
    tmem_ld16_wait(colO + ch * 16, ov);
#pragma unroll
    for (int x = 0; x < 16; ++x) ov[x] = __float_as_uint(__uint_as_float(ov[x]) * f);
    tmem_st16_wait(colO + ch * 16, ov);
  }
}

// One kept 64-key half of a tile, out of line so that both halves run the
// same, warm copy of the code (a jump over an inlined copy, when a half is not
// kept, missed the instruction cache for about a thousand cycles): loads S of
// the half (TMEM columns s_col .. s_col + 63), masks pad keys (nv valid), and
// raises the reference ms when the half's max exceeds it by more than the
// slack (to an integer, in log2 units; the other half's P already stored at
// s_col - 64 is then rescaled when `other` is set); stores P = 2^(S sl2 - ms)
// as bf16 over S columns s_col - 32 h .. (the half's own first 32 columns for
// half 0, columns 32-63 of the tile for half 1) and returns (ms, sum of P).
static __device__ __noinline__ float2 softmax_half_tmem(uint32_t s_col, int nv, float ms, float sl2, bool other) {
  uint32_t sv[64];
  tmem_ld32x2_wait(s_col, s_col + 32, sv);
  if (nv < kBN) mask_tail(sv, nv);
  const float mx = tile_max(sv, kBN) * sl2;
  const bool raise = mx > ms + kRescaleSlack;
  if (__any_sync(0xffffffffu, raise)) {
    const float mr = raise ? ceilf(mx) : ms;
    // the tile's first half (P at s_col - 64) follows the raised reference
    if (other) rescale_p_half(s_col - 64, raise && ms != -INFINITY ? ms - mr : 0.f);
    ms = mr;
  }
  uint32_t pw[32];
  float l;
  softmax_half(sv, sl2, ms, l, pw);
  // half 0: s_col is the tile's column 0, P goes to 0-31; half 1: s_col is
  // column 64, P goes to 32-63
  tmem_st32_wait(s_col - ((s_col & 64u) ? 32u : 0u), pw);
  return make_float2(ms, l);
}

// ---------------------------------------------------------------------------
// The kernel. 512 threads = 16 warps:
//   warps 0-3   softmax group 0 (even key tiles), warps 4-7 group 1 (odd key
//               tiles); warp w holds rows 32 (w % 4) .. + 31 of the unit (TMEM
//               lanes), one row per thread. At the end of a unit both groups
//               write the output, group g the columns g d / 2 .. (g + 1) d / 2:
//               O and the row sums merged with the skipped-block correction
//   warps 8-11  routing, one unit ahead; then the unit's Q tile by TMA once
//               every QK of the previous unit has completed
//   warp 12     TMA producer of the K tiles; publishes each tile's list entries
//   warp 13     MMA issuer for QK (one elected lane), up to two tiles ahead
//   warp 14     TMA producer of the V blocks
//   warp 15     MMA issuer for PV
// ---------------------------------------------------------------------------
template <int D, bool ROUTE>
__global__ void __launch_bounds__(kThreadsPP, 1)
    solattn_fwd_pp_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const Params P) {
  using SmemT = SmemPP<D>;
  constexpr int KS = SmemT::kKStages, VS = SmemT::kVStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* aligned = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  SmemT& sm = *reinterpret_cast<SmemT*>(aligned);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  DeviceStatus* st = P.status;
  volatile int* abort_flag = &sm.abort_flag;

  if (tid == 0) {
    for (int i = 0; i < KS; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
    }
    for (int i = 0; i < VS; ++i) {
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.v_empty[i], 1);
    }
    for (int i = 0; i < kSSlots; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], 4);  // the four warps of the tile's softmax group
      mbar_init(&sm.pv_done[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.route_full[i], 1);
      mbar_init(&sm.route_empty[i], 12);  // 2 producers + 2 MMA issuers + 8 softmax warps
      mbar_init(&sm.rfull[i], 1);
      mbar_init(&sm.o_free[i], 8);
      mbar_init(&sm.mma_done[i], 1);
    }
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_free, 1);
    for (int i = 0; i < 8; ++i) mbar_init(&sm.e_full[i], 1);
    for (int i = 0; i < 4; ++i) mbar_init(&sm.hand[i], 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 13) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 12 && lane == 0) {
    prefetch_tensormap(&tmQ);
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // Registers: the softmax warp groups take 152 per thread, the routing and
  // producer / issuer warp groups give theirs down to 104 (256 x 152 +
  // 256 x 104 = the 65,536 the CTA was launched with).
  if (warp >= 8 && warp < 12) {
    regs_dec<104>();
    // ======================= routing =======================
    const int rt = tid - 256;
    uint32_t chunk_ctr = 0;  // routing chunks consumed so far (buffer parity)
    uint32_t q_loads = 0;    // Q tiles requested so far (q_full phase)
    for (int n = 0;; ++n) {
      const int s = n & 1;
      if (n >= 2) {
        bool okw = true;
        if (rt == 0) okw = mbar_wait(&sm.route_empty[s], ((n >> 1) - 1) & 1, abort_flag, st, kSiteRouteEmpty, 0);
        if (named_bar_or(1, 128, !okw)) break;
      }
      if (rt == 0) sm.bcast = static_cast<int>(atomicAdd(&st->tile_counter, 1u));
      named_bar_sync(1, 128);
      const int u = sm.bcast;
      named_bar_sync(1, 128);
      if (u >= P.units) {
        if (rt == 0) {
          sm.unit[s] = -1;
          sm.count[s] = 0;
          mbar_arrive(&sm.route_full[s]);
        }
        break;
      }
      const int bh = u / P.npairs, pair = u % P.npairs;
      if constexpr (ROUTE) {
        if (!route_unit<D, 0>(sm, P, s, bh, pair, rt, chunk_ctr, abort_flag, st, u)) break;
      } else {
        if (rt == 0) {
          sm.count[s] = P.NB;
          sm.cden[s][0] = sm.cden[s][1] = 0.f;
          sm.cmax[s][0] = sm.cmax[s][1] = -INFINITY;
        }
      }
      named_bar_sync(1, 128);
      // the list is complete: producers may run ahead into this unit
      if (rt == 0) {
        sm.unit[s] = u;
        mbar_arrive(&sm.route_full[s]);
      }
      // the Q tile is free once every QK of the previous unit has completed
      bool okq = true;
      if (rt == 0) {
        if (n >= 1) okq = mbar_wait(&sm.q_free, (n - 1) & 1, abort_flag, st, kSiteQFree, u);
        if (okq) {
          ++q_loads;
          mbar_arrive_expect_tx(&sm.q_full, kBM * D * 2);
#pragma unroll
          for (int pnl = 0; pnl < D / 64; ++pnl)
            tma_load_4d(&sm.qt[pnl * kBM * 128], &tmQ, &sm.q_full, pnl * 64, pair * kBM, bh % P.H, bh / P.H);
        }
      }
      if (named_bar_or(1, 128, !okq)) break;
    }
    if (rt == 0 && q_loads > 0) mbar_wait_quiet(&sm.q_full, (q_loads - 1) & 1);  // teardown: the last Q copy landed
  } else if (warp == 12 || warp == 14) {
    regs_dec<104>();
    // ======================= TMA producers: warp 12 = K tiles, warp 14 = V blocks =======================
    const bool isK = warp == 12;
    uint32_t g = 0;  // K: global tile index; V: global block index
    for (int n = 0;; ++n) {
      const int s = n & 1;
      if (!warp_wait(&sm.route_full[s], (n >> 1) & 1, abort_flag, st, kSiteRouteFullProd, 0)) break;
      const int u = sm.unit[s];
      if (u < 0) break;
      const int T = sm.count[s];
      const int bh = u / P.npairs;
      bool ok = true;
      KeyWalk<ROUTE> walk(sm.bits[s][0], sm.bits[s][1]);
      if (isK) {
        const int TT = (T + 1) / 2;
        int t = 0;
        for (; t < TT; ++t) {
          const uint32_t gt = g + t, stg = gt % KS, r = gt / KS;
          if (r >= 1 && !warp_wait(&sm.k_empty[stg], (r - 1) & 1, abort_flag, st, kSiteKEmpty, u)) break;
          const int nb = (2 * t + 1 < T) ? 2 : 1;
          const uint32_t e0 = walk.next(), e1 = nb == 2 ? walk.next() : 0u;
          // Publish the tile's entries for the softmax groups. Slot reuse is
          // safe: this tile's stage was released by QK(t - 3), so the softmax
          // has finished tile t - 6, and with it, in the same group, t - 8.
          if (elect_one()) {
            sm.kentry[gt & 7][0] = e0;
            sm.kentry[gt & 7][1] = e1;
            mbar_arrive(&sm.e_full[gt & 7]);
          }
          __syncwarp();
#ifdef SOLATTN_TEST_HOOKS
          if (gt == 0 && static_cast<int>(blockIdx.x) == g_hook_skip_cta) continue;  // this tile never arrives
#endif
          if (elect_one()) {
            mbar_arrive_expect_tx(&sm.k_full[stg], nb * kBN * D * 2);
            const uint32_t jj[2] = {e0 & 0x3FFFu, e1 & 0x3FFFu};
            for (int h = 0; h < nb; ++h) {
#pragma unroll
              for (int pnl = 0; pnl < D / 64; ++pnl)
                tma_load_4d(&sm.kt[stg][pnl * kBM * 128 + h * kBN * 128], &tmK, &sm.k_full[stg], pnl * 64,
                            static_cast<int>(jj[h]) * kBN, bh % P.H, bh / P.H);
            }
          }
          __syncwarp();
        }
        g += t;
        ok = t == TT;
      } else {
        int t = 0;
        for (; t < T; ++t) {
          const int j = static_cast<int>(walk.next() & 0x3FFFu);
          const uint32_t gt = g + t, stg = gt % VS, r = gt / VS;
          if (r >= 1 && !warp_wait(&sm.v_empty[stg], (r - 1) & 1, abort_flag, st, kSiteVEmpty, u)) break;
          if (elect_one()) {
            mbar_arrive_expect_tx(&sm.v_full[stg], kBN * D * 2);
#pragma unroll
            for (int pnl = 0; pnl < D / 64; ++pnl)
              tma_load_4d(&sm.vt[stg][pnl * kBN * 128], &tmV, &sm.v_full[stg], pnl * 64, j * kBN, bh % P.H,
                          bh / P.H);
          }
          __syncwarp();
        }
        g += t;
        ok = t == T;
      }
      if (!ok) break;  // aborted
      if (elect_one()) mbar_arrive(&sm.route_empty[s]);
      __syncwarp();
    }
    if (lane == 0) {  // teardown: every issued copy lands before the CTA exits
      const uint32_t depth = isK ? KS : VS;
      for (uint32_t gt = g > depth ? g - depth : 0u; gt < g; ++gt) {
        if (isK) mbar_wait_quiet(&sm.k_full[gt % KS], (gt / KS) & 1);
        else mbar_wait_quiet(&sm.v_full[gt % VS], (gt / VS) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 13 || warp == 15) {
    regs_dec<104>();
    // ======================= MMA issuers: warp 13 = QK, warp 15 = PV =======================
    // QK(t) goes into S slot t % 3 as soon as its K tile has landed and the PV
    // that last read P from that slot (tile t - 3) has completed (MMAs into
    // different accumulators are not ordered with each other). PV(t) goes as
    // soon as the tile's softmax group stored P(t) and its V blocks landed;
    // PVs into O are ordered among themselves.
    const bool isQK = warp == 13;
    constexpr uint32_t idesc_qk2 = idesc_bf16_f32(kBM, 2 * kBN, false, false);
    constexpr uint32_t idesc_qk1 = idesc_bf16_f32(kBM, kBN, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
    const uint64_t qdesc = sw128_desc(smem_u32(&sm.qt[0]), 16, 1024);
    const uint64_t kdesc0 = sw128_desc(smem_u32(&sm.kt[0][0]), 16, 1024);
    const uint64_t vdesc0 = sw128_desc(smem_u32(&sm.vt[0][0]), 8192, 1024);
    const uint32_t colO = tmem + kColO;
    uint32_t gtile = 0, gblk = 0;
    uint32_t pv_waited = 0;  // QK issuer: tiles whose PV completion it has observed
    bool ok = true;
    for (int n = 0; ok; ++n) {
      const int s = n & 1;
      if (!warp_wait(&sm.route_full[s], (n >> 1) & 1, abort_flag, st, kSiteRouteFullMma, 0)) break;
      tc_fence_after();
      const int u = sm.unit[s];
      if (u < 0) break;
      const int T = sm.count[s];
      const int TT = (T + 1) / 2;
      if (isQK) {
        if (!warp_wait(&sm.q_full, n & 1, abort_flag, st, kSiteQFull, u)) break;
        if (TT == 0) {  // nothing to multiply: release the Q tile
          if (elect_one()) mma_commit(&sm.q_free);
          __syncwarp();
        }
        for (int t = 0; t < TT && ok; ++t) {
          const uint32_t gt = gtile + t, stg = gt % KS, slot = gt % kSSlots;
          for (; pv_waited + kSSlots <= gt && ok; ++pv_waited)
            ok = warp_wait(&sm.pv_done[pv_waited % kSSlots], (pv_waited / kSSlots) & 1, abort_flag, st,
                           kSitePvDone, u);
          if (ok) ok = warp_wait(&sm.k_full[stg], (gt / KS) & 1, abort_flag, st, kSiteKFull, u);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            const uint64_t kd = kdesc0 + ((stg * (kBM * D * 2)) >> 4);
            const uint32_t idesc = (2 * t + 1 < T) ? idesc_qk2 : idesc_qk1;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (((kk / 4) * kBM * 128) + (kk % 4) * 32) >> 4;
              mma_ss(tmem + slot * 128, qdesc + off, kd + off, idesc, kk > 0 ? 1u : 0u);
            }
            mma_commit(&sm.s_full[slot]);
            mma_commit(&sm.k_empty[stg]);
            if (t == TT - 1) mma_commit(&sm.q_free);
          }
          __syncwarp();
        }
      } else {
        // O is free once both groups' epilogues have read the previous unit's
        if (n >= 1 && !warp_wait(&sm.o_free[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag, st, kSiteOFree, u)) break;
        for (int t = 0; t < TT && ok; ++t) {
          const uint32_t gt = gtile + t;
          const int nb = (2 * t + 1 < T) ? 2 : 1;
          // V first: it has normally landed long before P, so once P is
          // stored only the issue remains
          uint32_t stv[2] = {0, 0};
          for (int h = 0; h < nb && ok; ++h) {
            const uint32_t gv = gblk + 2 * t + h;
            stv[h] = gv % VS;
            ok = warp_wait(&sm.v_full[stv[h]], (gv / VS) & 1, abort_flag, st, kSiteVFull, u);
          }
          if (ok) ok = warp_wait(&sm.p_full[gt % kSSlots], (gt / kSSlots) & 1, abort_flag, st, kSitePFull, u);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            const uint32_t colP = tmem + (gt % kSSlots) * 128;
            for (int h = 0; h < nb; ++h) {
              const uint64_t vd = vdesc0 + ((stv[h] * (kBN * D * 2)) >> 4);
#pragma unroll
              for (int kk = 0; kk < kBN / 16; ++kk)
                mma_ts(colO, colP + h * 32 + kk * 8, vd + ((kk * 2048) >> 4), idesc_pv,
                       (t > 0 || h > 0 || kk > 0) ? 1u : 0u);
              mma_commit(&sm.v_empty[stv[h]]);
            }
            mma_commit(&sm.pv_done[gt % kSSlots]);
          }
          __syncwarp();
        }
      }
      if (!ok) break;
      if (elect_one()) mbar_arrive(&sm.route_empty[s]);
      __syncwarp();
      gtile += TT;
      gblk += T;
    }
    const int me = isQK ? 0 : 1;
    if (elect_one()) mma_commit(&sm.mma_done[me]);  // teardown: issued MMAs complete before TMEM is freed
    __syncwarp();
    mbar_wait_quiet(&sm.mma_done[me], 0);
    __syncwarp();
  } else {
    regs_inc<152>();
    // ======================= softmax (warps 0-7) =======================
    const int grp = warp >> 2, wq = warp & 3;
    const int r = wq * 32 + lane;  // row of the unit == TMEM lane
    const int blk = r >> 6;        // query block of the row (warp-uniform)
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t colO = tmem + kColO + lane_off;
    const float sl2 = kLog2e * rsqrtf(static_cast<float>(D));
    const int nlast = P.N - (P.NB - 1) * kBN;
    uint64_t* hand = &sm.hand[wq];
    uint32_t gtile = 0;  // key tiles of the CTA so far (both groups)
    uint32_t hk = 0;     // handshakes of this row group so far (both directions)
    for (int n = 0;; ++n) {
      const int s = n & 1;
      if (!warp_wait<1>(&sm.route_full[s], (n >> 1) & 1, abort_flag, st, kSiteRouteFullSoft, 0)) break;
      tc_fence_after();
      const int u = sm.unit[s];
      if (u < 0) break;
      const int T = sm.count[s];
      const int TT = (T + 1) / 2;
      float m = -INFINITY;  // this group's view of the row's reference max
      float l = 0.f;        // this group's partial row sum, relative to m
      bool ok = true;
      for (int t = (static_cast<int>(gtile) + grp) & 1; t < TT; t += 2) {
        const uint32_t gt = gtile + t, slot = gt % kSSlots;
        const uint32_t colS = tmem + slot * 128 + lane_off;
        ok = warp_wait<1>(&sm.e_full[gt & 7], (gt >> 3) & 1, abort_flag, st, kSiteEFull, u);
        if (!ok) break;
        const int nb = (2 * t + 1 < T) ? 2 : 1;
        const uint32_t en0 = sm.kentry[gt & 7][0], en1 = sm.kentry[gt & 7][1];
        const bool kept0 = (en0 >> (14 + blk)) & 1u;
        const bool kept1 = nb == 2 && ((en1 >> (14 + blk)) & 1u);
        const int nv0 = (en0 & 0x3FFFu) == static_cast<uint32_t>(P.NB - 1) ? nlast : kBN;
        const int nv1 = (en1 & 0x3FFFu) == static_cast<uint32_t>(P.NB - 1) ? nlast : kBN;
        ok = warp_wait<1>(&sm.s_full[slot], (gt / kSSlots) & 1, abort_flag, st, kSiteSFull, u);
        if (!ok) break;
        tc_fence_after();
        // ---- P with this group's reference (raised by this tile if needed),
        // one kept 64-key half at a time (P of half h over S columns
        // 32 h .. 32 h + 31; S of keys 64-127 is read before half 1's P is
        // stored). A half the row's query block did not keep gets P = 0 below.
        float ms = m, lt = 0.f;
        if (kept0) {
          const float2 r0 = softmax_half_tmem(colS, nv0, ms, sl2, false);
          ms = r0.x;
          lt = r0.y;
        }
        if (kept1) {
          const float2 r1 = softmax_half_tmem(colS + 64, nv1, ms, sl2, kept0);
          // a raise in the second half rescaled the first half's P: its sum follows
          lt = (r1.x > ms && ms != -INFINITY) ? lt * pow2_f32(ms - r1.x) : lt;
          ms = r1.x;
          lt += r1.y;
        }
        // ---- the previous tile's reference, from the other group
        float mp = -INFINITY;
        if (t > 0) {
          ok = warp_wait<1>(hand, hk & 1, abort_flag, st, kSiteMlReady, u);
          ++hk;
          if (!ok) break;
          mp = sm.xm[r];
        }
        const float mf = fmaxf(ms, mp);
        // P was computed relative to ms: bring it to mf (rare)
        const bool fixp = mf > ms && ms != -INFINITY;
        if (__any_sync(0xffffffffu, fixp)) {
          for (int hh = 0; hh < nb; ++hh) rescale_p_half(colS + 32 * hh, fixp ? ms - mf : 0.f);
        }
        lt = (ms == -INFINITY) ? lt : lt * pow2_f32(ms - mf);
        // O holds the tiles before this one relative to mp: bring it to mf
        // once the previous tile's PV has completed (rare)
        const bool reso = mf > mp && mp != -INFINITY;
        if (__any_sync(0xffffffffu, reso)) {
          ok = warp_wait<1>(&sm.pv_done[(gt - 1) % kSSlots], ((gt - 1) / kSSlots) & 1, abort_flag, st,
                            kSitePvDone, u);
          if (!ok) break;
          tc_fence_after();
          rescale_o_row<D>(colO, reso ? mp - mf : 0.f);
        }
        l = ((m == -INFINITY) ? 0.f : l * pow2_f32(m - mf)) + lt;
        m = mf;
        // ---- zero P for the halves not kept: issued last (a TMEM store into a
        // slot soon after its QK completed stalls the warp), and after every
        // read of the slot's S; then pass the reference on
        if (!kept0) tmem_st32_zero(colS);
        if (nb == 2 && !kept1) tmem_st32_zero(colS + 32);
        sm.xm[r] = m;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(hand);
          mbar_arrive(&sm.p_full[slot]);
        }
        ++hk;
      }
      if (!ok) break;
      // ---------------- end of the unit: row max and row sum of both groups ----------------
      const int bh = u / P.npairs, pair = u % P.npairs;
      float mrow = -INFINITY, lrow = 0.f;
      if (TT > 0) {
        const int last = static_cast<int>((gtile + TT - 1) & 1);  // group of the last tile
        if (grp != last) {
          // receive the last tile's reference, send this group's sum, receive the total
          ok = warp_wait<1>(hand, hk & 1, abort_flag, st, kSiteMlReady, u);
          ++hk;
          if (!ok) break;
          mrow = sm.xm[r];
          sm.xl[r] = (m == -INFINITY) ? 0.f : l * pow2_f32(m - mrow);
          __syncwarp();
          if (lane == 0) mbar_arrive(hand);
          ++hk;
          ok = warp_wait<1>(hand, hk & 1, abort_flag, st, kSiteMlReady, u);
          ++hk;
          if (!ok) break;
          lrow = sm.xl[r];
        } else {
          ok = warp_wait<1>(hand, hk & 1, abort_flag, st, kSiteMlReady, u);
          ++hk;
          if (!ok) break;
          mrow = m;
          lrow = l + sm.xl[r];
          sm.xl[r] = lrow;
          __syncwarp();
          if (lane == 0) mbar_arrive(hand);
          ++hk;
        }
        // the unit's last PV has completed
        const uint32_t gl = gtile + TT - 1;
        if (!warp_wait<1>(&sm.pv_done[gl % kSSlots], (gl / kSSlots) & 1, abort_flag, st, kSitePvDone, u)) break;
        tc_fence_after();
      }
      // ---------------- epilogue: O and l merged with the correction ----------------
      const float mc = sm.cmax[s][blk] * kLog2e;
      const float cd = sm.cden[s][blk];
      const float mfin = fmaxf(mrow, mc);
      const float wa = (mrow == -INFINITY) ? 0.f : ex2_approx(mrow - mfin);
      const float wc = (mc == -INFINITY) ? 0.f : ex2_approx(mc - mfin);
      const float L = fmaf(lrow, wa, cd * wc);
      const float inv = 1.f / L;
      const int row = pair * kBM + r;
      const bool valid = row < P.N;
      constexpr int DH = D / 2;  // output columns written by this group
      uint16_t* orow =
          P.out + (bh / P.H) * P.sb + (bh % P.H) * P.sh + static_cast<long long>(row) * P.sn + grp * DH;
#pragma unroll 1
      for (int ch = 0; ch < DH / 16; ++ch) {
        float y[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) y[x] = ROUTE ? sm.cnum[s][blk][grp * DH + ch * 16 + x] * wc : 0.f;
        if (TT > 0) {
          uint32_t o[16];
          tmem_ld16_wait(colO + grp * DH + ch * 16, o);
#pragma unroll
          for (int x = 0; x < 16; ++x) y[x] = fmaf(__uint_as_float(o[x]), wa, y[x]);
        }
        if (valid) {
          uint32_t pk[8];
#pragma unroll
          for (int x = 0; x < 8; ++x) pk[x] = pack_bf16x2(y[2 * x] * inv, y[2 * x + 1] * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 16);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      if (valid && P.lse && grp == 0) P.lse[static_cast<long long>(bh) * P.N + row] = (mfin + __log2f(L)) * kLn2;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.o_free[s]);
        mbar_arrive(&sm.route_empty[s]);
      }
      gtile += TT;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool ROUTE>
cudaError_t launch_pp_t(const ForwardArgs& a, int num_sms, cudaStream_t stream) {
  CUtensorMap tmQ, tmK, tmV;
  const int B = a.BH / a.H;
  if (!make_map(&tmQ, a.q, B, a.H, a.N, D, a.st, kBM) || !make_map(&tmK, a.k, B, a.H, a.N, D, a.st, kBN) ||
      !make_map(&tmV, a.v, B, a.H, a.N, D, a.st, kBN))
    return cudaErrorInvalidValue;
  Params p{};
  p.q = a.q;
  p.out = a.out;
  p.lse = a.lse;
  p.density = a.density;
  p.qbar = a.pooled.qbar;
  p.kbar = a.pooled.kbar;
  p.vbar = a.pooled.vbar;
  p.kmean = a.pooled.kmean;
  p.kcov = a.pooled.kcov;
  p.beta = a.beta;
  p.n_forced = a.n_forced;
  p.BH = a.BH;
  p.H = a.H;
  p.sb = a.st.b;
  p.sh = a.st.h;
  p.sn = a.st.n;
  p.N = a.N;
  p.NB = (a.N + kBN - 1) / kBN;
  p.npairs = (p.NB + 1) / 2;
  p.units = a.BH * p.npairs;
  p.status = static_cast<DeviceStatus*>(a.status);
  const size_t smem = sizeof(SmemPP<D>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(solattn_fwd_pp_kernel<D, ROUTE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = p.units < num_sms ? p.units : num_sms;
  solattn_fwd_pp_kernel<D, ROUTE><<<grid, kThreadsPP, smem, stream>>>(tmQ, tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace

#ifdef SOLATTN_TEST_HOOKS
cudaError_t set_test_hooks_pp(int skip_cta, unsigned long long wait_budget_ns) {
  cudaError_t e = cudaMemcpyToSymbol(g_hook_skip_cta, &skip_cta, sizeof(skip_cta));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_wait_budget_ns, &wait_budget_ns, sizeof(wait_budget_ns));
  return e;
}

cudaError_t set_route_dump_pp(uint32_t* mask, float* stats) { return set_route_dump_here(mask, stats); }
#endif

cudaError_t launch_forward_pp(const ForwardArgs& a, int num_sms, cudaStream_t stream) {
  if (a.d == 64) return a.route ? launch_pp_t<64, true>(a, num_sms, stream) : launch_pp_t<64, false>(a, num_sms, stream);
  return a.route ? launch_pp_t<128, true>(a, num_sms, stream) : launch_pp_t<128, false>(a, num_sms, stream);
}

}  // namespace solattn
