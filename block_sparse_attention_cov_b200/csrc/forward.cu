// forward.cu -- fused Sol-Attn forward for sm_100a (tcgen05 + TMEM + TMA).
//
// Method: "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly
// Attention Sparsification" (pages: hotpaper.ai abstract; paithon.it sections
// "Una soglia per ogni riga" and "Scegliere mentre si calcola"). For every
// query block i the proxy scores s_hat_ij = qbar_i . kbar_j / sqrt(d) are
// produced one key block at a time and compared with tau_i = mu_i + beta sigma_i
// on the fly; blocks above tau_i are attended exactly; the others are folded in
// through the zeroth-order Taylor term n_j e^{s_hat_ij} (vbar_j in the
// numerator), into the same online-softmax state. The proxy row never leaves
// the SM.
//
// Work unit: two adjacent 64-token query blocks (128 rows, the full-rate
// tcgen05 tile height) of one head. The key blocks of a unit are the union of
// the two blocks' kept sets, taken two at a time as 128-key tiles (any two
// kept blocks, not only neighbours); a block kept by only one of the two
// query blocks is still multiplied for all 128 rows, and the other block's
// rows mask it out (their P is zero and their softmax state is untouched), so
// each block's result is exactly its own.
//
// One persistent CTA per SM, 512 threads (roles at the kernel below). S = Q K^T
// runs with both operands in shared memory (Q tile 128 x d, K tile 128 x d:
// at N = 128 the operand traffic fits the shared-memory bandwidth), O += P V
// with P in TMEM (written over its own S) and V in shared memory. Three S
// slots let the QKs of the next two tiles run while the softmax works on one;
// eight softmax warps split every 128-key tile in two 64-key halves (two warps
// per row group, agreeing on the row max), so two warps share each SM
// sub-partition's exponential unit.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "fwd_common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace solattn {

namespace {

constexpr int kThreads = 512;  // 16 warps, 128 registers per thread

template <int D, bool SEL = false>
struct __align__(1024) Smem {
  // K ring: one stage per 128-key tile (two blocks stacked in every 64-column
  // panel, as one N = 128 operand); V ring: one stage per block. Sizes are
  // multiples of 1 KB, so every stage stays 1024-aligned for the swizzle.
  // (with a top-k / top-p rule the proxy rows of the unit are kept in shared
  // memory for the selection, and the K ring gives up a stage for them)
  static constexpr int kKStages = D == 128 ? (SEL ? 2 : 3) : 4;
  static constexpr int kVStages = D == 128 ? 4 : 8;
  uint8_t qt[kBM * D * 2];               // Q tile of the unit, SW128 K-major panels of 128 rows
  uint8_t kt[kKStages][kBM * D * 2];     // K tiles, same layout
  uint8_t vt[kVStages][kBN * D * 2];     // V blocks, SW128 panels of 64 rows
  // Per-token correction: one extra K = 16 step of each pooled tile's QK adds,
  // for the row's query block g, columns 2g and 2g + 1 of the bias tile to the
  // score: -1e30 on the key blocks g kept (and on pads), else ln(n_j) sqrt(d)
  // as a bf16 hi + lo pair. ebias is the constant 0/1 query-side operand. Both are
  // K-major without swizzle (core matrices 8 rows x 16 B; 128 B between the
  // two along K, 256 B between groups of 8 rows).
  uint8_t ebias[kBM * 32];
  uint8_t kbias[kBM * 32];
  float rchunk[2][kChunk][D];        // routing: pooled keys of a chunk, double-buffered
  float cnum[2][2][D];               // correction numerator per slot and block
  float cden[2][2];
  float cmax[2][2];                  // reference max of the correction (natural units)
  int unit[2];
  int count[2];
  float rq[2][D];                    // routing: qbar of the unit's two query blocks
  float rstat[4][4];                 // routing: per-warp partial mu / quadratic form sums
  float rscore[2][kChunk];           // proxy scores of the chunk being routed
  float rweight[2][kChunk];          // correction weights n_j e^{s_hat - M} (0 if kept)
  float rscale[2];                   // rescale of the running correction sums
  float rmax[2];                     // running max of the skipped proxy scores
  float rden[2];                     // running correction denominators
  int rkept[2];                      // running kept counts
  uint32_t bits[2][2][kNbMax / 32];  // kept bitmaps [slot][query block][word]: the unit's key list
  float score[SEL ? 2 : 1][SEL ? kNbMax : 1];  // top-k / top-p: the unit's two proxy rows
  uint32_t cut[2];                   // top-k / top-p: order key of each row's cut
  int keep_none[2];                  // top-k / top-p: the row keeps no block by its rule
  uint64_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
  // Per S slot: QK landed / P stored by all four softmax warps / PV of the
  // slot's tile completed. Per-slot barriers keep a warp that runs a tile
  // ahead from arriving on the phase of the tile its neighbours are still on.
  uint64_t s_full[3], p_full[3], pv_done[3];
  uint64_t o_free[2];                // per unit slot: the epilogue has read O
  uint64_t q_full, q_free;
  uint64_t route_full[2], route_empty[2];
  uint64_t rfull[2];                 // routing chunk buffers landed
  uint64_t mma_done[2];
  uint64_t b_free;                   // per-token correction: the bias tile was read by its QK
  // Key-list entries of the key tiles (both halves), published by the K
  // producer, which walks the list anyway, for the softmax warps: a ring of 8
  // tiles, one barrier per slot
  uint32_t kentry[8][2];
  uint64_t e_full[8];
  float xm[kBM][2];                  // softmax: row max of each key half (exchange)
  float xl[kBM][2];                  // softmax: row sum of each key half (epilogue)
  uint32_t tmem_base;
  int bcast;
  int abort_flag;
};

// Dynamic shared memory per CTA on sm_100 is at most 227 KB (232448 bytes);
// one extra KB pays for the 1024-byte alignment of the TMA tiles.
static_assert(sizeof(Smem<128>) + 1024 <= 232448, "shared memory layout too large");
static_assert(sizeof(Smem<64>) + 1024 <= 232448, "shared memory layout too large");
static_assert(sizeof(Smem<128, true>) + 1024 <= 232448, "shared memory layout too large");
static_assert(sizeof(Smem<64, true>) + 1024 <= 232448, "shared memory layout too large");

// Tiles of a unit: TT of kept blocks (two per tile) and, with the per-token
// correction, TP of pooled keys (128 per tile, every key block of the head;
// columns are masked per query block to the blocks it skipped). V blocks: T
// kept ones, then the 64-key chunks of the pooled values.
struct UnitTiles {
  int T, TT, TP, VB;
  __device__ __forceinline__ UnitTiles(int T_, int NB, bool token)
      : T(T_), TT((T_ + 1) / 2), TP(token ? (NB + 127) / 128 : 0), VB(T_ + (token ? (NB + 63) / 64 : 0)) {}
  __device__ __forceinline__ int total() const { return TT + TP; }
  // key blocks (64-key halves) in tile t
  __device__ __forceinline__ int halves(int t, int NB) const {
    return t < TT ? ((2 * t + 1 < T) ? 2 : 1) : ((128 * (t - TT) + 64 < NB) ? 2 : 1);
  }
  // index of half h of tile t among the unit's V blocks
  __device__ __forceinline__ int vblock(int t, int h) const { return t < TT ? 2 * t + h : T + 2 * (t - TT) + h; }
};

// ---------------------------------------------------------------------------
// The kernel. 512 threads = 16 warps:
//   warps 0-7   softmax: warp w covers rows 32 (w % 4) .. + 31 of the unit
//               (TMEM lanes) and key block w / 4 of every 128-key tile; the
//               two warps of a row group agree on the row max through a
//               pairwise barrier. At the end of the unit, once its last PV has
//               completed, the epilogue (O and the row sum merged with the
//               skipped-block correction, out and lse written)
//   warps 8-11  routing, one unit ahead; then the unit's Q tile by TMA once
//               every QK of the previous unit has completed
//   warp 12     TMA producer of the K tiles (two kept blocks per stage)
//   warp 13     MMA issuer for QK (one elected lane), up to two tiles ahead
//   warp 14     TMA producer of the V blocks
//   warp 15     MMA issuer for PV
// TMEM: three S slots of 128 fp32 columns at 0 / 128 / 256 (the bf16 P of a
// tile is written over the first 64 columns of its own S) and O at 384. The
// QKs of the next two tiles are in flight while the softmax works on one.
// ---------------------------------------------------------------------------
template <int D, bool ROUTE, int RULE, bool TOKEN>
__global__ void __launch_bounds__(kThreads, 1)
    solattn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmKb,
                       const __grid_constant__ CUtensorMap tmVb, const Params P) {
  using SmemT = Smem<D, RULE != 0>;
  constexpr int KS = SmemT::kKStages, VS = SmemT::kVStages;
  constexpr uint32_t kColO = 3 * 128;
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
    for (int i = 0; i < 3; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_full[i], 8);
      mbar_init(&sm.pv_done[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.route_full[i], 1);
      mbar_init(&sm.route_empty[i], 12);  // 2 producers + 2 MMA issuers + 8 softmax warps
      mbar_init(&sm.rfull[i], 1);
    }
    mbar_init(&sm.o_free[0], 8);
    mbar_init(&sm.o_free[1], 8);
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_free, 1);
    mbar_init(&sm.mma_done[0], 1);
    mbar_init(&sm.mma_done[1], 1);
    mbar_init(&sm.b_free, 1);
    for (int i = 0; i < 8; ++i) mbar_init(&sm.e_full[i], 1);
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
    if (TOKEN) {
      prefetch_tensormap(&tmKb);
      prefetch_tensormap(&tmVb);
    }
  }
  if constexpr (TOKEN) {
    if (warp == 12) {
      // the constant query-side operand: row r of query block g = r / 64 has
      // ones in columns 2g, 2g + 1; columns 8-15 of both tiles stay zero
      for (int i = 0; i < 4; ++i) {
        const int r = lane * 4 + i;
        constexpr uint32_t kOnes = 0x3F803F80u;  // two bf16 ones
        uint8_t* e = &sm.ebias[(r >> 3) * 256 + (r & 7) * 16];
        *reinterpret_cast<uint4*>(e) = r < 64 ? make_uint4(kOnes, 0u, 0u, 0u) : make_uint4(0u, kOnes, 0u, 0u);
        *reinterpret_cast<uint4*>(e + 128) = make_uint4(0u, 0u, 0u, 0u);
        *reinterpret_cast<uint4*>(&sm.kbias[(r >> 3) * 256 + 128 + (r & 7) * 16]) = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp >= 8 && warp < 12) {
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
        if (!route_unit<D, RULE>(sm, P, s, bh, pair, rt, chunk_ctr, abort_flag, st, u)) break;
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
    // ======================= TMA producers: warp 12 = K tiles, warp 14 = V blocks =======================
    const bool isK = warp == 12;
    uint32_t g = 0;   // K: global tile index; V: global block index
    uint32_t gk = 0;  // K: key tiles published (entry ring position)
    uint32_t nbias = 0, wfull = 0, wlast = 0, wmask = 0;  // per-token correction: bias tiles written, entries
    if constexpr (TOKEN) {
      // a pooled key stands for the n_j keys of its block: ln(n_j) sqrt(d) in raw score units
      const float sd = sqrtf(static_cast<float>(D));
      wfull = bias_pair(logf(static_cast<float>(kBN)) * sd);
      wlast = bias_pair(logf(static_cast<float>(P.N - (P.NB - 1) * kBN)) * sd);
      wmask = pack_bf16x2(-1e30f, 0.f);
    }
    for (int n = 0;; ++n) {
      const int s = n & 1;
      if (!warp_wait(&sm.route_full[s], (n >> 1) & 1, abort_flag, st, kSiteRouteFullProd, 0)) break;
      const int u = sm.unit[s];
      if (u < 0) break;
      const int T = sm.count[s];
      const int bh = u / P.npairs;
      bool ok = true;
      KeyWalk<ROUTE> walk(sm.bits[s][0], sm.bits[s][1]);
      const UnitTiles ut(T, P.NB, TOKEN);
      if (isK) {
        const int TT = ut.total();
        int t = 0;
        for (; t < TT; ++t) {
          const uint32_t gt = g + t, stg = gt % KS, r = gt / KS;
          if (r >= 1 && !warp_wait(&sm.k_empty[stg], (r - 1) & 1, abort_flag, st, kSiteKEmpty, u)) break;
          const int nb = ut.halves(t, P.NB);
          const bool pooled = TOKEN && t >= ut.TT;  // a tile of pooled keys (per-token correction)
          int jj[2];
          if (!pooled) {
            const uint32_t e0 = walk.next(), e1 = nb == 2 ? walk.next() : 0u;
            jj[0] = e0 & 0x3FFF;
            jj[1] = e1 & 0x3FFF;
            // Publish the tile's entries for the softmax warps. Slot reuse is
            // safe: this tile's stage was released by QK(t - KS), so the softmax
            // has finished tile t - KS - 3 and is past every older slot user.
            const uint32_t ek = gk++;
            if (elect_one()) {
              sm.kentry[ek & 7][0] = e0;
              sm.kentry[ek & 7][1] = e1;
              mbar_arrive(&sm.e_full[ek & 7]);
            }
            __syncwarp();
          } else {
            jj[0] = 2 * (t - ut.TT);
            jj[1] = jj[0] + 1;
          }
          if constexpr (TOKEN) {
            if (pooled) {
              // the previous pooled tile's QK has read the bias tile
              if (nbias >= 1 && !warp_wait(&sm.b_free, (nbias - 1) & 1, abort_flag, st, kSiteBFree, u)) break;
              ++nbias;
              const int jb = jj[0] * kBN;  // first pooled key of the tile
              for (int i = 0; i < 4; ++i) {
                const int r = lane * 4 + i, j = jb + r;
                uint32_t w0 = wmask, w1 = wmask;
                if (j < P.NB) {
                  const uint32_t w = j == P.NB - 1 ? wlast : wfull;
                  if (!((sm.bits[s][0][j >> 5] >> (j & 31)) & 1u)) w0 = w;
                  if (!((sm.bits[s][1][j >> 5] >> (j & 31)) & 1u)) w1 = w;
                }
                *reinterpret_cast<uint4*>(&sm.kbias[(r >> 3) * 256 + (r & 7) * 16]) = make_uint4(w0, w1, 0u, 0u);
              }
              fence_proxy_async_smem();
              __syncwarp();
            }
          }
#ifdef SOLATTN_TEST_HOOKS
          if (gt == 0 && static_cast<int>(blockIdx.x) == g_hook_skip_cta) continue;  // this tile never arrives
#endif
          if (elect_one()) {
            mbar_arrive_expect_tx(&sm.k_full[stg], nb * kBN * D * 2);
            for (int h = 0; h < nb; ++h) {
#pragma unroll
              for (int pnl = 0; pnl < D / 64; ++pnl) {
                void* dst = &sm.kt[stg][pnl * kBM * 128 + h * kBN * 128];
                if (!pooled)
                  tma_load_4d(dst, &tmK, &sm.k_full[stg], pnl * 64, jj[h] * kBN, bh % P.H, bh / P.H);
                else  // rows 64 jj[h] .. of the head's bf16 pooled keys
                  tma_load_4d(dst, &tmKb, &sm.k_full[stg], pnl * 64, jj[h] * kBN, 0, bh);
              }
            }
          }
          __syncwarp();
        }
        g += t;
        ok = t == TT;
      } else {
        int t = 0;
        for (; t < ut.VB; ++t) {
          const bool pooled = TOKEN && t >= T;
          const int j = pooled ? t - T : (walk.next() & 0x3FFF);
          const uint32_t gt = g + t, stg = gt % VS, r = gt / VS;
          if (r >= 1 && !warp_wait(&sm.v_empty[stg], (r - 1) & 1, abort_flag, st, kSiteVEmpty, u)) break;
          if (elect_one()) {
            mbar_arrive_expect_tx(&sm.v_full[stg], kBN * D * 2);
#pragma unroll
            for (int pnl = 0; pnl < D / 64; ++pnl) {
              void* dst = &sm.vt[stg][pnl * kBN * 128];
              if (!pooled)
                tma_load_4d(dst, &tmV, &sm.v_full[stg], pnl * 64, j * kBN, bh % P.H, bh / P.H);
              else
                tma_load_4d(dst, &tmVb, &sm.v_full[stg], pnl * 64, j * kBN, 0, bh);
            }
          }
          __syncwarp();
        }
        g += t;
        ok = t == ut.VB;
      }
      if (!ok) break;  // aborted
      if (elect_one()) mbar_arrive(&sm.route_empty[s]);
      __syncwarp();
    }
    if (lane == 0) {  // teardown: every issued copy lands before the CTA exits
      const uint32_t depth = isK ? KS : VS;
      const uint32_t first = g > depth ? g - depth : 0u;
      for (uint32_t gt = first; gt < g; ++gt) {
        if (isK) mbar_wait_quiet(&sm.k_full[gt % KS], (gt / KS) & 1);
        else mbar_wait_quiet(&sm.v_full[gt % VS], (gt / VS) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 13 || warp == 15) {
    // ======================= MMA issuers: warp 13 = QK, warp 15 = PV =======================
    // QK(t) goes into S slot t % 3 as soon as its K tile has landed and the
    // PV that last read P from that slot (tile t - 3) has completed: QK and PV
    // come from different issuer threads, whose MMAs are not ordered with each
    // other, so the slot is reused only after pv_done (waited once per tile, in
    // order). The S ring
    // therefore runs up to two tiles ahead of the softmax. PV(t) goes as soon
    // as all eight softmax warps have stored P(t) and its V blocks have landed.
    const bool isQK = warp == 13;
    constexpr uint32_t idesc_qk2 = idesc_bf16_f32(kBM, 2 * kBN, false, false);
    constexpr uint32_t idesc_qk1 = idesc_bf16_f32(kBM, kBN, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
    const uint64_t qdesc = sw128_desc(smem_u32(&sm.qt[0]), 16, 1024);
    const uint64_t kdesc0 = sw128_desc(smem_u32(&sm.kt[0][0]), 16, 1024);
    const uint64_t vdesc0 = sw128_desc(smem_u32(&sm.vt[0][0]), 8192, 1024);
    const uint64_t edesc = nosw_desc(smem_u32(&sm.ebias[0]), 128, 256);
    const uint64_t bdesc = nosw_desc(smem_u32(&sm.kbias[0]), 128, 256);
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
      const UnitTiles ut(T, P.NB, TOKEN);
      const int TT = ut.total();
      if (isQK) {
        if (!warp_wait(&sm.q_full, n & 1, abort_flag, st, kSiteQFull, u)) break;
        if (TT == 0) {  // nothing to multiply: release the Q tile
          if (elect_one()) mma_commit(&sm.q_free);
          __syncwarp();
        }
        for (int t = 0; t < TT && ok; ++t) {
          const uint32_t gt = gtile + t, stg = gt % KS, slot = gt % 3;
          for (; pv_waited + 3 <= gt && ok; ++pv_waited)
            ok = warp_wait(&sm.pv_done[pv_waited % 3], (pv_waited / 3) & 1, abort_flag, st, kSitePvDone, u);
          if (ok) ok = warp_wait(&sm.k_full[stg], (gt / KS) & 1, abort_flag, st, kSiteKFull, u);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            const uint64_t kd = kdesc0 + ((stg * (kBM * D * 2)) >> 4);
            const uint32_t idesc = ut.halves(t, P.NB) == 2 ? idesc_qk2 : idesc_qk1;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (((kk / 4) * kBM * 128) + (kk % 4) * 32) >> 4;
              mma_ss(tmem + slot * 128, qdesc + off, kd + off, idesc, kk > 0 ? 1u : 0u);
            }
            const bool pooled = TOKEN && t >= ut.TT;
            if (pooled) mma_ss(tmem + slot * 128, edesc, bdesc, idesc, 1u);  // + the tile's mask and weights
            mma_commit(&sm.s_full[slot]);
            mma_commit(&sm.k_empty[stg]);
            if (pooled) mma_commit(&sm.b_free);
            if (t == TT - 1) mma_commit(&sm.q_free);
          }
          __syncwarp();
        }
      } else {
        // O is free once the epilogue has read the previous unit's
        if (n >= 1 && !warp_wait(&sm.o_free[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag, st, kSiteOFree, u)) break;
        for (int t = 0; t < TT && ok; ++t) {
          const uint32_t gt = gtile + t;
          const int nb = ut.halves(t, P.NB);
          // V first: it has normally landed long before P, so once P is
          // stored only the issue remains
          uint32_t stv[2];
          for (int h = 0; h < nb && ok; ++h) {
            const uint32_t gv = gblk + ut.vblock(t, h);
            stv[h] = gv % VS;
            ok = warp_wait(&sm.v_full[stv[h]], (gv / VS) & 1, abort_flag, st, kSiteVFull, u);
          }
          if (ok) ok = warp_wait(&sm.p_full[gt % 3], (gt / 3) & 1, abort_flag, st, kSitePFull, u);
          if (!ok) break;
          tc_fence_after();
          if (elect_one()) {
            const uint32_t colP = tmem + (gt % 3) * 128;
            for (int h = 0; h < nb; ++h) {
              const uint64_t vd = vdesc0 + ((stv[h] * (kBN * D * 2)) >> 4);
#pragma unroll
              for (int kk = 0; kk < kBN / 16; ++kk)
                mma_ts(colO, colP + h * 32 + kk * 8, vd + ((kk * 2048) >> 4), idesc_pv,
                       (t > 0 || h > 0 || kk > 0) ? 1u : 0u);
              mma_commit(&sm.v_empty[stv[h]]);
            }
            mma_commit(&sm.pv_done[gt % 3]);
          }
          __syncwarp();
        }
      }
      if (!ok) break;
      if (elect_one()) mma_commit(&sm.route_empty[s]);
      __syncwarp();
      gtile += TT;
      gblk += ut.VB;
    }
    const int me = isQK ? 0 : 1;
    if (elect_one()) mma_commit(&sm.mma_done[me]);  // teardown: issued MMAs complete before TMEM is freed
    __syncwarp();
    mbar_wait_quiet(&sm.mma_done[me], 0);
    __syncwarp();
  } else if (warp < 8) {
    // ======================= softmax =======================
    const int q4 = warp & 3, hh = warp >> 2;  // row group, key half of the tile
    const int r = q4 * 32 + lane;             // row of the unit == TMEM lane
    const int blk = r >> 6;                   // which of the two query blocks (warp-uniform)
    const int pb = 2 + q4;                    // named barrier of warps q4 and q4 + 4 (same rows)
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const float sl2 = kLog2e * rsqrtf(static_cast<float>(D));
    const int nlast = P.N - (P.NB - 1) * kBN;
    constexpr int DH = D / 2;                 // O / output columns owned by this warp
    const uint32_t colO = tmem + kColO + lane_off + hh * DH;
    uint32_t gtile = 0, gkey = 0;  // tiles / key tiles consumed so far
    for (int n = 0;; ++n) {
      const int s = n & 1;
      bool okr = warp_wait(&sm.route_full[s], (n >> 1) & 1, abort_flag, st, kSiteRouteFullSoft, 0);
      if (named_bar_or(pb, 64, !okr)) break;
      tc_fence_after();
      const int u = sm.unit[s];
      if (u < 0) break;
      const int T = sm.count[s];
      const UnitTiles ut(T, P.NB, TOKEN);
      const int TT = ut.total();
      float m = -INFINITY, l = 0.f;  // m: the row's shared reference max; l: this half's sum
      bool ok = true;
      for (int t = 0; t < TT; ++t) {
        const uint32_t gt = gtile + t, slot = gt % 3;
        const uint32_t colS = tmem + slot * 128 + lane_off;
        const int nb = ut.halves(t, P.NB);
        const bool pooled = TOKEN && t >= ut.TT;
        bool kept;
        int nv = kBN;
        bool oke = true;
        if (!pooled) {
          // this half's key-list entry, published by the K producer
          const uint32_t ek = gkey++;
          oke = warp_wait(&sm.e_full[ek & 7], (ek >> 3) & 1, abort_flag, st, kSiteEFull, u);
          const uint32_t entry = hh < nb ? sm.kentry[ek & 7][hh] : 0u;
          kept = (entry >> (14 + blk)) & 1u;
          nv = ((entry & 0x3FFF) == static_cast<uint32_t>(P.NB - 1)) ? nlast : kBN;
        } else {
          // pooled keys: the half counts while one of its columns is a block the
          // row's query block skipped (the QK's bias step put -1e30 on the rest)
          const int j0 = 128 * (t - ut.TT) + 64 * hh;  // first pooled key of this half
          kept = false;
          if (hh < nb) {
            const int valid = P.NB - j0;  // > 0
            const uint32_t u0 = ~sm.bits[s][blk][j0 >> 5] & (valid >= 32 ? ~0u : ((1u << valid) - 1u));
            const uint32_t u1 = valid <= 32 ? 0u
                                            : ~sm.bits[s][blk][(j0 >> 5) + 1] &
                                                  (valid >= 64 ? ~0u : ((1u << (valid - 32)) - 1u));
            kept = (u0 | u1) != 0u;
          }
        }
        const bool okw = oke && warp_wait(&sm.s_full[slot], (gt / 3) & 1, abort_flag, st, kSiteSFull, u);
        tc_fence_after();
        uint32_t sv[64];
        if (kept && okw) tmem_ld32x2_wait(colS + 64 * hh, colS + 64 * hh + 32, sv);
        const float mx = (kept && okw) ? tile_max(sv, nv) * sl2 : -INFINITY;
        // Does a row of this group need a new reference max (or did a wait fail)?
        // The barrier also orders this group's S reads before the other half's
        // P stores into the same columns.
        tc_fence_before();
        const bool any = named_bar_or(pb, 64, !okw || mx > m + kRescaleSlack);
        tc_fence_after();
        if (any) {
          sm.xm[r][hh] = okw ? mx : NAN;
          named_bar_sync(pb, 64);
          const float mo = sm.xm[r][hh ^ 1];
          if (__any_sync(0xffffffffu, !okw || mo != mo)) { ok = false; break; }  // identical in both warps
          const float mrow = fmaxf(mx, mo);
          float rescale = 1.f;
          bool need = false;
          if (mrow > m + kRescaleSlack) {
            need = m != -INFINITY;
            if (need) rescale = ex2_approx(m - mrow);
            m = mrow;
          }
          if (__any_sync(0xffffffffu, need)) {
            // O must hold every PV up to the previous tile before it is rescaled
            const uint32_t gp = gt - 1;
            const bool okp = warp_wait(&sm.pv_done[gp % 3], (gp / 3) & 1, abort_flag, st, kSitePvDone, u);
            if (named_bar_or(pb, 64, !okp)) { ok = false; break; }
            tc_fence_after();
            l *= rescale;
#pragma unroll 1
            for (int ch = 0; ch < DH / 16; ++ch) {
              uint32_t ov[16];
              tmem_ld16_wait(colO + ch * 16, ov);
#pragma unroll
              for (int c = 0; c < 16; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * rescale);
              tmem_st16_wait(colO + ch * 16, ov);
            }
          }
        }
        // ---- P = 2^(S sl2 - m) in bf16 for this key half, over S's first 64 columns
        if (hh < nb) {
          uint32_t pw[32];
          if (kept) {
            const uint64_t sc2 = f2_dup(sl2);
            const uint64_t nm2 = f2_dup(-m);
            uint64_t lsum = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q)
              softmax_slice(&sv[16 * q], sc2, nm2, lsum, *reinterpret_cast<uint32_t(*)[8]>(&pw[8 * q]));
            float l0, l1;
            f2_split(lsum, l0, l1);
            l += l0 + l1;
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) pw[c] = 0u;
          }
          tmem_st32_wait(colS + 32 * hh, pw);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[slot]);
      }
      if (!ok) break;
      // ---------------- epilogue: O and l merged with the correction ----------------
      const int bh = u / P.npairs, pair = u % P.npairs;
      const bool hasO = TT > 0;
      bool oke = true;
      if (hasO) {  // the unit's last PV has completed
        const uint32_t gl = gtile + TT - 1;
        oke = warp_wait(&sm.pv_done[gl % 3], (gl / 3) & 1, abort_flag, st, kSitePvDone, u);
      }
      sm.xl[r][hh] = l;
      if (named_bar_or(pb, 64, !oke)) break;
      tc_fence_after();
      const float lrow = sm.xl[r][0] + sm.xl[r][1];
      named_bar_sync(pb, 64);  // both halves have read xl
      // (with the per-token correction the skipped blocks came in as pooled tiles)
      const float mc = TOKEN ? -INFINITY : sm.cmax[s][blk] * kLog2e;
      const float cd = sm.cden[s][blk];
      const float mf = fmaxf(m, mc);
      const float wa = (m == -INFINITY) ? 0.f : ex2_approx(m - mf);
      const float wc = (mc == -INFINITY) ? 0.f : ex2_approx(mc - mf);
      const float L = fmaf(lrow, wa, cd * wc);
      const float inv = 1.f / L;
      const int row = pair * kBM + r;
      const bool valid = row < P.N;
      uint16_t* orow = P.out + (bh / P.H) * P.sb + (bh % P.H) * P.sh + static_cast<long long>(row) * P.sn + hh * DH;
#pragma unroll 1
      for (int ch = 0; ch < DH / 16; ++ch) {
        float y[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) y[e] = 0.f;
        if constexpr (ROUTE) {
#pragma unroll
          for (int e = 0; e < 16; ++e) y[e] = sm.cnum[s][blk][hh * DH + ch * 16 + e] * wc;
        }
        if (hasO) {
          uint32_t o[16];
          tmem_ld16_wait(colO + ch * 16, o);
#pragma unroll
          for (int e = 0; e < 16; ++e) y[e] = fmaf(__uint_as_float(o[e]), wa, y[e]);
        }
        if (valid) {
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) pk[e] = pack_bf16x2(y[2 * e] * inv, y[2 * e + 1] * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 16);
          dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
      if (valid && P.lse && hh == 0) P.lse[static_cast<long long>(bh) * P.N + row] = (mf + __log2f(L)) * kLn2;
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

template <int D, bool ROUTE, int RULE, bool TOKEN>
cudaError_t launch_fwd_t(const ForwardArgs& a, int num_sms, cudaStream_t stream) {
  CUtensorMap tmQ, tmK, tmV;
  const int B = a.BH / a.H;
  if (!make_map(&tmQ, a.q, B, a.H, a.N, D, a.st, kBM) || !make_map(&tmK, a.k, B, a.H, a.N, D, a.st, kBN) ||
      !make_map(&tmV, a.v, B, a.H, a.N, D, a.st, kBN))
    return cudaErrorInvalidValue;
  // bf16 pooled keys / values of every head, [BH][N_b][D], for the per-token correction
  CUtensorMap tmKb = tmK, tmVb = tmV;
  if (TOKEN) {
    const int NB = (a.N + kBN - 1) / kBN;
    const Strides ps{static_cast<long long>(NB) * D, static_cast<long long>(NB) * D, D};
    if (!make_map(&tmKb, a.pooled.kbar16, a.BH, 1, NB, D, ps, kBN) ||
        !make_map(&tmVb, a.pooled.vbar16, a.BH, 1, NB, D, ps, kBN))
      return cudaErrorInvalidValue;
  }
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
  p.topk = a.topk;
  p.topp = a.topp;
  p.n_forced = a.n_forced;
  p.token_corr = a.token_corr;
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
  const size_t smem = sizeof(Smem<D, RULE != 0>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(solattn_fwd_kernel<D, ROUTE, RULE, TOKEN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = p.units < num_sms ? p.units : num_sms;
  solattn_fwd_kernel<D, ROUTE, RULE, TOKEN><<<grid, kThreads, smem, stream>>>(tmQ, tmK, tmV, tmKb, tmVb, p);
  return cudaGetLastError();
}

}  // namespace

#ifdef SOLATTN_TEST_HOOKS
// Test builds only (this translation unit's copies of the hook variables).
cudaError_t set_test_hooks_fwd(int skip_cta, unsigned long long wait_budget_ns) {
  cudaError_t e = cudaMemcpyToSymbol(g_hook_skip_cta, &skip_cta, sizeof(skip_cta));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_wait_budget_ns, &wait_budget_ns, sizeof(wait_budget_ns));
  return e;
}

cudaError_t set_route_dump_fwd(uint32_t* mask, float* stats) { return set_route_dump_here(mask, stats); }
#endif


template <int D, bool ROUTE, int RULE>
cudaError_t launch_fwd_c(const ForwardArgs& a, int num_sms, cudaStream_t stream) {
  if constexpr (ROUTE) {
    if (a.token_corr) return launch_fwd_t<D, ROUTE, RULE, true>(a, num_sms, stream);
  }
  return launch_fwd_t<D, ROUTE, RULE, false>(a, num_sms, stream);
}

cudaError_t launch_forward(const ForwardArgs& a, int num_sms, cudaStream_t stream) {
  if (a.d == 64) {
    if (!a.route) return launch_fwd_c<64, false, 0>(a, num_sms, stream);
    if (a.rule == 1) return launch_fwd_c<64, true, 1>(a, num_sms, stream);
    if (a.rule == 2) return launch_fwd_c<64, true, 2>(a, num_sms, stream);
    return launch_fwd_c<64, true, 0>(a, num_sms, stream);
  }
  if (!a.route) return launch_fwd_c<128, false, 0>(a, num_sms, stream);
  if (a.rule == 1) return launch_fwd_c<128, true, 1>(a, num_sms, stream);
  if (a.rule == 2) return launch_fwd_c<128, true, 2>(a, num_sms, stream);
  return launch_fwd_c<128, true, 0>(a, num_sms, stream);
}

}  // namespace solattn
