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

#include "kernels.h"
#include "ptx.cuh"

namespace solattn {

#ifdef SOLATTN_TRACE
// Debug builds only: per-tile timestamps of CTA 0 (clock64), [event][index].
__device__ unsigned long long g_trace[40][4096];
#define SOLATTN_TRACE_EVENT(ev, idx)                                         \
  do {                                                                       \
    if (blockIdx.x == 0 && (idx) < 4096) g_trace[(ev)][(idx)] = clock64();   \
  } while (0)
#define SOLATTN_TRACE_VALUE(ev, idx, val)                                    \
  do {                                                                       \
    if (blockIdx.x == 0 && (idx) < 4096) g_trace[(ev)][(idx)] = (val);       \
  } while (0)
#else
#define SOLATTN_TRACE_EVENT(ev, idx) \
  do {                               \
  } while (0)
#define SOLATTN_TRACE_VALUE(ev, idx, val) \
  do {                                    \
  } while (0)
#endif

namespace {

constexpr int kBM = 128;      // rows per unit
constexpr int kBN = 64;       // keys per block (a tile holds two)
constexpr int kNbMax = 4096;  // key blocks per head supported
constexpr int kThreads = 512;  // 16 warps, 128 registers per thread
constexpr int kChunk = 16;    // pooled key blocks per routing chunk (4 per routing warp)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleSlack = 8.0f;  // log2 units a row max may grow before O is rescaled

// Wait-site ids reported in the status word when a bounded wait gives up.
enum : uint32_t {
  kSiteRouteEmpty = 1,
  kSiteRouteFullProd,
  kSiteKEmpty,
  kSiteVEmpty,
  kSiteMmaStall,
  kSiteRouteFullMma,
  kSiteKFull,
  kSiteSFree,
  kSiteOFree,
  kSitePFull,
  kSiteVFull,
  kSiteRouteFullSoft,
  kSiteSFull,
  kSiteOFull,
  kSiteRouteChunk,
  kSiteQFree,
  kSiteBFree,
  kSiteQFull,
  kSiteMlReady,
  kSitePvDone,
  kSiteEFull,
};

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

struct Params {
  const uint16_t* q;
  uint16_t* out;
  float* lse;
  int32_t* density;
  const float* qbar;
  const float* kbar;
  const float* vbar;
  const float* kmean;
  const float* kcov;
  float beta;
  int topk;         // top-k rule
  float topp;       // top-p rule
  int n_forced;     // leading key blocks always kept
  int token_corr;   // 1: skipped blocks attended per token as tiles of pooled keys
  long long sb, sh, sn;  // element strides of q, k, v and out (batch, head, token)
  int BH, H, N, NB, npairs, units;
  DeviceStatus* status;
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          DeviceStatus* st, uint32_t site, uint32_t unit) {
  const bool ok = mbar_wait(bar, parity, abort_flag, st, site, unit);
  return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------------------
// Routing (warps 8-11, 128 threads): the pooled keys of the head are streamed
// through shared memory in chunks of 16 key blocks (bulk async copies,
// double-buffered); the pooled values go from L2 to registers. Per chunk:
// every warp scores 4 key blocks against both query blocks of the unit (one
// float4 column slice per lane, transposed butterfly reduction), the rule sets
// the kept bits, and the skipped blocks' weights n_j e^{s_hat - M} are folded
// into per-column correction sums (one column per thread); no proxy map in HBM.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Helpers of the routing warps and of the top-k / top-p cut.
// Order-preserving map of a float to an unsigned key (x < y <=> key(x) < key(y)).
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// RULE 0: per-row threshold tau_i = mu_i + beta sigma_i, decided chunk by chunk
// as the scores are produced. RULE 1 / 2 (top-k / top-p): a first pass stores
// the unit's two proxy rows, a bisection on the order keys finds each row's cut,
// and a second pass decides and folds. False if a bounded wait gave up.
template <int D, int RULE>
__device__ bool route_unit(Smem<D, RULE != 0>& sm, const Params& P, int s, int bh, int pair, int rt, uint32_t& chunk_ctr,
                           volatile int* abort_flag, DeviceStatus* st, int u) {
  constexpr int VPL = D / 32;  // columns per lane in the scoring layout
  const int rw = rt / 32, lane = rt % 32;
  const int NB = P.NB;
  const int i0 = 2 * pair, i1 = 2 * pair + 1;
  const bool has1 = i1 < NB;
  const int nchunks = (NB + kChunk - 1) / kChunk;
  const float* kb = P.kbar + static_cast<long long>(bh) * NB * D;
  const float* vb = P.vbar + static_cast<long long>(bh) * NB * D;
  auto issue = [&](int c) {
    const int j0 = c * kChunk;
    const int nk = min(kChunk, NB - j0);
    const uint32_t buf = (chunk_ctr + c) & 1;
    const uint32_t bytes = static_cast<uint32_t>(nk) * D * 4;
    mbar_arrive_expect_tx(&sm.rfull[buf], bytes);
    bulk_copy_g2s(&sm.rchunk[buf][0][0], kb + static_cast<long long>(j0) * D, bytes, &sm.rfull[buf]);
  };
  if (rt == 0) issue(0);
  // pooled values: this thread's column of the chunk's blocks, loaded into
  // registers at the start of the chunk (D = 128: column rt; D = 64: rt % 64)
  const int vcol = rt % D;

  const float* qb = P.qbar + static_cast<long long>(bh) * NB * D;
  float q0[VPL], q1[VPL];
#pragma unroll
  for (int e = 0; e < VPL; ++e) {
    q0[e] = qb[static_cast<long long>(i0) * D + lane * VPL + e];
    q1[e] = has1 ? qb[static_cast<long long>(i1) * D + lane * VPL + e] : 0.f;
  }
  const float beta = P.beta;
  const float scale = rsqrtf(static_cast<float>(D));
  // tau_i = mu_i + beta sigma_i with mu_i = s qbar_i . kmean and
  // sigma_i = s sqrt(qbar_i^T C qbar_i), from the head's key mean and covariance
  // (the proxy row itself is never formed). sigma_i = 0 means a constant proxy
  // row (every score equals mu_i = tau_i): nothing is strictly above it, so no
  // block is kept, whatever rounding does to the individual scores.
  float tau0 = beta, tau1 = has1 ? beta : INFINITY;
  if (RULE == 0 && beta != -INFINITY && beta != INFINITY) {
    // D = 128: thread rt owns column rt of both blocks; D = 64: column rt % 64
    // of block rt / 64. y_b[c] = sum_r C[r][c] qbar_b[r] (C is symmetric).
    const int col = rt % D, b1 = rt / D;
    const float* C = P.kcov + static_cast<long long>(bh) * D * D;
    if constexpr (D == 128) {
      sm.rq[0][rt] = qb[static_cast<long long>(i0) * D + rt];
      sm.rq[1][rt] = has1 ? qb[static_cast<long long>(i1) * D + rt] : 0.f;
    } else {
      sm.rq[rt / 64][col] = (rt < 64 || has1) ? qb[static_cast<long long>(i0 + rt / 64) * D + col] : 0.f;
    }
    named_bar_sync(1, 128);
    float y0 = 0.f, y1 = 0.f;
#pragma unroll 16
    for (int r = 0; r < D; ++r) {
      const float c = __ldg(C + r * D + col);
      if constexpr (D == 128) {
        y0 = fmaf(sm.rq[0][r], c, y0);
        y1 = fmaf(sm.rq[1][r], c, y1);
      } else {
        y0 = fmaf(sm.rq[b1][r], c, y0);
      }
    }
    const float km = __ldg(P.kmean + static_cast<long long>(bh) * D + col);
    float part[4];  // mu_0, quad_0, mu_1, quad_1 (partial over this thread's column)
    if constexpr (D == 128) {
      part[0] = sm.rq[0][col] * km;
      part[1] = sm.rq[0][col] * y0;
      part[2] = sm.rq[1][col] * km;
      part[3] = sm.rq[1][col] * y1;
    } else {
      const float m = sm.rq[b1][col] * km, qd = sm.rq[b1][col] * y0;
      part[0] = b1 == 0 ? m : 0.f;
      part[1] = b1 == 0 ? qd : 0.f;
      part[2] = b1 == 1 ? m : 0.f;
      part[3] = b1 == 1 ? qd : 0.f;
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) {
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) part[x] += __shfl_xor_sync(0xffffffffu, part[x], off);
    }
    if (lane == 0) {
#pragma unroll
      for (int x = 0; x < 4; ++x) sm.rstat[rw][x] = part[x];
    }
    named_bar_sync(1, 128);
    float tot[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) tot[x] = (sm.rstat[0][x] + sm.rstat[1][x]) + (sm.rstat[2][x] + sm.rstat[3][x]);
    const float sg0 = scale * sqrtf(fmaxf(tot[1], 0.f)), sg1 = scale * sqrtf(fmaxf(tot[3], 0.f));
    tau0 = sg0 == 0.f ? INFINITY : scale * tot[0] + beta * sg0;
    tau1 = (!has1 || sg1 == 0.f) ? INFINITY : scale * tot[2] + beta * sg1;
  }
  const int nlast = P.N - (NB - 1) * kBN;
  if (rt < 2) {
    sm.rmax[rt] = -INFINITY;
    sm.rden[rt] = 0.f;
    sm.rkept[rt] = 0;
  }
  // correction accumulators: thread rt owns column rt (D = 128: both blocks;
  // D = 64: block rt / 64, column rt % 64)
  constexpr int NACC = D / 64;
  float acc[NACC];
#pragma unroll
  for (int a = 0; a < NACC; ++a) acc[a] = 0.f;

  bool ok = true;
  constexpr bool SEL = RULE != 0;
  for (int pass = SEL ? 0 : 1; pass < 2 && ok; ++pass) {
  const bool scoring = !SEL || pass == 0;  // scores computed from the streamed pooled keys
  const bool deciding = pass == 1;         // kept bits and corrections
  for (int c = 0; c < nchunks; ++c) {
    const uint32_t g = chunk_ctr + c, buf = g & 1;
    float vcur[kChunk];
    if (deciding) {
#pragma unroll
      for (int jj = 0; jj < kChunk; ++jj)
        vcur[jj] = (c * kChunk + jj < NB) ? __ldg(vb + static_cast<long long>(c * kChunk + jj) * D + vcol) : 0.f;
    }
    const int j0 = c * kChunk;
    const int nk = min(kChunk, NB - j0);
    if (scoring) {
    if (rt == 0 && c + 1 < nchunks) issue(c + 1);  // buffer (c+1)&1 was released by chunk c-1
    const bool landed = mbar_wait(&sm.rfull[buf], (g >> 1) & 1, abort_flag, st, kSiteRouteChunk, u);
    if (named_bar_or(1, 128, !landed || *abort_flag)) {
      // aborting: let the copies already issued (chunks c and c + 1) land first
      if (rt == 0) {
        mbar_wait_quiet(&sm.rfull[buf], (g >> 1) & 1);
        if (c + 1 < nchunks) mbar_wait_quiet(&sm.rfull[(g + 1) & 1], ((g + 1) >> 1) & 1);
      }
      ok = false;
      break;
    }
    // ---- scores: warp rw handles key blocks 4 rw .. 4 rw + 3 of the chunk
    float v[8];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const float* row = &sm.rchunk[buf][rw * 4 + kk][lane * VPL];
      float x[VPL];
      if constexpr (VPL == 4) {
        const float4 t = *reinterpret_cast<const float4*>(row);
        x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
      } else {
        const float2 t = *reinterpret_cast<const float2*>(row);
        x[0] = t.x; x[1] = t.y;
      }
      float d0 = 0.f, d1 = 0.f;
#pragma unroll
      for (int e = 0; e < VPL; ++e) {
        d0 = fmaf(q0[e], x[e], d0);
        d1 = fmaf(q1[e], x[e], d1);
      }
      v[2 * kk] = d0;
      v[2 * kk + 1] = d1;
    }
    // transposed butterfly: after it, lane l holds the full sum of value (l >> 2)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const bool up = lane & 16;
      const float send = up ? v[i] : v[4 + i];
      const float keep = up ? v[4 + i] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const bool up = lane & 8;
      const float send = up ? v[i] : v[2 + i];
      const float keep = up ? v[2 + i] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
    }
    {
      const bool up = lane & 4;
      const float send = up ? v[0] : v[1];
      const float keep = up ? v[1] : v[0];
      v[0] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
    }
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 2);
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], 1);
    if ((lane & 3) == 0) {
      const int idx = lane >> 2;  // = 2 * kk + block
      sm.rscore[idx & 1][rw * 4 + (idx >> 1)] = v[0] * scale;
      if constexpr (SEL) {
        if (rw * 4 + (idx >> 1) < nk) sm.score[idx & 1][j0 + rw * 4 + (idx >> 1)] = v[0] * scale;
      }
    }
    named_bar_sync(1, 128);
    }  // scoring
    if (!deciding) {
      named_bar_sync(1, 128);  // the chunk buffer is free again
      continue;
    }
    // ---- kept bits, correction weights (warp 0: block 0, warp 1: block 1)
    if (rw < 2) {
      const int b = rw;
      const bool valid = lane < nk && (b == 0 || has1);
      float sh;
      bool by_rule;
      if constexpr (SEL) {
        sh = sm.score[b][j0 + (lane < nk ? lane : 0)];
        by_rule = !sm.keep_none[b] && order_key(sh) >= sm.cut[b];
      } else {
        sh = sm.rscore[b][lane & (kChunk - 1)];
        by_rule = sh > (b == 0 ? tau0 : tau1);
      }
      const bool kept = valid && (by_rule || j0 + lane < P.n_forced);
      const bool skip = valid && !kept;
      const uint32_t kmask = __ballot_sync(0xffffffffu, kept);
      float mx = skip ? sh : -INFINITY;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float mold = sm.rmax[b];
      const float mnew = fmaxf(mold, mx);
      const float nj = static_cast<float>(j0 + lane == NB - 1 ? nlast : kBN);
      const float w = skip ? nj * ex2_approx((sh - mnew) * kLog2e) : 0.f;
      float wsum = w;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
      if (lane < kChunk) sm.rweight[b][lane] = w;
      if (lane == 0) {
        const float sc = (mold == -INFINITY) ? 0.f : ex2_approx((mold - mnew) * kLog2e);
        sm.rscale[b] = sc;
        sm.rden[b] = sm.rden[b] * sc + wsum;
        sm.rmax[b] = mnew;
        sm.rkept[b] += __popc(kmask);
        // two 16-block chunks per 32-bit bitmap word (even chunk first)
        if (c & 1) sm.bits[s][b][c >> 1] |= kmask << 16;
        else sm.bits[s][b][c >> 1] = kmask;
      }
    }
    named_bar_sync(1, 128);
    // ---- correction sums: sum_j w_bj vbar_j[col] (weights of kept and pad blocks are 0)
    {
      if constexpr (D == 128) {
        float a0 = acc[0] * sm.rscale[0], a1 = acc[1] * sm.rscale[1];
#pragma unroll
        for (int jj = 0; jj < kChunk; ++jj) {
          a0 = fmaf(sm.rweight[0][jj], vcur[jj], a0);
          a1 = fmaf(sm.rweight[1][jj], vcur[jj], a1);
        }
        acc[0] = a0;
        acc[1] = a1;
      } else {
        const int b = rt / 64;
        float a0 = acc[0] * sm.rscale[b];
#pragma unroll
        for (int jj = 0; jj < kChunk; ++jj) a0 = fmaf(sm.rweight[b][jj], vcur[jj], a0);
        acc[0] = a0;
      }
    }
    named_bar_sync(1, 128);  // chunk buffer and scratch free again
  }
  if (scoring) chunk_ctr += nchunks;
  if (SEL && pass == 0 && ok) {
    // ---- each row's cut: the largest order key K whose superlevel set
    // {j : key(s_hat_ij) >= K} still holds k blocks (top-k) or a fraction p of
    // the row's mass sum_j n_j e^{s_hat_ij} (top-p); bisection over the 32 key
    // bits, sums in a fixed order (warp 0: block 0, warp 1: block 1)
    if (rw < 2) {
      const int b = rw;
      uint32_t K = 0u;
      int none = (b == 1 && !has1) ? 1 : 0;
      if (!none) {
        if constexpr (RULE == 1) {
          const int kk = P.topk;
          if (kk <= 0) {
            none = 1;
          } else if (kk < NB) {
            for (int bit = 31; bit >= 0; --bit) {
              const uint32_t cand = K | (1u << bit);
              int cnt = 0;
              for (int j = lane; j < NB; j += 32) cnt += order_key(sm.score[b][j]) >= cand ? 1 : 0;
#pragma unroll
              for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
              if (cnt >= kk) K = cand;
            }
          }
        } else {
          const float p = P.topp;
          if (p <= 0.f) {
            none = 1;
          } else if (p < 1.f) {
            float M = -INFINITY;
            for (int j = lane; j < NB; j += 32) M = fmaxf(M, sm.score[b][j]);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
            auto mass_at_least = [&](uint32_t cand) {
              float w = 0.f;
              for (int j = lane; j < NB; j += 32) {
                const float sh = sm.score[b][j];
                if (order_key(sh) >= cand)
                  w += static_cast<float>(j == NB - 1 ? nlast : kBN) * ex2_approx((sh - M) * kLog2e);
              }
              return warp_sum(w);
            };
            const float target = p * mass_at_least(0u);
            for (int bit = 31; bit >= 0; --bit) {
              const uint32_t cand = K | (1u << bit);
              if (mass_at_least(cand) >= target) K = cand;
            }
          }
        }
      }
      if (lane == 0) {
        sm.cut[b] = K;
        sm.keep_none[b] = none;
      }
    }
    named_bar_sync(1, 128);
  }
  }  // passes
  if (!ok) return false;
  // ---- publish the unit's correction and kept list into slot s
  if constexpr (D == 128) {
    sm.cnum[s][0][rt] = acc[0];
    sm.cnum[s][1][rt] = acc[1];
  } else {
    sm.cnum[s][rt / 64][rt % 64] = acc[0];
  }
  if (rt < 2) {
    sm.cden[s][rt] = sm.rden[rt];
    sm.cmax[s][rt] = sm.rmax[rt];
  }
  if (rw == 0) {
    const int nwords = (nchunks + 1) / 2;  // one 32-bit word per two chunks
    int base = 0;
    for (int wi = lane; wi < nwords; wi += 32) base += __popc(sm.bits[s][0][wi] | sm.bits[s][1][wi]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) base += __shfl_xor_sync(0xffffffffu, base, off);
    if (lane == 0) {
      sm.count[s] = base;
      if (P.density) {
        P.density[static_cast<long long>(bh) * NB + i0] = sm.rkept[0];
        if (has1) P.density[static_cast<long long>(bh) * NB + i1] = sm.rkept[1];
      }
    }
  }
  return true;
}

// In-order walk over a unit's key list (the union of the two kept bitmaps of a
// slot; without routing, every block). next() returns j | keep-bits << 14
// (bit 14: kept by the first query block, bit 15: by the second). Every lane
// of a warp walks identically. A walk past the last word returns 0 (no keep
// bits), so a count that disagreed with the bitmaps could not read past them.
template <bool ROUTE>
struct KeyWalk {
  const uint32_t* b0;
  const uint32_t* b1;
  int w, pos;
  uint32_t rem, c0, c1;  // unvisited bits of word w, and the word itself (both bitmaps)
  __device__ __forceinline__ KeyWalk(const uint32_t* x0, const uint32_t* x1)
      : b0(x0), b1(x1), w(-1), pos(0), rem(0u), c0(0u), c1(0u) {}
  __device__ __forceinline__ uint32_t next() {
    if constexpr (!ROUTE) {
      return static_cast<uint32_t>(pos++) | 0xC000u;
    } else {
      // shared memory is read only when the walk moves to the next word: the
      // callers sit between barriers and fences, so nothing read here would
      // stay in registers across calls otherwise
      while (rem == 0u) {
        if (w + 1 >= kNbMax / 32) return 0u;
        ++w;
        c0 = b0[w];
        c1 = b1[w];
        rem = c0 | c1;
      }
      const int bit = __ffs(rem) - 1;
      rem &= rem - 1u;
      const uint32_t f = ((c0 >> bit) & 1u) | (((c1 >> bit) & 1u) << 1);
      return static_cast<uint32_t>(w * 32 + bit) | (f << 14);
    }
  }
};

// ---------------------------------------------------------------------------
// Softmax arithmetic of one row and one 64-key tile (log2 domain, lazily
// rescaled running max m, running sum l). sv/sw hold S columns 0-31 / 32-63,
// nv = valid keys of the tile. Writes the bf16 P row into pw; returns whether
// the row's O must be multiplied by `rescale` before this tile's PV.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ uint64_t f2_from_bits(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}

__device__ __forceinline__ void f2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// Sets the pad keys of a partial block (only the last block of a head) to -inf.
__device__ __forceinline__ void mask_tail(uint32_t (&sv)[64], int nv) {
  constexpr uint32_t kNegInf = 0xFF800000u;
  if (nv < 64) {
#pragma unroll
    for (int c = 0; c < 64; ++c)
      if (c >= nv) sv[c] = kNegInf;
  }
}

// Max over the valid keys of one 64-key block (raw S units); masks the pad keys.
__device__ __forceinline__ float tile_max(uint32_t (&sv)[64], int nv) {
  mask_tail(sv, nv);
  float t[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    t[i] = fmax3(fmax3(__uint_as_float(sv[8 * i]), __uint_as_float(sv[8 * i + 1]), __uint_as_float(sv[8 * i + 2])),
                 fmax3(__uint_as_float(sv[8 * i + 3]), __uint_as_float(sv[8 * i + 4]), __uint_as_float(sv[8 * i + 5])),
                 fmaxf(__uint_as_float(sv[8 * i + 6]), __uint_as_float(sv[8 * i + 7])));
  return fmaxf(fmax3(t[0], t[1], t[2]), fmax3(fmax3(t[3], t[4], t[5]), t[6], t[7]));
}

// 2^y for two packed fp32 values on the FMA pipe (relieves the MUFU unit):
// Cody-Waite split y = n + f with n = round(y) (adding 1.5 * 2^23 leaves n in
// the low mantissa bits), f in [-1/2, 1/2], 2^f by the degree-3 minimax
// polynomial fitted by fit_exp2_poly.py (max relative error 7.5e-5, below
// the bf16 rounding of P), and n added to the exponent field with one integer
// multiply-add. y is clamped to >= -125 so 2^n stays a normal float (keys
// masked to -inf give 2^-125 ~ 2e-38, against a zero V row).
constexpr float kPolyC0 = 0.9999280571937561f, kPolyC1 = 0.6932609677314758f;
constexpr float kPolyC2 = 0.2426111400127411f, kPolyC3 = 0.0551716648042202f;
constexpr int kPolyPairs = 0;  // column pairs per 16-column slice evaluated by the polynomial (0 = all MUFU)

__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ uint64_t f2_dup(float x) { return f2_from_bits(__float_as_uint(x), __float_as_uint(x)); }

__device__ __forceinline__ void exp2_poly2(float y0, float y1, float& p0, float& p1) {
  const uint64_t x = f2_from_bits(__float_as_uint(fmaxf(y0, -125.f)), __float_as_uint(fmaxf(y1, -125.f)));
  const uint64_t t = fadd2(x, f2_dup(12582912.f));           // 1.5 * 2^23 + round(y)
  const uint64_t n = fadd2(t, f2_dup(-12582912.f));          // round(y)
  const uint64_t f = ffma2(n, f2_dup(-1.f), x);              // y - round(y)
  uint64_t q = ffma2(f2_dup(kPolyC3), f, f2_dup(kPolyC2));
  q = ffma2(q, f, f2_dup(kPolyC1));
  q = ffma2(q, f, f2_dup(kPolyC0));
  float q0, q1, t0, t1;
  f2_split(q, q0, q1);
  f2_split(t, t0, t1);
  // exponent += n: the low bits of t hold n, (bits(t) << 23) == n << 23 (mod 2^32)
  p0 = __int_as_float(static_cast<int>(__float_as_uint(t0) * 8388608u + __float_as_uint(q0)));
  p1 = __int_as_float(static_cast<int>(__float_as_uint(t1) * 8388608u + __float_as_uint(q1)));
}

// P for 16 consecutive columns (x holds their raw S bits): 8 packed bf16x2
// words; adds the fp32 probabilities to the packed pair of partial sums l2.
// The first 8 - kPolyPairs column pairs use the MUFU ex2, the others the
// FMA-pipe polynomial.
__device__ __forceinline__ void softmax_slice(const uint32_t* x, uint64_t sc2, uint64_t nm2, uint64_t& l2,
                                              uint32_t (&pw)[8]) {
#pragma unroll
  for (int c = 0; c < 16; c += 2) {
    float y0, y1, p0, p1;
    f2_split(ffma2(f2_from_bits(x[c], x[c + 1]), sc2, nm2), y0, y1);
    if ((c >> 1) < 8 - kPolyPairs) {
      p0 = ex2_approx(y0);  // ex2(-inf) = 0 for masked keys
      p1 = ex2_approx(y1);
    } else {
      exp2_poly2(y0, y1, p0, p1);
    }
    l2 = fadd2(l2, f2_from_bits(__float_as_uint(p0), __float_as_uint(p1)));
    pw[c >> 1] = pack_bf16x2(p0, p1);
  }
}

// A bf16 hi + lo pair (hi in the low half) whose sum is w to about 16 bits.
__device__ __forceinline__ uint32_t bias_pair(float w) {
  const float hi = __uint_as_float((pack_bf16x2(w, 0.f) & 0xFFFFu) << 16);
  return pack_bf16x2(hi, w - hi);
}

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
      SOLATTN_TRACE_EVENT(13, rt == 0 ? n : 4096);
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
        SOLATTN_TRACE_EVENT(14, n);
        SOLATTN_TRACE_VALUE(19, n, static_cast<unsigned long long>(sm.count[s]));
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
            SOLATTN_TRACE_EVENT(15, gt);
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
            SOLATTN_TRACE_EVENT(16, gt);
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
    // PV that last read P from that slot (tile t - 3) has completed: MMAs into
    // different accumulators are not ordered with each other, so the slot is
    // reused only after pv_done (waited once per tile, in order). The S ring
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
          if (lane == 0) SOLATTN_TRACE_EVENT(17, gt);
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
            SOLATTN_TRACE_EVENT(10, gt);
          }
          __syncwarp();
        }
      } else {
        // O is free once the epilogue has read the previous unit's
        if (n >= 1 && !warp_wait(&sm.o_free[(n - 1) & 1], ((n - 1) >> 1) & 1, abort_flag, st, kSiteOFree, u)) break;
        for (int t = 0; t < TT && ok; ++t) {
          const uint32_t gt = gtile + t;
          const int nb = ut.halves(t, P.NB);
          if (!warp_wait(&sm.p_full[gt % 3], (gt / 3) & 1, abort_flag, st, kSitePFull, u)) { ok = false; break; }
          if (lane == 0) SOLATTN_TRACE_EVENT(12, gt);
          uint32_t stv[2];
          for (int h = 0; h < nb && ok; ++h) {
            const uint32_t gv = gblk + ut.vblock(t, h);
            stv[h] = gv % VS;
            ok = warp_wait(&sm.v_full[stv[h]], (gv / VS) & 1, abort_flag, st, kSiteVFull, u);
          }
          if (!ok) break;
          if (lane == 0) SOLATTN_TRACE_EVENT(18, gt);
          tc_fence_after();
          if (elect_one()) {
            SOLATTN_TRACE_EVENT(11, gt);
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
        if (lane == 0 && warp == 0) SOLATTN_TRACE_EVENT(9, gt);
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
        if (lane == 0 && warp == 0) SOLATTN_TRACE_EVENT(7, gt);
        const bool okw = oke && warp_wait(&sm.s_full[slot], (gt / 3) & 1, abort_flag, st, kSiteSFull, u);
        if (lane == 0 && warp == 0) SOLATTN_TRACE_EVENT(8, gt);
        tc_fence_after();
        if (lane == 0 && warp == 0) SOLATTN_TRACE_EVENT(0, gt);
        if (lane == 0 && warp == 4) SOLATTN_TRACE_EVENT(27, gt);
        uint32_t sv[64];
        if (kept && okw) tmem_ld32x2_wait(colS + 64 * hh, colS + 64 * hh + 32, sv);
        if (lane == 0 && (warp & 3) == 0) SOLATTN_TRACE_EVENT(warp == 0 ? 5 : 25, gt);
        const float mx = (kept && okw) ? tile_max(sv, nv) * sl2 : -INFINITY;
        if (lane == 0 && (warp & 3) == 0) SOLATTN_TRACE_EVENT(warp == 0 ? 6 : 26, gt);
        // Does a row of this group need a new reference max (or did a wait fail)?
        // The barrier also orders this group's S reads before the other half's
        // P stores into the same columns.
        tc_fence_before();
        const bool any = named_bar_or(pb, 64, !okw || mx > m + kRescaleSlack);
        tc_fence_after();
        if (lane == 0 && warp == 0) SOLATTN_TRACE_EVENT(1, gt);
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
        if (lane == 0 && warp == 0) SOLATTN_TRACE_EVENT(3, gt);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[slot]);
        if (lane == 0 && warp == 0) SOLATTN_TRACE_EVENT(4, gt);
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

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// q, k or v as a 4D tensor {D, N, H, B} (D fastest) with the caller's element
// strides; box = 64 columns x `rows` tokens of one (b, h), 128-byte swizzle;
// tokens past N read as zero.
bool make_map(CUtensorMap* map, const void* base, int B, int H, int N, int D, const Strides& st, int rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(st.n) * 2, static_cast<cuuint64_t>(st.h) * 2,
                           static_cast<cuuint64_t>(st.b) * 2};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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
// Test builds only: CTA `skip_cta` never requests its first K tile (-1: none)
// and every bounded wait gives up after `wait_budget_ns`.
extern "C" int solattn_test_set_hook(int skip_cta, unsigned long long wait_budget_ns) {
  if (cudaMemcpyToSymbol(g_hook_skip_cta, &skip_cta, sizeof(skip_cta)) != cudaSuccess) return 4;
  if (cudaMemcpyToSymbol(g_wait_budget_ns, &wait_budget_ns, sizeof(wait_budget_ns)) != cudaSuccess) return 4;
  return 0;
}
#endif

#ifdef SOLATTN_TRACE
extern "C" int solattn_trace_read(unsigned long long* host, size_t n) {
  return cudaMemcpyFromSymbol(host, g_trace, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 4;
}
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
