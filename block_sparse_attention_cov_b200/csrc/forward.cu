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
// tcgen05 tile height) of one head. The key tiles of a unit are the union of
// the two blocks' kept sets; a tile kept by only one of the two blocks is still
// multiplied for all 128 rows, and the other block's rows mask it out (their P
// row is zero and their softmax state is untouched), so each block's result is
// exactly its own.
//
// One persistent CTA per SM, 320 threads, warp roles:
//   warps 0-3  softmax / epilogue: thread r owns row r of the unit (TMEM lane r)
//   warps 4-7  routing, one unit ahead: fetch the next unit from the atomic
//              scheduler, copy its Q rows into TMEM, score every key block,
//              build the ordered kept list and the correction sums in shared
//              memory (double-buffered unit slots)
//   warp 8     TMA producer: K and V tiles of the kept list only
//   warp 9     MMA issuer (one thread): S = Q K^T and O += P V with A (Q, P)
//              in TMEM and B (K, V) in shared memory
// TMEM columns: Q slot 0/1 at 0/64, O at 128, S buffers at 256/320, P buffers
// at 384/416 (512 allocated).
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
#else
#define SOLATTN_TRACE_EVENT(ev, idx) \
  do {                               \
  } while (0)
#endif

namespace {

constexpr int kBM = 128;      // rows per unit
constexpr int kBN = 64;       // keys per tile (one block)
constexpr int kStages = 5;    // depth of the K ring and of the V ring
constexpr int kNbMax = 4096;  // key blocks per head supported
constexpr int kThreads = 512;
// Registers per thread after rebalancing (launched with 65536 / 512 = 128):
// 2 softmax warpgroups x 136 + routing 120 + producer/MMA 120, times 128 threads
// each = 65536.
constexpr int kRegsSoftmax = 136, kRegsRouting = 120, kRegsIssue = 120;
static_assert(128 * (2 * kRegsSoftmax + kRegsRouting + kRegsIssue) <= 65536, "register split exceeds the launch");
constexpr int kChunk = 16;    // pooled key blocks per routing chunk (4 per routing warp)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleSlack = 8.0f;  // log2 units a row max may grow before O is rescaled

constexpr uint32_t kColQ = 0, kColS = 64, kColP = 192, kColO = 256;  // + group * 64 / 32 / 128

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
  kSiteBDone,
};

template <int D>
struct __align__(1024) Smem {
  uint8_t kt[kStages][kBN * D * 2];  // SW128 K tiles (1024-aligned: size is a multiple of 8 KB)
  uint8_t vt[kStages][kBN * D * 2];  // SW128 V tiles
  float rchunk[2][2][kChunk][D];     // routing: [buffer][kbar | vbar][key block][column]
  uint16_t list[2][kNbMax];          // kept (union) list: j | keep-bits << 14
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
  uint32_t bits[2][kNbMax / 32];     // kept bitmaps of the unit being routed
  uint64_t k_full[kStages], v_full[kStages], k_empty[kStages], v_empty[kStages];
  uint64_t s_full[2], s_free[2], p_full[2], o_full[2];  // per softmax group
  uint64_t o_free, b_done, q_free;
  uint64_t route_full[2], route_empty[2];
  uint64_t rfull[2];                 // routing chunk buffers landed
  uint64_t mma_done[2];
  float mB[2][kBM];                  // group B's final running max / sum per row, per slot
  float lB[2][kBM];
  uint32_t tmem_base;
  int bcast;
  int abort_flag;
};

// Dynamic shared memory per CTA on sm_100 is at most 227 KB (232448 bytes);
// one extra KB pays for the 1024-byte alignment of the TMA tiles.
static_assert(sizeof(Smem<128>) + 1024 <= 232448, "shared memory layout too large");
static_assert(sizeof(Smem<64>) + 1024 <= 232448, "shared memory layout too large");

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
  int BH, N, NB, npairs, units;
  DeviceStatus* status;
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          DeviceStatus* st, uint32_t site, uint32_t unit) {
  const bool ok = mbar_wait(bar, parity, abort_flag, st, site, unit);
  return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------------------
// Routing (warps 4-7, 128 threads): the pooled keys and values of the head are
// streamed through shared memory in chunks of 32 key blocks (bulk async copies,
// double-buffered). Per chunk: every warp scores 8 key blocks against both
// query blocks of the unit (one float4 column slice per lane, transposed
// butterfly reduction), the threshold test sets the kept bits, and the skipped
// blocks' weights n_j e^{s_hat - M} are folded into per-column correction sums
// (one column per thread). The proxy row never leaves shared memory.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Returns false if a bounded wait gave up (the CTA is aborting).
template <int D>
__device__ bool route_unit(Smem<D>& sm, const Params& P, int s, int bh, int pair, int rt, uint32_t& chunk_ctr,
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
    mbar_arrive_expect_tx(&sm.rfull[buf], 2 * bytes);
    bulk_copy_g2s(&sm.rchunk[buf][0][0][0], kb + static_cast<long long>(j0) * D, bytes, &sm.rfull[buf]);
    bulk_copy_g2s(&sm.rchunk[buf][1][0][0], vb + static_cast<long long>(j0) * D, bytes, &sm.rfull[buf]);
  };
  if (rt == 0) issue(0);

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
  if (beta != -INFINITY && beta != INFINITY) {
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
  for (int c = 0; c < nchunks; ++c) {
    const uint32_t g = chunk_ctr + c, buf = g & 1;
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
    const int j0 = c * kChunk;
    const int nk = min(kChunk, NB - j0);
    // ---- scores: warp rw handles key blocks 4 rw .. 4 rw + 3 of the chunk
    float v[8];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const float* row = &sm.rchunk[buf][0][rw * 4 + kk][lane * VPL];
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
    }
    named_bar_sync(1, 128);
    // ---- threshold, kept bits, correction weights (warp 0: block 0, warp 1: block 1)
    if (rw < 2) {
      const int b = rw;
      const bool valid = lane < nk && (b == 0 || has1);
      const float sh = sm.rscore[b][lane & (kChunk - 1)];
      const bool kept = valid && sh > (b == 0 ? tau0 : tau1);
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
        if (c & 1) sm.bits[b][c >> 1] |= kmask << 16;
        else sm.bits[b][c >> 1] = kmask;
      }
    }
    named_bar_sync(1, 128);
    // ---- correction sums: sum_j w_bj vbar_j[col]
    {
      const float* vrows = &sm.rchunk[buf][1][0][0];
      if constexpr (D == 128) {
        const float sc0 = sm.rscale[0], sc1 = sm.rscale[1];
        float a0 = acc[0] * sc0, a1 = acc[1] * sc1;
        for (int jj = 0; jj < nk; ++jj) {
          const float x = vrows[jj * D + rt];
          a0 = fmaf(sm.rweight[0][jj], x, a0);
          a1 = fmaf(sm.rweight[1][jj], x, a1);
        }
        acc[0] = a0;
        acc[1] = a1;
      } else {
        const int b = rt / 64, col = rt % 64;
        float a0 = acc[0] * sm.rscale[b];
        for (int jj = 0; jj < nk; ++jj) a0 = fmaf(sm.rweight[b][jj], vrows[jj * D + col], a0);
        acc[0] = a0;
      }
    }
    named_bar_sync(1, 128);  // chunk buffer and scratch free again
  }
  chunk_ctr += nchunks;
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
    for (int w0 = 0; w0 < nwords; w0 += 32) {
      const int wi = w0 + lane;
      const uint32_t m0 = wi < nwords ? sm.bits[0][wi] : 0u;
      const uint32_t m1 = wi < nwords ? sm.bits[1][wi] : 0u;
      uint32_t un = m0 | m1;
      const int cnt = __popc(un);
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      int pos = base + incl - cnt;
      while (un) {
        const int bit = __ffs(un) - 1;
        const uint32_t flags = ((m0 >> bit) & 1u) | (((m1 >> bit) & 1u) << 1);
        sm.list[s][pos++] = static_cast<uint16_t>((wi * 32 + bit) | (flags << 14));
        un &= un - 1u;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
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

// Reads the unit's 128 Q rows (bf16 pairs = one 32-bit TMEM column per pair)
// into registers; rows past N are zero.
template <int D>
__device__ __forceinline__ void load_q_rows(const Params& P, int bh, int pair, int rt, uint32_t (&w)[D / 2]) {
  const int row = pair * kBM + rt;
  const uint4* src = reinterpret_cast<const uint4*>(P.q + (static_cast<long long>(bh) * P.N + row) * D);
  const bool ok = row < P.N;
#pragma unroll
  for (int x = 0; x < D / 8; ++x) {
    const uint4 t = ok ? __ldg(src + x) : make_uint4(0, 0, 0, 0);
    w[4 * x] = t.x; w[4 * x + 1] = t.y; w[4 * x + 2] = t.z; w[4 * x + 3] = t.w;
  }
}

template <int D>
__device__ __forceinline__ void store_q_tmem(uint32_t tmem, int rt, const uint32_t (&w)[D / 2]) {
  const uint32_t taddr = tmem + (static_cast<uint32_t>((rt / 32) * 32) << 16) + kColQ;
#pragma unroll
  for (int c = 0; c < D / 64; ++c) {
    uint32_t x[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = w[c * 32 + e];
    tmem_st32(taddr + c * 32, x);
  }
  tmem_wait_st();
}

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

// Masks the pad keys of a partial tile and folds the tile's row max into the
// lazily rescaled running max m (log2 units). Returns whether the row's O and
// l must be multiplied by `rescale` (= 2^(m_old - m_new)) before this tile.
__device__ __forceinline__ bool softmax_max(uint32_t (&sv)[32], uint32_t (&sw)[32], int nv, float sl2, float& m,
                                            float& rescale) {
  constexpr uint32_t kNegInf = 0xFF800000u;
  if (nv < 64) {  // only the last key block of a head can be partial
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      if (c >= nv) sv[c] = kNegInf;
      if (c + 32 >= nv) sw[c] = kNegInf;
    }
  }
  float t[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    t[i] = fmax3(fmax3(__uint_as_float(sv[8 * i]), __uint_as_float(sv[8 * i + 1]), __uint_as_float(sv[8 * i + 2])),
                 fmax3(__uint_as_float(sv[8 * i + 3]), __uint_as_float(sv[8 * i + 4]), __uint_as_float(sv[8 * i + 5])),
                 fmaxf(__uint_as_float(sv[8 * i + 6]), __uint_as_float(sv[8 * i + 7])));
    t[4 + i] = fmax3(fmax3(__uint_as_float(sw[8 * i]), __uint_as_float(sw[8 * i + 1]), __uint_as_float(sw[8 * i + 2])),
                     fmax3(__uint_as_float(sw[8 * i + 3]), __uint_as_float(sw[8 * i + 4]), __uint_as_float(sw[8 * i + 5])),
                     fmaxf(__uint_as_float(sw[8 * i + 6]), __uint_as_float(sw[8 * i + 7])));
  }
  const float mx = fmaxf(fmax3(t[0], t[1], t[2]), fmax3(fmax3(t[3], t[4], t[5]), t[6], t[7])) * sl2;
  rescale = 1.f;
  if (mx > m + kRescaleSlack) {
    const bool need = m != -INFINITY;
    if (need) rescale = ex2_approx(m - mx);
    m = mx;
    return need;
  }
  return false;
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
// words; adds the fp32 probabilities to l. The first 8 - kPolyPairs column
// pairs use the MUFU ex2, the others the FMA-pipe polynomial.
__device__ __forceinline__ void softmax_slice(const uint32_t* x, uint64_t sc2, uint64_t nm2, float& l,
                                              uint32_t (&pw)[8]) {
  float a0 = 0.f, a1 = 0.f;
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
    if (c & 2) a1 += p0 + p1; else a0 += p0 + p1;
    pw[c >> 1] = pack_bf16x2(p0, p1);
  }
  l += a0 + a1;
}

// ---------------------------------------------------------------------------
// The kernel. 512 threads = 16 warps:
//   warps 0-3   softmax group A (even global tiles) + epilogue
//   warps 4-7   softmax group B (odd global tiles)
//   warps 8-11  routing, one unit ahead (Q rows into TMEM after the previous
//               unit's last QK has completed)
//   warp 12     TMA producer of the K tiles of the kept list
//   warps 13/15 MMA issuers of group A / group B (one elected lane issues)
//   warp 14     TMA producer of the V tiles
// TMEM: Q at 0 (64 columns), S_A/S_B at 64/128, P_A/P_B at 192/224,
// O_A/O_B at 256/384. Each group keeps its own running max, sum and O; the
// epilogue merges the two with the skipped-block correction.
// ---------------------------------------------------------------------------
template <int D, bool ROUTE>
__global__ void __launch_bounds__(kThreads, 1)
    solattn_fwd_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const Params P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* aligned = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>(aligned);
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  DeviceStatus* st = P.status;
  volatile int* abort_flag = &sm.abort_flag;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&sm.k_full[i], 1);
      mbar_init(&sm.v_full[i], 1);
      mbar_init(&sm.k_empty[i], 1);
      mbar_init(&sm.v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_free[i], 4);
      mbar_init(&sm.p_full[i], 4);
      mbar_init(&sm.o_full[i], 1);
      mbar_init(&sm.route_full[i], 1);
      mbar_init(&sm.route_empty[i], 12);  // 2 producers + 2 MMA issuers + 8 softmax warps
      mbar_init(&sm.rfull[i], 1);
    }
    mbar_init(&sm.o_free, 4);
    mbar_init(&sm.b_done, 4);
    mbar_init(&sm.q_free, 2);  // one commit per MMA issuer
    mbar_init(&sm.mma_done[0], 1);
    mbar_init(&sm.mma_done[1], 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 13) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 12 && lane == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (warp >= 12) {
    regs_dec<kRegsIssue>();
  } else if (warp >= 8) {
    regs_dec<kRegsRouting>();
  } else {
    regs_inc<kRegsSoftmax>();
  }

  if (warp >= 8 && warp < 12) {
    // ======================= routing =======================
    const int rt = tid - 256;
    uint32_t chunk_ctr = 0;  // routing chunks consumed so far (buffer parity)
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
        if (!route_unit<D>(sm, P, s, bh, pair, rt, chunk_ctr, abort_flag, st, u)) break;
      } else {
        if (rt == 0) {
          sm.count[s] = P.NB;
          sm.cden[s][0] = sm.cden[s][1] = 0.f;
          sm.cmax[s][0] = sm.cmax[s][1] = -INFINITY;
        }
      }
      uint32_t qw[D / 2];
      load_q_rows<D>(P, bh, pair, rt, qw);
      if (n >= 1) {  // the Q slot is free once every QK of the previous unit has completed
        const bool okq = mbar_wait(&sm.q_free, (n - 1) & 1, abort_flag, st, kSiteQFree, u);
        if (named_bar_or(1, 128, !okq)) break;
      }
      tc_fence_after();
      store_q_tmem<D>(tmem, rt, qw);
      tc_fence_before();
      named_bar_sync(1, 128);
      if (rt == 0) {
        sm.unit[s] = u;
        mbar_arrive(&sm.route_full[s]);
        SOLATTN_TRACE_EVENT(14, n);
      }
    }
  } else if (warp == 12 || warp == 14) {
    // ======================= TMA producers: warp 12 = K tiles, warp 14 = V tiles =======================
    const bool isK = warp == 12;
    uint64_t* full = isK ? sm.k_full : sm.v_full;
    uint64_t* empty = isK ? sm.k_empty : sm.v_empty;
    const CUtensorMap* map = isK ? &tmK : &tmV;
    uint8_t* ring = isK ? &sm.kt[0][0] : &sm.vt[0][0];
    uint32_t g = 0;
    for (int n = 0;; ++n) {
      const int s = n & 1;
      if (!warp_wait(&sm.route_full[s], (n >> 1) & 1, abort_flag, st, kSiteRouteFullProd, 0)) break;
      const int u = sm.unit[s];
      if (u < 0) break;
      const int T = sm.count[s];
      const int bh = u / P.npairs;
      int t = 0;
      for (; t < T; ++t) {
        const int j = ROUTE ? (sm.list[s][t] & 0x3FFF) : t;
        const uint32_t gt = g + t, stg = gt % kStages, r = gt / kStages;
        if (r >= 1 && !warp_wait(&empty[stg], (r - 1) & 1, abort_flag, st, isK ? kSiteKEmpty : kSiteVEmpty, u)) break;
        if (elect_one()) {
          mbar_arrive_expect_tx(&full[stg], kBN * D * 2);
#pragma unroll
          for (int pnl = 0; pnl < D / 64; ++pnl)
            tma_load_3d(ring + stg * (kBN * D * 2) + pnl * 8192, map, &full[stg], pnl * 64, j * kBN, bh);
        }
        __syncwarp();
      }
      g += t;
      if (t < T) break;  // aborted
      if (elect_one()) mbar_arrive(&sm.route_empty[s]);
      __syncwarp();
    }
    if (lane == 0) {  // teardown: every issued copy lands before the CTA exits
      const uint32_t first = g > static_cast<uint32_t>(kStages) ? g - kStages : 0u;
      for (uint32_t gt = first; gt < g; ++gt) mbar_wait_quiet(&full[gt % kStages], (gt / kStages) & 1);
    }
    __syncwarp();
  } else if (warp == 13 || warp == 15) {
    // ======================= MMA issuers: warp 13 for group A, warp 15 for group B =======================
    // For the group's own tiles t (global tile parity = group): QK of the next
    // own tile as soon as the group has read the S of the current one (one S
    // buffer per group), then PV of the current one once its P is stored.
    // Waits sleep on their mbarrier (bounded); one lane issues.
    const int grp = warp == 13 ? 0 : 1;
    constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
    constexpr uint32_t kTileBytes = kBN * D * 2;
    const uint64_t kdesc0 = sw128_desc(smem_u32(&sm.kt[0][0]), 16, 1024);
    const uint64_t vdesc0 = sw128_desc(smem_u32(&sm.vt[0][0]), 8192, 1024);
    const uint32_t colS = tmem + kColS + grp * 64, colP = tmem + kColP + grp * 32, colO = tmem + kColO + grp * 128;
    uint32_t g = 0;
    bool ok = true;
    auto issue_qk = [&](uint32_t gt, int u, bool last) -> bool {
      const uint32_t stg = gt % kStages, use = gt >> 1;
      if (use >= 1 && !warp_wait(&sm.s_free[grp], (use - 1) & 1, abort_flag, st, kSiteSFree, u)) return false;
      if (!warp_wait(&sm.k_full[stg], (gt / kStages) & 1, abort_flag, st, kSiteKFull, u)) return false;
      tc_fence_after();
      if (elect_one()) {
        const uint64_t kd = kdesc0 + ((stg * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ts(colS, tmem + kColQ + kk * 8, kd + ((((kk / 4) * 8192) + (kk % 4) * 32) >> 4), idesc_qk,
                 kk > 0 ? 1u : 0u);
        mma_commit(&sm.s_full[grp]);
        mma_commit(&sm.k_empty[stg]);
        if (last) mma_commit(&sm.q_free);
        SOLATTN_TRACE_EVENT(10, gt);
      }
      __syncwarp();
      return true;
    };
    for (int n = 0; ok; ++n) {
      const int s = n & 1;
      if (!warp_wait(&sm.route_full[s], (n >> 1) & 1, abort_flag, st, kSiteRouteFullMma, 0)) break;
      tc_fence_after();
      const int u = sm.unit[s];
      if (u < 0) break;
      const int T = sm.count[s];
      const int t0 = ((g & 1u) == static_cast<uint32_t>(grp)) ? 0 : 1;  // first own tile of the unit
      if (t0 >= T) {  // no own tile: still release the Q slot and keep o_free's phase
        if (elect_one()) mma_commit(&sm.q_free);
        __syncwarp();
        if (n >= 1 && !warp_wait(&sm.o_free, (n - 1) & 1, abort_flag, st, kSiteOFree, u)) break;
      } else {
        ok = issue_qk(g + t0, u, t0 + 2 >= T);
        if (ok && n >= 1 && !warp_wait(&sm.o_free, (n - 1) & 1, abort_flag, st, kSiteOFree, u)) ok = false;
        for (int t = t0; t < T && ok; t += 2) {
          if (t + 2 < T && !(ok = issue_qk(g + t + 2, u, t + 4 >= T))) break;
          const uint32_t gp = g + t, stp = gp % kStages, usep = gp >> 1;
          if (!warp_wait(&sm.p_full[grp], usep & 1, abort_flag, st, kSitePFull, u)) { ok = false; break; }
          if (!warp_wait(&sm.v_full[stp], (gp / kStages) & 1, abort_flag, st, kSiteVFull, u)) { ok = false; break; }
          tc_fence_after();
          if (elect_one()) {
            SOLATTN_TRACE_EVENT(11, gp);
            const uint64_t vd = vdesc0 + ((stp * kTileBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk)
              mma_ts(colO, colP + kk * 8, vd + ((kk * 2048) >> 4), idesc_pv, (t > t0 || kk > 0) ? 1u : 0u);
            mma_commit(&sm.v_empty[stp]);
            mma_commit(&sm.o_full[grp]);
          }
          __syncwarp();
        }
      }
      if (!ok) break;
      if (elect_one()) mma_commit(&sm.route_empty[s]);
      __syncwarp();
      g += T;
    }
    if (elect_one()) mma_commit(&sm.mma_done[grp]);  // teardown: issued MMAs complete before TMEM is freed
    __syncwarp();
    mbar_wait_quiet(&sm.mma_done[grp], 0);
    __syncwarp();
  } else {
    // ======================= softmax groups A (warps 0-3) and B (4-7) =======================
    const int grp = warp >> 2;   // 0 = A (even global tiles), 1 = B (odd)
    const int r = tid & 127;     // row of the unit == TMEM lane
    const int blk = r >> 6;      // which of the two query blocks
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const float sl2 = kLog2e * rsqrtf(static_cast<float>(D));
    const int nlast = P.N - (P.NB - 1) * kBN;
    const uint32_t colS = tmem + kColS + grp * 64 + lane_off;
    const uint32_t colP = tmem + kColP + grp * 32 + lane_off;
    const uint32_t colO = tmem + kColO + grp * 128 + lane_off;
    uint32_t g = 0;
    for (int n = 0;; ++n) {
      const int s = n & 1;
      if (!warp_wait(&sm.route_full[s], (n >> 1) & 1, abort_flag, st, kSiteRouteFullSoft, 0)) break;
      tc_fence_after();
      const int u = sm.unit[s];
      if (u < 0) break;
      const int T = sm.count[s];
      const int bh = u / P.npairs, pair = u % P.npairs;
      float m = -INFINITY, l = 0.f;
      bool ok = true, first = true;
      uint32_t last_use = 0;
      for (int t = ((g & 1u) == static_cast<uint32_t>(grp)) ? 0 : 1; t < T; t += 2) {
        const uint32_t gt = g + t, use = gt >> 1;
        const uint32_t entry = ROUTE ? sm.list[s][t] : (static_cast<uint32_t>(t) | 0xC000u);
        const int j = entry & 0x3FFF;
        const bool mine = (entry >> (14 + blk)) & 1u;  // warp-uniform
        if (!warp_wait(&sm.s_full[grp], use & 1, abort_flag, st, kSiteSFull, u)) { ok = false; break; }
        tc_fence_after();
        if ((tid & 127) == 0) SOLATTN_TRACE_EVENT(grp * 5 + 0, gt);
        uint32_t sv[32], sw[32];
        if (mine) {
          tmem_ld32(colS, sv);
          tmem_ld32(colS + 32, sw);
          tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if ((tid & 127) == 0) SOLATTN_TRACE_EVENT(grp * 5 + 1, gt);
        if (lane == 0) mbar_arrive(&sm.s_free[grp]);
        float rescale = 1.f;
        bool need = false;
        uint32_t pw[32];
        if (mine) {
          need = softmax_max(sv, sw, (j == P.NB - 1) ? nlast : kBN, sl2, m, rescale);
          if (need) l *= rescale;
          if ((tid & 127) == 0) SOLATTN_TRACE_EVENT(grp * 5 + 2, gt);
          const uint64_t sc2 = f2_dup(sl2);
          const uint64_t nm2 = f2_dup(-m);
          softmax_slice(&sv[0], sc2, nm2, l, *reinterpret_cast<uint32_t(*)[8]>(&pw[0]));
          softmax_slice(&sv[16], sc2, nm2, l, *reinterpret_cast<uint32_t(*)[8]>(&pw[8]));
          softmax_slice(&sw[0], sc2, nm2, l, *reinterpret_cast<uint32_t(*)[8]>(&pw[16]));
          softmax_slice(&sw[16], sc2, nm2, l, *reinterpret_cast<uint32_t(*)[8]>(&pw[24]));
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) pw[c] = 0u;
        }
        // this group's previous PV must be complete: it read the P buffer and wrote O
        if (!first && !warp_wait(&sm.o_full[grp], (use - 1) & 1, abort_flag, st, kSiteOFull, u)) { ok = false; break; }
        tc_fence_after();
        if ((tid & 127) == 0) SOLATTN_TRACE_EVENT(grp * 5 + 3, gt);
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int ch = 0; ch < D / 16; ++ch) {
            uint32_t ov[16];
            tmem_ld16(colO + ch * 16, ov);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * rescale);
            tmem_st16(colO + ch * 16, ov);
          }
        }
        tmem_st32(colP, pw);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[grp]);
        if ((tid & 127) == 0) SOLATTN_TRACE_EVENT(grp * 5 + 4, gt);
        first = false;
        last_use = use;
      }
      if (!ok) break;
      // this group's last PV of the unit
      if (!first) {
        if (!warp_wait(&sm.o_full[grp], last_use & 1, abort_flag, st, kSiteOFull, u)) break;
        tc_fence_after();
      }
      if (grp == 1) {
        sm.mB[s][r] = m;
        sm.lB[s][r] = l;
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sm.b_done);
          mbar_arrive(&sm.route_empty[s]);
        }
        g += T;
        continue;
      }
      // ---------------- epilogue (group A): merge A, B and the correction ----------------
      if (!warp_wait(&sm.b_done, n & 1, abort_flag, st, kSiteBDone, u)) break;
      const bool hasA = !first;
      const int tilesB = ((g & 1u) == 1u) ? (T + 1) / 2 : T / 2;
      const bool hasB = tilesB > 0;
      const float mB = sm.mB[s][r], lB = sm.lB[s][r];
      const float mc = sm.cmax[s][blk] * kLog2e;
      const float cd = sm.cden[s][blk];
      const float mf = fmax3(m, mB, mc);
      const float wa = (m == -INFINITY) ? 0.f : ex2_approx(m - mf);
      const float wb = (mB == -INFINITY) ? 0.f : ex2_approx(mB - mf);
      const float wc = (mc == -INFINITY) ? 0.f : ex2_approx(mc - mf);
      const float L = fmaf(l, wa, fmaf(lB, wb, cd * wc));
      const float inv = 1.f / L;
      const int row = pair * kBM + r;
      const bool valid = row < P.N;
      uint16_t* orow = P.out + (static_cast<long long>(bh) * P.N + row) * D;
      for (int ch = 0; ch < D / 16; ++ch) {
        float y[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) y[e] = 0.f;
        if constexpr (ROUTE) {
#pragma unroll
          for (int e = 0; e < 16; ++e) y[e] = sm.cnum[s][blk][ch * 16 + e] * wc;
        }
        uint32_t o[16];
        if (hasA) {
          tmem_ld16(colO + ch * 16, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) y[e] = fmaf(__uint_as_float(o[e]), wa, y[e]);
        }
        if (hasB) {
          tmem_ld16(colO + 128 + ch * 16, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) y[e] = fmaf(__uint_as_float(o[e]), wb, y[e]);
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
      if (valid && P.lse) P.lse[static_cast<long long>(bh) * P.N + row] = (mf + __log2f(L)) * kLn2;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.o_free);
        mbar_arrive(&sm.route_empty[s]);
      }
      g += T;
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

// [BH][N][D] bf16 viewed as a 3D tensor (D fastest); box = 64 columns x 64 rows,
// 128-byte swizzle; rows past N read as zero.
bool make_kv_map(CUtensorMap* map, const void* base, int BH, int N, int D) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(N) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kBN), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, bool ROUTE>
cudaError_t launch_fwd_t(const ForwardArgs& a, int num_sms, cudaStream_t stream) {
  CUtensorMap tmK, tmV;
  if (!make_kv_map(&tmK, a.k, a.BH, a.N, D) || !make_kv_map(&tmV, a.v, a.BH, a.N, D))
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
  p.BH = a.BH;
  p.N = a.N;
  p.NB = (a.N + kBN - 1) / kBN;
  p.npairs = (p.NB + 1) / 2;
  p.units = a.BH * p.npairs;
  p.status = static_cast<DeviceStatus*>(a.status);
  const size_t smem = sizeof(Smem<D>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(solattn_fwd_kernel<D, ROUTE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = p.units < num_sms ? p.units : num_sms;
  solattn_fwd_kernel<D, ROUTE><<<grid, kThreads, smem, stream>>>(tmK, tmV, p);
  return cudaGetLastError();
}

}  // namespace

#ifdef SOLATTN_TRACE
extern "C" int solattn_trace_read(unsigned long long* host, size_t n) {
  return cudaMemcpyFromSymbol(host, g_trace, n * sizeof(unsigned long long)) == cudaSuccess ? 0 : 4;
}
#endif

cudaError_t launch_forward(const ForwardArgs& a, int num_sms, cudaStream_t stream) {
  if (a.d == 64) return a.route ? launch_fwd_t<64, true>(a, num_sms, stream) : launch_fwd_t<64, false>(a, num_sms, stream);
  return a.route ? launch_fwd_t<128, true>(a, num_sms, stream) : launch_fwd_t<128, false>(a, num_sms, stream);
}

}  // namespace solattn
