// fwd_common.cuh -- pieces shared by the two fused forward kernels (forward.cu,
// forward_pp.cu): kernel parameters, the routing warps' per-unit work (proxy
// scores, per-row threshold, kept bitmaps, zeroth-order correction sums), the
// walk over a unit's key list, softmax arithmetic helpers and the host-side
// tensor-map encoder.
//
// Method: "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly
// Attention Sparsification" (pages: hotpaper.ai abstract; paithon.it sections
// "Una soglia per ogni riga" and "Scegliere mentre si calcola").
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cmath>
#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace solattn {
namespace {

constexpr int kBM = 128;      // rows per unit
constexpr int kBN = 64;       // keys per block (a tile holds two)
constexpr int kNbMax = 4096;  // key blocks per head supported
constexpr int kChunk = 16;    // pooled key blocks per routing chunk (4 per routing warp)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleSlack = 16.0f;  // log2 units a row max may grow before O is rescaled

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

#ifdef SOLATTN_TEST_HOOKS
// Test builds only: when set, the routing warps copy every unit's kept bitmaps
// ([BH][N_b][ceil(N_b / 32)] words, bit j % 32 of word j / 32 = key block j
// kept) and its rows' mu, sigma, tau ([BH][N_b][3] floats) to these buffers.
// One copy per translation unit; set through set_route_dump_<kernel>().
static __device__ uint32_t* g_hook_route_mask = nullptr;
static __device__ float* g_hook_route_stats = nullptr;

inline cudaError_t set_route_dump_here(uint32_t* mask, float* stats) {
  cudaError_t e = cudaMemcpyToSymbol(g_hook_route_mask, &mask, sizeof(mask));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(g_hook_route_stats, &stats, sizeof(stats));
  return e;
}
#endif

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

template <int REGION = 0>
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          DeviceStatus* st, uint32_t site, uint32_t unit) {
  const bool ok = mbar_wait<REGION>(bar, parity, abort_flag, st, site, unit);
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

// Read-only global load that does not allocate in L1: the routing warps stream
// the head's pooled values and covariance (hundreds of KB per unit) from L2,
// and L1 (what shared memory leaves of it) is better kept for the other warps.
__device__ __forceinline__ float ld_stream_f32(const float* p) {
  float v;
  asm volatile("ld.global.nc.L1::no_allocate.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
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
template <int D, int RULE, class SM>
__device__ bool route_unit(SM& sm, const Params& P, int s, int bh, int pair, int rt, uint32_t& chunk_ctr,
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
  float mu0 = NAN, mu1 = NAN, sig0 = NAN, sig1 = NAN;  // reported by test builds only
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
      const float c = ld_stream_f32(C + r * D + col);
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
    mu0 = scale * tot[0];
    mu1 = scale * tot[2];
    sig0 = sg0;
    sig1 = sg1;
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
        vcur[jj] = (c * kChunk + jj < NB) ? ld_stream_f32(vb + static_cast<long long>(c * kChunk + jj) * D + vcol) : 0.f;
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
#ifdef SOLATTN_TEST_HOOKS
  // Test builds only: the unit's kept bitmaps and row statistics, for the
  // element-by-element comparison of the kept sets with the oracle's.
  if (g_hook_route_mask) {
    const int nwords = (nchunks + 1) / 2;
    uint32_t* m0 = g_hook_route_mask + (static_cast<long long>(bh) * NB + i0) * nwords;
    for (int w = rt; w < nwords; w += 128) {
      m0[w] = sm.bits[s][0][w];
      if (has1) m0[nwords + w] = sm.bits[s][1][w];
    }
    if (rt == 0) {
      float* r0 = g_hook_route_stats + (static_cast<long long>(bh) * NB + i0) * 3;
      r0[0] = mu0;
      r0[1] = sig0;
      r0[2] = RULE == 0 ? tau0 : NAN;
      if (has1) {
        r0[3] = mu1;
        r0[4] = sig1;
        r0[5] = RULE == 0 ? tau1 : NAN;
      }
    }
  }
#endif
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

__device__ __forceinline__ uint64_t fadd2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ uint64_t f2_dup(float x) { return f2_from_bits(__float_as_uint(x), __float_as_uint(x)); }

// P for 16 consecutive columns (x holds their raw S bits): 8 packed bf16x2
// words; adds the fp32 probabilities to the packed pair of partial sums l2.
__device__ __forceinline__ void softmax_slice(const uint32_t* x, uint64_t sc2, uint64_t nm2, uint64_t& l2,
                                              uint32_t (&pw)[8]) {
#pragma unroll
  for (int c = 0; c < 16; c += 2) {
    float y0, y1;
    f2_split(ffma2(f2_from_bits(x[c], x[c + 1]), sc2, nm2), y0, y1);
    const float p0 = ex2_approx(y0);  // ex2(-inf) = 0 for masked keys
    const float p1 = ex2_approx(y1);
    l2 = fadd2(l2, f2_from_bits(__float_as_uint(p0), __float_as_uint(p1)));
    pw[c >> 1] = pack_bf16x2(p0, p1);
  }
}

// A bf16 hi + lo pair (hi in the low half) whose sum is w to about 16 bits.
__device__ __forceinline__ uint32_t bias_pair(float w) {
  const float hi = __uint_as_float((pack_bf16x2(w, 0.f) & 0xFFFFu) << 16);
  return pack_bf16x2(hi, w - hi);
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

}  // namespace
}  // namespace solattn
