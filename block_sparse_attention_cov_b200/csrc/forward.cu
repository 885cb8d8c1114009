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

namespace {

constexpr int kBM = 128;      // rows per unit
constexpr int kBN = 64;       // keys per tile (one block)
constexpr int kStages = 4;    // K/V ring depth
constexpr int kNbMax = 4096;  // key blocks per head supported
constexpr int kThreads = 320;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleSlack = 8.0f;  // log2 units a row max may grow before O is rescaled

constexpr uint32_t kColQ = 0, kColO = 128, kColS = 256, kColP = 384;

// Wait-site ids reported in the status word when a bounded wait gives up.
enum : uint32_t {
  kSiteRouteEmpty = 1,
  kSiteRouteFullProd,
  kSiteKvEmpty,
  kSiteRouteFullMma,
  kSiteKFull,
  kSiteSFree,
  kSiteOFree,
  kSitePFull,
  kSiteVFull,
  kSiteRouteFullSoft,
  kSiteSFull,
  kSiteOFull,
};

template <int D>
struct __align__(1024) Smem {
  uint8_t kt[kStages][kBN * D * 2];  // SW128 K tiles (1024-aligned: size is a multiple of 8 KB)
  uint8_t vt[kStages][kBN * D * 2];  // SW128 V tiles
  uint16_t list[2][kNbMax];          // kept (union) list: j | keep-bits << 14
  float cnum[2][2][D];               // correction numerator per slot and block
  float cden[2][2];
  float cmax[2][2];                  // reference max of the correction (natural units)
  int unit[2];
  int count[2];
  float wnum[4][2][D];               // per routing warp partial corrections
  float wden[4][2];
  float wmax[4][2];
  uint32_t bits[2][kNbMax / 32];     // kept bitmaps of the unit being routed
  uint64_t k_full[kStages], v_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_free[2], p_full[2];
  uint64_t o_full, o_free;
  uint64_t route_full[2], route_empty[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int bcast;
  int abort_flag;
};

struct Params {
  const uint16_t* q;
  uint16_t* out;
  float* lse;
  int32_t* density;
  const float* qbar;
  const float* kbar;
  const float* vbar;
  const float* mu;
  const float* sigma;
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
// Routing: scores of both query blocks against every key block, kept bitmaps,
// correction sums. 128 threads (warps 4-7), one key block per warp per trip.
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void corr_add(float& M, float& den, float (&num)[D / 32], float sh, float nj,
                                         const float (&vv)[D / 32]) {
  if (sh > M) {
    const float sc = ex2_approx((M - sh) * kLog2e);  // 0 when M = -inf
    den *= sc;
#pragma unroll
    for (int e = 0; e < D / 32; ++e) num[e] *= sc;
    M = sh;
  }
  const float w = nj * ex2_approx((sh - M) * kLog2e);
  den += w;
#pragma unroll
  for (int e = 0; e < D / 32; ++e) num[e] = fmaf(w, vv[e], num[e]);
}

template <int D>
__device__ __forceinline__ void load_vec(const float* p, float (&x)[D / 32]) {
  if constexpr (D == 128) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(p));
    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
  } else {
    const float2 t = __ldg(reinterpret_cast<const float2*>(p));
    x[0] = t.x; x[1] = t.y;
  }
}

template <int D>
__device__ void route_unit(Smem<D>& sm, const Params& P, int s, int bh, int pair, int rt) {
  constexpr int VPL = D / 32;
  const int rw = rt / 32, lane = rt % 32;
  const int NB = P.NB;
  const int i0 = 2 * pair, i1 = 2 * pair + 1;
  const bool has1 = i1 < NB;
  const int nwords = (NB + 31) / 32;
  for (int w = rt; w < nwords; w += 128) {
    sm.bits[0][w] = 0u;
    sm.bits[1][w] = 0u;
  }
  const float* qb = P.qbar + static_cast<long long>(bh) * NB * D;
  float q0[VPL], q1[VPL];
  load_vec<D>(qb + static_cast<long long>(i0) * D + lane * VPL, q0);
  if (has1) {
    load_vec<D>(qb + static_cast<long long>(i1) * D + lane * VPL, q1);
  } else {
#pragma unroll
    for (int e = 0; e < VPL; ++e) q1[e] = 0.f;
  }
  const float beta = P.beta;
  // tau_i = mu_i + beta sigma_i. sigma_i = 0 means a constant proxy row (every
  // score equals mu_i = tau_i): nothing is strictly above it, so no block is
  // kept, whatever rounding does to the individual scores.
  auto tau_of = [&](int i) -> float {
    if (beta == -INFINITY) return -INFINITY;
    if (beta == INFINITY) return INFINITY;
    const float sg = P.sigma[static_cast<long long>(bh) * NB + i];
    if (sg == 0.f) return INFINITY;
    return P.mu[static_cast<long long>(bh) * NB + i] + beta * sg;
  };
  const float tau0 = tau_of(i0);
  const float tau1 = has1 ? tau_of(i1) : INFINITY;
  const float scale = rsqrtf(static_cast<float>(D));
  const int nlast = P.N - (NB - 1) * kBN;
  named_bar_sync(1, 128);  // bitmaps cleared

  float M0 = -INFINITY, M1 = -INFINITY, den0 = 0.f, den1 = 0.f;
  float num0[VPL], num1[VPL];
#pragma unroll
  for (int e = 0; e < VPL; ++e) num0[e] = num1[e] = 0.f;
  const float* kb = P.kbar + static_cast<long long>(bh) * NB * D + lane * VPL;
  const float* vb = P.vbar + static_cast<long long>(bh) * NB * D + lane * VPL;
  for (int j = rw; j < NB; j += 4) {
    float kv[VPL];
    load_vec<D>(kb + static_cast<long long>(j) * D, kv);
    float d0 = 0.f, d1 = 0.f;
#pragma unroll
    for (int e = 0; e < VPL; ++e) {
      d0 = fmaf(q0[e], kv[e], d0);
      d1 = fmaf(q1[e], kv[e], d1);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      d0 += __shfl_xor_sync(0xffffffffu, d0, off);
      d1 += __shfl_xor_sync(0xffffffffu, d1, off);
    }
    const float sh0 = d0 * scale, sh1 = d1 * scale;
    const bool k0 = sh0 > tau0;
    const bool k1 = has1 && (sh1 > tau1);
    if (lane == 0) {
      if (k0) atomicOr(&sm.bits[0][j >> 5], 1u << (j & 31));
      if (k1) atomicOr(&sm.bits[1][j >> 5], 1u << (j & 31));
    }
    const bool c0 = !k0, c1 = has1 && !k1;
    if (c0 || c1) {
      float vv[VPL];
      load_vec<D>(vb + static_cast<long long>(j) * D, vv);
      const float nj = static_cast<float>(j == NB - 1 ? nlast : kBN);
      if (c0) corr_add<D>(M0, den0, num0, sh0, nj, vv);
      if (c1) corr_add<D>(M1, den1, num1, sh1, nj, vv);
    }
  }
  // per-warp partials -> shared
#pragma unroll
  for (int e = 0; e < VPL; ++e) {
    sm.wnum[rw][0][lane * VPL + e] = num0[e];
    sm.wnum[rw][1][lane * VPL + e] = num1[e];
  }
  if (lane == 0) {
    sm.wden[rw][0] = den0;
    sm.wden[rw][1] = den1;
    sm.wmax[rw][0] = M0;
    sm.wmax[rw][1] = M1;
  }
  named_bar_sync(1, 128);
  // combine the four warps (fixed order)
  for (int idx = rt; idx < 2 * D; idx += 128) {
    const int b = idx / D, e = idx % D;
    float Mb = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) Mb = fmaxf(Mb, sm.wmax[w][b]);
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float mw = sm.wmax[w][b];
      if (mw != -INFINITY) acc = fmaf(sm.wnum[w][b][e], ex2_approx((mw - Mb) * kLog2e), acc);
    }
    sm.cnum[s][b][e] = acc;
  }
  if (rt < 2) {
    const int b = rt;
    float Mb = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) Mb = fmaxf(Mb, sm.wmax[w][b]);
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float mw = sm.wmax[w][b];
      if (mw != -INFINITY) acc = fmaf(sm.wden[w][b], ex2_approx((mw - Mb) * kLog2e), acc);
    }
    sm.cden[s][b] = acc;
    sm.cmax[s][b] = Mb;
  }
  // ordered union list from the bitmaps (warp 0 of the routing group)
  if (rw == 0) {
    int base = 0, kept0 = 0, kept1 = 0;
    for (int w0 = 0; w0 < nwords; w0 += 32) {
      const int wi = w0 + lane;
      const uint32_t m0 = wi < nwords ? sm.bits[0][wi] : 0u;
      const uint32_t m1 = wi < nwords ? sm.bits[1][wi] : 0u;
      uint32_t un = m0 | m1;
      const int c = __popc(un);
      int incl = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      int pos = base + incl - c;
      while (un) {
        const int bit = __ffs(un) - 1;
        const uint32_t flags = ((m0 >> bit) & 1u) | (((m1 >> bit) & 1u) << 1);
        sm.list[s][pos++] = static_cast<uint16_t>((wi * 32 + bit) | (flags << 14));
        un &= un - 1u;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
      kept0 += __popc(m0);
      kept1 += __popc(m1);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      kept0 += __shfl_xor_sync(0xffffffffu, kept0, off);
      kept1 += __shfl_xor_sync(0xffffffffu, kept1, off);
    }
    if (lane == 0) {
      sm.count[s] = base;
      if (P.density) {
        P.density[static_cast<long long>(bh) * NB + i0] = kept0;
        if (has1) P.density[static_cast<long long>(bh) * NB + i1] = kept1;
      }
    }
  }
}

// Copies the unit's 128 Q rows (bf16 pairs, one 32-bit TMEM column per pair)
// into the Q slot; rows past N are zero.
template <int D>
__device__ __forceinline__ void load_q_to_tmem(const Params& P, uint32_t tmem, int s, int bh, int pair, int rt) {
  const int row = pair * kBM + rt;
  const uint32_t taddr = tmem + (static_cast<uint32_t>((rt / 32) * 32) << 16) + kColQ + s * 64;
  const uint4* src = reinterpret_cast<const uint4*>(P.q + (static_cast<long long>(bh) * P.N + row) * D);
  const bool ok = row < P.N;
#pragma unroll
  for (int c = 0; c < D / 64; ++c) {
    uint32_t w[32];
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const uint4 t = ok ? __ldg(src + c * 8 + x) : make_uint4(0, 0, 0, 0);
      w[4 * x] = t.x; w[4 * x + 1] = t.y; w[4 * x + 2] = t.z; w[4 * x + 3] = t.w;
    }
    tmem_st32(taddr + c * 32, w);
  }
  tmem_wait_st();
}

// ---------------------------------------------------------------------------
// The kernel
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
      mbar_init(&sm.kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_free[i], 4);
      mbar_init(&sm.p_full[i], 4);
      mbar_init(&sm.route_full[i], 1);
      mbar_init(&sm.route_empty[i], 6);
    }
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.o_free, 4);
    mbar_init(&sm.mma_done, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&tmK);
    prefetch_tensormap(&tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp >= 4 && warp < 8) {
    // ======================= routing =======================
    const int rt = tid - 128;
    for (int n = 0;; ++n) {
      const int s = n & 1;
      if (n >= 2) {
        if (rt == 0)
          sm.bcast = mbar_wait(&sm.route_empty[s], ((n >> 1) - 1) & 1, abort_flag, st, kSiteRouteEmpty, 0) ? 1 : 0;
        named_bar_sync(1, 128);
        const int ok = sm.bcast;
        named_bar_sync(1, 128);
        if (!ok) break;
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
      load_q_to_tmem<D>(P, tmem, s, bh, pair, rt);
      if constexpr (ROUTE) {
        route_unit<D>(sm, P, s, bh, pair, rt);
      } else {
        if (rt == 0) {
          sm.count[s] = P.NB;
          sm.cden[s][0] = sm.cden[s][1] = 0.f;
          sm.cmax[s][0] = sm.cmax[s][1] = -INFINITY;
        }
      }
      tc_fence_before();
      named_bar_sync(1, 128);
      if (rt == 0) {
        sm.unit[s] = u;
        mbar_arrive(&sm.route_full[s]);
      }
    }
  } else if (warp == 8) {
    // ======================= TMA producer (lane 0 issues) =======================
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
        if (r >= 1 && !warp_wait(&sm.kv_empty[stg], (r - 1) & 1, abort_flag, st, kSiteKvEmpty, u)) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&sm.k_full[stg], kBN * D * 2);
#pragma unroll
          for (int pnl = 0; pnl < D / 64; ++pnl)
            tma_load_3d(&sm.kt[stg][pnl * 8192], &tmK, &sm.k_full[stg], pnl * 64, j * kBN, bh);
          mbar_arrive_expect_tx(&sm.v_full[stg], kBN * D * 2);
#pragma unroll
          for (int pnl = 0; pnl < D / 64; ++pnl)
            tma_load_3d(&sm.vt[stg][pnl * 8192], &tmV, &sm.v_full[stg], pnl * 64, j * kBN, bh);
        }
        __syncwarp();
      }
      g += t;
      if (t < T) break;  // aborted
      if (lane == 0) mbar_arrive(&sm.route_empty[s]);
      __syncwarp();
    }
    // teardown: let every issued copy land before the CTA exits
    if (lane == 0) {
      const uint32_t first = g > static_cast<uint32_t>(kStages) ? g - kStages : 0u;
      for (uint32_t gt = first; gt < g; ++gt) {
        mbar_wait_quiet(&sm.k_full[gt % kStages], (gt / kStages) & 1);
        mbar_wait_quiet(&sm.v_full[gt % kStages], (gt / kStages) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ======================= MMA issuer (lane 0 issues) =======================
    constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, false, true);
    uint32_t g = 0;
    bool ok = true;
    for (int n = 0; ok; ++n) {
      const int s = n & 1;
      if (!warp_wait(&sm.route_full[s], (n >> 1) & 1, abort_flag, st, kSiteRouteFullMma, 0)) break;
      tc_fence_after();
      const int u = sm.unit[s];
      if (u < 0) break;
      const int T = sm.count[s];
      const uint32_t qaddr = tmem + kColQ + s * 64;
      for (int t = 0; t <= T; ++t) {
        if (t < T) {
          const uint32_t gt = g + t, stg = gt % kStages, b = gt & 1, use = gt >> 1;
          if (!warp_wait(&sm.k_full[stg], (gt / kStages) & 1, abort_flag, st, kSiteKFull, u)) { ok = false; break; }
          if (use >= 1 && !warp_wait(&sm.s_free[b], (use - 1) & 1, abort_flag, st, kSiteSFree, u)) { ok = false; break; }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t kaddr = smem_u32(&sm.kt[stg][0]);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t bdesc = sw128_desc(kaddr + (kk / 4) * 8192 + (kk % 4) * 32, 16, 1024);
              mma_ts(tmem + kColS + b * 64, qaddr + kk * 8, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
            }
            mma_commit(&sm.s_full[b]);
          }
          __syncwarp();
        }
        if (t >= 1) {
          const int tp = t - 1;
          const uint32_t gp = g + tp, stp = gp % kStages, bp = gp & 1, usep = gp >> 1;
          if (tp == 0 && n >= 1 && !warp_wait(&sm.o_free, (n - 1) & 1, abort_flag, st, kSiteOFree, u)) { ok = false; break; }
          if (!warp_wait(&sm.p_full[bp], usep & 1, abort_flag, st, kSitePFull, u)) { ok = false; break; }
          if (!warp_wait(&sm.v_full[stp], (gp / kStages) & 1, abort_flag, st, kSiteVFull, u)) { ok = false; break; }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t vaddr = smem_u32(&sm.vt[stp][0]);
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk) {
              const uint64_t bdesc = sw128_desc(vaddr + kk * 2048, 8192, 1024);
              mma_ts(tmem + kColO, tmem + kColP + bp * 32 + kk * 8, bdesc, idesc_pv, (tp > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&sm.kv_empty[stp]);
            mma_commit(&sm.o_full);
          }
          __syncwarp();
        }
      }
      if (!ok) break;
      if (T == 0 && n >= 1 && !warp_wait(&sm.o_free, (n - 1) & 1, abort_flag, st, kSiteOFree, u)) break;
      if (lane == 0) mma_commit(&sm.route_empty[s]);
      __syncwarp();
      g += T;
    }
    // teardown: every issued MMA completes before TMEM is released
    if (lane == 0) mma_commit(&sm.mma_done);
    __syncwarp();
    mbar_wait_quiet(&sm.mma_done, 0);
    __syncwarp();
  } else {
    // ======================= softmax + epilogue (warps 0-3) =======================
    const int r = tid;           // row of the unit == TMEM lane
    const int blk = r >> 6;      // which of the two query blocks
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = kLog2e * rsqrtf(static_cast<float>(D));
    const int nlast = P.N - (P.NB - 1) * kBN;
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
      bool ok = true;
      for (int t = 0; t < T; ++t) {
        const uint32_t gt = g + t, b = gt & 1, use = gt >> 1;
        const uint32_t entry = ROUTE ? sm.list[s][t] : (static_cast<uint32_t>(t) | 0xC000u);
        const int j = entry & 0x3FFF;
        const bool mine = (entry >> (14 + blk)) & 1u;  // warp-uniform
        if (!warp_wait(&sm.s_full[b], use & 1, abort_flag, st, kSiteSFull, u)) { ok = false; break; }
        tc_fence_after();
        uint32_t sv[32], sw[32];  // S columns 0-31 and 32-63 of this row
        if (mine) {
          tmem_ld32(tmem + kColS + b * 64 + lane_off, sv);
          tmem_ld32(tmem + kColS + b * 64 + 32 + lane_off, sw);
          tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_free[b]);
        uint32_t pw[32];
        float rescale = 1.f;
        bool need = false;
        if (mine) {
          const int nv = (j == P.NB - 1) ? nlast : kBN;
          float mx = -INFINITY;
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            mx = fmaxf(mx, c < nv ? __uint_as_float(sv[c]) : -INFINITY);
            mx = fmaxf(mx, c + 32 < nv ? __uint_as_float(sw[c]) : -INFINITY);
          }
          mx *= sl2;
          if (mx > m + kRescaleSlack) {
            if (m != -INFINITY) {
              need = true;
              rescale = ex2_approx(m - mx);
              l *= rescale;
            }
            m = mx;
          }
          float sum = 0.f;
#pragma unroll
          for (int c = 0; c < 32; c += 2) {
            const float p0 = c < nv ? ex2_approx(fmaf(__uint_as_float(sv[c]), sl2, -m)) : 0.f;
            const float p1 = c + 1 < nv ? ex2_approx(fmaf(__uint_as_float(sv[c + 1]), sl2, -m)) : 0.f;
            const float p2 = c + 32 < nv ? ex2_approx(fmaf(__uint_as_float(sw[c]), sl2, -m)) : 0.f;
            const float p3 = c + 33 < nv ? ex2_approx(fmaf(__uint_as_float(sw[c + 1]), sl2, -m)) : 0.f;
            sum += (p0 + p1) + (p2 + p3);
            pw[c / 2] = pack_bf16x2(p0, p1);
            pw[16 + c / 2] = pack_bf16x2(p2, p3);
          }
          l += sum;
        } else {
#pragma unroll
          for (int c = 0; c < 32; ++c) pw[c] = 0u;
        }
        // PV of the previous tile must be complete: its P buffer and O are touched next
        if (t >= 1 && !warp_wait(&sm.o_full, (gt - 1) & 1, abort_flag, st, kSiteOFull, u)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll
          for (int ch = 0; ch < D / 32; ++ch) {
            uint32_t ov[32];
            tmem_ld32(tmem + kColO + ch * 32 + lane_off, ov);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 32; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * rescale);
            tmem_st32(tmem + kColO + ch * 32 + lane_off, ov);
          }
        }
        tmem_st32(tmem + kColP + b * 32 + lane_off, pw);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[b]);
      }
      if (!ok) break;
      // ---------------- epilogue ----------------
      if (T >= 1) {
        if (!warp_wait(&sm.o_full, (g + T - 1) & 1, abort_flag, st, kSiteOFull, u)) break;
        tc_fence_after();
      }
      const float mc = sm.cmax[s][blk] * kLog2e;
      const float cd = sm.cden[s][blk];
      const float mf = fmaxf(m, mc);
      const float a = (m == -INFINITY) ? 0.f : ex2_approx(m - mf);
      const float c = (mc == -INFINITY) ? 0.f : ex2_approx(mc - mf);
      const float L = fmaf(l, a, cd * c);
      const float inv = 1.f / L;
      const int row = pair * kBM + r;
      const bool valid = row < P.N;
      uint16_t* orow = P.out + (static_cast<long long>(bh) * P.N + row) * D;
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t ov[32];
        if (T >= 1) {
          tmem_ld32(tmem + kColO + ch * 32 + lane_off, ov);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) ov[e] = 0u;
        }
        uint32_t packed[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float y0, y1;
          if constexpr (ROUTE) {
            const float* cn = &sm.cnum[s][blk][ch * 32 + e];
            y0 = fmaf(__uint_as_float(ov[e]), a, cn[0] * c) * inv;
            y1 = fmaf(__uint_as_float(ov[e + 1]), a, cn[1] * c) * inv;
          } else {
            y0 = __uint_as_float(ov[e]) * a * inv;
            y1 = __uint_as_float(ov[e + 1]) * a * inv;
          }
          packed[e / 2] = pack_bf16x2(y0, y1);
        }
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x)
            dst[x] = make_uint4(packed[4 * x], packed[4 * x + 1], packed[4 * x + 2], packed[4 * x + 3]);
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
  if (warp == 9) {
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
  p.mu = a.pooled.mu;
  p.sigma = a.pooled.sigma;
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

cudaError_t launch_forward(const ForwardArgs& a, int num_sms, cudaStream_t stream) {
  if (a.d == 64) return a.route ? launch_fwd_t<64, true>(a, num_sms, stream) : launch_fwd_t<64, false>(a, num_sms, stream);
  return a.route ? launch_fwd_t<128, true>(a, num_sms, stream) : launch_fwd_t<128, false>(a, num_sms, stream);
}

}  // namespace solattn
