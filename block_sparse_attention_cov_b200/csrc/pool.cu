// pool.cu -- pooled statistics for Sol-Attn routing.
//
// "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly Attention
// Sparsification" (paithon.it): the proxy score of (query block i, key block j)
// is the product of the block-mean query and the block-mean key ("Perché
// l'attenzione pesa tanto nei video"), and each row's mean and standard
// deviation come from the mean of the pooled keys and their d x d second-moment
// matrix, without forming the row ("Una soglia per ogni riga", last paragraph).
//
// Two launches:
//   pool_means_kernel  -- HBM-bound: reads q, k, v once with 128-bit loads and
//                         writes the fp32 block means (qbar, kbar, vbar).
//   key_stats_kernel   -- per head: mean of kbar and its covariance (two-pass,
//                         divided by N_b), one cluster of CTAs per head.
// The per-row statistics mu_i, sigma_i are evaluated by the forward kernel's
// routing warps from kmean and kcov.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "kernels.h"

namespace solattn {

namespace {

constexpr int kBlock = 64;

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4 w) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] += __uint_as_float(u[i] << 16);
    acc[2 * i + 1] += __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// One CTA (256 threads) reduces one 64-token block of one tensor per loop trip.
// Thread t owns 8 consecutive columns (chunk t % (D/8)) of the rows
// t / (D/8) + k * (256 / (D/8)). A warp therefore reads whole rows: coalesced.
template <int D>
__global__ void __launch_bounds__(256) pool_means_kernel(const uint16_t* __restrict__ q,
                                                         const uint16_t* __restrict__ k,
                                                         const uint16_t* __restrict__ v, float* __restrict__ qbar,
                                                         float* __restrict__ kbar, float* __restrict__ vbar,
                                                         uint16_t* __restrict__ kbar16, uint16_t* __restrict__ vbar16,
                                                         int BH, int H, int N, int NB, Strides st) {
  constexpr int CH = D / 8;       // 16-byte chunks per row
  constexpr int RG = 256 / CH;    // row groups
  constexpr int RPT = kBlock / RG;  // rows per thread
  __shared__ float part[8][D];
  const int tid = threadIdx.x;
  const int c = tid % CH;
  const int g = tid / CH;
  const long long items = 3ll * BH * NB;
  for (long long item = blockIdx.x; item < items; item += gridDim.x) {
    const int which = static_cast<int>(item / (static_cast<long long>(BH) * NB));
    const long long rem = item - static_cast<long long>(which) * BH * NB;
    const int bh = static_cast<int>(rem / NB);
    const int j = static_cast<int>(rem - static_cast<long long>(bh) * NB);
    const uint16_t* src = which == 0 ? q : (which == 1 ? k : v);
    float* dst = which == 0 ? qbar : (which == 1 ? kbar : vbar);
    const int row0 = j * kBlock;
    const int n = min(kBlock, N - row0);
    const uint16_t* base = src + (bh / H) * st.b + (bh % H) * st.h + static_cast<long long>(row0) * st.n + c * 8;
    uint4 w[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const int row = g + r * RG;
      w[r] = row < n ? ld_stream_v4(base + static_cast<long long>(row) * st.n) : make_uint4(0, 0, 0, 0);
    }
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int r = 0; r < RPT; ++r) add_bf16x8(acc, w[r]);
    // lanes with the same chunk inside a warp: lane % CH equal
#pragma unroll
    for (int off = CH; off < 32; off <<= 1) {
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    }
    const int warp = tid / 32, lane = tid % 32;
    if (lane < CH) {
#pragma unroll
      for (int e = 0; e < 8; ++e) part[warp][lane * 8 + e] = acc[e];
    }
    __syncthreads();
    if (tid < D) {
      float s = 0.f;
#pragma unroll
      for (int w8 = 0; w8 < 8; ++w8) s += part[w8][tid];
      const float mean = s / static_cast<float>(n);
      const long long o = (static_cast<long long>(bh) * NB + j) * D + tid;
      dst[o] = mean;
      if (which > 0) {  // bf16 copies of the pooled keys / values (round to nearest even)
        uint16_t* d16 = which == 1 ? kbar16 : vbar16;
        d16[o] = static_cast<uint16_t>(__bfloat16_as_ushort(__float2bfloat16_rn(mean)));
      }
    }
    __syncthreads();
  }
}

// Mean and covariance of the pooled keys of one head, two-pass, by a cluster of
// kSplit CTAs (one per contiguous slice of key blocks), 256 threads each:
//   1. every CTA sums its slice's columns; the cluster exchanges the kSplit
//      partial sums through distributed shared memory and every CTA forms the
//      same mean (fixed order);
//   2. every CTA accumulates the outer products of its slice's deviations
//      (kbar_j - mean) into a D x D partial, staged 32 key blocks at a time;
//   3. CTA r adds the kSplit partials of rows r*D/kSplit.. in rank order and
//      writes them divided by N_b. The summation order is fixed: every call
//      gives the same bits.
// Thread (ta, tb) of step 2 owns rows {4 ta + e, 64 + 4 ta + e} and columns
// {4 tb + e, 64 + 4 tb + e} (D = 128; D = 64: the first set only), so the
// float4 reads of a staged row by one quarter-warp touch 128 contiguous bytes.
constexpr int kSplit = 8;   // CTAs per head (portable cluster size)
constexpr int kRows = 32;   // key blocks staged per trip

template <int D>
struct KeyStatsSmem {
  float part[D][D];         // this CTA's sum of deviation outer products
  float dev[2][kRows][D];   // staged deviations, double-buffered
  float colpart[256 / (D / 4)][D];
  float csum[D];            // this CTA's column sums (read by the whole cluster)
  float mean[D];
};

template <int D>
__global__ void __cluster_dims__(kSplit, 1, 1) __launch_bounds__(256)
    key_stats_kernel(const float* __restrict__ kbar, float* __restrict__ kmean, float* __restrict__ kcov, int NB) {
  namespace cg = cooperative_groups;
  extern __shared__ __align__(16) unsigned char ks_raw[];
  KeyStatsSmem<D>& sm = *reinterpret_cast<KeyStatsSmem<D>*>(ks_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x;
  const int rank = static_cast<int>(cluster.block_rank());
  const int bh = blockIdx.y;
  const int per = (NB + kSplit - 1) / kSplit;
  const int j0 = min(NB, rank * per), j1 = min(NB, j0 + per);
  const float* kb = kbar + static_cast<long long>(bh) * NB * D;

  // ---- 1. column sums of the slice, then the head mean
  {
    constexpr int C4 = D / 4, RL = 256 / C4;
    const int c4 = tid % C4, rl = tid / C4;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    int j = j0 + rl;
    for (; j + RL < j1; j += 2 * RL) {
      const float4 x = __ldg(reinterpret_cast<const float4*>(kb + static_cast<long long>(j) * D) + c4);
      const float4 y = __ldg(reinterpret_cast<const float4*>(kb + static_cast<long long>(j + RL) * D) + c4);
      a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
      b.x += y.x; b.y += y.y; b.z += y.z; b.w += y.w;
    }
    if (j < j1) {
      const float4 x = __ldg(reinterpret_cast<const float4*>(kb + static_cast<long long>(j) * D) + c4);
      a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
    }
    *reinterpret_cast<float4*>(&sm.colpart[rl][c4 * 4]) = make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
    __syncthreads();
    if (tid < D) {
      float t = 0.f;
#pragma unroll
      for (int r = 0; r < RL; ++r) t += sm.colpart[r][tid];
      sm.csum[tid] = t;
    }
  }
  cluster.sync();
  if (tid < D) {
    float t = 0.f;
    for (int r = 0; r < kSplit; ++r) t += cluster.map_shared_rank(sm.csum, r)[tid];
    sm.mean[tid] = t / static_cast<float>(NB);
  }
  __syncthreads();

  // ---- 2. sum of the deviations' outer products over the slice
  constexpr int TT = D / 16;  // rows (and columns) per thread: 8 or 4
  const int ta = tid / 16, tb = tid % 16;
  float acc[TT][TT];
#pragma unroll
  for (int x = 0; x < TT; ++x)
#pragma unroll
    for (int y = 0; y < TT; ++y) acc[x][y] = 0.f;
  // staged through registers: the next 32 key blocks are in flight while the
  // current ones are multiplied
  constexpr int PER = kRows * D / 4 / 256;  // float4 per thread per stage
  float4 pre[PER];
  auto fetch = [&](int c0) {
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = tid + 256 * i, r = e / (D / 4), c = (e % (D / 4)) * 4;
      pre[i] = (c0 + r < j1) ? __ldg(reinterpret_cast<const float4*>(kb + static_cast<long long>(c0 + r) * D + c))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  if (j0 < j1) fetch(j0);
  for (int c0 = j0, it = 0; c0 < j1; c0 += kRows, ++it) {
    const int nr = min(kRows, j1 - c0);
    float (*dv)[D] = sm.dev[it & 1];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = tid + 256 * i, r = e / (D / 4), c = (e % (D / 4)) * 4;
      float4 x = pre[i];
      if (r < nr) {
        x.x -= sm.mean[c]; x.y -= sm.mean[c + 1]; x.z -= sm.mean[c + 2]; x.w -= sm.mean[c + 3];
      }
      *reinterpret_cast<float4*>(&dv[r][c]) = x;  // rows past the slice stay zero
    }
    __syncthreads();
    if (c0 + kRows < j1) fetch(c0 + kRows);
    for (int r = 0; r < nr; ++r) {
      float av[TT], bv[TT];
#pragma unroll
      for (int h = 0; h < TT / 4; ++h) {
        const float4 x = *reinterpret_cast<const float4*>(&dv[r][64 * h + 4 * ta]);
        const float4 y = *reinterpret_cast<const float4*>(&dv[r][64 * h + 4 * tb]);
        av[4 * h] = x.x; av[4 * h + 1] = x.y; av[4 * h + 2] = x.z; av[4 * h + 3] = x.w;
        bv[4 * h] = y.x; bv[4 * h + 1] = y.y; bv[4 * h + 2] = y.z; bv[4 * h + 3] = y.w;
      }
#pragma unroll
      for (int x = 0; x < TT; ++x)
#pragma unroll
        for (int y = 0; y < TT; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
    }
  }
#pragma unroll
  for (int x = 0; x < TT; ++x) {
    const int row = 64 * (x / 4) + 4 * ta + x % 4;
#pragma unroll
    for (int h = 0; h < TT / 4; ++h)
      *reinterpret_cast<float4*>(&sm.part[row][64 * h + 4 * tb]) =
          make_float4(acc[x][4 * h], acc[x][4 * h + 1], acc[x][4 * h + 2], acc[x][4 * h + 3]);
  }
  cluster.sync();

  // ---- 3. rows rank * D / kSplit .. of the covariance: partials in rank order
  {
    constexpr int R = D / kSplit;          // rows per CTA: 16 or 8
    constexpr int V4 = R * D / 4 / 256;    // float4 per thread: 2 or 1 (D = 64: 128 threads idle)
    const float inv = 1.f / static_cast<float>(NB);
    float* out = kcov + static_cast<long long>(bh) * D * D + static_cast<long long>(rank) * R * D;
#pragma unroll
    for (int v = 0; v < (V4 > 0 ? V4 : 1); ++v) {
      const int e = tid + 256 * v;
      if (e < R * D / 4) {
        const int row = rank * R + e / (D / 4), c = (e % (D / 4)) * 4;
        float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < kSplit; ++r) {
          const float4 y = *reinterpret_cast<const float4*>(&cluster.map_shared_rank(&sm.part[0][0], r)[row * D + c]);
          t.x += y.x; t.y += y.y; t.z += y.z; t.w += y.w;
        }
        reinterpret_cast<float4*>(out)[e] = make_float4(t.x * inv, t.y * inv, t.z * inv, t.w * inv);
      }
    }
    if (rank == 0 && tid < D) kmean[static_cast<long long>(bh) * D + tid] = sm.mean[tid];
  }
  cluster.sync();  // no CTA leaves while another still reads its shared memory
}

template <int D>
cudaError_t launch_pool_d(const uint16_t* q, const uint16_t* k, const uint16_t* v, const PooledPtrs& p, int BH,
                          int H, int N, const Strides& st, int num_sms, cudaStream_t stream) {
  const int NB = (N + kBlock - 1) / kBlock;
  const long long items = 3ll * BH * NB;
  const int grid1 = static_cast<int>(items < num_sms * 8ll ? items : num_sms * 8ll);
  pool_means_kernel<D><<<grid1, 256, 0, stream>>>(q, k, v, p.qbar, p.kbar, p.vbar, p.kbar16, p.vbar16, BH, H, N,
                                                   NB, st);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int smem = static_cast<int>(sizeof(KeyStatsSmem<D>));
  e = cudaFuncSetAttribute(key_stats_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  key_stats_kernel<D><<<dim3(kSplit, BH), 256, smem, stream>>>(p.kbar, p.kmean, p.kcov, NB);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool(const uint16_t* q, const uint16_t* k, const uint16_t* v, const PooledPtrs& p, int BH,
                        int H, int N, int d, const Strides& st, int num_sms, cudaStream_t stream) {
  if (d == 64) return launch_pool_d<64>(q, k, v, p, BH, H, N, st, num_sms, stream);
  return launch_pool_d<128>(q, k, v, p, BH, H, N, st, num_sms, stream);
}

}  // namespace solattn
