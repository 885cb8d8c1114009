// pool.cu -- pooled statistics for Sol-Attn routing.
//
// "Sol-Attn: Accelerating Video Generation Inference via On-the-Fly Attention
// Sparsification" (paithon.it): the proxy score of (query block i, key block j)
// is the product of the block-mean query and the block-mean key ("Perché
// l'attenzione pesa tanto nei video"), and each row's mean and standard
// deviation come from the mean of the pooled keys and their d x d second-moment
// matrix, without forming the row ("Una soglia per ogni riga", last paragraph).
//
// Three launches:
//   pool_means_kernel  -- HBM-bound: reads q, k, v once with 128-bit loads and
//                         writes the fp32 block means (qbar, kbar, vbar).
//   key_stats_kernel   -- per head: mean of kbar and its covariance (two-pass,
//                         divided by N_b), one 64x64 tile of it per CTA.
//   row_stats_kernel   -- per query block: mu_i = s qbar_i . kmean and
//                         sigma_i = s sqrt(max(0, qbar_i^T C qbar_i)).
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
                                                         float* __restrict__ kbar, float* __restrict__ vbar, int BH,
                                                         int N, int NB) {
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
    const uint16_t* base = src + (static_cast<long long>(bh) * N + row0) * D + c * 8;
    uint4 w[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
      const int row = g + r * RG;
      w[r] = row < n ? ld_stream_v4(base + static_cast<long long>(row) * D) : make_uint4(0, 0, 0, 0);
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
      dst[(static_cast<long long>(bh) * NB + j) * D + tid] = s / static_cast<float>(n);
    }
    __syncthreads();
  }
}

// grid = (T*T, BH) with T = D/64; CTA (ta, tb) writes kcov[ta*64.., tb*64..].
template <int D>
__global__ void __launch_bounds__(256) key_stats_kernel(const float* __restrict__ kbar, float* __restrict__ kmean,
                                                        float* __restrict__ kcov, int NB) {
  constexpr int T = D / 64;
  constexpr int JC = 32;  // pooled keys staged per trip
  __shared__ float mean_part[256 / D][D];
  __shared__ float mean_s[D];
  __shared__ float da[JC][64];
  __shared__ float db[JC][64];
  const int tid = threadIdx.x;
  const int bh = blockIdx.y;
  const int ta = blockIdx.x / T, tb = blockIdx.x % T;
  const float* kb = kbar + static_cast<long long>(bh) * NB * D;
  // pass 1: mean, fixed summation order
  {
    const int col = tid % D, part = tid / D;
    float s = 0.f;
    for (int j = part; j < NB; j += 256 / D) s += kb[static_cast<long long>(j) * D + col];
    mean_part[part][col] = s;
  }
  __syncthreads();
  if (tid < D) {
    float s = 0.f;
#pragma unroll
    for (int p = 0; p < 256 / D; ++p) s += mean_part[p][tid];
    mean_s[tid] = s / static_cast<float>(NB);
    if (blockIdx.x == 0) kmean[static_cast<long long>(bh) * D + tid] = mean_s[tid];
  }
  __syncthreads();
  // pass 2: covariance tile from deviations
  const int a0 = (tid / 16) * 4, b0 = (tid % 16) * 4;
  float acc[4][4];
#pragma unroll
  for (int x = 0; x < 4; ++x)
#pragma unroll
    for (int y = 0; y < 4; ++y) acc[x][y] = 0.f;
  for (int j0 = 0; j0 < NB; j0 += JC) {
    for (int e = tid; e < JC * 64; e += 256) {
      const int jj = e / 64, cc = e % 64, j = j0 + jj;
      const bool ok = j < NB;
      da[jj][cc] = ok ? kb[static_cast<long long>(j) * D + ta * 64 + cc] - mean_s[ta * 64 + cc] : 0.f;
      db[jj][cc] = ok ? kb[static_cast<long long>(j) * D + tb * 64 + cc] - mean_s[tb * 64 + cc] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int jj = 0; jj < JC; ++jj) {
      float av[4], bv[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) av[x] = da[jj][a0 + x];
#pragma unroll
      for (int y = 0; y < 4; ++y) bv[y] = db[jj][b0 + y];
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(av[x], bv[y], acc[x][y]);
    }
    __syncthreads();
  }
  const float inv = 1.f / static_cast<float>(NB);
  float* out = kcov + static_cast<long long>(bh) * D * D;
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    float4 r = make_float4(acc[x][0] * inv, acc[x][1] * inv, acc[x][2] * inv, acc[x][3] * inv);
    *reinterpret_cast<float4*>(out + static_cast<long long>(ta * 64 + a0 + x) * D + tb * 64 + b0) = r;
  }
}

// grid = (chunks, BH), 256 threads = 8 warps; dynamic smem holds C (D*D fp32).
template <int D>
__global__ void __launch_bounds__(256) row_stats_kernel(const float* __restrict__ qbar,
                                                        const float* __restrict__ kmean,
                                                        const float* __restrict__ kcov, float* __restrict__ mu,
                                                        float* __restrict__ sigma, int NB) {
  extern __shared__ __align__(16) float smem_f[];
  float* C = smem_f;            // [D][D]
  float* km = C + D * D;        // [D]
  float* qs = km + D;           // [8][D]
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int bh = blockIdx.y;
  const float* cg = kcov + static_cast<long long>(bh) * D * D;
  for (int e = tid; e < D * D / 4; e += 256)
    reinterpret_cast<float4*>(C)[e] = reinterpret_cast<const float4*>(cg)[e];
  if (tid < D) km[tid] = kmean[static_cast<long long>(bh) * D + tid];
  __syncthreads();
  const float s = rsqrtf(static_cast<float>(D));
  constexpr int M = D / 32;
  for (int i = blockIdx.x * 8 + warp; i < NB; i += gridDim.x * 8) {
    const float* qg = qbar + (static_cast<long long>(bh) * NB + i) * D;
    float qv[M];
#pragma unroll
    for (int m = 0; m < M; ++m) {
      qv[m] = qg[lane + 32 * m];
      qs[warp * D + lane + 32 * m] = qv[m];
    }
    __syncwarp();
    float y[M];
#pragma unroll
    for (int m = 0; m < M; ++m) y[m] = 0.f;
    for (int b = 0; b < D; ++b) {
      const float qb = qs[warp * D + b];
#pragma unroll
      for (int m = 0; m < M; ++m) y[m] = fmaf(C[b * D + lane + 32 * m], qb, y[m]);  // C symmetric
    }
    float quad = 0.f, dot = 0.f;
#pragma unroll
    for (int m = 0; m < M; ++m) {
      quad = fmaf(qv[m], y[m], quad);
      dot = fmaf(qv[m], km[lane + 32 * m], dot);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      quad += __shfl_xor_sync(0xffffffffu, quad, off);
      dot += __shfl_xor_sync(0xffffffffu, dot, off);
    }
    if (lane == 0) {
      mu[static_cast<long long>(bh) * NB + i] = s * dot;
      sigma[static_cast<long long>(bh) * NB + i] = s * sqrtf(fmaxf(quad, 0.f));
    }
    __syncwarp();
  }
}

template <int D>
cudaError_t launch_pool_d(const uint16_t* q, const uint16_t* k, const uint16_t* v, const PooledPtrs& p, int BH,
                          int N, int num_sms, cudaStream_t stream) {
  const int NB = (N + kBlock - 1) / kBlock;
  const long long items = 3ll * BH * NB;
  const int grid1 = static_cast<int>(items < num_sms * 8ll ? items : num_sms * 8ll);
  pool_means_kernel<D><<<grid1, 256, 0, stream>>>(q, k, v, p.qbar, p.kbar, p.vbar, BH, N, NB);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  constexpr int T = D / 64;
  key_stats_kernel<D><<<dim3(T * T, BH), 256, 0, stream>>>(p.kbar, p.kmean, p.kcov, NB);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = (static_cast<size_t>(D) * D + D + 8 * D) * sizeof(float);
  e = cudaFuncSetAttribute(row_stats_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int chunks = (NB + 63) / 64;  // 64 query blocks per CTA
  row_stats_kernel<D><<<dim3(chunks, BH), 256, smem, stream>>>(p.qbar, p.kmean, p.kcov, p.mu, p.sigma, NB);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool(const uint16_t* q, const uint16_t* k, const uint16_t* v, const PooledPtrs& p, int BH,
                        int N, int d, int num_sms, cudaStream_t stream) {
  if (d == 64) return launch_pool_d<64>(q, k, v, p, BH, N, num_sms, stream);
  return launch_pool_d<128>(q, k, v, p, BH, N, num_sms, stream);
}

}  // namespace solattn
