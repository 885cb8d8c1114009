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
//                         divided by N_b), one 32x32 tile (and its mirror) per CTA.
//   row_stats_kernel   -- per query block: mu_i = s qbar_i . kmean and
//                         sigma_i = s sqrt(max(0, qbar_i^T C qbar_i)), 64 blocks per CTA.
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

// Covariance of the pooled keys, two-pass. grid = (number of 32x32 tiles on or
// above the diagonal, BH); CTA (ta <= tb) computes tile (ta, tb) and writes it
// and its mirror (tb, ta). Pass 1: mean of the 64 columns it needs (fixed
// order); pass 2: sum over key blocks of the deviations' outer products, 64
// key blocks staged in shared memory per trip.
template <int D>
__global__ void __launch_bounds__(256) key_stats_kernel(const float* __restrict__ kbar, float* __restrict__ kmean,
                                                        float* __restrict__ kcov, int NB) {
  constexpr int T = D / 32;
  constexpr int JC = 128;
  __shared__ float mpart[8][64];
  __shared__ float mcol[64];        // means of columns ta*32.. (0-31) and tb*32.. (32-63)
  __shared__ float da[JC][33];      // deviations, padded against bank conflicts
  __shared__ __align__(16) float db[JC][32];
  const int tid = threadIdx.x;
  const int bh = blockIdx.y;
  int ta = 0, tb = 0;
  {  // blockIdx.x -> (ta, tb), ta <= tb, row-major over the upper triangle
    int rem = blockIdx.x;
    for (ta = 0; ta < T; ++ta) {
      if (rem < T - ta) { tb = ta + rem; break; }
      rem -= T - ta;
    }
  }
  const float* kb = kbar + static_cast<long long>(bh) * NB * D;
  {
    // 4 partial sums per column, each over rows part, part + 4, ...; 8
    // independent accumulators keep 8 loads in flight (fixed summation order)
    const int c = tid % 64, part = tid / 64;
    const int col = c < 32 ? ta * 32 + c : tb * 32 + (c - 32);
    float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int j = part;
    for (; j + 28 < NB; j += 32) {
#pragma unroll
      for (int u = 0; u < 8; ++u) acc8[u] += kb[static_cast<long long>(j + 4 * u) * D + col];
    }
    for (int u = 0; j < NB; j += 4, ++u) acc8[u & 7] += kb[static_cast<long long>(j) * D + col];
    mpart[part][c] = ((acc8[0] + acc8[1]) + (acc8[2] + acc8[3])) + ((acc8[4] + acc8[5]) + (acc8[6] + acc8[7]));
  }
  __syncthreads();
  if (tid < 64) {
    mcol[tid] = ((mpart[0][tid] + mpart[1][tid]) + (mpart[2][tid] + mpart[3][tid])) / static_cast<float>(NB);
    if (ta == tb && tid < 32) kmean[static_cast<long long>(bh) * D + ta * 32 + tid] = mcol[tid];
  }
  __syncthreads();
  const int a = tid / 8, b0 = (tid % 8) * 4;  // this thread: row a, columns b0..b0+3 of the tile
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int j0 = 0; j0 < NB; j0 += JC) {
    for (int e = tid; e < JC * 32; e += 256) {
      const int jj = e / 32, cc = e % 32, j = j0 + jj;
      const bool ok = j < NB;
      da[jj][cc] = ok ? kb[static_cast<long long>(j) * D + ta * 32 + cc] - mcol[cc] : 0.f;
      db[jj][cc] = ok ? kb[static_cast<long long>(j) * D + tb * 32 + cc] - mcol[32 + cc] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int jj = 0; jj < JC; ++jj) {
      const float x = da[jj][a];
      const float4 y = *reinterpret_cast<const float4*>(&db[jj][b0]);
      acc[0] = fmaf(x, y.x, acc[0]);
      acc[1] = fmaf(x, y.y, acc[1]);
      acc[2] = fmaf(x, y.z, acc[2]);
      acc[3] = fmaf(x, y.w, acc[3]);
    }
    __syncthreads();
  }
  const float inv = 1.f / static_cast<float>(NB);
  float* out = kcov + static_cast<long long>(bh) * D * D;
  const int row = ta * 32 + a, col = tb * 32 + b0;
  *reinterpret_cast<float4*>(out + static_cast<long long>(row) * D + col) =
      make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
  if (ta != tb) {
#pragma unroll
    for (int x = 0; x < 4; ++x) out[static_cast<long long>(col + x) * D + row] = acc[x] * inv;
  }
}

// mu_i = s qbar_i . kmean and sigma_i = s sqrt(max(0, qbar_i^T C qbar_i)) for 64
// query blocks per CTA: thread t owns block t / 4 and a quarter of the columns
// of y = C qbar (C symmetric), then reduces qbar . y over the 4 threads.
// grid = (ceil(NB / 64), BH); dynamic smem = C (D*D) + 64 padded qbar rows.
template <int D>
__global__ void __launch_bounds__(256) row_stats_kernel(const float* __restrict__ qbar,
                                                        const float* __restrict__ kmean,
                                                        const float* __restrict__ kcov, float* __restrict__ mu,
                                                        float* __restrict__ sigma, int NB) {
  constexpr int QS = D + 4;     // padded row stride of the staged qbar rows
  constexpr int CW = D / 4;     // columns per thread
  extern __shared__ __align__(16) float smem_f[];
  float* C = smem_f;            // [D][D]
  float* Q = C + D * D;         // [64][QS]
  float* km = Q + 64 * QS;      // [D]
  const int tid = threadIdx.x;
  const int bh = blockIdx.y;
  const int i0 = blockIdx.x * 64;
  const float* cg = kcov + static_cast<long long>(bh) * D * D;
  for (int e = tid; e < D * D / 4; e += 256)
    reinterpret_cast<float4*>(C)[e] = reinterpret_cast<const float4*>(cg)[e];
  for (int e = tid; e < 64 * D; e += 256) {
    const int r = e / D, c = e % D;
    Q[r * QS + c] = (i0 + r < NB) ? qbar[(static_cast<long long>(bh) * NB + i0 + r) * D + c] : 0.f;
  }
  if (tid < D) km[tid] = kmean[static_cast<long long>(bh) * D + tid];
  __syncthreads();
  // thread (r, c4): columns c4 * 4 + 16 m .. + 3 (m < D / 16): the four threads
  // of a row read 64 contiguous bytes of C per step (no bank conflicts)
  const int r = tid / 4, c4 = tid % 4;
  const float* qrow = Q + r * QS;
  float y[CW];
#pragma unroll
  for (int c = 0; c < CW; ++c) y[c] = 0.f;
#pragma unroll 4
  for (int k = 0; k < D; ++k) {
    const float qk = qrow[k];
    const float* crow = C + k * D + c4 * 4;
#pragma unroll
    for (int m = 0; m < CW / 4; ++m) {
      const float4 cv = *reinterpret_cast<const float4*>(crow + 16 * m);
      y[4 * m] = fmaf(qk, cv.x, y[4 * m]);
      y[4 * m + 1] = fmaf(qk, cv.y, y[4 * m + 1]);
      y[4 * m + 2] = fmaf(qk, cv.z, y[4 * m + 2]);
      y[4 * m + 3] = fmaf(qk, cv.w, y[4 * m + 3]);
    }
  }
  float quad = 0.f, dot = 0.f;
#pragma unroll
  for (int m = 0; m < CW / 4; ++m) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int c = c4 * 4 + 16 * m + e;
      quad = fmaf(qrow[c], y[4 * m + e], quad);
      dot = fmaf(qrow[c], km[c], dot);
    }
  }
  quad += __shfl_xor_sync(0xffffffffu, quad, 1);
  dot += __shfl_xor_sync(0xffffffffu, dot, 1);
  quad += __shfl_xor_sync(0xffffffffu, quad, 2);
  dot += __shfl_xor_sync(0xffffffffu, dot, 2);
  const int i = i0 + r;
  if ((tid % 4) == 0 && i < NB) {
    const float s = rsqrtf(static_cast<float>(D));
    mu[static_cast<long long>(bh) * NB + i] = s * dot;
    sigma[static_cast<long long>(bh) * NB + i] = s * sqrtf(fmaxf(quad, 0.f));
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
  constexpr int T = D / 32;
  key_stats_kernel<D><<<dim3(T * (T + 1) / 2, BH), 256, 0, stream>>>(p.kbar, p.kmean, p.kcov, NB);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = (static_cast<size_t>(D) * D + 64 * (D + 4) + D) * sizeof(float);
  e = cudaFuncSetAttribute(row_stats_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  row_stats_kernel<D><<<dim3((NB + 63) / 64, BH), 256, smem, stream>>>(p.qbar, p.kmean, p.kcov, p.mu, p.sigma, NB);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool(const uint16_t* q, const uint16_t* k, const uint16_t* v, const PooledPtrs& p, int BH,
                        int N, int d, int num_sms, cudaStream_t stream) {
  if (d == 64) return launch_pool_d<64>(q, k, v, p, BH, N, num_sms, stream);
  return launch_pool_d<128>(q, k, v, p, BH, N, num_sms, stream);
}

}  // namespace solattn
