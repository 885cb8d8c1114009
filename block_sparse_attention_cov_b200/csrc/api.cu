// api.cu -- the C ABI declared in include/solattn.h: argument checks, buffer
// layout helpers and stream-ordered launches. No allocation happens here.
#include <cuda_runtime.h>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/solattn.h"
#include "kernels.h"
#include "ptx.cuh"

namespace {

#ifdef SOLATTN_TEST_HOOKS
bool g_force_one_unit = false;  // test builds: run every forward on the one-unit kernel
#endif

using solattn::DeviceStatus;
using solattn::PooledPtrs;

static_assert(sizeof(DeviceStatus) <= SOLATTN_WORKSPACE_BYTES, "workspace too small for the status block");

constexpr int kMaxDevices = 64;
// Multiprocessor count per device: 0 = not yet queried, -1 = not an sm_100
// device. Filled lazily; concurrent first calls may both query the device and
// store the same value, which the atomic makes well defined.
std::atomic<int> g_sms[kMaxDevices];

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

int check_shape(int B, int H, int N, int d) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0) return SOLATTN_ERR_ARG;
  if (d != 64 && d != 128) return SOLATTN_ERR_UNSUPPORTED;
  if (N > SOLATTN_MAX_TOKENS) return SOLATTN_ERR_UNSUPPORTED;
  const long long bh = static_cast<long long>(B) * H;
  const long long nb = (N + SOLATTN_BLOCK - 1) / SOLATTN_BLOCK;
  if (bh * ((nb + 1) / 2) >= (1ll << 31) || bh >= (1ll << 31)) return SOLATTN_ERR_UNSUPPORTED;
  return SOLATTN_OK;
}

int check_qkv(const void* q, const void* k, const void* v) {
  if (!q || !k || !v) return SOLATTN_ERR_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return SOLATTN_ERR_ALIGN;
  return SOLATTN_OK;
}

int check_pooled(const solattn_pooled_t* p) {
  if (!p) return SOLATTN_ERR_ARG;
  const void* ptrs[7] = {p->qbar, p->kbar, p->vbar, p->kmean, p->kcov, p->kbar16, p->vbar16};
  for (const void* x : ptrs)
    if (!x) return SOLATTN_ERR_ARG;
  for (const void* x : ptrs)
    if (!aligned16(x)) return SOLATTN_ERR_ALIGN;
  return SOLATTN_OK;
}

// Multiprocessor count of the current device, or an error code (negative).
int current_device_sms(int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SOLATTN_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SOLATTN_ERR_DEVICE;
  int n = g_sms[dev].load(std::memory_order_acquire);
  if (n == 0) {
    int major = 0, minor = 0, count = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return SOLATTN_ERR_CUDA;
    n = (major == 10 && minor == 0) ? count : -1;
    g_sms[dev].store(n, std::memory_order_release);
  }
  if (n < 0) return SOLATTN_ERR_DEVICE;
  *sms = n;
  return SOLATTN_OK;
}

// Strides of q, k, v, out: all zero means contiguous [B][H][N][d]; otherwise
// every stride a multiple of 8 elements (16 bytes: 128-bit loads, TMA), the
// token stride at least d, and the head (batch) stride non-zero when there is
// more than one head (batch): out shares these strides, and two heads writing
// the same rows would race.
int resolve_strides(const solattn_strides_t* in, int B, int H, int N, int d, solattn::Strides* out) {
  if (!in || (in->batch == 0 && in->head == 0 && in->token == 0)) {
    *out = solattn::Strides{static_cast<long long>(H) * N * d, static_cast<long long>(N) * d, d};
    return SOLATTN_OK;
  }
  if (in->batch < 0 || in->head < 0 || in->token < d) return SOLATTN_ERR_ARG;
  if ((H > 1 && in->head == 0) || (B > 1 && in->batch == 0)) return SOLATTN_ERR_ARG;
  if ((in->batch | in->head | in->token) & 7) return SOLATTN_ERR_ARG;
  *out = solattn::Strides{in->batch, in->head, in->token};
  return SOLATTN_OK;
}

PooledPtrs to_ptrs(const solattn_pooled_t* p) {
  return PooledPtrs{p->qbar, p->kbar, p->vbar, p->kmean, p->kcov, static_cast<uint16_t*>(p->kbar16),
                    static_cast<uint16_t*>(p->vbar16)};
}

// reset_status: false leaves the status word as it is (only the scheduler
// counter restarts), so that a sequence of calls keeps the first error.
int run_forward(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                const solattn_pooled_t* pooled, const solattn_options_t& opt, bool route, void* out, float* lse,
                int32_t* density, void* workspace, size_t workspace_bytes, void* stream, bool reset_status = true) {
  const float beta = opt.beta;
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if ((rc = check_qkv(q, k, v))) return rc;
  if (!out) return SOLATTN_ERR_ARG;
  if (!aligned16(out)) return SOLATTN_ERR_ALIGN;
  if ((lse && !aligned4(lse)) || (density && !aligned4(density))) return SOLATTN_ERR_ALIGN;
  solattn::Strides strides;
  if ((rc = resolve_strides(&opt.strides, B, H, N, d, &strides))) return rc;
  if (route) {
    if (std::isnan(beta) || std::isnan(opt.topp) || opt.n_forced < 0) return SOLATTN_ERR_ARG;
    if (opt.rule != SOLATTN_RULE_THRESHOLD && opt.rule != SOLATTN_RULE_TOPK && opt.rule != SOLATTN_RULE_TOPP)
      return SOLATTN_ERR_ARG;
    if (opt.correction != 0 && opt.correction != 1) return SOLATTN_ERR_ARG;
    if ((rc = check_pooled(pooled))) return rc;
  }
  if (!workspace || workspace_bytes < SOLATTN_WORKSPACE_BYTES) return SOLATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return SOLATTN_ERR_ALIGN;
  int sms = 0;
  if ((rc = current_device_sms(&sms))) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the scheduler counter (and, normally, the status word) start at zero
  if (cudaMemsetAsync(workspace, 0, reset_status ? sizeof(DeviceStatus) : sizeof(unsigned int), s) != cudaSuccess)
    return SOLATTN_ERR_CUDA;
  solattn::ForwardArgs a{};
  a.q = static_cast<const uint16_t*>(q);
  a.k = static_cast<const uint16_t*>(k);
  a.v = static_cast<const uint16_t*>(v);
  a.out = static_cast<uint16_t*>(out);
  a.lse = lse;
  a.density = route ? density : nullptr;
  if (route) a.pooled = to_ptrs(pooled);
  a.beta = beta;
  a.rule = route ? opt.rule : SOLATTN_RULE_THRESHOLD;
  a.topk = opt.topk;
  a.topp = opt.topp;
  a.n_forced = route ? opt.n_forced : 0;
  a.token_corr = route ? opt.correction : 0;
  a.route = route;
  a.BH = B * H;
  a.H = H;
  a.N = N;
  a.d = d;
  a.st = strides;
  a.status = workspace;
  // the threshold rule with the block-level correction (the method) and the
  // dense path run on the two-group kernel (forward_pp.cu); the ablation rules
  // and the per-token correction on the one-unit kernel (forward.cu)
  bool pp = a.rule == SOLATTN_RULE_THRESHOLD && a.token_corr == 0;
#ifdef SOLATTN_TEST_HOOKS
  if (g_force_one_unit) pp = false;
#endif
  const cudaError_t e = pp ? solattn::launch_forward_pp(a, sms, s) : solattn::launch_forward(a, sms, s);
  return e == cudaSuccess ? SOLATTN_OK : SOLATTN_ERR_CUDA;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

int run_pool(const void* q, const void* k, const void* v, int B, int H, int N, int d,
             const solattn_strides_t* strides, const solattn_pooled_t* pooled, void* stream) {
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  solattn::Strides st;
  if ((rc = resolve_strides(strides, B, H, N, d, &st))) return rc;
  if ((rc = check_qkv(q, k, v))) return rc;
  if ((rc = check_pooled(pooled))) return rc;
  int sms = 0;
  if ((rc = current_device_sms(&sms))) return rc;
  const cudaError_t e =
      solattn::launch_pool(static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(k),
                           static_cast<const uint16_t*>(v), to_ptrs(pooled), B * H, H, N, d, st, sms,
                           static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SOLATTN_OK : SOLATTN_ERR_CUDA;
}

}  // namespace

extern "C" {

int solattn_version(void) { return 10000; }

const char* solattn_strerror(int code) {
  switch (code) {
    case SOLATTN_OK: return "ok";
    case SOLATTN_ERR_ARG: return "invalid argument (null pointer, non-positive size or NaN beta)";
    case SOLATTN_ERR_UNSUPPORTED: return "unsupported shape (d must be 64 or 128, N <= 262144)";
    case SOLATTN_ERR_ALIGN: return "device pointer not aligned (16 bytes for tensors, 4 for lse/density)";
    case SOLATTN_ERR_CUDA: return "CUDA runtime error";
    case SOLATTN_ERR_TIMEOUT: return "a bounded wait inside the kernel expired; outputs are invalid";
    case SOLATTN_ERR_DEVICE: return "current device is not an sm_100 (B200-class) GPU";
    case SOLATTN_ERR_WORKSPACE: return "workspace missing or smaller than SOLATTN_WORKSPACE_BYTES";
    case SOLATTN_ERR_SCRATCH: return "problem too large for the static scratch of solattn_forward_noalloc";
    default: return "unknown status code";
  }
}

int solattn_pooled_layout(int B, int H, int N, int d, void* base, solattn_pooled_t* pooled, size_t* bytes) {
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if (!bytes && !pooled) return SOLATTN_ERR_ARG;
  const size_t bh = static_cast<size_t>(B) * H;
  const size_t nb = (static_cast<size_t>(N) + SOLATTN_BLOCK - 1) / SOLATTN_BLOCK;
  const size_t f = sizeof(float);
  const size_t sizes[7] = {bh * nb * d * f, bh * nb * d * f, bh * nb * d * f, bh * d * f,
                           bh * static_cast<size_t>(d) * d * f, bh * nb * d * 2, bh * nb * d * 2};
  size_t off[7], total = 0;
  for (int i = 0; i < 7; ++i) {
    off[i] = total;
    total += round256(sizes[i]);
  }
  if (bytes) *bytes = total;
  if (pooled && base) {
    char* b = static_cast<char*>(base);
    if (!aligned16(base)) return SOLATTN_ERR_ALIGN;
    pooled->qbar = reinterpret_cast<float*>(b + off[0]);
    pooled->kbar = reinterpret_cast<float*>(b + off[1]);
    pooled->vbar = reinterpret_cast<float*>(b + off[2]);
    pooled->kmean = reinterpret_cast<float*>(b + off[3]);
    pooled->kcov = reinterpret_cast<float*>(b + off[4]);
    pooled->kbar16 = b + off[5];
    pooled->vbar16 = b + off[6];
  } else if (pooled && !base) {
    return SOLATTN_ERR_ARG;
  }
  return SOLATTN_OK;
}

int solattn_pool(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                 const solattn_pooled_t* pooled, void* stream) {
  return solattn_pool_ex(q, k, v, B, H, N, d, nullptr, pooled, stream);
}

int solattn_pool_ex(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                    const solattn_strides_t* strides, const solattn_pooled_t* pooled, void* stream) {
  return run_pool(q, k, v, B, H, N, d, strides, pooled, stream);
}

int solattn_forward(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                    const solattn_pooled_t* pooled, float beta, void* out, float* lse, int32_t* density_out,
                    void* workspace, size_t workspace_bytes, void* stream) {
  const solattn_options_t opt{SOLATTN_RULE_THRESHOLD, beta, 0, 0.f, 0, {0, 0, 0}, 0};
  return run_forward(q, k, v, B, H, N, d, pooled, opt, true, out, lse, density_out, workspace, workspace_bytes,
                     stream);
}

int solattn_forward_ex(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                       const solattn_pooled_t* pooled, const solattn_options_t* opts, void* out, float* lse,
                       int32_t* density_out, void* workspace, size_t workspace_bytes, void* stream) {
  if (!opts) return SOLATTN_ERR_ARG;
  return run_forward(q, k, v, B, H, N, d, pooled, *opts, true, out, lse, density_out, workspace, workspace_bytes,
                     stream);
}

int solattn_dense(const void* q, const void* k, const void* v, int B, int H, int N, int d, void* out, float* lse,
                  void* workspace, size_t workspace_bytes, void* stream) {
  const solattn_options_t opt{SOLATTN_RULE_THRESHOLD, -INFINITY, 0, 0.f, 0, {0, 0, 0}, 0};
  return run_forward(q, k, v, B, H, N, d, nullptr, opt, false, out, lse, nullptr, workspace, workspace_bytes,
                     stream);
}

#ifdef SOLATTN_TEST_HOOKS
// Test builds only (libsolattn_testhooks.so; not declared in include/solattn.h):
// CTA `skip_cta` never requests its first K tile (-1: none) and every bounded
// wait gives up after `wait_budget_ns`.
int solattn_test_set_hook(int skip_cta, unsigned long long wait_budget_ns) {
  const bool ok = solattn::set_test_hooks_fwd(skip_cta, wait_budget_ns) == cudaSuccess &&
                  solattn::set_test_hooks_pp(skip_cta, wait_budget_ns) == cudaSuccess;
  return ok ? SOLATTN_OK : SOLATTN_ERR_CUDA;
}

// Test builds only: every later forward copies its units' kept bitmaps to `mask`
// ([B*H][N_b][ceil(N_b / 32)] uint32, bit j % 32 of word j / 32 = key block j
// kept) and mu_i, sigma_i, tau_i to `stats` ([B*H][N_b][3] float; NaN where the
// rule does not define them). NULL, NULL switches the copy off.
// Test builds only: 1 runs every forward and dense call on the one-unit kernel
// (forward.cu), 0 restores the normal choice.
int solattn_test_force_one_unit(int on) {
  g_force_one_unit = on != 0;
  return SOLATTN_OK;
}

int solattn_test_set_route_dump(uint32_t* mask, float* stats) {
  const bool ok = solattn::set_route_dump_fwd(mask, stats) == cudaSuccess &&
                  solattn::set_route_dump_pp(mask, stats) == cudaSuccess;
  return ok ? SOLATTN_OK : SOLATTN_ERR_CUDA;
}
#endif

int solattn_status(const void* workspace, void* stream) {
  if (!workspace) return SOLATTN_ERR_WORKSPACE;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SOLATTN_ERR_CUDA;
  DeviceStatus h{};
  if (cudaMemcpy(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return SOLATTN_ERR_CUDA;
  return h.error == 0 ? SOLATTN_OK : static_cast<int>(h.error);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free forward: pooled statistics and workspace live in a static
// device array instead of caller-provided buffers.
// ---------------------------------------------------------------------------
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[SOLATTN_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kMaxDevices];  // device address of g_noalloc_scratch, per device

// Device address of the static scratch on the current device (looked up once
// per device, with that device current), or nullptr on failure.
void* noalloc_scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_addr[dev] = ptr;
  }
  return g_noalloc_addr[dev];
}

}  // namespace

extern "C" {

int solattn_forward_noalloc(const void* q, const void* k, const void* v, int B, int H, int N, int d, float beta,
                            void* out, float* lse, int32_t* density_out, void* stream) {
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if ((rc = check_qkv(q, k, v))) return rc;
  if (!out) return SOLATTN_ERR_ARG;
  if (!aligned16(out)) return SOLATTN_ERR_ALIGN;
  if ((lse && !aligned4(lse)) || (density_out && !aligned4(density_out))) return SOLATTN_ERR_ALIGN;
  if (std::isnan(beta)) return SOLATTN_ERR_ARG;
  size_t pooled_bytes = 0;
  if ((rc = solattn_pooled_layout(B, H, N, d, nullptr, nullptr, &pooled_bytes))) return rc;
  const size_t need = SOLATTN_WORKSPACE_BYTES + pooled_bytes;
  if (need > SOLATTN_NOALLOC_SCRATCH_BYTES) return SOLATTN_ERR_SCRATCH;
  int sms = 0;
  if ((rc = current_device_sms(&sms))) return rc;
  char* scratch = static_cast<char*>(noalloc_scratch_address());
  if (!scratch) return SOLATTN_ERR_CUDA;
  solattn_pooled_t pooled;
  if ((rc = solattn_pooled_layout(B, H, N, d, scratch + SOLATTN_WORKSPACE_BYTES, &pooled, nullptr))) return rc;
  if ((rc = solattn_pool(q, k, v, B, H, N, d, &pooled, stream))) return rc;
  return solattn_forward(q, k, v, B, H, N, d, &pooled, beta, out, lse, density_out, scratch,
                         SOLATTN_WORKSPACE_BYTES, stream);
}

int solattn_noalloc_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SOLATTN_ERR_CUDA;
  DeviceStatus h{};
  // the status block sits at the start of the static array; a copy from the
  // symbol allocates nothing
  if (cudaMemcpyFromSymbol(&h, g_noalloc_scratch, sizeof(h)) != cudaSuccess) return SOLATTN_ERR_CUDA;
  return h.error == 0 ? SOLATTN_OK : static_cast<int>(h.error);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// End-to-end forward on host buffers: the B*H (b, h) pairs go through the
// device in chunks, double-buffered in the caller's scratch. Three streams:
// copies to the device, the caller's stream (pool + forward), copies back;
// events order chunk i's copy in after chunk i - 2 has left the same buffer.
// ---------------------------------------------------------------------------
namespace {

struct HostChunkLayout {
  size_t q, k, v, out, lse, dens, pooled;  // offsets inside one buffer
  size_t buffer;                           // bytes of one buffer
  size_t pooled_bytes;
};

int default_chunk_heads(int BH) {
  // about 16 chunks: the copy-in of the first and the copy-back of the last
  // chunk are the only transfers not hidden behind other work
  const int c = (BH + 15) / 16;
  return c < 1 ? 1 : c;
}

int host_chunk_layout(int N, int d, int C, HostChunkLayout* L) {
  size_t pooled_bytes = 0;
  int rc = solattn_pooled_layout(1, C, N, d, nullptr, nullptr, &pooled_bytes);
  if (rc) return rc;
  const size_t nb = (static_cast<size_t>(N) + SOLATTN_BLOCK - 1) / SOLATTN_BLOCK;
  const size_t tensor = static_cast<size_t>(C) * N * d * 2;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += round256(bytes);
    return at;
  };
  L->q = take(tensor);
  L->k = take(tensor);
  L->v = take(tensor);
  L->out = take(tensor);
  L->lse = take(static_cast<size_t>(C) * N * sizeof(float));
  L->dens = take(static_cast<size_t>(C) * nb * sizeof(int32_t));
  L->pooled = take(pooled_bytes);
  L->buffer = off;
  L->pooled_bytes = pooled_bytes;
  return SOLATTN_OK;
}

// Streams and events of one solattn_forward_host call; released at the end of
// the call (the runtime defers the release until their work has completed).
struct HostPipeline {
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t start = nullptr;
  cudaEvent_t ev[3][4] = {};  // [copied in, computed, copied back][chunk % 4]
  bool ok = true;
  HostPipeline() {
    ok = cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking) == cudaSuccess &&
         cudaStreamCreateWithFlags(&down, cudaStreamNonBlocking) == cudaSuccess &&
         cudaEventCreateWithFlags(&start, cudaEventDisableTiming) == cudaSuccess;
    for (auto& row : ev)
      for (auto& e : row) ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
  }
  ~HostPipeline() {
    for (auto& row : ev)
      for (auto& e : row)
        if (e) cudaEventDestroy(e);
    if (start) cudaEventDestroy(start);
    if (up) cudaStreamDestroy(up);
    if (down) cudaStreamDestroy(down);
  }
};

}  // namespace

extern "C" {

int solattn_host_scratch_bytes(int B, int H, int N, int d, int chunk_heads, size_t* bytes) {
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if (!bytes || chunk_heads < 0) return SOLATTN_ERR_ARG;
  const int BH = B * H;
  const int C = chunk_heads == 0 ? default_chunk_heads(BH) : (chunk_heads < BH ? chunk_heads : BH);
  HostChunkLayout L;
  if ((rc = host_chunk_layout(N, d, C, &L))) return rc;
  *bytes = SOLATTN_WORKSPACE_BYTES + 2 * L.buffer;
  return SOLATTN_OK;
}

int solattn_forward_host(const void* q, const void* k, const void* v, int B, int H, int N, int d, float beta,
                         void* out, float* lse, int32_t* density_out, int chunk_heads, void* scratch,
                         size_t scratch_bytes, void* stream) {
  int rc = check_shape(B, H, N, d);
  if (rc) return rc;
  if (!q || !k || !v || !out || chunk_heads < 0 || std::isnan(beta)) return SOLATTN_ERR_ARG;
  if (!scratch) return SOLATTN_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(scratch) & 255u) != 0) return SOLATTN_ERR_ALIGN;
  const int BH = B * H;
  const int C = chunk_heads == 0 ? default_chunk_heads(BH) : (chunk_heads < BH ? chunk_heads : BH);
  HostChunkLayout L;
  if ((rc = host_chunk_layout(N, d, C, &L))) return rc;
  if (scratch_bytes < SOLATTN_WORKSPACE_BYTES + 2 * L.buffer) return SOLATTN_ERR_WORKSPACE;
  int sms = 0;
  if ((rc = current_device_sms(&sms))) return rc;

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  HostPipeline pl;
  if (!pl.ok) return SOLATTN_ERR_CUDA;
  char* ws = static_cast<char*>(scratch);
  char* buf[2] = {ws + SOLATTN_WORKSPACE_BYTES, ws + SOLATTN_WORKSPACE_BYTES + L.buffer};
  const size_t nb = (static_cast<size_t>(N) + SOLATTN_BLOCK - 1) / SOLATTN_BLOCK;
  const size_t head_bytes = static_cast<size_t>(N) * d * 2;
  const char* hq = static_cast<const char*>(q);
  const char* hk = static_cast<const char*>(k);
  const char* hv = static_cast<const char*>(v);
  char* ho = static_cast<char*>(out);
  const solattn_options_t opt{SOLATTN_RULE_THRESHOLD, beta, 0, 0.f, 0, {0, 0, 0}, 0};
  auto cuda_ok = [](cudaError_t e) { return e == cudaSuccess; };

  // everything earlier on the caller's stream (an earlier call on this
  // scratch included) comes first; the status block starts clean
  if (!cuda_ok(cudaMemsetAsync(ws, 0, SOLATTN_WORKSPACE_BYTES, s)) || !cuda_ok(cudaEventRecord(pl.start, s)) ||
      !cuda_ok(cudaStreamWaitEvent(pl.up, pl.start, 0)) || !cuda_ok(cudaStreamWaitEvent(pl.down, pl.start, 0)))
    return SOLATTN_ERR_CUDA;
  const int chunks = (BH + C - 1) / C;
  for (int i = 0; i < chunks; ++i) {
    const int c0 = i * C, nc = (BH - c0 < C) ? BH - c0 : C;
    char* b = buf[i & 1];
    cudaEvent_t* in = pl.ev[0];
    cudaEvent_t* done = pl.ev[1];
    cudaEvent_t* back = pl.ev[2];
    // copy in: the buffer's inputs are free once chunk i - 2 has been computed
    if (i >= 2 && !cuda_ok(cudaStreamWaitEvent(pl.up, done[(i - 2) & 3], 0))) return SOLATTN_ERR_CUDA;
    const size_t bytes = head_bytes * nc, at = head_bytes * c0;
    if (!cuda_ok(cudaMemcpyAsync(b + L.q, hq + at, bytes, cudaMemcpyHostToDevice, pl.up)) ||
        !cuda_ok(cudaMemcpyAsync(b + L.k, hk + at, bytes, cudaMemcpyHostToDevice, pl.up)) ||
        !cuda_ok(cudaMemcpyAsync(b + L.v, hv + at, bytes, cudaMemcpyHostToDevice, pl.up)) ||
        !cuda_ok(cudaEventRecord(in[i & 3], pl.up)))
      return SOLATTN_ERR_CUDA;
    // compute: its outputs overwrite chunk i - 2's, which must have been copied back
    if (!cuda_ok(cudaStreamWaitEvent(s, in[i & 3], 0))) return SOLATTN_ERR_CUDA;
    if (i >= 2 && !cuda_ok(cudaStreamWaitEvent(s, back[(i - 2) & 3], 0))) return SOLATTN_ERR_CUDA;
    solattn_pooled_t pooled;
    if ((rc = solattn_pooled_layout(1, nc, N, d, b + L.pooled, &pooled, nullptr))) return rc;
    if ((rc = run_pool(b + L.q, b + L.k, b + L.v, 1, nc, N, d, nullptr, &pooled, stream))) return rc;
    if ((rc = run_forward(b + L.q, b + L.k, b + L.v, 1, nc, N, d, &pooled, opt, true, b + L.out,
                          lse ? reinterpret_cast<float*>(b + L.lse) : nullptr,
                          density_out ? reinterpret_cast<int32_t*>(b + L.dens) : nullptr, ws,
                          SOLATTN_WORKSPACE_BYTES, stream, false)))
      return rc;
    if (!cuda_ok(cudaEventRecord(done[i & 3], s))) return SOLATTN_ERR_CUDA;
    // copy back
    if (!cuda_ok(cudaStreamWaitEvent(pl.down, done[i & 3], 0)) ||
        !cuda_ok(cudaMemcpyAsync(ho + at, b + L.out, bytes, cudaMemcpyDeviceToHost, pl.down)))
      return SOLATTN_ERR_CUDA;
    if (lse && !cuda_ok(cudaMemcpyAsync(lse + static_cast<size_t>(c0) * N, b + L.lse,
                                        static_cast<size_t>(nc) * N * sizeof(float), cudaMemcpyDeviceToHost,
                                        pl.down)))
      return SOLATTN_ERR_CUDA;
    if (density_out && !cuda_ok(cudaMemcpyAsync(density_out + static_cast<size_t>(c0) * nb, b + L.dens,
                                                static_cast<size_t>(nc) * nb * sizeof(int32_t),
                                                cudaMemcpyDeviceToHost, pl.down)))
      return SOLATTN_ERR_CUDA;
    if (!cuda_ok(cudaEventRecord(back[i & 3], pl.down))) return SOLATTN_ERR_CUDA;
  }
  // the results are on the host once the caller's stream has passed this point
  if (!cuda_ok(cudaStreamWaitEvent(s, pl.ev[2][(chunks - 1) & 3], 0))) return SOLATTN_ERR_CUDA;
  return SOLATTN_OK;
}

}  // extern "C"
