// kernels.h -- internal launch interface between the C ABI layer and the CUDA
// kernels (not part of the public ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace solattn {

struct PooledPtrs {
  float* qbar;
  float* kbar;
  float* vbar;
  float* kmean;
  float* kcov;
  uint16_t* kbar16;  // bf16 copies for the per-token correction
  uint16_t* vbar16;
};

// Element strides of q, k, v and out; the d elements of a token are contiguous.
struct Strides {
  long long b, h, n;
};

struct ForwardArgs {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  uint16_t* out;
  float* lse;          // may be null
  int32_t* density;    // may be null
  PooledPtrs pooled;   // unused when route == false
  float beta;
  int rule;            // 0 threshold, 1 top-k, 2 top-p (solattn_rule)
  int topk;
  float topp;
  int n_forced;        // leading key blocks always kept
  int token_corr;      // 1: per-token correction through pooled-key tiles
  bool route;          // false: dense attention (no routing, no correction)
  int BH, H, N, d;
  Strides st;          // of q, k, v and out
  void* status;        // DeviceStatus in the caller's workspace
};

cudaError_t launch_pool(const uint16_t* q, const uint16_t* k, const uint16_t* v, const PooledPtrs& p, int BH,
                        int H, int N, int d, const Strides& st, int num_sms, cudaStream_t stream);

// Fused forward with per-unit key lists (any kept-set rule, either
// correction): one unit in flight per CTA (forward.cu).
cudaError_t launch_forward(const ForwardArgs& a, int num_sms, cudaStream_t stream);

// Fused forward with two units in flight per CTA (forward_pp.cu): threshold
// rule with the block-level correction (forced blocks allowed), and the dense
// path.
cudaError_t launch_forward_pp(const ForwardArgs& a, int num_sms, cudaStream_t stream);

#ifdef SOLATTN_TEST_HOOKS
// Test builds only: hook variables of each kernel's translation unit.
cudaError_t set_test_hooks_fwd(int skip_cta, unsigned long long wait_budget_ns);
cudaError_t set_route_dump_fwd(uint32_t* mask, float* stats);
cudaError_t set_test_hooks_pp(int skip_cta, unsigned long long wait_budget_ns);
cudaError_t set_route_dump_pp(uint32_t* mask, float* stats);
#endif

}  // namespace solattn
