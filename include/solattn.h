/*
 * solattn.h -- C ABI of the Sol-Attn block-sparse attention forward for
 * NVIDIA B200 (sm_100a).
 *
 * The method is Sol-Attn ("Sol-Attn: Accelerating Video Generation Inference
 * via On-the-Fly Attention Sparsification", arXiv 2607.24027), as described on
 * the pages hotpaper.ai (abstract), agihunt.info (digest) and paithon.it
 * (article). Section names below are the paithon.it headings.
 *
 * Notation: B batch, H heads, N tokens, d head dimension (64 or 128),
 * 64-token blocks ("Perché l'attenzione pesa tanto nei video"),
 * N_b = ceil(N / 64), n_j = valid tokens of block j (64, or fewer for the last),
 * s = 1/sqrt(d).
 *
 * Layouts (row-major; contiguous unless solattn_pool_ex / solattn_forward_ex
 * are given other strides):
 *   q, k, v, out        bf16 [B][H][N][d]   (passed as raw 16-bit words)
 *   lse                 fp32 [B][H][N]      natural log of the softmax sum
 *   density_out         int32 [B][H][N_b]   |S_i| = kept key blocks per query block
 *   pooled buffers      fp32 (plus bf16 copies of kbar, vbar), see solattn_pooled_t
 *
 * Ownership: the caller allocates every buffer, on the device unless a function
 * says otherwise. No call allocates device memory. Nothing is retained after a
 * call returns. Every device pointer must be 16-byte aligned.
 *
 * Ordering: every call that takes `stream` (a cudaStream_t, NULL = legacy
 * default stream) is asynchronous on that stream and returns once its work is
 * enqueued. Argument errors are reported before anything is enqueued.
 *
 * Errors: every int-returning call returns SOLATTN_OK (0) or one of the codes
 * below; solattn_strerror() names them. Errors that happen on the device (a
 * bounded wait that expired) are recorded in the caller's workspace and
 * reported by solattn_status().
 */
#ifndef SOLATTN_H_
#define SOLATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define SOLATTN_BLOCK 64          /* tokens per block */
#define SOLATTN_MAX_TOKENS 262144 /* N limit (N_b <= 4096) */
#define SOLATTN_WORKSPACE_BYTES 256

enum solattn_status_code {
  SOLATTN_OK = 0,
  SOLATTN_ERR_ARG = 1,         /* null pointer, non-positive size, NaN beta */
  SOLATTN_ERR_UNSUPPORTED = 2, /* d not in {64,128}, N > SOLATTN_MAX_TOKENS, B*H too large */
  SOLATTN_ERR_ALIGN = 3,       /* a device pointer is not 16-byte aligned */
  SOLATTN_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  SOLATTN_ERR_TIMEOUT = 5,     /* a bounded device wait expired (device side) */
  SOLATTN_ERR_DEVICE = 6,      /* current device is not an sm_100 GPU */
  SOLATTN_ERR_WORKSPACE = 7,   /* workspace missing or smaller than SOLATTN_WORKSPACE_BYTES */
  SOLATTN_ERR_SCRATCH = 8      /* problem needs more than SOLATTN_NOALLOC_SCRATCH_BYTES of scratch */
};

/*
 * Pooled statistics of one (q, k, v) triple, written by solattn_pool and read
 * by solattn_forward. All fp32, device memory, caller-owned:
 *   qbar, kbar, vbar  [B][H][N_b][d]  block means over valid tokens
 *   kmean             [B][H][d]       mean of the pooled keys (each block counts once)
 *   kcov              [B][H][d][d]    covariance of the pooled keys, divided by N_b
 *   kbar16, vbar16    [B][H][N_b][d]  kbar and vbar rounded to bf16 (operands of the
 *                                     per-token correction's MMAs)
 * (paithon.it, "Una soglia per ogni riga", last paragraph: the mean and the
 * d x d second-moment matrix of the pooled keys give every proxy row's mean and
 * spread; solattn_forward evaluates them per query block from kmean and kcov.)
 */
typedef struct {
  float* qbar;
  float* kbar;
  float* vbar;
  float* kmean;
  float* kcov;
  void* kbar16;
  void* vbar16;
} solattn_pooled_t;

/*
 * Size in bytes of one contiguous buffer holding every pooled array, and (when
 * base != NULL) the pointers into it, each 256-byte aligned. base may be a
 * device pointer; it is only used for address arithmetic, never dereferenced.
 * Host-only; enqueues nothing.
 */
int solattn_pooled_layout(int B, int H, int N, int d, void* base, solattn_pooled_t* pooled,
                          size_t* bytes);

/*
 * Pooling (paithon.it, "Perché l'attenzione pesa tanto nei video": proxy scores
 * are products of block-mean queries and keys; "Una soglia per ogni riga",
 * last paragraph: the row statistics come from the mean and d x d
 * second-moment matrix of the pooled keys).
 * Reads q, k, v once and writes every array of `pooled` (the struct itself is
 * host memory, its pointers are device memory):
 *   qbar_i = mean of the valid query tokens of block i (likewise kbar, vbar);
 *   kmean  = (1/N_b) sum_j kbar_j;
 *   kcov   = (1/N_b) sum_j (kbar_j - kmean)(kbar_j - kmean)^T  (two-pass, fp32,
 *            fixed summation order: the result is the same on every call).
 */
int solattn_pool(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                 const solattn_pooled_t* pooled, void* stream);

/*
 * Element strides of q, k, v and out (the pages fix no layout): token (b, h, n)
 * starts at b * batch + h * head + n * token elements from the base pointer and
 * its d elements are contiguous. {H*N*d, N*d, d} is [B][H][N][d]; {N*H*d, d,
 * H*d} is [B][N][H][d]. Every stride must be a multiple of 8 elements (16
 * bytes), token >= d, head != 0 when H > 1 and batch != 0 when B > 1 (out
 * shares the strides: two heads must not write the same rows); all zero means
 * contiguous [B][H][N][d]. The four tensors share one set of strides.
 */
typedef struct {
  long long batch;
  long long head;
  long long token;
} solattn_strides_t;

/*
 * solattn_pool on q, k, v laid out with *strides (host memory, read during
 * the call; NULL = contiguous). The pooled arrays are always contiguous.
 * SOLATTN_ERR_ARG for strides that break the rules above.
 */
int solattn_pool_ex(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                    const solattn_strides_t* strides, const solattn_pooled_t* pooled, void* stream);

/*
 * Sol-Attn forward (hotpaper.ai abstract: routing, sparse computation and
 * correction in one online-softmax pass; paithon.it "Una soglia per ogni riga":
 * tau_i = mu_i + beta sigma_i, S_i = {j : s_hat_ij > tau_i}; "Scegliere mentre si
 * calcola": proxy scores compared with tau_i as they are produced, kept blocks
 * attended exactly, skipped blocks approximated by the zeroth-order Taylor term
 * that reuses their proxy scores, both in the same softmax state).
 *
 * For every query block i, with s = 1/sqrt(d) and s_hat_ij = s qbar_i . kbar_j,
 * the row statistics are evaluated in the routing warps from kmean and kcov:
 *   mu_i = s qbar_i . kmean,  sigma_i = s sqrt(max(0, qbar_i^T kcov qbar_i)),
 *   tau_i = mu_i + beta sigma_i  (tau_i = +inf when sigma_i = 0: a constant row
 *   has no block strictly above its mean).
 * For every query token t of block i:
 *   out_t = (sum_{j in S_i} sum_{u in j} e^{s q_t.k_u} v_u + sum_{j not in S_i} n_j e^{s_hat_ij} vbar_j)
 *         / (sum_{j in S_i} sum_{u in j} e^{s q_t.k_u}     + sum_{j not in S_i} n_j e^{s_hat_ij})
 *   lse_t = natural log of the denominator;   density_out_i = |S_i|.
 * beta = -INFINITY keeps every block (dense attention); beta = +INFINITY skips
 * every block. The proxy map s_hat is never written to memory.
 *
 * pooled must hold solattn_pool's results for the same q and k. lse and
 * density_out may be NULL. workspace: device memory of at least
 * SOLATTN_WORKSPACE_BYTES, owned by the caller, used by one call at a time
 * (calls sharing a workspace must not overlap on the device); its contents
 * need no initialisation and are rewritten by every call.
 */
int solattn_forward(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                    const solattn_pooled_t* pooled, float beta, void* out, float* lse,
                    int32_t* density_out, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Kept-set rules other than the per-row threshold, and always-kept blocks.
 * The pages compare the threshold with the top-k and top-p routing of earlier
 * methods (paithon.it, "Una soglia per ogni riga": a shared budget or a sort
 * per row; "I numeri": routing time of threshold vs top-k vs top-p) and keep
 * the text tokens of joint attention exact ("Dove leggere con attenzione"):
 *   SOLATTN_RULE_THRESHOLD  S_i = {j : s_hat_ij > mu_i + beta sigma_i}
 *   SOLATTN_RULE_TOPK       S_i = {j : s_hat_ij >= the topk-th largest s_hat_i.}
 *                           (topk clamped to [0, N_b]; equal scores at the cut
 *                           are all kept)
 *   SOLATTN_RULE_TOPP       S_i = {j : s_hat_ij >= v*_i}, v*_i the largest score
 *                           whose superlevel set carries a fraction >= topp of
 *                           sum_j n_j e^{s_hat_ij}; topp <= 0 keeps nothing,
 *                           topp >= 1 everything
 * and in every rule blocks 0 .. n_forced - 1 are added to S_i. Skipped blocks
 * get the same zeroth-order correction as with the threshold.
 */
enum solattn_rule {
  SOLATTN_RULE_THRESHOLD = 0,
  SOLATTN_RULE_TOPK = 1,
  SOLATTN_RULE_TOPP = 2
};

typedef struct {
  int rule;      /* enum solattn_rule */
  float beta;    /* threshold rule (NaN rejected) */
  int topk;      /* top-k rule: key blocks kept per query block */
  float topp;    /* top-p rule: mass fraction (NaN rejected) */
  int n_forced;  /* leading key blocks always kept, >= 0 (0 = none) */
  solattn_strides_t strides;  /* of q, k, v and out; all zero = contiguous [B][H][N][d] */
  int correction;  /* 0: block-level proxy score s_hat_ij for a skipped block (the
                      library's definition); 1: per token, s q_t . kbar_j (the
                      literal reading of "Scegliere mentre si calcola": each token
                      of a skipped block carries the block's mean key), value
                      vbar_j either way */
} solattn_options_t;

/*
 * solattn_forward with the kept-set rule, forced blocks and tensor strides of
 * *opts (host memory, read during the call). solattn_forward(..., beta, ...)
 * equals this call with {SOLATTN_RULE_THRESHOLD, beta, 0, 0, 0, {0, 0, 0}, 0}.
 * Errors as for solattn_forward, plus SOLATTN_ERR_ARG for a null opts, an
 * unknown rule, a NaN beta/topp, a negative n_forced, invalid strides or a
 * correction other than 0 / 1. With correction = 1 the skipped blocks of the
 * unit's two query blocks are attended as extra 128-key tiles of pooled keys
 * (kbar16, vbar16), each column weighted by n_j.
 */
int solattn_forward_ex(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                       const solattn_pooled_t* pooled, const solattn_options_t* opts, void* out,
                       float* lse, int32_t* density_out, void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * Dense softmax attention with scale 1/sqrt(d) by the same kernel with routing
 * switched off: equal to solattn_forward with beta = -INFINITY, without the
 * pooled statistics. lse may be NULL. workspace as for solattn_forward.
 */
int solattn_dense(const void* q, const void* k, const void* v, int B, int H, int N, int d, void* out,
                  float* lse, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronises `stream`, then returns the device-side status recorded in
 * `workspace` by the last forward or dense call that used it: SOLATTN_OK or
 * SOLATTN_ERR_TIMEOUT (a bounded wait inside the kernel gave up; the kernel
 * returned early and its outputs are invalid). SOLATTN_ERR_CUDA if the
 * synchronisation or the read fails.
 */
int solattn_status(const void* workspace, void* stream);

/*
 * Allocation-free forward, for callers that cannot allocate device memory
 * themselves: code running where cudaMalloc is unavailable or forbidden (for
 * example inside a host framework that owns every allocation, a plugin that
 * may only receive tensors, or an embedded runtime with a fixed memory plan).
 * There is no counterpart on the pages: it is solattn_pool followed by
 * solattn_forward, with the pooled statistics and the workspace placed in one
 * file-scope static device array of SOLATTN_NOALLOC_SCRATCH_BYTES that every
 * GPU loading this library holds until the process exits.
 *
 * Arguments, layouts and results are those of solattn_pool + solattn_forward
 * (the caller passes inputs and outputs only; lse and density_out may be NULL).
 * The scratch needed is SOLATTN_WORKSPACE_BYTES plus the solattn_pooled_layout
 * size; larger problems are rejected with SOLATTN_ERR_SCRATCH before anything is
 * enqueued. Nothing is allocated (no cudaMalloc, cudaFree or allocating library
 * call). The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call before
 * any stream capture. All calls share the one array and it keeps the last
 * call's contents: calls that overlap on the GPU (other streams, other host
 * threads) race and must be serialised by the caller. The scheduler counter and
 * status word at the start of the array are cleared by every call; a bounded
 * device wait that expires ends the kernel early (instead of hanging) and is
 * reported by solattn_noalloc_status, not by this call's return code.
 */
#define SOLATTN_NOALLOC_SCRATCH_BYTES (16u << 20)
int solattn_forward_noalloc(const void* q, const void* k, const void* v, int B, int H, int N, int d, float beta,
                            void* out, float* lse, int32_t* density_out, void* stream);

/*
 * Device status of the last solattn_forward_noalloc call on the current device
 * (no counterpart on the pages): synchronises `stream`, then copies the status
 * block out of the static array (no allocation) and returns SOLATTN_OK or
 * SOLATTN_ERR_TIMEOUT (a bounded wait gave up; that call's outputs are
 * invalid); SOLATTN_ERR_CUDA if the synchronisation or the copy fails. Calls on
 * other streams that overlap the one being checked race on the same block.
 */
int solattn_noalloc_status(void* stream);

/*
 * End-to-end forward on HOST buffers (no counterpart on the pages): the
 * computation of solattn_pool + solattn_forward (threshold rule, block-level
 * correction) for q, k, v in host memory, with out, lse and density_out
 * written to host memory. Layouts are the contiguous ones of solattn_forward;
 * lse and density_out may be NULL.
 *
 * The B*H (batch, head) pairs are independent (every statistic and every
 * kept set is per pair), so they go through the device in chunks of
 * chunk_heads consecutive pairs (0 = about B*H / 16, at least 1): while chunk i
 * is pooled and attended on `stream`, chunk i + 1 is copied to the device and
 * chunk i - 1's results are copied back, on two streams of the call's own.
 * Host buffers must be page-locked (cudaHostAlloc / cudaHostRegister) for the
 * copies to overlap the computation; pageable memory gives the same results
 * with the copies serialised by the CUDA runtime.
 *
 * scratch: device memory of at least solattn_host_scratch_bytes(B, H, N, d,
 * chunk_heads) bytes, 256-byte aligned, owned by the caller and used by one
 * call at a time (two chunk buffers of inputs, outputs and pooled statistics;
 * its first SOLATTN_WORKSPACE_BYTES are the workspace, so
 * solattn_status(scratch, stream) reports the call's device status: the first
 * error of any chunk). The call only enqueues work; the results are in host
 * memory once `stream` has completed (the call makes `stream` wait for the
 * last copy back). Errors: as for solattn_forward, plus SOLATTN_ERR_ARG for a
 * null host buffer, a negative chunk_heads or a NaN beta, and
 * SOLATTN_ERR_WORKSPACE for a missing or short scratch; nothing is enqueued
 * when the arguments are rejected.
 */
int solattn_host_scratch_bytes(int B, int H, int N, int d, int chunk_heads, size_t* bytes);
int solattn_forward_host(const void* q, const void* k, const void* v, int B, int H, int N, int d, float beta,
                         void* out, float* lse, int32_t* density_out, int chunk_heads, void* scratch,
                         size_t scratch_bytes, void* stream);

/* Static description of a status code. */
const char* solattn_strerror(int code);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
int solattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SOLATTN_H_ */
