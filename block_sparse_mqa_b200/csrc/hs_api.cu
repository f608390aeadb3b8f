// Host side of the libhs C ABI: argument validation, kernel choice, the
// device status word and error reporting.  See include/hs.h for the contract
// of every entry point.

#include <cuda_runtime.h>
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "hs.h"
#include "hs_internal.h"

namespace {

// Device-side status word: kernels record the first device-detected problem
// here (one copy per device that loads the library).
__device__ int g_device_status;

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices];
std::mutex g_status_mu;

std::atomic<int> g_force_simt{0};
std::atomic<long long> g_wait_limit{0};  // 0 = the kernels' default bound

thread_local char g_last_error[512];
// Kernel family of the calling thread's most recent successful compute call
// (hs_last_path), -1 before the first one.
thread_local int g_last_path = -1;

hs_status fail(hs_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return st;
}

hs_status cuda_fail(cudaError_t e, const char* what) {
  return fail(HS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Address of the status word on the current device (looked up once per
// device with that device current).
hs_status status_ptr(int** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(HS_ERR_UNSUPPORTED, "device id %d", dev);
  std::lock_guard<std::mutex> lk(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_device_status);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  *out = g_status_ptr[dev];
  return HS_OK;
}

bool valid_block(int b) { return b == 16 || b == 32 || b == 64 || b == 128; }

int nbmax_of(int max_seqlen, int block_size) {
  return (max_seqlen + block_size - 1) / block_size;
}

constexpr int kMaxHeads = 128;
constexpr int kMaxDim = 1024;

// Checks shared by the calls that read q and k; fills p (status excluded).
hs_status check_problem(hs::Problem& p, const void* q, int64_t qrs, int64_t qhs, const void* k,
                        int64_t krs, const int32_t* cu, int num_docs, int total_tokens,
                        int max_seqlen, int num_heads, int dk, int dv, hs_dtype dtype,
                        float scale) {
  if (total_tokens < 0) return fail(HS_ERR_INVALID_ARG, "total_tokens < 0");
  if (num_docs < 0) return fail(HS_ERR_INVALID_ARG, "num_docs < 0");
  if (total_tokens > 0 && num_docs < 1)
    return fail(HS_ERR_INVALID_ARG, "num_docs must be >= 1 when total_tokens > 0");
  if (total_tokens > 0 && max_seqlen < 1)
    return fail(HS_ERR_INVALID_ARG, "max_seqlen must be >= 1");
  if (!cu) return fail(HS_ERR_INVALID_ARG, "cu_seqlens is NULL");
  if (!q || !k) return fail(HS_ERR_INVALID_ARG, "q or k is NULL");
  if (dtype != HS_F32 && dtype != HS_BF16) return fail(HS_ERR_UNSUPPORTED, "dtype %d", (int)dtype);
  if (num_heads < 1 || num_heads > kMaxHeads)
    return fail(HS_ERR_UNSUPPORTED, "num_heads %d not in [1, %d]", num_heads, kMaxHeads);
  if (dk < 1 || dk > kMaxDim) return fail(HS_ERR_UNSUPPORTED, "dk %d not in [1, %d]", dk, kMaxDim);
  if (dv < 0 || dv > kMaxDim) return fail(HS_ERR_UNSUPPORTED, "dv %d not in [1, %d]", dv, kMaxDim);
  if (qhs < dk) return fail(HS_ERR_INVALID_ARG, "q_head_stride %lld < dk", (long long)qhs);
  if (qrs < (int64_t)num_heads * qhs)
    return fail(HS_ERR_INVALID_ARG, "q_row_stride %lld < num_heads * q_head_stride", (long long)qrs);
  if (krs < dk) return fail(HS_ERR_INVALID_ARG, "k_row_stride %lld < dk", (long long)krs);
  if (!(isfinite(scale))) return fail(HS_ERR_INVALID_ARG, "softmax_scale is not finite");
  p.q = q;
  p.q_row_stride = qrs;
  p.q_head_stride = qhs;
  p.k = k;
  p.k_row_stride = krs;
  p.v = nullptr;
  p.v_row_stride = 0;
  p.cu_seqlens = cu;
  p.num_docs = num_docs;
  p.total_tokens = total_tokens;
  p.max_seqlen = max_seqlen;
  p.num_heads = num_heads;
  p.dk = dk;
  p.dv = dv;
  p.dtype = dtype;
  p.scale = scale > 0.f ? scale : 1.0f / sqrtf((float)dk);
  p.status = nullptr;
  return HS_OK;
}

// The backward's workspace: the delta / sink terms of every path, then (for
// shapes the tensor-core passes take) the dk / dv pass's partial sums at a
// 256-byte boundary.
size_t bwd_simt_bytes(int total_tokens, int num_heads) {
  return (hs::simt_backward_workspace(total_tokens, num_heads) + 255) & ~(size_t)255;
}
size_t bwd_workspace(int total_tokens, int num_heads, int dk, int dv, hs_dtype dtype) {
  size_t need = bwd_simt_bytes(total_tokens, num_heads);
  if (!g_force_simt.load() && hs::tc_backward_shape_ok(dtype, num_heads, dk, dv))
    need += hs::tc_bwd_dkdv_workspace(total_tokens, dk, dv);
  return need;
}

hs_status launched(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return cuda_fail(e, what);
  return HS_OK;
}

// launched(), and on success records `path` as the call's kernel family.
hs_status launched_on(cudaError_t e, const char* what, int path) {
  hs_status r = launched(e, what);
  if (r == HS_OK) g_last_path = path;
  return r;
}

}  // namespace

namespace hs {
// Lets other translation units of the library report a host-side failure
// through hs_last_error().
hs_status report_error(hs_status st, const char* msg) { return fail(st, "%s", msg); }

// Host checks of hs_block_score's arguments, without any device work.
hs_status check_score_args(const void* q, int64_t qrs, int64_t qhs, const void* k, int64_t krs,
                           const int32_t* cu, int num_docs, int total_tokens, int max_seqlen,
                           int num_heads, int dk, hs_dtype dtype, float scale, int block_size,
                           const float* lse, const float* block_score, int nb_stride) {
  Problem p{};
  hs_status r = check_problem(p, q, qrs, qhs, k, krs, cu, num_docs, total_tokens, max_seqlen,
                              num_heads, dk, 0, dtype, scale);
  if (r != HS_OK) return r;
  if (!valid_block(block_size))
    return fail(HS_ERR_UNSUPPORTED, "block_size %d not in {16, 32, 64, 128}", block_size);
  if (!lse || !block_score) return fail(HS_ERR_INVALID_ARG, "lse or block_score is NULL");
  if (total_tokens > 0 && nb_stride < nbmax_of(max_seqlen, block_size))
    return fail(HS_ERR_INVALID_ARG, "nb_stride %d < ceil(max_seqlen / block_size) = %d", nb_stride,
                nbmax_of(max_seqlen, block_size));
  return HS_OK;
}
}  // namespace hs

extern "C" {

int hs_version(void) { return 300; }

const char* hs_status_string(hs_status s) {
  switch (s) {
    case HS_OK: return "HS_OK";
    case HS_ERR_INVALID_ARG: return "HS_ERR_INVALID_ARG";
    case HS_ERR_UNSUPPORTED: return "HS_ERR_UNSUPPORTED";
    case HS_ERR_CUDA: return "HS_ERR_CUDA";
    case HS_ERR_INVALID_INDEX: return "HS_ERR_INVALID_INDEX";
    case HS_ERR_TIMEOUT: return "HS_ERR_TIMEOUT";
    case HS_ERR_WORKSPACE: return "HS_ERR_WORKSPACE";
  }
  return "HS_ERR_UNKNOWN";
}

const char* hs_last_error(void) { return g_last_error; }

int hs_last_path(void) { return g_last_path; }

void hs_set_force_simt(int on) { g_force_simt.store(on ? 1 : 0); }

hs_status hs_selftest_wait(long long limit_ns, hs_stream_t stream) {
  if (limit_ns < 1 || limit_ns > 1000000000ll)
    return fail(HS_ERR_INVALID_ARG, "limit_ns %lld not in [1, 1e9]", limit_ns);
  int* st = nullptr;
  hs_status r = status_ptr(&st);
  if (r != HS_OK) return r;
  return launched(hs::launch_selftest_wait(limit_ns, st, stream), "self-test wait");
}

int hs_path(int op, hs_dtype dtype, int num_heads, int dk, int dv, int block_size) {
  if (dtype != HS_F32 && dtype != HS_BF16) return -1;
  switch (op) {
    case HS_OP_SELECT_TOPK: return HS_PATH_SIMT;
    case HS_OP_BLOCK_SCORE:
      if (dtype == HS_BF16 && !g_force_simt.load() &&
          hs::tc_block_score_supported(num_heads, dk, block_size, 0))
        return HS_PATH_TCGEN05;
      return HS_PATH_SIMT;
    case HS_OP_SPARSE_MQA_BWD:
    case HS_OP_SWA_MQA_BWD:
      if (!g_force_simt.load() && hs::tc_backward_shape_ok(dtype, num_heads, dk, dv))
        return HS_PATH_MMA;
      return HS_PATH_SIMT;
    case HS_OP_SPARSE_MQA:
    case HS_OP_SWA_MQA:
    case HS_OP_BLOCK_SCORE_ATTN:  // fused, or the attention then the score kernel
    case HS_OP_SWA_LAYER:         // the sparse branch, then the window branch combining
      if (dtype == HS_BF16 && !g_force_simt.load() &&
          hs::tc_attention_supported(num_heads, dk, dv, block_size, op == HS_OP_SPARSE_MQA))
        return HS_PATH_TCGEN05;
      return HS_PATH_SIMT;
  }
  return -1;
}

size_t hs_workspace_size(int op, int total_tokens, int num_docs, int max_seqlen, int num_heads,
                         int dk, int dv, hs_dtype dtype, int block_size) {
  if ((op == HS_OP_SPARSE_MQA_BWD || op == HS_OP_SWA_MQA_BWD) && total_tokens > 0 &&
      num_heads > 0)
    return bwd_workspace(total_tokens, num_heads, dk, dv, dtype);
  if ((op != HS_OP_BLOCK_SCORE && op != HS_OP_BLOCK_SCORE_ATTN) || total_tokens <= 0 ||
      !valid_block(block_size))
    return 0;
  const int nbmax = nbmax_of(max_seqlen, block_size);
  size_t need = 0;
  if (dtype == HS_BF16 && !g_force_simt.load() &&
      hs::tc_block_score_supported(num_heads, dk, block_size, nbmax))
    need = hs::tc_block_score_workspace(total_tokens, num_docs, num_heads, nbmax);
  // the fused kernel's scratch (the call falls back to the score kernel when
  // pointer alignment rules the fused one out, so cover both)
  if (op == HS_OP_BLOCK_SCORE_ATTN && dtype == HS_BF16 && !g_force_simt.load() &&
      hs::tc_full_supported(num_heads, dk, dv, block_size)) {
    const size_t f = hs::tc_full_workspace(total_tokens, nbmax);
    if (f > need) need = f;
  }
  return need;
}

hs_status hs_poll_status(hs_stream_t stream) {
  int* st = nullptr;
  hs_status r = status_ptr(&st);
  if (r != HS_OK) return r;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int host = 0;
  e = cudaMemcpyFromSymbol(&host, g_device_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read status");
  const int zero = 0;
  e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "clear status");
  if (host != 0)
    return fail((hs_status)host, "device reported %s", hs_status_string((hs_status)host));
  return HS_OK;
}

hs_status hs_block_score(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                         const void* k, int64_t k_row_stride, const int32_t* cu_seqlens,
                         int num_docs, int total_tokens, int max_seqlen, int num_heads, int dk,
                         hs_dtype dtype, float softmax_scale, int block_size, float* lse,
                         float* block_score, int nb_stride, float* block_lse, void* workspace,
                         size_t workspace_bytes, hs_stream_t stream) {
  hs::ScoreArgs a{};
  hs_status r = check_problem(a.p, q, q_row_stride, q_head_stride, k, k_row_stride, cu_seqlens,
                              num_docs, total_tokens, max_seqlen, num_heads, dk, 0, dtype,
                              softmax_scale);
  if (r != HS_OK) return r;
  if (!valid_block(block_size))
    return fail(HS_ERR_UNSUPPORTED, "block_size %d not in {16, 32, 64, 128}", block_size);
  if (!lse || !block_score) return fail(HS_ERR_INVALID_ARG, "lse or block_score is NULL");
  if (total_tokens == 0) return HS_OK;
  const int nbmax = nbmax_of(max_seqlen, block_size);
  if (nb_stride < nbmax)
    return fail(HS_ERR_INVALID_ARG, "nb_stride %d < ceil(max_seqlen / block_size) = %d", nb_stride,
                nbmax);
  a.block_size = block_size;
  a.nbmax = nbmax;
  a.nb_stride = nb_stride;
  a.lse = lse;
  a.block_score = block_score;
  a.block_lse = block_lse;
  a.workspace = workspace;
  a.workspace_bytes = workspace_bytes;
  r = status_ptr(&a.p.status);
  if (r != HS_OK) return r;
  const bool tc = dtype == HS_BF16 && !g_force_simt.load() &&
                  hs::tc_block_score_supported(num_heads, dk, block_size, nbmax) &&
                  hs::tc_block_score_eligible(a);
  if (tc) {
    const size_t need = hs::tc_block_score_workspace(total_tokens, num_docs, num_heads, nbmax);
    if (need > 0 && (!workspace || workspace_bytes < need))
      return fail(HS_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                  workspace ? workspace_bytes : (size_t)0);
    return launched_on(hs::launch_tc_block_score(a, g_wait_limit.load(), stream),
                       "tc block score", HS_PATH_TCGEN05);
  }
  int dev = 0, optin = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (hs::simt_block_score_smem(num_heads, dk, nbmax) > (size_t)optin)
    return fail(HS_ERR_UNSUPPORTED, "num_heads * dk + blocks too large for the CUDA-core kernel");
  return launched_on(hs::launch_simt_block_score(a, stream), "simt block score", HS_PATH_SIMT);
}

hs_status hs_select_topk(const float* block_score, int nb_stride, const int32_t* cu_seqlens,
                         int num_docs, int total_tokens, int max_seqlen, int block_size, int topk,
                         int32_t* idx, hs_stream_t stream) {
  if (total_tokens < 0 || num_docs < 0) return fail(HS_ERR_INVALID_ARG, "negative size");
  if (total_tokens > 0 && (num_docs < 1 || max_seqlen < 1))
    return fail(HS_ERR_INVALID_ARG, "num_docs and max_seqlen must be >= 1");
  if (!block_score || !cu_seqlens || !idx) return fail(HS_ERR_INVALID_ARG, "NULL pointer");
  if (!valid_block(block_size))
    return fail(HS_ERR_UNSUPPORTED, "block_size %d not in {16, 32, 64, 128}", block_size);
  if (topk < 1 || topk > 256) return fail(HS_ERR_UNSUPPORTED, "topk %d not in [1, 256]", topk);
  if (total_tokens == 0) return HS_OK;
  const int nbmax = nbmax_of(max_seqlen, block_size);
  if (nb_stride < nbmax)
    return fail(HS_ERR_INVALID_ARG, "nb_stride %d < ceil(max_seqlen / block_size) = %d", nb_stride,
                nbmax);
  if (nbmax > hs::kMaxSelectBlocks)
    return fail(HS_ERR_UNSUPPORTED, "ceil(max_seqlen / block_size) = %d blocks > %d", nbmax,
                hs::kMaxSelectBlocks);
  int* st = nullptr;
  hs_status r = status_ptr(&st);
  if (r != HS_OK) return r;
  return launched_on(hs::launch_select_topk(block_score, nb_stride, cu_seqlens, num_docs,
                                            total_tokens, max_seqlen, block_size, topk, idx, st,
                                            stream),
                     "select topk", HS_PATH_SIMT);
}

static hs_status attention_common(hs::AttnArgs& a, bool sparse, const void* q, int64_t qrs,
                                  int64_t qhs, const void* k, int64_t krs, const void* v,
                                  int64_t vrs, const int32_t* cu, int num_docs, int total_tokens,
                                  int max_seqlen, int num_heads, int dk, int dv, hs_dtype dtype,
                                  float scale, const float* sink, void* out, float* lse,
                                  hs_stream_t stream) {
  hs_status r = check_problem(a.p, q, qrs, qhs, k, krs, cu, num_docs, total_tokens, max_seqlen,
                              num_heads, dk, dv, dtype, scale);
  if (r != HS_OK) return r;
  if (dv < 1) return fail(HS_ERR_UNSUPPORTED, "dv must be >= 1");
  if (!v) return fail(HS_ERR_INVALID_ARG, "v is NULL");
  if (vrs < dv) return fail(HS_ERR_INVALID_ARG, "v_row_stride %lld < dv", (long long)vrs);
  if (!out || !lse) return fail(HS_ERR_INVALID_ARG, "out or lse is NULL");
  a.p.v = v;
  a.p.v_row_stride = vrs;
  a.sink = sink;
  a.out = out;
  a.lse = lse;
  if (total_tokens == 0) return HS_OK;
  r = status_ptr(&a.p.status);
  if (r != HS_OK) return r;
  const bool tc = dtype == HS_BF16 && !g_force_simt.load() &&
                  hs::tc_attention_supported(num_heads, dk, dv, a.block_size, sparse) &&
                  hs::tc_attention_eligible(a);
  if (tc) return launched_on(hs::launch_tc_attention(a, sparse, g_wait_limit.load(), stream),
                             sparse ? "tc sparse attention" : "tc swa attention",
                             HS_PATH_TCGEN05);
  return launched_on(hs::launch_simt_attention(a, sparse, stream),
                     sparse ? "simt sparse attention" : "simt swa attention", HS_PATH_SIMT);
}

hs_status hs_sparse_mqa_fwd(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                            const void* k, int64_t k_row_stride, const void* v,
                            int64_t v_row_stride, const int32_t* cu_seqlens, int num_docs,
                            int total_tokens, int max_seqlen, int num_heads, int dk, int dv,
                            hs_dtype dtype, float softmax_scale, const int32_t* idx, int topk,
                            int block_size, const float* sink, void* out, float* lse,
                            hs_stream_t stream) {
  if (!valid_block(block_size))
    return fail(HS_ERR_UNSUPPORTED, "block_size %d not in {16, 32, 64, 128}", block_size);
  if (topk < 1 || topk > 256) return fail(HS_ERR_UNSUPPORTED, "topk %d not in [1, 256]", topk);
  if (!idx) return fail(HS_ERR_INVALID_ARG, "idx is NULL");
  hs::AttnArgs a{};
  a.idx = idx;
  a.topk = topk;
  a.block_size = block_size;
  a.window = 0;
  return attention_common(a, true, q, q_row_stride, q_head_stride, k, k_row_stride, v,
                          v_row_stride, cu_seqlens, num_docs, total_tokens, max_seqlen,
                          num_heads, dk, dv, dtype, softmax_scale, sink, out, lse, stream);
}

hs_status hs_swa_mqa_fwd(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                         const void* k, int64_t k_row_stride, const void* v, int64_t v_row_stride,
                         const int32_t* cu_seqlens, int num_docs, int total_tokens,
                         int max_seqlen, int num_heads, int dk, int dv, hs_dtype dtype,
                         float softmax_scale, int window, const float* sink, void* out,
                         float* lse, hs_stream_t stream) {
  if (window < 1) return fail(HS_ERR_INVALID_ARG, "window %d < 1", window);
  hs::AttnArgs a{};
  a.idx = nullptr;
  a.topk = 0;
  a.block_size = 64;  // block size plays no part in the window; any valid value
  a.window = window;
  return attention_common(a, false, q, q_row_stride, q_head_stride, k, k_row_stride, v,
                          v_row_stride, cu_seqlens, num_docs, total_tokens, max_seqlen,
                          num_heads, dk, dv, dtype, softmax_scale, sink, out, lse, stream);
}

hs_status hs_block_score_attn_fwd(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                                  const void* k, int64_t k_row_stride, const void* v,
                                  int64_t v_row_stride, const int32_t* cu_seqlens, int num_docs,
                                  int total_tokens, int max_seqlen, int num_heads, int dk, int dv,
                                  hs_dtype dtype, float softmax_scale, int block_size, void* out,
                                  float* lse, float* block_score, int nb_stride, float* block_lse,
                                  void* workspace, size_t workspace_bytes, hs_stream_t stream) {
  hs::FullArgs f{};
  hs_status r = check_problem(f.p, q, q_row_stride, q_head_stride, k, k_row_stride, cu_seqlens,
                              num_docs, total_tokens, max_seqlen, num_heads, dk, dv, dtype,
                              softmax_scale);
  if (r != HS_OK) return r;
  if (!valid_block(block_size))
    return fail(HS_ERR_UNSUPPORTED, "block_size %d not in {16, 32, 64, 128}", block_size);
  if (dv < 1) return fail(HS_ERR_UNSUPPORTED, "dv must be >= 1");
  if (!v) return fail(HS_ERR_INVALID_ARG, "v is NULL");
  if (v_row_stride < dv) return fail(HS_ERR_INVALID_ARG, "v_row_stride %lld < dv",
                                     (long long)v_row_stride);
  if (!out || !lse || !block_score) return fail(HS_ERR_INVALID_ARG, "out, lse or block_score is NULL");
  if (total_tokens == 0) return HS_OK;
  const int nbmax = nbmax_of(max_seqlen, block_size);
  if (nb_stride < nbmax)
    return fail(HS_ERR_INVALID_ARG, "nb_stride %d < ceil(max_seqlen / block_size) = %d", nb_stride,
                nbmax);
  f.p.v = v;
  f.p.v_row_stride = v_row_stride;
  f.block_size = block_size;
  f.nbmax = nbmax;
  f.nb_stride = nb_stride;
  f.out = out;
  f.lse = lse;
  f.block_score = block_score;
  f.block_lse = block_lse;
  f.workspace = workspace;
  r = status_ptr(&f.p.status);
  if (r != HS_OK) return r;
  hs::AttnArgs a{};  // the attention part, for the eligibility test and the two-kernel path
  a.p = f.p;
  a.block_size = block_size;
  a.window = max_seqlen;  // covers every document: dense causal
  a.sink = nullptr;
  a.out = out;
  a.lse = lse;
  const bool fused = dtype == HS_BF16 && !g_force_simt.load() &&
                     hs::tc_full_supported(num_heads, dk, dv, block_size) &&
                     hs::tc_attention_eligible(a);
  if (fused) {
    const size_t need = hs::tc_full_workspace(total_tokens, nbmax);
    if (!workspace || workspace_bytes < need)
      return fail(HS_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                  workspace ? workspace_bytes : (size_t)0);
    return launched_on(hs::launch_tc_full(f, g_wait_limit.load(), stream), "tc full layer",
                       HS_PATH_TCGEN05);
  }
  // two kernels: the attention (its lse is the same quantity; the score
  // kernel then writes lse again), then step 1
  const bool tca = dtype == HS_BF16 && !g_force_simt.load() &&
                   hs::tc_attention_supported(num_heads, dk, dv, block_size, false) &&
                   hs::tc_attention_eligible(a);
  r = launched(tca ? hs::launch_tc_attention(a, false, g_wait_limit.load(), stream)
                   : hs::launch_simt_attention(a, false, stream),
               "full layer attention");
  if (r != HS_OK) return r;
  r = hs_block_score(q, q_row_stride, q_head_stride, k, k_row_stride, cu_seqlens, num_docs,
                     total_tokens, max_seqlen, num_heads, dk, dtype, softmax_scale, block_size,
                     lse, block_score, nb_stride, block_lse, workspace, workspace_bytes, stream);
  if (r == HS_OK && !tca) g_last_path = HS_PATH_SIMT;  // the attention ran on CUDA cores
  return r;
}

hs_status hs_swa_layer_fwd(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                           const void* k, int64_t k_row_stride, const void* v,
                           int64_t v_row_stride, const void* k_shared,
                           int64_t k_shared_row_stride, const void* v_shared,
                           int64_t v_shared_row_stride, const int32_t* cu_seqlens, int num_docs,
                           int total_tokens, int max_seqlen, int num_heads, int dk, int dv,
                           hs_dtype dtype, float softmax_scale, int window, const float* sink_swa,
                           const int32_t* idx, int topk, int block_size,
                           const float* sink_sparse, const float* gate_swa,
                           const float* gate_sparse, void* out, float* lse_swa,
                           float* lse_sparse, hs_stream_t stream) {
  if (window < 1) return fail(HS_ERR_INVALID_ARG, "window %d < 1", window);
  if (!valid_block(block_size))
    return fail(HS_ERR_UNSUPPORTED, "block_size %d not in {16, 32, 64, 128}", block_size);
  if (topk < 1 || topk > 256) return fail(HS_ERR_UNSUPPORTED, "topk %d not in [1, 256]", topk);
  if (!idx) return fail(HS_ERR_INVALID_ARG, "idx is NULL");
  if (!k_shared || !v_shared) return fail(HS_ERR_INVALID_ARG, "k_shared or v_shared is NULL");
  if (k_shared_row_stride < dk)
    return fail(HS_ERR_INVALID_ARG, "k_shared_row_stride %lld < dk", (long long)k_shared_row_stride);
  if (v_shared_row_stride < dv)
    return fail(HS_ERR_INVALID_ARG, "v_shared_row_stride %lld < dv", (long long)v_shared_row_stride);
  if (!lse_sparse || !lse_swa) return fail(HS_ERR_INVALID_ARG, "lse_swa or lse_sparse is NULL");
  // the window branch's own arguments, checked before the first launch
  if (!k || !v) return fail(HS_ERR_INVALID_ARG, "k or v is NULL");
  if (k_row_stride < dk) return fail(HS_ERR_INVALID_ARG, "k_row_stride %lld < dk",
                                     (long long)k_row_stride);
  if (v_row_stride < dv) return fail(HS_ERR_INVALID_ARG, "v_row_stride %lld < dv",
                                     (long long)v_row_stride);
  // the sparse branch over the shared KV, written to out
  hs::AttnArgs sp{};
  sp.idx = idx;
  sp.topk = topk;
  sp.block_size = block_size;
  sp.window = 0;
  hs_status r = attention_common(sp, true, q, q_row_stride, q_head_stride, k_shared,
                                 k_shared_row_stride, v_shared, v_shared_row_stride, cu_seqlens,
                                 num_docs, total_tokens, max_seqlen, num_heads, dk, dv, dtype,
                                 softmax_scale, sink_sparse, out, lse_sparse, stream);
  if (r != HS_OK) return r;
  const int sparse_path = g_last_path;
  // the window branch, whose epilogue adds the gated sparse result from out
  hs::AttnArgs w{};
  w.idx = nullptr;
  w.topk = 0;
  w.block_size = 64;
  w.window = window;
  w.prev = out;
  w.gate_own = gate_swa;
  w.gate_prev = gate_sparse;
  r = attention_common(w, false, q, q_row_stride, q_head_stride, k, k_row_stride, v,
                       v_row_stride, cu_seqlens, num_docs, total_tokens, max_seqlen, num_heads,
                       dk, dv, dtype, softmax_scale, sink_swa, out, lse_swa, stream);
  if (r == HS_OK && sparse_path == HS_PATH_SIMT) g_last_path = HS_PATH_SIMT;
  return r;
}

static hs_status backward_common(hs::BwdArgs& a, bool sparse, const void* q, int64_t qrs,
                                 int64_t qhs, const void* k, int64_t krs, const void* v,
                                 int64_t vrs, const int32_t* cu, int num_docs, int total_tokens,
                                 int max_seqlen, int num_heads, int dk, int dv, hs_dtype dtype,
                                 float scale, const float* sink, const void* out,
                                 const float* lse, const void* dout, float* dq, float* dkey,
                                 float* dval, float* dsink, void* workspace,
                                 size_t workspace_bytes, hs_stream_t stream) {
  hs_status r = check_problem(a.p, q, qrs, qhs, k, krs, cu, num_docs, total_tokens, max_seqlen,
                              num_heads, dk, dv, dtype, scale);
  if (r != HS_OK) return r;
  if (dv < 1) return fail(HS_ERR_UNSUPPORTED, "dv must be >= 1");
  if (!v) return fail(HS_ERR_INVALID_ARG, "v is NULL");
  if (vrs < dv) return fail(HS_ERR_INVALID_ARG, "v_row_stride %lld < dv", (long long)vrs);
  if (!out || !lse || !dout) return fail(HS_ERR_INVALID_ARG, "out, lse or dout is NULL");
  if (!dq || !dkey || !dval) return fail(HS_ERR_INVALID_ARG, "dq, dk or dv is NULL");
  a.p.v = v;
  a.p.v_row_stride = vrs;
  a.sink = sink;
  a.out = out;
  a.lse = lse;
  a.dout = dout;
  a.dq = dq;
  a.dkey = dkey;
  a.dval = dval;
  a.dsink = dsink;
  if (total_tokens == 0) return HS_OK;
  const size_t need = bwd_workspace(total_tokens, num_heads, dk, dv, dtype);
  if (!workspace || workspace_bytes < need)
    return fail(HS_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                workspace ? workspace_bytes : (size_t)0);
  if ((reinterpret_cast<uintptr_t>(workspace) & 15) != 0)
    return fail(HS_ERR_INVALID_ARG, "workspace is not 16-byte aligned");
  a.workspace = workspace;
  a.dkdv_ws = need > bwd_simt_bytes(total_tokens, num_heads)
                  ? static_cast<char*>(workspace) + bwd_simt_bytes(total_tokens, num_heads)
                  : nullptr;
  r = status_ptr(&a.p.status);
  if (r != HS_OK) return r;
  int path = HS_PATH_SIMT;
  return launched_on(hs::launch_simt_backward(a, sparse, !g_force_simt.load(), &path, stream),
                     sparse ? "sparse attention backward" : "swa attention backward", path);
}

hs_status hs_sparse_mqa_bwd(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                            const void* k, int64_t k_row_stride, const void* v,
                            int64_t v_row_stride, const int32_t* cu_seqlens, int num_docs,
                            int total_tokens, int max_seqlen, int num_heads, int dk, int dv,
                            hs_dtype dtype, float softmax_scale, const int32_t* idx, int topk,
                            int block_size, const float* sink, const void* out, const float* lse,
                            const void* dout, float* dq, float* dkey, float* dval, float* dsink,
                            void* workspace, size_t workspace_bytes, hs_stream_t stream) {
  if (!valid_block(block_size))
    return fail(HS_ERR_UNSUPPORTED, "block_size %d not in {16, 32, 64, 128}", block_size);
  if (topk < 1 || topk > 256) return fail(HS_ERR_UNSUPPORTED, "topk %d not in [1, 256]", topk);
  if (!idx) return fail(HS_ERR_INVALID_ARG, "idx is NULL");
  hs::BwdArgs a{};
  a.idx = idx;
  a.topk = topk;
  a.block_size = block_size;
  a.window = 0;
  return backward_common(a, true, q, q_row_stride, q_head_stride, k, k_row_stride, v,
                         v_row_stride, cu_seqlens, num_docs, total_tokens, max_seqlen, num_heads,
                         dk, dv, dtype, softmax_scale, sink, out, lse, dout, dq, dkey, dval,
                         dsink, workspace, workspace_bytes, stream);
}

hs_status hs_swa_mqa_bwd(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                         const void* k, int64_t k_row_stride, const void* v, int64_t v_row_stride,
                         const int32_t* cu_seqlens, int num_docs, int total_tokens,
                         int max_seqlen, int num_heads, int dk, int dv, hs_dtype dtype,
                         float softmax_scale, int window, const float* sink, const void* out,
                         const float* lse, const void* dout, float* dq, float* dkey, float* dval,
                         float* dsink, void* workspace, size_t workspace_bytes,
                         hs_stream_t stream) {
  if (window < 1) return fail(HS_ERR_INVALID_ARG, "window %d < 1", window);
  hs::BwdArgs a{};
  a.idx = nullptr;
  a.topk = 0;
  a.block_size = 64;
  a.window = window;
  return backward_common(a, false, q, q_row_stride, q_head_stride, k, k_row_stride, v,
                         v_row_stride, cu_seqlens, num_docs, total_tokens, max_seqlen, num_heads,
                         dk, dv, dtype, softmax_scale, sink, out, lse, dout, dq, dkey, dval,
                         dsink, workspace, workspace_bytes, stream);
}

}  // extern "C"
