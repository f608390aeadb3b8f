// Internal declarations shared by the libhs translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "hs.h"

namespace hs {

// Arguments common to the attention-style calls, after host validation.
struct Problem {
  const void* q;
  int64_t q_row_stride, q_head_stride;
  const void* k;
  int64_t k_row_stride;
  const void* v;
  int64_t v_row_stride;
  const int32_t* cu_seqlens;
  int num_docs, total_tokens, max_seqlen;
  int num_heads, dk, dv;
  hs_dtype dtype;
  float scale;  // resolved (> 0)
  int* status;  // device status word of the current device
};

struct ScoreArgs {
  Problem p;
  int block_size, nbmax, nb_stride;
  float* lse;
  float* block_score;
  float* block_lse;  // may be null
  void* workspace;
  size_t workspace_bytes;
};

struct AttnArgs {
  Problem p;
  const int32_t* idx;  // sparse only
  int topk, block_size;
  int window;          // swa only
  const float* sink;   // may be null
  void* out;
  float* lse;
  // optional combining epilogue (the SWA layer): out = gate_own * result +
  // gate_prev * prev; prev [T, H, Dv] of dtype, may alias out; gates [T, H]
  // fp32 or null (= 1).  prev == null: plain output.
  const void* prev = nullptr;
  const float* gate_own = nullptr;
  const float* gate_prev = nullptr;
};

// The full layer's fused forward (after host validation): dense causal
// attention without a sink plus step 1's outputs.
struct FullArgs {
  Problem p;
  int block_size, nbmax, nb_stride;
  void* out;
  float* lse;
  float* block_score;
  float* block_lse;  // may be null
  void* workspace;   // tc_full_workspace() bytes on the tensor-core path
};

// Backward of the attention calls (after host validation).
struct BwdArgs {
  Problem p;
  const int32_t* idx;  // sparse only
  int topk, block_size;
  int window;          // swa only
  const float* sink;   // may be null
  const void* out;
  const float* lse;
  const void* dout;
  float* dq;
  float* dkey;
  float* dval;
  float* dsink;        // may be null
  void* workspace;     // simt_backward_workspace() bytes
  void* dkdv_ws;       // the tensor-core dk / dv pass's partial sums, or null
};

// Launchers; each returns cudaSuccess or the launch error.
cudaError_t launch_simt_block_score(const ScoreArgs& a, cudaStream_t s);
// Longest score row hs_select_topk takes (its keys staged in shared memory):
// NBmax = ceil(max_seqlen / block_size) <= kMaxSelectBlocks.
constexpr int kMaxSelectBlocks = 56 * 1024;
cudaError_t launch_select_topk(const float* block_score, int nb_stride, const int32_t* cu,
                               int num_docs, int total_tokens, int max_seqlen, int block_size,
                               int topk, int32_t* idx, int* status, cudaStream_t s);
cudaError_t launch_simt_attention(const AttnArgs& a, bool sparse, cudaStream_t s);
size_t simt_backward_workspace(int total_tokens, int num_heads);
// *path (may be null) receives the kernel family the dq and dk / dv passes use.
cudaError_t launch_simt_backward(const BwdArgs& a, bool sparse, bool allow_mma, int* path,
                                 cudaStream_t s);
// The backward's tcgen05 passes: bf16, 64 heads, Dk <= 576 and Dv <= 512,
// multiples of 64, 16-byte aligned operands; delta = the workspace's [T, H]
// array.  dq query-major (tc_bwd_dq.cu); dk / dv key-major, a cluster of
// four CTAs per 32-key tile (tc_bwd_dkdv.cu).
bool tc_backward_shape_ok(hs_dtype dtype, int num_heads, int dk, int dv);
bool tc_bwd_dq_supported(const Problem& p);
bool tc_bwd_dkdv_supported(const Problem& p);
// Bytes of the dk / dv pass's partial sums (per query range, per key row).
size_t tc_bwd_dkdv_workspace(int total_tokens, int dk, int dv);
cudaError_t launch_tc_bwd_dq(const BwdArgs& a, bool sparse, const float* delta,
                             long long wait_limit, cudaStream_t s);
cudaError_t launch_tc_bwd_dkdv(const BwdArgs& a, bool sparse, const float* delta,
                               long long wait_limit, cudaStream_t s);

// Shared-memory bytes the CUDA-core block-score kernel needs (0 if it cannot run).
size_t simt_block_score_smem(int num_heads, int dk, int nbmax);

// tcgen05 kernels (bf16).  *_supported() decides eligibility on the host.
bool tc_block_score_supported(int num_heads, int dk, int block_size, int nbmax);
size_t tc_block_score_workspace(int total_tokens, int num_docs, int num_heads, int nbmax);
bool tc_block_score_eligible(const ScoreArgs& a);  // alignment / doc-count conditions
cudaError_t launch_tc_block_score(const ScoreArgs& a, long long wait_limit, cudaStream_t s);

bool tc_attention_supported(int num_heads, int dk, int dv, int block_size, bool sparse);
bool tc_attention_eligible(const AttnArgs& a);  // alignment conditions
cudaError_t launch_tc_attention(const AttnArgs& a, bool sparse, long long wait_limit,
                                cudaStream_t s);
// Full-layer mode of the same kernel (block sizes 32, 64, 128).
bool tc_full_supported(int num_heads, int dk, int dv, int block_size);
size_t tc_full_workspace(int total_tokens, int nbmax);
cudaError_t launch_tc_full(const FullArgs& f, long long wait_limit, cudaStream_t s);

// Records msg as the calling thread's hs_last_error() and returns st.
hs_status report_error(hs_status st, const char* msg);

// hs_block_score's host-side argument checks (no device work); HS_OK or the
// status hs_block_score would return for them, with hs_last_error() set.
hs_status check_score_args(const void* q, int64_t qrs, int64_t qhs, const void* k, int64_t krs,
                           const int32_t* cu, int num_docs, int total_tokens, int max_seqlen,
                           int num_heads, int dk, hs_dtype dtype, float scale, int block_size,
                           const float* lse, const float* block_score, int nb_stride);

// One thread waits (bounded) on an mbarrier nothing arrives at.
cudaError_t launch_selftest_wait(long long limit_ns, int* status, cudaStream_t s);

}  // namespace hs
