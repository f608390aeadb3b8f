/*
 * hs.h -- C ABI of libhs, the B200 (sm_100a) HySparse MQA attention path.
 *
 * The method: "HySparse MQA sparse attention (FA4 block scoring + SWA MQA +
 * block-sparse DSA gather)", PaddleFleet pull request 1470 ("Core" list and
 * the Copilot per-file table), in the absorbed-MLA MQA layout of its
 * "FlashMLA sparse kernel constraints" section: H query heads share ONE key
 * head of width Dk (latent + RoPE) and one value head of width Dv.
 *
 * Four calls form the forward path, in this order:
 *   hs_block_score     causal QK^T pass -> per-head row LSE, per-head block
 *                      LSE (optional) and head-summed block score
 *   hs_select_topk     per-query top-k key blocks inside its document
 *   hs_sparse_mqa_fwd  softmax attention over the selected blocks + sink
 *   hs_swa_mqa_fwd     sliding-window attention + sink (Dk != Dv allowed)
 *
 * and two calls give the backward of the two attention steps:
 *   hs_sparse_mqa_bwd  dq, dk, dv and the sink gradient of hs_sparse_mqa_fwd
 *   hs_swa_mqa_bwd     the same for hs_swa_mqa_fwd
 *
 * hs_block_score_attn_fwd is the full layer's forward: dense causal
 * attention that emits step 1's outputs from the same pass, replacing
 * hs_block_score where the model runs that layer anyway.  hs_swa_layer_fwd
 * is the SWA layer: its window attention plus a block-sparse branch over the
 * full layer's shared KV, combined.
 *
 * Conventions shared by every call
 * --------------------------------
 * Pointers named q, k, v, out, lse, block_score, block_lse, idx, sink and
 * cu_seqlens are DEVICE pointers.  Element strides are in elements, not
 * bytes; the innermost dimension of every tensor is contiguous.
 *
 *   q      [T, H, Dk]  row (token) stride q_row_stride, head stride
 *                      q_head_stride.
 *   k      [T, Dk]     row stride k_row_stride.
 *   v      [T, Dv]     row stride v_row_stride; may alias k (for example
 *                      v = k with Dv < Dk reads the first Dv columns, the
 *                      absorbed-MLA latent region).
 *   cu_seqlens [num_docs + 1] int32: packed documents; cu_seqlens[0] = 0,
 *                      non-decreasing, cu_seqlens[num_docs] = T.  Document d
 *                      is tokens [cu_seqlens[d], cu_seqlens[d+1]).  No
 *                      attention, block or window crosses a document end.
 *   max_seqlen         host-side upper bound of every document's length; it
 *                      sizes grids and the block count NBmax =
 *                      ceil(max_seqlen / block_size).
 *   dtype              HS_BF16 or HS_F32 for q, k, v and out (all the same).
 *                      Accumulation is fp32 in every case.
 *   softmax_scale      logits are s = softmax_scale * <q, k>; a value <= 0
 *                      selects Dk^-1/2 (the default sm_scale of the SWA
 *                      wrapper, per-file table entry "swa_attn.py").
 *   stream             a cudaStream_t (NULL = legacy default stream).  All
 *                      calls are asynchronous on it.
 *
 * Blocks.  Key blocks of size B are laid on each document separately from
 * its first token (the per-document block_bos of the block-score PyLayer in
 * the review of PaddleFleet pull request 1453); the last block of a
 * document may be partial.  Block ids are document-local.  For a query t
 * of document [bos, eos), its own block is bq(t) = (t - bos) / B.
 *
 * Ownership.  The caller owns every buffer, its allocation and lifetime.
 * The library never allocates, frees or synchronises inside these four
 * calls; any scratch it needs is the caller's `workspace` argument.
 *
 * Errors.  Every call validates its host-visible arguments before any
 * launch and returns a non-zero hs_status without touching the GPU when
 * they are wrong.  Device-detected problems (a malformed cu_seqlens, an
 * out-of-range block id, a pipeline wait that ran out of its iteration
 * limit) never trap: the kernel records a status word, skips the bad work
 * and exits; hs_poll_status() returns it.  hs_last_error() describes the
 * most recent host-side failure of the calling thread.
 */
#ifndef HS_H_
#define HS_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* hs_stream_t; /* == cudaStream_t */

typedef enum hs_status {
  HS_OK = 0,
  HS_ERR_INVALID_ARG = 1,   /* bad pointer, size, stride or cu_seqlens     */
  HS_ERR_UNSUPPORTED = 2,   /* valid but not implemented (dtype, dims)     */
  HS_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed        */
  HS_ERR_INVALID_INDEX = 4, /* device: a block id outside [-1, bq]         */
  HS_ERR_TIMEOUT = 5,       /* device: a bounded pipeline wait ran out     */
  HS_ERR_WORKSPACE = 6      /* workspace missing or smaller than required  */
} hs_status;

typedef enum hs_dtype { HS_F32 = 0, HS_BF16 = 1 } hs_dtype;

/* Operation ids for hs_path() and hs_workspace_size(). */
typedef enum hs_op {
  HS_OP_BLOCK_SCORE = 0,
  HS_OP_SELECT_TOPK = 1,
  HS_OP_SPARSE_MQA = 2,
  HS_OP_SWA_MQA = 3,
  HS_OP_SPARSE_MQA_BWD = 4,
  HS_OP_SWA_MQA_BWD = 5,
  HS_OP_BLOCK_SCORE_ATTN = 6,
  HS_OP_SWA_LAYER = 7
} hs_op;

/* Kernel family a call will use, as returned by hs_path(). */
typedef enum hs_kernel_path {
  HS_PATH_SIMT = 0,    /* CUDA-core kernel: fp32 inputs, unusual shapes    */
  HS_PATH_TCGEN05 = 1, /* tcgen05 tensor-core kernel (TMEM accumulators)   */
  HS_PATH_MMA = 2      /* the backward's tensor-core path (tcgen05: a
                          query-major dq pass and a key-major dk / dv pass) */
} hs_kernel_path;

/*
 * Step 1 -- causal block scoring.
 * Source: "HySparse MQA sparse attention ...", PaddleFleet pull request
 * 1470, "Core" list (FA4-fused block scoring) and per-file table
 * (pipeline.py: the block score is recovered as exp(block_logit - lse)
 * before top-k); review of pull request 1453 (per-document block_bos).
 *
 * For query t in document [bos, eos), head h, s_j = scale * <q[t,h], k[j]>
 * over the causal keys j in [bos, t]:
 *   lse[t,h]          = log sum_j exp(s_j)                 (no sink)
 *   block_lse[t,h,b]  = log sum_{j in block b, j <= t} exp(s_j)
 *   block_score[t,b]  = sum_h exp(block_lse[t,h,b] - lse[t,h])
 * for b <= bq(t); for bq(t) < b < NBmax, block_score = 0 and block_lse =
 * -inf.  Columns NBmax .. nb_stride-1 are not written.  Logs are natural.
 *
 *   lse          [T, H] fp32, output.
 *   block_score  [T, nb_stride] fp32, output; nb_stride >= NBmax.
 *   block_lse    [T, H, nb_stride] fp32, optional output (NULL = skip).
 *   workspace    device scratch of at least
 *                hs_workspace_size(HS_OP_BLOCK_SCORE, ...) bytes (may be
 *                NULL when that size is 0).  Its contents on entry do not
 *                matter; concurrent calls must not share one workspace.
 *                On the tensor-core path it is two [NBmax, 128] fp32 rows
 *                per CTA, one CTA per SM: 128 is the row count of a query
 *                tile (tokens x heads), independent of H (9.7 MB for
 *                NBmax 64 on 148 SMs).
 *   block_size   16, 32, 64 or 128.
 */
hs_status hs_block_score(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                         const void* k, int64_t k_row_stride,
                         const int32_t* cu_seqlens, int num_docs, int total_tokens,
                         int max_seqlen, int num_heads, int dk, hs_dtype dtype,
                         float softmax_scale, int block_size,
                         float* lse, float* block_score, int nb_stride, float* block_lse,
                         void* workspace, size_t workspace_bytes, hs_stream_t stream);

/*
 * Step 2 -- per-query top-k block selection.
 * Source: per-file table of pull request 1470 (pipeline.py: top-k block
 * selection over the recovered block scores).  Rule: candidates are blocks
 * 0..bq(t) of the query's document; the own block bq(t) and the first
 * block 0 are always selected and count toward topk; when bq(t) + 1 <=
 * topk all candidates are selected; otherwise the remaining slots go to
 * the highest block_score values, an exact fp32 tie going to the lower
 * block id.
 *
 *   block_score  [T, nb_stride] fp32 (as written by hs_block_score); only
 *                columns 0..bq(t) of row t are read.
 *   idx          [T, topk] int32 output: document-local block ids in
 *                ascending order, unused slots = -1.
 *   topk         1..256.  topk = 1 selects only the own block (the first
 *                block is then not forced).
 *   NBmax = ceil(max_seqlen / block_size) <= 57344 (a row's keys are staged
 *   in shared memory; e.g. documents up to 917504 tokens at block size 16);
 *   longer rows are HS_ERR_UNSUPPORTED.
 * One warp per query reads its row once; the selection is exact (no
 * approximation) and bit-for-bit deterministic.
 */
hs_status hs_select_topk(const float* block_score, int nb_stride,
                         const int32_t* cu_seqlens, int num_docs, int total_tokens,
                         int max_seqlen, int block_size, int topk, int32_t* idx,
                         hs_stream_t stream);

/*
 * Step 3 -- block-sparse MQA attention with a per-head sink.
 * Source: pull request 1470, "Core" list (block-sparse DSA gather with a
 * learnable per-head attn_sink) and "FlashMLA sparse kernel constraints";
 * the sink is a softmax offset ("Support attn sink in fa3", pull request
 * 1415, dense-path review thread): a logit in the denominator only.
 *
 * Keys of query t: S_t = union over the ids b >= 0 in idx[t] of the keys of
 * block b that are <= t.  With s_j = scale * <q[t,h], k[j]>:
 *   lse[t,h] = log(exp(sink[h]) + sum_{j in S_t} exp(s_j))
 *   out[t,h] = sum_{j in S_t} exp(s_j - lse[t,h]) * v[j]
 * sink is in the scaled logit space (not multiplied by softmax_scale).
 *
 *   idx    [T, topk] int32: ascending distinct ids in [0, bq(t)], then -1
 *          padding (the output of hs_select_topk).  An entry b >= 0 is used
 *          when b <= bq(t) and b is larger than the entry before it; any
 *          other non-negative entry is skipped and reported as
 *          HS_ERR_INVALID_INDEX (the row's output is then unspecified).
 *   sink   [H] fp32 or NULL (NULL = no sink, i.e. -inf).
 *   out    [T, H, Dv] of `dtype`, contiguous, output.
 *   lse    [T, H] fp32, output.
 */
hs_status hs_sparse_mqa_fwd(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                            const void* k, int64_t k_row_stride,
                            const void* v, int64_t v_row_stride,
                            const int32_t* cu_seqlens, int num_docs, int total_tokens,
                            int max_seqlen, int num_heads, int dk, int dv, hs_dtype dtype,
                            float softmax_scale, const int32_t* idx, int topk,
                            int block_size, const float* sink,
                            void* out, float* lse, hs_stream_t stream);

/*
 * Step 4 -- sliding-window MQA attention with a per-head sink.
 * Source: pull request 1470, "Core" list (SWA sliding-window MQA) and
 * per-file table (windowed_mqa_attn*.py: Dk != Dv, optional attn_sink);
 * review of pull request 1453 (per-row bos/eos key ranges).
 *
 * Keys of query t: the `window` keys ending at t, clipped at its document
 * start: j in [max(bos, t - window + 1), t].  Same lse/out/sink formulas
 * as hs_sparse_mqa_fwd.  window >= 1.
 */
hs_status hs_swa_mqa_fwd(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                         const void* k, int64_t k_row_stride,
                         const void* v, int64_t v_row_stride,
                         const int32_t* cu_seqlens, int num_docs, int total_tokens,
                         int max_seqlen, int num_heads, int dk, int dv, hs_dtype dtype,
                         float softmax_scale, int window, const float* sink,
                         void* out, float* lse, hs_stream_t stream);

/*
 * Backward of step 3 (block-sparse MQA with a per-head sink).
 * Source: pull request 1470, "Core" list (the block-sparse MQA and SWA
 * kernels come with backward passes; the learnable per-head attn_sink has an
 * analytic gradient) and per-file table (block-sparse DSA gather backend:
 * analytic sink gradient).  The pages give no formulas; this is the exact
 * gradient of hs_sparse_mqa_fwd for a loss L with dL/dout = dout.  With the
 * forward's key sets S_t, s_j = scale * <q[t,h], k[j]>, p_j = exp(s_j -
 * lse[t,h]) (lse includes the sink) and delta[t,h] = <dout[t,h], out[t,h]>:
 *   ds_j     = p_j * (<dout[t,h], v[j]> - delta[t,h])
 *   dq[t,h]  = scale * sum_{j in S_t} ds_j * k[j]
 *   dk[j]    = scale * sum over (t,h) with j in S_t of ds_j * q[t,h]
 *   dv[j]    = sum over (t,h) with j in S_t of p_j * dout[t,h]
 *   dsink[h] = -sum_t exp(sink[h] - lse[t,h]) * delta[t,h]
 *
 * Inputs are those of the forward call plus:
 *   out, dout  [T, H, Dv] of `dtype`, contiguous: the forward's output and
 *              the gradient of the loss with respect to it.
 *   lse        [T, H] fp32: the forward's lse (sink included).
 * Outputs (fp32, contiguous, fully overwritten; keys no query selected get
 * zero gradients):
 *   dq         [T, H, Dk]
 *   dkey       [T, Dk]   gradient with respect to the T rows of k
 *   dval       [T, Dv]   gradient with respect to the T rows of v (when v
 *                        aliases the first Dv columns of k, the caller adds
 *                        dval into those columns of dkey)
 *   dsink      [H], or NULL to skip; ignored when sink is NULL.
 *   workspace  device scratch of at least hs_workspace_size(
 *              HS_OP_SPARSE_MQA_BWD, ...) bytes, 16-byte aligned; its
 *              contents on entry do not matter; concurrent calls must not
 *              share one.  A missing or short workspace is HS_ERR_WORKSPACE
 *              before any device work.  Size: 8 * T * H rounded up to 256,
 *              plus, for shapes the tensor-core passes take, the dk / dv
 *              pass's fp32 partial sums, nrange * T * (Dk + Dv) * 4 bytes,
 *              with nrange = ceil(T / max(512, ceil(T / 8))) <= 8 query
 *              ranges (143 MB at T = 4096, Dk 576, Dv 512).
 * idx entries follow the forward's rule; offending entries are skipped and
 * reported as HS_ERR_INVALID_INDEX.  Results are deterministic (every sum
 * runs in a fixed order).  bf16 inputs with 64 heads and Dk, Dv multiples of
 * 64 (Dk <= 576, Dv <= 512, 16-byte aligned) run on tcgen05 tensor cores
 * (hs_path: HS_PATH_MMA); other inputs on CUDA cores.  The dk / dv pass is a
 * four-CTA cluster kernel (single CTAs where the device cannot place the
 * cluster) whose work items are (32-key tile, query range) pairs; their
 * partial sums are added per key in a fixed range order by a second kernel.
 */
hs_status hs_sparse_mqa_bwd(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                            const void* k, int64_t k_row_stride,
                            const void* v, int64_t v_row_stride,
                            const int32_t* cu_seqlens, int num_docs, int total_tokens,
                            int max_seqlen, int num_heads, int dk, int dv, hs_dtype dtype,
                            float softmax_scale, const int32_t* idx, int topk,
                            int block_size, const float* sink,
                            const void* out, const float* lse, const void* dout,
                            float* dq, float* dkey, float* dval, float* dsink,
                            void* workspace, size_t workspace_bytes, hs_stream_t stream);

/*
 * Backward of step 4 (sliding-window MQA with a per-head sink).
 * Source: pull request 1470, "Core" list (SWA sliding-window MQA) and
 * per-file table (windowed_mqa_attn*.py: fwd/bwd with Dk != Dv, attn_sink and
 * a guard for ragged sequence lengths in the backward).  Same formulas,
 * arguments and outputs as hs_sparse_mqa_bwd with the forward's window key
 * sets j in [max(bos, t - window + 1), t]; workspace size from
 * hs_workspace_size(HS_OP_SWA_MQA_BWD, ...).
 */
hs_status hs_swa_mqa_bwd(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                         const void* k, int64_t k_row_stride,
                         const void* v, int64_t v_row_stride,
                         const int32_t* cu_seqlens, int num_docs, int total_tokens,
                         int max_seqlen, int num_heads, int dk, int dv, hs_dtype dtype,
                         float softmax_scale, int window, const float* sink,
                         const void* out, const float* lse, const void* dout,
                         float* dq, float* dkey, float* dval, float* dsink,
                         void* workspace, size_t workspace_bytes, hs_stream_t stream);

/*
 * The full layer's forward with step 1 fused in.
 * Source: pull request 1470, "Core" list (FA4-fused block scoring), the
 * Copilot overview (the HySparse full layer produces the shared KV and the
 * block indices) and per-file table (block_score_fa4.py: the full layer's
 * flash-attention forward emits the scaled block_logit; pipeline.py: the
 * score is recovered as exp(block_logit - lse)); review of pull request 1453
 * (the PyLayer saves out and lse; per-document block_bos).
 *
 * For query t in document [bos, eos), head h, s_j = scale * <q[t,h], k[j]>
 * over every causal key j in [bos, t], with no sink:
 *   lse[t,h]          = log sum_j exp(s_j)
 *   out[t,h]          = sum_j exp(s_j - lse[t,h]) * v[j]
 *   block_lse[t,h,b]  = log sum_{j in block b, j <= t} exp(s_j)
 *   block_score[t,b]  = sum_h exp(block_lse[t,h,b] - lse[t,h])
 * lse, block_score and block_lse are exactly what hs_block_score defines
 * (blocks past bq(t) up to NBmax: score 0, block_lse -inf; columns NBmax ..
 * nb_stride-1 not written); out is hs_swa_mqa_fwd's output for a window
 * covering every document without a sink.
 *
 *   out          [T, H, Dv] of `dtype`, contiguous, output.
 *   lse          [T, H] fp32, output.
 *   block_score  [T, nb_stride] fp32, output; nb_stride >= NBmax.
 *   block_lse    [T, H, nb_stride] fp32, optional output (NULL = skip).
 *   workspace    device scratch of at least hs_workspace_size(
 *                HS_OP_BLOCK_SCORE_ATTN, ...) bytes; contents on entry do
 *                not matter; concurrent calls must not share one.  A missing
 *                or short workspace is HS_ERR_WORKSPACE before any launch.
 *   block_size   16, 32, 64 or 128.
 * bf16 with 64 heads, Dk and Dv multiples of 64 (Dk <= 576, Dv <= 512),
 * block sizes 32..128 and 16-byte aligned q, k, v, out run as ONE tcgen05
 * kernel (its scratch: two [NBmax, 64] fp32 rows per SM, one per head of
 * the 64).  Other inputs run
 * the attention and hs_block_score's kernel one after the other on the same
 * stream (same results, two passes over the logits).
 */
hs_status hs_block_score_attn_fwd(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                                  const void* k, int64_t k_row_stride,
                                  const void* v, int64_t v_row_stride,
                                  const int32_t* cu_seqlens, int num_docs, int total_tokens,
                                  int max_seqlen, int num_heads, int dk, int dv,
                                  hs_dtype dtype, float softmax_scale, int block_size,
                                  void* out, float* lse, float* block_score, int nb_stride,
                                  float* block_lse, void* workspace, size_t workspace_bytes,
                                  hs_stream_t stream);

/*
 * The HySparse SWA layer: window branch + sparse branch on the shared KV.
 * Source: pull request 1470, "What" (NSA-style, three cooperating
 * structures) and Copilot overview (the SWA kernel is wired into the SWA
 * layer's main branch; the full layer produces the shared KV and the block
 * indices); review of pull request 1453 (the SWA layer consumes shared_kv
 * in a sparse branch).  The pages do not say how the branches combine; as in
 * NSA, each branch is its own softmax and the output is their gated sum:
 *   out[t,h] = gate_swa[t,h]    * swa(q, k, v; window, sink_swa)[t,h]
 *            + gate_sparse[t,h] * sparse(q, k_shared, v_shared; idx, sink_sparse)[t,h]
 * with the two branches defined exactly as hs_swa_mqa_fwd and
 * hs_sparse_mqa_fwd, over the same queries q (the SWA layer's own).
 *
 *   k, v                [T, Dk], [T, Dv]: the SWA layer's own keys / values.
 *   k_shared, v_shared  [T, Dk], [T, Dv]: the full layer's keys / values
 *                       (same dims; v_shared may alias k_shared).
 *   idx                 [T, topk]: the full layer's block lists (the rule
 *                       of hs_sparse_mqa_fwd).
 *   gate_swa, gate_sparse  [T, H] fp32, or NULL for 1 (then a plain sum).
 *   out                 [T, H, Dv] of `dtype`, contiguous, output.
 *   lse_swa, lse_sparse [T, H] fp32 outputs: each branch's lse (with its sink).
 * No workspace.  The call runs the sparse branch into `out`, then the window
 * attention whose epilogue adds the gated sparse result it reads back from
 * `out` (fp32 arithmetic, one rounding to bf16 for the sum's window part and
 * one for the sum); 16-byte-aligned bf16 inputs with 64 heads use the
 * tcgen05 kernels for both.
 */
hs_status hs_swa_layer_fwd(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                           const void* k, int64_t k_row_stride,
                           const void* v, int64_t v_row_stride,
                           const void* k_shared, int64_t k_shared_row_stride,
                           const void* v_shared, int64_t v_shared_row_stride,
                           const int32_t* cu_seqlens, int num_docs, int total_tokens,
                           int max_seqlen, int num_heads, int dk, int dv, hs_dtype dtype,
                           float softmax_scale, int window, const float* sink_swa,
                           const int32_t* idx, int topk, int block_size,
                           const float* sink_sparse, const float* gate_swa,
                           const float* gate_sparse, void* out, float* lse_swa,
                           float* lse_sparse, hs_stream_t stream);

/*
 * Step 1 for callers that cannot allocate device memory.
 * The method has no counterpart of this call; it is a deployment aid.
 *
 * hs_block_score needs a caller-provided workspace.  Some callers cannot
 * allocate one: code running where an allocator call is not allowed (inside
 * a framework's kernel-launch hook, a real-time loop that must not take the
 * allocator's locks or synchronisation, a process whose device memory is
 * fixed up front).  This call computes exactly what hs_block_score computes,
 * with the same arguments minus the workspace, and takes its scratch from a
 * 16 MiB array in the library's own device memory (every GPU on which the
 * library is loaded holds that array until the process exits).  It calls no
 * allocation or free routine.
 *
 *   - Arguments are validated first (the same checks as hs_block_score).
 *     Then problems whose tensor-core scratch would exceed 16 MiB
 *     (hs_workspace_size of HS_OP_BLOCK_SCORE > 16 MiB: two [NBmax, 128]
 *     fp32 rows per SM, so with 148 SMs about 110 key blocks per document,
 *     e.g. max_seqlen 7040 at block size 64) are rejected on the host with
 *     HS_ERR_WORKSPACE before any device work; use hs_block_score with a
 *     workspace for them.  The limit is applied from the shape alone, so it
 *     is conservative for a call that would run the CUDA-core kernel (which
 *     needs no scratch) because of its pointer alignment or document count.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) while that device is current and keeps it for
 *     the life of the process; make that first call before any stream
 *     capture, and do not use the library across a cudaDeviceReset (the
 *     kept address would then be stale; the device status word of every
 *     call is kept the same way).
 *   - All calls share the one array and nothing is cleared between calls
 *     (no scratch value is read before the kernel writes it, so the previous
 *     contents do not matter).  Calls that may overlap on the GPU (other
 *     streams, other host threads) race on the array: serialise them.
 */
hs_status hs_block_score_static(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                                const void* k, int64_t k_row_stride,
                                const int32_t* cu_seqlens, int num_docs, int total_tokens,
                                int max_seqlen, int num_heads, int dk, hs_dtype dtype,
                                float softmax_scale, int block_size,
                                float* lse, float* block_score, int nb_stride, float* block_lse,
                                hs_stream_t stream);

/* ---------------------------------------------------------------- helpers */

/* Bytes of `workspace` that op needs for these sizes (0 = none).
 * HS_OP_BLOCK_SCORE, HS_OP_BLOCK_SCORE_ATTN and the two backward ops use a
 * workspace. */
size_t hs_workspace_size(int op, int total_tokens, int num_docs, int max_seqlen,
                         int num_heads, int dk, int dv, hs_dtype dtype, int block_size);

/* Which kernel family op would run for these parameters (hs_kernel_path),
 * or -1 when the parameters are unsupported.  It sees only the shape: a
 * call whose pointers are not 16-byte aligned, whose strides are not
 * multiples of 8 elements or (block scoring) whose cu_seqlens holds more
 * than 1024 documents runs on the CUDA-core kernels even where hs_path
 * says HS_PATH_TCGEN05; hs_last_path() reports what a call actually ran. */
int hs_path(int op, hs_dtype dtype, int num_heads, int dk, int dv, int block_size);

/* Kernel family (hs_kernel_path) that the calling thread's most recent
 * successful compute call launched, or -1 before its first one.  A call
 * that launches several kernels reports HS_PATH_SIMT when any part of its
 * attention or scoring work ran on CUDA cores (top-k selection is always
 * HS_PATH_SIMT: it is no contraction).  This is how a caller detects that a
 * call left the tensor-core path because of its pointers or strides, which
 * hs_path() cannot see.  Thread-local; failed calls leave it unchanged. */
int hs_last_path(void);

/* Synchronises `stream`, then returns and clears the device-side status
 * word (HS_OK when no kernel recorded a problem).  This is the only call
 * that waits for the GPU. */
hs_status hs_poll_status(hs_stream_t stream);

/* Testing aid: when on != 0 every call uses the CUDA-core kernels even
 * where a tensor-core kernel exists.  Process-wide; not for production. */
void hs_set_force_simt(int on);

/* Failure-detection self test (no counterpart in the method): launches one
 * thread that waits on an mbarrier nothing will ever arrive at, with the
 * same bounded-wait routine the tensor-core pipelines use and a limit of
 * limit_ns nanoseconds (1 .. 10^9).  The wait gives up, the kernel records
 * HS_ERR_TIMEOUT in the device status word and returns normally; the next
 * hs_poll_status() reports it.  Nothing is in flight when it gives up. */
hs_status hs_selftest_wait(long long limit_ns, hs_stream_t stream);

const char* hs_status_string(hs_status status);

/* Message of the calling thread's most recent failed call ("" if none). */
const char* hs_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int hs_version(void);

#ifdef __cplusplus
} /* extern "C" */
#endif

#endif /* HS_H_ */
