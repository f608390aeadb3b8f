// Top-k key-block selection, one warp per query token.
//
// Rule ("HySparse MQA sparse attention ...", PaddleFleet pull request 1470,
// per-file table, pipeline.py: top-k over the recovered block scores; the
// forced blocks and the tie rule are this library's stated contract): the
// query's own block bq and the document's first block 0 are always taken and
// count toward k; the other k - 2 slots go to the largest scores among blocks
// 1 .. bq-1, an exact fp32 tie going to the lower block id.  Output ascending,
// padded with -1.
//
// Selection without sorting: the m-th largest score is found by a 32-step
// bitwise search over an order-preserving uint32 image of the fp32 scores
// (each step counts, with one warp reduction, how many candidates reach the
// trial value).  Everything above that threshold is taken, then the first
// r equal ones in index order; a ballot prefix count writes the chosen ids in
// ascending order.  The score row is read straight from global memory; its
// 32 re-reads hit L1.

#include "hs_device.cuh"
#include "hs_internal.h"

namespace hs {

namespace {

constexpr int kSelWarps = 8;

// Monotone map of fp32 to uint32 (larger float -> larger integer).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kSelWarps * 32)
select_topk_kernel(const float* __restrict__ block_score, int nb_stride,
                   const int32_t* __restrict__ cu, int num_docs, int total_tokens,
                   int max_seqlen, int block_size, int topk, int32_t* __restrict__ idx,
                   int* status) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kSelWarps + (threadIdx.x >> 5);
  if (t >= total_tokens) return;
  int32_t* out = idx + (int64_t)t * topk;
  int bos, eos;
  if (!find_doc(cu, num_docs, total_tokens, max_seqlen, t, bos, eos, status)) {
    for (int i = lane; i < topk; i += 32) out[i] = -1;
    return;
  }
  const int bq = (t - bos) / block_size;
  if (bq + 1 <= topk) {  // every candidate fits
    for (int i = lane; i < topk; i += 32) out[i] = (i <= bq) ? i : -1;
    return;
  }
  // here bq >= topk >= 1
  const bool two = topk >= 2;           // block 0 forced as well
  const int flo = two ? 1 : 0;          // free candidates [flo, bq)
  const int m = topk - (two ? 2 : 1);   // free slots
  const float* row = block_score + (int64_t)t * nb_stride;

  uint32_t theta = 0;
  if (m > 0) {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t trial = theta | (1u << bit);
      unsigned cnt = 0;
      for (int c = flo + lane; c < bq; c += 32) cnt += order_key(__ldg(row + c)) >= trial;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if ((int)cnt >= m) theta = trial;
    }
  }
  unsigned above = 0;
  if (m > 0) {
    for (int c = flo + lane; c < bq; c += 32) above += order_key(__ldg(row + c)) > theta;
    above = __reduce_add_sync(0xffffffffu, above);
  }
  const int r = m - (int)above;  // equal-to-threshold ids still to take

  const unsigned lt = (1u << lane) - 1u;
  int pos = 0, eq_seen = 0;
  for (int base = 0; base <= bq; base += 32) {
    const int c = base + lane;
    const bool in = c <= bq;
    const bool is_free = m > 0 && in && c >= flo && c < bq;
    const uint32_t key = is_free ? order_key(__ldg(row + c)) : 0u;
    const bool eq = is_free && key == theta;
    const unsigned eq_mask = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eq_mask & lt);
    const bool sel = in && (c == bq || (two && c == 0) ||
                            (is_free && (key > theta || (eq && eq_rank < r))));
    const unsigned sel_mask = __ballot_sync(0xffffffffu, sel);
    if (sel) {
      const int o = pos + __popc(sel_mask & lt);
      if (o < topk) out[o] = c;
    }
    pos += __popc(sel_mask);
    eq_seen += __popc(eq_mask);
  }
  for (int i = pos + lane; i < topk; i += 32) out[i] = -1;  // only if pos < topk
}

}  // namespace

cudaError_t launch_select_topk(const float* block_score, int nb_stride, const int32_t* cu,
                               int num_docs, int total_tokens, int max_seqlen, int block_size,
                               int topk, int32_t* idx, int* status, cudaStream_t s) {
  const int grid = (total_tokens + kSelWarps - 1) / kSelWarps;
  select_topk_kernel<<<grid, kSelWarps * 32, 0, s>>>(block_score, nb_stride, cu, num_docs,
                                                     total_tokens, max_seqlen, block_size, topk,
                                                     idx, status);
  return cudaGetLastError();
}

}  // namespace hs
