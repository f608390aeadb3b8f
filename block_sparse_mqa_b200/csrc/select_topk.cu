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
// Selection without sorting.  Each score is mapped to an order-preserving
// uint32 key; the row is read from global memory ONCE, with coalesced loads,
// into the warp's registers (32 keys per lane at most, rows of up to 1024
// candidates) or, for longer rows, into the warp's slice of shared memory.
// The m-th largest key is then found by a bitwise search over the staged
// keys: theta is built from the top bit down, and a bit is kept when at least
// m keys reach theta with that bit set (one warp reduction per bit).  Two
// things shorten the search without changing its result:
//   * bits above the highest bit in which the candidates' keys differ are
//     the same in every key, so theta starts as that common prefix;
//   * once exactly m keys reach a trial value, the top-m set is exactly
//     {key >= trial} and the search stops there.
// Finally everything above theta is taken, then the first r keys equal to it
// in block order (r = m minus the count above), and a ballot prefix count
// writes the chosen ids in ascending order.  With the early stop, theta may
// sit below the m-th largest key, but only when exactly m keys reach it,
// so no key equals the m-th without being taken: the set is the same.
//
// Rows of more than 64 candidates with m <= 32 first narrow the search:
// each lane keeps its two largest keys, and the m-th largest p of those 64
// values is found by the same search.  At least m distinct candidates reach
// p, so the top m of the row, and every key equal to the m-th largest, are
// among {key >= p}.  Those keys are copied, in block order, into a 64-entry
// list in shared memory (two per lane), and the search and the output run
// over that list instead of the whole row.  A row whose list would exceed
// 64 entries (mass ties around p) takes the full search above.

#include "hs_device.cuh"
#include "hs_internal.h"

namespace hs {

namespace {

constexpr int kSelWarps = 8;         // queries per CTA
constexpr int kRegChunks = 32;       // register path: up to 32 x 32 = 1024 candidates
constexpr int kListSlots = 2;        // narrowed list: two keys per lane
constexpr int kListCap = 32 * kListSlots;
// Longer rows are staged in shared memory: at most kMaxSelectBlocks keys
// (224 KB) plus the narrowed list (keys and ids) for one warp, within the
// 227 KB a CTA may use.
constexpr size_t kStageLimit = ((size_t)kMaxSelectBlocks + 2 * kListCap) * sizeof(uint32_t);
static_assert(kStageLimit <= 232448, "staged row and list of one warp");

// Monotone map of fp32 to uint32 (larger float -> larger integer).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Loops over a row's 32-candidate chunks run to NCH when it is a
// compile-time bound (> 0: fully unrolled, so a register array is indexed by
// constants) and stop at the row's own chunk count nch (warp-uniform).
template <int NCH>
__host__ __device__ constexpr int loop_bound() { return NCH > 0 ? NCH : 1 << 30; }

// The search over the staged keys.  KeyAt(i) returns the key of lane
// candidate i (candidates c = 32 i + lane); non-candidates hold 0, which no
// trial value (always > 0) reaches.  nch = number of 32-candidate chunks that
// can hold candidates.  Returns theta; *r_out = equal keys still to take.
template <int NCH, typename KeyAt>
__device__ __forceinline__ uint32_t search_theta(KeyAt key_at, int nch, int m, int* r_out) {
  // common prefix of every candidate key (non-candidates do not take part)
  uint32_t kand = 0xffffffffu, kor = 0u;
#pragma unroll
  for (int i = 0; i < loop_bound<NCH>(); ++i) {
    if (i >= nch) break;
    const uint32_t k = key_at(i);
    if (k != 0u) {
      kand &= k;
      kor |= k;
    }
  }
  kand = __reduce_and_sync(0xffffffffu, kand);
  kor = __reduce_or_sync(0xffffffffu, kor);
  const uint32_t diff = kand ^ kor;
  uint32_t theta;
  int bit;
  if (diff == 0u) {  // every candidate key is equal: that key is the m-th largest
    theta = kand;
    bit = -1;
  } else {
    bit = 31 - __clz(diff);
    theta = bit == 31 ? 0u : (kand >> (bit + 1)) << (bit + 1);
  }
  for (; bit >= 0; --bit) {
    const uint32_t trial = theta | (1u << bit);
    unsigned cnt = 0;
#pragma unroll
    for (int i = 0; i < loop_bound<NCH>(); ++i) {
      if (i >= nch) break;
      cnt += key_at(i) >= trial;
    }
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if ((int)cnt >= m) {
      theta = trial;
      if ((int)cnt == m) break;  // exactly the top m reach trial
    }
  }
  unsigned above = 0;
#pragma unroll
  for (int i = 0; i < loop_bound<NCH>(); ++i) {
    if (i >= nch) break;
    above += key_at(i) > theta;
  }
  above = __reduce_add_sync(0xffffffffu, above);
  *r_out = m - (int)above;
  return theta;
}

// Ascending output of the selected ids (forced blocks, keys above theta, and
// the first r keys equal to theta in block order), then -1 padding.
template <int NCH, typename KeyAt>
__device__ __forceinline__ void write_selection(KeyAt key_at, int nch, int bq, bool two,
                                                uint32_t theta, int r, int topk, int32_t* out) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  int pos = 0, eq_seen = 0;
#pragma unroll
  for (int i = 0; i < loop_bound<NCH>(); ++i) {
    if (i >= nch) break;
    const int c = 32 * i + lane;
    const bool in = c <= bq;
    const uint32_t key = key_at(i);  // 0 unless c is a free candidate
    const bool eq = key != 0u && key == theta;
    const unsigned eq_mask = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eq_mask & lt);
    const bool sel = in && (c == bq || (two && c == 0) ||
                            (key != 0u && (key > theta || (eq && eq_rank < r))));
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

// The narrowed selection for rows with 1 <= m <= 32 free slots (see the
// file comment).  list_key / list_id: this warp's kListCap-entry buffers in
// shared memory.  nch is a multiple of G (chunks past the row hold 0), so
// the loops test their bound once per G chunks.  Returns false, having
// written nothing, when more than kListCap keys reach the pivot; the caller
// then runs the full search.
template <int NCH, int G, typename KeyAt>
__device__ __forceinline__ bool select_narrowed(KeyAt key_at, int nch, int m, int bq, bool two,
                                                int32_t* out, uint32_t* list_key,
                                                uint32_t* list_id) {
  const int lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  uint32_t a = 0u, b = 0u;  // this lane's largest and second-largest key
#pragma unroll
  for (int i = 0; i < loop_bound<NCH>(); ++i) {
    if (i % G == 0 && i >= nch) break;
    const uint32_t k = key_at(i);
    b = max(b, min(a, k));
    a = max(a, k);
  }
  // pivot: the m-th largest of the 64 values, or 1 (every candidate) when
  // fewer than m of them are candidates
  uint32_t pivot = 1u;
  const int nz = __popc(__ballot_sync(0xffffffffu, a != 0u)) +
                 __popc(__ballot_sync(0xffffffffu, b != 0u));
  if (nz >= m) {
    int r_unused;
    auto two_at = [&](int j) -> uint32_t { return j == 0 ? a : b; };
    pivot = max(search_theta<kListSlots>(two_at, kListSlots, m, &r_unused), 1u);
  }
  // copy every key >= pivot into the list, in block order
  int n = 0;
#pragma unroll
  for (int i = 0; i < loop_bound<NCH>(); ++i) {
    if (i % G == 0 && i >= nch) break;
    const uint32_t k = key_at(i);
    const bool in = k >= pivot;
    const unsigned mask = __ballot_sync(0xffffffffu, in);
    const int o = n + __popc(mask & lt);
    if (in && o < kListCap) {
      list_key[o] = k;
      list_id[o] = (uint32_t)(32 * i + lane);
    }
    n += __popc(mask);
  }
  if (n > kListCap) return false;
  __syncwarp();
  uint32_t lk[kListSlots], li[kListSlots];
#pragma unroll
  for (int j = 0; j < kListSlots; ++j) {
    const int q = 32 * j + lane;
    lk[j] = q < n ? list_key[q] : 0u;
    li[j] = q < n ? list_id[q] : 0u;
  }
  int r;
  auto list_at = [&](int j) -> uint32_t { return lk[j]; };
  const uint32_t theta = search_theta<kListSlots>(list_at, kListSlots, m, &r);
  // output: block 0 (forced), the chosen list entries in block order, bq
  int pos = two ? 1 : 0, eq_seen = 0;
#pragma unroll
  for (int j = 0; j < kListSlots; ++j) {
    const uint32_t key = lk[j];
    const bool eq = key != 0u && key == theta;
    const unsigned eq_mask = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eq_mask & lt);
    const bool sel = key != 0u && (key > theta || (eq && eq_rank < r));
    const unsigned sel_mask = __ballot_sync(0xffffffffu, sel);
    if (sel) out[pos + __popc(sel_mask & lt)] = (int32_t)li[j];
    pos += __popc(sel_mask);
    eq_seen += __popc(eq_mask);
  }
  if (lane == 0) {  // pos == topk - 1: exactly m free blocks were taken
    if (two) out[0] = 0;
    out[pos] = bq;
  }
  return true;
}

// Per-query set-up shared by the kernels.  Returns false when the row is
// finished already (no document, or every candidate fits).
__device__ __forceinline__ bool begin_row(const int32_t* cu, int num_docs, int total_tokens,
                                          int max_seqlen, int block_size, int topk, int t,
                                          int32_t* out, int* status, int& bq) {
  const int lane = threadIdx.x & 31;
  int bos, eos;
  if (!find_doc(cu, num_docs, total_tokens, max_seqlen, t, bos, eos, status)) {
    for (int i = lane; i < topk; i += 32) out[i] = -1;
    return false;
  }
  bq = (t - bos) / block_size;
  if (bq + 1 <= topk) {  // every candidate fits
    for (int i = lane; i < topk; i += 32) out[i] = (i <= bq) ? i : -1;
    return false;
  }
  return true;  // here bq >= topk >= 1
}

// Rows of up to 32 * NCH candidates: the keys live in registers.
template <int NCH>
__global__ void __launch_bounds__(kSelWarps * 32, NCH >= 32 ? 5 : 6)
select_topk_reg_kernel(const float* __restrict__ block_score, int nb_stride,
                       const int32_t* __restrict__ cu, int num_docs, int total_tokens,
                       int max_seqlen, int block_size, int topk, int32_t* __restrict__ idx,
                       int* status) {
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * kSelWarps + (threadIdx.x >> 5);
  if (t >= total_tokens) return;
  int32_t* out = idx + (int64_t)t * topk;
  int bq;
  if (!begin_row(cu, num_docs, total_tokens, max_seqlen, block_size, topk, t, out, status, bq))
    return;
  const bool two = topk >= 2;          // block 0 forced as well
  const int flo = two ? 1 : 0;         // free candidates [flo, bq)
  const int m = topk - (two ? 2 : 1);  // free slots
  const int nch = bq / 32 + 1;         // chunks holding candidates 0 .. bq
  const float* row = block_score + (int64_t)t * nb_stride;
  // chunks are loaded in groups of four (NCH >= 4): entries past the row's
  // last group are never read, those between nch and the group's end hold 0
  constexpr int G = NCH >= 4 ? 4 : 1;
  const int nchg = (nch + G - 1) / G * G;
  uint32_t key[NCH];
#pragma unroll
  for (int i = 0; i < NCH; ++i) {  // one coalesced pass over the row
    if (i % G == 0 && i >= nchg) break;
    const int c = 32 * i + lane;
    key[i] = (c >= flo && c < bq) ? order_key(__ldg(row + c)) : 0u;
  }
  // every loop over the chunks is unrolled to NCH, so i is a constant here
  auto key_at = [&](int i) -> uint32_t { return key[i]; };
  if (NCH > 2 && nch > 2 && m >= 1 && m <= 32) {
    __shared__ uint32_t list[kSelWarps][2][kListCap];
    const int w = threadIdx.x >> 5;
    if (select_narrowed<NCH, G>(key_at, nchg, m, bq, two, out, list[w][0], list[w][1])) return;
  }
  uint32_t theta = 0xffffffffu;  // no free slot (m = 0): no key is above theta
  int r = 0;
  if (m > 0) theta = search_theta<NCH>(key_at, nch, m, &r);
  write_selection<NCH>(key_at, nch, bq, two, theta, r, topk, out);
}

// Longer rows: the keys are staged in this warp's slice of shared memory.
__global__ void __launch_bounds__(kSelWarps * 32)
select_topk_long_kernel(const float* __restrict__ block_score, int nb_stride,
                        const int32_t* __restrict__ cu, int num_docs, int total_tokens,
                        int max_seqlen, int block_size, int topk, int32_t* __restrict__ idx,
                        int* status, int slice) {
  extern __shared__ uint32_t stage[];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int t = blockIdx.x * (blockDim.x >> 5) + w;
  if (t >= total_tokens) return;
  int32_t* out = idx + (int64_t)t * topk;
  int bq;
  if (!begin_row(cu, num_docs, total_tokens, max_seqlen, block_size, topk, t, out, status, bq))
    return;
  const bool two = topk >= 2;
  const int flo = two ? 1 : 0;
  const int m = topk - (two ? 2 : 1);
  const int nch = bq / 32 + 1;
  const float* row = block_score + (int64_t)t * nb_stride;
  uint32_t* keys = stage + (size_t)w * (slice + 2 * kListCap);
  for (int i = 0; i < nch; ++i) {  // one coalesced pass over the row
    const int c = 32 * i + lane;
    keys[c] = (c >= flo && c < bq) ? order_key(__ldg(row + c)) : 0u;
  }
  __syncwarp();
  auto key_at = [&](int i) -> uint32_t { return keys[32 * i + lane]; };
  if (m >= 1 && m <= 32 &&
      select_narrowed<0, 1>(key_at, nch, m, bq, two, out, keys + slice, keys + slice + kListCap))
    return;
  uint32_t theta = 0xffffffffu;  // no free slot (m = 0): no key is above theta
  int r = 0;
  if (m > 0) theta = search_theta<0>(key_at, nch, m, &r);
  write_selection<0>(key_at, nch, bq, two, theta, r, topk, out);
}

template <int NCH>
cudaError_t launch_reg(const float* bs, int nbs, const int32_t* cu, int nd, int T, int ms, int B,
                       int k, int32_t* idx, int* st, cudaStream_t s) {
  const int grid = (T + kSelWarps - 1) / kSelWarps;
  select_topk_reg_kernel<NCH><<<grid, kSelWarps * 32, 0, s>>>(bs, nbs, cu, nd, T, ms, B, k, idx,
                                                              st);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select_topk(const float* block_score, int nb_stride, const int32_t* cu,
                               int num_docs, int total_tokens, int max_seqlen, int block_size,
                               int topk, int32_t* idx, int* status, cudaStream_t s) {
  // candidates of a row: blocks 0 .. bq <= NBmax - 1
  const int nbmax = (max_seqlen + block_size - 1) / block_size;
  const int nch = (nbmax + 31) / 32;
  auto a = [&](auto fn) {
    return fn(block_score, nb_stride, cu, num_docs, total_tokens, max_seqlen, block_size, topk,
              idx, status, s);
  };
  if (nch <= 1) return a(launch_reg<1>);
  if (nch <= 2) return a(launch_reg<2>);
  if (nch <= 4) return a(launch_reg<4>);
  if (nch <= 8) return a(launch_reg<8>);
  if (nch <= 16) return a(launch_reg<16>);
  if (nch <= kRegChunks) return a(launch_reg<kRegChunks>);
  // longer rows: one warp's slice of shared memory holds a row's keys (the
  // host has refused rows past kMaxSelectBlocks)
  const int slice = nch * 32;
  const size_t per_warp = ((size_t)slice + 2 * kListCap) * sizeof(uint32_t);
  if (per_warp > kStageLimit) return cudaErrorInvalidValue;
  int warps = (int)(kStageLimit / per_warp);
  if (warps > kSelWarps) warps = kSelWarps;
  const size_t smem = (size_t)warps * per_warp;
  cudaError_t e = cudaFuncSetAttribute(select_topk_long_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = (total_tokens + warps - 1) / warps;
  select_topk_long_kernel<<<grid, warps * 32, smem, s>>>(block_score, nb_stride, cu, num_docs,
                                                         total_tokens, max_seqlen, block_size,
                                                         topk, idx, status, slice);
  return cudaGetLastError();
}

}  // namespace hs
