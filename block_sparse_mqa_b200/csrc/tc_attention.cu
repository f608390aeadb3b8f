// hs_sparse_mqa_fwd, hs_swa_mqa_fwd and the full layer's fused forward
// (hs_block_score_attn_fwd) on tcgen05 tensor cores (bf16 in, fp32
// accumulate), 64 query heads over one KV head.
//
// Definitions ("HySparse MQA sparse attention ...", PaddleFleet pull request
// 1470, "Core" list: block-sparse DSA gather and SWA sliding-window MQA, both
// with a learnable per-head attn_sink; "Support attn sink in fa3", pull
// request 1415: the sink is a softmax-denominator offset):
//   lse[t,h] = log(exp(sink_h) + sum_{j in S_t} exp(s_j)),
//   out[t,h] = sum_{j in S_t} exp(s_j - lse[t,h]) v_j,
// with S_t the selected blocks (causal inside the own block) or the window.
// The full layer ("Core" list: FA4-fused block scoring; the Copilot overview:
// the HySparse full layer yields the block indices) attends every causal key
// without a sink and also emits, from the same fp32 exponentials,
//   block_lse[t,h,b] = log sum_{j in block b, j <= t} exp(s_j),
//   block_score[t,b] = sum_h exp(block_lse[t,h,b] - lse[t,h]).
//
// Design.  Every query token has its own key set, so its 64 heads are the
// only rows that share a key tile.  The kernel therefore works transposed:
//   S^T[128 keys x 64 heads]  = K_tile (A, K-major) . Q_t^T (B, K-major)
//   O^T[Dv x 64 heads]       += V_tile^T (A, MN-major) . P^T (B, MN-major)
// so every MMA has M = 128 (full tcgen05 rate) and N = 64.  TMEM holds the
// four 128-row dv chunks of O^T (256 columns) and two S^T buffers (128).
// One persistent CTA per SM walks tokens; per token the key tiles are
// 128 keys: 128/B selected blocks gathered by per-block TMA boxes (unused
// slots repeat the own block, masked), or one contiguous window slice.
// Two rings of two 32 KB slots carry K (two 64-column chunks per stage) and
// V (one 128-row dv chunk per stage); two MMA-issuing threads consume them:
// one issues every QK (S^T of tile i+1 runs while the softmax works on tile
// i), the other every PV once the softmax has written P.  The softmax
// warps (thread = key row) reduce per-head maxima across the 128 rows with a
// 32-lane transpose-reduction plus a 4-warp combine, keep the running max
// per head (raised only when a tile beats it by more than 2^8, which then
// rescales O^T in TMEM), write P^T as bf16 into one 128-byte-swizzled buffer
// and accumulate per-head sums in registers.  The sink joins in the
// epilogue, which reads O^T back per dv row, stages each 128-row dv chunk
// as [head][dv] in the P^T buffer and stores it to out[t, h, :] with one TMA
// tensor store per warpgroup.
// Warp 0 = K producer, warp 10 = V producer, warp 1 = QK issuer / TMEM
// owner, warp 11 = PV issuer, warps 2-9 = two softmax warpgroups, each
// owning 32 of the 64 heads (per-head state never crosses warpgroups).  All
// waits are bounded (HS_ERR_TIMEOUT, drain, free).
//
// Full-layer mode: each key tile covers 128 / B whole blocks (B >= 32, so a
// block is one or more whole warps of key rows).  After the exponentials
// every warp transposes-and-sums its 32 rows per head; at the warpgroup's
// next rendezvous the warps of each block add their sums and write
// log2(sum) + running max (the block's LSE in log2 units) to a per-CTA
// scratch row [block][head] in global memory (L2-resident; two rows per CTA,
// alternating by token, since one token's rows are read while the next
// token's are written).  After the token's last tile both warpgroups meet
// (a bounded 256-thread barrier) and each warp turns blocks into scores:
// lanes take two heads each, exp2(block LSE - row LSE), a fixed-order warp
// sum.

#include <math.h>

#include "hs_device.cuh"
#include "hs_internal.h"
#include "tc_common.cuh"
#include "tc_host.h"

namespace hs {
namespace {

using namespace tc;

constexpr int kThreads = 384;  // 2 producers, 2 MMA issuers, 2 softmax warpgroups
constexpr int kH = 64;              // heads (N of every MMA)
constexpr int kTile = 128;          // keys per tile (M of the QK MMA)
constexpr int kSlots = 2;           // slots of each ring (K ring, V ring)
constexpr int kSlotBytes = 32768;   // two 128 x 64 bf16 panels
constexpr int kVProdWarp = 10;      // V producer warp
constexpr int kPvWarp = 11;         // PV MMA-issuing warp
constexpr int kPanel = 16384;
constexpr int kQChunkBytes = kH * 64 * 2;  // 8 KB
constexpr int kMaxQChunks = 9;      // Dk <= 576
constexpr int kPBytes = kTile * kH * 2;    // 16 KB
constexpr int kSCol = 256;          // S^T buffers at 256 and 320
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kRescaleLog2 = 8.f;  // raise the running max only past 2^8

// kModeSwaLayer: the window attention with the combining epilogue
constexpr int kModeSwa = 0, kModeSparse = 1, kModeFull = 2, kModeSwaLayer = 3;

struct AttnParams {
  const int32_t* cu;
  int num_docs, T, max_seqlen;
  const int32_t* idx;
  int topk, B, window;
  int nck, nvc;  // 64-column K chunks, 128-row V chunks (the last may be half past Dv)
  int dv;
  float scale_log2;
  const float* sink;
  __nv_bfloat16* out;
  float* lse;
  int* status;
  long long wait_ns;
  // full-layer mode only
  float* blk;          // scratch: [gridDim.x][2][nbmax][kH] block LSEs (log2 units)
  int nbmax, nb_stride;
  float* block_score;  // [T, nb_stride]
  float* block_lse;    // [T, kH, nb_stride] or null
  // combining epilogue (the SWA layer): out = gate_own * this attention +
  // gate_prev * prev, prev [T, kH, Dv] bf16 (may be out itself); null = off
  const __nv_bfloat16* prev;
  const float* gate_own;   // [T, kH] or null (= 1)
  const float* gate_prev;  // [T, kH] or null (= 1)
};

struct Shared {
  uint64_t kfull[kSlots], kempty[kSlots];  // K ring
  uint64_t vfull[kSlots], vempty[kSlots];  // V ring
  uint64_t qfull[kMaxQChunks], qempty[kMaxQChunks];
  uint64_t sfull[2], sempty[2];
  uint64_t pfull, pvdone, ofull, oempty, drain, drain_pv;
  uint64_t ochunk[4];        // O^T chunk c read out of TMEM (early epilogue)
  uint64_t rv[2];            // rendezvous inside softmax warpgroup wg (128 threads)
  uint64_t rv_all;           // rendezvous of both softmax warpgroups (full-layer mode)
  float red[2][4][32];       // [warpgroup][warp][lane] partial reductions
  float bsum[2][4][32];      // [warpgroup][warp][head] one tile's exp sums (full layer)
  float lse2[kH];            // row LSE per head, log2 units (full layer)
  float gprev[kH];           // gate of prev per head (combining epilogue)
  float mrun[kH];            // running max per head (log2 domain)
  float alpha[kH];           // rescale factor per head
  float lsum[kH];            // output multiplier per head
  int rescale[2][2];         // [warpgroup][tile parity]: some head's max rose
  int plist[2][256];         // each producer's (K, V) selected-block list of its token
  int blist[2][256];         // each softmax warpgroup's list of its token
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kSmemBytes =
    1024 + (size_t)2 * kSlots * kSlotBytes + (size_t)kMaxQChunks * kQChunkBytes + kPBytes +
    sizeof(Shared);

__device__ __forceinline__ bool aborted(Shared* sh) {
  return *reinterpret_cast<volatile int*>(&sh->abort_flag) != 0;
}
__device__ __forceinline__ void give_up(Shared* sh, int* status) {
  record_status(status, HS_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&sh->abort_flag) = 1;
}

// Token bookkeeping shared by all roles (each role derives it on its own,
// deterministically, from cu_seqlens and idx).
struct TokenPlan {
  bool ok;
  int bos, eos, bq;
  int wlo;    // window start (SWA)
  int nkeys;  // SWA: keys in the window
  int nsel;   // sparse: valid selected blocks
  int ntile;
};

// Index rule shared by every role: entry s of idx[t] is a selected block when
// 0 <= b <= bq(t) and b is larger than the raw entry before it (ascending,
// no duplicates; -1 padding fails the first test).  Rows that break it get
// the offending entries skipped and HS_ERR_INVALID_INDEX reported.
__device__ __forceinline__ bool entry_ok(const int32_t* row, int s, int bq, int& b) {
  b = __ldg(row + s);
  return b >= 0 && b <= bq && (s == 0 || b > __ldg(row + s - 1));
}

template <bool kSparse>
__device__ __forceinline__ TokenPlan plan_token(const AttnParams& p, int t, bool report) {
  TokenPlan tp;
  tp.ok = find_doc(p.cu, p.num_docs, p.T, p.max_seqlen, t, tp.bos, tp.eos,
                   report ? p.status : nullptr);
  tp.bq = tp.ok ? (t - tp.bos) / p.B : 0;
  tp.wlo = 0;
  tp.nkeys = 0;
  tp.nsel = 0;
  tp.ntile = 0;
  if (!tp.ok) return tp;
  if (kSparse) {
    const int32_t* row = p.idx + (int64_t)t * p.topk;
    int n = 0;
    bool bad = false;
    for (int s = 0; s < p.topk; ++s) {
      int b;
      if (entry_ok(row, s, tp.bq, b)) ++n;
      else if (b >= 0) bad = true;
    }
    if (bad && report) record_status(p.status, HS_ERR_INVALID_INDEX);
    tp.nsel = n;
    const int per = kTile / p.B;
    tp.ntile = (n + per - 1) / per;
  } else {
    tp.wlo = max(tp.bos, t - p.window + 1);
    tp.nkeys = t - tp.wlo + 1;
    tp.ntile = (tp.nkeys + kTile - 1) / kTile;
  }
  return tp;
}

// The same plan computed by a whole warp (every lane calls it and gets the
// result): the idx row is read with one coalesced load per 32 entries and
// the index rule is evaluated per lane, the raw entry before it coming from
// the neighbouring lane.  When `list` is not null the selected blocks are
// written to it in order (compacted by ballot).  One L2 round trip per 32
// entries instead of a serial walk over the row.
template <bool kSparse>
__device__ __forceinline__ TokenPlan plan_token_warp(const AttnParams& p, int t, bool report,
                                                     int* list) {
  const int lane = threadIdx.x & 31;
  TokenPlan tp;
  tp.ok = find_doc(p.cu, p.num_docs, p.T, p.max_seqlen, t, tp.bos, tp.eos,
                   (report && lane == 0) ? p.status : nullptr);
  tp.bq = tp.ok ? (t - tp.bos) / p.B : 0;
  tp.wlo = 0;
  tp.nkeys = 0;
  tp.nsel = 0;
  tp.ntile = 0;
  if (!tp.ok) return tp;
  if (kSparse) {
    const int32_t* row = p.idx + (int64_t)t * p.topk;
    int n = 0, prev_last = 0;
    bool bad = false;
    for (int base = 0; base < p.topk; base += 32) {
      const int s = base + lane;
      const int b = s < p.topk ? __ldg(row + s) : -1;
      int prev = __shfl_up_sync(0xffffffffu, b, 1);
      if (lane == 0) prev = prev_last;  // the previous 32 entries' last one
      const bool v = b >= 0 && b <= tp.bq && (s == 0 || b > prev);
      const unsigned m = __ballot_sync(0xffffffffu, v);
      if (list && v) list[n + __popc(m & ((1u << lane) - 1u))] = b;
      n += __popc(m);
      bad = __any_sync(0xffffffffu, b >= 0 && !v) || bad;
      prev_last = __shfl_sync(0xffffffffu, b, 31);
    }
    if (bad && report && lane == 0) record_status(p.status, HS_ERR_INVALID_INDEX);
    tp.nsel = n;
    const int per = kTile / p.B;
    tp.ntile = (n + per - 1) / per;
  } else {
    tp.wlo = max(tp.bos, t - p.window + 1);
    tp.nkeys = t - tp.wlo + 1;
    tp.ntile = (tp.nkeys + kTile - 1) / kTile;
  }
  return tp;
}

// 32-lane transpose reductions: lane i receives op over lanes of v[i].
__device__ __forceinline__ float tr_max(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < off; ++j) {
      const float send = upper ? v[j] : v[j + off];
      const float keep = upper ? v[j + off] : v[j];
      v[j] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, off));
    }
  }
  return v[0];
}
__device__ __forceinline__ float tr_sum(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < off; ++j) {
      const float send = upper ? v[j] : v[j + off];
      const float keep = upper ? v[j + off] : v[j];
      v[j] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0];
}

// Bounded rendezvous of the 128 threads of softmax warpgroup wg.
__device__ __forceinline__ bool rendezvous(Shared* sh, int wg, uint32_t& ph, long long lim) {
  mbar_arrive(&sh->rv[wg]);
  const bool ok = mbar_wait(&sh->rv[wg], ph, lim);
  ph ^= 1;
  return ok;
}

// An SS MMA issued only when `on` (a guard predicate on the instruction,
// not a branch around it).
__device__ __forceinline__ void umma_ss_if(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate, uint32_t on) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 q, %5, 0;\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(on)
      : "memory");
}

// NP K chunks with a compile-time first accumulate flag (the narrow-Dk
// instantiations; see mma_run_qk).
template <int NP, bool FIRST>
__device__ __forceinline__ void mma_run(uint32_t d, uint64_t a0, uint64_t b0, uint32_t idesc) {
#pragma unroll
  for (int pn = 0; pn < NP; ++pn)
#pragma unroll
    for (int k = 0; k < 4; ++k)
      umma_ss(d, a0 + (uint64_t)((pn * kPanel) >> 4) + 2 * k,
              b0 + (uint64_t)((pn * kQChunkBytes) >> 4) + 2 * k, idesc,
              (FIRST && pn == 0 && k == 0) ? 0u : 1u);
}

// One K stage: two K chunks (4 MMAs each, M=128 keys, N=64 heads, K=16)
// into S^T at d; A = K panels 16 KB apart, B = Q chunks 8 KB apart.  The
// second chunk is issued only when `two`; the chunk count and the first
// accumulate flag are runtime values, with no branch between the MMAs.  The
// wide-Dk instantiations (Dk > 256) use this form (sparse 0.771 -> 0.753 ms,
// SWA 0.408 -> 0.398 ms at Dk 576); the narrow ones keep the earlier issuer
// code with the templated variants above (the wide code measured ~6 %
// slower at Dk 192 / Dv 128).
__device__ __forceinline__ void mma_run_qk(uint32_t d, uint64_t a0, uint64_t b0, uint32_t idesc,
                                           uint32_t acc0, uint32_t two) {
#pragma unroll
  for (int k = 0; k < 4; ++k)
    umma_ss(d, a0 + 2 * k, b0 + 2 * k, idesc, k == 0 ? acc0 : 1u);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    umma_ss_if(d, a0 + (uint64_t)(kPanel >> 4) + 2 * k, b0 + (uint64_t)(kQChunkBytes >> 4) + 2 * k,
               idesc, 1u, two);
}

// One 128-row dv chunk: O^T[c] (+)= V^T (MN-major, two 64-row panels) . P^T
// over 128 keys = 8 MMAs (K=16 keys each, 16 key rows = 2 KB per step).
__device__ __forceinline__ void pv_run(uint32_t d, uint64_t a0, uint64_t b0, uint32_t idesc,
                                       uint32_t acc0) {
#pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk)
    umma_ss(d, a0 + (uint64_t)(kk * 128), b0 + (uint64_t)(kk * 128), idesc,
            kk == 0 ? acc0 : 1u);
}

// pv_run with a compile-time first accumulate flag (narrow-Dk instantiations).
template <bool FIRST>
__device__ __forceinline__ void pv_run_t(uint32_t d, uint64_t a0, uint64_t b0, uint32_t idesc) {
#pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk)
    umma_ss(d, a0 + (uint64_t)(kk * 128), b0 + (uint64_t)(kk * 128), idesc,
            (FIRST && kk == 0) ? 0u : 1u);
}

template <int kMode, bool kWide>
__global__ void __launch_bounds__(kThreads, 1)
tc_attention_kernel(const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap,
                    const __grid_constant__ CUtensorMap qmap,
                    const __grid_constant__ CUtensorMap omap, const AttnParams p) {
  constexpr bool kSparse = kMode == kModeSparse;
  constexpr bool kFull = kMode == kModeFull;
  constexpr bool kCombine = kMode == kModeSwaLayer;
  // The plain modes defer a token's epilogue until the next token's first P
  // tile is written, and release O^T chunk by chunk to that token's first PV
  // (the other modes stage their output through the P^T buffer).
  constexpr bool kEarly = kMode == kModeSwa || kMode == kModeSparse;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ring = base;
  uint8_t* vring = ring + kSlots * kSlotBytes;
  uint8_t* qbuf = vring + kSlots * kSlotBytes;
  uint8_t* pbuf = qbuf + kMaxQChunks * kQChunkBytes;
  Shared* sh = reinterpret_cast<Shared*>(pbuf + kPBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sh->kfull[s], 1);
      mbar_init(&sh->kempty[s], 1);
      mbar_init(&sh->vfull[s], 1);
      mbar_init(&sh->vempty[s], 1);
    }
    for (int c = 0; c < kMaxQChunks; ++c) {
      mbar_init(&sh->qfull[c], 1);
      mbar_init(&sh->qempty[c], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh->sfull[b], 1);
      mbar_init(&sh->sempty[b], 256);
      mbar_init(&sh->rv[b], 128);
    }
    mbar_init(&sh->rv_all, 256);
    mbar_init(&sh->pfull, 256);
    mbar_init(&sh->pvdone, 1);
    mbar_init(&sh->ofull, 1);
    mbar_init(&sh->oempty, 256);
    for (int c = 0; c < 4; ++c) mbar_init(&sh->ochunk[c], 256);
    mbar_init(&sh->drain, 1);
    mbar_init(&sh->drain_pv, 1);
    fence_barrier_init();
    sh->abort_flag = 0;
    sh->rescale[0][0] = sh->rescale[0][1] = sh->rescale[1][0] = sh->rescale[1][1] = 0;
  }
  if (warp == 1) tmem_alloc(&sh->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const int G = gridDim.x;
  const long long lim = p.wait_ns;
  const int per = kSparse ? kTile / p.B : 1;  // boxes per panel
  const int box_rows = kSparse ? p.B : kTile;

  if (warp == 0 || warp == kVProdWarp) {
    // ------------------------------------------------------------ producers
    // Warp 0 feeds the K ring (and the token's q chunks), warp kVProdWarp
    // the V ring, each in its consumer's order.  The whole warp issues: lane
    // 0 waits for a free slot and arms its barrier with the stage's bytes,
    // then the stage's TMA boxes are spread over the lanes (a single thread
    // issues a box only every few hundred cycles, too slow for the
    // per-block gather).
    const bool is_v = warp == kVProdWarp;
    uint64_t* const fullb = is_v ? sh->vfull : sh->kfull;
    uint64_t* const emptyb = is_v ? sh->vempty : sh->kempty;
    uint8_t* const rbase = is_v ? vring : ring;
    const CUtensorMap* const map = is_v ? &vmap : &kmap;
    int* const plist = sh->plist[is_v ? 1 : 0];
    if (lane == 0) {
      tma_prefetch_desc(map);
      if (!is_v) tma_prefetch_desc(&qmap);
    }
    int fills[kSlots], qfills[kMaxQChunks];
    for (int s = 0; s < kSlots; ++s) fills[s] = 0;
    for (int c = 0; c < kMaxQChunks; ++c) qfills[c] = 0;
    uint32_t slot = 0, ph = 0;
    bool stop = false;
    // one ring stage: K (two 64-column chunks) or V (one 128-row dv chunk)
    auto load_stage = [&](const TokenPlan& tp, int tile, int idx2) -> bool {
      const int npanel = is_v ? 2 : min(2, p.nck - 2 * idx2);
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait(&emptyb[slot], ph ^ 1, lim);
        if (ok) mbar_expect_tx(&fullb[slot], npanel * kPanel);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) return false;
      __syncwarp();
      uint8_t* dst = rbase + slot * kSlotBytes;
      for (int bx = lane; bx < npanel * per; bx += 32) {
        const int pn = bx / per, j = bx - pn * per;
        const int col = (idx2 * 2 + pn) * 64;
        int row0;
        if (kSparse) {
          const int slotn = tile * per + j;  // past the list: masked filler (own block)
          const int b = slotn < tp.nsel ? plist[slotn] : tp.bq;
          row0 = tp.bos + b * p.B;
        } else {
          row0 = tp.wlo + tile * kTile;
        }
        tma_load_2d(dst + pn * kPanel + j * box_rows * 128, map, &fullb[slot], col, row0);
      }
      ++fills[slot];
      if (++slot == kSlots) {
        slot = 0;
        ph ^= 1;
      }
      return true;
    };
    const int nst = is_v ? p.nvc : (p.nck + 1) / 2;  // stages per tile
    for (int t = blockIdx.x; t < p.T && !stop; t += G) {
      // the token's plan and selected blocks (plist), read by the whole warp
      const TokenPlan tp = plan_token_warp<kSparse>(p, t, !is_v, kSparse ? plist : nullptr);
      if (!tp.ok || tp.ntile == 0) continue;
      __syncwarp();  // plist complete before any lane reads it
      if (!is_v) {
        // Q_t chunks (lane c loads chunk c), each as soon as the previous
        // token's last QK released it
        int qok = 1;
        if (lane < p.nck) {
          const int c = lane;
          if (qfills[c] > 0) qok = mbar_wait(&sh->qempty[c], (qfills[c] - 1) & 1, lim);
          if (qok) {
            mbar_expect_tx(&sh->qfull[c], kQChunkBytes);
            tma_load_3d(qbuf + c * kQChunkBytes, &qmap, &sh->qfull[c], c * 64, 0, t);
            ++qfills[c];
          }
        }
        if (!__all_sync(0xffffffffu, qok)) {
          stop = true;
          break;
        }
      }
      for (int i = 0; i < tp.ntile && !stop; ++i)
        for (int s = 0; s < nst && !stop; ++s) stop = !load_stage(tp, i, s);
      __syncwarp();  // plist is rewritten for the next token only after all lanes used it
    }
    if (stop && lane == 0) give_up(sh, p.status);
    // no copy may still be landing when the CTA exits
    if (lane == 0)
      for (int s = 0; s < kSlots; ++s)
        if (fills[s] > 0) mbar_wait(&fullb[s], (fills[s] - 1) & 1, kDefaultWaitNs);
    if (!is_v && lane < p.nck && qfills[lane] > 0)
      mbar_wait(&sh->qfull[lane], (qfills[lane] - 1) & 1, kDefaultWaitNs);
  } else if (warp == 1 || warp == kPvWarp) {
    // ------------------------------------------------------------ MMA issuers
    // Two independent instruction streams (QK on warp 1, PV on warp
    // kPvWarp): each thread's waits and bookkeeping between its runs of
    // MMAs overlap with the other thread's MMAs (measured: 88 -> 53 cycles
    // per N=64 MMA with two issuers instead of one).
    const bool is_pv = warp == kPvWarp;
    if (lane == 0) {
      constexpr uint32_t id_qk = idesc_bf16_f32(128, kH, false, false);
      constexpr uint32_t id_pv = idesc_bf16_f32(128, kH, true, true);
      const uint64_t ring_desc_k = umma_desc_sw128(smem_u32(ring), 16, 1024);
      const uint64_t ring_desc_v = umma_desc_sw128(smem_u32(vring), kPanel, 1024);
      const uint64_t q_desc = umma_desc_sw128(smem_u32(qbuf), 16, 1024);
      const uint64_t p_desc = umma_desc_sw128(smem_u32(pbuf), kPanel, 1024);
      uint32_t slot = 0, ph = 0, sidx = 0, npv = 0, ntok = 0;
      int qtok = 0;
      bool issued = false, stop = false;
      auto next_slot = [&]() {
        if (++slot == kSlots) {
          slot = 0;
          ph ^= 1;
        }
      };
      // S^T(tile) = K_tile . Q^T into S buffer sidx & 1.  Each ring stage
      // (two 64-column chunks) is one run of MMAs with no branch inside.
      auto qk_stage = [&](uint32_t d, uint64_t a, uint64_t b, int s, bool two) {
        if constexpr (kWide) {
          mma_run_qk(d, a, b, id_qk, s == 0 ? 0u : 1u, two ? 1u : 0u);
        } else if (s == 0) {
          if (two) mma_run<2, true>(d, a, b, id_qk); else mma_run<1, true>(d, a, b, id_qk);
        } else {
          if (two) mma_run<2, false>(d, a, b, id_qk); else mma_run<1, false>(d, a, b, id_qk);
        }
      };
      auto qk = [&](bool first_tile, bool last_tile) -> bool {
        const uint32_t buf = sidx & 1, use = sidx >> 1;
        if (!mbar_wait_spin(&sh->sempty[buf], (use & 1) ^ 1, lim)) return false;
        tc_fence_after();
        const uint32_t d = tmem + kSCol + buf * kH;
        for (int s = 0; s < (p.nck + 1) / 2; ++s) {
          const int c0 = 2 * s;
          const bool two = c0 + 1 < p.nck;
          if (!mbar_wait_spin(&sh->kfull[slot], ph, lim)) return false;  // TMA stage
          if (first_tile) {  // the token's q chunks (resident for all its tiles)
            if (!mbar_wait_spin(&sh->qfull[c0], qtok & 1, lim)) return false;
            if (two && !mbar_wait_spin(&sh->qfull[c0 + 1], qtok & 1, lim)) return false;
          }
          const uint64_t a = ring_desc_k + (uint64_t)((slot * kSlotBytes) >> 4);
          const uint64_t b = q_desc + (uint64_t)((c0 * kQChunkBytes) >> 4);
          qk_stage(d, a, b, s, two);
          if (last_tile) {  // the token's last QK has read these Q chunks
            umma_commit(&sh->qempty[c0]);
            if (two) umma_commit(&sh->qempty[c0 + 1]);
          }
          umma_commit(&sh->kempty[slot]);
          next_slot();
        }
        umma_commit(&sh->sfull[buf]);
        ++sidx;
        issued = true;
        return true;
      };
      // O^T += V_tile^T . P^T (waits for P of this tile); 8 MMAs per stage
      // A token's middle tiles (neither its first nor its last) run the same
      // stages without the first / last tile's q waits and releases, so that
      // no branch on them sits between two stages' runs of MMAs (the wide-Dk
      // instantiations; the narrow ones run every tile through qk / pv,
      // which measured faster there: the issuing thread's code shape moves
      // the Dk 192 / Dv 128 window kernel by ~6 %).
      auto qk_mid = [&]() -> bool {
        const uint32_t buf = sidx & 1, use = sidx >> 1;
        if (!mbar_wait_spin(&sh->sempty[buf], (use & 1) ^ 1, lim)) return false;
        tc_fence_after();
        const uint32_t d = tmem + kSCol + buf * kH;
        for (int s = 0; s < (p.nck + 1) / 2; ++s) {
          const int c0 = 2 * s;
          const bool two = c0 + 1 < p.nck;
          if (!mbar_wait_spin(&sh->kfull[slot], ph, lim)) return false;  // TMA stage
          const uint64_t a = ring_desc_k + (uint64_t)((slot * kSlotBytes) >> 4);
          const uint64_t b = q_desc + (uint64_t)((c0 * kQChunkBytes) >> 4);
          qk_stage(d, a, b, s, two);
          umma_commit(&sh->kempty[slot]);
          next_slot();
        }
        umma_commit(&sh->sfull[buf]);
        ++sidx;
        issued = true;
        return true;
      };
      auto pv_mid = [&]() -> bool {
        if (!mbar_wait_spin(&sh->pfull, npv & 1, lim)) return false;
        tc_fence_after();
        for (int c = 0; c < p.nvc; ++c) {
          if (!mbar_wait_spin(&sh->vfull[slot], ph, lim)) return false;  // TMA stage
          const uint64_t a0 = ring_desc_v + (uint64_t)((slot * kSlotBytes) >> 4);
          pv_run(tmem + c * kH, a0, p_desc, id_pv, 1u);
          umma_commit(&sh->vempty[slot]);
          next_slot();
        }
        umma_commit(&sh->pvdone);
        ++npv;
        issued = true;
        return true;
      };
      auto pv = [&](bool first_tile) -> bool {
        if (!mbar_wait_spin(&sh->pfull, npv & 1, lim)) return false;
        tc_fence_after();
        for (int c = 0; c < p.nvc; ++c) {
          if (!mbar_wait_spin(&sh->vfull[slot], ph, lim)) return false;  // TMA stage
          if (kEarly && first_tile && ntok > 0) {  // previous token's chunk c read out
            if (!mbar_wait_spin(&sh->ochunk[c], (ntok - 1) & 1, lim)) return false;
            tc_fence_after();
          }
          const uint64_t a0 = ring_desc_v + (uint64_t)((slot * kSlotBytes) >> 4);
          const uint32_t d = tmem + c * kH;
          if constexpr (kWide) {
            pv_run(d, a0, p_desc, id_pv, first_tile ? 0u : 1u);
          } else {
            if (first_tile) pv_run_t<true>(d, a0, p_desc, id_pv);
            else pv_run_t<false>(d, a0, p_desc, id_pv);
          }
          umma_commit(&sh->vempty[slot]);
          next_slot();
        }
        umma_commit(&sh->pvdone);
        ++npv;
        issued = true;
        return true;
      };
      // lane 0 alone walks the tokens (the other lanes of the warp stay idle:
      // divergent work beside the issuing lane was measured to slow MMA issue)
      for (int t = blockIdx.x; t < p.T && !stop; t += G) {
        const TokenPlan tp = plan_token<kSparse>(p, t, false);
        if (!tp.ok || tp.ntile == 0) continue;
        if (!is_pv) {
          if constexpr (kWide) {
            for (int i = 0; i < tp.ntile; ++i) {
              const bool ok2 =
                  (i > 0 && i + 1 < tp.ntile) ? qk_mid() : qk(i == 0, i + 1 == tp.ntile);
              if (!ok2) { stop = true; break; }
            }
          } else {
            for (int i = 0; i < tp.ntile; ++i)
              if (!qk(i == 0, i + 1 == tp.ntile)) { stop = true; break; }
          }
          ++qtok;
        } else {
          // O^T of the previous token must have been read out before PV(0)
          // (the plain modes wait per chunk inside pv)
          if (!kEarly && ntok > 0 && !mbar_wait(&sh->oempty, (ntok - 1) & 1, lim)) {
            stop = true;
            break;
          }
          tc_fence_after();
          if constexpr (kWide) {
            for (int i = 0; i < tp.ntile; ++i)
              if (!(i > 0 ? pv_mid() : pv(true))) { stop = true; break; }
          } else {
            for (int i = 0; i < tp.ntile; ++i)
              if (!pv(i == 0)) { stop = true; break; }
          }
          if (stop) break;
          if (!kEarly) umma_commit(&sh->ofull);
          ++ntok;
        }
      }
      if (stop) give_up(sh, p.status);
      if (issued) {  // this thread's MMAs done before TMEM is released
        uint64_t* db = is_pv ? &sh->drain_pv : &sh->drain;
        umma_commit(db);
        mbar_wait(db, 0, kDefaultWaitNs);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    // Two warpgroups; warpgroup wg owns heads [32 wg, 32 wg + 32).  Thread
    // (warp, lane) owns key row r of S^T and value row r of each O^T chunk.
    const int wg = (warp - 2) >> 2;
    const int g4 = warp & 3;
    const int r = 32 * g4 + lane;
    const int hb = 32 * wg;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * g4) << 16);
    const float sl2 = p.scale_log2;
    const int dvs = p.dv;  // row stride of out
    uint32_t sidx = 0, npv = 0, rvph = 0, ntok = 0, gt = 0, rvph_all = 0;
    bool ok = true;
    // full layer: blocks per tile, warps per block, the running max (log2)
    // of this lane's head that the last tile's exponentials used
    const int nbt = kFull ? kTile / p.B : 0;
    const int wpb = kFull ? p.B / 32 : 1;
    float m_used = 0.f;
    // Plain modes: the token whose output is still in TMEM (-1: none).  Its
    // epilogue runs once the next token's first P tile is written: each
    // 128-row dv chunk of O^T is read into registers, released at once to the
    // next token's first PV (ochunk[c]), normalised by the token's sh->lsum
    // and stored as bf16 straight to out (a warp writes 32 consecutive dv of
    // one head per store).  The last PV of that token must be complete.
    int pend_t = -1;
    auto early_epilogue = [&]() {
      __nv_bfloat16* const obase = p.out + ((int64_t)pend_t * kH + hb) * dvs;
      float ls[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) ls[k] = sh->lsum[hb + k];
      for (int c = 0; c < p.nvc; ++c) {
        uint32_t w[32];
        tmem_ld32(lane_base + c * kH + hb, w);
        tmem_ld_wait();
        reg_fence(w);
        tc_fence_before();
        mbar_arrive(&sh->ochunk[c]);
        const int col = c * 128 + r;
        if (col < dvs) {
#pragma unroll
          for (int k = 0; k < 32; ++k)
            obase[(int64_t)k * dvs + col] = __float2bfloat16_rn(__uint_as_float(w[k]) * ls[k]);
        }
      }
      pend_t = -1;
    };
    for (int t = blockIdx.x; t < p.T && ok && !aborted(sh); t += G) {
      // the token's plan; warp 0 of the group also compacts its selected
      // blocks into blist
      const TokenPlan tp =
          plan_token_warp<kSparse>(p, t, false, (kSparse && g4 == 0) ? sh->blist[wg] : nullptr);
      if (!tp.ok) continue;
      float* const blkrow =
          kFull ? p.blk + ((size_t)blockIdx.x * 2 + (ntok & 1)) * (size_t)p.nbmax * kH : nullptr;
      // block LSEs (log2 units) of tile `tile`: the warps of each block add
      // their per-head sums; blocks past the query's own are not stored
      auto flush_blocks = [&](int tile) {
        if (g4 < nbt) {
          float sum = 0.f;
          for (int w = 0; w < wpb; ++w) sum += sh->bsum[wg][g4 * wpb + w][lane];
          const int b = tile * nbt + g4;
          if (b <= tp.bq) blkrow[(size_t)b * kH + hb + lane] = m_used + fast_log2(sum);
        }
      };
      if (tp.ntile == 0) {  // no valid block: empty softmax, only the sink
        for (int e = r; e < 32 * dvs; e += 128)
          p.out[((int64_t)t * kH + hb) * dvs + e] = __float2bfloat16_rn(0.f);
        if (r < 32) p.lse[(int64_t)t * kH + hb + r] = p.sink ? __ldg(p.sink + hb + r) : -INFINITY;
        continue;
      }
      if (kSparse) {  // blist is complete for every warp of the group after this
        if (!rendezvous(sh, wg, rvph, lim)) { ok = false; break; }
      }
      if (kCombine) {  // this warpgroup's rows of prev towards L2 for the epilogue
        const char* pb = reinterpret_cast<const char*>(p.prev + ((int64_t)t * kH + hb) * dvs);
        for (int off = r * 128; off < 32 * dvs * 2; off += 128 * 128)
          asm volatile("prefetch.global.L2 [%0];" ::"l"(pb + off));
      }
      float lpart[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) lpart[k] = 0.f;
      for (int i = 0; i < tp.ntile && ok; ++i) {
        const uint32_t buf = sidx & 1, use = sidx >> 1;
        if (!mbar_wait(&sh->sfull[buf], use & 1, lim)) { ok = false; break; }
        tc_fence_after();
        uint32_t u[32];
        tmem_ld32(lane_base + kSCol + buf * kH + hb, u);
        tmem_ld_wait();
        reg_fence(u);
        tc_fence_before();
        mbar_arrive(&sh->sempty[buf]);
        ++sidx;
        // key of this row and its validity
        bool valid;
        if (kSparse) {
          const int slotn = i * (kTile / p.B) + r / p.B;
          const int b = slotn < tp.nsel ? sh->blist[wg][slotn] : tp.bq;
          const int key = tp.bos + b * p.B + (r % p.B);
          valid = slotn < tp.nsel && key <= t;
        } else {
          valid = tp.wlo + i * kTile + r <= t;
        }
        float x[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) x[k] = valid ? __uint_as_float(u[k]) * sl2 : -INFINITY;
        // per-head max over the 128 key rows
        {
          float a[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) a[k] = x[k];
          sh->red[wg][g4][lane] = tr_max(a);
        }
        if (!rendezvous(sh, wg, rvph, lim)) { ok = false; break; }
        if (kFull && i > 0) flush_blocks(i - 1);  // sums written before this rendezvous
        if (g4 == 0) {
          const int hh = hb + lane;
          const float tm = fmaxf(fmaxf(sh->red[wg][0][lane], sh->red[wg][1][lane]),
                                 fmaxf(sh->red[wg][2][lane], sh->red[wg][3][lane]));
          const float mo = (i == 0) ? -INFINITY : sh->mrun[hh];
          float mn = mo;
          if (i == 0 || tm > mo + kRescaleLog2) mn = tm;
          sh->alpha[hh] = (i == 0 || mn == mo) ? 1.f : fast_exp2(mo - mn);
          sh->mrun[hh] = mn;
          if (i > 0 && mn != mo) sh->rescale[wg][gt & 1] = 1;
          // the other parity's flag was last read before this rendezvous
          if (lane == 0) sh->rescale[wg][(gt + 1) & 1] = 0;
        }
        if (!rendezvous(sh, wg, rvph, lim)) { ok = false; break; }
        const bool resc = i > 0 && sh->rescale[wg][gt & 1] != 0;
        ++gt;
        // exp2(x - m_h) for heads hb..hb+31 of row r, packed as bf16 pairs,
        // before waiting for the P^T buffer: after PV of the previous tile
        // has released it only the stores remain
        if (resc) {
#pragma unroll
          for (int k = 0; k < 32; ++k) lpart[k] *= sh->alpha[hb + k];
        }
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float e0 = fast_exp2(x[2 * k] - sh->mrun[hb + 2 * k]);
          const float e1 = fast_exp2(x[2 * k + 1] - sh->mrun[hb + 2 * k + 1]);
          lpart[2 * k] += e0;
          lpart[2 * k + 1] += e1;
          __nv_bfloat162 pr = __floats2bfloat162_rn(e0, e1);
          pk[k] = *reinterpret_cast<uint32_t*>(&pr);
          if (kFull) {
            x[2 * k] = e0;
            x[2 * k + 1] = e1;
          }
        }
        if (kFull) {  // this warp's 32 key rows summed per head (lane = head)
          sh->bsum[wg][g4][lane] = tr_sum(x);
          m_used = sh->mrun[hb + lane];
        }
        // P^T may be rewritten once PV of the previous tile has read it, and
        // on a token's first tile once BOTH warpgroups have finished staging
        // the previous token's output in the same buffer (each warpgroup's
        // staging half spans rows that hold the other warpgroup's P^T columns)
        if (i > 0 || (kEarly && pend_t >= 0)) {
          if (!mbar_wait(&sh->pvdone, npv & 1, lim)) { ok = false; break; }
          ++npv;
          tc_fence_after();
        } else if (!kEarly && ntok > 0) {
          if (!mbar_wait(&sh->oempty, (ntok - 1) & 1, lim)) { ok = false; break; }
        }
        if (resc) {  // rare: some head's running max rose; rescale its O^T columns
#pragma unroll 1
          for (int c = 0; c < p.nvc; ++c) {
            uint32_t w[32];
            const uint32_t ta = lane_base + c * kH + hb;
            tmem_ld32(ta, w);
            tmem_ld_wait();
            reg_fence(w);
#pragma unroll
            for (int k = 0; k < 32; ++k)
              w[k] = __float_as_uint(__uint_as_float(w[k]) * sh->alpha[hb + k]);
            tmem_st32(ta, w);
          }
          tmem_st_wait();
        }
        // P^T row r, 128-byte swizzled
        uint8_t* prow = pbuf + r * 128;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int cidx = 4 * wg + q4;
          *reinterpret_cast<uint4*>(prow + ((cidx ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        mbar_arrive(&sh->pfull);
        if (kEarly && pend_t >= 0) early_epilogue();  // the previous token's output
      }
      if (!ok) break;
      // ---------------- epilogue: per-head sums, sink, normalisation
      sh->red[wg][g4][lane] = tr_sum(lpart);
      if (!rendezvous(sh, wg, rvph, lim)) { ok = false; break; }
      if (kFull) flush_blocks(tp.ntile - 1);
      if (g4 == 0) {
        const int hh = hb + lane;
        const float l = (sh->red[wg][0][lane] + sh->red[wg][1][lane]) +
                        (sh->red[wg][2][lane] + sh->red[wg][3][lane]);
        const float m = sh->mrun[hh];  // finite: tile 0 always holds a valid key
        const float sk = p.sink ? __ldg(p.sink + hh) * kLog2e : -INFINITY;
        const float M = fmaxf(m, sk);
        const float den = l * fast_exp2(m - M) + fast_exp2(sk - M);
        sh->lsum[hh] = fast_exp2(m - M) / den;
        if (kCombine) {
          if (p.gate_own) sh->lsum[hh] *= __ldg(p.gate_own + (int64_t)t * kH + hh);
          sh->gprev[hh] = p.gate_prev ? __ldg(p.gate_prev + (int64_t)t * kH + hh) : 1.f;
        }
        sh->lse2[hh] = M + fast_log2(den);
        p.lse[(int64_t)t * kH + hh] = sh->lse2[hh] * kLn2;
      }
      if (kEarly) {
        ++ntok;
        pend_t = t;
        // lsum is visible to the whole warpgroup, and red / mrun / blist may
        // be rewritten for the next token, only after this
        if (!rendezvous(sh, wg, rvph, lim)) { ok = false; break; }
        continue;
      }
      // the last PV of this token must be complete before O^T is read
      if (!mbar_wait(&sh->pvdone, npv & 1, lim)) { ok = false; break; }
      ++npv;
      if (!mbar_wait(&sh->ofull, ntok & 1, lim)) { ok = false; break; }
      tc_fence_after();
      if (!rendezvous(sh, wg, rvph, lim)) { ok = false; break; }
      // O^T chunk c (dv rows x this warpgroup's 32 heads) is normalised,
      // staged as [head][128 dv] bf16 in this warpgroup's half of the P^T
      // buffer (free: the token's last PV is complete) and written out by
      // one TMA tensor store of that box (the combining mode instead adds the
      // other branch and writes 16-byte units, a head's 256 contiguous bytes
      // per half-warp).  The storing thread waits until TMA has read the box
      // before the next chunk is staged.  No wait inside this loop can fail,
      // so all 128 threads meet each named barrier.
      {
        __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(pbuf) + wg * (32 * 128);
        __nv_bfloat16* obase = p.out + ((int64_t)t * kH + hb) * dvs;
        float ls[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) ls[k] = sh->lsum[hb + k];
        for (int c = 0; c < p.nvc; ++c) {
          // combining epilogue: the 16-byte units of prev this thread will
          // overwrite, loaded before the TMEM read so the latency overlaps
          uint4 pv[4];
          if (kCombine) {
            const __nv_bfloat16* pbase = p.prev + ((int64_t)t * kH + hb) * dvs;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const int u = r + 128 * q4;
              const int col = c * 128 + (u & 15) * 8;
              pv[q4] = col < dvs ? *reinterpret_cast<const uint4*>(
                                       pbase + (int64_t)(u >> 4) * dvs + col)
                                 : make_uint4(0u, 0u, 0u, 0u);
            }
          }
          uint32_t w[32];
          tmem_ld32(lane_base + c * kH + hb, w);
          tmem_ld_wait();
          reg_fence(w);
#pragma unroll
          for (int k = 0; k < 32; ++k)
            stage[k * 128 + r] = __float2bfloat16_rn(__uint_as_float(w[k]) * ls[k]);
          if (!kCombine) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          named_bar(1 + wg, 128);
          if (kCombine) {
            // the gated other branch joins in fp32
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              const int u = r + 128 * q4;
              const int col = c * 128 + (u & 15) * 8;
              if (col < dvs) {
                uint4 v = reinterpret_cast<const uint4*>(stage)[u];
                const float g = sh->gprev[hb + (u >> 4)];
                uint32_t* vw = reinterpret_cast<uint32_t*>(&v);
                const uint32_t* pw = reinterpret_cast<const uint32_t*>(&pv[q4]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vw[e]));
                  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pw[e]));
                  __nv_bfloat162 o = __floats2bfloat162_rn(fmaf(g, b.x, a.x), fmaf(g, b.y, a.y));
                  vw[e] = *reinterpret_cast<uint32_t*>(&o);
                }
                *reinterpret_cast<uint4*>(obase + (int64_t)(u >> 4) * dvs + col) = v;
              }
            }
          } else {
            // one thread stores the staged [32 heads][128 dv] box with TMA
            // (columns past Dv fall outside the tensor and are not written)
            if (r == 0) {
              asm volatile(
                  "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
                  ::"l"(reinterpret_cast<uint64_t>(&omap)), "r"(smem_u32(stage)), "r"(c * 128),
                  "r"(hb), "r"(t)
                  : "memory");
              asm volatile("cp.async.bulk.commit_group;" ::: "memory");
              asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            }
          }
          named_bar(1 + wg, 128);
        }
      }
      tc_fence_before();
      mbar_arrive(&sh->oempty);
      if (kFull) {
        // both warpgroups' block LSEs and row LSEs are in place after this
        __threadfence_block();
        mbar_arrive(&sh->rv_all);
        if (!mbar_wait(&sh->rv_all, rvph_all, lim)) { ok = false; break; }
        rvph_all ^= 1;
        const float la = sh->lse2[lane], lb = sh->lse2[lane + 32];
        float* const srow = p.block_score + (int64_t)t * p.nb_stride;
        float* const lrow = p.block_lse ? p.block_lse + (int64_t)t * kH * p.nb_stride : nullptr;
        for (int b = wg * 4 + g4; b < p.nbmax; b += 8) {  // one block per warp
          float sc = 0.f, va = -INFINITY, vb = -INFINITY;
          if (b <= tp.bq) {
            va = __ldcg(blkrow + (size_t)b * kH + lane);
            vb = __ldcg(blkrow + (size_t)b * kH + lane + 32);
            float e = fast_exp2(va - la) + fast_exp2(vb - lb);
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) e += __shfl_xor_sync(0xffffffffu, e, off);
            sc = e;
          }
          if (lane == 0) srow[b] = sc;
          if (lrow) {
            lrow[(int64_t)lane * p.nb_stride + b] = va * kLn2;
            lrow[(int64_t)(lane + 32) * p.nb_stride + b] = vb * kLn2;
          }
        }
      }
      ++ntok;
      // lsum / mrun / blist are rewritten for the next token only after this
      if (!rendezvous(sh, wg, rvph, lim)) { ok = false; break; }
    }
    if (kEarly && ok && pend_t >= 0 && !aborted(sh)) {  // the last token's output
      if (mbar_wait(&sh->pvdone, npv & 1, lim)) {
        ++npv;
        tc_fence_after();
        early_epilogue();
      } else {
        ok = false;
      }
    }
    if (!ok) give_up(sh, p.status);
    if (!kCombine && r == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace

bool tc_attention_supported(int num_heads, int dk, int dv, int block_size, bool sparse) {
  (void)sparse;
  return num_heads == kH && dk % 64 == 0 && dk >= 64 && dk <= 64 * kMaxQChunks &&
         dv % 64 == 0 && dv >= 64 && dv <= 512 &&
         (block_size == 16 || block_size == 32 || block_size == 64 || block_size == 128);
}

bool tc_attention_eligible(const AttnArgs& a) {
  const Problem& p = a.p;
  auto al16 = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15) == 0; };
  return al16(p.q) && al16(p.k) && al16(p.v) && al16(a.out) && al16(a.prev) &&
         p.q_row_stride % 8 == 0 &&
         p.q_head_stride % 8 == 0 && p.k_row_stride % 8 == 0 && p.v_row_stride % 8 == 0;
}

namespace {

cudaError_t launch_mode(const AttnArgs& a, int mode, const FullArgs* fa, long long wait_limit,
                        cudaStream_t s) {
  const bool sparse = mode == kModeSparse;
  const Problem& p = a.p;
  const uint32_t rows = sparse ? (uint32_t)a.block_size : (uint32_t)kTile;
  CUtensorMap kmap, vmap, qmap, omap;
  {
    const uint64_t dims[2] = {(uint64_t)p.dk, (uint64_t)p.total_tokens};
    const uint64_t strides[1] = {(uint64_t)p.k_row_stride * 2};
    const uint32_t box[2] = {64, rows};
    if (!encode_bf16_map(&kmap, p.k, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {(uint64_t)p.dv, (uint64_t)p.total_tokens};
    const uint64_t strides[1] = {(uint64_t)p.v_row_stride * 2};
    const uint32_t box[2] = {64, rows};
    if (!encode_bf16_map(&vmap, p.v, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {(uint64_t)p.dk, (uint64_t)p.num_heads, (uint64_t)p.total_tokens};
    const uint64_t strides[2] = {(uint64_t)p.q_head_stride * 2, (uint64_t)p.q_row_stride * 2};
    const uint32_t box[3] = {64, (uint32_t)kH, 1};
    if (!encode_bf16_map(&qmap, p.q, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {(uint64_t)p.dv, (uint64_t)p.num_heads, (uint64_t)p.total_tokens};
    const uint64_t strides[2] = {(uint64_t)p.dv * 2, (uint64_t)p.num_heads * p.dv * 2};
    const uint32_t box[3] = {128, 32, 1};
    if (!encode_bf16_map(&omap, a.out, 3, dims, strides, box, false)) return cudaErrorInvalidValue;
  }
  AttnParams ap;
  ap.cu = p.cu_seqlens;
  ap.num_docs = p.num_docs;
  ap.T = p.total_tokens;
  ap.max_seqlen = p.max_seqlen;
  ap.idx = a.idx;
  ap.topk = a.topk;
  ap.B = a.block_size;
  ap.window = mode == kModeFull ? (1 << 30) : a.window;  // full layer: every causal key
  ap.nck = p.dk / 64;
  ap.nvc = (p.dv + 127) / 128;  // a panel past Dv is zero-filled by TMA
  ap.dv = p.dv;
  ap.scale_log2 = p.scale * kLog2e;
  ap.sink = a.sink;
  ap.out = static_cast<__nv_bfloat16*>(a.out);
  ap.lse = a.lse;
  ap.status = p.status;
  ap.wait_ns = wait_limit > 0 ? wait_limit : kDefaultWaitNs;
  ap.blk = fa ? static_cast<float*>(fa->workspace) : nullptr;
  ap.nbmax = fa ? fa->nbmax : 0;
  ap.nb_stride = fa ? fa->nb_stride : 0;
  ap.block_score = fa ? fa->block_score : nullptr;
  ap.block_lse = fa ? fa->block_lse : nullptr;
  ap.prev = static_cast<const __nv_bfloat16*>(a.prev);
  ap.gate_own = a.gate_own;
  ap.gate_prev = a.gate_prev;
  const int grid = p.total_tokens < sm_count() ? p.total_tokens : sm_count();
  // the issuers' form of a QK stage is chosen per instantiation (Dk > 256:
  // runtime flags, else templated variants)
  auto kern = ap.nck > 4 ? (mode == kModeSparse     ? tc_attention_kernel<kModeSparse, true>
                            : mode == kModeFull     ? tc_attention_kernel<kModeFull, true>
                            : mode == kModeSwaLayer ? tc_attention_kernel<kModeSwaLayer, true>
                                                    : tc_attention_kernel<kModeSwa, true>)
                         : (mode == kModeSparse     ? tc_attention_kernel<kModeSparse, false>
                            : mode == kModeFull     ? tc_attention_kernel<kModeFull, false>
                            : mode == kModeSwaLayer ? tc_attention_kernel<kModeSwaLayer, false>
                                                    : tc_attention_kernel<kModeSwa, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemBytes, s>>>(kmap, vmap, qmap, omap, ap);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_attention(const AttnArgs& a, bool sparse, long long wait_limit,
                                cudaStream_t s) {
  if (a.prev && sparse) return cudaErrorInvalidValue;  // combining is a window-branch mode
  return launch_mode(a, sparse ? kModeSparse : a.prev ? kModeSwaLayer : kModeSwa, nullptr,
                     wait_limit, s);
}

bool tc_full_supported(int num_heads, int dk, int dv, int block_size) {
  return tc_attention_supported(num_heads, dk, dv, block_size, false) && block_size >= 32;
}

size_t tc_full_workspace(int total_tokens, int nbmax) {
  const int grid = total_tokens < sm_count() ? total_tokens : sm_count();
  return (size_t)grid * 2 * (size_t)nbmax * kH * sizeof(float);
}

cudaError_t launch_tc_full(const FullArgs& f, long long wait_limit, cudaStream_t s) {
  AttnArgs a{};
  a.p = f.p;
  a.idx = nullptr;
  a.topk = 0;
  a.block_size = f.block_size;
  a.window = 0;
  a.sink = nullptr;
  a.out = f.out;
  a.lse = f.lse;
  return launch_mode(a, kModeFull, &f, wait_limit, s);
}

}  // namespace hs
