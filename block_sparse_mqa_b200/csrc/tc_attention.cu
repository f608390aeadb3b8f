// hs_sparse_mqa_fwd and hs_swa_mqa_fwd on tcgen05 tensor cores (bf16 in,
// fp32 accumulate), 64 query heads over one KV head.
//
// Definitions ("HySparse MQA sparse attention ...", PaddleFleet pull request
// 1470, "Core" list: block-sparse DSA gather and SWA sliding-window MQA, both
// with a learnable per-head attn_sink; "Support attn sink in fa3", pull
// request 1415: the sink is a softmax-denominator offset):
//   lse[t,h] = log(exp(sink_h) + sum_{j in S_t} exp(s_j)),
//   out[t,h] = sum_{j in S_t} exp(s_j - lse[t,h]) v_j,
// with S_t the selected blocks (causal inside the own block) or the window.
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
// A 4-slot ring of 32 KB stages carries K (two 64-column chunks per stage)
// and V (one 128-row dv chunk per stage) in exactly the order the MMA warp
// consumes them: QK(0), then for each tile i: QK(i+1), PV(i).  The softmax
// warps (thread = key row) reduce per-head maxima across the 128 rows with a
// 32-lane transpose-reduction plus a 4-warp combine, keep the running max
// per head (raised only when a tile beats it by more than 2^8, which then
// rescales O^T in TMEM), write P^T as bf16 into one 128-byte-swizzled buffer
// and accumulate per-head sums in registers.  The sink joins in the
// epilogue, which reads O^T back per dv row and writes out[t, h, :].
// Warp 0 = TMA producer, warp 1 = MMA issuer / TMEM owner, warps 2-5 =
// softmax + epilogue.  All waits are bounded (HS_ERR_TIMEOUT, drain, free).

#include <math.h>

#include "hs_device.cuh"
#include "hs_internal.h"
#include "tc_common.cuh"
#include "tc_host.h"

namespace hs {
namespace {

using namespace tc;

constexpr int kThreads = 192;
constexpr int kH = 64;              // heads (N of every MMA)
constexpr int kTile = 128;          // keys per tile (M of the QK MMA)
constexpr int kSlots = 4;           // ring slots
constexpr int kSlotBytes = 32768;   // two 128 x 64 bf16 panels
constexpr int kPanel = 16384;
constexpr int kQChunkBytes = kH * 64 * 2;  // 8 KB
constexpr int kMaxQChunks = 9;      // Dk <= 576
constexpr int kPBytes = kTile * kH * 2;    // 16 KB
constexpr int kSCol = 256;          // S^T buffers at 256 and 320
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;
constexpr float kRescaleLog2 = 8.f;  // raise the running max only past 2^8

struct AttnParams {
  const int32_t* cu;
  int num_docs, T, max_seqlen;
  const int32_t* idx;
  int topk, B, window;
  int nck, nvc;  // 64-column K chunks, 128-row V chunks
  float scale_log2;
  const float* sink;
  __nv_bfloat16* out;
  float* lse;
  int* status;
  long long wait_ns;
};

struct Shared {
  uint64_t full[kSlots], empty[kSlots];
  uint64_t qfull[kMaxQChunks], qempty[kMaxQChunks];
  uint64_t sfull[2], sempty[2];
  uint64_t pfull, pvdone, ofull, oempty, rv, drain;
  float red[4][kH];
  float mrun[kH];
  float alpha[kH];
  float lsum[kH];
  int rescale[2];  // per tile parity: some head's running max rose
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kSmemBytes =
    1024 + (size_t)kSlots * kSlotBytes + (size_t)kMaxQChunks * kQChunkBytes + kPBytes + sizeof(Shared);

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
    int prev = -1, n = 0;
    bool bad = false;
    for (int s = 0; s < p.topk; ++s) {
      const int b = __ldg(row + s);
      if (b < 0) continue;
      if (b > tp.bq || b <= prev) {
        bad = true;
        continue;
      }
      prev = b;
      ++n;
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

// The n-th valid selected block of token t (same validation as plan_token),
// or the own block when n is past the last one (a masked filler slot).
__device__ __forceinline__ int nth_block(const AttnParams& p, int t, int bq, int n) {
  const int32_t* row = p.idx + (int64_t)t * p.topk;
  int prev = -1, k = 0;
  for (int s = 0; s < p.topk; ++s) {
    const int b = __ldg(row + s);
    if (b < 0 || b > bq || b <= prev) continue;
    prev = b;
    if (k == n) return b;
    ++k;
  }
  return bq;
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

// Bounded rendezvous of the 128 softmax threads.
__device__ __forceinline__ bool rendezvous(Shared* sh, uint32_t& ph, long long lim) {
  mbar_arrive(&sh->rv);
  const bool ok = mbar_wait(&sh->rv, ph, lim);
  ph ^= 1;
  return ok;
}

template <bool kSparse>
__global__ void __launch_bounds__(kThreads, 1)
tc_attention_kernel(const __grid_constant__ CUtensorMap kmap,
                    const __grid_constant__ CUtensorMap vmap,
                    const __grid_constant__ CUtensorMap qmap, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ring = base;
  uint8_t* qbuf = ring + kSlots * kSlotBytes;
  uint8_t* pbuf = qbuf + kMaxQChunks * kQChunkBytes;
  Shared* sh = reinterpret_cast<Shared*>(pbuf + kPBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], 1);
    }
    for (int c = 0; c < kMaxQChunks; ++c) {
      mbar_init(&sh->qfull[c], 1);
      mbar_init(&sh->qempty[c], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh->sfull[b], 1);
      mbar_init(&sh->sempty[b], 128);
    }
    mbar_init(&sh->pfull, 128);
    mbar_init(&sh->pvdone, 1);
    mbar_init(&sh->ofull, 1);
    mbar_init(&sh->oempty, 128);
    mbar_init(&sh->rv, 128);
    mbar_init(&sh->drain, 1);
    fence_barrier_init();
    sh->abort_flag = 0;
    sh->rescale[0] = sh->rescale[1] = 0;
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      tma_prefetch_desc(&qmap);
      int fills[kSlots], qfills[kMaxQChunks];
      for (int s = 0; s < kSlots; ++s) fills[s] = 0;
      for (int c = 0; c < kMaxQChunks; ++c) qfills[c] = 0;
      uint32_t slot = 0, ph = 0;
      bool stop = false;
      // one ring stage: K (two 64-column chunks) or V (one 128-row dv chunk)
      auto load_stage = [&](const TokenPlan& tp, int t, int tile, bool is_v, int idx2) -> bool {
        if (!mbar_wait(&sh->empty[slot], ph ^ 1, lim)) return false;
        const int npanel = is_v ? 2 : min(2, p.nck - 2 * idx2);
        mbar_expect_tx(&sh->full[slot], npanel * kPanel);
        uint8_t* dst = ring + slot * kSlotBytes;
        for (int pn = 0; pn < npanel; ++pn) {
          const int col = is_v ? (idx2 * 2 + pn) * 64 : (idx2 * 2 + pn) * 64;
          for (int j = 0; j < per; ++j) {
            int row0;
            if (kSparse) {
              const int b = nth_block(p, t, tp.bq, tile * per + j);
              row0 = tp.bos + b * p.B;
            } else {
              row0 = tp.wlo + tile * kTile;
            }
            tma_load_2d(dst + pn * kPanel + j * box_rows * 128, is_v ? &vmap : &kmap,
                        &sh->full[slot], col, row0);
          }
        }
        ++fills[slot];
        if (++slot == kSlots) {
          slot = 0;
          ph ^= 1;
        }
        return true;
      };
      const int nks = (p.nck + 1) / 2;  // K stages per tile
      for (int t = blockIdx.x; t < p.T && !stop; t += G) {
        const TokenPlan tp = plan_token<kSparse>(p, t, true);
        if (!tp.ok || tp.ntile == 0) continue;
        // Q_t chunks, each as soon as the previous token's last QK released it
        for (int c = 0; c < p.nck; ++c) {
          if (qfills[c] > 0 && !mbar_wait(&sh->qempty[c], (qfills[c] - 1) & 1, lim)) {
            stop = true;
            break;
          }
          mbar_expect_tx(&sh->qfull[c], kQChunkBytes);
          tma_load_3d(qbuf + c * kQChunkBytes, &qmap, &sh->qfull[c], c * 64, 0, t);
          ++qfills[c];
        }
        if (stop) break;
        for (int s = 0; s < nks && !stop; ++s) stop = !load_stage(tp, t, 0, false, s);
        for (int i = 0; i < tp.ntile && !stop; ++i) {
          if (i + 1 < tp.ntile)
            for (int s = 0; s < nks && !stop; ++s) stop = !load_stage(tp, t, i + 1, false, s);
          for (int c = 0; c < p.nvc && !stop; ++c) stop = !load_stage(tp, t, i, true, c);
        }
      }
      if (stop) give_up(sh, p.status);
      for (int s = 0; s < kSlots; ++s)
        if (fills[s] > 0) mbar_wait(&sh->full[s], (fills[s] - 1) & 1, kDefaultWaitNs);
      for (int c = 0; c < kMaxQChunks; ++c)
        if (qfills[c] > 0) mbar_wait(&sh->qfull[c], (qfills[c] - 1) & 1, kDefaultWaitNs);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_qk = idesc_bf16_f32(128, kH, false, false);
      constexpr uint32_t id_pv = idesc_bf16_f32(128, kH, true, true);
      const uint64_t ring_desc_k = umma_desc_sw128(smem_u32(ring), 16, 1024);
      const uint64_t ring_desc_v = umma_desc_sw128(smem_u32(ring), kPanel, 1024);
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
      // S^T(tile) = K_tile . Q^T into S buffer sidx & 1
      auto qk = [&](bool last_tile) -> bool {
        const uint32_t buf = sidx & 1, use = sidx >> 1;
        if (!mbar_wait(&sh->sempty[buf], (use & 1) ^ 1, lim)) return false;
        tc_fence_after();
        const uint32_t d = tmem + kSCol + buf * kH;
        for (int s = 0; s < (p.nck + 1) / 2; ++s) {
          if (!mbar_wait(&sh->full[slot], ph, lim)) return false;
          tc_fence_after();
          const int np = min(2, p.nck - 2 * s);
          for (int pn = 0; pn < np; ++pn) {
            const int c = 2 * s + pn;
            if (!mbar_wait(&sh->qfull[c], qtok & 1, lim)) return false;
            tc_fence_after();
            const uint64_t a = ring_desc_k + (uint64_t)((slot * kSlotBytes + pn * kPanel) >> 4);
            const uint64_t b = q_desc + (uint64_t)((c * kQChunkBytes) >> 4);
#pragma unroll
            for (int k = 0; k < 4; ++k)
              umma_ss(d, a + 2 * k, b + 2 * k, id_qk, (c | k) != 0);
            if (last_tile) umma_commit(&sh->qempty[c]);
          }
          umma_commit(&sh->empty[slot]);
          next_slot();
        }
        umma_commit(&sh->sfull[buf]);
        ++sidx;
        issued = true;
        return true;
      };
      // O^T += V_tile^T . P^T (waits for P of this tile)
      auto pv = [&](bool first_tile) -> bool {
        if (!mbar_wait(&sh->pfull, npv & 1, lim)) return false;
        tc_fence_after();
        for (int c = 0; c < p.nvc; ++c) {
          if (!mbar_wait(&sh->full[slot], ph, lim)) return false;
          tc_fence_after();
          const uint64_t a0 = ring_desc_v + (uint64_t)((slot * kSlotBytes) >> 4);
          const uint32_t d = tmem + c * kH;
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_ss(d, a0 + (uint64_t)(kk * 128), p_desc + (uint64_t)(kk * 128), id_pv,
                    (!first_tile || kk > 0) ? 1u : 0u);
          umma_commit(&sh->empty[slot]);
          next_slot();
        }
        umma_commit(&sh->pvdone);
        ++npv;
        return true;
      };
      for (int t = blockIdx.x; t < p.T && !stop; t += G) {
        const TokenPlan tp = plan_token<kSparse>(p, t, false);
        if (!tp.ok || tp.ntile == 0) continue;
        if (!qk(tp.ntile == 1)) { stop = true; break; }
        // O^T of the previous token must have been read out before PV(0)
        if (ntok > 0 && !mbar_wait(&sh->oempty, (ntok - 1) & 1, lim)) { stop = true; break; }
        tc_fence_after();
        for (int i = 0; i < tp.ntile; ++i) {
          if (i + 1 < tp.ntile && !qk(i + 2 == tp.ntile)) { stop = true; break; }
          if (!pv(i == 0)) { stop = true; break; }
        }
        if (stop) break;
        umma_commit(&sh->ofull);
        ++ntok;
        ++qtok;
      }
      if (stop) give_up(sh, p.status);
      if (issued) {
        umma_commit(&sh->drain);
        mbar_wait(&sh->drain, 0, kDefaultWaitNs);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int g4 = warp & 3;
    const int r = 32 * g4 + lane;  // key row of S^T / dv row of O^T
    const uint32_t lane_base = tmem + ((uint32_t)(32 * g4) << 16);
    uint32_t sidx = 0, npv = 0, rvph = 0, ntok = 0, gt = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.T && ok && !aborted(sh); t += G) {
      const TokenPlan tp = plan_token<kSparse>(p, t, false);
      if (!tp.ok) continue;
      if (tp.ntile == 0) {  // no valid block: empty softmax, only the sink
        const int dvs = p.nvc * 128;
        for (int e = r; e < kH * dvs; e += 128)
          p.out[(int64_t)t * kH * dvs + e] = __float2bfloat16_rn(0.f);
        if (r < kH) p.lse[(int64_t)t * kH + r] = p.sink ? __ldg(p.sink + r) : -INFINITY;
        continue;
      }
      float lpart[kH];
#pragma unroll
      for (int h = 0; h < kH; ++h) lpart[h] = 0.f;
      for (int i = 0; i < tp.ntile && ok; ++i) {
        const uint32_t buf = sidx & 1, use = sidx >> 1;
        if (!mbar_wait(&sh->sfull[buf], use & 1, lim)) { ok = false; break; }
        tc_fence_after();
        float x[kH];
#pragma unroll
        for (int j = 0; j < kH / 32; ++j) {
          uint32_t u[32];
          tmem_ld32(lane_base + kSCol + buf * kH + j * 32, u);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) x[j * 32 + k] = __uint_as_float(u[k]);
        }
        tc_fence_before();
        mbar_arrive(&sh->sempty[buf]);
        ++sidx;
        // key of this row and its validity
        bool valid;
        if (kSparse) {
          const int slotn = i * (kTile / p.B) + r / p.B;
          const int b = nth_block(p, t, tp.bq, slotn);
          const int key = tp.bos + b * p.B + (r % p.B);
          valid = slotn < tp.nsel && key <= t;
        } else {
          const int key = tp.wlo + i * kTile + r;
          valid = key <= t;
        }
#pragma unroll
        for (int h = 0; h < kH; ++h) x[h] = valid ? x[h] * p.scale_log2 : -INFINITY;
        // per-head max over the 128 rows
        {
          float a[32], b2[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            a[k] = x[k];
            b2[k] = x[k + 32];
          }
          const float m0 = tr_max(a), m1 = tr_max(b2);
          sh->red[g4][lane] = m0;
          sh->red[g4][lane + 32] = m1;
        }
        if (!rendezvous(sh, rvph, lim)) { ok = false; break; }
        if (r < kH) {
          const float tm = fmaxf(fmaxf(sh->red[0][r], sh->red[1][r]),
                                 fmaxf(sh->red[2][r], sh->red[3][r]));
          float mo = (i == 0) ? -INFINITY : sh->mrun[r];
          float mn = mo;
          if (i == 0) mn = tm;
          else if (tm > mo + kRescaleLog2) mn = tm;
          // a head whose keys are all masked so far keeps -inf: use 0 as
          // reference so that exp2 stays finite (all its P are zero anyway)
          sh->alpha[r] = (i == 0 || mn == mo) ? 1.f : fast_exp2(mo - mn);
          sh->mrun[r] = mn;
          if (i > 0 && mn != mo) sh->rescale[gt & 1] = 1;
        }
        // the other parity's flag was last read before the rendezvous above
        if (r == 0) sh->rescale[(gt + 1) & 1] = 0;
        if (!rendezvous(sh, rvph, lim)) { ok = false; break; }
        const bool resc = i > 0 && sh->rescale[gt & 1] != 0;
        ++gt;
        // P^T may be written once PV of the previous tile has read it
        if (i > 0) {
          if (!mbar_wait(&sh->pvdone, npv & 1, lim)) { ok = false; break; }
          ++npv;
          tc_fence_after();
        }
        if (resc) {
          // rare: the running max of some head rose; rescale O^T columns
#pragma unroll 1
          for (int c = 0; c < p.nvc; ++c) {
#pragma unroll
            for (int j = 0; j < kH / 32; ++j) {
              uint32_t u[32];
              const uint32_t ta = lane_base + c * kH + j * 32;
              tmem_ld32(ta, u);
              tmem_ld_wait();
#pragma unroll
              for (int k = 0; k < 32; ++k)
                u[k] = __float_as_uint(__uint_as_float(u[k]) * sh->alpha[j * 32 + k]);
              tmem_st32(ta, u);
            }
          }
          tmem_st_wait();
#pragma unroll
          for (int h = 0; h < kH; ++h) lpart[h] *= sh->alpha[h];
        }
        // P^T row r: exp2(x - m_h) as bf16, 128-byte swizzled (MN-major B)
        uint8_t* prow = pbuf + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int h0 = c * 8 + 2 * k;
            const float mh0 = sh->mrun[h0], mh1 = sh->mrun[h0 + 1];
            const float e0 = fast_exp2(x[h0] - (mh0 == -INFINITY ? 0.f : mh0));
            const float e1 = fast_exp2(x[h0 + 1] - (mh1 == -INFINITY ? 0.f : mh1));
            lpart[h0] += e0;
            lpart[h0 + 1] += e1;
            __nv_bfloat162 pr = __floats2bfloat162_rn(e0, e1);
            w[k] = *reinterpret_cast<uint32_t*>(&pr);
          }
          *reinterpret_cast<uint4*>(prow + ((c ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        mbar_arrive(&sh->pfull);
      }
      if (!ok) break;
      // ---------------- epilogue: per-head sums, sink, normalisation
      {
        float a[32], b2[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          a[k] = lpart[k];
          b2[k] = lpart[k + 32];
        }
        const float s0 = tr_sum(a), s1 = tr_sum(b2);
        sh->red[g4][lane] = s0;
        sh->red[g4][lane + 32] = s1;
      }
      if (!rendezvous(sh, rvph, lim)) { ok = false; break; }
      if (r < kH) {
        const float l = (sh->red[0][r] + sh->red[1][r]) + (sh->red[2][r] + sh->red[3][r]);
        const float mh = sh->mrun[r];
        const float m = (mh == -INFINITY) ? 0.f : mh;  // log2 reference used for P
        const float sk = p.sink ? __ldg(p.sink + r) * kLog2e : -INFINITY;
        const float M = fmaxf(m, sk);
        const float den = l * fast_exp2(m - M) + fast_exp2(sk - M);
        sh->lsum[r] = fast_exp2(m - M) / den;  // multiplier of O
        p.lse[(int64_t)t * kH + r] = (M + fast_log2(den)) * kLn2;
      }
      // the last PV of this token must be complete before O^T is read
      if (!mbar_wait(&sh->pvdone, npv & 1, lim)) { ok = false; break; }
      ++npv;
      if (!mbar_wait(&sh->ofull, ntok & 1, lim)) { ok = false; break; }
      tc_fence_after();
      if (!rendezvous(sh, rvph, lim)) { ok = false; break; }
      __nv_bfloat16* orow = p.out + (int64_t)t * kH * (p.nvc * 128);
      const int dvs = p.nvc * 128;
      for (int c = 0; c < p.nvc; ++c) {
#pragma unroll
        for (int j = 0; j < kH / 32; ++j) {
          uint32_t u[32];
          tmem_ld32(lane_base + c * kH + j * 32, u);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int h = j * 32 + k;
            orow[(int64_t)h * dvs + c * 128 + r] =
                __float2bfloat16_rn(__uint_as_float(u[k]) * sh->lsum[h]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&sh->oempty);
      ++ntok;
      // lsum / mrun are rewritten for the next token only after everyone is done
      if (!rendezvous(sh, rvph, lim)) { ok = false; break; }
    }
    if (!ok) give_up(sh, p.status);
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
         dv % 128 == 0 && dv >= 128 && dv <= 512 &&
         (block_size == 16 || block_size == 32 || block_size == 64 || block_size == 128);
}

bool tc_attention_eligible(const AttnArgs& a) {
  const Problem& p = a.p;
  auto al16 = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15) == 0; };
  return al16(p.q) && al16(p.k) && al16(p.v) && p.q_row_stride % 8 == 0 &&
         p.q_head_stride % 8 == 0 && p.k_row_stride % 8 == 0 && p.v_row_stride % 8 == 0;
}

cudaError_t launch_tc_attention(const AttnArgs& a, bool sparse, long long wait_limit,
                                cudaStream_t s) {
  const Problem& p = a.p;
  const uint32_t rows = sparse ? (uint32_t)a.block_size : (uint32_t)kTile;
  CUtensorMap kmap, vmap, qmap;
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
  AttnParams ap;
  ap.cu = p.cu_seqlens;
  ap.num_docs = p.num_docs;
  ap.T = p.total_tokens;
  ap.max_seqlen = p.max_seqlen;
  ap.idx = a.idx;
  ap.topk = a.topk;
  ap.B = a.block_size;
  ap.window = a.window;
  ap.nck = p.dk / 64;
  ap.nvc = p.dv / 128;
  ap.scale_log2 = p.scale * kLog2e;
  ap.sink = a.sink;
  ap.out = static_cast<__nv_bfloat16*>(a.out);
  ap.lse = a.lse;
  ap.status = p.status;
  ap.wait_ns = wait_limit > 0 ? wait_limit : kDefaultWaitNs;
  const int grid = p.total_tokens < sm_count() ? p.total_tokens : sm_count();
  auto kern = sparse ? tc_attention_kernel<true> : tc_attention_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemBytes, s>>>(kmap, vmap, qmap, ap);
  return cudaGetLastError();
}

}  // namespace hs
