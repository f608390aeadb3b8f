// dq of hs_sparse_mqa_bwd / hs_swa_mqa_bwd on tcgen05 tensor cores (bf16
// in, fp32 accumulate), 64 query heads over one KV head.
//
// Definition (the backward of the forward in tc_attention.cu; "HySparse MQA
// sparse attention ...", PaddleFleet pull request 1470, "Core" list: the
// DSA gather and windowed MQA backward, with the learnable attn_sink of pull
// request 1415 entering only through lse): with P_j = exp(s_j - lse[t,h]),
// s_j = scale <q[t,h], k_j>, dP_j = <dout[t,h], v_j> and
// delta[t,h] = <dout[t,h], out[t,h]>,
//   dq[t,h] = scale * sum_{j in S_t} P_j (dP_j - delta[t,h]) k_j.
//
// Design.  Query-major like the forward: one persistent CTA per SM walks
// tokens; q_t (64 heads x Dk) and dout_t (64 heads x Dv) stay in shared
// memory for all of the token's 128-key tiles, and every MMA is transposed
// so that M = 128 keys or 128 rows of Dk:
//   S^T[128 keys x 64]  = K_tile . q_t^T          (A: K tile, K-major)
//   dP^T[128 keys x 64] = V_tile . dout_t^T       (A: V tile, K-major)
//   dQ^T[Dk x 64]      += K_tile^T . dS^T         (A: the K tile again, MN-major)
// TMEM: dQ^T in five 64-column chunks (Dk <= 640), two S^T buffers and one
// dP^T buffer (512 columns).  One ring of two 32 KB slots carries, in the
// issuing order, the K stages of QK(i+1), the K stages of dQ(i) (the K tile
// is read a second time, after the softmax) and the V stages of dP(i+1), so
// that QK(i+1) runs while the dS warps work on tile i.  The dS warps (thread
// = key row, two warpgroups of 32 heads) need no reduction: lse and delta
// come from the forward and from the delta pass, so
//   dS = exp2(s log2e scale - lse log2e) (dP - delta)
// is written straight to a 128-byte-swizzled [key][head] bf16 tile (the B
// operand of dQ).  After the token's last tile they read dQ^T back (lane =
// Dk row) and store scale * dQ as fp32 rows of dq.  All waits are bounded.

#include <math.h>

#include "hs_device.cuh"
#include "hs_internal.h"
#include "tc_common.cuh"
#include "tc_host.h"

namespace hs {
namespace {

using namespace tc;

constexpr int kThreads = 384;  // producer, issuer, 2 dS warpgroups, 2 idle warps
constexpr int kH = 64;
constexpr int kTile = 128;
constexpr int kSlots = 2;
constexpr int kSlotBytes = 32768;     // two 128 x 64 bf16 panels
constexpr int kPanel = 16384;
constexpr int kChunkBytes = kH * 64 * 2;  // 8 KB: 64 heads x 64 columns
constexpr int kMaxQC = 9;             // Dk <= 576
constexpr int kMaxDC = 8;             // Dv <= 512
constexpr int kDsBytes = kTile * kH * 2;  // 16 KB
constexpr int kSCol = 320;            // S^T buffers at 320 and 384
constexpr int kDPCol = 448;           // dP^T buffer
constexpr float kLog2e = 1.44269504088896340736f;

struct DqParams {
  const int32_t* cu;
  int num_docs, T, max_seqlen;
  const int32_t* idx;
  int topk, B, window;
  int nck, ndc, dk;
  float scale, scale_log2;
  const float* lse;
  const float* delta;
  float* dq;
  int* status;
  long long wait_ns;
};

struct Shared {
  uint64_t full[kSlots], empty[kSlots];
  uint64_t qfull[kMaxQC], qempty[kMaxQC];
  uint64_t dofull[kMaxDC], doempty[kMaxDC];
  uint64_t sfull[2], sempty[2];
  uint64_t dpfull, dpempty, dsfull, dsempty, dqfull, dqempty, drain;
  uint64_t rv[2];
  float lse2[kH];   // this token's lse per head, log2 units
  float del[kH];    // this token's delta per head
  int plist[256];   // the producer's selected blocks of its token
  int blist[2][256];
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kSmemBytes = 1024 + (size_t)kSlots * kSlotBytes + (size_t)kMaxQC * kChunkBytes +
                              (size_t)kMaxDC * kChunkBytes + kDsBytes + sizeof(Shared);
static_assert(kSmemBytes <= 232448, "shared memory of one CTA");

__device__ __forceinline__ bool aborted(Shared* sh) {
  return *reinterpret_cast<volatile int*>(&sh->abort_flag) != 0;
}
__device__ __forceinline__ void give_up(Shared* sh, int* status) {
  record_status(status, HS_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&sh->abort_flag) = 1;
}

struct TokenPlan {
  bool ok;
  int bos, bq, wlo, nsel, ntile;
};

// The forward's index rule: entry s is used when 0 <= b <= bq and b is larger
// than the raw entry before it.
__device__ __forceinline__ bool entry_ok(const int32_t* row, int s, int bq, int& b) {
  b = __ldg(row + s);
  return b >= 0 && b <= bq && (s == 0 || b > __ldg(row + s - 1));
}

template <bool kSparse>
__device__ __forceinline__ TokenPlan plan_token(const DqParams& p, int t) {
  TokenPlan tp;
  int eos;
  tp.ok = find_doc(p.cu, p.num_docs, p.T, p.max_seqlen, t, tp.bos, eos, nullptr);
  tp.bq = tp.ok ? (t - tp.bos) / p.B : 0;
  tp.wlo = 0;
  tp.nsel = 0;
  tp.ntile = 0;
  if (!tp.ok) return tp;
  if (kSparse) {
    const int32_t* row = p.idx + (int64_t)t * p.topk;
    int n = 0;
    for (int s = 0; s < p.topk; ++s) {
      int b;
      if (entry_ok(row, s, tp.bq, b)) ++n;
    }
    tp.nsel = n;
    const int per = kTile / p.B;
    tp.ntile = (n + per - 1) / per;
  } else {
    tp.wlo = max(tp.bos, t - p.window + 1);
    tp.ntile = (t - tp.wlo + 1 + kTile - 1) / kTile;
  }
  return tp;
}

__device__ __forceinline__ bool rendezvous(Shared* sh, int wg, uint32_t& ph, long long lim) {
  mbar_arrive(&sh->rv[wg]);
  const bool ok = mbar_wait(&sh->rv[wg], ph, lim);
  ph ^= 1;
  return ok;
}

// One K-major stage: up to two 64-column chunks of the A stage (panels 16 KB
// apart) against B chunks 8 KB apart, 4 MMAs (M = 128, N = 64, K = 16) per
// chunk into d.  The first accumulate flag and whether the second chunk is
// issued are runtime values (a guard predicate, not a branch between MMA
// runs: 1.66 -> 1.62 ms block-sparse, 0.99 -> 0.96 ms window).
__device__ __forceinline__ void kmajor_run_rt(uint32_t d, uint64_t a0, uint64_t b0, uint32_t idesc,
                                              uint32_t acc0, uint32_t two) {
#pragma unroll
  for (int k = 0; k < 4; ++k) umma_ss(d, a0 + 2 * k, b0 + 2 * k, idesc, k == 0 ? acc0 : 1u);
#pragma unroll
  for (int k = 0; k < 4; ++k)
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "setp.ne.b32 q, %5, 0;\n\t"
        "@q tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a0 + (uint64_t)(kPanel >> 4) + 2 * k), "l"(b0 + (uint64_t)(kChunkBytes >> 4) + 2 * k),
        "r"(idesc), "r"(1u), "r"(two)
        : "memory");
}
// One 128-row Dk chunk of dQ^T (+)= K_tile^T (MN-major, two 64-row panels)
// . dS^T (MN-major) over 128 keys: 8 MMAs of 16 keys; acc0 = 0 opens it.
__device__ __forceinline__ void mnmajor_run_rt(uint32_t d, uint64_t a0, uint64_t b0, uint32_t idesc,
                                               uint32_t acc0) {
#pragma unroll
  for (int kk = 0; kk < kTile / 16; ++kk)
    umma_ss(d, a0 + (uint64_t)(kk * 128), b0 + (uint64_t)(kk * 128), idesc, kk == 0 ? acc0 : 1u);
}

template <bool kSparse>
__global__ void __launch_bounds__(kThreads, 1)
tc_bwd_dq_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                 const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap dmap,
                 const DqParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* ring = base;
  uint8_t* qbuf = ring + kSlots * kSlotBytes;
  uint8_t* dobuf = qbuf + kMaxQC * kChunkBytes;
  uint8_t* dsbuf = dobuf + kMaxDC * kChunkBytes;
  Shared* sh = reinterpret_cast<Shared*>(dsbuf + kDsBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], 1);
    }
    for (int c = 0; c < kMaxQC; ++c) {
      mbar_init(&sh->qfull[c], 1);
      mbar_init(&sh->qempty[c], 1);
    }
    for (int c = 0; c < kMaxDC; ++c) {
      mbar_init(&sh->dofull[c], 1);
      mbar_init(&sh->doempty[c], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh->sfull[b], 1);
      mbar_init(&sh->sempty[b], 256);
      mbar_init(&sh->rv[b], 128);
    }
    mbar_init(&sh->dpfull, 1);
    mbar_init(&sh->dpempty, 256);
    mbar_init(&sh->dsfull, 256);
    mbar_init(&sh->dsempty, 1);
    mbar_init(&sh->dqfull, 1);
    mbar_init(&sh->dqempty, 256);
    mbar_init(&sh->drain, 1);
    fence_barrier_init();
    sh->abort_flag = 0;
  }
  if (warp == 1) tmem_alloc(&sh->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const int G = gridDim.x;
  const long long lim = p.wait_ns;
  const int per = kSparse ? kTile / p.B : 1;
  const int box_rows = kSparse ? p.B : kTile;
  const int nsk = (p.nck + 1) / 2;  // K stages per tile (two 64-column chunks each)
  const int nsv = (p.ndc + 1) / 2;  // V stages per tile

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // The ring's stages in the issuing order: per token K(QK 0), V(dP 0),
    // then per tile i: K(QK i+1), K(dQ i), V(dP i+1).  Lane 0 waits for a
    // free slot and arms it; the stage's TMA boxes are spread over the lanes.
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&vmap);
      tma_prefetch_desc(&qmap);
      tma_prefetch_desc(&dmap);
    }
    int fills[kSlots] = {0, 0};
    int qfills = 0, dfills = 0;  // per lane: its q chunk / dout chunk
    uint32_t slot = 0, ph = 0;
    bool stop = false;
    auto load_stage = [&](const TokenPlan& tp, int tile, int st, bool is_v) -> bool {
      const int nch = is_v ? p.ndc : p.nck;
      const int npanel = min(2, nch - 2 * st);
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait(&sh->empty[slot], ph ^ 1, lim);
        if (ok) mbar_expect_tx(&sh->full[slot], npanel * kPanel);
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) return false;
      __syncwarp();
      uint8_t* dst = ring + slot * kSlotBytes;
      for (int bx = lane; bx < npanel * per; bx += 32) {
        const int pn = bx / per, j = bx - pn * per;
        const int col = (2 * st + pn) * 64;
        int row0;
        if (kSparse) {
          const int slotn = tile * per + j;  // past the list: masked filler (own block)
          const int b = slotn < tp.nsel ? sh->plist[slotn] : tp.bq;
          row0 = tp.bos + b * p.B;
        } else {
          row0 = tp.wlo + tile * kTile;
        }
        tma_load_2d(dst + pn * kPanel + j * box_rows * 128, is_v ? &vmap : &kmap, &sh->full[slot],
                    col, row0);
      }
      ++fills[slot];
      if (++slot == kSlots) {
        slot = 0;
        ph ^= 1;
      }
      return true;
    };
    auto load_tile = [&](const TokenPlan& tp, int tile, bool is_v) -> bool {
      const int n = is_v ? nsv : nsk;
      for (int s = 0; s < n; ++s)
        if (!load_stage(tp, tile, s, is_v)) return false;
      return true;
    };
    for (int t = blockIdx.x; t < p.T && !stop; t += G) {
      const TokenPlan tp = plan_token<kSparse>(p, t);
      if (!tp.ok || tp.ntile == 0) continue;
      if (kSparse) {
        if (lane == 0) {
          const int32_t* row = p.idx + (int64_t)t * p.topk;
          int n = 0;
          for (int s2 = 0; s2 < p.topk; ++s2) {
            int b;
            if (entry_ok(row, s2, tp.bq, b)) sh->plist[n++] = b;
          }
        }
        __syncwarp();
      }
      // q_t and dout_t chunks (lane c: q chunk c and dout chunk c), each
      // once the previous token's last QK / dP has released it
      int ok = 1;
      if (lane < p.nck) {
        if (qfills > 0) ok = mbar_wait(&sh->qempty[lane], (qfills - 1) & 1, lim);
        if (ok) {
          mbar_expect_tx(&sh->qfull[lane], kChunkBytes);
          tma_load_3d(qbuf + lane * kChunkBytes, &qmap, &sh->qfull[lane], lane * 64, 0, t);
          ++qfills;
        }
      }
      if (ok && lane < p.ndc) {
        if (dfills > 0) ok = mbar_wait(&sh->doempty[lane], (dfills - 1) & 1, lim);
        if (ok) {
          mbar_expect_tx(&sh->dofull[lane], kChunkBytes);
          tma_load_3d(dobuf + lane * kChunkBytes, &dmap, &sh->dofull[lane], lane * 64, 0, t);
          ++dfills;
        }
      }
      if (!__all_sync(0xffffffffu, ok)) {
        stop = true;
        break;
      }
      stop = !load_tile(tp, 0, false) || !load_tile(tp, 0, true);
      for (int i = 0; i < tp.ntile && !stop; ++i) {
        if (i + 1 < tp.ntile && !load_tile(tp, i + 1, false)) { stop = true; break; }
        if (!load_tile(tp, i, false)) { stop = true; break; }
        if (i + 1 < tp.ntile && !load_tile(tp, i + 1, true)) { stop = true; break; }
      }
      __syncwarp();  // plist is rewritten for the next token only after all lanes used it
    }
    if (stop && lane == 0) give_up(sh, p.status);
    if (lane == 0)
      for (int s = 0; s < kSlots; ++s)
        if (fills[s] > 0) mbar_wait(&sh->full[s], (fills[s] - 1) & 1, kDefaultWaitNs);
    if (lane < p.nck && qfills > 0) mbar_wait(&sh->qfull[lane], (qfills - 1) & 1, kDefaultWaitNs);
    if (lane < p.ndc && dfills > 0)
      mbar_wait(&sh->dofull[lane], (dfills - 1) & 1, kDefaultWaitNs);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_k = idesc_bf16_f32(128, kH, false, false);
      constexpr uint32_t id_mn = idesc_bf16_f32(128, kH, true, true);
      const uint64_t ring_k = umma_desc_sw128(smem_u32(ring), 16, 1024);
      const uint64_t ring_mn = umma_desc_sw128(smem_u32(ring), kPanel, 1024);
      const uint64_t q_desc = umma_desc_sw128(smem_u32(qbuf), 16, 1024);
      const uint64_t do_desc = umma_desc_sw128(smem_u32(dobuf), 16, 1024);
      const uint64_t ds_desc = umma_desc_sw128(smem_u32(dsbuf), kPanel, 1024);
      uint32_t slot = 0, ph = 0, sidx = 0, ndp = 0, nds = 0, ntok = 0, qtok = 0;
      bool issued = false, stop = false;
      auto next_slot = [&]() {
        if (++slot == kSlots) {
          slot = 0;
          ph ^= 1;
        }
      };
      // S^T (QK) or dP^T (dP) of one tile: K-major stages against the
      // resident q / dout chunks; the token's last tile releases them
      auto kmajor = [&](bool is_dp, bool first_tile, bool last_tile) -> bool {
        uint32_t d;
        if (is_dp) {
          if (!mbar_wait_spin(&sh->dpempty, (ndp & 1) ^ 1, lim)) return false;
          d = tmem + kDPCol;
        } else {
          const uint32_t buf = sidx & 1, use = sidx >> 1;
          if (!mbar_wait_spin(&sh->sempty[buf], (use & 1) ^ 1, lim)) return false;
          d = tmem + kSCol + buf * kH;
        }
        tc_fence_after();
        const int nch = is_dp ? p.ndc : p.nck;
        const int ns = is_dp ? nsv : nsk;
        uint64_t* fullc = is_dp ? sh->dofull : sh->qfull;
        uint64_t* emptyc = is_dp ? sh->doempty : sh->qempty;
        const uint64_t bdesc = is_dp ? do_desc : q_desc;
        for (int s = 0; s < ns; ++s) {
          const int c0 = 2 * s;
          const bool two = c0 + 1 < nch;
          if (!mbar_wait_spin(&sh->full[slot], ph, lim)) return false;
          if (first_tile) {
            if (!mbar_wait_spin(&fullc[c0], qtok & 1, lim)) return false;
            if (two && !mbar_wait_spin(&fullc[c0 + 1], qtok & 1, lim)) return false;
          }
          const uint64_t a = ring_k + (uint64_t)((slot * kSlotBytes) >> 4);
          const uint64_t b = bdesc + (uint64_t)((c0 * kChunkBytes) >> 4);
          kmajor_run_rt(d, a, b, id_k, s == 0 ? 0u : 1u, two ? 1u : 0u);
          if (last_tile) {
            umma_commit(&emptyc[c0]);
            if (two) umma_commit(&emptyc[c0 + 1]);
          }
          umma_commit(&sh->empty[slot]);
          next_slot();
        }
        if (is_dp) {
          umma_commit(&sh->dpfull);
          ++ndp;
        } else {
          umma_commit(&sh->sfull[sidx & 1]);
          ++sidx;
        }
        issued = true;
        return true;
      };
      // dQ^T += K_tile^T . dS^T for one tile (the K tile's second pass)
      auto dq = [&](bool first_tile, bool last_tile) -> bool {
        if (!mbar_wait_spin(&sh->dsfull, nds & 1, lim)) return false;
        if (first_tile && ntok > 0 && !mbar_wait_spin(&sh->dqempty, (ntok - 1) & 1, lim))
          return false;
        tc_fence_after();
        for (int m = 0; m < nsk; ++m) {
          if (!mbar_wait_spin(&sh->full[slot], ph, lim)) return false;
          const uint64_t a0 = ring_mn + (uint64_t)((slot * kSlotBytes) >> 4);
          const uint32_t d = tmem + m * kH;
          mnmajor_run_rt(d, a0, ds_desc, id_mn, first_tile ? 0u : 1u);
          umma_commit(&sh->empty[slot]);
          next_slot();
        }
        umma_commit(&sh->dsempty);
        ++nds;
        if (last_tile) umma_commit(&sh->dqfull);
        issued = true;
        return true;
      };
      for (int t = blockIdx.x; t < p.T && !stop; t += G) {
        const TokenPlan tp = plan_token<kSparse>(p, t);
        if (!tp.ok || tp.ntile == 0) continue;
        const int n = tp.ntile;
        if (!kmajor(false, true, n == 1) || !kmajor(true, true, n == 1)) { stop = true; break; }
        for (int i = 0; i < n; ++i) {
          if (i + 1 < n && !kmajor(false, false, i + 2 == n)) { stop = true; break; }
          if (!dq(i == 0, i + 1 == n)) { stop = true; break; }
          if (i + 1 < n && !kmajor(true, false, i + 2 == n)) { stop = true; break; }
        }
        if (stop) break;
        ++qtok;
        ++ntok;
      }
      if (stop) give_up(sh, p.status);
      if (issued) {
        umma_commit(&sh->drain);
        mbar_wait(&sh->drain, 0, kDefaultWaitNs);
      }
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------ dS + epilogue
    // Warpgroup wg owns heads [32 wg, 32 wg + 32); thread (warp, lane) owns
    // key row r of S^T / dP^T / dS^T and Dk row r of each dQ^T chunk.
    const int wg = (warp - 2) >> 2;
    const int g4 = warp & 3;
    const int r = 32 * g4 + lane;
    const int hb = 32 * wg;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * g4) << 16);
    const float sl2 = p.scale_log2;
    uint32_t sidx = 0, ndp = 0, nds = 0, ntok = 0, rvph = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.T && ok && !aborted(sh); t += G) {
      const TokenPlan tp = plan_token<kSparse>(p, t);
      if (!tp.ok) continue;
      float* const dqt = p.dq + ((int64_t)t * kH + hb) * p.dk;
      if (tp.ntile == 0) {  // no valid block: dq is zero
        for (int e = r; e < 32 * p.dk; e += 128) dqt[e] = 0.f;
        continue;
      }
      if (r < 32) {
        sh->lse2[hb + r] = __ldg(p.lse + (int64_t)t * kH + hb + r) * kLog2e;
        sh->del[hb + r] = __ldg(p.delta + (int64_t)t * kH + hb + r);
      }
      if (kSparse && g4 == 0) {
        const int32_t* row = p.idx + (int64_t)t * p.topk;
        int n = 0;
        for (int base0 = 0; base0 < p.topk; base0 += 32) {
          const int s2 = base0 + lane;
          int b = -1;
          const bool v = s2 < p.topk && entry_ok(row, s2, tp.bq, b);
          const unsigned mask = __ballot_sync(0xffffffffu, v);
          if (v) sh->blist[wg][n + __popc(mask & ((1u << lane) - 1u))] = b;
          n += __popc(mask);
        }
      }
      if (!rendezvous(sh, wg, rvph, lim)) { ok = false; break; }
      for (int i = 0; i < tp.ntile && ok; ++i) {
        const uint32_t buf = sidx & 1, use = sidx >> 1;
        if (!mbar_wait(&sh->sfull[buf], use & 1, lim) || !mbar_wait(&sh->dpfull, ndp & 1, lim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t u[32], w[32];
        tmem_ld32(lane_base + kSCol + buf * kH + hb, u);
        tmem_ld32(lane_base + kDPCol + hb, w);
        tmem_ld_wait();
        reg_fence(u);
        reg_fence(w);
        tc_fence_before();
        mbar_arrive(&sh->sempty[buf]);
        mbar_arrive(&sh->dpempty);
        ++sidx;
        ++ndp;
        bool valid;
        if (kSparse) {
          const int slotn = i * per + r / p.B;
          const int b = slotn < tp.nsel ? sh->blist[wg][slotn] : tp.bq;
          const int key = tp.bos + b * p.B + (r % p.B);
          valid = slotn < tp.nsel && key <= t;
        } else {
          valid = tp.wlo + i * kTile + r <= t;
        }
        uint32_t pk[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          float ds0 = 0.f, ds1 = 0.f;
          if (valid) {
            const float p0 = fast_exp2(__uint_as_float(u[2 * k]) * sl2 - sh->lse2[hb + 2 * k]);
            const float p1 =
                fast_exp2(__uint_as_float(u[2 * k + 1]) * sl2 - sh->lse2[hb + 2 * k + 1]);
            ds0 = p0 * (__uint_as_float(w[2 * k]) - sh->del[hb + 2 * k]);
            ds1 = p1 * (__uint_as_float(w[2 * k + 1]) - sh->del[hb + 2 * k + 1]);
          }
          __nv_bfloat162 pr = __floats2bfloat162_rn(ds0, ds1);
          pk[k] = *reinterpret_cast<uint32_t*>(&pr);
        }
        // dS^T may be rewritten once dQ of the previous tile has read it
        if (!mbar_wait(&sh->dsempty, (nds & 1) ^ 1, lim)) { ok = false; break; }
        ++nds;
        uint8_t* prow = dsbuf + r * 128;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int cidx = 4 * wg + q4;
          *reinterpret_cast<uint4*>(prow + ((cidx ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&sh->dsfull);
      }
      if (!ok) break;
      // ---------------- epilogue: dq[t, h, :] = scale * dQ^T[:, h] (fp32)
      if (!mbar_wait(&sh->dqfull, ntok & 1, lim)) { ok = false; break; }
      tc_fence_after();
      for (int m = 0; m < nsk; ++m) {
        uint32_t w[32];
        tmem_ld32(lane_base + m * kH + hb, w);
        tmem_ld_wait();
        reg_fence(w);
        const int d = m * 128 + r;
        if (d < p.dk) {
#pragma unroll
          for (int k = 0; k < 32; ++k) dqt[(int64_t)k * p.dk + d] = p.scale * __uint_as_float(w[k]);
        }
      }
      tc_fence_before();
      mbar_arrive(&sh->dqempty);
      ++ntok;
      // lse2 / del / blist are rewritten for the next token only after this
      if (!rendezvous(sh, wg, rvph, lim)) { ok = false; break; }
    }
    if (!ok) give_up(sh, p.status);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace

bool tc_bwd_dq_supported(const Problem& p) {
  auto al16 = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15) == 0; };
  return p.dtype == HS_BF16 && p.num_heads == kH && p.dk % 64 == 0 && p.dk >= 64 &&
         p.dk <= 64 * kMaxQC && p.dv % 64 == 0 && p.dv >= 64 && p.dv <= 64 * kMaxDC &&
         al16(p.q) && al16(p.k) && al16(p.v) && p.q_row_stride % 8 == 0 &&
         p.q_head_stride % 8 == 0 && p.k_row_stride % 8 == 0 && p.v_row_stride % 8 == 0;
}

cudaError_t launch_tc_bwd_dq(const BwdArgs& b, bool sparse, const float* delta,
                             long long wait_limit, cudaStream_t s) {
  const Problem& p = b.p;
  const uint32_t rows = sparse ? (uint32_t)b.block_size : (uint32_t)kTile;
  if (sparse && b.block_size != 16 && b.block_size != 32 && b.block_size != 64 &&
      b.block_size != 128)
    return cudaErrorInvalidValue;
  if (reinterpret_cast<uintptr_t>(b.dout) & 15) return cudaErrorInvalidValue;
  CUtensorMap kmap, vmap, qmap, dmap;
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
  {  // dout [T, H, Dv] contiguous
    const uint64_t dims[3] = {(uint64_t)p.dv, (uint64_t)p.num_heads, (uint64_t)p.total_tokens};
    const uint64_t strides[2] = {(uint64_t)p.dv * 2, (uint64_t)p.num_heads * p.dv * 2};
    const uint32_t box[3] = {64, (uint32_t)kH, 1};
    if (!encode_bf16_map(&dmap, b.dout, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  DqParams a;
  a.cu = p.cu_seqlens;
  a.num_docs = p.num_docs;
  a.T = p.total_tokens;
  a.max_seqlen = p.max_seqlen;
  a.idx = b.idx;
  a.topk = b.topk;
  a.B = b.block_size;
  a.window = b.window;
  a.nck = p.dk / 64;
  a.ndc = p.dv / 64;
  a.dk = p.dk;
  a.scale = p.scale;
  a.scale_log2 = p.scale * kLog2e;
  a.lse = b.lse;
  a.delta = delta;
  a.dq = b.dq;
  a.status = p.status;
  a.wait_ns = wait_limit > 0 ? wait_limit : kDefaultWaitNs;
  auto kern = sparse ? tc_bwd_dq_kernel<true> : tc_bwd_dq_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int grid = p.total_tokens < sm_count() ? p.total_tokens : sm_count();
  kern<<<grid, kThreads, kSmemBytes, s>>>(kmap, vmap, qmap, dmap, a);
  return cudaGetLastError();
}

}  // namespace hs
