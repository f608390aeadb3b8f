// dk / dv of hs_sparse_mqa_bwd / hs_swa_mqa_bwd on tcgen05 tensor cores
// (bf16 in, fp32 accumulate), 64 query heads over one KV head.
//
// Definitions (the backward of the forward in tc_attention.cu; "HySparse MQA
// sparse attention ...", PaddleFleet pull request 1470, "Core" list: the DSA
// gather and windowed MQA backward): for every key j and every (t, h) with
// j in S_t,
//   dk[j] += scale * ds * q[t,h],  dv[j] += p * dout[t,h],
//   p = exp(scale <q[t,h], k[j]> - lse[t,h]),  ds = p (<dout[t,h], v[j]> - delta[t,h]).
//
// Design.  Key-major: a 32-key tile's accumulators stay in TMEM as
//   dV^T [Dv x 32 keys] (four 128-row chunks, 128 columns) and
//   dK^T [Dk x 32 keys] (five 128-row chunks, 160 columns),
// beside the per-member scores, which use the heads as M:
//   S  [64 heads x 32 keys] = q_t . K_tile^T     (M = 64, N = 32, A = q_t K-major)
//   dP [64 heads x 32 keys] = dout_t . V_tile^T  (M = 64, N = 32)
//   dV^T += dout_t^T . P,  dK^T += q_t^T . dS     (M = 128 rows of Dv / Dk,
//        A = the same resident dout_t / q_t read MN-major, B = P / dS)
// An M = 64 result lands in TMEM lanes 32w .. 32w+15 for rows 16w .. 16w+15
// (w = 0..3, measured), so the dS warps (one per lane quarter) each own 16
// heads, one head per lane: p and ds need only that head's lse and delta,
// with no reduction.  P and dS are written as 64-byte-swizzled MN-major
// [head][key] bf16 tiles (the B operands).  A cluster of four CTAs shares a
// key tile (split at document boundaries): each scans every candidate query
// (the forward's index rule; the window for SWA) and takes every fourth
// member in ascending order, and the four partial sums are added in rank
// order through distributed shared memory, so a tile every query selects (a
// document's first block) is spread over four SMs.  Per member the producer
// loads q_t and dout_t by TMA chunk by chunk, each 64-column chunk once the
// previous member's dK^T / dV^T MMAs have read it, and two threads issue the
// MMAs (the q side and the dout side).  Sums run in a fixed order: results
// are deterministic.
// All waits are bounded (HS_ERR_TIMEOUT).

#include <algorithm>
#include <cooperative_groups.h>
#include <math.h>

#include "hs_device.cuh"
#include "hs_internal.h"
#include "tc_common.cuh"
#include "tc_host.h"

namespace hs {
namespace {

using namespace tc;
namespace cg = cooperative_groups;

constexpr int kThreads = 256;       // 8 warps: producer, 2 issuers, 1 idle, 4 dS / epilogue
constexpr int kCluster = 4;         // CTAs sharing one key tile
constexpr int kKT = 32;             // keys per tile
constexpr int kH = 64;
constexpr int kMaxQC = 9;           // Dk <= 576
constexpr int kMaxDC = 8;           // Dv <= 512
constexpr int kRowChunk = kKT * 64 * 2;  // 4 KB: a tile's 32 rows x 64 columns
constexpr int kTokChunk = kH * 64 * 2;   // 8 KB: a token's 64 heads x 64 columns
constexpr int kPBytes = kH * kKT * 2;    // 4 KB: [64 heads][32 keys] bf16
constexpr int kColS = 0, kColDP = 32, kColDV = 64, kColDK = 192;  // TMEM columns
constexpr int kDSWarp = 4;          // first dS / epilogue warp
constexpr float kLog2e = 1.44269504088896340736f;

struct DkdvParams {
  const int32_t* cu;
  int num_docs, T, max_seqlen;
  const int32_t* idx;
  int topk, B, window;
  int nck, ndc, dk, dv;
  float scale, scale_log2;
  const float* lse;
  const float* delta;
  float* dkey;
  float* dval;
  int* status;
  long long wait_ns;
  // work items: (32-key tile, query range) pairs, range-major
  int rlen, nrange;    // query-range length, number of ranges
  int nitems;          // items that can hold members (see item_of)
  float* part;         // [nrange][T][Dk + Dv] partial sums of the items (fp32)
};

// The tiles whose keys a query in [r0, r1) can attend: every earlier tile for
// block-sparse attention, the tiles within one window before it for SWA.
__host__ __device__ __forceinline__ void range_tiles(bool sparse, int rg, int rlen, int T,
                                                     int window, int& tlo, int& thi) {
  const int r0 = rg * rlen, r1 = min(T, r0 + rlen);
  thi = (r1 + kKT - 1) / kKT;
  tlo = sparse ? 0 : max(0, (r0 - window - kKT + 1) / kKT);
  if (tlo > thi) tlo = thi;
}

// Work item k -> (tile, range): range-major, so the clusters that run at the
// same time take members from the same range of queries (whose q_t and
// dout_t then stay in L2), and a tile every query selects is spread over all
// ranges instead of one cluster.
__host__ __device__ __forceinline__ bool item_of(bool sparse, int k, int rlen, int nrange, int T,
                                                 int window, int& tile, int& rg) {
  for (rg = 0; rg < nrange; ++rg) {
    int tlo, thi;
    range_tiles(sparse, rg, rlen, T, window, tlo, thi);
    if (k < thi - tlo) {
      tile = tlo + k;
      return true;
    }
    k -= thi - tlo;
  }
  return false;
}

struct Shared {
  uint64_t tile_full, sdp_full, sdp_empty, pds_full, pds_free, acc_done;
  // per 64-column chunk of q_t / dout_t: loaded, and read by the member's MMAs
  uint64_t qfull[kMaxQC], qfree[kMaxQC], dfull[kMaxDC], dfree[kMaxDC];
  int mem[kThreads];      // a candidate chunk's members (query tokens)
  int memmask[kThreads];  // and the tile keys each attends (bit jj = key s0 + jj)
  int wcount[kThreads / 32];
  int abort_flag;
  uint32_t tmem_base;
};

constexpr size_t kSmemBytes = 1024 + (size_t)kMaxQC * kRowChunk + (size_t)kMaxDC * kRowChunk +
                              (size_t)kMaxQC * kTokChunk + (size_t)kMaxDC * kTokChunk +
                              2 * (size_t)kPBytes + sizeof(Shared);
static_assert(kSmemBytes <= 232448, "shared memory of one CTA");
// the partial sums [32 keys][Dk + Dv] fp32 reuse the q_t / dout_t buffers
static_assert((size_t)kKT * (64 * kMaxQC + 64 * kMaxDC) * 4 <=
                  (size_t)(kMaxQC + kMaxDC) * kTokChunk,
              "partial sums fit the token buffers");

__device__ __forceinline__ bool aborted(Shared* sh) {
  return *reinterpret_cast<volatile int*>(&sh->abort_flag) != 0;
}
__device__ __forceinline__ void give_up(Shared* sh, int* status) {
  record_status(status, HS_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&sh->abort_flag) = 1;
}

// The forward's index rule.
__device__ __forceinline__ bool entry_used(const int32_t* row, int s, int bq, int& b) {
  b = __ldg(row + s);
  return b >= 0 && b <= bq && (s == 0 || b > __ldg(row + s - 1));
}
__device__ __forceinline__ bool selects(const int32_t* row, int topk, int bq, int b) {
  for (int s = 0; s < topk; ++s) {
    int e;
    if (entry_used(row, s, bq, e) && e == b) return true;
  }
  return false;
}

// 64-byte-swizzle descriptor of an MN-major B operand with 32 bf16 (64 B) per
// K row: 8-row groups of 512 B.
__device__ __forceinline__ uint64_t desc_sw64(uint32_t addr) {
  return umma_desc_sw64(addr, 4096, 512);
}

template <bool kSparse>
__global__ void __launch_bounds__(kThreads, 1)
tc_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap,
                   const __grid_constant__ CUtensorMap qmap,
                   const __grid_constant__ CUtensorMap dmap, const DkdvParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* kt = base;                               // [9][32 x 64] K tile
  uint8_t* vt = kt + kMaxQC * kRowChunk;            // [8][32 x 64] V tile
  uint8_t* qb = vt + kMaxDC * kRowChunk;            // [9][64 x 64] q_t
  uint8_t* db = qb + kMaxQC * kTokChunk;            // [8][64 x 64] dout_t
  uint8_t* pb = db + kMaxDC * kTokChunk;            // P  [64 heads][32 keys]
  uint8_t* sb = pb + kPBytes;                       // dS [64 heads][32 keys]
  Shared* sh = reinterpret_cast<Shared*>(sb + kPBytes);
  float* part = reinterpret_cast<float*>(qb);       // [32][Dk + Dv] partial sums (tile end)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  cg::cluster_group cl = cg::this_cluster();
  const int crank = (int)cl.block_rank(), csize = (int)cl.num_blocks();
  const int ncl = gridDim.x / csize;
  const long long lim = p.wait_ns;
  const int NT = p.T, dk = p.dk, dv = p.dv, W = dk + dv;
  const int nmk = (p.nck + 1) / 2, nmv = (p.ndc + 1) / 2;  // 128-row chunks of dK^T, dV^T

  if (tid == 0) {
    mbar_init(&sh->tile_full, 1);
    for (int c = 0; c < kMaxQC; ++c) {
      mbar_init(&sh->qfull[c], 1);
      mbar_init(&sh->qfree[c], 1);
    }
    for (int c = 0; c < kMaxDC; ++c) {
      mbar_init(&sh->dfull[c], 1);
      mbar_init(&sh->dfree[c], 1);
    }
    mbar_init(&sh->sdp_full, 2);   // both issuers' commits
    mbar_init(&sh->sdp_empty, 128);
    mbar_init(&sh->pds_full, 128);
    mbar_init(&sh->pds_free, 2);
    mbar_init(&sh->acc_done, 2);
    fence_barrier_init();
    sh->abort_flag = 0;
  }
  if (warp == 1) tmem_alloc(&sh->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&kmap);
    tma_prefetch_desc(&vmap);
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&dmap);
  }
  // pipeline counters (each role keeps its own copy where it uses them)
  uint32_t ntile_loads = 0;   // producer / issuer: K/V tile loads issued / consumed
  uint32_t nmem = 0;          // members processed by this CTA (all roles)
  uint32_t nacc = 0;          // tiles with at least one member (issuer / epilogue)
  bool ok = true;
  // issuer state
  const uint32_t id_s = idesc_bf16_f32(64, kKT, false, false);
  const uint32_t id_acc = idesc_bf16_f32(128, kKT, true, true);

  // The tile, segment and candidate-chunk loops depend only on the inputs,
  // never on a CTA's own failures: every CTA of a cluster meets every cluster
  // barrier.  A CTA that gave up skips its members' work.
  for (int item = blockIdx.x / csize; item < p.nitems; item += ncl) {
    int tile, rg;
    if (!item_of(kSparse, item, p.rlen, p.nrange, NT, p.window, tile, rg)) break;
    const int r0 = rg * p.rlen, r1 = min(NT, r0 + p.rlen);  // this item's queries
    const int j1 = min(NT, tile * kKT + kKT);
    for (int s0 = tile * kKT; s0 < j1;) {  // one document segment at a time
      int bos, eos;
      // a malformed cu_seqlens fails alike in every CTA of the cluster
      if (!find_doc(p.cu, p.num_docs, NT, p.max_seqlen, s0, bos, eos, p.status)) break;
      const int s1 = min(j1, eos), n = s1 - s0;
      // the segment's candidate queries [s0, tend) inside this item's range
      const int tend_all = kSparse ? eos : min(eos, s1 - 1 + p.window);
      const int c_lo = max(s0, r0), tend = min(tend_all, r1);
      if (c_lo >= tend) {  // none: no partial sum for this segment and range
        s0 = s1;
        continue;
      }
      // the segment's K and V rows (32 from s0; rows past the segment are
      // never a member's key; rows past T are zero-filled)
      if (warp == 0 && lane == 0) {
        mbar_expect_tx(&sh->tile_full, (uint32_t)(p.nck + p.ndc) * kRowChunk);
        for (int c = 0; c < p.nck; ++c)
          tma_load_2d(kt + c * kRowChunk, &kmap, &sh->tile_full, c * 64, s0);
        for (int c = 0; c < p.ndc; ++c)
          tma_load_2d(vt + c * kRowChunk, &vmap, &sh->tile_full, c * 64, s0);
      }
      ++ntile_loads;
      bool tile_waited = false;
      bool any = false;
      const int b_lo = kSparse ? (s0 - bos) / p.B : 0;
      const int b_hi = kSparse ? (s1 - 1 - bos) / p.B : 0;
      for (int c0 = c_lo; c0 < tend; c0 += kThreads) {
        // candidate query t = c0 + tid: which of the segment's keys it attends
        const int t = c0 + tid;
        uint32_t mask = 0;
        if (t < tend) {
          if (kSparse) {
            const int bq = (t - bos) / p.B;
            const int32_t* row = p.idx + (int64_t)t * p.topk;
            bool f[3];  // the segment's keys lie in at most three blocks (B >= 16)
#pragma unroll
            for (int q = 0; q < 3; ++q)
              f[q] = b_lo + q <= b_hi && selects(row, p.topk, bq, b_lo + q);
            for (int jj = 0; jj < n; ++jj) {
              const int j = s0 + jj;
              if (j <= t && f[(j - bos) / p.B - b_lo]) mask |= 1u << jj;
            }
          } else {
            for (int jj = 0; jj < n; ++jj) {
              const int j = s0 + jj;
              if (j <= t && j > t - p.window) mask |= 1u << jj;
            }
          }
        }
        const unsigned bal = __ballot_sync(0xffffffffu, mask != 0);
        if (lane == 0) sh->wcount[warp] = __popc(bal);
        __syncthreads();
        int off = 0, nm = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
          if (w < warp) off += sh->wcount[w];
          nm += sh->wcount[w];
        }
        if (mask) {
          const int pos = off + __popc(bal & ((1u << lane) - 1u));
          sh->mem[pos] = t;
          sh->memmask[pos] = (int)mask;
        }
        __syncthreads();
        // ---- this CTA's members of the chunk (every csize-th, ascending)
        if (warp == 0) {
          // producer: q_t and dout_t of each member, chunk c by lane c, each
          // chunk once the previous member's MMAs have read it (the next
          // member's loads overlap this member's last MMAs)
          uint32_t m = nmem;
          for (int mi = crank; mi < nm && ok; mi += csize, ++m) {
            const int tt = sh->mem[mi];
            int good = 1;
            if (lane < p.nck) {
              if (m > 0) good = mbar_wait(&sh->qfree[lane], (m - 1) & 1, lim);
              if (good) {
                mbar_expect_tx(&sh->qfull[lane], kTokChunk);
                tma_load_3d(qb + lane * kTokChunk, &qmap, &sh->qfull[lane], lane * 64, 0, tt);
              }
            }
            if (good && lane < p.ndc) {
              if (m > 0) good = mbar_wait(&sh->dfree[lane], (m - 1) & 1, lim);
              if (good) {
                mbar_expect_tx(&sh->dfull[lane], kTokChunk);
                tma_load_3d(db + lane * kTokChunk, &dmap, &sh->dfull[lane], lane * 64, 0, tt);
              }
            }
            if (!__all_sync(0xffffffffu, good)) { ok = false; break; }
          }
        } else if (warp == 1 || warp == 2) {
          // two MMA-issuing threads: warp 1 issues the q side (S, then dK^T),
          // warp 2 the dout side (dP, then dV^T); one thread issues an MMA
          // only every ~90 cycles, so the two streams halve a member's issue
          if (lane == 0) {
            const bool qside = warp == 1;
            const uint64_t a_k = umma_desc_sw128(smem_u32(qside ? qb : db), 16, 1024);
            const uint64_t b_k = umma_desc_sw128(smem_u32(qside ? kt : vt), 16, 1024);
            const uint64_t a_mn = umma_desc_sw128(smem_u32(qside ? qb : db), kTokChunk, 1024);
            const uint64_t b_pd = desc_sw64(smem_u32(qside ? sb : pb));
            const int nch = qside ? p.nck : p.ndc;
            const int nmc = qside ? nmk : nmv;
            const uint32_t col_s = qside ? kColS : kColDP;
            const uint32_t col_acc = qside ? kColDK : kColDV;
            uint64_t* const full_b = qside ? sh->qfull : sh->dfull;
            uint64_t* const free_b = qside ? sh->qfree : sh->dfree;
            uint32_t m = nmem;
            for (int mi = crank; mi < nm && ok; mi += csize, ++m) {
              if (!tile_waited) {
                if (!mbar_wait(&sh->tile_full, (ntile_loads - 1) & 1, lim)) { ok = false; break; }
                tile_waited = true;
              }
              // S (or dP) of this member, once the previous member's were read
              if (m > 0 && !mbar_wait_spin(&sh->sdp_empty, (m - 1) & 1, lim)) {
                ok = false;
                break;
              }
              tc_fence_after();
              bool got = true;
              if (nch == 9 || nch == 8) {
                // Dk 576 / 512, Dv 512: every chunk landed first, then the
                // member's runs back to back with no wait or loop branch
                // between them (4.67 -> 4.48 ms block-sparse, 2.63 -> 2.53 ms
                // window, bit-identical); chunks arrive early enough that
                // waiting for the last one costs less than the branches did
                for (int c = 0; c < nch && got; ++c)
                  if (!mbar_wait_spin(&full_b[c], m & 1, lim)) got = false;
                if (!got) { ok = false; break; }
#pragma unroll
                for (int c = 0; c < 8; ++c)
#pragma unroll
                  for (int k = 0; k < 4; ++k)
                    umma_ss(tmem + col_s, a_k + (uint64_t)((c * kTokChunk) >> 4) + 2 * k,
                            b_k + (uint64_t)((c * kRowChunk) >> 4) + 2 * k, id_s,
                            (c == 0 && k == 0) ? 0u : 1u);
                if (nch == 9) {
#pragma unroll
                  for (int k = 0; k < 4; ++k)
                    umma_ss(tmem + col_s, a_k + (uint64_t)((8 * kTokChunk) >> 4) + 2 * k,
                            b_k + (uint64_t)((8 * kRowChunk) >> 4) + 2 * k, id_s, 1u);
                }
              } else {
                for (int c = 0; c < nch && got; ++c) {
                  if (!mbar_wait_spin(&full_b[c], m & 1, lim)) { got = false; break; }
#pragma unroll
                  for (int k = 0; k < 4; ++k)
                    umma_ss(tmem + col_s, a_k + (uint64_t)((c * kTokChunk) >> 4) + 2 * k,
                            b_k + (uint64_t)((c * kRowChunk) >> 4) + 2 * k, id_s,
                            (c == 0 && k == 0) ? 0u : 1u);
                }
              }
              if (!got) { ok = false; break; }
              umma_commit(&sh->sdp_full);
              // dK^T += q_t^T . dS (or dV^T += dout_t^T . P) once P and dS are
              // written (the tile's first member opens the sums)
              if (!mbar_wait_spin(&sh->pds_full, m & 1, lim)) { ok = false; break; }
              tc_fence_after();
              const uint32_t first = any ? 1u : 0u;
              auto acc_run = [&](int c) {
#pragma unroll
                for (int k = 0; k < 4; ++k)
                  umma_ss(tmem + col_acc + c * kKT,
                          a_mn + (uint64_t)((2 * c * kTokChunk) >> 4) + (uint64_t)(k * 128),
                          b_pd + (uint64_t)(k * 64), id_acc, (k == 0) ? first : 1u);
              };
              if (nch == 9 || nch == 8) {  // Dk 576 / 512, Dv 512: unrolled (-3 %)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                  acc_run(c);
                  // this chunk pair of q_t (or dout_t) is read: the next
                  // member's copies may land there
                  umma_commit(&free_b[2 * c]);
                  umma_commit(&free_b[2 * c + 1]);
                }
                if (nch == 9) {
                  acc_run(4);
                  umma_commit(&free_b[8]);
                }
              } else {
                for (int c = 0; c < nmc; ++c) {
                  acc_run(c);
                  umma_commit(&free_b[2 * c]);
                  if (2 * c + 1 < nch) umma_commit(&free_b[2 * c + 1]);
                }
              }
              umma_commit(&sh->pds_free);
              any = true;
            }
          }
        } else if (warp >= kDSWarp) {
          // dS warps: head h = 16 (warp - kDSWarp) + lane for lanes 0-15 (the
          // M = 64 layout); all 32 lanes take part in loads and barriers
          const int wq = warp - kDSWarp;
          const int h = 16 * wq + (lane & 15);
          const bool act = lane < 16;
          const uint32_t lane_base = tmem + ((uint32_t)(32 * wq) << 16);
          uint32_t m = nmem;
          for (int mi = crank; mi < nm && ok; mi += csize, ++m) {
            const int tt = sh->mem[mi];
            const uint32_t mk = (uint32_t)sh->memmask[mi];
            const float lse2 = __ldg(p.lse + (int64_t)tt * kH + h) * kLog2e;
            const float del = __ldg(p.delta + (int64_t)tt * kH + h);
            if (!mbar_wait(&sh->sdp_full, m & 1, lim)) { ok = false; break; }
            tc_fence_after();
            uint32_t u[32], w[32];
            tmem_ld32(lane_base + kColS, u);
            tmem_ld32(lane_base + kColDP, w);
            tmem_ld_wait();
            reg_fence(u);
            reg_fence(w);
            tc_fence_before();
            mbar_arrive(&sh->sdp_empty);
            uint32_t pp[16], pd[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              float p0 = 0.f, p1 = 0.f;
              if ((mk >> (2 * k)) & 1u) p0 = fast_exp2(__uint_as_float(u[2 * k]) * p.scale_log2 - lse2);
              if ((mk >> (2 * k + 1)) & 1u)
                p1 = fast_exp2(__uint_as_float(u[2 * k + 1]) * p.scale_log2 - lse2);
              const float d0 = p0 * (__uint_as_float(w[2 * k]) - del);
              const float d1 = p1 * (__uint_as_float(w[2 * k + 1]) - del);
              __nv_bfloat162 a = __floats2bfloat162_rn(p0, p1);
              __nv_bfloat162 b = __floats2bfloat162_rn(d0, d1);
              pp[k] = *reinterpret_cast<uint32_t*>(&a);
              pd[k] = *reinterpret_cast<uint32_t*>(&b);
            }
            // P / dS may be rewritten once the previous member's dV / dK read them
            if (m > 0 && !mbar_wait(&sh->pds_free, (m - 1) & 1, lim)) { ok = false; break; }
            if (act) {
              // row h of each [head][32 keys] tile: 64 bytes, 64-byte swizzle
              const int sw = (h >> 1) & 3;
#pragma unroll
              for (int q4 = 0; q4 < 4; ++q4) {
                const int off = h * 64 + ((q4 ^ sw) << 4);
                *reinterpret_cast<uint4*>(pb + off) =
                    make_uint4(pp[4 * q4], pp[4 * q4 + 1], pp[4 * q4 + 2], pp[4 * q4 + 3]);
                *reinterpret_cast<uint4*>(sb + off) =
                    make_uint4(pd[4 * q4], pd[4 * q4 + 1], pd[4 * q4 + 2], pd[4 * q4 + 3]);
              }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(&sh->pds_full);
          }
        }
        // every role has handled this chunk's members; the member list is
        // rewritten for the next chunk only after this
        const int mine = nm > crank ? (nm - crank + csize - 1) / csize : 0;
        if (mine > 0) any = true;
        nmem += (uint32_t)mine;
        if (aborted(sh)) ok = false;
        if (!ok) give_up(sh, p.status);
        __syncthreads();
        if (aborted(sh)) ok = false;
      }
      // the tile load's phase is consumed even without members
      if ((warp == 1 || warp == 2) && lane == 0 && !tile_waited)
        if (!mbar_wait(&sh->tile_full, (ntile_loads - 1) & 1, kDefaultWaitNs)) give_up(sh, p.status);
      // ---- this CTA's partial sums -> its shared memory (the token buffers
      // are free once every MMA has completed), then the cluster adds them
      if (any && ok) {
        if ((warp == 1 || warp == 2) && lane == 0) umma_commit(&sh->acc_done);
        __syncwarp();
        if (warp >= kDSWarp) {
          const int r = 32 * (warp - kDSWarp) + lane;  // TMEM lane = Dv / Dk row
          const uint32_t lb = tmem + ((uint32_t)(32 * (warp - kDSWarp)) << 16);
          if (!mbar_wait(&sh->acc_done, nacc & 1, lim)) {
            give_up(sh, p.status);
          } else {
            tc_fence_after();
            for (int c = 0; c < nmv; ++c) {
              uint32_t w[32];
              tmem_ld32(lb + kColDV + c * kKT, w);
              tmem_ld_wait();
              reg_fence(w);
              const int d = c * 128 + r;
              if (d < dv)
                for (int jj = 0; jj < kKT; ++jj) part[jj * W + dk + d] = __uint_as_float(w[jj]);
            }
            for (int c = 0; c < nmk; ++c) {
              uint32_t w[32];
              tmem_ld32(lb + kColDK + c * kKT, w);
              tmem_ld_wait();
              reg_fence(w);
              const int d = c * 128 + r;
              if (d < dk)
                for (int jj = 0; jj < kKT; ++jj) part[jj * W + d] = __uint_as_float(w[jj]);
            }
          }
        }
        ++nacc;
      } else {
        // no member here: a zero partial sum
        for (int e = tid; e < kKT * W; e += kThreads) part[e] = 0.f;
      }
      tc_fence_before();
      cl.sync();
      tc_fence_after();
      if (aborted(sh)) ok = false;
      const int mine_keys = n > crank ? (n - crank + csize - 1) / csize : 0;
      for (int e = tid; e < mine_keys * W; e += kThreads) {
        const int kk = crank + (e / W) * csize, col = e - (e / W) * W;
        float sum = 0.f;
        for (int rr = 0; rr < csize; ++rr) sum += cl.map_shared_rank(part, rr)[kk * W + col];
        p.part[((int64_t)rg * NT + s0 + kk) * W + col] = sum;  // this range's share
      }
      cl.sync();  // no CTA reuses its shared memory while another still reads it
      s0 = s1;
    }
  }
  // every TMA copy issued has landed before the CTA exits
  if (warp == 0 && nmem > 0) {
    if (lane < p.nck) mbar_wait(&sh->qfull[lane], (nmem - 1) & 1, kDefaultWaitNs);
    if (lane < p.ndc) mbar_wait(&sh->dfull[lane], (nmem - 1) & 1, kDefaultWaitNs);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// dk / dv from the items' partial sums: each key adds its rows over the
// ranges its candidate queries fall in (the span the items used), in
// increasing range order, and dk is scaled.
template <bool kSparse>
__global__ void __launch_bounds__(256) dkdv_reduce_kernel(const DkdvParams p) {
  const int W = p.dk + p.dv;
  const int64_t total = (int64_t)p.T * W;
  for (int64_t e = (int64_t)blockIdx.x * 256 + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * 256) {
    const int j = (int)(e / W), col = (int)(e - (int64_t)j * W);
    int bos, eos;
    float sum = 0.f;
    if (find_doc(p.cu, p.num_docs, p.T, p.max_seqlen, j, bos, eos, nullptr)) {
      const int tile0 = (j / kKT) * kKT;
      const int s0 = max(bos, tile0), s1 = min(tile0 + kKT, eos);
      const int tend = kSparse ? eos : min(eos, s1 - 1 + p.window);
      for (int rg = s0 / p.rlen; rg < p.nrange && rg * p.rlen < tend; ++rg)
        sum += __ldcs(p.part + ((int64_t)rg * p.T + j) * W + col);
    }
    if (col < p.dk)
      p.dkey[(int64_t)j * p.dk + col] = p.scale * sum;
    else
      p.dval[(int64_t)j * p.dv + (col - p.dk)] = sum;
  }
}

// Query-range length and count of the work items: ranges of at least 512
// queries (q_t and dout_t of one range, ~70 MB at 64 heads x 1088, fit in
// L2), at most 8 of them (which bounds the partial-sum workspace).
void range_split(int T, int& rlen, int& nrange) {
  rlen = (T + 7) / 8;
  if (rlen < 512) rlen = 512;
  nrange = T > 0 ? (T + rlen - 1) / rlen : 0;
}

}  // namespace

size_t tc_bwd_dkdv_workspace(int total_tokens, int dk, int dv) {
  int rlen, nrange;
  range_split(total_tokens, rlen, nrange);
  return (size_t)nrange * (size_t)total_tokens * (size_t)(dk + dv) * sizeof(float);
}

bool tc_backward_shape_ok(hs_dtype dtype, int num_heads, int dk, int dv) {
  return dtype == HS_BF16 && num_heads == kH && dk % 64 == 0 && dk >= 64 && dk <= 64 * kMaxQC &&
         dv % 64 == 0 && dv >= 64 && dv <= 64 * kMaxDC;
}

bool tc_bwd_dkdv_supported(const Problem& p) {
  auto al16 = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15) == 0; };
  return p.dtype == HS_BF16 && p.num_heads == kH && p.dk % 64 == 0 && p.dk >= 64 &&
         p.dk <= 64 * kMaxQC && p.dv % 64 == 0 && p.dv >= 64 && p.dv <= 64 * kMaxDC &&
         al16(p.q) && al16(p.k) && al16(p.v) && p.q_row_stride % 8 == 0 &&
         p.q_head_stride % 8 == 0 && p.k_row_stride % 8 == 0 && p.v_row_stride % 8 == 0;
}

cudaError_t launch_tc_bwd_dkdv(const BwdArgs& b, bool sparse, const float* delta,
                               long long wait_limit, cudaStream_t s) {
  const Problem& p = b.p;
  if (reinterpret_cast<uintptr_t>(b.dout) & 15) return cudaErrorInvalidValue;
  CUtensorMap kmap, vmap, qmap, dmap;
  {
    const uint64_t dims[2] = {(uint64_t)p.dk, (uint64_t)p.total_tokens};
    const uint64_t strides[1] = {(uint64_t)p.k_row_stride * 2};
    const uint32_t box[2] = {64, (uint32_t)kKT};
    if (!encode_bf16_map(&kmap, p.k, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[2] = {(uint64_t)p.dv, (uint64_t)p.total_tokens};
    const uint64_t strides[1] = {(uint64_t)p.v_row_stride * 2};
    const uint32_t box[2] = {64, (uint32_t)kKT};
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
  DkdvParams a;
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
  a.dv = p.dv;
  a.scale = p.scale;
  a.scale_log2 = p.scale * kLog2e;
  a.lse = b.lse;
  a.delta = delta;
  a.dkey = b.dkey;
  a.dval = b.dval;
  a.status = p.status;
  a.wait_ns = wait_limit > 0 ? wait_limit : kDefaultWaitNs;
  range_split(p.total_tokens, a.rlen, a.nrange);
  a.nitems = 0;
  for (int rg = 0; rg < a.nrange; ++rg) {
    int tlo, thi;
    range_tiles(sparse, rg, a.rlen, p.total_tokens, a.window, tlo, thi);
    a.nitems += thi - tlo;
  }
  a.part = static_cast<float*>(b.dkdv_ws);
  if (!a.part) return cudaErrorInvalidValue;
  auto kern = sparse ? tc_bwd_dkdv_kernel<true> : tc_bwd_dkdv_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const int items = a.nitems;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(items * kCluster);
  int nclusters = 0;
  if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) != cudaSuccess || nclusters < 1) {
    (void)cudaGetLastError();
    attr[0].val.clusterDim.x = 1;  // single CTAs: each takes every member of its item
    cfg.gridDim = dim3(items);
  }
  if (items > 0) {
    cudaError_t le = cudaLaunchKernelEx(&cfg, kern, kmap, vmap, qmap, dmap, a);
    if (le != cudaSuccess) return le;
  }
  const int64_t total = (int64_t)p.total_tokens * (p.dk + p.dv);
  const int rgrid = (int)std::min<int64_t>((total + 255) / 256, (int64_t)sm_count() * 8);
  if (sparse)
    dkdv_reduce_kernel<true><<<rgrid, 256, 0, s>>>(a);
  else
    dkdv_reduce_kernel<false><<<rgrid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace hs
