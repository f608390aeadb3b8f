// hs_block_score on tcgen05 tensor cores (bf16 in, fp32 accumulate).
//
// Definition ("HySparse MQA sparse attention ...", PaddleFleet pull request
// 1470: "Core" list, FA4-fused block scoring; per-file table, pipeline.py:
// block score = exp(block_logit - lse)): for query t, head h and block b <=
// bq(t) of t's document, blockLSE = log sum_{j in block b, j <= t} exp(s_j),
// LSE = log sum_{j <= t} exp(s_j), score[t, b] = sum_h exp(blockLSE - LSE).
//
// Design (one persistent CTA per SM, 12 warps):
//  * A query tile is 128 rows = (128 / H) consecutive tokens x H heads of one
//    document; q[T, H, Dk] rows are (token, head) pairs, so a tile is a
//    plain 128-row slab.  The first min(Dk, 512) columns of the tile live in
//    TMEM as the A operand (TS form): TMA brings them through the ring and
//    the MMA thread copies them into TMEM with tcgen05.cp (the same swizzled
//    K-major slabs an SS MMA would read); any remaining 64-column chunk (the
//    RoPE part of Dk = 576) stays a shared-memory tile (SS form).
//  * Keys stream in tiles of 128 (always a whole number of blocks, starting
//    at the document's first token) as 64-column K chunks (one 16 KB TMA box
//    each); three chunks form one 48 KB stage, so every pipeline wait of an
//    MMA thread is followed by 12 M=128, N=128, K=16 MMAs issued without a
//    branch between them (a branch between two MMAs costs about half the
//    issue rate).  The shared-memory (RoPE) chunk goes last, so that a query
//    tile's first key tiles need not wait for it.  Key tiles
//    alternate between two MMA-issuing threads, each with its own producer
//    and two-slot ring and its own S buffer in TMEM: a wait costs one issuing
//    thread a few hundred cycles (measured: the stage waits took ~650 of the
//    ~3800 cycles of a key tile with one issuer), and with two the tensor
//    pipe runs the other thread's MMAs meanwhile.
//  * Softmax warps (thread = row) read S (tcgen05.ld), compute per-block
//    log-sum-exp in the log2 domain with the block's own max (no underflow
//    for far-below-max blocks) and keep the running row max and sum.  Block
//    values go to a per-CTA global workspace slot [2][NBmax][128] (coalesced,
//    L2 resident; halves alternate by query tile).  At the end of the tile each row has its LSE; the head
//    sum of exp2(blockLSE - LSE) is a 32-lane transpose-reduction per warp
//    plus a fixed-order sum over the warps of a token (deterministic).
//  * Warps 0 / 10 = TMA producers of rings 0 / 1 (each also loads half of
//    the query tile's TMEM q chunks into its ring; warp 0 loads the RoPE
//    chunk), warps 1 / 11 = MMA issuers of key tiles of even / odd index
//    (each copies its ring's half of q into TMEM; warp 1 owns TMEM),
//    warps 2-9 = two softmax warpgroups
//    that take the alternate S tiles (one S buffer each) and share the
//    epilogue.  Per-row running
//    (max, sum) pairs of the two warpgroups are merged at the end of the
//    tile.  Each warpgroup loads its whole 128-column S tile into registers
//    (four tcgen05.ld in flight at once) and releases the S buffer before
//    any arithmetic, so the issuer's next MMAs into that buffer overlap the
//    softmax of this tile (measured: 0.548 -> 0.481 ms at 4096 tokens,
//    159.6 -> 142.8 ms at 65536, against reading and computing chunk by
//    chunk and releasing after the third).
//    Every wait is bounded; a timeout records HS_ERR_TIMEOUT, drains
//    in-flight copies and MMAs, frees TMEM.

#include <math.h>

#include "hs_device.cuh"
#include "hs_internal.h"
#include "tc_common.cuh"
#include "tc_host.h"

namespace hs {
namespace {

using namespace tc;

constexpr int kThreads = 384;  // 2 producers, 2 MMA issuers, 2 softmax warpgroups
constexpr int kProdB = 10;     // producer of ring 1
constexpr int kMmaB = 11;      // MMA issuer of ring 1
constexpr int kKeyTile = 128;
constexpr int kChunkBytes = kKeyTile * 64 * 2;   // one TMA box: 128 keys x 64 bf16
constexpr int kChunksPerStage = 3;               // 12 MMAs per pipeline wait
constexpr int kStageBytes = kChunksPerStage * kChunkBytes;
constexpr int kSlots = 2;                        // slots per ring (two rings)
constexpr int kStages = 2 * kSlots;
constexpr int kMaxQhi = 1;                       // shared-memory Q chunks (Dk <= 576)
constexpr int kMaxTmemQ = 8;                     // TMEM Q chunks (first 512 columns)
constexpr int kMaxDocs = 1024;
constexpr int kSCol = 256;                       // S buffers at TMEM columns 256, 384
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;

struct BSParams {
  const int32_t* cu;
  int num_docs, T, max_seqlen;
  const __nv_bfloat16* q;
  int64_t qrs, qhs;
  int H, nck, nq_tmem, nq_smem, tpt, nbmax, nbs;
  float scale_log2;
  float* lse;
  float* block_score;
  float* block_lse;
  float* ws;
  int* status;
  long long wait_ns;
};

struct Shared {
  uint64_t kfull[kStages], kempty[kStages];
  uint64_t qhi_full, qhi_empty;  // the shared-memory q chunk (empty: both issuers)
  uint64_t qdone;                // a query tile's MMAs of both issuers have completed
  uint64_t qready;               // both issuers' copies of q into TMEM have completed
  uint64_t drain[2];
  uint64_t sfull[2], sempty[2];
  uint64_t epi_all;    // rendezvous of both softmax warpgroups (256 threads)
  uint64_t epi_wg[2];  // rendezvous inside one warpgroup (128 threads)
  int prefix[kMaxDocs + 1];
  float ml[2][2][2][128];  // [tile parity][warpgroup][max | sum][row]
  float red[2][4][32];
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kSmemBytes =
    1024 + (size_t)kStages * kStageBytes + (size_t)kMaxQhi * kChunkBytes + sizeof(Shared);

struct Tile {
  int t0, tend, bos;
};

__device__ __forceinline__ Tile tile_of(int g, const int* prefix, int nd, const int32_t* cu,
                                        int tpt) {
  int lo = 0, hi = nd;  // last d with prefix[d] <= g
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= g) lo = mid; else hi = mid;
  }
  const int local = g - prefix[lo];
  const int ntd = prefix[lo + 1] - prefix[lo];
  const int li = ntd - 1 - local;  // longest tile of the document first
  Tile t;
  t.bos = __ldg(cu + lo);
  t.t0 = t.bos + li * tpt;
  t.tend = min(t.t0 + tpt, (int)__ldg(cu + lo + 1));
  return t;
}

__device__ __forceinline__ bool aborted(Shared* sh) {
  return *reinterpret_cast<volatile int*>(&sh->abort_flag) != 0;
}

__device__ __forceinline__ void give_up(Shared* sh, int* status) {
  record_status(status, HS_ERR_TIMEOUT);
  *reinterpret_cast<volatile int*>(&sh->abort_flag) = 1;
}

// Sum of v[i] over the 32 lanes of the warp, delivered to lane i.
__device__ __forceinline__ float transpose_reduce_sum(float (&v)[32]) {
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

// One ring stage = NC (three, fewer in the last stage when Dk is not a
// multiple of 192) 64-column K chunks = 4 NC MMAs (M=128, N=128, K=16) into S
// accumulator d.  FIRST: the stage opens the S tile (its first MMA
// overwrites d).  The stage's chunks come from TMEM q chunks tpos, tpos+1,
// ...; SS_LAST: its last chunk is the shared-memory q chunk (descriptor qd).
template <bool FIRST, bool SS_LAST, int NC = kChunksPerStage>
__device__ __forceinline__ void issue_stage(uint32_t d, uint32_t tmem, int tpos, uint64_t qd,
                                            uint64_t b0, uint32_t idesc) {
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const uint64_t bc = b0 + (uint64_t)((c * kChunkBytes) >> 4);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t acc = (FIRST && c == 0 && k == 0) ? 0u : 1u;
      if (SS_LAST && c == NC - 1)
        umma_ss(d, qd + 2 * k, bc + 2 * k, idesc, acc);
      else
        umma_ts(d, tmem + (uint32_t)((tpos + c) * 32 + k * 8), bc + 2 * k, idesc, acc);
    }
  }
}

template <int B>
__global__ void __launch_bounds__(kThreads, 1)
tc_block_score_kernel(const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap qmap, const BSParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* stages = base;
  uint8_t* qhi = base + kStages * kStageBytes;
  Shared* sh = reinterpret_cast<Shared*>(qhi + kMaxQhi * kChunkBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nd = p.num_docs;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh->kfull[s], 1);
      mbar_init(&sh->kempty[s], 1);
    }
    mbar_init(&sh->qhi_full, 1);
    mbar_init(&sh->qhi_empty, 2);
    mbar_init(&sh->qdone, 2);
    mbar_init(&sh->qready, 2);
    mbar_init(&sh->drain[0], 1);
    mbar_init(&sh->drain[1], 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sh->sfull[b], 1);
      mbar_init(&sh->sempty[b], 128);
    }
    mbar_init(&sh->epi_all, 256);
    mbar_init(&sh->epi_wg[0], 128);
    mbar_init(&sh->epi_wg[1], 128);
    fence_barrier_init();
    sh->abort_flag = 0;
    // tiles per document (validating cu_seqlens on the way)
    bool bad = __ldg(p.cu) != 0 || __ldg(p.cu + nd) != p.T;
    int acc = 0;
    sh->prefix[0] = 0;
    for (int d = 0; d < nd; ++d) {
      const int b0 = __ldg(p.cu + d), e0 = __ldg(p.cu + d + 1);
      const int len = e0 - b0;
      if (b0 < 0 || len < 0 || len > p.max_seqlen || e0 > p.T) bad = true;
      else acc += (len + p.tpt - 1) / p.tpt;
      sh->prefix[d + 1] = acc;
    }
    if (bad) record_status(p.status, HS_ERR_INVALID_ARG);
  }
  if (warp == 1) tmem_alloc(&sh->tmem_base, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const int total = sh->prefix[nd];
  const int G = gridDim.x, cta = blockIdx.x;
  const long long lim = p.wait_ns;

  if (warp == 0 || warp == kProdB) {
    // ------------------------------------------------------------ producers
    // Producer r fills ring r with the stages of the key tiles whose global
    // index (key tiles counted over this CTA's query tiles) has parity r,
    // preceded in each query tile by its half of the tile's TMEM q chunks;
    // producer 0 also loads the shared-memory (RoPE) q chunk.
    const int r = warp == 0 ? 0 : 1;
    if (lane == 0) {
      tma_prefetch_desc(&kmap);
      tma_prefetch_desc(&qmap);
      int fills[kSlots];
#pragma unroll
      for (int s2 = 0; s2 < kSlots; ++s2) fills[s2] = 0;
      int qfills = 0, sbase = 0;
      uint32_t kst = 0, kph = 0;
      bool stop = false;
      // next stage of ring r: wait for the slot, arm its barrier
      auto open_stage = [&](int bytes) -> uint8_t* {
        const int sl = r * kSlots + (int)kst;
        if (!mbar_wait(&sh->kempty[sl], kph ^ 1, lim)) return nullptr;
        mbar_expect_tx(&sh->kfull[sl], bytes);
        return stages + sl * kStageBytes;
      };
      auto close_stage = [&]() {
        ++fills[kst];
        if (++kst == kSlots) {
          kst = 0;
          kph ^= 1;
        }
      };
      for (int it = 0; it * G < total && !stop && !aborted(sh); ++it) {
        const int g = it * G + ((it & 1) ? (G - 1 - cta) : cta);
        if (g >= total) continue;
        const Tile tl = tile_of(g, sh->prefix, nd, p.cu, p.tpt);
        const int nkt = (tl.tend - tl.bos + kKeyTile - 1) / kKeyTile;
        if (r == 0) {
          // warm L2 with the next tile's q rows (the softmax warps read them)
          {
            const int it2 = it + 1, g2 = it2 * G + ((it2 & 1) ? (G - 1 - cta) : cta);
            if (g2 < total) {
              const Tile t2 = tile_of(g2, sh->prefix, nd, p.cu, p.tpt);
              for (int ch = 0; ch < p.nck; ++ch) tma_prefetch_3d(&qmap, ch * 64, 0, t2.t0);
            }
          }
        }
        {
          // the tile's q chunks that live in TMEM: half of them pass through
          // each ring (at most three per stage) and that ring's MMA issuer
          // copies them into TMEM with tcgen05.cp.  They need only ring
          // slots, which the previous tile's last stages of the ring free.
          const int qlo = r == 0 ? 0 : (p.nq_tmem + 1) / 2;
          const int qhi_end = r == 0 ? (p.nq_tmem + 1) / 2 : p.nq_tmem;
          for (int q0 = qlo; q0 < qhi_end; q0 += kChunksPerStage) {
            const int n = min(kChunksPerStage, qhi_end - q0);
            uint8_t* dst = open_stage(n * kChunkBytes);
            if (!dst) { stop = true; break; }
            const int sl = r * kSlots + (int)kst;
            for (int j = 0; j < n; ++j)
              tma_load_3d(dst + j * kChunkBytes, &qmap, &sh->kfull[sl], (q0 + j) * 64, 0, tl.t0);
            close_stage();
          }
          if (stop) break;
        }
        if (r == 0) {
          // the shared-memory chunk comes after them: its buffer is free only
          // once both issuers' MMAs of the previous tile are complete
          if (p.nq_smem > 0) {
            if (qfills > 0 && !mbar_wait(&sh->qhi_empty, (qfills - 1) & 1, lim)) {
              stop = true;
              break;
            }
            mbar_expect_tx(&sh->qhi_full, p.nq_smem * kChunkBytes);
            for (int j = 0; j < p.nq_smem; ++j)
              tma_load_3d(qhi + j * kChunkBytes, &qmap, &sh->qhi_full, (p.nq_tmem + j) * 64, 0,
                          tl.t0);
            ++qfills;
          }
        }
        // this ring's key tiles: stages of three K chunks in the MMA's order,
        // the TMEM chunks 0, 1, ... first, then the shared-memory (RoPE) chunk
        const int spt = (p.nck + kChunksPerStage - 1) / kChunksPerStage;  // stages per key tile
        for (int kt = 0; kt < nkt && !stop; ++kt) {
          if (((sbase + kt) & 1) != r) continue;
          for (int st = 0; st < spt; ++st) {
            const int nst = min(kChunksPerStage, p.nck - st * kChunksPerStage);
            uint8_t* dst = open_stage(nst * kChunkBytes);
            if (!dst) { stop = true; break; }
            const int sl = r * kSlots + (int)kst;
            for (int j = 0; j < nst; ++j) {
              const int ch = st * kChunksPerStage + j;  // K chunk = q chunk position
              tma_load_2d(dst + j * kChunkBytes, &kmap, &sh->kfull[sl], ch * 64,
                          tl.bos + kt * kKeyTile);
            }
            close_stage();
          }
        }
        sbase += nkt;
      }
      if (stop) give_up(sh, p.status);
      // no copy may still be landing when the CTA exits
      for (int s2 = 0; s2 < kSlots; ++s2)
        if (fills[s2] > 0)
          mbar_wait(&sh->kfull[r * kSlots + s2], (fills[s2] - 1) & 1, kDefaultWaitNs);
      if (qfills > 0) mbar_wait(&sh->qhi_full, (qfills - 1) & 1, kDefaultWaitNs);
    }
  } else if (warp == 1 || warp == kMmaB) {
    // ------------------------------------------------------------ MMA issuers
    // Issuer r issues the key tiles of global parity r from ring r into S
    // buffer r (the softmax warpgroup r reads it); two instruction streams,
    // so each one's pipeline waits overlap the other's MMAs.  Each issuer
    // also copies the half of a query tile's q that came through its ring
    // into TMEM, once both issuers' MMAs of the previous tile are complete
    // (qdone counts both), and commits qready; both wait for qready (count
    // 2: both halves copied) before their first MMA of the tile.
    const int r = warp == 1 ? 0 : 1;
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
      uint64_t qhi_desc[kMaxQhi];
#pragma unroll
      for (int j = 0; j < kMaxQhi; ++j)
        qhi_desc[j] = umma_desc_sw128(smem_u32(qhi + j * kChunkBytes), 16, 1024);
      const uint64_t stage_desc0 = umma_desc_sw128(smem_u32(stages), 16, 1024);
      uint32_t kst = 0, kph = 0, myidx = 0;
      int qtile = 0, sbase = 0;
      bool issued = false, ok = true;
      auto next_slot = [&]() {
        if (++kst == kSlots) {
          kst = 0;
          kph ^= 1;
        }
      };
      for (int it = 0; it * G < total && ok && !aborted(sh); ++it) {
        const int g = it * G + ((it & 1) ? (G - 1 - cta) : cta);
        if (g >= total) continue;
        const Tile tl = tile_of(g, sh->prefix, nd, p.cu, p.tpt);
        const int nkt = (tl.tend - tl.bos + kKeyTile - 1) / kKeyTile;
        {
          // this ring's half of q enters TMEM by tcgen05.cp, once every MMA
          // of the previous tile (which read the old q) has completed
          if (qtile > 0 && !mbar_wait_spin(&sh->qdone, (qtile - 1) & 1, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int qlo = r == 0 ? 0 : (p.nq_tmem + 1) / 2;
          const int qhi_end = r == 0 ? (p.nq_tmem + 1) / 2 : p.nq_tmem;
          for (int q0 = qlo; q0 < qhi_end; q0 += kChunksPerStage) {
            const int n = min(kChunksPerStage, qhi_end - q0);
            const int sl = r * kSlots + (int)kst;
            if (!mbar_wait_spin(&sh->kfull[sl], kph, lim)) {  // TMA stage
              ok = false;
              break;
            }
            const uint64_t b0 = stage_desc0 + (uint64_t)((sl * kStageBytes) >> 4);
            for (int j = 0; j < n; ++j)
#pragma unroll
              for (int k = 0; k < 4; ++k)  // 128 rows x 16 elements per copy
                tmem_cp_128x256b(tmem + (uint32_t)((q0 + j) * 32 + k * 8),
                                 b0 + (uint64_t)((j * kChunkBytes) >> 4) + 2 * k);
            umma_commit(&sh->kempty[sl]);  // the copies have read the stage
            next_slot();
          }
          if (!ok) break;
          umma_commit(&sh->qready);  // arrives once this issuer's copies have completed
          issued = true;
          // both halves in TMEM (every tile's phase is waited for)
          if (!mbar_wait_spin(&sh->qready, qtile & 1, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        const int spt = (p.nck + kChunksPerStage - 1) / kChunksPerStage;
        // the shared-memory q chunk is waited for once per tile, before its
        // first use (the last stage of a key tile), or at the tile's end
        bool qhi_seen = p.nq_smem == 0;
        for (int kt = 0; kt < nkt && ok; ++kt) {
          if (((sbase + kt) & 1) != r) continue;
          if (!mbar_wait_spin(&sh->sempty[r], (myidx & 1) ^ 1, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + kSCol + r * 128;
          if (p.nck == 9 && p.nq_smem > 0) {
            // Dk 576: the key tile's three stages written out, no dispatch
            // branch between their runs of MMAs
            auto stage_wait = [&](int& slo) -> bool {
              slo = r * kSlots + (int)kst;
              return mbar_wait_spin(&sh->kfull[slo], kph, lim);
            };
            int sl;
            if (!stage_wait(sl)) { ok = false; break; }
            issue_stage<true, false>(d, tmem, 0, 0,
                                     stage_desc0 + (uint64_t)((sl * kStageBytes) >> 4), idesc);
            umma_commit(&sh->kempty[sl]);
            next_slot();
            if (!stage_wait(sl)) { ok = false; break; }
            issue_stage<false, false>(d, tmem, 3, 0,
                                      stage_desc0 + (uint64_t)((sl * kStageBytes) >> 4), idesc);
            umma_commit(&sh->kempty[sl]);
            next_slot();
            if (!stage_wait(sl)) { ok = false; break; }
            if (!qhi_seen) {
              if (!mbar_wait(&sh->qhi_full, qtile & 1, lim)) { ok = false; break; }
              qhi_seen = true;
            }
            issue_stage<false, true>(d, tmem, 6, qhi_desc[0],
                                     stage_desc0 + (uint64_t)((sl * kStageBytes) >> 4), idesc);
            umma_commit(&sh->kempty[sl]);
            next_slot();
            issued = true;
            umma_commit(&sh->sfull[r]);
            ++myidx;
            continue;
          }
          for (int st = 0; st < spt; ++st) {
            const int sl = r * kSlots + (int)kst;
            if (!mbar_wait_spin(&sh->kfull[sl], kph, lim)) {  // TMA stage (no fence needed)
              ok = false;
              break;
            }
            const uint64_t b0 = stage_desc0 + (uint64_t)((sl * kStageBytes) >> 4);
            // 12 MMAs without a branch between them (a branch between two
            // tcgen05.mma costs about half the issue rate); one stage pattern
            // is chosen per stage
            const int tpos = st * kChunksPerStage;  // first TMEM chunk
            // a shorter last stage (Dk not a multiple of 192) only occurs
            // without a shared-memory q chunk (that needs 9 chunks: the last
            // stage is then TMEM chunks 6, 7 and the shared-memory chunk)
            const int nst = min(kChunksPerStage, p.nck - st * kChunksPerStage);
            if (st == spt - 1 && p.nq_smem > 0) {
              if (!qhi_seen) {
                if (!mbar_wait(&sh->qhi_full, qtile & 1, lim)) {
                  ok = false;
                  break;
                }
                qhi_seen = true;
              }
              issue_stage<false, true>(d, tmem, tpos, qhi_desc[0], b0, idesc);
            } else if (nst == kChunksPerStage) {
              if (st == 0) issue_stage<true, false>(d, tmem, tpos, 0, b0, idesc);
              else issue_stage<false, false>(d, tmem, tpos, 0, b0, idesc);
            } else if (nst == 2) {
              if (st == 0) issue_stage<true, false, 2>(d, tmem, tpos, 0, b0, idesc);
              else issue_stage<false, false, 2>(d, tmem, tpos, 0, b0, idesc);
            } else {
              if (st == 0) issue_stage<true, false, 1>(d, tmem, tpos, 0, b0, idesc);
              else issue_stage<false, false, 1>(d, tmem, tpos, 0, b0, idesc);
            }
            issued = true;
            umma_commit(&sh->kempty[sl]);
            next_slot();
          }
          if (!ok) break;
          umma_commit(&sh->sfull[r]);
          ++myidx;
        }
        if (!ok) break;
        // every tile's phase of the shared-memory chunk is waited for, even
        // with no key tile of this parity (a parity wait must never run two
        // phases ahead of its barrier)
        if (!qhi_seen && !mbar_wait(&sh->qhi_full, qtile & 1, lim)) {
          ok = false;
          break;
        }
        // this issuer is done with the tile's q (both commit; count 2)
        if (p.nq_smem > 0) umma_commit(&sh->qhi_empty);
        umma_commit(&sh->qdone);
        ++qtile;
        sbase += nkt;
      }
      if (!ok) give_up(sh, p.status);
      if (issued) {  // every MMA and copy done before TMEM is released
        umma_commit(&sh->drain[r]);
        mbar_wait(&sh->drain[r], 0, kDefaultWaitNs);
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    // Two warpgroups; warpgroup wg owns S buffer wg, i.e. every other S tile.
    // Per-row (max, sum) pairs are combined at the end of the query tile.
    const int wg = (warp - 2) >> 2;
    const int g4 = warp & 3;
    const int r = 32 * g4 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * g4) << 16);
    const int H = p.H;
    const int hp = H / 32;  // warps per token
    const float sl2 = p.scale_log2;
    // two workspace halves by query-tile parity: one warpgroup may already
    // write the next tile's block values while the other still reads this
    // tile's in its epilogue (they are never more than one tile apart)
    float* const ws_cta = p.ws + (size_t)blockIdx.x * 2 * p.nbmax * 128 + r;
    uint32_t sbase = 0, all_ph = 0, wg_ph = 0;
    bool ok = true;
    auto tile_at = [&](int it2, Tile& out) -> bool {
      if (it2 * G >= total) return false;
      const int g2 = it2 * G + ((it2 & 1) ? (G - 1 - cta) : cta);
      if (g2 >= total) return false;
      out = tile_of(g2, sh->prefix, nd, p.cu, p.tpt);
      return true;
    };
    Tile cur;
    bool have = tile_at(0, cur);
    for (int it = 0; have && ok && !aborted(sh); ++it) {
      const Tile tl = cur;
      const int tok = tl.t0 + r / H;
      const int h = r % H;
      const bool valid = tok < tl.tend;
      const int tok_c = valid ? tok : tl.tend - 1;
      const int nkt = (tl.tend - tl.bos + kKeyTile - 1) / kKeyTile;
      float m = -INFINITY, l = 0.f;  // log2 domain
      float* const ws_row = ws_cta + (size_t)(it & 1) * p.nbmax * 128;
      for (int kt = 0; kt < nkt; ++kt) {
        const uint32_t gs = sbase + kt;
        if ((int)(gs & 1) != wg) continue;
        if (!mbar_wait(&sh->sfull[wg], (gs >> 1) & 1, lim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int key0 = tl.bos + kt * kKeyTile;
        const bool need_mask = key0 + kKeyTile - 1 > tl.t0;
        const uint32_t sa = lane_base + kSCol + wg * 128;
        float bm = -INFINITY, bs = 0.f;  // running block max (raw logits) and sum
        auto finish_block = [&](int bidx) {
          float blse = -INFINITY;
          if (bm != -INFINITY) {
            blse = fmaf(bm, sl2, fast_log2(bs));
            const float mn = fmaxf(m, blse);
            l = l * fast_exp2(m - mn) + fast_exp2(blse - mn);
            m = mn;
          }
          const int bg = kt * (kKeyTile / B) + bidx;
          if (bg < p.nbmax) ws_row[(size_t)bg * 128] = blse;
          bm = -INFINITY;
          bs = 0.f;
        };
        // one 32-column chunk of S (raw logits in u)
        auto chunk = [&](int j, uint32_t (&u)[32]) {
          if (need_mask) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (key0 + 32 * j + i > tok_c) u[i] = 0xff800000u;  // -inf
          }
          float (&x)[32] = reinterpret_cast<float (&)[32]>(u);
          if (B >= 32) {
            float cm = x[0];
#pragma unroll
            for (int i = 1; i < 32; ++i) cm = fmaxf(cm, x[i]);
            if (cm > bm) {
              bs *= fast_exp2((bm - cm) * sl2);
              bm = cm;
            }
            if (bm != -INFINITY) {
              const float nb = -bm * sl2;
              float a0 = 0.f, a1 = 0.f;
#pragma unroll
              for (int i = 0; i < 32; i += 2) {
                a0 += fast_exp2(fmaf(x[i], sl2, nb));
                a1 += fast_exp2(fmaf(x[i + 1], sl2, nb));
              }
              bs += a0 + a1;
            }
            if (((32 * j + 32) % B) == 0) finish_block((32 * j) / B);
          } else {
#pragma unroll
            for (int hb = 0; hb < 32 / B; ++hb) {
              float cm = x[hb * B];
#pragma unroll
              for (int i = 1; i < B; ++i) cm = fmaxf(cm, x[hb * B + i]);
              bm = cm;
              if (bm != -INFINITY) {
                const float nb = -bm * sl2;
                float a0 = 0.f;
#pragma unroll
                for (int i = 0; i < B; ++i) a0 += fast_exp2(fmaf(x[hb * B + i], sl2, nb));
                bs = a0;
              }
              finish_block((32 * j) / B + hb);
            }
          }
        };
        uint32_t u0[32], u1[32], u2[32], u3[32];
        tmem_ld32(sa, u0);
        tmem_ld32(sa + 32, u1);
        tmem_ld32(sa + 64, u2);
        tmem_ld32(sa + 96, u3);
        tmem_ld_wait();
        reg_fence(u0);
        reg_fence(u1);
        reg_fence(u2);
        reg_fence(u3);
        tc_fence_before();
        mbar_arrive(&sh->sempty[wg]);  // whole tile is in registers
        chunk(0, u0);
        chunk(1, u1);
        chunk(2, u2);
        chunk(3, u3);
      }
      if (!ok) break;
      sbase += nkt;
      // ---- combine the two warpgroups' row statistics
      const int mb = it & 1;
      sh->ml[mb][wg][0][r] = m;
      sh->ml[mb][wg][1][r] = l;
      mbar_arrive(&sh->epi_all);
      if (!mbar_wait(&sh->epi_all, all_ph, lim)) { ok = false; break; }
      all_ph ^= 1;
      const float m0 = sh->ml[mb][0][0][r], l0 = sh->ml[mb][0][1][r];
      const float m1 = sh->ml[mb][1][0][r], l1 = sh->ml[mb][1][1][r];
      const float M = fmaxf(m0, m1);
      const float L = (m0 == -INFINITY ? 0.f : l0 * fast_exp2(m0 - M)) +
                      (m1 == -INFINITY ? 0.f : l1 * fast_exp2(m1 - M));
      const float lse2 = M + fast_log2(L);
      if (wg == 0 && valid) p.lse[(int64_t)tok * H + h] = lse2 * kLn2;
      have = tile_at(it + 1, cur);
      // ---- head-summed block masses (and optional per-head block LSE)
      const int bq = valid ? (tok - tl.bos) / B : -1;
      float* blo = (valid && p.block_lse) ? p.block_lse + ((int64_t)tok * H + h) * p.nbs : nullptr;
      const int tkw = g4 / hp;
      const bool first = (g4 % hp) == 0;
      const int tok_w = tl.t0 + tkw;
      const int nbatch = (p.nbmax + 31) / 32;
      for (int bi = wg; bi < nbatch; bi += 2) {
        const int bb0 = bi * 32;
        // all 32 workspace loads first: interleaved with the block_lse
        // stores, which may alias them, they would run one L2 round trip at
        // a time
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = bb0 + j <= bq ? ws_row[(size_t)(bb0 + j) * 128] : 0.f;
        if (blo) {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int b = bb0 + j;
            if (b <= bq) blo[b] = v[j] * kLn2;
            else if (b < p.nbmax) blo[b] = -INFINITY;
          }
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = bb0 + j <= bq ? fast_exp2(v[j] - lse2) : 0.f;
        const float s = transpose_reduce_sum(v);
        sh->red[wg][g4][lane] = s;
        mbar_arrive(&sh->epi_wg[wg]);
        if (!mbar_wait(&sh->epi_wg[wg], wg_ph, lim)) { ok = false; break; }
        wg_ph ^= 1;
        if (first && tok_w < tl.tend && bb0 + lane < p.nbmax) {
          float acc = 0.f;
          for (int i = 0; i < hp; ++i) acc += sh->red[wg][g4 + i][lane];
          p.block_score[(int64_t)tok_w * p.nbs + bb0 + lane] = acc;
        }
        mbar_arrive(&sh->epi_wg[wg]);
        if (!mbar_wait(&sh->epi_wg[wg], wg_ph, lim)) { ok = false; break; }
        wg_ph ^= 1;
      }
    }
    if (!ok) give_up(sh, p.status);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

int grid_for(int total_tokens, int num_docs, int num_heads) {
  const int tpt = 128 / num_heads;
  const long long tiles = (long long)(total_tokens + tpt - 1) / tpt + num_docs;
  return (int)(tiles < sm_count() ? tiles : sm_count());
}

}  // namespace

bool tc_block_score_supported(int num_heads, int dk, int block_size, int nbmax) {
  (void)nbmax;
  // 64-column chunks, at most kMaxTmemQ in TMEM and kMaxQhi in shared memory
  return (num_heads == 32 || num_heads == 64 || num_heads == 128) && dk % 64 == 0 &&
         dk >= 64 && dk <= 64 * (kMaxTmemQ + kMaxQhi) &&
         (block_size == 16 || block_size == 32 || block_size == 64 || block_size == 128);
}

size_t tc_block_score_workspace(int total_tokens, int num_docs, int num_heads, int nbmax) {
  return (size_t)grid_for(total_tokens, num_docs, num_heads) * 2 * nbmax * 128 * sizeof(float);
}

// Data-dependent conditions of the tensor-core path (alignment, doc count).
bool tc_block_score_eligible(const ScoreArgs& a) {
  const Problem& p = a.p;
  return p.num_docs <= kMaxDocs && (reinterpret_cast<uintptr_t>(p.q) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(p.k) & 15) == 0 && p.q_row_stride % 8 == 0 &&
         p.q_head_stride % 8 == 0 && p.k_row_stride % 8 == 0;
}

cudaError_t launch_tc_block_score(const ScoreArgs& a, long long wait_limit, cudaStream_t s) {
  const Problem& p = a.p;
  CUtensorMap kmap, qmap;
  {
    const uint64_t dims[2] = {(uint64_t)p.dk, (uint64_t)p.total_tokens};
    const uint64_t strides[1] = {(uint64_t)p.k_row_stride * 2};
    const uint32_t box[2] = {64, kKeyTile};
    if (!encode_bf16_map(&kmap, p.k, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  const int tpt = 128 / p.num_heads;
  {
    const uint64_t dims[3] = {(uint64_t)p.dk, (uint64_t)p.num_heads, (uint64_t)p.total_tokens};
    const uint64_t strides[2] = {(uint64_t)p.q_head_stride * 2, (uint64_t)p.q_row_stride * 2};
    const uint32_t box[3] = {64, (uint32_t)p.num_heads, (uint32_t)tpt};
    if (!encode_bf16_map(&qmap, p.q, 3, dims, strides, box)) return cudaErrorInvalidValue;
  }
  BSParams bp;
  bp.cu = p.cu_seqlens;
  bp.num_docs = p.num_docs;
  bp.T = p.total_tokens;
  bp.max_seqlen = p.max_seqlen;
  bp.q = static_cast<const __nv_bfloat16*>(p.q);
  bp.qrs = p.q_row_stride;
  bp.qhs = p.q_head_stride;
  bp.H = p.num_heads;
  bp.nck = p.dk / 64;
  bp.nq_tmem = bp.nck < kMaxTmemQ ? bp.nck : kMaxTmemQ;
  bp.nq_smem = bp.nck - bp.nq_tmem;
  bp.tpt = tpt;
  bp.nbmax = a.nbmax;
  bp.nbs = a.nb_stride;
  bp.scale_log2 = p.scale * kLog2e;
  bp.lse = a.lse;
  bp.block_score = a.block_score;
  bp.block_lse = a.block_lse;
  bp.ws = static_cast<float*>(a.workspace);
  bp.status = p.status;
  bp.wait_ns = wait_limit > 0 ? wait_limit : kDefaultWaitNs;
  const int grid = grid_for(p.total_tokens, p.num_docs, p.num_heads);
  void (*kern)(const CUtensorMap, const CUtensorMap, const BSParams) = nullptr;
  switch (a.block_size) {
    case 16: kern = tc_block_score_kernel<16>; break;
    case 32: kern = tc_block_score_kernel<32>; break;
    case 64: kern = tc_block_score_kernel<64>; break;
    default: kern = tc_block_score_kernel<128>; break;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  kern<<<grid, kThreads, kSmemBytes, s>>>(kmap, qmap, bp);
  return cudaGetLastError();
}

}  // namespace hs
