// The dk / dv pass of the attention backward on warp-level tensor-core MMAs
// (mma.sync m16n8k16, bf16 in, fp32 accumulate), for bf16 inputs with 64
// heads, Dk and Dv multiples of 64 (Dk <= 576, Dv <= 512); the dq pass runs
// on tcgen05 (tc_bwd_dq.cu).
//
// Definitions as in simt_backward.cu ("HySparse MQA sparse attention ...",
// PaddleFleet pull request 1470, "Core" list: SWA and block-sparse MQA
// backward): for every key j and every (t, h) with j in S_t,
//   dk[j] += scale * ds * q[t,h],  dv[j] += p * dout[t,h],
//   p = exp(scale <q[t,h], k[j]> - lse[t,h]),  ds = p (<dout[t,h], v[j]> - delta[t,h]).
//
// Why warp-level MMAs here: a key tile's dk and dv accumulators (keys x
// (Dk + Dv) fp32) do not fit the 512 TMEM columns beside the score tiles at
// Dk 576 / Dv 512, while registers spread over 16 warps hold them for a tile
// of 32 keys.  A cluster of four CTAs per 32-key tile (split at document
// boundaries); each keeps the tile's K and V rows in shared memory, finds the
// queries whose key set meets the tile by scanning candidate idx rows (or the
// window), takes every fourth of them in ascending order, and the four
// partial sums are added in rank order through distributed shared memory
// (a tile every query selects, such as a document's first block, is then
// spread over four SMs).  Per member token t (all 64 heads):
//   S^T [32 keys x 64 heads]  = K_tile . q_t^T      (warps 0-7, 16x16 each)
//   dP^T[32 x 64]             = V_tile . dout_t^T   (warps 8-15, 16x16 each)
//   P^T, dS^T (bf16)          -> shared memory      (dP^T passed to the S^T
//                                                    warps through it, fp32)
//   dK[32 x Dk] += dS^T . q_t,  dV[32 x Dv] += P^T . dout_t   (registers)
// Sums run in a fixed order: results are deterministic.

#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <math.h>

#include "hs_device.cuh"
#include "hs_internal.h"

namespace hs {
namespace {

namespace cg = cooperative_groups;

constexpr int kThreads = 512;   // 16 warps
constexpr int kCluster = 4;     // CTAs sharing one key tile (dk / dv pass)
constexpr int kKT = 32;         // keys per tile (two m16 tiles)
constexpr int kH = 64;          // heads
constexpr int kPad = 8;         // bf16 elements of row padding (16 bytes)
constexpr int kMaxNK = 9;       // Dk / 64 n-tiles per warp (Dk <= 576)
constexpr int kMaxNV = 8;       // Dv / 64 (Dv <= 512)
constexpr int kPS = kH + kPad;  // row stride of the P^T / dS^T tiles

struct MmaBwdParams {
  Problem p;
  const int32_t* idx;
  int topk, B, window;
  const float* lse;
  const float* delta;
  const __nv_bfloat16* dout;
  float* dkey;
  float* dval;
  float* dq;
};

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two 8x8 bf16 matrices stored row-major by k (rows k0..k0+15, 8 columns n0..)
// loaded transposed: the B fragment (k pairs per n) of an m16n8k16 MMA.
// Lanes 0-15 give the row addresses.
__device__ __forceinline__ void ldsm_x2_trans(uint32_t& b0, uint32_t& b1, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(b0), "=r"(b1)
               : "r"(addr));
}

// Four 8x8 bf16 matrices, row addresses from lanes 8i..8i+7 for matrix i
// (not transposed): the A fragment of an m16n8k16 MMA (rows 0-15 x k 0-15),
// or the B fragments of two n8 tiles stored as [n][k] rows.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t lds32(const __nv_bfloat16* p) {
  return *reinterpret_cast<const uint32_t*>(p);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

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

// Asynchronous 16-byte global -> shared copy (completion: cp_async_wait_all).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

// q_t and dout_t of one token, all heads, into padded shared-memory tiles
// (asynchronous copies, all in flight at once; the caller waits and syncs).
__device__ __forceinline__ void stage_token(__nv_bfloat16* Qs, int KS, __nv_bfloat16* Ds, int VS,
                                            const __nv_bfloat16* qg, int64_t qrs, int64_t qhs,
                                            const __nv_bfloat16* dout, int t, int dk, int dv) {
  const int vq = dk >> 3, vd = dv >> 3;
  for (int e = threadIdx.x; e < kH * vq; e += kThreads) {
    const int h = e / vq, c = (e - h * vq) << 3;
    cp_async16(Qs + h * KS + c, qg + (int64_t)t * qrs + (int64_t)h * qhs + c);
  }
  for (int e = threadIdx.x; e < kH * vd; e += kThreads) {
    const int h = e / vd, c = (e - h * vd) << 3;
    cp_async16(Ds + h * VS + c, dout + ((int64_t)t * kH + h) * dv + c);
  }
}

// 16-byte copy of `rows` rows of `cols` bf16 (cols % 8 == 0) into a padded
// shared-memory tile; row r of the source starts at src + r * stride.
// Rows past `rows` (up to zero_rows_to) are zeroed.  Asynchronous for the
// copied rows: the caller waits (cp_async_wait_all) and syncs.
__device__ __forceinline__ void copy_rows(__nv_bfloat16* dst, int dst_stride,
                                          const __nv_bfloat16* src, int64_t stride, int rows,
                                          int cols, int zero_rows_to) {
  const int vpr = cols >> 3;  // 16-byte vectors per row
  for (int e = threadIdx.x; e < zero_rows_to * vpr; e += kThreads) {
    const int r = e / vpr, c = (e - r * vpr) << 3;
    if (r < rows)
      cp_async16(dst + r * dst_stride + c, src + (int64_t)r * stride + c);
    else
      *reinterpret_cast<uint4*>(dst + r * dst_stride + c) = make_uint4(0u, 0u, 0u, 0u);
  }
}

inline size_t mma_dkdv_smem_bytes(int dk, int dv) {
  const int KS = dk + kPad, VS = dv + kPad;
  return 2 * ((size_t)kKT * KS + (size_t)kKT * VS + (size_t)kH * KS + (size_t)kH * VS +
              2 * (size_t)kKT * kPS) +
         4 * 2 * (size_t)kH + 4 * 2 * (size_t)kThreads;
}

template <bool kSparse>
__global__ void __launch_bounds__(kThreads, 1) bwd_dkdv_mma_kernel(const MmaBwdParams a) {
  extern __shared__ __align__(16) uint8_t smraw[];
  __shared__ int wcount[kThreads / 32];
  const Problem& P = a.p;
  const int dk = P.dk, dv = P.dv, KS = dk + kPad, VS = dv + kPad;
  __nv_bfloat16* Kt = reinterpret_cast<__nv_bfloat16*>(smraw);  // [kKT][KS]
  __nv_bfloat16* Vt = Kt + kKT * KS;                             // [kKT][VS]
  __nv_bfloat16* Qs = Vt + kKT * VS;                             // [kH][KS]  q_t
  __nv_bfloat16* Ds = Qs + kH * KS;                              // [kH][VS]  dout_t
  __nv_bfloat16* Ps = Ds + kH * VS;                              // [kKT][kPS] P^T
  __nv_bfloat16* Ss = Ps + kKT * kPS;                            // [kKT][kPS] dS^T
  float* lse_s = reinterpret_cast<float*>(Ss + kKT * kPS);
  float* del_s = lse_s + kH;
  int* mem = reinterpret_cast<int*>(del_s + kH);                 // [kThreads]
  int* memmask = mem + kThreads;                                 // [kThreads]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, tig = lane & 3;
  const int wm = warp >> 3;  // 16-key half of the tile
  const int wn = warp & 7;   // 8-head tile (scores) / n-tile phase (dk, dv)
  const int nK = dk >> 6, nV = dv >> 6;
  const float scale = P.scale;
  const int NT = P.total_tokens;
  const uint32_t qs_base = (uint32_t)__cvta_generic_to_shared(Qs);
  const uint32_t ds_base = (uint32_t)__cvta_generic_to_shared(Ds);
  const __nv_bfloat16* qg = static_cast<const __nv_bfloat16*>(P.q);
  const __nv_bfloat16* kg = static_cast<const __nv_bfloat16*>(P.k);
  const __nv_bfloat16* vg = static_cast<const __nv_bfloat16*>(P.v);
  // Score phase: warp w < 8 computes S^T, warp w + 8 the dP^T block at the
  // same place: keys 16 mt.., heads 16 np.. (two n8 tiles sharing each A
  // fragment; ldmatrix for A and B).  dP^T goes to the S^T warp through an
  // fp32 tile [kKT][kDP] laid over the P^T / dS^T buffers.
  const bool s_warp = warp < 8;
  const int mt = (warp >> 2) & 1, np = warp & 3;
  constexpr int kDP = 72;  // fp32 row stride of the dP^T hand-over tile
  static_assert(kKT * kDP * 4 <= 2 * kKT * kPS * 2, "dP tile must fit the P / dS buffers");
  float* dpx = reinterpret_cast<float*>(Ps);
  const uint32_t a_sc = (uint32_t)__cvta_generic_to_shared(s_warp ? Kt : Vt) +
                        (uint32_t)(((mt * 16 + (lane & 15)) * (s_warp ? KS : VS) +
                                    (lane >> 4) * 8) * 2);
  const uint32_t b_sc = (s_warp ? qs_base : ds_base) +
                        (uint32_t)(((np * 16 + (lane & 7) + ((lane >> 4) << 3)) *
                                        (s_warp ? KS : VS) +
                                    ((lane >> 3) & 1) * 8) * 2);
  const int kend_sc = s_warp ? dk : dv;
  // The CTAs of a cluster share one key tile: each scans every candidate
  // (so all see the same member list) and takes every csize-th member; their
  // partial sums are added in rank order through distributed shared memory.
  cg::cluster_group cl = cg::this_cluster();
  const int crank = (int)cl.block_rank(), csize = (int)cl.num_blocks();
  const int ncl = gridDim.x / csize;
  for (int tile = blockIdx.x / csize; tile * kKT < NT; tile += ncl) {
    const int j1 = min(NT, tile * kKT + kKT);
    for (int s0 = tile * kKT; s0 < j1;) {  // one document segment at a time
      int bos, eos;
      if (!find_doc(P.cu_seqlens, P.num_docs, NT, P.max_seqlen, s0, bos, eos, P.status)) break;
      const int s1 = min(j1, eos), n = s1 - s0;
      copy_rows(Kt, KS, kg + (int64_t)s0 * P.k_row_stride, P.k_row_stride, n, dk, kKT);
      copy_rows(Vt, VS, vg + (int64_t)s0 * P.v_row_stride, P.v_row_stride, n, dv, kKT);
      cp_async_wait_all();  // published by the candidate loop's first barrier
      float accK[kMaxNK][4], accV[kMaxNV][4];
#pragma unroll
      for (int i = 0; i < kMaxNK; ++i) accK[i][0] = accK[i][1] = accK[i][2] = accK[i][3] = 0.f;
#pragma unroll
      for (int i = 0; i < kMaxNV; ++i) accV[i][0] = accV[i][1] = accV[i][2] = accV[i][3] = 0.f;
      const int tend = kSparse ? eos : min(eos, s1 - 1 + a.window);
      const int b_lo = kSparse ? (s0 - bos) / a.B : 0;
      const int b_hi = kSparse ? (s1 - 1 - bos) / a.B : 0;
      for (int c0 = s0; c0 < tend; c0 += kThreads) {
        // candidate query t = c0 + tid: which of the segment's keys it attends
        const int t = c0 + tid;
        uint32_t mask = 0;
        if (t < tend) {
          if (kSparse) {
            const int bq = (t - bos) / a.B;
            const int32_t* row = a.idx + (int64_t)t * a.topk;
            bool f[3];  // the segment's keys lie in at most three blocks (B >= 16)
#pragma unroll
            for (int q = 0; q < 3; ++q) f[q] = b_lo + q <= b_hi && selects(row, a.topk, bq, b_lo + q);
            for (int jj = 0; jj < n; ++jj) {
              const int j = s0 + jj;
              if (j <= t && f[(j - bos) / a.B - b_lo]) mask |= 1u << jj;
            }
          } else {
            for (int jj = 0; jj < n; ++jj) {
              const int j = s0 + jj;
              if (j <= t && j > t - a.window) mask |= 1u << jj;
            }
          }
        }
        const unsigned bal = __ballot_sync(0xffffffffu, mask != 0);
        if (lane == 0) wcount[warp] = __popc(bal);
        __syncthreads();
        int off = 0, nm = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
          if (w < warp) off += wcount[w];
          nm += wcount[w];
        }
        if (mask) {
          const int pos = off + __popc(bal & ((1u << lane) - 1u));
          mem[pos] = t;
          memmask[pos] = (int)mask;
        }
        __syncthreads();
        for (int mi = crank; mi < nm; mi += csize) {
          const int tt = mem[mi];
          const uint32_t mk = (uint32_t)memmask[mi];
          // q_t and dout_t, all heads, and the token's lse / delta
          stage_token(Qs, KS, Ds, VS, qg, P.q_row_stride, P.q_head_stride, a.dout, tt, dk, dv);
          if (tid < kH) {
            lse_s[tid] = __ldg(a.lse + (int64_t)tt * kH + tid);
            del_s[tid] = __ldg(a.delta + (int64_t)tt * kH + tid);
          }
          cp_async_wait_all();
          __syncthreads();
          // S^T (warps 0-7) or dP^T (warps 8-15) for keys 16 mt.. x heads 16 np..
          float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
          for (int k0 = 0; k0 < kend_sc; k0 += 16) {
            uint32_t af[4], bf[4];
            ldsm_x4(af, a_sc + (uint32_t)(k0 * 2));
            ldsm_x4(bf, b_sc + (uint32_t)(k0 * 2));
            mma16816(acc2[0], af, bf[0], bf[1]);
            mma16816(acc2[1], af, bf[2], bf[3]);
          }
          const int r0 = mt * 16 + g;
          if (!s_warp) {  // hand dP^T over (the P^T / dS^T buffers are free here)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int h = np * 16 + 8 * j + 2 * tig;
              *reinterpret_cast<float2*>(dpx + r0 * kDP + h) = make_float2(acc2[j][0], acc2[j][1]);
              *reinterpret_cast<float2*>(dpx + (r0 + 8) * kDP + h) =
                  make_float2(acc2[j][2], acc2[j][3]);
            }
          }
          __syncthreads();
          float dpv[2][4];
          if (s_warp) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int h = np * 16 + 8 * j + 2 * tig;
              const float2 lo = *reinterpret_cast<const float2*>(dpx + r0 * kDP + h);
              const float2 hi = *reinterpret_cast<const float2*>(dpx + (r0 + 8) * kDP + h);
              dpv[j][0] = lo.x;
              dpv[j][1] = lo.y;
              dpv[j][2] = hi.x;
              dpv[j][3] = hi.y;
            }
          }
          __syncthreads();  // every dP^T value read before P^T / dS^T overwrite the tile
          // P^T = exp(s - lse) on member keys, dS^T = P^T (dP^T - delta)
          if (s_warp) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              const int h0 = np * 16 + 8 * j + 2 * tig;
              float pv[4], dsv[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int key = r0 + ((q & 2) ? 8 : 0), head = h0 + (q & 1);
                const float pr =
                    ((mk >> key) & 1u) ? expf(acc2[j][q] * scale - lse_s[head]) : 0.f;
                pv[q] = pr;
                dsv[q] = pr * (dpv[j][q] - del_s[head]);
              }
              *reinterpret_cast<uint32_t*>(Ps + r0 * kPS + h0) = pack_bf16(pv[0], pv[1]);
              *reinterpret_cast<uint32_t*>(Ps + (r0 + 8) * kPS + h0) = pack_bf16(pv[2], pv[3]);
              *reinterpret_cast<uint32_t*>(Ss + r0 * kPS + h0) = pack_bf16(dsv[0], dsv[1]);
              *reinterpret_cast<uint32_t*>(Ss + (r0 + 8) * kPS + h0) = pack_bf16(dsv[2], dsv[3]);
            }
          }
          __syncthreads();
          // dK += dS^T . q_t and dV += P^T . dout_t over the 64 heads
#pragma unroll
          for (int ks = 0; ks < kH / 16; ++ks) {
            const __nv_bfloat16* sa = Ss + (wm * 16 + g) * kPS + ks * 16 + 2 * tig;
            const uint32_t afs[4] = {lds32(sa), lds32(sa + 8 * kPS), lds32(sa + 8),
                                     lds32(sa + 8 * kPS + 8)};
            const __nv_bfloat16* pa = Ps + (wm * 16 + g) * kPS + ks * 16 + 2 * tig;
            const uint32_t afp[4] = {lds32(pa), lds32(pa + 8 * kPS), lds32(pa + 8),
                                     lds32(pa + 8 * kPS + 8)};
            const int brow = ks * 16 + (lane & 15);
            const uint32_t qrow = qs_base + (uint32_t)(brow * KS) * 2u;
            const uint32_t drow = ds_base + (uint32_t)(brow * VS) * 2u;
#pragma unroll
            for (int i = 0; i < kMaxNK; ++i) {
              if (i < nK) {
                uint32_t b0, b1;
                ldsm_x2_trans(b0, b1, qrow + (uint32_t)((wn + 8 * i) * 16));
                mma16816(accK[i], afs, b0, b1);
              }
            }
#pragma unroll
            for (int i = 0; i < kMaxNV; ++i) {
              if (i < nV) {
                uint32_t b0, b1;
                ldsm_x2_trans(b0, b1, drow + (uint32_t)((wn + 8 * i) * 16));
                mma16816(accV[i], afp, b0, b1);
              }
            }
          }
          __syncthreads();
        }
      }
      // this CTA's partial sums -> its shared memory (the q / dout staging
      // area is free: [kKT][Dk + Dv] fp32); the cluster adds them in rank
      // order, rank r writing keys r, r + csize, ... of the segment
      {
        const int W = dk + dv, r0 = wm * 16 + g;
        float* part = reinterpret_cast<float*>(Qs);
#pragma unroll
        for (int i = 0; i < kMaxNK; ++i) {
          if (i < nK) {
            const int col = (wn + 8 * i) * 8 + 2 * tig;
            *reinterpret_cast<float2*>(part + r0 * W + col) = make_float2(accK[i][0], accK[i][1]);
            *reinterpret_cast<float2*>(part + (r0 + 8) * W + col) =
                make_float2(accK[i][2], accK[i][3]);
          }
        }
#pragma unroll
        for (int i = 0; i < kMaxNV; ++i) {
          if (i < nV) {
            const int col = dk + (wn + 8 * i) * 8 + 2 * tig;
            *reinterpret_cast<float2*>(part + r0 * W + col) = make_float2(accV[i][0], accV[i][1]);
            *reinterpret_cast<float2*>(part + (r0 + 8) * W + col) =
                make_float2(accV[i][2], accV[i][3]);
          }
        }
        cl.sync();
        const int mine = n > crank ? (n - crank + csize - 1) / csize : 0;
        for (int e = tid; e < mine * W; e += kThreads) {
          const int kk = crank + (e / W) * csize, col = e - (e / W) * W;
          float sum = 0.f;
          for (int rr = 0; rr < csize; ++rr) sum += cl.map_shared_rank(part, rr)[kk * W + col];
          if (col < dk)
            a.dkey[(int64_t)(s0 + kk) * dk + col] = scale * sum;
          else
            a.dval[(int64_t)(s0 + kk) * dv + (col - dk)] = sum;
        }
        cl.sync();  // no CTA reuses its shared memory while another still reads it
      }
      s0 = s1;
    }
  }
}

}  // namespace

bool mma_backward_shape_ok(hs_dtype dtype, int num_heads, int dk, int dv) {
  return dtype == HS_BF16 && num_heads == kH && dk % 64 == 0 && dk >= 64 && dk <= 64 * kMaxNK &&
         dv % 64 == 0 && dv >= 64 && dv <= 64 * kMaxNV;
}

bool mma_backward_supported(const Problem& p) {
  auto al16 = [](const void* x) { return (reinterpret_cast<uintptr_t>(x) & 15) == 0; };
  return mma_backward_shape_ok(p.dtype, p.num_heads, p.dk, p.dv) &&
         al16(p.q) && al16(p.k) && al16(p.v) && p.q_row_stride % 8 == 0 &&
         p.q_head_stride % 8 == 0 && p.k_row_stride % 8 == 0 && p.v_row_stride % 8 == 0 &&
         mma_dkdv_smem_bytes(p.dk, p.dv) <= 227 * 1024;
}

cudaError_t launch_mma_dkdv(const BwdArgs& b, bool sparse, const float* delta, cudaStream_t s) {
  MmaBwdParams a;
  a.p = b.p;
  a.idx = b.idx;
  a.topk = b.topk;
  a.B = b.block_size;
  a.window = b.window;
  a.lse = b.lse;
  a.delta = delta;
  a.dout = static_cast<const __nv_bfloat16*>(b.dout);
  a.dkey = b.dkey;
  a.dval = b.dval;
  a.dq = nullptr;
  const size_t bytes = mma_dkdv_smem_bytes(b.p.dk, b.p.dv);
  auto kern = sparse ? bwd_dkdv_mma_kernel<true> : bwd_dkdv_mma_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
  if (e != cudaSuccess) return e;
  const int tiles = (b.p.total_tokens + kKT - 1) / kKT;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kCluster;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = bytes;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // clusters of kCluster CTAs when the device can place them, else single CTAs
  int nclusters = 0;
  cfg.gridDim = dim3(tiles * kCluster);
  if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) != cudaSuccess || nclusters < 1) {
    (void)cudaGetLastError();
    attr[0].val.clusterDim.x = 1;
    cfg.gridDim = dim3(tiles);
  }
  return cudaLaunchKernelEx(&cfg, kern, a);
}

}  // namespace hs
