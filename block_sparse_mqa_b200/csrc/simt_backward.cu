// Backward of hs_sparse_mqa_fwd and hs_swa_mqa_fwd on CUDA cores (fp32
// arithmetic, bf16 or fp32 inputs).
//
// Definitions ("HySparse MQA sparse attention ...", PaddleFleet pull request
// 1470, "Core" list: the SWA and block-sparse MQA kernels have backward
// passes and the learnable per-head attn_sink an analytic gradient; per-file
// table: windowed MQA fwd/bwd with Dk != Dv and attn_sink).  The backward is
// the exact gradient of the forward; with s_j = scale <q[t,h], k[j]>,
// p_j = exp(s_j - lse[t,h]) (lse includes the sink), dp_j = <dout[t,h], v[j]>:
//   delta[t,h] = <dout[t,h], out[t,h]>
//   ds_j       = p_j (dp_j - delta[t,h])
//   dq[t,h]    = scale sum_{j in S_t} ds_j k[j]
//   dk[j]      = scale sum_{(t,h): j in S_t} ds_j q[t,h]
//   dv[j]      = sum_{(t,h): j in S_t} p_j dout[t,h]
//   dsink[h]   = -sum_t exp(sink[h] - lse[t,h]) delta[t,h]
//
// Four kernels, every sum in a fixed order (results are deterministic):
//   delta      one warp per (t, h): delta and the token's sink term
//   dsink      one CTA per head: the sink terms summed over t
//   dq         query-major, one CTA per token: heads in groups of G, the
//              token's key set in tiles of KT keys staged in shared memory
//   dkdv       key-major, one CTA per tile of 16 consecutive keys: the tokens
//              whose key set meets the tile (found by scanning candidate
//              tokens' idx rows, or the window) are visited in ascending
//              order and their contributions accumulated in shared memory

#include <math.h>

#include "hs_device.cuh"
#include "hs_internal.h"

namespace hs {
namespace {

constexpr int kThreads = 256;
constexpr int kKeyTile = 16;  // keys per dk/dv tile (<= the smallest block size)

struct BwdParams {
  Problem p;
  const int32_t* idx;
  int topk, B, window;
  const float* sink;
  const void* out;
  const float* lse;
  const void* dout;
  float* dq;
  float* dkey;
  float* dval;
  float* dsink;
  float* delta;       // workspace [T, H]
  float* dsink_part;  // workspace [T, H]
  int G, KT;          // heads per group, keys per dq tile
};

template <typename T>
__device__ __forceinline__ float ld(const void* base, int64_t i) {
  return to_f32<T>(static_cast<const T*>(base)[i]);
}

// Entry s of idx row `row` is a selected block when 0 <= b <= bq and b is
// larger than the raw entry before it (the forward kernels' rule).
__device__ __forceinline__ bool entry_used(const int32_t* row, int s, int bq, int& b) {
  b = __ldg(row + s);
  return b >= 0 && b <= bq && (s == 0 || b > __ldg(row + s - 1));
}

// Is block b among the selected blocks of query t (doc-local bq)?
__device__ __forceinline__ bool selects(const int32_t* row, int topk, int bq, int b) {
  for (int s = 0; s < topk; ++s) {
    int e;
    if (entry_used(row, s, bq, e) && e == b) return true;
  }
  return false;
}

// ---------------------------------------------------------------- delta
template <typename T>
__global__ void __launch_bounds__(kThreads) bwd_delta_kernel(const BwdParams a) {
  const int warp = (blockIdx.x * kThreads + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  const int H = a.p.num_heads, dv = a.p.dv;
  if (warp >= a.p.total_tokens * H) return;
  const int t = warp / H, h = warp - t * H;
  const int64_t base = ((int64_t)t * H + h) * dv;
  float acc = 0.f;
  for (int e = lane; e < dv; e += 32) acc += ld<T>(a.dout, base + e) * ld<T>(a.out, base + e);
  acc = warp_sum(acc);
  if (lane == 0) {
    a.delta[(int64_t)t * H + h] = acc;
    a.dsink_part[(int64_t)t * H + h] =
        a.sink ? -expf(__ldg(a.sink + h) - __ldg(a.lse + (int64_t)t * H + h)) * acc : 0.f;
  }
}

// ---------------------------------------------------------------- dsink
__global__ void __launch_bounds__(kThreads) bwd_dsink_kernel(const BwdParams a) {
  __shared__ float red[kThreads];
  const int h = blockIdx.x, H = a.p.num_heads;
  float acc = 0.f;
  for (int t = threadIdx.x; t < a.p.total_tokens; t += kThreads)
    acc += a.dsink_part[(int64_t)t * H + h];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int o = kThreads / 2; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) a.dsink[h] = red[0];
}

// ---------------------------------------------------------------- dq
// Shared memory (floats): q group [G][dk|1], dout group [G][dv|1], K tile
// [KT][dk|1], V tile [KT][dv|1], dq group [G][dk], s/p [G][KT], dp/ds [G][KT],
// lse and delta [G]; then the token's selected blocks (ints, sparse).  Odd
// row strides keep the dot-product phase free of bank conflicts.
__host__ __device__ inline size_t dq_smem_floats(int G, int KT, int dk, int dv) {
  const int dkp = dk | 1, dvp = dv | 1;
  return (size_t)G * dkp + (size_t)G * dvp + (size_t)KT * dkp + (size_t)KT * dvp +
         (size_t)G * dk + 2 * (size_t)G * KT + 2 * (size_t)G;
}

template <typename T, bool kSparse>
__global__ void __launch_bounds__(kThreads) bwd_dq_kernel(const BwdParams a) {
  extern __shared__ float sm[];
  __shared__ int nblk;
  const Problem& P = a.p;
  const int G = a.G, KT = a.KT, H = P.num_heads, dk = P.dk, dv = P.dv, tid = threadIdx.x;
  const int dkp = dk | 1, dvp = dv | 1;
  float* qs = sm;
  float* dos = qs + G * dkp;
  float* ks = dos + G * dvp;
  float* vs = ks + KT * dkp;
  float* dqs = vs + KT * dvp;
  float* sp = dqs + G * dk;
  float* dsp = sp + G * KT;
  float* lse_s = dsp + G * KT;
  float* del_s = lse_s + G;
  int* blist = reinterpret_cast<int*>(del_s + G);
  const float scale = P.scale;
  for (int t = blockIdx.x; t < P.total_tokens; t += gridDim.x) {
    int bos, eos;
    if (!find_doc(P.cu_seqlens, P.num_docs, P.total_tokens, P.max_seqlen, t, bos, eos,
                  P.status))
      continue;
    if (kSparse) {
      if (tid == 0) {
        const int bq = (t - bos) / a.B;
        const int32_t* row = a.idx + (int64_t)t * a.topk;
        int n = 0;
        bool bad = false;
        for (int s = 0; s < a.topk; ++s) {
          int b;
          if (entry_used(row, s, bq, b)) blist[n++] = b;
          else if (b >= 0) bad = true;
        }
        if (bad) record_status(P.status, HS_ERR_INVALID_INDEX);
        nblk = n;
      }
      __syncthreads();
    }
    const int nseg = kSparse ? nblk : 1;
    for (int g0 = 0; g0 < H; g0 += G) {
      const int gn = min(G, H - g0);
      for (int e = tid; e < gn * dk; e += kThreads) {
        const int g = e / dk, d = e - g * dk;
        qs[g * dkp + d] = ld<T>(P.q, (int64_t)t * P.q_row_stride + (int64_t)(g0 + g) * P.q_head_stride + d);
        dqs[e] = 0.f;
      }
      for (int e = tid; e < gn * dv; e += kThreads) {
        const int g = e / dv, d = e - g * dv;
        dos[g * dvp + d] = ld<T>(a.dout, ((int64_t)t * H + g0 + g) * dv + d);
      }
      if (tid < gn) {
        lse_s[tid] = a.lse[(int64_t)t * H + g0 + tid];
        del_s[tid] = a.delta[(int64_t)t * H + g0 + tid];
      }
      __syncthreads();
      for (int sg = 0; sg < nseg; ++sg) {
        int lo, hi;
        if (kSparse) {
          lo = bos + blist[sg] * a.B;
          hi = min(min(lo + a.B, eos), t + 1);
        } else {
          lo = max(bos, t - a.window + 1);
          hi = t + 1;
        }
        for (int j0 = lo; j0 < hi; j0 += KT) {
          const int n = min(KT, hi - j0);
          for (int e = tid; e < n * dk; e += kThreads) {
            const int jj = e / dk, d = e - jj * dk;
            ks[jj * dkp + d] = ld<T>(P.k, (int64_t)(j0 + jj) * P.k_row_stride + d);
          }
          for (int e = tid; e < n * dv; e += kThreads) {
            const int jj = e / dv, d = e - jj * dv;
            vs[jj * dvp + d] = ld<T>(P.v, (int64_t)(j0 + jj) * P.v_row_stride + d);
          }
          __syncthreads();
          for (int i = tid; i < 2 * gn * KT; i += kThreads) {
            const bool isdp = i >= gn * KT;
            const int ii = isdp ? i - gn * KT : i, g = ii / KT, jj = ii - g * KT;
            float acc = 0.f;
            if (jj < n) {
              if (!isdp) {
                for (int d = 0; d < dk; ++d) acc += qs[g * dkp + d] * ks[jj * dkp + d];
              } else {
                for (int d = 0; d < dv; ++d) acc += dos[g * dvp + d] * vs[jj * dvp + d];
              }
            }
            (isdp ? dsp : sp)[ii] = acc;
          }
          __syncthreads();
          for (int i = tid; i < gn * KT; i += kThreads) {
            const int g = i / KT, jj = i - g * KT;
            const float pr = jj < n ? expf(sp[i] * scale - lse_s[g]) : 0.f;
            dsp[i] = pr * (dsp[i] - del_s[g]);
          }
          __syncthreads();
          for (int e = tid; e < gn * dk; e += kThreads) {
            const int g = e / dk, d = e - g * dk;
            float acc = 0.f;
            for (int jj = 0; jj < n; ++jj) acc += dsp[g * KT + jj] * ks[jj * dkp + d];
            dqs[e] += scale * acc;
          }
          __syncthreads();
        }
      }
      for (int e = tid; e < gn * dk; e += kThreads) {
        const int g = e / dk, d = e - g * dk;
        a.dq[((int64_t)t * H + g0 + g) * dk + d] = dqs[e];
      }
      __syncthreads();
    }
  }
}

// ---------------------------------------------------------------- dk, dv
// Shared memory (floats): K tile [KT][dk|1], V tile [KT][dv|1], q group
// [G][dk|1], dout group [G][dv|1], dk accumulators [KT][dk], dv accumulators
// [KT][dv], p [G][KT], ds [G][KT], lse and delta [G]; then the member tokens
// of the current candidate chunk and their key masks (ints).
__host__ __device__ inline size_t dkdv_smem_floats(int G, int KT, int dk, int dv) {
  const int dkp = dk | 1, dvp = dv | 1;
  return (size_t)KT * dkp + (size_t)KT * dvp + (size_t)G * dkp + (size_t)G * dvp +
         (size_t)KT * dk + (size_t)KT * dv + 2 * (size_t)G * KT + 2 * (size_t)G;
}

template <typename T, bool kSparse>
__global__ void __launch_bounds__(kThreads) bwd_dkdv_kernel(const BwdParams a, int KT) {
  extern __shared__ float sm[];
  __shared__ int wcount[kThreads / 32];
  const Problem& P = a.p;
  const int G = a.G, H = P.num_heads, dk = P.dk, dv = P.dv, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int dkp = dk | 1, dvp = dv | 1;
  float* ks = sm;
  float* vs = ks + KT * dkp;
  float* qs = vs + KT * dvp;
  float* dos = qs + G * dkp;
  float* dks = dos + G * dvp;
  float* dvs = dks + KT * dk;
  float* sp = dvs + KT * dv;
  float* dsp = sp + G * KT;
  float* lse_s = dsp + G * KT;
  float* del_s = lse_s + G;
  int* mem = reinterpret_cast<int*>(del_s + G);  // [kThreads] member tokens
  int* memmask = mem + kThreads;                 // [kThreads] their key masks
  const float scale = P.scale;
  const int NT = P.total_tokens;
  for (int tile = blockIdx.x; tile * KT < NT; tile += gridDim.x) {
    const int j1 = min(NT, tile * KT + KT);
    // the tile's keys, one document segment [s0, s1) at a time
    for (int s0 = tile * KT; s0 < j1;) {
      int bos, eos;
      if (!find_doc(P.cu_seqlens, P.num_docs, NT, P.max_seqlen, s0, bos, eos, P.status)) break;
      const int s1 = min(j1, eos), n = s1 - s0;
      for (int e = tid; e < n * dk; e += kThreads) {
        const int jj = e / dk, d = e - jj * dk;
        ks[jj * dkp + d] = ld<T>(P.k, (int64_t)(s0 + jj) * P.k_row_stride + d);
        dks[e] = 0.f;
      }
      for (int e = tid; e < n * dv; e += kThreads) {
        const int jj = e / dv, d = e - jj * dv;
        vs[jj * dvp + d] = ld<T>(P.v, (int64_t)(s0 + jj) * P.v_row_stride + d);
        dvs[e] = 0.f;
      }
      // candidate queries t (those whose key set can meet [s0, s1)), in
      // chunks of kThreads: thread i tests t = c0 + i
      const int tend = kSparse ? eos : min(eos, s1 - 1 + a.window);
      const int ba = kSparse ? (s0 - bos) / a.B : 0, bb = kSparse ? (s1 - 1 - bos) / a.B : 0;
      for (int c0 = s0; c0 < tend; c0 += kThreads) {
        const int t = c0 + tid;
        uint32_t mask = 0;
        if (t < tend) {
          if (kSparse) {
            const int bq = (t - bos) / a.B;
            const int32_t* row = a.idx + (int64_t)t * a.topk;
            const bool fa = selects(row, a.topk, bq, ba);
            const bool fb = bb == ba ? fa : selects(row, a.topk, bq, bb);
            for (int jj = 0; jj < n; ++jj) {
              const int j = s0 + jj;
              if (j <= t && ((j - bos) / a.B == ba ? fa : fb)) mask |= 1u << jj;
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
        for (int mi = 0; mi < nm; ++mi) {
          const int tt = mem[mi];
          const uint32_t mk = (uint32_t)memmask[mi];
          for (int g0 = 0; g0 < H; g0 += G) {
            const int gn = min(G, H - g0);
            for (int e = tid; e < gn * dk; e += kThreads) {
              const int g = e / dk, d = e - g * dk;
              qs[g * dkp + d] = ld<T>(P.q, (int64_t)tt * P.q_row_stride +
                                              (int64_t)(g0 + g) * P.q_head_stride + d);
            }
            for (int e = tid; e < gn * dv; e += kThreads) {
              const int g = e / dv, d = e - g * dv;
              dos[g * dvp + d] = ld<T>(a.dout, ((int64_t)tt * H + g0 + g) * dv + d);
            }
            if (tid < gn) {
              lse_s[tid] = a.lse[(int64_t)tt * H + g0 + tid];
              del_s[tid] = a.delta[(int64_t)tt * H + g0 + tid];
            }
            __syncthreads();
            for (int i = tid; i < 2 * gn * KT; i += kThreads) {
              const bool isdp = i >= gn * KT;
              const int ii = isdp ? i - gn * KT : i, g = ii / KT, jj = ii - g * KT;
              float acc = 0.f;
              if (jj < n && ((mk >> jj) & 1u)) {
                if (!isdp) {
                  for (int d = 0; d < dk; ++d) acc += qs[g * dkp + d] * ks[jj * dkp + d];
                } else {
                  for (int d = 0; d < dv; ++d) acc += dos[g * dvp + d] * vs[jj * dvp + d];
                }
              }
              (isdp ? dsp : sp)[ii] = acc;
            }
            __syncthreads();
            for (int i = tid; i < gn * KT; i += kThreads) {
              const int g = i / KT, jj = i - g * KT;
              const bool member = jj < n && ((mk >> jj) & 1u);
              const float pr = member ? expf(sp[i] * scale - lse_s[g]) : 0.f;
              dsp[i] = pr * (dsp[i] - del_s[g]);
              sp[i] = pr;
            }
            __syncthreads();
            for (int e = tid; e < n * dk; e += kThreads) {
              const int jj = e / dk, d = e - jj * dk;
              float acc = 0.f;
              for (int g = 0; g < gn; ++g) acc += dsp[g * KT + jj] * qs[g * dkp + d];
              dks[e] += scale * acc;
            }
            for (int e = tid; e < n * dv; e += kThreads) {
              const int jj = e / dv, d = e - jj * dv;
              float acc = 0.f;
              for (int g = 0; g < gn; ++g) acc += sp[g * KT + jj] * dos[g * dvp + d];
              dvs[e] += acc;
            }
            __syncthreads();
          }
        }
      }
      for (int e = tid; e < n * dk; e += kThreads) {
        const int jj = e / dk, d = e - jj * dk;
        a.dkey[(int64_t)(s0 + jj) * dk + d] = dks[e];
      }
      for (int e = tid; e < n * dv; e += kThreads) {
        const int jj = e / dv, d = e - jj * dv;
        a.dval[(int64_t)(s0 + jj) * dv + d] = dvs[e];
      }
      __syncthreads();
      s0 = s1;
    }
  }
}

constexpr size_t kMaxSmem = 227 * 1024;

template <typename T, bool kSparse>
cudaError_t launch_typed(BwdParams a, bool cuda_core_passes, cudaStream_t s) {
  const Problem& P = a.p;
  const int NT = P.total_tokens, H = P.num_heads;
  const int pairs = NT * H;
  bwd_delta_kernel<T><<<(pairs + kThreads / 32 - 1) / (kThreads / 32), kThreads, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.dsink && a.sink) {
    bwd_dsink_kernel<<<H, kThreads, 0, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // dq: the largest head group (and key tile) whose staging fits (unless the
  // caller runs the tensor-core passes instead)
  if (cuda_core_passes) {
    int G = 16, KT = 16;
    const size_t ints = 256 * sizeof(int);
    while (G > 1 && dq_smem_floats(G, KT, P.dk, P.dv) * 4 + ints > kMaxSmem) G >>= 1;
    while (KT > 1 && dq_smem_floats(G, KT, P.dk, P.dv) * 4 + ints > kMaxSmem) KT >>= 1;
    const size_t bytes = dq_smem_floats(G, KT, P.dk, P.dv) * 4 + ints;
    if (bytes > kMaxSmem) return cudaErrorInvalidConfiguration;
    a.G = G;
    a.KT = KT;
    auto kern = bwd_dq_kernel<T, kSparse>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    kern<<<NT, kThreads, bytes, s>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // dk, dv: key tiles of at most kKeyTile keys (unless the caller runs the
  // tensor-core key-major pass instead)
  if (cuda_core_passes) {
    int G = 16, KT = kKeyTile;
    const size_t ints = 2 * kThreads * sizeof(int);
    while (KT > 4 && dkdv_smem_floats(G, KT, P.dk, P.dv) * 4 + ints > kMaxSmem) KT >>= 1;
    while (G > 1 && dkdv_smem_floats(G, KT, P.dk, P.dv) * 4 + ints > kMaxSmem) G >>= 1;
    const size_t bytes = dkdv_smem_floats(G, KT, P.dk, P.dv) * 4 + ints;
    if (bytes > kMaxSmem) return cudaErrorInvalidConfiguration;
    a.G = G;
    auto kern = bwd_dkdv_kernel<T, kSparse>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    kern<<<(NT + KT - 1) / KT, kThreads, bytes, s>>>(a, KT);
    e = cudaGetLastError();
  }
  return e;
}

}  // namespace

size_t simt_backward_workspace(int total_tokens, int num_heads) {
  return (size_t)2 * total_tokens * num_heads * sizeof(float);
}

cudaError_t launch_simt_backward(const BwdArgs& b, bool sparse, bool allow_mma, int* path,
                                 cudaStream_t s) {
  BwdParams a{};
  a.p = b.p;
  a.idx = b.idx;
  a.topk = b.topk;
  a.B = b.block_size;
  a.window = b.window;
  a.sink = b.sink;
  a.out = b.out;
  a.lse = b.lse;
  a.dout = b.dout;
  a.dq = b.dq;
  a.dkey = b.dkey;
  a.dval = b.dval;
  a.dsink = b.dsink;
  a.delta = static_cast<float*>(b.workspace);
  a.dsink_part = a.delta + (size_t)b.p.total_tokens * b.p.num_heads;
  if (b.p.dtype == HS_BF16) {
    // tensor cores: dq and dk / dv on tcgen05 (else every pass on CUDA cores)
    const bool mma = allow_mma && tc_bwd_dq_supported(b.p) && tc_bwd_dkdv_supported(b.p) &&
                     (reinterpret_cast<uintptr_t>(b.dout) & 15) == 0 && b.dkdv_ws != nullptr;
    if (path) *path = mma ? HS_PATH_MMA : HS_PATH_SIMT;
    cudaError_t e = sparse ? launch_typed<__nv_bfloat16, true>(a, !mma, s)
                           : launch_typed<__nv_bfloat16, false>(a, !mma, s);
    if (e != cudaSuccess || !mma) return e;
    e = launch_tc_bwd_dq(b, sparse, a.delta, 0, s);
    if (e != cudaSuccess) return e;
    return launch_tc_bwd_dkdv(b, sparse, a.delta, 0, s);
  }
  if (path) *path = HS_PATH_SIMT;
  return sparse ? launch_typed<float, true>(a, true, s) : launch_typed<float, false>(a, true, s);
}

}  // namespace hs
