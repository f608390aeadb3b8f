// CUDA-core kernels for block scoring and for sparse / sliding-window MQA
// attention.  They serve fp32 inputs (where bf16 tensor-core arithmetic would
// not meet the accuracy bound) and shapes the tcgen05 kernels do not cover.
// Arithmetic is fp32 throughout.
//
// Definitions: "HySparse MQA sparse attention (FA4 block scoring + SWA MQA +
// block-sparse DSA gather)", PaddleFleet pull request 1470, "Core" list and
// per-file table; the sink is a softmax-denominator offset as in "Support
// attn sink in fa3", pull request 1415.

#include <math.h>

#include "hs_device.cuh"
#include "hs_internal.h"

namespace hs {

namespace {

constexpr int kScoreThreads = 256;
constexpr int kScoreChunk = 2048;  // keys per pass; a multiple of every block size
constexpr int kAttnThreads = 128;
constexpr int kMaxDvPerThread = 8;  // dv <= 1024

template <typename T>
__device__ __forceinline__ float dot_row(const float* __restrict__ qs, const T* __restrict__ kr,
                                         int dk) {
  float acc = 0.f;
  for (int d = 0; d < dk; ++d) acc = fmaf(qs[d], to_f32<T>(kr[d]), acc);
  return acc;
}

// One CTA per query token.  For every head in turn: logits of all causal
// keys (in chunks), per-block log-sum-exp, the row LSE as the log-sum-exp of
// the block values, then the head's block masses are added to the token's
// score accumulators (heads in increasing order).
template <typename T>
__global__ void __launch_bounds__(kScoreThreads)
simt_block_score_kernel(ScoreArgs a) {
  extern __shared__ float smem[];
  const Problem& p = a.p;
  const int t = blockIdx.x;
  if (t >= p.total_tokens) return;
  int bos, eos;
  if (!find_doc(p.cu_seqlens, p.num_docs, p.total_tokens, p.max_seqlen, t, bos, eos, p.status))
    return;
  const int H = p.num_heads, Dk = p.dk, B = a.block_size, nbmax = a.nbmax;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = kScoreThreads / 32;
  float* qs = smem;                // [H * Dk]
  float* sbuf = qs + H * Dk;       // [kScoreChunk]
  float* blse = sbuf + kScoreChunk;  // [nbmax]
  float* acc = blse + nbmax;       // [nbmax]
  float* red = acc + nbmax;        // [32]

  const T* qt = reinterpret_cast<const T*>(p.q) + (int64_t)t * p.q_row_stride;
  for (int i = tid; i < H * Dk; i += kScoreThreads) {
    int h = i / Dk, d = i - h * Dk;
    qs[i] = to_f32<T>(qt[(int64_t)h * p.q_head_stride + d]);
  }
  const int n = t - bos + 1;
  const int nb = (n + B - 1) / B;
  for (int b = tid; b < nbmax; b += kScoreThreads) acc[b] = 0.f;
  __syncthreads();

  const T* kb = reinterpret_cast<const T*>(p.k);
  for (int h = 0; h < H; ++h) {
    const float* qh = qs + h * Dk;
    for (int c0 = 0; c0 < n; c0 += kScoreChunk) {
      const int cn = min(kScoreChunk, n - c0);
      for (int i = tid; i < cn; i += kScoreThreads)
        sbuf[i] = p.scale * dot_row<T>(qh, kb + (int64_t)(bos + c0 + i) * p.k_row_stride, Dk);
      __syncthreads();
      const int nbc = (cn + B - 1) / B;
      for (int bb = warp; bb < nbc; bb += nwarps) {
        const int lo = bb * B, hi = min(lo + B, cn);
        float m = -INFINITY;
        for (int i = lo + lane; i < hi; i += 32) m = fmaxf(m, sbuf[i]);
        m = warp_max(m);
        float s = 0.f;
        for (int i = lo + lane; i < hi; i += 32) s += expf(sbuf[i] - m);
        s = warp_sum(s);
        if (lane == 0) blse[c0 / B + bb] = m + logf(s);
      }
      __syncthreads();
    }
    if (warp == 0) {
      float m = -INFINITY;
      for (int b = lane; b < nb; b += 32) m = fmaxf(m, blse[b]);
      m = warp_max(m);
      float s = 0.f;
      for (int b = lane; b < nb; b += 32) s += expf(blse[b] - m);
      s = warp_sum(s);
      if (lane == 0) {
        const float L = m + logf(s);
        red[0] = L;
        a.lse[(int64_t)t * H + h] = L;
      }
    }
    __syncthreads();
    const float L = red[0];
    float* bl = a.block_lse ? a.block_lse + ((int64_t)t * H + h) * a.nb_stride : nullptr;
    for (int b = tid; b < nbmax; b += kScoreThreads) {
      if (b < nb) {
        acc[b] += expf(blse[b] - L);
        if (bl) bl[b] = blse[b];
      } else if (bl) {
        bl[b] = -INFINITY;
      }
    }
    __syncthreads();
  }
  float* bs = a.block_score + (int64_t)t * a.nb_stride;
  for (int b = tid; b < nbmax; b += kScoreThreads) bs[b] = (b < nb) ? acc[b] : 0.f;
}

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_max(v);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < kAttnThreads / 32; ++w) r = fmaxf(r, red[w]);
  __syncthreads();
  return r;
}

__device__ __forceinline__ float block_reduce_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
  for (int w = 1; w < kAttnThreads / 32; ++w) r += red[w];
  __syncthreads();
  return r;
}

// One CTA per (query token, head).  Keys come in segments of at most 128
// (one selected block, or one slice of the window); an online softmax keeps
// the running max m, the running denominator l and the output accumulators
// (thread i owns value columns i, i + 128, ...).  The sink joins at the end.
template <typename T, bool kSparse>
__global__ void __launch_bounds__(kAttnThreads)
simt_attention_kernel(AttnArgs a) {
  extern __shared__ float smem[];
  const Problem& p = a.p;
  const int t = blockIdx.x, h = blockIdx.y;
  if (t >= p.total_tokens || h >= p.num_heads) return;
  int bos, eos;
  if (!find_doc(p.cu_seqlens, p.num_docs, p.total_tokens, p.max_seqlen, t, bos, eos, p.status))
    return;
  const int Dk = p.dk, Dv = p.dv, tid = threadIdx.x;
  float* qs = smem;          // [Dk]
  float* pbuf = qs + Dk;     // [128]
  float* red = pbuf + 128;   // [32]
  const T* qh = reinterpret_cast<const T*>(p.q) + (int64_t)t * p.q_row_stride +
                (int64_t)h * p.q_head_stride;
  for (int d = tid; d < Dk; d += kAttnThreads) qs[d] = to_f32<T>(qh[d]);
  __syncthreads();

  const T* kb = reinterpret_cast<const T*>(p.k);
  const T* vb = reinterpret_cast<const T*>(p.v);
  float acc[kMaxDvPerThread];
#pragma unroll
  for (int r = 0; r < kMaxDvPerThread; ++r) acc[r] = 0.f;
  float m = -INFINITY, l = 0.f;

  int nseg, wlo = 0;
  if (kSparse) {
    nseg = a.topk;
  } else {
    wlo = max(bos, t - a.window + 1);
    nseg = (t + 1 - wlo + 127) / 128;
  }
  const int bq = (t - bos) / a.block_size;
  for (int sgi = 0; sgi < nseg; ++sgi) {
    int lo, hi;
    if (kSparse) {
      // a block id must lie in [0, bq] and exceed the entry before it
      const int32_t* row = a.idx + (int64_t)t * a.topk;
      const int b = __ldg(row + sgi);
      if (b < 0) continue;
      if (b > bq || (sgi > 0 && b <= __ldg(row + sgi - 1))) {
        if (tid == 0) record_status(p.status, HS_ERR_INVALID_INDEX);
        continue;
      }
      lo = bos + b * a.block_size;
      hi = min(lo + a.block_size, t + 1);
    } else {
      lo = wlo + sgi * 128;
      hi = min(lo + 128, t + 1);
    }
    const int cnt = hi - lo;
    float s = -INFINITY;
    if (tid < cnt) s = p.scale * dot_row<T>(qs, kb + (int64_t)(lo + tid) * p.k_row_stride, Dk);
    const float bmax = block_reduce_max(s, red);
    const float mn = fmaxf(m, bmax);
    const float alpha = expf(m - mn);  // 0 on the first segment
    const float pv = (tid < cnt) ? expf(s - mn) : 0.f;
    pbuf[tid] = pv;
    const float psum = block_reduce_sum(pv, red);  // also orders the pbuf writes
    l = l * alpha + psum;
#pragma unroll
    for (int r = 0; r < kMaxDvPerThread; ++r) {
      const int d = tid + r * kAttnThreads;
      if (d < Dv) {
        float x = acc[r] * alpha;
        for (int i = 0; i < cnt; ++i)
          x = fmaf(pbuf[i], to_f32<T>(vb[(int64_t)(lo + i) * p.v_row_stride + d]), x);
        acc[r] = x;
      }
    }
    m = mn;
    __syncthreads();
  }

  const float sk = a.sink ? __ldg(a.sink + h) : -INFINITY;
  const float M = fmaxf(m, sk);
  float lse, inv;
  if (M == -INFINITY) {  // no key and no sink: empty softmax
    lse = -INFINITY;
    inv = 0.f;
  } else {
    const float em = expf(m - M);
    const float denom = l * em + expf(sk - M);
    lse = M + logf(denom);
    inv = em / denom;
  }
  T* o = reinterpret_cast<T*>(a.out) + ((int64_t)t * p.num_heads + h) * Dv;
  const int64_t th = (int64_t)t * p.num_heads + h;
  const float gown = a.gate_own ? __ldg(a.gate_own + th) : 1.f;
  const float gprev = a.gate_prev ? __ldg(a.gate_prev + th) : 1.f;
  const T* pr = a.prev ? reinterpret_cast<const T*>(a.prev) + th * Dv : nullptr;
#pragma unroll
  for (int r = 0; r < kMaxDvPerThread; ++r) {
    const int d = tid + r * kAttnThreads;
    if (d < Dv) {
      float x = acc[r] * inv * gown;
      if (pr) x = fmaf(gprev, to_f32<T>(pr[d]), x);  // read before the write below
      o[d] = from_f32<T>(x);
    }
  }
  if (tid == 0) a.lse[(int64_t)t * p.num_heads + h] = lse;
}

}  // namespace

size_t simt_block_score_smem(int num_heads, int dk, int nbmax) {
  return sizeof(float) * ((size_t)num_heads * dk + kScoreChunk + 2 * (size_t)nbmax + 32);
}

cudaError_t launch_simt_block_score(const ScoreArgs& a, cudaStream_t s) {
  const size_t smem = simt_block_score_smem(a.p.num_heads, a.p.dk, a.nbmax);
  if (a.p.dtype == HS_BF16) {
    auto kern = simt_block_score_kernel<__nv_bfloat16>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<a.p.total_tokens, kScoreThreads, smem, s>>>(a);
  } else {
    auto kern = simt_block_score_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<a.p.total_tokens, kScoreThreads, smem, s>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_simt_attention(const AttnArgs& a, bool sparse, cudaStream_t s) {
  if (a.p.dv > kAttnThreads * kMaxDvPerThread) return cudaErrorInvalidValue;
  const size_t smem = sizeof(float) * ((size_t)a.p.dk + 128 + 32);
  dim3 grid(a.p.total_tokens, a.p.num_heads);
  if (a.p.dtype == HS_BF16) {
    if (sparse) simt_attention_kernel<__nv_bfloat16, true><<<grid, kAttnThreads, smem, s>>>(a);
    else simt_attention_kernel<__nv_bfloat16, false><<<grid, kAttnThreads, smem, s>>>(a);
  } else {
    if (sparse) simt_attention_kernel<float, true><<<grid, kAttnThreads, smem, s>>>(a);
    else simt_attention_kernel<float, false><<<grid, kAttnThreads, smem, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace hs
