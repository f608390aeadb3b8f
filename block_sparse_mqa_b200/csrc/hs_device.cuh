// Device helpers shared by the libhs kernels: document lookup, status
// recording and element loads.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hs.h"

namespace hs {

// Record a device-detected problem.  The first non-zero status wins; kernels
// never trap, they record and skip the offending work.
__device__ __forceinline__ void record_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Document [bos, eos) that holds token t: the last d with cu[d] <= t.
// Returns false (and records HS_ERR_INVALID_ARG) when cu_seqlens is
// inconsistent with t, total_tokens or max_seqlen.
__device__ __forceinline__ bool find_doc(const int32_t* __restrict__ cu, int num_docs,
                                         int total_tokens, int max_seqlen, int t, int& bos,
                                         int& eos, int* status) {
  int lo = 0, hi = num_docs;  // invariant: answer in [lo, hi)
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (__ldg(cu + mid) <= t) lo = mid; else hi = mid;
  }
  bos = __ldg(cu + lo);
  eos = __ldg(cu + lo + 1);
  bool ok = (bos >= 0) && (bos <= t) && (t < eos) && (eos <= total_tokens) &&
            (eos - bos <= max_seqlen);
  if (!ok) record_status(status, HS_ERR_INVALID_ARG);
  return ok;
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Warp reductions.
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace hs
