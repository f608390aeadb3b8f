// hs_block_score_static: block scoring for callers that cannot allocate.
//
// hs_block_score needs a device workspace from its caller.  Some callers
// cannot provide one: code that runs where no allocator may be called (for
// example inside a framework's custom-op kernel launch path that forbids
// cudaMalloc, a real-time loop that must not hit the allocator or its
// synchronisation, or a process whose memory pool is fixed up front).  This
// entry point gives them the same computation with the scratch taken from a
// fixed array that lives in the library's own device memory.
//
// The array is a file-scope __device__ variable, so every GPU on which the
// library is loaded holds it (kStaticScratchBytes) until the process exits.
// Host code cannot use the array's name as a device address; the address is
// looked up once per device with cudaGetSymbolAddress, on the first call made
// while that device is current, and kept for the life of the process (so
// the library must not be used across a cudaDeviceReset, after which the
// module is reloaded and the kept address would be stale).  Nothing is
// allocated, freed or zeroed by a call: the kernel writes every scratch
// value before reading it, so the contents left by a previous call do not
// matter.  All calls share the one
// array, so calls that may run at the same time on the GPU (different
// streams, or different host threads) race on it and must be serialised by
// the caller.

#include <cuda_runtime.h>
#include <stdio.h>

#include <mutex>

#include "hs.h"
#include "hs_internal.h"

namespace {

// 16 MiB: enough for the 4096-token, 64-head, block-64 workload (about 10 MB
// with 148 SMs); larger problems must use hs_block_score with a workspace.
constexpr size_t kStaticScratchBytes = 16u << 20;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices];  // device address of the array, per device
std::mutex g_scratch_mu;

// Device address of the array on the current device (looked up once).
hs_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return hs::report_error(HS_ERR_CUDA, "cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices)
    return hs::report_error(HS_ERR_UNSUPPORTED, "device id out of range for the static scratch");
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char msg[256];
      snprintf(msg, sizeof(msg), "cudaGetSymbolAddress(static scratch): %s",
               cudaGetErrorString(e));
      return hs::report_error(HS_ERR_CUDA, msg);
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return HS_OK;
}

}  // namespace

extern "C" {

hs_status hs_block_score_static(const void* q, int64_t q_row_stride, int64_t q_head_stride,
                                const void* k, int64_t k_row_stride,
                                const int32_t* cu_seqlens, int num_docs, int total_tokens,
                                int max_seqlen, int num_heads, int dk, hs_dtype dtype,
                                float softmax_scale, int block_size, float* lse,
                                float* block_score, int nb_stride, float* block_lse,
                                hs_stream_t stream) {
  // the arguments first (a negative max_seqlen must not reach the sizing),
  // then the size check, all on the host before any device work
  hs_status r = hs::check_score_args(q, q_row_stride, q_head_stride, k, k_row_stride, cu_seqlens,
                                     num_docs, total_tokens, max_seqlen, num_heads, dk, dtype,
                                     softmax_scale, block_size, lse, block_score, nb_stride);
  if (r != HS_OK) return r;
  if (total_tokens == 0) return HS_OK;
  // The limit follows from the shape alone, so it is conservative for a call
  // that pointer alignment or its document count sends to the CUDA-core
  // kernel, which needs no scratch.
  const size_t need = hs_workspace_size(HS_OP_BLOCK_SCORE, total_tokens, num_docs, max_seqlen,
                                        num_heads, dk, 0, dtype, block_size);
  if (need > kStaticScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "problem needs %zu bytes of scratch, the static scratch holds %zu; "
             "use hs_block_score with a workspace",
             need, kStaticScratchBytes);
    return hs::report_error(HS_ERR_WORKSPACE, msg);
  }
  void* scratch = nullptr;
  r = scratch_address(&scratch);
  if (r != HS_OK) return r;
  return hs_block_score(q, q_row_stride, q_head_stride, k, k_row_stride, cu_seqlens, num_docs,
                        total_tokens, max_seqlen, num_heads, dk, dtype, softmax_scale,
                        block_size, lse, block_score, nb_stride, block_lse, scratch,
                        kStaticScratchBytes, stream);
}

}  // extern "C"
