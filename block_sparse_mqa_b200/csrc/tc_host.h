// Host helpers of the tensor-core kernels: TMA tensor-map encoding.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hs {
namespace tc {

// Encodes a bf16 tiled tensor map with 128-byte swizzle and zero fill for
// out-of-range elements.  dims/box are innermost first; strides (bytes) are
// given for dimensions 1..rank-1.  Returns false if the driver rejects it.
// swizzle128 = false gives a plain (unswizzled, row-major) box layout in
// shared memory, e.g. for stores of a dense staged tile.
bool encode_bf16_map(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box,
                     bool swizzle128 = true);

// Number of SMs of the current device (cached per device).
int sm_count();

}  // namespace tc
}  // namespace hs
