// Host-side creation of TMA tensor maps (cuTensorMapEncodeTiled through the runtime's
// driver entry point, so the library does not link libcuda directly).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {

// bf16 tensor of `rank` dims (dims[0] contiguous), strides in bytes for dims 1..rank-1,
// box in elements, 128-byte swizzle (64-byte when swizzle64), out-of-bounds elements
// read as zero.  Returns false if the driver rejects the description.
bool make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, bool swizzle64 = false);

// uint8 (f32 false) or float32 tensor, otherwise as above; swizzle_bytes 0, 64 or 128.
bool make_tmap_raw(CUtensorMap* map, const void* base, bool f32, int rank,
                   const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                   int swizzle_bytes);

}  // namespace mla
