// Host-side creation of TMA tensor maps over a [B, H, W, C] bf16 map, through
// the driver entry point (no link-time dependency on libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace bra {

// Tensor map whose box is one head (32 channels) of a box_w x box_h block of
// tokens of one image, 64-byte swizzled in shared memory.  Returns false if
// the driver entry point is missing or the encoder rejects the map.
bool encode_region_map(CUtensorMap* map, const void* base, int B, int H, int W, int C, int box_w,
                       int box_h);

// Number of SMs of the current device (cached per device).
int sm_count();

}  // namespace bra
