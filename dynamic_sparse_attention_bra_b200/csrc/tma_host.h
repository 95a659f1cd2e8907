// Host-side creation of TMA tensor maps over a [B, H, W, C] bf16 map, through
// the driver entry point (no link-time dependency on libcuda).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace bra {

// Tensor map whose box is box_c channels (32: one head, 64-byte swizzle in
// shared memory; 64: two heads, 128-byte swizzle) of a box_w x box_h block of
// tokens of one image.  Returns false if the driver entry point is missing or
// the encoder rejects the map.
bool encode_region_map(CUtensorMap* map, const void* base, int B, int H, int W, int C, int box_w,
                       int box_h, int box_c);

// Tensor map over the same map viewed as (channel, x in region, y in region,
// region column, image x region row), whose box is one head's channels of
// every region of one image, landing region-major (region r's tokens in rows
// r * ws * hs ... in their in-region order).
bool encode_region_major_map(CUtensorMap* map, const void* base, int B, int H, int W, int C, int ws, int hs,
                             int S);

// Tensor map whose box is 64 channels (a head pair) of a box_w x box_h block
// of tokens of one image, unswizzled (128-byte token rows in shared memory);
// boxes reaching past the map are zero-filled.
bool encode_halo_map(CUtensorMap* map, const void* base, int B, int H, int W, int C, int box_w, int box_h);

// Number of SMs of the current device (cached per device).
int sm_count();

}  // namespace bra
