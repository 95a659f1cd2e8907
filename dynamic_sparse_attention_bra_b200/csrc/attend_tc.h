// Tensor-core (tcgen05) token attention for bf16, head dim 32 (internal).
#pragma once

#include <cuda_runtime.h>

#include "../../include/bra.h"
#include "common.cuh"

namespace bra {

// Launches the tcgen05 attention for ``g`` when it covers the shape; returns
// BRA_ERR_UNSUPPORTED (and launches nothing) when it does not.
bra_status attend_tc_launch(const Geometry& g, const void* q, const void* k, const void* v,
                            const int32_t* idx, void* o, int* status, cudaStream_t stream);

// Persistent warp-specialised variant for regions of 16..64 tokens (n % 16
// == 0) whose keys per query region (topk * n) are a multiple of 32 and at
// most 256; BRA_ERR_UNSUPPORTED (nothing launched) otherwise.
bra_status attend_stack_launch(const Geometry& g, const void* q, const void* k, const void* v,
                               const int32_t* idx, void* o, int* status, cudaStream_t stream);

// The same kernel with the local context term (a 5 x 5 depthwise filter of V
// plus bias, fp32) added in its epilogue before O is rounded and stored: 8 x 8
// regions, an even number of heads, C <= 128.
bool attend_stack_lce_covers(const Geometry& g);
bra_status attend_stack_lce_launch(const Geometry& g, const void* q, const void* k, const void* v,
                                   const float* weight, const float* bias, const int32_t* idx, void* o, int* status,
                                   cudaStream_t stream);

// Persistent variant for maps of at most 256 tokens (BiFormer stage 3): each
// (batch, head) slice's Q, K, V in shared memory, S dense over the slice,
// each query's softmax masked to its routed regions' keys.
bool attend_slice_covers(const Geometry& g);
bra_status attend_slice_launch(const Geometry& g, const void* q, const void* k, const void* v,
                               const int32_t* idx, void* o, int* status, cudaStream_t stream);

// Warp-level MMA variant for small regions (n % 16 == 0, topk * n of 32, 64
// or 128, maps of at most 256 x 256) whose (batch, head) K and V slices fit
// twice in an SM's shared memory (BiFormer stage 2): persistent, one CTA per
// SM over an equal share of the items, slices double-buffered, routed rows
// gathered by per-lane operand addresses.
bool attend_warp_covers(const Geometry& g);
bra_status attend_warp_launch(const Geometry& g, const void* q, const void* k, const void* v,
                              const int32_t* idx, void* o, int* status, cudaStream_t stream);

// Persistent flash-style variant for regions of a multiple of 128 tokens
// (the dense-prediction map): 128-query tiles, keys streamed in blocks of 128
// with a running maximum, output accumulated in registers.
bool attend_flash_covers(const Geometry& g);
bra_status attend_flash_launch(const Geometry& g, const void* q, const void* k, const void* v,
                               const int32_t* idx, void* o, int* status, cudaStream_t stream);

}  // namespace bra
