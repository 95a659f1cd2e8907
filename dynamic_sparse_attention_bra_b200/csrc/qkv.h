// Q, K, V projection with the region-mean epilogue (internal).
#pragma once

#include "../../include/bra.h"
#include "common.cuh"

namespace bra {

// BRA_OK when the fused projection covers ``g`` (bf16, C = 64 or 128,
// regions of at most 128 tokens), else BRA_ERR_UNSUPPORTED.  Host only.
bra_status qkv_check(const Geometry& g);

// [q | k | v] = x w^T (+ bias) in bf16 and the fp32 region means of q and k
// ([B, heads, R, 32]).  A device-side wait that gives up records kDevTimeout
// in ``status``.
bra_status qkv_launch(const Geometry& g, const void* x, const void* w, const float* bias, void* q, void* k, void* v,
                      float* qr, float* kr, int* status, cudaStream_t stream);

}  // namespace bra
