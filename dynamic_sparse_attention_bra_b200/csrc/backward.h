// Gradients of the token attention for a fixed routing (internal).
#pragma once

#include "common.cuh"

namespace bra {

// Dynamic shared memory the backward kernel needs for ``g`` (0: too much).
size_t backward_smem_bytes(const Geometry& g);

// dq, dk, dv (fp32 [B, H, W, C]) must be zero; dq is written, dk and dv
// accumulated.  Out-of-range routes record kDevBadRoute in ``status``.
cudaError_t launch_attend_backward(bool bf16, const void* q, const void* k, const void* v, const int32_t* idx,
                                   const void* grad_o, float* dq, float* dk, float* dv, const Geometry& g,
                                   int* status, cudaStream_t stream);

// The tensor-core backward (bf16, d = 32, regions of 16..64 tokens in steps
// of 16, topk * n <= 128 keys, topk <= 8).  dk and dv must be zero; dq is
// written in full (zero for a region with an out-of-range route).
bool backward_mma_covers(const Geometry& g);
cudaError_t launch_attend_backward_mma(const void* q, const void* k, const void* v, const int32_t* idx,
                                       const void* grad_o, float* dq, float* dk, float* dv, const Geometry& g,
                                       int* status, cudaStream_t stream);

}  // namespace bra
