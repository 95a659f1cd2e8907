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

}  // namespace bra
