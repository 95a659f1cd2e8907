// bra_route_noalloc: region-level routing whose scratch (the fp32 region
// means Q^r and K^r) lives in a fixed array inside this library instead of
// in a caller-supplied workspace, for callers that cannot allocate device
// memory themselves.  It runs the same pool and route kernels as bra_route.
//
// Set-up: every call looks up the current device's address of the array
// with cudaGetSymbolAddress (which allocates nothing; the device must be
// current, which it is for the caller's stream), so the address is never
// stale, even after a device reset has reloaded the library's module.  The
// first call on a device may load the module, so it should come before any
// stream capture.  The array's name in host code is only a host-side handle,
// never a device address, so kernels are always given the looked-up pointer.
//
// Every call on a device shares the one array and leaves the last call's
// means in it; nothing in it needs to start at zero (the pool kernel writes
// every mean the route kernel reads).  Calls that overlap on the GPU (two
// streams, or two host threads) race on the array.
#include <cuda_runtime.h>

#include "../../include/bra.h"
#include "common.cuh"
#include "kernels.h"

namespace bra {
namespace {

// Q^r and K^r, each up to kNoAllocMeans floats (B * heads * S*S * d).
constexpr size_t kNoAllocMeans = BRA_NOALLOC_MAX_MEANS;
static __device__ __align__(256) float g_route_scratch[2 * kNoAllocMeans];

// Device address of g_route_scratch on the current device, or nullptr.
float* scratch_for_current_device() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess) return nullptr;
    return static_cast<float*>(p);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace bra

extern "C" bra_status bra_route_noalloc(const bra_shape* shape, const void* q, const void* k,
                                        int32_t* idx, void* stream) {
    using namespace bra;
    // Same size rules as bra_route (bra_workspace_bytes is 0 for a bad shape).
    if (!shape) return BRA_ERR_INVALID_ARG;
    const size_t ws = bra_workspace_bytes(shape);
    if (ws == 0) {
        bra_shape probe = *shape;  // tell "invalid" from "unsupported" the way bra_route does
        return bra_route(&probe, q, k, idx, nullptr, stream);
    }
    if (!q || !k || !idx || !aligned16(q) || !aligned16(k) || !aligned16(idx))
        return BRA_ERR_INVALID_ARG;
    Geometry g;
    g.B = shape->B; g.H = shape->H; g.W = shape->W; g.C = shape->C; g.heads = shape->heads;
    g.S = shape->S; g.topk = shape->topk;
    g.d = g.C / g.heads; g.R = g.S * g.S; g.hs = g.H / g.S; g.ws = g.W / g.S; g.n = g.hs * g.ws;
    const size_t means = (size_t)g.B * g.heads * g.R * g.d;
    if (means > kNoAllocMeans) return BRA_ERR_UNSUPPORTED;
    if (g.B == 0) return BRA_OK;
    float* scratch = scratch_for_current_device();
    if (!scratch) return BRA_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const bool bf16 = shape->dtype == BRA_DTYPE_BF16;
    if (launch_pool(bf16, q, k, scratch, scratch + kNoAllocMeans, g, st) != cudaSuccess)
        return BRA_ERR_CUDA;
    if (launch_route(scratch, scratch + kNoAllocMeans, idx, g, st) != cudaSuccess)
        return BRA_ERR_CUDA;
    return BRA_OK;
}
