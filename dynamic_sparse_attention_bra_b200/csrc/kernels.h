// Kernel entry points and launch constants of the BRA library (internal).
#pragma once

#include "common.cuh"

namespace bra {

constexpr int kPoolThreads = 128;
constexpr int kPoolWarpThreads = 128;  // 4 regions per CTA in the warp form
constexpr int kRouteThreads = 256;
constexpr int kMaxRegions = 256;   // S * S limit: 8 affinity columns per lane
constexpr int kSimtThreads = 128;
constexpr int kSimtKeyBlock = 64;  // keys staged in shared memory per step

// Host-side launchers (each defined next to its kernel).  All launch on
// ``stream`` and return cudaGetLastError() of the launch.
cudaError_t launch_pool(bool bf16, const void* q, const void* k, float* qr, float* kr,
                        const Geometry& g, cudaStream_t stream);
cudaError_t launch_route(const float* qr, const float* kr, int32_t* idx, const Geometry& g,
                         cudaStream_t stream);
// Bounded-wait self-test: waits on an mbarrier nobody arrives at (unless
// ``arrive``) for at most ``tries`` polls, then records kDevTimeout.
cudaError_t launch_bounded_wait_selftest(int* status, uint32_t tries, bool arrive, cudaStream_t stream);
// Local context enhancement: o += bias + 5x5 depthwise filter of v.
cudaError_t launch_lce(bool bf16, const void* v, const float* w, const float* bias, void* o, const Geometry& g,
                       cudaStream_t stream);

// SIMT token attention, any dtype, head dim 32.
struct SimtPlan {
    int chunk;      // queries per CTA (<= kSimtThreads)
    int group;      // threads per query (power of two, <= 32)
    int chunks;     // CTAs per region
};
SimtPlan simt_plan(const Geometry& g);
cudaError_t launch_attend_simt(bool bf16, const void* q, const void* k, const void* v,
                               const int32_t* idx, void* o, const Geometry& g, int* status,
                               cudaStream_t stream);

}  // namespace bra
