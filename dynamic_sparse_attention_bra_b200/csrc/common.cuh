// Device helpers shared by the BRA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace bra {

// Geometry of one call, derived on the host from bra_shape.
struct Geometry {
    int B, H, W, C, heads, S, topk;
    int d;    // head dim C / heads
    int R;    // S * S regions
    int hs;   // rows per region H / S
    int ws;   // columns per region W / S
    int n;    // tokens per region hs * ws
};

// Status words at the start of the workspace status block.
enum DeviceStatus : int { kDevOk = 0, kDevTimeout = 4, kDevBadRoute = 5, kDevBounds = 6 };

__device__ __forceinline__ void raise_status(int* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// Index checks of a debug build (compiled with -DBRA_DEBUG): an access whose
// last element ``last`` is not below ``count`` elements of its buffer is
// recorded as kDevBounds in the status block and skipped.  A normal build
// compiles the checks away (the function returns true).
__device__ __forceinline__ bool in_bounds(size_t last, size_t count, int* status) {
#ifdef BRA_DEBUG
    if (last >= count) {
        raise_status(status, kDevBounds);
        return false;
    }
#else
    (void)last;
    (void)count;
    (void)status;
#endif
    return true;
}

// Elements of a [B, H, W, C] map.
__host__ __device__ __forceinline__ size_t map_elems(const Geometry& g) {
    return (size_t)g.B * g.H * g.W * g.C;
}

// Element loads/stores widened to fp32.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Unpack one 16-byte vector into fp32 lanes: 4 floats or 8 bf16.
__device__ __forceinline__ void unpack16(const uint4& u, float* out, const float*) {
    out[0] = __uint_as_float(u.x);
    out[1] = __uint_as_float(u.y);
    out[2] = __uint_as_float(u.z);
    out[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ void unpack16(const uint4& u, float* out, const __nv_bfloat16*) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        out[2 * i] = __uint_as_float(w[i] << 16);
        out[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

// Global memory offset (in elements) of token t of region r, channel 0, batch b.
__device__ __forceinline__ size_t token_offset(const Geometry& g, int b, int r, int t) {
    const int ri = r / g.S, rj = r - ri * g.S;
    const int ty = t / g.ws, tx = t - ty * g.ws;
    const size_t y = (size_t)ri * g.hs + ty, x = (size_t)rj * g.ws + tx;
    return (((size_t)b * g.H + y) * g.W + x) * g.C;
}

}  // namespace bra

namespace bra {

// Programmatic dependent launch: a kernel launched with
// launch_after_previous() may start while the previous kernel on the stream
// is finishing; it must call grid_dependency_wait() before touching anything
// the previous kernel writes or reads.  A kernel calls allow_dependents()
// once the kernel after it may begin its own set-up.
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void allow_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_after_previous(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                  cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace bra
