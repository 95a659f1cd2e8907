// C ABI of the BRA library: argument checks, workspace layout and launches.
// Declarations and the contract of every entry point are in include/bra.h.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <cstring>

#include "../../include/bra.h"
#include "attend_tc.h"
#include "backward.h"
#include "common.cuh"
#include "kernels.h"
#include "qkv.h"

namespace bra {
namespace {

constexpr size_t kStatusBytes = 256;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t elem_bytes(int dtype) { return dtype == BRA_DTYPE_BF16 ? 2 : 4; }

// Checks ``s``; fills ``g``.  BRA_OK, BRA_ERR_INVALID_ARG or BRA_ERR_UNSUPPORTED.
bra_status make_geometry(const bra_shape* s, Geometry* g) {
    if (!s) return BRA_ERR_INVALID_ARG;
    if (s->B < 0 || s->H <= 0 || s->W <= 0 || s->C <= 0 || s->heads <= 0 || s->S <= 0)
        return BRA_ERR_INVALID_ARG;
    if (s->H % s->S || s->W % s->S || s->C % s->heads) return BRA_ERR_INVALID_ARG;
    if (s->S > 65535 / s->S || s->topk < 1 || s->topk > s->S * s->S) return BRA_ERR_INVALID_ARG;
    if (s->dtype != BRA_DTYPE_F32 && s->dtype != BRA_DTYPE_BF16) return BRA_ERR_INVALID_ARG;
    // All index arithmetic inside the kernels is 64-bit from the token offset
    // up; per-dimension sizes must still fit the grid.
    if ((int64_t)s->H * s->W > (int64_t)1 << 30 || s->B > 65535) return BRA_ERR_UNSUPPORTED;
    g->B = s->B; g->H = s->H; g->W = s->W; g->C = s->C; g->heads = s->heads; g->S = s->S;
    g->topk = s->topk;
    g->d = s->C / s->heads;
    g->R = s->S * s->S;
    g->hs = s->H / s->S;
    g->ws = s->W / s->S;
    g->n = g->hs * g->ws;
    if (g->d != 32) return BRA_ERR_UNSUPPORTED;
    if (g->R > kMaxRegions) return BRA_ERR_UNSUPPORTED;
    if (s->heads > 65535) return BRA_ERR_UNSUPPORTED;
    // pool: the 16-byte channel vectors of one token must fit the CTA's threads
    if ((size_t)s->C * elem_bytes(s->dtype) > 16u * kPoolThreads) return BRA_ERR_UNSUPPORTED;
    if ((int64_t)s->B * s->heads > 0x7fffffff) return BRA_ERR_UNSUPPORTED;
    return BRA_OK;
}

size_t means_bytes(const Geometry& g) {
    return round_up((size_t)g.B * g.heads * g.R * g.d * sizeof(float), 256);
}

struct Workspace {
    float* qr;
    float* kr;
    int* status;
};

Workspace carve(const Geometry& g, void* ws) {
    char* base = static_cast<char*>(ws);
    const size_t mb = means_bytes(g);
    return {reinterpret_cast<float*>(base), reinterpret_cast<float*>(base + mb),
            reinterpret_cast<int*>(base + 2 * mb)};
}

// Attention kernel selection.  The environment variable BRA_ATTEND_KERNEL
// (read on every call) pins one kernel for testing: "slice" (persistent
// tcgen05, a map of at most 256 tokens per (batch, head), dense with a
// routing mask), "warp" (warp-level MMAs over a (batch, head) slice's K and V
// resident in shared memory, small regions), "flash" (persistent tcgen05,
// regions of a multiple of 128 tokens, keys streamed in blocks with a running
// maximum), "stack" (persistent tcgen05, regions of 16..64 tokens), "tiled" (tcgen05 per 128-query tile), "simt" (CUDA cores); a
// pinned kernel that does not cover the shape makes the call return
// BRA_ERR_UNSUPPORTED.  Unset or "auto": the slice kernel for small maps,
// else the warp kernel when it covers the shape and each query region routes
// to several regions (a gather per query tile would re-read K and V topk
// times), else the first of flash, stack, tiled, simt that covers it
// (tensor-core kernels for bf16 only).
enum class AttendKernel { kAuto, kSlice, kWarp, kFlash, kStack, kTiled, kSimt };

AttendKernel attend_kernel_choice() {
    const char* e = getenv("BRA_ATTEND_KERNEL");
    if (!e) return AttendKernel::kAuto;
    if (!strcmp(e, "slice")) return AttendKernel::kSlice;
    if (!strcmp(e, "warp")) return AttendKernel::kWarp;
    if (!strcmp(e, "flash")) return AttendKernel::kFlash;
    if (!strcmp(e, "stack")) return AttendKernel::kStack;
    if (!strcmp(e, "tiled")) return AttendKernel::kTiled;
    if (!strcmp(e, "simt")) return AttendKernel::kSimt;
    return AttendKernel::kAuto;
}

bra_status route_impl(const bra_shape* s, const Geometry& g, const void* q, const void* k,
                      int32_t* idx, const Workspace& w, cudaStream_t st) {
    if (g.B == 0) return BRA_OK;
    const bool bf16 = s->dtype == BRA_DTYPE_BF16;
    if (launch_pool(bf16, q, k, w.qr, w.kr, g, st) != cudaSuccess) return BRA_ERR_CUDA;
    if (launch_route(w.qr, w.kr, idx, g, st) != cudaSuccess) return BRA_ERR_CUDA;
    return BRA_OK;
}

bra_status attend_impl(const bra_shape* s, const Geometry& g, const void* q, const void* k,
                       const void* v, const int32_t* idx, void* o, const Workspace& w,
                       cudaStream_t st) {
    if (g.B == 0) return BRA_OK;
    const bool bf16 = s->dtype == BRA_DTYPE_BF16;
    const AttendKernel choice = attend_kernel_choice();
    if (bf16 && (choice == AttendKernel::kSlice || (choice == AttendKernel::kAuto && attend_slice_covers(g)))) {
        const bra_status rc = attend_slice_launch(g, q, k, v, idx, o, w.status, st);
        if (rc != BRA_ERR_UNSUPPORTED || choice == AttendKernel::kSlice) return rc;
    }
    if (choice == AttendKernel::kSlice) return BRA_ERR_UNSUPPORTED;
    if (bf16 && (choice == AttendKernel::kWarp ||
                 (choice == AttendKernel::kAuto && g.topk > 1 && attend_warp_covers(g)))) {
        const bra_status rc = attend_warp_launch(g, q, k, v, idx, o, w.status, st);
        if (rc != BRA_ERR_UNSUPPORTED || choice == AttendKernel::kWarp) return rc;
    }
    if (choice == AttendKernel::kWarp) return BRA_ERR_UNSUPPORTED;
    if (bf16 && (choice == AttendKernel::kFlash || (choice == AttendKernel::kAuto && attend_flash_covers(g)))) {
        const bra_status rc = attend_flash_launch(g, q, k, v, idx, o, w.status, st);
        if (rc != BRA_ERR_UNSUPPORTED || choice == AttendKernel::kFlash) return rc;
    }
    if (choice == AttendKernel::kFlash) return BRA_ERR_UNSUPPORTED;
    if (bf16 && (choice == AttendKernel::kAuto || choice == AttendKernel::kStack)) {
        const bra_status rc = attend_stack_launch(g, q, k, v, idx, o, w.status, st);
        if (rc != BRA_ERR_UNSUPPORTED || choice == AttendKernel::kStack) return rc;
    }
    if (bf16 && (choice == AttendKernel::kAuto || choice == AttendKernel::kTiled)) {
        const bra_status rc = attend_tc_launch(g, q, k, v, idx, o, w.status, st);
        if (rc != BRA_ERR_UNSUPPORTED || choice == AttendKernel::kTiled) return rc;
    }
    if (choice == AttendKernel::kStack || choice == AttendKernel::kTiled) return BRA_ERR_UNSUPPORTED;
    if ((int64_t)g.R * simt_plan(g).chunks > 0x7fffffff) return BRA_ERR_UNSUPPORTED;
    if (launch_attend_simt(bf16, q, k, v, idx, o, g, w.status, st) != cudaSuccess)
        return BRA_ERR_CUDA;
    return BRA_OK;
}

}  // namespace
}  // namespace bra

using namespace bra;

extern "C" {

size_t bra_workspace_bytes(const bra_shape* shape) {
    Geometry g;
    if (make_geometry(shape, &g) != BRA_OK) return 0;
    return 2 * means_bytes(g) + kStatusBytes;
}

bra_status bra_route(const bra_shape* shape, const void* q, const void* k, int32_t* idx,
                     void* workspace, void* stream) {
    Geometry g;
    bra_status rc = make_geometry(shape, &g);
    if (rc != BRA_OK) return rc;
    if (!q || !k || !idx || !workspace) return BRA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(idx) || !aligned16(workspace))
        return BRA_ERR_INVALID_ARG;
    return route_impl(shape, g, q, k, idx, carve(g, workspace), static_cast<cudaStream_t>(stream));
}

bra_status bra_attend(const bra_shape* shape, const void* q, const void* k, const void* v,
                      const int32_t* idx, void* o, void* workspace, void* stream) {
    Geometry g;
    bra_status rc = make_geometry(shape, &g);
    if (rc != BRA_OK) return rc;
    if (!q || !k || !v || !idx || !o || !workspace) return BRA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(o) ||
        !aligned16(workspace))
        return BRA_ERR_INVALID_ARG;
    return attend_impl(shape, g, q, k, v, idx, o, carve(g, workspace),
                       static_cast<cudaStream_t>(stream));
}

bra_status bra_forward(const bra_shape* shape, const void* q, const void* k, const void* v,
                       void* o, int32_t* idx, void* workspace, void* stream) {
    Geometry g;
    bra_status rc = make_geometry(shape, &g);
    if (rc != BRA_OK) return rc;
    if (!q || !k || !v || !idx || !o || !workspace) return BRA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(o) ||
        !aligned16(workspace))
        return BRA_ERR_INVALID_ARG;
    const Workspace w = carve(g, workspace);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = route_impl(shape, g, q, k, idx, w, st);
    if (rc != BRA_OK) return rc;
    return attend_impl(shape, g, q, k, v, idx, o, w, st);
}

bra_status bra_lce(const bra_shape* shape, const void* v, const float* weight, const float* bias, void* o,
                   void* stream) {
    Geometry g;
    bra_status rc = make_geometry(shape, &g);
    if (rc != BRA_OK) return rc;
    if (!v || !weight || !o) return BRA_ERR_INVALID_ARG;
    if (!aligned16(v) || !aligned16(o) || !aligned16(weight) || (bias && !aligned16(bias)))
        return BRA_ERR_INVALID_ARG;
    if ((int64_t)g.H > (int64_t)65535 * 8) return BRA_ERR_UNSUPPORTED;  // grid rows of 8 outputs
    return launch_lce(shape->dtype == BRA_DTYPE_BF16, v, weight, bias, o, g, static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? BRA_OK
               : BRA_ERR_CUDA;
}

bra_status bra_forward_lce(const bra_shape* shape, const void* q, const void* k, const void* v, const float* weight,
                           const float* bias, void* o, int32_t* idx, void* workspace, void* stream) {
    Geometry g;
    bra_status rc = make_geometry(shape, &g);
    if (rc != BRA_OK) return rc;
    if (!q || !k || !v || !weight || !idx || !o || !workspace) return BRA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(weight) || (bias && !aligned16(bias)) ||
        !aligned16(idx) || !aligned16(o) || !aligned16(workspace))
        return BRA_ERR_INVALID_ARG;
    if ((int64_t)g.H > (int64_t)65535 * 8) return BRA_ERR_UNSUPPORTED;  // as bra_lce
    const Workspace w = carve(g, workspace);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = route_impl(shape, g, q, k, idx, w, st);
    if (rc != BRA_OK || g.B == 0) return rc;
    const AttendKernel choice = attend_kernel_choice();
    if (shape->dtype == BRA_DTYPE_BF16 && (choice == AttendKernel::kAuto || choice == AttendKernel::kStack) &&
        attend_stack_lce_covers(g)) {
        rc = attend_stack_lce_launch(g, q, k, v, weight, bias, idx, o, w.status, st);
        if (rc != BRA_ERR_UNSUPPORTED) return rc;
    }
    // other shapes: attention, then the filter added in place
    rc = attend_impl(shape, g, q, k, v, idx, o, w, st);
    if (rc != BRA_OK) return rc;
    return launch_lce(shape->dtype == BRA_DTYPE_BF16, v, weight, bias, o, g, st) == cudaSuccess ? BRA_OK
                                                                                                 : BRA_ERR_CUDA;
}

bra_status bra_attend_backward(const bra_shape* shape, const void* q, const void* k, const void* v,
                               const int32_t* idx, const void* grad_o, float* dq, float* dk, float* dv,
                               void* workspace, void* stream) {
    Geometry g;
    bra_status rc = make_geometry(shape, &g);
    if (rc != BRA_OK) return rc;
    if (!q || !k || !v || !idx || !grad_o || !dq || !dk || !dv || !workspace) return BRA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(idx) || !aligned16(grad_o) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(workspace))
        return BRA_ERR_INVALID_ARG;
    if (backward_smem_bytes(g) == 0) return BRA_ERR_UNSUPPORTED;
    if ((long long)g.B * g.heads > 65535) return BRA_ERR_UNSUPPORTED;  // one grid row per (batch, head)
    if (g.B == 0) return BRA_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t bytes = (size_t)g.B * g.H * g.W * g.C * sizeof(float);
    // BRA_BACKWARD_KERNEL pins the kernel: "mma" (tensor cores) or "simt"
    // (CUDA cores, fp32 throughout); by default the tensor-core kernel
    // wherever it covers the shape.
    const char* pin = getenv("BRA_BACKWARD_KERNEL");
    const bool want_mma = !pin || strcmp(pin, "simt") != 0;
    if (shape->dtype == BRA_DTYPE_BF16 && want_mma && backward_mma_covers(g)) {
        // dq is written in full by the kernel; dk and dv accumulate
        if (cudaMemsetAsync(dk, 0, bytes, st) != cudaSuccess || cudaMemsetAsync(dv, 0, bytes, st) != cudaSuccess)
            return BRA_ERR_CUDA;
        const cudaError_t e = launch_attend_backward_mma(q, k, v, idx, grad_o, dq, dk, dv, g,
                                                         carve(g, workspace).status, st);
        return e == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
    }
    if (pin && !strcmp(pin, "mma")) return BRA_ERR_UNSUPPORTED;
    if (cudaMemsetAsync(dq, 0, bytes, st) != cudaSuccess || cudaMemsetAsync(dk, 0, bytes, st) != cudaSuccess ||
        cudaMemsetAsync(dv, 0, bytes, st) != cudaSuccess)
        return BRA_ERR_CUDA;
    const cudaError_t e = launch_attend_backward(shape->dtype == BRA_DTYPE_BF16, q, k, v, idx, grad_o, dq, dk, dv, g,
                                                 carve(g, workspace).status, st);
    return e == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

bra_status bra_qkv_project(const bra_shape* shape, const void* x, const void* w_qkv, const float* b_qkv, void* q,
                           void* k, void* v, float* q_r, float* k_r, void* workspace, void* stream) {
    Geometry g;
    bra_status rc = make_geometry(shape, &g);
    if (rc != BRA_OK) return rc;
    if (!x || !w_qkv || !q || !k || !v || !q_r || !k_r || !workspace) return BRA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_qkv) || (b_qkv && !aligned16(b_qkv)) || !aligned16(q) || !aligned16(k) ||
        !aligned16(v) || !aligned16(q_r) || !aligned16(k_r) || !aligned16(workspace))
        return BRA_ERR_INVALID_ARG;
    if (shape->dtype != BRA_DTYPE_BF16 || qkv_check(g) != BRA_OK) return BRA_ERR_UNSUPPORTED;
    if (g.B == 0) return BRA_OK;
    return qkv_launch(g, x, w_qkv, b_qkv, q, k, v, q_r, k_r, carve(g, workspace).status,
                      static_cast<cudaStream_t>(stream));
}

bra_status bra_forward_qkv(const bra_shape* shape, const void* x, const void* w_qkv, const float* b_qkv, void* q,
                           void* k, void* v, void* o, int32_t* idx, void* workspace, void* stream) {
    Geometry g;
    bra_status rc = make_geometry(shape, &g);
    if (rc != BRA_OK) return rc;
    if (!x || !w_qkv || !q || !k || !v || !o || !idx || !workspace) return BRA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(w_qkv) || (b_qkv && !aligned16(b_qkv)) || !aligned16(q) || !aligned16(k) ||
        !aligned16(v) || !aligned16(o) || !aligned16(idx) || !aligned16(workspace))
        return BRA_ERR_INVALID_ARG;
    if (shape->dtype != BRA_DTYPE_BF16 || qkv_check(g) != BRA_OK) return BRA_ERR_UNSUPPORTED;
    if (g.B == 0) return BRA_OK;
    const Workspace w = carve(g, workspace);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    rc = qkv_launch(g, x, w_qkv, b_qkv, q, k, v, w.qr, w.kr, w.status, st);
    if (rc != BRA_OK) return rc;
    if (launch_route(w.qr, w.kr, idx, g, st) != cudaSuccess) return BRA_ERR_CUDA;
    return attend_impl(shape, g, q, k, v, idx, o, w, st);
}

bra_status bra_selftest_bounded_wait(const bra_shape* shape, void* workspace, unsigned int tries, int arrive,
                                     void* stream) {
    Geometry g;
    bra_status rc = make_geometry(shape, &g);
    if (rc != BRA_OK) return rc;
    if (!workspace || !aligned16(workspace) || tries == 0 || tries > (1u << 24)) return BRA_ERR_INVALID_ARG;
    return launch_bounded_wait_selftest(carve(g, workspace).status, tries, arrive != 0,
                                        static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? BRA_OK
               : BRA_ERR_CUDA;
}

bra_status bra_device_status(const bra_shape* shape, void* workspace, void* stream) {
    Geometry g;
    bra_status rc = make_geometry(shape, &g);
    if (rc != BRA_OK) return rc;
    if (!workspace || !aligned16(workspace)) return BRA_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int* status = carve(g, workspace).status;
    int host = 0;
    if (cudaMemcpyAsync(&host, status, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return BRA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return BRA_ERR_CUDA;
    if (cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess) return BRA_ERR_CUDA;
    if (host == kDevTimeout) return BRA_ERR_TIMEOUT;
    if (host == kDevBadRoute) return BRA_ERR_BAD_ROUTE;
    if (host == kDevBounds) return BRA_ERR_BOUNDS;
    return host == 0 ? BRA_OK : BRA_ERR_CUDA;
}

const char* bra_status_string(bra_status status) {
    switch (status) {
        case BRA_OK: return "ok";
        case BRA_ERR_INVALID_ARG: return "invalid argument";
        case BRA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case BRA_ERR_CUDA: return "CUDA error";
        case BRA_ERR_TIMEOUT: return "device-side wait timed out";
        case BRA_ERR_BAD_ROUTE: return "routing index out of range";
        case BRA_ERR_BOUNDS: return "index outside its buffer (debug build)";
    }
    return "unknown status";
}

int bra_version(void) { return 100; }

}  // extern "C"
