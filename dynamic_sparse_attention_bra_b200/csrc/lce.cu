// Local context enhancement (blog "BiFormer Reshapes Visual Attention with
// Bi-Level Routing", Part 2 section 2.2, step 4 third bullet; the pseudocode's
// step 7 adds "dwconv(value)" to the attention output):
//   o[b, y, x, c] += bias[c] + sum_{i, j = 0..4} w[c][i][j] * v[b, y + i - 2, x + j - 2, c]
// with v = 0 outside the map (5x5 depthwise filter, zero padding 2).
//
// A memory-bound stencil on CUDA cores, fp32 accumulation.  A tile is 8
// rows x 32 columns of one 128-byte channel group (64 bf16 or 32 fp32
// channels).  The kernel is persistent, two CTAs per SM: each CTA walks its
// tiles and, while it computes one, copies the next one's 12 x 36 halo of v
// into the other of two shared-memory buffers with 16-byte cp.async (zeros
// outside the map, which is the zero padding), so loading and arithmetic
// overlap.  Lane l owns channel pair 2l, 2l + 1 (bf16) or channel l (fp32) of
// the group with its 25 taps in registers, and warp w computes columns
// 4w .. 4w + 3 of the tile, each as a strip of 8 outputs down the column: the
// strip's o values are fetched first, its 12 input rows are read from shared
// memory once (5 taps each, 128 contiguous bytes per warp read) and added to
// the (up to 5) outputs each row reaches.
// HBM traffic: v read about once (halo reads mostly hit L2), o read and
// written once.
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace bra {
namespace {

constexpr int kLceRows = 8;                // outputs per strip (tile rows)
constexpr int kLceCols = 32;               // tile columns
constexpr int kLceStrips = 4;              // columns per warp
constexpr int kLceThreads = 256;           // 8 warps x 4 strips = 32 columns
constexpr int kHaloRows = kLceRows + 4, kHaloCols = kLceCols + 4;
constexpr int kHaloChunks = kHaloRows * kHaloCols * 8;  // 16-byte chunks of the halo tile

// Two fp32 lanes in one 64-bit register (x in the low half): sm_100a
// multiplies and adds both with one fma.rn.f32x2, rounding each as fmaf would.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
// bf16 pair -> packed fp32 pair (each bf16 is the high half of its float)
__device__ __forceinline__ uint64_t f2_from_bf16x2(uint32_t r) {
    return f2_pack(__uint_as_float(r << 16), __uint_as_float(r & 0xffff0000u));
}

template <typename T>
struct LceVec;  // the channels of one lane: 2 bf16 or 1 float
template <>
struct LceVec<__nv_bfloat16> {
    static constexpr int kCh = 2;
    using Raw = uint32_t;
    __device__ static void unpack(Raw r, float* f) {
        f[0] = __uint_as_float(r << 16);
        f[1] = __uint_as_float(r & 0xffff0000u);
    }
    __device__ static Raw pack(const float* f) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(f[0], f[1]);
        return *reinterpret_cast<const uint32_t*>(&h);
    }
};
template <>
struct LceVec<float> {
    static constexpr int kCh = 1;
    using Raw = float;
    __device__ static void unpack(Raw r, float* f) { f[0] = r; }
    __device__ static Raw pack(const float* f) { return f[0]; }
};

struct LceTiles {
    int tiles_x, tiles_y, groups, count;  // tiles across, down, channel groups; all tiles
};

template <typename T>
__global__ void __launch_bounds__(kLceThreads, 2)
bra_lce_kernel(const T* __restrict__ v, const float* __restrict__ w, const float* __restrict__ bias,
               T* __restrict__ o, int B, int H, int W, int C, LceTiles tl) {
    using V = LceVec<T>;
    using Raw = typename V::Raw;
    constexpr int CH = V::kCh;
    extern __shared__ uint4 lce_raw[];  // two buffers of kHaloChunks 16-byte chunks
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gbytes_all = C * (int)sizeof(T);
    const size_t token_bytes = (size_t)gbytes_all, row_bytes = (size_t)W * token_bytes;
    // tile t = ((b * tiles_y + ty) * tiles_x + tx) * groups + grp
    auto coords = [&](int t, int& b, int& y0, int& x0, int& grp) {
        grp = t % tl.groups;
        int u = t / tl.groups;
        x0 = (u % tl.tiles_x) * kLceCols;
        u /= tl.tiles_x;
        y0 = (u % tl.tiles_y) * kLceRows;
        b = u / tl.tiles_y;
    };
    auto stage = [&](int t, int buf) {
        int b, y0, x0, grp;
        coords(t, b, y0, x0, grp);
        const int gbytes = min(128, gbytes_all - grp * 128);
        const char* vb = reinterpret_cast<const char*>(v) + (size_t)b * H * row_bytes + (size_t)grp * 128;
        const uint32_t base = ptx::smem_addr(lce_raw + (size_t)buf * kHaloChunks);
#pragma unroll 4
        for (int k = threadIdx.x; k < kHaloChunks; k += kLceThreads) {
            const int row = k / (kHaloCols * 8), rem = k - row * (kHaloCols * 8);
            const int col = rem >> 3, q = rem & 7;
            const int y = y0 - 2 + row, x = x0 - 2 + col;
            const bool in = y >= 0 && y < H && x >= 0 && x < W && q * 16 < gbytes;
            const char* src = in ? vb + (size_t)y * row_bytes + (size_t)x * token_bytes + q * 16 : vb;
            ptx::cp_async16_zfill(base + (uint32_t)k * 16u, src, in ? 16u : 0u);
        }
    };
    int t = blockIdx.x;
    if (t < tl.count) stage(t, 0);
    ptx::cp_async_commit();
    int wgrp = -1;  // channel group whose taps are in registers
    float wt[CH][25], b0[CH];
    uint64_t wt2[25], b2 = 0;  // the bf16 path keeps its two channels' taps packed
    for (int i = 0; t < tl.count; ++i, t += gridDim.x) {
        // the next tile streams into the other buffer while this one is computed
        if (t + (int)gridDim.x < tl.count) stage(t + gridDim.x, (i + 1) & 1);
        ptx::cp_async_commit();
        ptx::cp_async_wait_group<1>();  // this tile's copies (all but the newest group) are done
        __syncthreads();
        int b, y0, x0, grp;
        coords(t, b, y0, x0, grp);
        const int c0 = grp * (128 / (int)sizeof(T)) + lane * CH;  // this lane's first channel
        if (c0 < C) {
            const Raw* tile = reinterpret_cast<const Raw*>(lce_raw + (size_t)(i & 1) * kHaloChunks);  // 32 Raw per token
            if constexpr (CH == 2) {
                // bf16: the lane's two channels ride together in packed fp32 pairs
                if (grp != wgrp) {
#pragma unroll
                    for (int tp = 0; tp < 25; ++tp)
                        wt2[tp] = f2_pack(__ldg(w + (size_t)c0 * 25 + tp), __ldg(w + (size_t)(c0 + 1) * 25 + tp));
                    b2 = bias ? f2_pack(__ldg(bias + c0), __ldg(bias + c0 + 1)) : f2_pack(0.f, 0.f);
                    wgrp = grp;
                }
                for (int st = 0; st < kLceStrips; ++st) {
                    const int cx = warp * kLceStrips + st;  // column inside the tile
                    const int x = x0 + cx;
                    if (x >= W) break;
                    T* ob = o + ((size_t)b * H * W + (size_t)x) * C + c0;
                    Raw cur_raw[kLceRows];
#pragma unroll
                    for (int r = 0; r < kLceRows; ++r)
                        cur_raw[r] = y0 + r < H ? *reinterpret_cast<const Raw*>(ob + (size_t)(y0 + r) * W * C) : Raw(0);
                    uint64_t acc[kLceRows];
#pragma unroll
                    for (int r = 0; r < kLceRows; ++r) acc[r] = b2;
                    const Raw* colp = tile + cx * 32 + lane;
#pragma unroll
                    for (int k = 0; k < kHaloRows; ++k) {
                        uint64_t f[5];
#pragma unroll
                        for (int j = 0; j < 5; ++j) f[j] = f2_from_bf16x2(colp[(k * kHaloCols + j) * 32]);
#pragma unroll
                        for (int r = 0; r < kLceRows; ++r) {
                            const int ti = k - r;
                            if (ti < 0 || ti > 4) continue;
#pragma unroll
                            for (int j = 0; j < 5; ++j) acc[r] = f2_fma(wt2[ti * 5 + j], f[j], acc[r]);
                        }
                    }
#pragma unroll
                    for (int r = 0; r < kLceRows; ++r) {
                        if (y0 + r >= H) break;
                        float cur[2], sum[2];
                        V::unpack(cur_raw[r], cur);
                        f2_unpack(acc[r], sum[0], sum[1]);
                        sum[0] += cur[0];
                        sum[1] += cur[1];
                        *reinterpret_cast<Raw*>(ob + (size_t)(y0 + r) * W * C) = V::pack(sum);
                    }
                }
            } else {
            if (grp != wgrp) {
#pragma unroll
                for (int e = 0; e < CH; ++e) {
#pragma unroll
                    for (int tp = 0; tp < 25; ++tp) wt[e][tp] = __ldg(w + (size_t)(c0 + e) * 25 + tp);
                    b0[e] = bias ? __ldg(bias + c0 + e) : 0.f;
                }
                wgrp = grp;
            }
            for (int st = 0; st < kLceStrips; ++st) {
                const int cx = warp * kLceStrips + st;  // column inside the tile
                const int x = x0 + cx;
                if (x >= W) break;
                // o of the strip, fetched now and used at the end
                T* ob = o + ((size_t)b * H * W + (size_t)x) * C + c0;
                Raw cur_raw[kLceRows];
#pragma unroll
                for (int r = 0; r < kLceRows; ++r)
                    cur_raw[r] = y0 + r < H ? *reinterpret_cast<const Raw*>(ob + (size_t)(y0 + r) * W * C) : Raw(0);
                float acc[kLceRows][CH];
#pragma unroll
                for (int r = 0; r < kLceRows; ++r)
#pragma unroll
                    for (int e = 0; e < CH; ++e) acc[r][e] = b0[e];
                const Raw* colp = tile + cx * 32 + lane;
#pragma unroll
                for (int k = 0; k < kHaloRows; ++k) {  // input row y0 - 2 + k
                    float f[5][CH];
#pragma unroll
                    for (int j = 0; j < 5; ++j) V::unpack(colp[(k * kHaloCols + j) * 32], f[j]);
                    // output row y0 + r sees this input row through tap row i = k - r
#pragma unroll
                    for (int r = 0; r < kLceRows; ++r) {
                        const int ti = k - r;
                        if (ti < 0 || ti > 4) continue;
#pragma unroll
                        for (int j = 0; j < 5; ++j)
#pragma unroll
                            for (int e = 0; e < CH; ++e) acc[r][e] = fmaf(wt[e][ti * 5 + j], f[j][e], acc[r][e]);
                    }
                }
#pragma unroll
                for (int r = 0; r < kLceRows; ++r) {
                    if (y0 + r >= H) break;
                    float cur[CH], sum[CH];
                    V::unpack(cur_raw[r], cur);
#pragma unroll
                    for (int e = 0; e < CH; ++e) sum[e] = cur[e] + acc[r][e];
                    *reinterpret_cast<Raw*>(ob + (size_t)(y0 + r) * W * C) = V::pack(sum);
                }
            }
        }
            }
        __syncthreads();  // the buffer is free for the tile after next
    }
    ptx::cp_async_wait_all();
}

}  // namespace

cudaError_t launch_lce(bool bf16, const void* v, const float* w, const float* bias, void* o, const Geometry& g,
                       cudaStream_t stream) {
    if (g.B == 0) return cudaSuccess;
    LceTiles tl;
    tl.groups = (g.C * (bf16 ? 2 : 4) + 127) / 128;
    tl.tiles_x = (g.W + kLceCols - 1) / kLceCols;
    tl.tiles_y = (g.H + kLceRows - 1) / kLceRows;
    const long long count = (long long)g.B * tl.tiles_y * tl.tiles_x * tl.groups;
    if (count > 0x7fffffffLL) return cudaErrorInvalidValue;
    tl.count = (int)count;
    int sms = sm_count();
    if (sms <= 0) sms = 148;
    const int grid = tl.count < 2 * sms ? tl.count : 2 * sms;  // two persistent CTAs per SM
    const size_t smem = (size_t)2 * kHaloChunks * 16;         // two halo buffers
    if (bf16) {
        auto k = bra_lce_kernel<__nv_bfloat16>;
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return cudaGetLastError();
        k<<<grid, kLceThreads, smem, stream>>>(static_cast<const __nv_bfloat16*>(v), w, bias,
                                               static_cast<__nv_bfloat16*>(o), g.B, g.H, g.W, g.C, tl);
    } else {
        auto k = bra_lce_kernel<float>;
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return cudaGetLastError();
        k<<<grid, kLceThreads, smem, stream>>>(static_cast<const float*>(v), w, bias, static_cast<float*>(o), g.B,
                                               g.H, g.W, g.C, tl);
    }
    return cudaGetLastError();
}

}  // namespace bra
