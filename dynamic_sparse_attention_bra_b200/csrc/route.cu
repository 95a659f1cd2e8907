// Region-level routing kernels (blog "BiFormer Reshapes Visual Attention with
// Bi-Level Routing", Part 2 section 2.2, step 3):
//   bra_pool_kernel   Q^r, K^r = per-region means of Q and K (fp32)
//   bra_route_kernel  A^r = Q^r (K^r)^T in fp32, then row-wise top-k -> I^r
#include "common.cuh"
#include "kernels.h"

namespace bra {

// ---------------------------------------------------------------------------
// Pool: one CTA of 128 threads per (region, batch).  Thread t owns one 16-byte
// channel vector cv = t % nv of the C channels (nv = C / (16 / sizeof(T)))
// and every sp-th token of the region, sp = 128 / nv, for Q and for K, so a
// warp reads whole 16-byte runs of consecutive tokens and each thread keeps
// up to 8 loads in flight.  The sp partial sums per channel meet in shared
// memory; the means are written in fp32 [B, heads, R, d] order (channel
// c = h * d + i of region r).
// HBM traffic: Q and K read once (2 * B*H*W*C*sizeof(T) bytes), means written.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
bra_pool_kernel(const T* __restrict__ q, const T* __restrict__ k, float* __restrict__ qr,
                float* __restrict__ kr, Geometry g) {
    constexpr int VEC = 16 / sizeof(T);
    constexpr int kUnroll = 4;
    extern __shared__ float pool_smem[];  // [2][sp][C] partial sums
    const int r = blockIdx.x, b = blockIdx.y;
    const int nv = g.C / VEC;
    const int sp = kPoolThreads / nv;  // host guarantees 1 <= nv <= kPoolThreads
    const int tid = threadIdx.x;
    const int cv = tid % nv, j = tid / nv;

    float aq[VEC], ak[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) aq[i] = ak[i] = 0.f;

    if (j < sp) {
        const size_t base = token_offset(g, b, r, 0) + (size_t)cv * VEC;
        const size_t row_stride = (size_t)g.W * g.C;
        int t = j;
        for (; t + (kUnroll - 1) * sp < g.n; t += kUnroll * sp) {
            uint4 uq[kUnroll], uk[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int tt = t + u * sp;
                const int ty = tt / g.ws, tx = tt - ty * g.ws;
                const size_t off = base + ty * row_stride + (size_t)tx * g.C;
                uq[u] = __ldg(reinterpret_cast<const uint4*>(q + off));
                uk[u] = __ldg(reinterpret_cast<const uint4*>(k + off));
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                float fq[VEC], fk[VEC];
                unpack16(uq[u], fq, q);
                unpack16(uk[u], fk, k);
#pragma unroll
                for (int i = 0; i < VEC; ++i) {
                    aq[i] += fq[i];
                    ak[i] += fk[i];
                }
            }
        }
        for (; t < g.n; t += sp) {
            const int ty = t / g.ws, tx = t - ty * g.ws;
            const size_t off = base + ty * row_stride + (size_t)tx * g.C;
            float fq[VEC], fk[VEC];
            unpack16(__ldg(reinterpret_cast<const uint4*>(q + off)), fq, q);
            unpack16(__ldg(reinterpret_cast<const uint4*>(k + off)), fk, k);
#pragma unroll
            for (int i = 0; i < VEC; ++i) {
                aq[i] += fq[i];
                ak[i] += fk[i];
            }
        }
        float* sq = pool_smem + (size_t)j * g.C + cv * VEC;
        float* sk = pool_smem + (size_t)(sp + j) * g.C + cv * VEC;
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
            sq[i] = aq[i];
            sk[i] = ak[i];
        }
    }
    __syncthreads();
    allow_dependents();  // the route kernel may launch; it waits for this grid's writes
    const float inv_n = 1.f / (float)g.n;
    for (int c = tid; c < 2 * g.C; c += kPoolThreads) {
        const int which = c / g.C, ch = c - which * g.C;
        const float* src = pool_smem + (size_t)which * sp * g.C + ch;
        float s = 0.f;
        for (int jj = 0; jj < sp; ++jj) s += src[(size_t)jj * g.C];
        const int h = ch / g.d, i = ch - h * g.d;
        float* out = which ? kr : qr;
        out[(((size_t)b * g.heads + h) * g.R + r) * g.d + i] = s * inv_n;
    }
}

// ---------------------------------------------------------------------------
// Pool, strip form: one CTA per (region row i, batch) covers the hs image rows
// of that row of regions, which are one contiguous run of hs * W * C
// elements.  Thread t owns column x = t / nv and channel vector cv = t % nv,
// so a warp reads consecutive 16-byte vectors of an image row, and sums its
// column over the hs rows (all loads of a thread issued back to back).  The
// per-column sums meet in shared memory, where each output channel of each of
// the S regions adds its ws columns.  Used when there are enough (i, b) pairs
// to fill the GPU; the region form above covers the rest.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kStripMaxThreads)
bra_pool_strip_kernel(const T* __restrict__ q, const T* __restrict__ k, float* __restrict__ qr,
                      float* __restrict__ kr, Geometry g) {
    constexpr int VEC = 16 / sizeof(T);
    extern __shared__ float strip_smem[];  // [2][W][C] column sums of Q and K
    const int i = blockIdx.x, b = blockIdx.y;
    const int nv = g.C / VEC;
    const int t = threadIdx.x;
    const size_t row_elems = (size_t)g.W * g.C;
    const size_t base = ((size_t)b * g.H + (size_t)i * g.hs) * row_elems;
    if (t < g.W * nv) {
        const int x = t / nv, cv = t - x * nv;
        const size_t off0 = base + (size_t)x * g.C + (size_t)cv * VEC;
        float aq[VEC], ak[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) aq[e] = ak[e] = 0.f;
        // All rows of up to 8 at once: 16 independent 16-byte loads per thread.
        int y = 0;
        for (; y + 7 < g.hs; y += 8) {
            uint4 uq[8], uk[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                uq[u] = __ldg(reinterpret_cast<const uint4*>(q + off0 + (size_t)(y + u) * row_elems));
                uk[u] = __ldg(reinterpret_cast<const uint4*>(k + off0 + (size_t)(y + u) * row_elems));
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                float fq[VEC], fk[VEC];
                unpack16(uq[u], fq, q);
                unpack16(uk[u], fk, k);
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    aq[e] += fq[e];
                    ak[e] += fk[e];
                }
            }
        }
        for (; y + 3 < g.hs; y += 4) {
            uint4 uq[4], uk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                uq[u] = __ldg(reinterpret_cast<const uint4*>(q + off0 + (size_t)(y + u) * row_elems));
                uk[u] = __ldg(reinterpret_cast<const uint4*>(k + off0 + (size_t)(y + u) * row_elems));
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float fq[VEC], fk[VEC];
                unpack16(uq[u], fq, q);
                unpack16(uk[u], fk, k);
#pragma unroll
                for (int e = 0; e < VEC; ++e) {
                    aq[e] += fq[e];
                    ak[e] += fk[e];
                }
            }
        }
        for (; y < g.hs; ++y) {
            float fq[VEC], fk[VEC];
            unpack16(__ldg(reinterpret_cast<const uint4*>(q + off0 + (size_t)y * row_elems)), fq, q);
            unpack16(__ldg(reinterpret_cast<const uint4*>(k + off0 + (size_t)y * row_elems)), fk, k);
#pragma unroll
            for (int e = 0; e < VEC; ++e) {
                aq[e] += fq[e];
                ak[e] += fk[e];
            }
        }
        float* sq = strip_smem + (size_t)x * g.C + cv * VEC;
        float* sk = strip_smem + row_elems + (size_t)x * g.C + cv * VEC;
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
            sq[e] = aq[e];
            sk[e] = ak[e];
        }
    }
    __syncthreads();
    allow_dependents();  // the route kernel may launch; it waits for this grid's writes
    const float inv_n = 1.f / (float)g.n;
    const int outs = 2 * g.S * g.C;
    for (int oo = t; oo < outs; oo += blockDim.x) {
        const int which = oo / (g.S * g.C);
        const int rem = oo - which * g.S * g.C;
        const int j = rem / g.C, c = rem - j * g.C;
        const float* src = strip_smem + which * row_elems + (size_t)j * g.ws * g.C + c;
        float s = 0.f;
        for (int xx = 0; xx < g.ws; ++xx) s += src[(size_t)xx * g.C];
        const int h = c / g.d, e = c - h * g.d;
        float* out = which ? kr : qr;
        out[(((size_t)b * g.heads + h) * g.R + i * g.S + j) * g.d + e] = s * inv_n;
    }
}

// ---------------------------------------------------------------------------
// Route: one CTA per (batch, head).  Q^r and K^r of the slice go to shared
// memory (rows padded to d + 1 floats so that 32 lanes reading 32 different
// K^r rows hit 32 banks).  A warp owns one row r at a time: lane l computes
// A[r][j] for j = l, l + 32, ... (fp32, channels in order), then topk rounds
// of a warp-wide argmax under the key (value descending, index ascending)
// pick the routed regions in order.  A^r never leaves registers.
// ---------------------------------------------------------------------------
constexpr int kMaxColsPerLane = kMaxRegions / 32;

__device__ __forceinline__ bool route_before(float va, int ia, float vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

__global__ void __launch_bounds__(kRouteThreads)
bra_route_kernel(const float* __restrict__ qr, const float* __restrict__ kr,
                 int32_t* __restrict__ idx, Geometry g) {
    constexpr int D = 32;                      // head dim (checked on the host)
    constexpr int LD = D + 4;                  // padded row: 16-byte aligned, 8 lanes hit 32 banks
    constexpr int kRows = kRouteThreads / 32;  // one row of A^r per warp
    extern __shared__ float4 route_smem4[];    // K^r of the slice, [R][LD]
    float* sk = reinterpret_cast<float*>(route_smem4);
    grid_dependency_wait();  // the pool kernel's means are complete and visible
    allow_dependents();      // the attention kernel may start its set-up
    const int R = g.R;
    const size_t bh = blockIdx.x;
    const int row0 = blockIdx.y * kRows;
    const float4* gk = reinterpret_cast<const float4*>(kr + bh * R * D);
    for (int e0 = threadIdx.x; e0 < R * (D / 4); e0 += 4 * kRouteThreads) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = e0 + u * kRouteThreads;
            if (e < R * (D / 4)) v[u] = __ldg(gk + e);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = e0 + u * kRouteThreads;
            if (e < R * (D / 4)) *reinterpret_cast<float4*>(sk + (e / (D / 4)) * LD + (e % (D / 4)) * 4) = v[u];
        }
    }
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int r = row0 + warp;
    if (r >= R) return;
    // This warp's query mean, in registers (same 128 bytes for all lanes).
    float qv[D];
    const float4* gq = reinterpret_cast<const float4*>(qr + (bh * R + r) * D);
#pragma unroll
    for (int c = 0; c < D / 4; ++c) {
        const float4 t = __ldg(gq + c);
        qv[4 * c] = t.x; qv[4 * c + 1] = t.y; qv[4 * c + 2] = t.z; qv[4 * c + 3] = t.w;
    }
    const int cols = (R + 31) / 32;
    float a[kMaxColsPerLane];
#pragma unroll
    for (int i = 0; i < kMaxColsPerLane; ++i) {
        a[i] = -INFINITY;
        const int jcol = lane + 32 * i;
        if (i < cols && jcol < R) {
            const float* krow = sk + jcol * LD;
            float s = 0.f;
#pragma unroll
            for (int c = 0; c < D / 4; ++c) {
                const float4 k4 = *reinterpret_cast<const float4*>(krow + 4 * c);
                s = fmaf(qv[4 * c], k4.x, s);
                s = fmaf(qv[4 * c + 1], k4.y, s);
                s = fmaf(qv[4 * c + 2], k4.z, s);
                s = fmaf(qv[4 * c + 3], k4.w, s);
            }
            a[i] = s;
        }
    }
    uint32_t taken = 0;  // bit i: column lane + 32 i already routed
    int32_t* out = idx + (bh * R + r) * g.topk;
    for (int m = 0; m < g.topk; ++m) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < kMaxColsPerLane; ++i) {
            const int jcol = lane + 32 * i;
            if (i < cols && jcol < R && !(taken >> i & 1u) && route_before(a[i], jcol, bv, bi)) {
                bv = a[i];
                bi = jcol;
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
            if (route_before(ov, oi, bv, bi)) {
                bv = ov;
                bi = oi;
            }
        }
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (lane == 0) out[m] = bi;
    }
}

cudaError_t launch_pool(bool bf16, const void* q, const void* k, float* qr, float* kr,
                        const Geometry& g, cudaStream_t stream) {
    const int vec = bf16 ? 8 : 4;
    {
        // Strip form when a row of regions fits one CTA and there are enough rows.
        const int threads = (g.W * (g.C / vec) + 31) / 32 * 32;
        const size_t smem = (size_t)2 * g.W * g.C * sizeof(float);
        if (threads <= kStripMaxThreads && smem <= 48 * 1024 && (long long)g.B * g.S >= 148) {
            const dim3 grid(g.S, g.B);
            if (bf16)
                bra_pool_strip_kernel<__nv_bfloat16><<<grid, threads, smem, stream>>>(
                    static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), qr, kr, g);
            else
                bra_pool_strip_kernel<float><<<grid, threads, smem, stream>>>(
                    static_cast<const float*>(q), static_cast<const float*>(k), qr, kr, g);
            return cudaGetLastError();
        }
    }
    const int nv = g.C / vec;
    const int sp = kPoolThreads / nv;
    const size_t smem = (size_t)2 * sp * g.C * sizeof(float);
    const dim3 grid(g.R, g.B);
    if (bf16)
        bra_pool_kernel<__nv_bfloat16><<<grid, kPoolThreads, smem, stream>>>(
            static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), qr, kr, g);
    else
        bra_pool_kernel<float><<<grid, kPoolThreads, smem, stream>>>(
            static_cast<const float*>(q), static_cast<const float*>(k), qr, kr, g);
    return cudaGetLastError();
}

cudaError_t launch_route(const float* qr, const float* kr, int32_t* idx, const Geometry& g,
                         cudaStream_t stream) {
    const size_t smem = (size_t)g.R * (32 + 4) * sizeof(float);
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(
            bra_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    const dim3 grid(g.B * g.heads, (g.R + kRouteThreads / 32 - 1) / (kRouteThreads / 32));
    return launch_after_previous(bra_route_kernel, grid, dim3(kRouteThreads), smem, stream, qr, kr, idx, g);
}

}  // namespace bra
