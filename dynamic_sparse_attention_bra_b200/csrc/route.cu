// Region-level routing kernels (blog "BiFormer Reshapes Visual Attention with
// Bi-Level Routing", Part 2 section 2.2, step 3):
//   bra_pool_kernel   Q^r, K^r = per-region means of Q and K (fp32)
//   bra_route_kernel  A^r = Q^r (K^r)^T in fp32, then row-wise top-k -> I^r
#include "common.cuh"
#include "kernels.h"

namespace bra {

// ---------------------------------------------------------------------------
// Pool: one CTA per (region, batch).  The region's rows are contiguous runs
// of ws * C elements, so a CTA streams them with 16-byte vector loads: thread
// tid owns vector column (tid % nv) of the channels and every (G)-th token,
// where nv = C / (16 / sizeof(T)) vectors per token and G = 256 / nv token
// groups.  Partial sums meet in shared memory; the means are written in
// fp32 [B, heads, R, d] order (channel c = h * d + i of region r).
// HBM traffic: Q and K read once (2 * B*H*W*C*sizeof(T) bytes), means written.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
bra_pool_kernel(const T* __restrict__ q, const T* __restrict__ k, float* __restrict__ qr,
                float* __restrict__ kr, Geometry g) {
    constexpr int VEC = 16 / sizeof(T);
    extern __shared__ float pool_smem[];  // [groups][C] for Q then for K
    const int r = blockIdx.x, b = blockIdx.y;
    const int nv = g.C / VEC;
    const int groups = kPoolThreads / nv;  // host guarantees nv <= kPoolThreads
    const int tid = threadIdx.x;
    const int col = tid % nv, grp = tid / nv;

    float aq[VEC], ak[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) aq[i] = ak[i] = 0.f;

    if (grp < groups) {
        // Unroll by 4 tokens to keep several 16-byte loads in flight per thread.
        int t = grp;
        for (; t + 3 * groups < g.n; t += 4 * groups) {
            uint4 uq[4], uk[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const size_t off = token_offset(g, b, r, t + u * groups) + (size_t)col * VEC;
                uq[u] = __ldg(reinterpret_cast<const uint4*>(q + off));
                uk[u] = __ldg(reinterpret_cast<const uint4*>(k + off));
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
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
        for (; t < g.n; t += groups) {
            const size_t off = token_offset(g, b, r, t) + (size_t)col * VEC;
            float fq[VEC], fk[VEC];
            unpack16(__ldg(reinterpret_cast<const uint4*>(q + off)), fq, q);
            unpack16(__ldg(reinterpret_cast<const uint4*>(k + off)), fk, k);
#pragma unroll
            for (int i = 0; i < VEC; ++i) {
                aq[i] += fq[i];
                ak[i] += fk[i];
            }
        }
        float* sq = pool_smem + (size_t)grp * g.C + col * VEC;
        float* sk = pool_smem + (size_t)(groups + grp) * g.C + col * VEC;
#pragma unroll
        for (int i = 0; i < VEC; ++i) {
            sq[i] = aq[i];
            sk[i] = ak[i];
        }
    }
    __syncthreads();
    const float inv_n = 1.f / (float)g.n;
    for (int c = tid; c < 2 * g.C; c += kPoolThreads) {
        const int which = c / g.C, ch = c - which * g.C;
        const float* base = pool_smem + (size_t)which * groups * g.C + ch;
        float s = 0.f;
        for (int j = 0; j < groups; ++j) s += base[(size_t)j * g.C];
        const int h = ch / g.d, i = ch - h * g.d;
        float* out = which ? kr : qr;
        out[(((size_t)b * g.heads + h) * g.R + r) * g.d + i] = s * inv_n;
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
    extern __shared__ float route_smem[];
    const int R = g.R, d = g.d, ld = d + 1;
    float* sq = route_smem;
    float* sk = route_smem + (size_t)R * ld;
    const size_t bh = blockIdx.x;
    const float* gq = qr + bh * R * d;
    const float* gk = kr + bh * R * d;
    for (int e = threadIdx.x; e < R * d; e += kRouteThreads) {
        const int row = e / d, c = e - row * d;
        sq[row * ld + c] = gq[e];
        sk[row * ld + c] = gk[e];
    }
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int cols = (R + 31) / 32;
    for (int r = warp; r < R; r += kRouteThreads / 32) {
        float a[kMaxColsPerLane];
#pragma unroll
        for (int i = 0; i < kMaxColsPerLane; ++i) {
            a[i] = -INFINITY;
            const int j = lane + 32 * i;
            if (i < cols && j < R) {
                float s = 0.f;
                for (int c = 0; c < d; ++c) s = fmaf(sq[r * ld + c], sk[j * ld + c], s);
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
                const int j = lane + 32 * i;
                if (i < cols && j < R && !(taken >> i & 1u) && route_before(a[i], j, bv, bi)) {
                    bv = a[i];
                    bi = j;
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
}

cudaError_t launch_pool(bool bf16, const void* q, const void* k, float* qr, float* kr,
                        const Geometry& g, cudaStream_t stream) {
    const int vec = bf16 ? 8 : 4;
    const int nv = g.C / vec;
    const int groups = kPoolThreads / nv;
    const size_t smem = (size_t)2 * groups * g.C * sizeof(float);
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
    const size_t smem = (size_t)2 * g.R * (g.d + 1) * sizeof(float);
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(
            bra_route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    bra_route_kernel<<<g.B * g.heads, kRouteThreads, smem, stream>>>(qr, kr, idx, g);
    return cudaGetLastError();
}

}  // namespace bra
