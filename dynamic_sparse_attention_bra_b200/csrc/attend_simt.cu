// Token-to-token attention over routed regions on the CUDA cores (blog
// "BiFormer Reshapes Visual Attention with Bi-Level Routing", Part 2 section
// 2.2, step 4).  This kernel serves the fp32 path (exact fp32 products) and
// any shape the tensor-core kernel does not take.
//
// One CTA per (query chunk of a region, head, batch).  Each query is owned by
// a group of ``plan.group`` lanes of one warp that split its keys; the routed
// keys are staged through shared memory 64 at a time, converted to fp32, so
// the gathered K/V never travel back to HBM.  Each lane keeps a base-2 online
// softmax (running max m, sum l, accumulator acc[D]) and the group merges its
// partial states with shuffles at the end.
#include "common.cuh"
#include "kernels.h"

namespace bra {

template <typename T, int D>
__global__ void __launch_bounds__(kSimtThreads)
bra_attend_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                       const int32_t* __restrict__ idx, T* __restrict__ o, Geometry g,
                       SimtPlan plan, int* status) {
    constexpr int VEC = 16 / sizeof(T);
    constexpr int NV = D / VEC;  // 16-byte vectors per head row
    constexpr int LD = D + 4;    // padded fp32 row: 8 lanes on 8 rows hit 32 banks
    __shared__ __align__(16) float ks[kSimtKeyBlock][LD];
    __shared__ __align__(16) float vs[kSimtKeyBlock][LD];
    __shared__ int routes[kMaxRegions];
    __shared__ uint32_t seen[kMaxRegions / 32];
    __shared__ int bad, nroutes;

    const int chunk_id = blockIdx.x % plan.chunks, r = blockIdx.x / plan.chunks;
    const int h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x;
    const int32_t* row = idx + (((size_t)b * g.heads + h) * g.R + r) * g.topk;
    // The routed regions, each once: a caller-given row may repeat a region,
    // and attention runs over the union of the routed regions' tokens.
    if (tid == 0) {
        bad = 0;
        nroutes = 0;
        for (int w = 0; w < kMaxRegions / 32; ++w) seen[w] = 0;
        for (int m = 0; m < g.topk; ++m) {
            const int rr = row[m];
            if (rr < 0 || rr >= g.R) {
                bad = 1;
                break;
            }
            if (!((seen[rr >> 5] >> (rr & 31)) & 1u)) {
                seen[rr >> 5] |= 1u << (rr & 31);
                routes[nroutes++] = rr;
            }
        }
    }
    __syncthreads();
    if (bad) {
        if (tid == 0) raise_status(status, kDevBadRoute);
        return;
    }

    const int qi = tid / plan.group, sub = tid % plan.group;
    const int t = chunk_id * plan.chunk + qi;
    const bool active = qi < plan.chunk && t < g.n;
    const size_t qoff = active ? token_offset(g, b, r, t) + (size_t)h * D : 0;

    // q pre-scaled so that exp2(q.k) = exp(q.k / sqrt(D)).
    float qv[D];
    const float qscale = 1.4426950408889634f / sqrtf((float)D);
#pragma unroll
    for (int c = 0; c < NV; ++c) {
        uint4 u = make_uint4(0, 0, 0, 0);
        if (active) u = __ldg(reinterpret_cast<const uint4*>(q + qoff) + c);
        unpack16(u, qv + c * VEC, q);
    }
#pragma unroll
    for (int c = 0; c < D; ++c) qv[c] *= qscale;

    float mx = -INFINITY, l = 0.f, acc[D];
#pragma unroll
    for (int c = 0; c < D; ++c) acc[c] = 0.f;

    const int kn = nroutes * g.n;
    for (int j0 = 0; j0 < kn; j0 += kSimtKeyBlock) {
        const int nb = min(kSimtKeyBlock, kn - j0);
        __syncthreads();
        for (int e = tid; e < nb * NV; e += kSimtThreads) {
            const int jj = e / NV, cv = e - jj * NV;
            const int j = j0 + jj, m = j / g.n, tt = j - m * g.n;
            const size_t off = token_offset(g, b, routes[m], tt) + (size_t)h * D + cv * VEC;
            float fk[VEC], fv[VEC];
            unpack16(__ldg(reinterpret_cast<const uint4*>(k + off)), fk, k);
            unpack16(__ldg(reinterpret_cast<const uint4*>(v + off)), fv, v);
#pragma unroll
            for (int i = 0; i < VEC; ++i) {
                ks[jj][cv * VEC + i] = fk[i];
                vs[jj][cv * VEC + i] = fv[i];
            }
        }
        __syncthreads();
        if (active) {
            for (int jj = sub; jj < nb; jj += plan.group) {
                float s = 0.f;
#pragma unroll
                for (int c = 0; c < D; ++c) s = fmaf(qv[c], ks[jj][c], s);
                if (s > mx) {
                    const float corr = exp2f(mx - s);
                    l *= corr;
#pragma unroll
                    for (int c = 0; c < D; ++c) acc[c] *= corr;
                    mx = s;
                }
                const float p = exp2f(s - mx);
                l += p;
#pragma unroll
                for (int c = 0; c < D; ++c) acc[c] = fmaf(p, vs[jj][c], acc[c]);
            }
        }
    }

    // Merge the partial softmax states of the lanes that share a query.
    for (int off = plan.group >> 1; off > 0; off >>= 1) {
        const float m2 = __shfl_xor_sync(0xffffffffu, mx, off);
        const float l2 = __shfl_xor_sync(0xffffffffu, l, off);
        const float mn = fmaxf(mx, m2);
        const float c1 = (mx == -INFINITY) ? 0.f : exp2f(mx - mn);
        const float c2 = (m2 == -INFINITY) ? 0.f : exp2f(m2 - mn);
        l = l * c1 + l2 * c2;
#pragma unroll
        for (int c = 0; c < D; ++c) {
            const float a2 = __shfl_xor_sync(0xffffffffu, acc[c], off);
            acc[c] = acc[c] * c1 + a2 * c2;
        }
        mx = mn;
    }
    if (active && sub == 0) {
        const float inv = 1.f / l;
        T* out = o + qoff;
        if (in_bounds(qoff + D - 1, map_elems(g), status)) {
#pragma unroll
            for (int c = 0; c < D; ++c) out[c] = from_f32<T>(acc[c] * inv);
        }
    }
}

SimtPlan simt_plan(const Geometry& g) {
    SimtPlan p;
    p.chunk = g.n < kSimtThreads ? g.n : kSimtThreads;
    p.group = 1;
    while (p.group < 32 && p.chunk * p.group * 2 <= kSimtThreads) p.group *= 2;
    p.chunks = (g.n + p.chunk - 1) / p.chunk;
    return p;
}

cudaError_t launch_attend_simt(bool bf16, const void* q, const void* k, const void* v,
                               const int32_t* idx, void* o, const Geometry& g, int* status,
                               cudaStream_t stream) {
    const SimtPlan p = simt_plan(g);
    const dim3 grid(g.R * p.chunks, g.heads, g.B);
    if (bf16)
        bra_attend_simt_kernel<__nv_bfloat16, 32><<<grid, kSimtThreads, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
            static_cast<const __nv_bfloat16*>(v), idx, static_cast<__nv_bfloat16*>(o), g, p, status);
    else
        bra_attend_simt_kernel<float, 32><<<grid, kSimtThreads, 0, stream>>>(
            static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
            idx, static_cast<float*>(o), g, p, status);
    return cudaGetLastError();
}

}  // namespace bra
