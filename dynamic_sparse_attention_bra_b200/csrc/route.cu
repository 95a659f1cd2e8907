// Region-level routing kernels (blog "BiFormer Reshapes Visual Attention with
// Bi-Level Routing", Part 2 section 2.2, step 3):
//   bra_pool_warp_kernel / bra_pool_kernel
//                     Q^r, K^r = per-region means of Q and K (fp32)
//   bra_route_kernel  A^r = Q^r (K^r)^T in fp32, then row-wise top-k -> I^r
#include "common.cuh"
#include "kernels.h"
#include "tma_host.h"

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
// Pool, warp form: one warp per (tensor, batch, region).  Row ty of region
// (ri, rj) is one contiguous run of ws * C elements, i.e. RC = ws * CG
// 16-byte vectors with CG = C / VEC vectors per token.  Vector e of the
// region (row e / RC, vector e % RC of the row) holds channel group e % CG,
// and lane l takes e = l, l + 32, ... .  When CG divides 32 the lane's channel
// group is always l % CG (NACC = 1) and the lanes sharing a group meet by
// butterfly shuffles; when 32 divides CG the lane cycles through NACC = CG / 32
// groups l + 32 a.  A lane issues 4 loads before it sums any of them, and a
// CTA of 4 warps holds 4 regions; twelve CTAs fit an SM, so the whole of Q
// and K of the common shapes streams through in one wave, many 16-byte loads
// in flight per SM.
// HBM traffic: Q and K read once, means written (2 * B*heads*R*d floats).
// ---------------------------------------------------------------------------
template <typename T, int NACC>
__global__ void __launch_bounds__(kPoolWarpThreads, NACC == 1 ? 12 : 6)
bra_pool_warp_kernel(const T* __restrict__ q, const T* __restrict__ k, float* __restrict__ qr,
                     float* __restrict__ kr, Geometry g) {
    constexpr int VEC = 16 / sizeof(T);
    constexpr int kUnroll = 4;
    const int lane = threadIdx.x & 31;
    const int unit = blockIdx.x * (kPoolWarpThreads / 32) + (threadIdx.x >> 5);
    if (unit >= 2 * g.B * g.R) return;
    // unit = (which * B + b) * R + r: neighbouring warps read neighbouring runs
    const int r = unit % g.R;
    const int b = (unit / g.R) % g.B;
    const int which = unit / (g.R * g.B);
    const int ri = r / g.S, rj = r - ri * g.S;
    const int CG = g.C / VEC;
    const int RC = g.ws * CG;
    const int total = g.hs * RC;
    const T* src = (which ? k : q) + (((size_t)b * g.H + (size_t)ri * g.hs) * g.W + (size_t)rj * g.ws) * g.C;
    // Running position of vector e = lane + 32 i: its column ci in its row and
    // its address; stepping 32 vectors may cross one or more row ends.
    const size_t wrap = (size_t)g.W * g.C - (size_t)RC * VEC;  // a row's end -> the next row's start
    int ci = lane % RC;
    const T* ptr = src + (size_t)(lane / RC) * g.W * g.C + (size_t)ci * VEC;

    float acc[NACC][VEC];
#pragma unroll
    for (int a = 0; a < NACC; ++a)
#pragma unroll
        for (int i = 0; i < VEC; ++i) acc[a][i] = 0.f;

    for (int e0 = lane; e0 < total; e0 += 32 * kUnroll) {
        uint4 u[kUnroll];
#pragma unroll
        for (int uu = 0; uu < kUnroll; ++uu) {
            u[uu] = make_uint4(0, 0, 0, 0);  // +0 adds nothing to the sums
            if (e0 + 32 * uu < total) u[uu] = __ldg(reinterpret_cast<const uint4*>(ptr));
            ci += 32;
            ptr += 32 * VEC;
            while (ci >= RC) {
                ci -= RC;
                ptr += wrap;
            }
        }
#pragma unroll
        for (int uu = 0; uu < kUnroll; ++uu) {
            float f[VEC];
            unpack16(u[uu], f, src);
            // (e0 - lane) / 32 is a multiple of kUnroll, itself a multiple of NACC
#pragma unroll
            for (int i = 0; i < VEC; ++i) acc[uu % NACC][i] += f[i];
        }
    }
    if (NACC == 1) {
        for (int off = 16; off >= CG; off >>= 1)
#pragma unroll
            for (int i = 0; i < VEC; ++i) acc[0][i] += __shfl_xor_sync(0xffffffffu, acc[0][i], off);
    }
    allow_dependents();  // the route kernel may launch; it waits for this grid's writes
    const float inv_n = 1.f / (float)g.n;
    float* out = which ? kr : qr;
#pragma unroll
    for (int a = 0; a < NACC; ++a) {
        const int cg = lane + 32 * a;
        if (cg >= CG) continue;
        const int c = cg * VEC, h = c / g.d, i0 = c - h * g.d;  // VEC divides d: one head
        float4* dst = reinterpret_cast<float4*>(out + (((size_t)b * g.heads + h) * g.R + r) * g.d + i0);
#pragma unroll
        for (int i = 0; i < VEC; i += 4)
            dst[i / 4] = make_float4(acc[a][i] * inv_n, acc[a][i + 1] * inv_n, acc[a][i + 2] * inv_n,
                                     acc[a][i + 3] * inv_n);
    }
}

// ---------------------------------------------------------------------------
// Route: a CTA owns rows [row0, row0 + rows) of one (batch, head) slice.  It
// stages all of K^r of the slice and its own rows of Q^r in shared memory
// with one batch of loads (one round trip to L2), rows padded to d + 4 floats
// so that 8 lanes reading 8 different K^r rows cover all 32 banks.  A warp
// owns one row r at a time: lane l computes A[r][j] for j = l + 32 e,
// e < E (fp32, channels in order).  I^r[r] lists the topk columns first
// under the key (value descending, index ascending): each score becomes an
// order-preserving 32-bit key (larger float, larger key; -0 counts as +0 and
// a non-finite score as -inf so that the order is total), and each of topk
// rounds takes the warp maximum with one redux and the lowest column holding
// it with one ballot per slot e (all of slot e's columns precede slot e + 1's).
// A taken or padding column gets key 0, below the key of -inf.
// A^r never reaches global memory.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t route_key(float s) {
    if (!isfinite(s)) s = -INFINITY;
    const uint32_t u = __float_as_uint(s + 0.f);  // -0 + 0 = +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

template <int E>
__global__ void __launch_bounds__(kRouteThreads, 4)
bra_route_kernel(const float* __restrict__ qr, const float* __restrict__ kr,
                 int32_t* __restrict__ idx, Geometry g, int rows_per_cta) {
    constexpr int D = 32;      // head dim (checked on the host)
    constexpr int LD = D + 4;  // padded row: 16-byte aligned, 8 lanes hit 32 banks
    constexpr int kWarps = kRouteThreads / 32;
    extern __shared__ float4 route_smem4[];  // [R][LD] K^r of the slice, [rows][LD] this CTA's Q^r rows
    float* sk = reinterpret_cast<float*>(route_smem4);
    const int R = g.R;
    const size_t bh = blockIdx.x;
    const int row0 = blockIdx.y * rows_per_cta;
    const int rows = min(rows_per_cta, R - row0);
    float* sq = sk + (size_t)R * LD;
    grid_dependency_wait();  // the pool kernel's means are complete and visible
    allow_dependents();      // the attention kernel may start its set-up
    const float4* gk = reinterpret_cast<const float4*>(kr + bh * R * D);
    const float4* gq = reinterpret_cast<const float4*>(qr + (bh * R + row0) * D);
    const int nk = R * (D / 4), nall = (R + rows) * (D / 4);
    for (int e0 = threadIdx.x; e0 < nall; e0 += 4 * kRouteThreads) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = e0 + u * kRouteThreads;
            if (e < nall) v[u] = __ldg(e < nk ? gk + e : gq + (e - nk));
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int e = e0 + u * kRouteThreads;
            if (e < nall) *reinterpret_cast<float4*>(sk + (e / (D / 4)) * LD + (e % (D / 4)) * 4) = v[u];
        }
    }
    __syncthreads();

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int rr = warp; rr < rows; rr += kWarps) {
        const int r = row0 + rr;
        const float* qrow = sq + rr * LD;  // the same 128 bytes for every lane: broadcast reads
        uint32_t key[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            key[e] = 0u;
            const int jcol = lane + 32 * e;
            if (jcol < R) {
                const float* krow = sk + jcol * LD;
                float s = 0.f;
#pragma unroll
                for (int c = 0; c < D / 4; ++c) {
                    const float4 k4 = *reinterpret_cast<const float4*>(krow + 4 * c);
                    const float4 q4 = *reinterpret_cast<const float4*>(qrow + 4 * c);
                    s = fmaf(q4.x, k4.x, s);
                    s = fmaf(q4.y, k4.y, s);
                    s = fmaf(q4.z, k4.z, s);
                    s = fmaf(q4.w, k4.w, s);
                }
                key[e] = route_key(s);
            }
        }
        int32_t* out = idx + (bh * R + r) * g.topk;
        for (int m = 0; m < g.topk; ++m) {
            uint32_t best = key[0];
#pragma unroll
            for (int e = 1; e < E; ++e) best = max(best, key[e]);
            const uint32_t top = __reduce_max_sync(0xffffffffu, best);
            int win = 0;
#pragma unroll
            for (int e = E - 1; e >= 0; --e) {
                const uint32_t hit = __ballot_sync(0xffffffffu, key[e] == top);
                if (hit) win = 32 * e + __ffs(hit) - 1;  // the lowest slot with a hit wins
            }
#pragma unroll
            for (int e = 0; e < E; ++e)
                if (win == lane + 32 * e) key[e] = 0u;
            if (lane == 0) out[m] = win;
        }
    }
}

namespace {

template <typename T>
cudaError_t launch_pool_t(const T* q, const T* k, float* qr, float* kr, const Geometry& g,
                          cudaStream_t stream) {
    constexpr int VEC = 16 / sizeof(T);
    const int cg = g.C / VEC;
    const int units = 2 * g.B * g.R;
    const dim3 grid((units + kPoolWarpThreads / 32 - 1) / (kPoolWarpThreads / 32));
    if (units == 0) return cudaSuccess;
    // Warp form whenever a token's 16-byte vectors tile a warp evenly.
    if (32 % cg == 0)
        bra_pool_warp_kernel<T, 1><<<grid, kPoolWarpThreads, 0, stream>>>(q, k, qr, kr, g);
    else if (cg == 64)
        bra_pool_warp_kernel<T, 2><<<grid, kPoolWarpThreads, 0, stream>>>(q, k, qr, kr, g);
    else if (cg == 128)
        bra_pool_warp_kernel<T, 4><<<grid, kPoolWarpThreads, 0, stream>>>(q, k, qr, kr, g);
    else {
        const int sp = kPoolThreads / cg;
        const size_t smem = (size_t)2 * sp * g.C * sizeof(float);
        bra_pool_kernel<T><<<dim3(g.R, g.B), kPoolThreads, smem, stream>>>(q, k, qr, kr, g);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool(bool bf16, const void* q, const void* k, float* qr, float* kr,
                        const Geometry& g, cudaStream_t stream) {
    if (bf16)
        return launch_pool_t(static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k), qr,
                             kr, g, stream);
    return launch_pool_t(static_cast<const float*>(q), static_cast<const float*>(k), qr, kr, g, stream);
}

namespace {

int route_rows_per_cta(const Geometry& g, int sms) {
    // Enough CTAs for about two per SM, each with at least one row per warp.
    const long long slices = (long long)g.B * g.heads;
    if (slices <= 0) return g.R;
    long long target = ((long long)g.R * slices + 2LL * sms - 1) / (2LL * sms);
    if (target < kRouteThreads / 32) target = kRouteThreads / 32;
    if (target > g.R) target = g.R;
    const int blocks = (int)((g.R + target - 1) / target);
    return (g.R + blocks - 1) / blocks;  // balanced: row blocks differ by at most one row
}

}  // namespace

cudaError_t launch_route(const float* qr, const float* kr, int32_t* idx, const Geometry& g,
                         cudaStream_t stream) {
    if ((long long)g.B * g.heads == 0) return cudaSuccess;
    const int sms = sm_count();
    const int rows = route_rows_per_cta(g, sms > 0 ? sms : 148);
    const size_t smem = (size_t)(g.R + rows) * (32 + 4) * sizeof(float);
    const int e = (g.R + 31) / 32;  // columns per lane, R <= kMaxRegions
    void (*kernel)(const float*, const float*, int32_t*, Geometry, int) =
        e == 1 ? bra_route_kernel<1> : e == 2 ? bra_route_kernel<2> : e <= 4 ? bra_route_kernel<4>
                                                                             : bra_route_kernel<8>;
    static_assert(kMaxRegions <= 8 * 32, "route kernel covers at most 8 columns per lane");
    if (smem > 48 * 1024) {
        const cudaError_t err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
    }
    const dim3 grid(g.B * g.heads, (g.R + rows - 1) / rows);
    return launch_after_previous(kernel, grid, dim3(kRouteThreads), smem, stream, qr, kr, idx, g, rows);
}

}  // namespace bra
