// Token attention for small regions with one (batch, head) slice's keys and
// values resident in shared memory, on warp-level tensor-core MMAs (blog
// "BiFormer Reshapes Visual Attention with Bi-Level Routing", Part 2 section
// 2.2, step 4: gather the routed key-value regions, then token attention
// over their union).
//
// Why this form for BiFormer's stage 2 (28 x 28 map, 49 regions of 4 x 4
// tokens, 4 routes, head dim 32).  Every query region attends to its own 64
// keys, scattered over the slice 16 at a time.  A tcgen05 product is at least
// 64 rows and costs about 26 ns to issue even when small, and its operands
// must sit at a uniform stride in shared memory, so that form needs either a
// copy of the routed keys per tile or several hundred small products per
// slice.  A warp-level m16n8k16 product instead takes its operand rows from
// per-lane addresses (ldmatrix), so the gather is free: each warp takes one
// 16-query chunk of a region, reads the routed regions' K and V rows in place
// from the resident slice, keeps S, the softmax and P in registers (the
// accumulator layout of S is the operand layout of P), and writes O.  Each
// slice's K and V cross the load path once; Q is read once (straight into
// registers) and O written once.  Two CTAs share an SM, so one's slice load
// overlaps the other's arithmetic.
//
// Work: one CTA per slice (grid = B * heads); 12 warps take the slice's
// (region, 16-query chunk) items in turn.  The slice's K and V arrive as one
// 4-D TMA box per region each (64-byte rows, 64-byte swizzle, region r at
// byte r * n * 64), completion on one mbarrier (bounded wait; on expiry the
// CTA records kDevTimeout and writes nothing).  Routes: a region listed more
// than once counts once (later listings are masked), and a query region with
// an out-of-range route is reported (BRA_ERR_BAD_ROUTE) and not written.
#include <cuda.h>
#include <stdlib.h>

#include "attend_tc.h"
#include "kernels.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace bra {
namespace {

constexpr int kWarps = 12;
constexpr int kThreads = 32 * kWarps;
constexpr uint32_t kWait = 1u << 22;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kMaxSliceBytes = 2u * 50u * 1024u;  // K + V: two CTAs per SM

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// D += A B for one m16n8k16 tile (bf16 in, fp32 accumulate).
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Byte address of 16-byte chunk c (0..3) of row ``row`` of a slice buffer
// written by TMA with the 64-byte swizzle (chunk index XOR bits 7-8 of the
// row's byte offset).
__device__ __forceinline__ uint32_t swz64(uint32_t base, int row, int c) {
    return base + (uint32_t)row * 64u + (uint32_t)((c ^ ((row >> 1) & 3)) << 4);
}

// KN: keys per query region (topk * n), a multiple of 16, at most 128.
template <int KN>
__global__ void __launch_bounds__(kThreads, 2)
bra_attend_warp_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                       const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ idx,
                       __nv_bfloat16* __restrict__ o, Geometry g, int* status) {
    constexpr int NT = KN / 8;  // 8-key column tiles of S
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t region_bytes = (uint32_t)g.n * 64u;
    const uint32_t slice_bytes = (uint32_t)g.R * region_bytes;
    const uint32_t k_base = ptx::smem_addr(smem), v_base = k_base + slice_bytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + 2 * slice_bytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x, b = bh / g.heads, hd = bh - b * g.heads;

    if (threadIdx.x == 0) {
        ptx::mbar_init(full, 1);
        ptx::mbar_init_fence();
    }
    __syncthreads();
    grid_dependency_wait();
    if (warp == 0) {
        if (lane == 0) {
            ptx::tma_prefetch_desc(&tk);
            ptx::tma_prefetch_desc(&tv);
            ptx::mbar_arrive_expect_tx(full, 2u * slice_bytes);
        }
        __syncwarp();
        for (int j = lane; j < 2 * g.R; j += 32) {
            const int r = j >> 1, ri = r / g.S, rj = r - ri * g.S;
            const bool is_v = j & 1;
            ptx::tma_load_4d((is_v ? v_base : k_base) + (uint32_t)r * region_bytes,
                             is_v ? (const void*)&tv : (const void*)&tk, hd * 32, rj * g.ws, ri * g.hs, b, full);
        }
    }

    const int gq = lane >> 2, tq = lane & 3;  // fragment row group and column pair
    const float sl = kLog2e * rsqrtf(32.f);
    const int chunks = g.n / 16;              // 16-query chunks per region
    const int items = g.R * chunks;
    const int32_t* routes = idx + (size_t)bh * g.R * g.topk;
    bool landed = false;
    for (int it = warp; it < items; it += kWarps) {
        const int r = it / chunks, ch = it - r * chunks;
        // routes of region r: lane m < topk holds route m; live: in range and
        // its first listing; any route out of range skips the region
        const int my_r = lane < g.topk ? __ldg(routes + r * g.topk + lane) : 0;
        const uint32_t badm = __ballot_sync(0xffffffffu, lane < g.topk && (my_r < 0 || my_r >= g.R));
        if (badm) {
            if (lane == 0) raise_status(status, kDevBadRoute);
            continue;
        }
        bool dup = false;
        for (int dd = 1; dd < g.topk; ++dd) {
            const int other = __shfl_up_sync(0xffffffffu, my_r, dd);
            if (dd <= lane && other == my_r) dup = true;
        }
        const uint32_t live = __ballot_sync(0xffffffffu, lane < g.topk && !dup);
        const int my_base = my_r * g.n;  // first slice row of route ``lane``
        // this chunk's 16 query tokens: rows t0 + gq and t0 + gq + 8 of the region
        const int t0 = ch * 16;
        const size_t orow0 = token_offset(g, b, r, t0 + gq) + (size_t)hd * 32;
        const size_t orow1 = token_offset(g, b, r, t0 + gq + 8) + (size_t)hd * 32;
        uint32_t qa[2][4];
#pragma unroll
        for (int kc = 0; kc < 2; ++kc) {
            const int c0 = 16 * kc + 2 * tq;
            qa[kc][0] = __ldg(reinterpret_cast<const uint32_t*>(q + orow0 + c0));
            qa[kc][1] = __ldg(reinterpret_cast<const uint32_t*>(q + orow1 + c0));
            qa[kc][2] = __ldg(reinterpret_cast<const uint32_t*>(q + orow0 + c0 + 8));
            qa[kc][3] = __ldg(reinterpret_cast<const uint32_t*>(q + orow1 + c0 + 8));
        }
        if (!landed) {
            if (!ptx::mbar_wait(full, 0, kWait)) {
                if (lane == 0) raise_status(status, kDevTimeout);
                break;
            }
            landed = true;
        }
        // S = Q K^T over the routed keys: column tile j is keys 8j..8j+7 of the
        // stacked list (route j*8/n, key (8j) % n of that region)
        float s[NT][4];
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
            const int m = (8 * j) / g.n;  // route of the tile (the same for every lane)
            const int base = __shfl_sync(0xffffffffu, my_base, m < 32 ? m : 0);
            if (8 * j >= g.topk * g.n) continue;
            const int row = base + (8 * j) % g.n + (lane & 7);
            uint32_t b0, b1, b2, b3;
            ldsm_x4(swz64(k_base, row, lane >> 3), b0, b1, b2, b3);
            mma16816(s[j], qa[0][0], qa[0][1], qa[0][2], qa[0][3], b0, b1);
            mma16816(s[j], qa[1][0], qa[1][1], qa[1][2], qa[1][3], b2, b3);
        }
        // masked base-2 softmax over each row (rows gq and gq + 8; a row's 16
        // values of a tile sit in the 4 lanes of its group)
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const int m = (8 * j) / g.n;
            const bool on = 8 * j < g.topk * g.n && ((live >> m) & 1u);
            if (!on) s[j][0] = s[j][1] = s[j][2] = s[j][3] = -INFINITY;
            mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
            mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float m0 = mx0 * sl, m1 = mx1 * sl;
        // P as bf16 pairs (the A operand of P V), and the row sums of those bf16 values
        uint32_t pa[NT][2];
        float l0 = 0.f, l1 = 0.f;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            pa[j][0] = ptx::pack_bf16x2(ptx::ex2(fmaf(s[j][0], sl, -m0)), ptx::ex2(fmaf(s[j][1], sl, -m0)));
            pa[j][1] = ptx::pack_bf16x2(ptx::ex2(fmaf(s[j][2], sl, -m1)), ptx::ex2(fmaf(s[j][3], sl, -m1)));
            l0 += __uint_as_float(pa[j][0] << 16) + __uint_as_float(pa[j][0] & 0xffff0000u);
            l1 += __uint_as_float(pa[j][1] << 16) + __uint_as_float(pa[j][1] & 0xffff0000u);
        }
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        // O = P V: 16 keys per step (tiles 2k, 2k + 1 of P), V rows of the routed
        // region read transposed by ldmatrix; 4 tiles of 8 channels
        float acc[4][4];
#pragma unroll
        for (int n = 0; n < 4; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < NT / 2; ++kk) {
            const int m = (16 * kk) / g.n;
            const int base = __shfl_sync(0xffffffffu, my_base, m < 32 ? m : 0);
            if (16 * kk >= g.topk * g.n) continue;
            // matrices: (keys 0-7, ch c..c+7), (keys 8-15, ch c..), (keys 0-7, ch c+8..), (keys 8-15, ch c+8..)
            const int row = base + (16 * kk) % g.n + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(swz64(v_base, row, 2 * half + (lane >> 4)), b0, b1, b2, b3);
                mma16816(acc[2 * half], pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1], b0, b1);
                mma16816(acc[2 * half + 1], pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1], b2,
                         b3);
            }
        }
        // O rows gq and gq + 8: channels 8n + 2tq, 8n + 2tq + 1
        const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
        if (!in_bounds((orow0 > orow1 ? orow0 : orow1) + 31, map_elems(g), status)) continue;
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            const int c = 8 * n + 2 * tq;
            __stcs(reinterpret_cast<uint32_t*>(o + orow0 + c), ptx::pack_bf16x2(acc[n][0] * i0, acc[n][1] * i0));
            __stcs(reinterpret_cast<uint32_t*>(o + orow1 + c), ptx::pack_bf16x2(acc[n][2] * i1, acc[n][3] * i1));
        }
    }
    // every copy this CTA issued must land before it exits
    if (!landed && warp == 0 && lane == 0) ptx::mbar_wait(full, 0, kWait);
    __syncthreads();
}

}  // namespace

bool attend_warp_covers(const Geometry& g) {
    const int kn = g.topk * g.n;
    return g.d == 32 && g.n % 16 == 0 && kn <= 128 && (kn == 32 || kn == 64 || kn == 128) &&
           2u * (uint32_t)g.R * (uint32_t)g.n * 64u <= kMaxSliceBytes;
}

bra_status attend_warp_launch(const Geometry& g, const void* q, const void* k, const void* v, const int32_t* idx,
                              void* o, int* status, cudaStream_t stream) {
    if (!attend_warp_covers(g)) return BRA_ERR_UNSUPPORTED;
    CUtensorMap tk, tv;
    if (!encode_region_map(&tk, k, g.B, g.H, g.W, g.C, g.ws, g.hs, 32) ||
        !encode_region_map(&tv, v, g.B, g.H, g.W, g.C, g.ws, g.hs, 32))
        return BRA_ERR_UNSUPPORTED;
    const long long slices = (long long)g.B * g.heads;
    if (slices > 0x7fffffffLL) return BRA_ERR_UNSUPPORTED;
    const uint32_t smem = 2u * (uint32_t)g.R * (uint32_t)g.n * 64u + 64u + 1024u;
    using KernelFn = void (*)(CUtensorMap, CUtensorMap, const __nv_bfloat16*, const int32_t*, __nv_bfloat16*, Geometry,
                              int*);
    const int kn = g.topk * g.n;
    const KernelFn kernel = kn == 32 ? bra_attend_warp_kernel<32>
                                     : (kn == 64 ? bra_attend_warp_kernel<64> : bra_attend_warp_kernel<128>);
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return BRA_ERR_CUDA;
    const cudaError_t e = launch_after_previous(kernel, dim3((unsigned)slices), dim3(kThreads), smem, stream, tk, tv,
                                                static_cast<const __nv_bfloat16*>(q), idx,
                                                static_cast<__nv_bfloat16*>(o), g, status);
    return e == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

}  // namespace bra
