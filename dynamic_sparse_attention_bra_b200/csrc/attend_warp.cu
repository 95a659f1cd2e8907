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
// slice's K and V cross the load path once per CTA that works on it; Q is
// read once (straight into registers) and O written once.
//
// Work: persistent, one CTA per SM.  All (slice, region, 16-query chunk)
// items are split into equal contiguous ranges, one per CTA (a CTA's range
// spans two or three slices on stage 2), so no SM gets a whole extra slice.
// A producer warp loads the slices of the CTA's range into a two-buffer ring,
// so the next slice lands while the compute warps work on the current one;
// the compute warps take the range's items in turn and release a buffer once
// done with its slice.  A slice's K (and its V) is one 5-D TMA box: the map
// viewed as (channel, x in region, y in region, region column, image x region
// row) lands region-major, region r's n tokens in 64-byte rows r * n .. r * n
// + n - 1 (64-byte swizzle).  Routed regions then start at multiples of 16
// rows, so each lane's ldmatrix addresses are its route's base plus constants
// (the swizzle included) and the per-tile offsets are compile-time constants
// of the region size.
// Every wait is bounded (on expiry: kDevTimeout, all roles stop, copies in
// flight are waited for).  Routes: a region listed more than once counts
// once (later listings are masked), and a query region with an out-of-range
// route is reported (BRA_ERR_BAD_ROUTE) and not written.
#include <cuda.h>
#include <stdlib.h>

#include "attend_tc.h"
#include "kernels.h"
#include "tc_ptx.cuh"
#include "tma_host.h"
#include "warp_mma.cuh"

namespace bra {
namespace {

// Compute warps per CTA (one CTA per SM), one more warp being the producer:
// 19 for up to 64 keys per query, 12 for 128 (a warp's S row block needs
// more registers).
constexpr int compute_warps_for(int kn) { return kn <= 64 ? 19 : 12; }
constexpr uint32_t kMaxSliceBytes = 55u * 1024u;  // K or V of one slice; two slices of K + V resident

constexpr uint32_t kWait = 1u << 22;
constexpr float kLog2e = 1.4426950408889634f;

using wmma16::ldsm_x4;
using wmma16::ldsm_x4_t;
using wmma16::mma16816;

// Byte address of 16-byte chunk c (0..3) of row ``row`` of a slice buffer
// written by TMA with the 64-byte swizzle (chunk index XOR bits 7-8 of the
// row's byte offset).
__device__ __forceinline__ uint32_t swz64(uint32_t base, int row, int c) {
    return base + (uint32_t)row * 64u + (uint32_t)((c ^ ((row >> 1) & 3)) << 4);
}

struct RingBarriers {
    uint64_t full[2];   // slice buffer b holds its slice (TMA bytes landed)
    uint64_t empty[2];  // every compute warp is done with slice buffer b
    int issued;         // slices whose loads the producer has issued
    int abort;
};

__device__ __forceinline__ bool ring_aborted(RingBarriers* rb) {
    return *reinterpret_cast<volatile int*>(&rb->abort) != 0;
}
__device__ __forceinline__ bool ring_wait(uint64_t* bar, uint32_t parity, RingBarriers* rb, int* status) {
    for (uint32_t i = 0; i < kWait; ++i) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 63u && ring_aborted(rb)) return false;
    }
    raise_status(status, kDevTimeout);
    *reinterpret_cast<volatile int*>(&rb->abort) = 1;
    return false;
}

// KN: keys per query region (topk * n); N: tokens per region (a power of two,
// 16..KN).  Both are template parameters so that the route and in-region
// offset of every 8-key tile of S and every 16-key step of P V are constants.
// Registers per thread: the most that lets one CTA of compute_warps_for(KN) + 1
// warps fit (warps are spread over the SM's four 16 K-register files: 20
// warps put 5 on each, 5 x 32 x 96 <= 16 K; 13 warps put 4 on one, 4 x 32 x 128).
constexpr int max_regs_for(int kn) { return kn <= 64 ? 96 : 128; }

template <int KN, int N>
__global__ void __maxnreg__(max_regs_for(KN))
bra_attend_warp_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                       const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ idx,
                       __nv_bfloat16* __restrict__ o, Geometry g, int* status) {
    constexpr int NT = KN / 8;     // 8-key column tiles of S
    constexpr int TOPK = KN / N;   // routes per query region
    constexpr int CHUNKS = N / 16; // 16-query chunks per region
    constexpr int kCompute = compute_warps_for(KN);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t slice_bytes = (uint32_t)g.R * (uint32_t)N * 64u;
    const uint32_t ring_base = ptx::smem_addr(smem);  // buffer b: K at ring_base + b * 2 * slice_bytes, then V
    RingBarriers* rb = reinterpret_cast<RingBarriers*>(smem + 4 * slice_bytes);
    int* qcorner = reinterpret_cast<int*>(smem + 4 * slice_bytes + ((sizeof(RingBarriers) + 15) & ~size_t(15)));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int lg_ws = __ffs(g.ws) - 1;
    const int per_slice = g.R * CHUNKS;
    // this CTA's contiguous share of all (slice, region, chunk) items (the
    // host checks that their number fits an int)
    const long long total = (long long)g.B * g.heads * per_slice;
    const int lo = (int)(total * blockIdx.x / gridDim.x), hi = (int)(total * (blockIdx.x + 1) / gridDim.x);
    const int s_first = lo / per_slice;
    const int n_slices = hi > lo ? (hi - 1) / per_slice - s_first + 1 : 0;

    // map offset of each query region's token (0, 0)
    for (int r = threadIdx.x; r < g.R; r += blockDim.x) {
        const int ri = r / g.S;
        qcorner[r] = ri * g.hs * g.W + (r - ri * g.S) * g.ws;
    }
    if (threadIdx.x == 0) {
        ptx::mbar_init(&rb->full[0], 1);
        ptx::mbar_init(&rb->full[1], 1);
        ptx::mbar_init(&rb->empty[0], kCompute);
        ptx::mbar_init(&rb->empty[1], kCompute);
        rb->abort = 0;
        rb->issued = 0;
        ptx::mbar_init_fence();
    }
    __syncthreads();
    grid_dependency_wait();

    if (warp == kCompute) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            ptx::tma_prefetch_desc(&tk);
            ptx::tma_prefetch_desc(&tv);
        }
        for (int k = 0; k < n_slices; ++k) {
            const int buf = k & 1;
            if (k >= 2 && !ring_wait(&rb->empty[buf], ((k - 2) >> 1) & 1, rb, status)) break;
            const int bh = s_first + k, b = bh / g.heads, hd = bh - b * g.heads;
            const uint32_t k_base = ring_base + (uint32_t)buf * 2u * slice_bytes, v_base = k_base + slice_bytes;
            // one head of every region of the image, region-major: region r's
            // tokens are buffer rows r * N .. r * N + N - 1 in their in-region order
            if (lane == 0) {
                ptx::mbar_arrive_expect_tx(&rb->full[buf], 2u * slice_bytes);
                ptx::tma_load_5d(k_base, &tk, hd * 32, 0, 0, 0, b * g.S, &rb->full[buf]);
                ptx::tma_load_5d(v_base, &tv, hd * 32, 0, 0, 0, b * g.S, &rb->full[buf]);
                rb->issued = k + 1;
            }
            __syncwarp();
        }
    } else {
        // --------------------------------------------------------- compute warps
        const int gq = lane >> 2, tq = lane & 3;  // fragment row group and column pair
        const float sl = kLog2e * rsqrtf(32.f);
        constexpr uint32_t kOnes = 0x3f803f80u;   // a bf16 pair of ones: the B operand of the row sums
        // Shared-memory byte offsets of this lane's ldmatrix rows.  A routed
        // region starts at a multiple of 16 rows and every tile or step at a
        // multiple of 8 rows inside it, so the 64-byte swizzle (chunk XOR bits
        // 1-2 of the row) depends on the lane alone.
        const int kl = lane & 7, vrow = kl + ((lane >> 3) & 1) * 8;
        const uint32_t s_lane = (uint32_t)kl * 64u + ((uint32_t)((lane >> 3) ^ ((kl >> 1) & 3)) << 4);
        const uint32_t v_lane0 = (uint32_t)vrow * 64u + ((uint32_t)((0 + (lane >> 4)) ^ ((kl >> 1) & 3)) << 4);
        const uint32_t v_lane1 = (uint32_t)vrow * 64u + ((uint32_t)((2 + (lane >> 4)) ^ ((kl >> 1) & 3)) << 4);
        int it = lo + warp;  // items lo + warp, lo + warp + kCompute, ...
        for (int k = 0; k < n_slices; ++k) {
            const int buf = k & 1;
            const int bh = s_first + k, b = bh / g.heads, hd = bh - b * g.heads;
            const int s_end = hi < (bh + 1) * per_slice ? hi : (bh + 1) * per_slice;
            const uint32_t k_base = ring_base + (uint32_t)buf * 2u * slice_bytes;
            const int32_t* routes = idx + (size_t)bh * g.R * TOPK;
            const size_t img = (size_t)b * g.H * g.W;
            bool landed = false, stop = false;
            for (; it < s_end; it += kCompute) {
                const int item = it - bh * per_slice;
                const int r = item / CHUNKS, ch = item - r * CHUNKS;
                // routes of region r: lane m < topk holds route m; live: in range and
                // its first listing; any route out of range skips the region
                const int my_r = lane < TOPK ? __ldg(routes + r * TOPK + lane) : 0;
                const uint32_t badm = __ballot_sync(0xffffffffu, lane < TOPK && (my_r < 0 || my_r >= g.R));
                if (badm) {
                    if (lane == 0) raise_status(status, kDevBadRoute);
                    continue;
                }
                bool dup = false;
#pragma unroll
                for (int dd = 1; dd < TOPK; ++dd) {
                    const int other = __shfl_up_sync(0xffffffffu, my_r, dd);
                    if (dd <= lane && other == my_r) dup = true;
                }
                const uint32_t live = __ballot_sync(0xffffffffu, lane < TOPK && !dup);
                constexpr uint32_t kAll = TOPK >= 32 ? 0xffffffffu : (1u << TOPK) - 1u;
                // K of route ``lane`` starts at this byte (V one slice further)
                const uint32_t my_kb = k_base + (uint32_t)my_r * (uint32_t)N * 64u;
                // this chunk's 16 query tokens: rows t0 and t0 + 8 of the region
                const int t0 = ch * 16 + gq, t1 = t0 + 8;
                const size_t corner = img + (size_t)qcorner[r];
                const size_t orow0 = (corner + (size_t)((t0 >> lg_ws) * g.W + (t0 & (g.ws - 1)))) * g.C + (size_t)hd * 32;
                const size_t orow1 = (corner + (size_t)((t1 >> lg_ws) * g.W + (t1 & (g.ws - 1)))) * g.C + (size_t)hd * 32;
                uint32_t qa[2][4];
#pragma unroll
                for (int kc = 0; kc < 2; ++kc) {
                    const int c0 = 16 * kc + 2 * tq;
                    qa[kc][0] = __ldg(reinterpret_cast<const uint32_t*>(q + orow0 + c0));
                    qa[kc][1] = __ldg(reinterpret_cast<const uint32_t*>(q + orow1 + c0));
                    qa[kc][2] = __ldg(reinterpret_cast<const uint32_t*>(q + orow0 + c0 + 8));
                    qa[kc][3] = __ldg(reinterpret_cast<const uint32_t*>(q + orow1 + c0 + 8));
                }
                uint32_t kb[TOPK];
#pragma unroll
                for (int m = 0; m < TOPK; ++m) kb[m] = __shfl_sync(0xffffffffu, my_kb, m);
                if (!landed) {
                    if (!ring_wait(&rb->full[buf], (k >> 1) & 1, rb, status)) {
                        stop = true;
                        break;
                    }
                    landed = true;
                }
                // S = Q K^T over the routed keys: column tile j is keys 8j..8j+7 of the
                // stacked list (route 8j / N, keys (8j) % N .. of that region)
                float s[NT][4];
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kb[(8 * j) / N] + (uint32_t)((8 * j) % N) * 64u + s_lane, b0, b1, b2, b3);
                    mma16816(s[j], qa[0][0], qa[0][1], qa[0][2], qa[0][3], b0, b1);
                    mma16816(s[j], qa[1][0], qa[1][1], qa[1][2], qa[1][3], b2, b3);
                }
                // masked base-2 softmax over each row (rows gq and gq + 8; a row's 16
                // values of a tile sit in the 4 lanes of its group)
                if (live != kAll) {
#pragma unroll
                    for (int j = 0; j < NT; ++j)
                        if (!((live >> ((8 * j) / N)) & 1u)) s[j][0] = s[j][1] = s[j][2] = s[j][3] = -INFINITY;
                }
                float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    mx0 = fmaxf(mx0, fmaxf(s[j][0], s[j][1]));
                    mx1 = fmaxf(mx1, fmaxf(s[j][2], s[j][3]));
                }
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
                const float m0 = mx0 * sl, m1 = mx1 * sl;
                // P as bf16 pairs (the A operand of P V)
                uint32_t pa[NT][2];
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    pa[j][0] = ptx::pack_bf16x2(ptx::ex2(fmaf(s[j][0], sl, -m0)), ptx::ex2(fmaf(s[j][1], sl, -m0)));
                    pa[j][1] = ptx::pack_bf16x2(ptx::ex2(fmaf(s[j][2], sl, -m1)), ptx::ex2(fmaf(s[j][3], sl, -m1)));
                }
                // O = P V: 16 keys per step (tiles 2kk, 2kk + 1 of P), V rows of the
                // routed region read transposed by ldmatrix; 4 tiles of 8 channels.
                // The row sums of the bf16 P come from one more product per step
                // against ones (every column of ls holds its row's sum).
                float acc[4][4], ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int nn = 0; nn < 4; ++nn) acc[nn][0] = acc[nn][1] = acc[nn][2] = acc[nn][3] = 0.f;
#pragma unroll
                for (int kk = 0; kk < NT / 2; ++kk) {
                    mma16816(ls, pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1], kOnes, kOnes);
                    // matrices: (keys 0-7, ch c..c+7), (keys 8-15, ch c..), (keys 0-7, ch c+8..), (keys 8-15, ch c+8..)
                    const uint32_t vstep = kb[(16 * kk) / N] + slice_bytes + (uint32_t)((16 * kk) % N) * 64u;
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vstep + v_lane0, b0, b1, b2, b3);
                    mma16816(acc[0], pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1], b0, b1);
                    mma16816(acc[1], pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1], b2, b3);
                    ldsm_x4_t(vstep + v_lane1, b0, b1, b2, b3);
                    mma16816(acc[2], pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1], b0, b1);
                    mma16816(acc[3], pa[2 * kk][0], pa[2 * kk][1], pa[2 * kk + 1][0], pa[2 * kk + 1][1], b2, b3);
                }
                // O rows gq and gq + 8: channels 8n + 2tq, 8n + 2tq + 1
                const float i0 = ls[0] > 0.f ? 1.f / ls[0] : 0.f, i1 = ls[2] > 0.f ? 1.f / ls[2] : 0.f;
                if (!in_bounds((orow0 > orow1 ? orow0 : orow1) + 31, map_elems(g), status)) continue;
#pragma unroll
                for (int nn = 0; nn < 4; ++nn) {
                    const int c = 8 * nn + 2 * tq;
                    __stcs(reinterpret_cast<uint32_t*>(o + orow0 + c), ptx::pack_bf16x2(acc[nn][0] * i0, acc[nn][1] * i0));
                    __stcs(reinterpret_cast<uint32_t*>(o + orow1 + c), ptx::pack_bf16x2(acc[nn][2] * i1, acc[nn][3] * i1));
                }
            }
            if (stop) break;
            // a warp with no item in this slice still waits for its load before
            // releasing the buffer: an early release would count toward this
            // buffer's previous slice
            if (!landed && !ring_wait(&rb->full[buf], (k >> 1) & 1, rb, status)) break;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&rb->empty[buf]);
        }
    }
    __syncthreads();
    // every copy this CTA issued must land before it exits: the last use of each
    // buffer is its latest phase (already complete unless a wait gave up)
    if (threadIdx.x == 0) {
        const int issued = rb->issued;
        for (int k = issued - 2 < 0 ? 0 : issued - 2; k < issued; ++k)
            ptx::mbar_wait(&rb->full[k & 1], (k >> 1) & 1, kWait);
    }
}

}  // namespace

bool attend_warp_covers(const Geometry& g) {
    const int kn = g.topk * g.n;
    // kn in {32, 64, 128} and 16 | n make n, ws and hs powers of two (checked
    // anyway: the kernel's index arithmetic relies on it)
    return g.d == 32 && g.n % 16 == 0 && (kn == 32 || kn == 64 || kn == 128) && (g.n & (g.n - 1)) == 0 &&
           (g.ws & (g.ws - 1)) == 0 && g.W <= 256 && g.H <= 256 &&  // one TMA box per map
           (uint32_t)g.R * (uint32_t)g.n * 64u <= kMaxSliceBytes;
}

bra_status attend_warp_launch(const Geometry& g, const void* q, const void* k, const void* v, const int32_t* idx,
                              void* o, int* status, cudaStream_t stream) {
    if (!attend_warp_covers(g)) return BRA_ERR_UNSUPPORTED;
    CUtensorMap tk, tv;
    if (!encode_region_major_map(&tk, k, g.B, g.H, g.W, g.C, g.ws, g.hs, g.S) ||
        !encode_region_major_map(&tv, v, g.B, g.H, g.W, g.C, g.ws, g.hs, g.S))
        return BRA_ERR_UNSUPPORTED;
    const long long items = (long long)g.B * g.heads * g.R * (g.n / 16);
    if (items > 0x7fffffffLL) return BRA_ERR_UNSUPPORTED;
    const int sms = sm_count();
    if (sms <= 0) return BRA_ERR_CUDA;
    const int grid = items < sms ? (int)items : sms;
    const uint32_t smem = 4u * (uint32_t)g.R * (uint32_t)g.n * 64u + (((uint32_t)sizeof(RingBarriers) + 15u) & ~15u) +
                          (uint32_t)g.R * 4u + 1024u;
    using KernelFn = void (*)(CUtensorMap, CUtensorMap, const __nv_bfloat16*, const int32_t*, __nv_bfloat16*, Geometry,
                              int*);
    const int kn = g.topk * g.n;
    const unsigned threads = 32u * (unsigned)(compute_warps_for(kn) + 1);
    KernelFn kernel = nullptr;
    switch (kn * 1000 + g.n) {
        case 32016: kernel = bra_attend_warp_kernel<32, 16>; break;
        case 32032: kernel = bra_attend_warp_kernel<32, 32>; break;
        case 64016: kernel = bra_attend_warp_kernel<64, 16>; break;
        case 64032: kernel = bra_attend_warp_kernel<64, 32>; break;
        case 64064: kernel = bra_attend_warp_kernel<64, 64>; break;
        case 128016: kernel = bra_attend_warp_kernel<128, 16>; break;
        case 128032: kernel = bra_attend_warp_kernel<128, 32>; break;
        case 128064: kernel = bra_attend_warp_kernel<128, 64>; break;
        case 128128: kernel = bra_attend_warp_kernel<128, 128>; break;
        default: return BRA_ERR_UNSUPPORTED;
    }
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return BRA_ERR_CUDA;
    const cudaError_t e = launch_after_previous(kernel, dim3((unsigned)grid), dim3(threads), smem, stream, tk, tv,
                                                static_cast<const __nv_bfloat16*>(q), idx,
                                                static_cast<__nv_bfloat16*>(o), g, status);
    return e == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

}  // namespace bra
