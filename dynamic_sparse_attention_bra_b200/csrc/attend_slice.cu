// Persistent tcgen05 attention for small maps, one (batch, head) slice at a
// time, dense over the slice with the routing applied as a mask (blog
// "BiFormer Reshapes Visual Attention with Bi-Level Routing", Part 2 section
// 2.2, step 4: token attention over the union of the routed regions' tokens).
//
// Why.  When a map holds at most 256 tokens (BiFormer stage 3: 14 x 14, with
// 49 regions of 2 x 2 tokens and 16 routes per region), a region is too small
// for a tensor-core tile and gathering its routed regions one by one costs
// more than the whole slice: here a slice's Q, K and V are each one TMA box
// (every token of the map, one head, 64-byte rows), S = Q K^T is computed for
// every query against every key of the slice (M = 128 queries, N = the slice's
// tokens rounded up to 16), and each query's softmax reads only the keys of
// its routed regions (a per-region key mask built from I^r); P is zero
// elsewhere, so O = P V over the whole slice equals attention over the union
// of the routed tokens.  Each softmax thread forms its own mask as the OR of
// its region's routed regions' token bitmaps (a table that depends on the map
// geometry only, built once per CTA), so a region listed twice sets its keys
// once; a query region with an out-of-range route is reported and its outputs
// are skipped.
//
// Roles (one CTA per SM, slices strided by the grid):
//   warp 0     producer: the slice's Q, K, V boxes into a two-stage ring,
//              then, while they land, each query region's key mask (lane per
//              region: the OR of its routed regions' token bits) into the
//              stage's mask buffer, so the softmax threads read a finished mask;
//   warp 1     issues S = Q K^T for each 128-query unit of a slice;
//   warp 2     issues O = P V (with the row sums of P) for each unit;
//   two softmax warp groups, units alternating between them, one query row
//   per thread: masked base-2 softmax, P as bf16 into shared memory, then
//   O = (P V) / l to global memory.
// Every mbarrier wait is bounded; on expiry the kernel records kDevTimeout,
// stops all roles, drains its MMAs and frees TMEM.
#include <cuda.h>
#include <stdlib.h>

#include "attend_tc.h"
#include "kernels.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace bra {
namespace {

constexpr int kStages = 2;
constexpr int kGroups = 2;
constexpr int kCtrl = 3;  // producer, S issuer, P V issuer
constexpr int kThreads = 32 * kCtrl + 128 * kGroups;
constexpr int kMaxTokens = 256;
constexpr int kMaxWords = kMaxTokens / 32;
constexpr uint32_t kWait = 1u << 22;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kSmemBudget = 227 * 1024;

struct SlicePlan {
    int HW;                 // tokens of the slice (<= 256)
    int Np;                 // keys rounded up to 16 (MMA N of S)
    int mt;                 // 128-query units per slice (1 or 2)
    int words;              // 32-bit mask words per query region: ceil(Np / 32)
    int slices;             // B * heads
    uint32_t q_bytes;       // mt * 128 rows x 64 B
    uint32_t kv_bytes;      // Np rows x 64 B
    uint32_t k_off, v_off;  // inside a stage
    uint32_t stage_bytes;
    uint32_t p_off;         // two P buffers (one per softmax group)
    uint32_t p_bytes;       // ceil(Np / 64) atom columns of 128 rows x 128 B
    uint32_t ones_off;      // 16 rows x 64 B of bf16 ones
    uint32_t tok_off;       // R x words of uint32: the tokens of each region as key bits
    int pre_mask;           // 1: the producer builds each query region's key mask per stage
    uint32_t mask_off;      // per stage: R x words of uint32 (pre_mask)
    uint32_t mask_bytes;    // R * words * 4 rounded up to 16
    uint32_t bar_off;
    uint32_t smem_bytes;
};

struct Barriers {
    uint64_t full[kStages];   // the slice's boxes landed (and its masks are written)
    uint64_t empty[kStages];  // the slice's last P V is done: stage free
    uint64_t s_full[kGroups], o_full[kGroups], s_free[kGroups], p_full[kGroups];
    uint64_t drain[2];
    uint32_t tmem;
    int abort;
};

__device__ __forceinline__ bool aborted(Barriers* sb) {
    return *reinterpret_cast<volatile int*>(&sb->abort) != 0;
}

__device__ __forceinline__ void set_abort(Barriers* sb, int* status) {
    *reinterpret_cast<volatile int*>(&sb->abort) = 1;
    raise_status(status, kDevTimeout);
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Barriers* sb, int* status) {
    for (uint32_t i = 0; i < kWait; ++i) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((i & 1023) == 1023 && aborted(sb)) return false;
    }
    set_abort(sb, status);
    return false;
}

__global__ void __launch_bounds__(kThreads, 1)
bra_attend_slice_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                        const __grid_constant__ CUtensorMap tv, const int32_t* __restrict__ idx,
                        __nv_bfloat16* __restrict__ o, Geometry g, SlicePlan p, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_addr(smem);
    Barriers* sb = reinterpret_cast<Barriers*>(smem + p.bar_off);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int my_slices =
        (int)blockIdx.x < p.slices ? (p.slices - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
    const int my_units = my_slices * p.mt;
    const uint32_t ones = sbase + p.ones_off;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&sb->full[s], p.pre_mask ? 1 + 32 : 1);  // + each producer lane's masks
            ptx::mbar_init(&sb->empty[s], 1);
        }
        for (int b = 0; b < kGroups; ++b) {
            ptx::mbar_init(&sb->s_full[b], 1);
            ptx::mbar_init(&sb->o_full[b], 1);
            ptx::mbar_init(&sb->s_free[b], 128);
            ptx::mbar_init(&sb->p_full[b], 128);
        }
        ptx::mbar_init(&sb->drain[0], 1);
        ptx::mbar_init(&sb->drain[1], 1);
        sb->abort = 0;
        ptx::mbar_init_fence();
    }
    if (warp == 1) {
        ptx::tmem_alloc(&sb->tmem, 512);
        ptx::tmem_relinquish();
        ptx::tc_fence_before();
    }
    // Zero, once, the V rows past the slice's last token (P is zero there,
    // and 0 times a stale non-finite value would not be); the boxes never
    // write them.  Then the ones block.
    {
        const uint32_t tail0 = (uint32_t)p.HW * 64u / 16u, tail1 = p.kv_bytes / 16u;
        for (int s = 0; s < kStages; ++s)
            for (uint32_t i = tail0 + threadIdx.x; i < tail1; i += kThreads)
                reinterpret_cast<uint4*>(smem + s * p.stage_bytes + p.v_off)[i] = make_uint4(0, 0, 0, 0);
        for (uint32_t i = p.ones_off / 16 + threadIdx.x; i < p.tok_off / 16; i += kThreads)
            reinterpret_cast<uint4*>(smem)[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
        // key bits of each region's tokens (token t = y * W + x is bit t)
        uint32_t* tok = reinterpret_cast<uint32_t*>(smem + p.tok_off);
        for (int i = threadIdx.x; i < g.R * p.words; i += kThreads) tok[i] = 0u;
        __syncthreads();
        for (int t = threadIdx.x; t < p.HW; t += kThreads) {
            const int y = t / g.W, x = t - y * g.W;
            const int r = (y / g.hs) * g.S + x / g.ws;
            atomicOr(&tok[r * p.words + (t >> 5)], 1u << (t & 31));
        }
    }
    ptx::fence_proxy_async_smem();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sb->tmem;
    // Everything above overlaps the routing kernel; from here on the routes
    // are read and O is written.
    grid_dependency_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            ptx::tma_prefetch_desc(&tq);
            ptx::tma_prefetch_desc(&tk);
            ptx::tma_prefetch_desc(&tv);
        }
        for (int j = 0; j < my_slices; ++j) {
            const int s = j % kStages;
            if (j >= kStages && !wait_or_abort(&sb->empty[s], ((j / kStages) - 1) & 1, sb, status)) break;
            const int bh = (int)blockIdx.x + j * (int)gridDim.x;
            const int b = bh / g.heads, hd = bh - b * g.heads;
            const uint32_t stage = sbase + (uint32_t)s * p.stage_bytes;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_expect_tx(&sb->full[s], (uint32_t)p.HW * 64u * 3u);
            __syncwarp();
            if (lane < 3) {
                const CUtensorMap* map = lane == 0 ? &tq : (lane == 1 ? &tk : &tv);
                const uint32_t off = lane == 0 ? 0u : (lane == 1 ? p.k_off : p.v_off);
                ptx::tma_load_4d(stage + off, map, hd * 32, 0, 0, b, &sb->full[s]);
            }
            if (p.pre_mask) {
                // the slice's key masks, lane per query region; a region with an
                // out-of-range route gets an empty mask (l = 0: nothing written)
                const int32_t* rsrc = idx + (size_t)bh * g.R * g.topk;
                const uint32_t* tok = reinterpret_cast<const uint32_t*>(smem + p.tok_off);
                uint32_t* mdst = reinterpret_cast<uint32_t*>(smem + p.mask_off + (uint32_t)s * p.mask_bytes);
                for (int r = lane; r < g.R; r += 32) {
                    uint32_t mk[kMaxWords];
#pragma unroll
                    for (int w = 0; w < kMaxWords; ++w) mk[w] = 0u;
                    bool bad = false;
                    for (int m = 0; m < g.topk; ++m) {
                        const int rr = __ldg(rsrc + (size_t)r * g.topk + m);
                        if (rr < 0 || rr >= g.R) {
                            bad = true;
                            continue;
                        }
#pragma unroll
                        for (int w = 0; w < kMaxWords; ++w)
                            if (w < p.words) mk[w] |= tok[rr * p.words + w];
                    }
                    if (bad) raise_status(status, kDevBadRoute);
#pragma unroll
                    for (int w = 0; w < kMaxWords; ++w)
                        if (w < p.words) mdst[r * p.words + w] = bad ? 0u : mk[w];
                }
                ptx::mbar_arrive(&sb->full[s]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- S = Q K^T issuer
        if (lane == 0) {
            const uint32_t idesc_qk = ptx::idesc_bf16_f32(128, p.Np, false, false);
            for (int u = 0; u < my_units; ++u) {
                const int j = u / p.mt, mt = u - j * p.mt, s = j % kStages, buf = u % kGroups;
                if (!wait_or_abort(&sb->full[s], (j / kStages) & 1, sb, status)) break;
                if (u >= kGroups && !wait_or_abort(&sb->s_free[buf], ((u / kGroups) - 1) & 1, sb, status)) break;
                ptx::tc_fence_after();
                const uint32_t stage = sbase + (uint32_t)s * p.stage_bytes;
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const uint64_t a = ptx::smem_desc(stage + (uint32_t)mt * 8192u + kk * 32, 16, 512, ptx::kSwizzle64B);
                    const uint64_t bd = ptx::smem_desc(stage + p.k_off + kk * 32, 16, 512, ptx::kSwizzle64B);
                    ptx::mma_bf16(tmem + (uint32_t)buf * 256u, a, bd, idesc_qk, kk);
                }
                ptx::mma_commit(&sb->s_full[buf]);
            }
            ptx::mma_commit(&sb->drain[0]);
            ptx::mbar_wait(&sb->drain[0], 0, kWait);
        }
        __syncwarp();
    } else if (warp == 2) {
        // --------------------------------------------------- O = P V issuer
        if (lane == 0) {
            // N = 48: columns 0..31 are V, 32..47 the ones block (row sums of P).
            const uint32_t idesc_pv = ptx::idesc_bf16_f32(128, 48, false, true);
            const int steps = p.Np / 16;
            for (int u = 0; u < my_units; ++u) {
                const int j = u / p.mt, mt = u - j * p.mt, s = j % kStages, buf = u % kGroups;
                if (!wait_or_abort(&sb->p_full[buf], (u / kGroups) & 1, sb, status)) break;
                ptx::tc_fence_after();
                const uint32_t vbase = sbase + (uint32_t)s * p.stage_bytes + p.v_off;
                const uint32_t pbase = sbase + p.p_off + (uint32_t)buf * p.p_bytes;
                for (int kk = 0; kk < steps; ++kk) {
                    const uint32_t vaddr = vbase + (uint32_t)kk * 1024u;
                    const uint64_t a = ptx::smem_desc(pbase + (uint32_t)(kk >> 2) * 16384u + (kk & 3) * 32, 16, 1024,
                                                      ptx::kSwizzle128B);
                    const uint64_t bd = ptx::smem_desc(vaddr, ones - vaddr, 512, ptx::kSwizzle64B);
                    ptx::mma_bf16(tmem + (uint32_t)buf * 256u, a, bd, idesc_pv, kk);
                }
                ptx::mma_commit(&sb->o_full[buf]);
                if (mt == p.mt - 1) ptx::mma_commit(&sb->empty[s]);
            }
            ptx::mma_commit(&sb->drain[1]);
            ptx::mbar_wait(&sb->drain[1], 0, kWait);
        }
        __syncwarp();
    } else {
        // --------------------------------------------------- softmax + epilogue
        const int grp = (warp - kCtrl) >> 2;
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        const int row = 32 * q + lane;
        const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
        const float sl = kLog2e * rsqrtf(32.f);
        const int nch = p.Np / 16;
        for (int u = grp; u < my_units; u += kGroups) {
            const int j = u / p.mt, mt = u - j * p.mt, s = j % kStages, buf = u % kGroups;
            const int bh = (int)blockIdx.x + j * (int)gridDim.x;
            const int b = bh / g.heads, hd = bh - b * g.heads;
            const int t = mt * 128 + row;  // this thread's query token in the slice
            const bool valid = t < p.HW;
            const int y = t / g.W, x = t - y * g.W;
            const int reg = valid ? (y / g.hs) * g.S + x / g.ws : 0;
            // this query region's key mask: the OR of its routed regions' token bits
            uint32_t mk[kMaxWords];
#pragma unroll
            for (int w = 0; w < kMaxWords; ++w) mk[w] = 0u;
            if (valid && !p.pre_mask) {
                const int32_t* rows = idx + ((size_t)bh * g.R + reg) * g.topk;
                const uint32_t* tok = reinterpret_cast<const uint32_t*>(smem + p.tok_off);
                bool bad = false;
                for (int m0 = 0; m0 < g.topk; m0 += 8) {
                    int rr[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) rr[e] = m0 + e < g.topk ? __ldg(rows + m0 + e) : 0;
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        if (m0 + e >= g.topk) continue;
                        if (rr[e] < 0 || rr[e] >= g.R) {
                            bad = true;
                            continue;
                        }
#pragma unroll
                        for (int w = 0; w < kMaxWords; ++w)
                            if (w < p.words) mk[w] |= tok[rr[e] * p.words + w];
                    }
                }
                if (bad) {
                    // a region with an out-of-range route keeps its outputs
                    // untouched: an empty mask gives l = 0, and nothing is written
                    raise_status(status, kDevBadRoute);
#pragma unroll
                    for (int w = 0; w < kMaxWords; ++w) mk[w] = 0u;
                }
            }
            if (!wait_or_abort(&sb->full[s], (j / kStages) & 1, sb, status)) break;
            if (valid && p.pre_mask) {  // the producer's mask of this query region
                const uint32_t* msrc =
                    reinterpret_cast<const uint32_t*>(smem + p.mask_off + (uint32_t)s * p.mask_bytes) + reg * p.words;
#pragma unroll
                for (int w = 0; w < kMaxWords; ++w)
                    if (w < p.words) mk[w] = msrc[w];
            }
            if (!wait_or_abort(&sb->s_full[buf], (u / kGroups) & 1, sb, status)) break;
            ptx::tc_fence_after();
            const uint32_t sbuf = tmem + lane_addr + (uint32_t)buf * 256u;
            // max over the routed keys
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < kMaxTokens / 16; ++c) {
                if (c < nch) {
                    uint32_t r[16];
                    ptx::tmem_ld16(sbuf + (uint32_t)c * 16u, r);
                    ptx::tmem_wait16(r);
                    const uint32_t bits = (mk[c >> 1] >> (16 * (c & 1))) & 0xFFFFu;
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        if ((bits >> e) & 1u) m4[e & 3] = fmaxf(m4[e & 3], __uint_as_float(r[e]));
                }
            }
            const float msl = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl;
            // p = 2^(s * sl - max) on the routed keys, 0 elsewhere, as bf16 into
            // the 128-byte swizzled K-major P buffer of this group
            const uint32_t prow = sbase + p.p_off + (uint32_t)buf * p.p_bytes + (uint32_t)row * 128u;
#pragma unroll
            for (int c = 0; c < kMaxTokens / 16; ++c) {
                if (c < nch) {
                    uint32_t r[16];
                    ptx::tmem_ld16(sbuf + (uint32_t)c * 16u, r);
                    ptx::tmem_wait16(r);
                    const uint32_t bits = (mk[c >> 1] >> (16 * (c & 1))) & 0xFFFFu;
                    uint32_t packed[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float x0 = ((bits >> (2 * e)) & 1u) ? fmaf(__uint_as_float(r[2 * e]), sl, -msl) : -INFINITY;
                        const float x1 =
                            ((bits >> (2 * e + 1)) & 1u) ? fmaf(__uint_as_float(r[2 * e + 1]), sl, -msl) : -INFINITY;
                        packed[e] = ptx::pack_bf16x2(ptx::ex2(x0), ptx::ex2(x1));
                    }
                    const uint32_t atom = prow + (uint32_t)(c >> 2) * 16384u;
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int chunk = ((c & 3) << 1) + cc;
                        ptx::st_shared_v4(atom + ((chunk ^ (row & 7)) << 4), packed[4 * cc], packed[4 * cc + 1],
                                          packed[4 * cc + 2], packed[4 * cc + 3]);
                    }
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            ptx::mbar_arrive(&sb->p_full[buf]);
            // epilogue: O = (P V) / l, then release the TMEM buffer
            if (!wait_or_abort(&sb->o_full[buf], (u / kGroups) & 1, sb, status)) break;
            ptx::tc_fence_after();
            uint32_t r[16], lw = 0;
            ptx::tmem_ld16(sbuf, r);
            lw = ptx::tmem_ld1(sbuf + 32);
            ptx::tmem_wait17(r, lw);
            const float l = __uint_as_float(lw);
            const bool write = valid && l > 0.f;
            const float inv = write ? 1.f / l : 0.f;
            const size_t ooff = write ? (((size_t)b * g.H + y) * g.W + x) * g.C + (size_t)hd * 32 : 0;
            int4* dst = write && in_bounds(ooff + 31, map_elems(g), status) ? reinterpret_cast<int4*>(o + ooff) : nullptr;
#pragma unroll
            for (int h16 = 0; h16 < 2; ++h16) {
                if (h16 == 1) {
                    ptx::tmem_ld16(sbuf + 16, r);
                    ptx::tmem_wait16(r);
                }
                if (dst) {
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            w[e] = ptx::pack_bf16x2(__uint_as_float(r[8 * c + 2 * e]) * inv,
                                                    __uint_as_float(r[8 * c + 2 * e + 1]) * inv);
                        __stcs(dst + 2 * h16 + c, make_int4((int)w[0], (int)w[1], (int)w[2], (int)w[3]));
                    }
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&sb->s_free[buf]);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

bool make_slice_plan(const Geometry& g, SlicePlan* p) {
    const int HW = g.H * g.W;
    if (g.d != 32 || HW > kMaxTokens || g.W > 256 || g.H > 256 || g.R > kMaxTokens) return false;
    p->HW = HW;
    p->Np = (HW + 15) / 16 * 16;
    p->mt = (HW + 127) / 128;
    p->words = (p->Np + 31) / 32;
    const long long slices = (long long)g.B * g.heads;
    if (slices * p->mt > 0x7fffffffLL) return false;
    p->slices = (int)slices;
    p->q_bytes = (uint32_t)p->mt * 8192u;
    p->kv_bytes = (uint32_t)p->Np * 64u;
    p->k_off = p->q_bytes;
    p->v_off = p->k_off + ((p->kv_bytes + 1023) / 1024) * 1024;
    p->stage_bytes = p->v_off + ((p->kv_bytes + 1023) / 1024) * 1024;
    p->p_off = kStages * p->stage_bytes;
    p->p_bytes = (uint32_t)((p->Np + 63) / 64) * 16384u;
    p->ones_off = p->p_off + kGroups * p->p_bytes;
    p->tok_off = p->ones_off + 1024;
    p->mask_off = p->tok_off + ((uint32_t)g.R * p->words * 4u + 15) / 16 * 16;
    p->mask_bytes = ((uint32_t)g.R * p->words * 4u + 15) / 16 * 16;
    // the producer-built masks where two stages of them fit, else each softmax
    // thread builds its own from the routes in global memory
    for (int pre = 1; pre >= 0; --pre) {
        p->pre_mask = pre;
        p->bar_off = p->mask_off + (pre ? kStages * p->mask_bytes : 0u);
        p->smem_bytes = p->bar_off + (uint32_t)sizeof(Barriers) + 1024;
        if (p->smem_bytes <= kSmemBudget) return true;
    }
    return false;
}

}  // namespace

bool attend_slice_covers(const Geometry& g) {
    SlicePlan p;
    return make_slice_plan(g, &p);
}

bra_status attend_slice_launch(const Geometry& g, const void* q, const void* k, const void* v, const int32_t* idx,
                               void* o, int* status, cudaStream_t stream) {
    SlicePlan p;
    if (!make_slice_plan(g, &p)) return BRA_ERR_UNSUPPORTED;
    CUtensorMap tq, tk, tv;
    if (!encode_region_map(&tq, q, g.B, g.H, g.W, g.C, g.W, g.H, 32) ||
        !encode_region_map(&tk, k, g.B, g.H, g.W, g.C, g.W, g.H, 32) ||
        !encode_region_map(&tv, v, g.B, g.H, g.W, g.C, g.W, g.H, 32))
        return BRA_ERR_UNSUPPORTED;
    const int sms = sm_count();
    if (sms <= 0) return BRA_ERR_CUDA;
    const int grid = p.slices < sms ? p.slices : sms;
    if (cudaFuncSetAttribute(bra_attend_slice_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)p.smem_bytes) != cudaSuccess)
        return BRA_ERR_CUDA;
    const cudaError_t e = launch_after_previous(bra_attend_slice_kernel, dim3(grid), dim3(kThreads), p.smem_bytes,
                                                stream, tq, tk, tv, idx, static_cast<__nv_bfloat16*>(o), g, p,
                                                status);
    return e == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

}  // namespace bra
