// Persistent, warp-specialised tcgen05 attention for large regions (blog
// "BiFormer Reshapes Visual Attention with Bi-Level Routing", Part 2 section
// 2.2, step 4: gather the routed key-value regions, then token attention over
// them), for regions of a multiple of 128 tokens such as the dense-prediction
// map (128 x 128 tokens, S = 8: 256 tokens per region, 4 routes, 1024 keys per
// query), where the products, not the bytes, set the time.
//
// Tiling.  A tile is 128 query tokens of one region (one (batch, head, region,
// part)); its keys are its routed regions' tokens in blocks of 128 (a region
// of n tokens is n / 128 blocks of 128 / ws image rows), streamed through a
// ring of shared-memory stages by TMA.  For every block, S = Q K^T (M = 128,
// N = 128) lands in TMEM, a softmax thread per query row updates its running
// maximum and writes P = 2^(s - max) as bf16 to shared memory, and O_blk = P V
// (M = 128, N = 48: V next to a block of bf16 ones, so the row sums of P come
// out of the same product) overwrites the block's S columns; the thread folds
// O_blk into its fp32 output registers, rescaled by 2^(old max - new max).
// Every routed region is attended once (a region repeated in a row has P = 0
// for its later listings); a tile whose routes are out of range is reported
// (BRA_ERR_BAD_ROUTE) and not written.
//
// Roles (one CTA per SM, tiles strided by the grid; two tiles in flight, one
// per softmax group, their blocks interleaved):
//   warp 0     producer: routes, each tile's Q box, each block's K and V boxes;
//   warp 1     issues S = Q K^T per block;
//   warp 2     issues O_blk = P V per block and releases the block's stage;
//   two softmax warp groups, one query row per thread.
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

constexpr int kGroups = 2;
constexpr int kCtrl = 3;  // producer, S issuer, P V issuer
constexpr int kThreads = 32 * kCtrl + 128 * kGroups;
constexpr int kMaxRoutes = 32;  // one lane per route
constexpr int kStages = 4;          // K + V blocks in flight
constexpr uint32_t kQBytes = 8192;  // 128 rows x 64 B
constexpr uint32_t kKvBytes = 8192; // one block of K (or V)
constexpr uint32_t kPBytes = 32768; // 128 rows x 128 keys of bf16 (two 128-byte swizzle atoms of 64 keys)
constexpr uint32_t kWait = 1u << 22;
constexpr float kLog2e = 1.4426950408889634f;

struct FlashPlan {
    int parts;      // 128-token query tiles per region (n / 128)
    int kb;         // key blocks per route (n / 128)
    int nb;         // key blocks per tile (topk * kb)
    int box_h;      // image rows per block (128 / ws)
    int tiles;      // B * heads * R * parts
};

// shared memory (1024-aligned): Q [2] | K/V stages [kStages] x (K | V) | P [2 groups][2] | ones | barriers
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffKv = kOffQ + 2 * kQBytes;
constexpr uint32_t kOffP = kOffKv + kStages * 2 * kKvBytes;
constexpr uint32_t kOffOnes = kOffP + kGroups * 2 * kPBytes;
constexpr uint32_t kOffBar = kOffOnes + 1024;

struct Barriers {
    uint64_t q_full[kGroups], q_empty[kGroups];
    uint64_t kv_full[kStages], kv_empty[kStages];
    uint64_t s_full[kGroups][2], s_free[kGroups][2], p_full[kGroups][2], o_full[kGroups][2];
    uint64_t drain[2];
    uint32_t tmem;
    int abort;
};
constexpr uint32_t kSmemBytes = kOffBar + (uint32_t)sizeof(Barriers) + 1024;

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

// The CTA's steps interleave the blocks of two tiles: step s belongs to local
// tile pair s / (2 nb); within a pair, block b of the even tile, then block b of
// the odd tile.  Returns false past the end (an odd last tile has no partner).
struct Step {
    int tile;  // local tile index (group = tile % 2)
    int b;     // key block of the tile
};
__device__ __forceinline__ bool step_at(const FlashPlan& p, int my_tiles, int s, Step& st) {
    const int pair = s / (2 * p.nb), r = s - pair * 2 * p.nb;
    st.b = r >> 1;
    st.tile = 2 * pair + (r & 1);
    return st.tile < my_tiles;
}

// Global coordinates of local tile i of this CTA.
__device__ __forceinline__ void tile_coords(const FlashPlan& p, const Geometry& g, int i, int& bh, int& r, int& part) {
    const int t = (int)blockIdx.x + i * (int)gridDim.x;
    part = t % p.parts;
    const int rr = t / p.parts;
    r = rr % g.R;
    bh = rr / g.R;
}

// The tile's routes as the softmax sees them: bit m of ``live`` set when
// route m is in range and its first listing; ``bad`` when any route is out
// of range.  Every lane of the calling warp gets the same result.  (Each
// softmax warp reads them itself: a value handed over by the producer could
// be overwritten for the group's next tile before a short tile's softmax has
// read it.)
__device__ __forceinline__ void tile_routes(const Geometry& g, const int32_t* __restrict__ idx, int bh, int r,
                                            int lane, uint32_t& live, bool& bad) {
    int my_r = lane < g.topk ? __ldg(idx + ((size_t)bh * g.R + r) * g.topk + lane) : 0;
    const bool out = lane < g.topk && (my_r < 0 || my_r >= g.R);
    bad = __ballot_sync(0xffffffffu, out) != 0u;
    bool dup = false;
    for (int dd = 1; dd < g.topk; ++dd) {
        const int other = __shfl_up_sync(0xffffffffu, my_r, dd);
        if (dd <= lane && other == my_r) dup = true;
    }
    live = __ballot_sync(0xffffffffu, lane < g.topk && !out && !dup);
}

// Columns c0 .. c0 + 63 of this warp's TMEM rows at ``taddr``: four x16 loads,
// one wait; the empty asm statements after the wait name the other three
// groups of registers so that no use of them is scheduled before it.
__device__ __forceinline__ void tmem_ld64_grouped(uint32_t taddr, uint32_t (&r)[4][16]) {
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) ptx::tmem_ld16(taddr + (uint32_t)cc * 16u, r[cc]);
    ptx::tmem_wait16(r[0]);
#pragma unroll
    for (int cc = 1; cc < 4; ++cc)
        asm volatile(""
                     : "+r"(r[cc][0]), "+r"(r[cc][1]), "+r"(r[cc][2]), "+r"(r[cc][3]), "+r"(r[cc][4]),
                       "+r"(r[cc][5]), "+r"(r[cc][6]), "+r"(r[cc][7]), "+r"(r[cc][8]), "+r"(r[cc][9]),
                       "+r"(r[cc][10]), "+r"(r[cc][11]), "+r"(r[cc][12]), "+r"(r[cc][13]), "+r"(r[cc][14]),
                       "+r"(r[cc][15])
                     :
                     : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
bra_attend_flash_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                        const __grid_constant__ CUtensorMap tv, const int32_t* __restrict__ idx,
                        __nv_bfloat16* __restrict__ o, Geometry g, FlashPlan p, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_addr(smem);
    Barriers* sb = reinterpret_cast<Barriers*>(smem + kOffBar);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int my_tiles =
        (int)blockIdx.x < p.tiles ? (p.tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
    const int steps = ((my_tiles + 1) / 2) * 2 * p.nb;  // including the empty slots of an odd last tile

    if (threadIdx.x == 0) {
        for (int x = 0; x < kGroups; ++x) {
            ptx::mbar_init(&sb->q_full[x], 1);
            ptx::mbar_init(&sb->q_empty[x], 1);
            for (int y = 0; y < 2; ++y) {
                ptx::mbar_init(&sb->s_full[x][y], 1);
                ptx::mbar_init(&sb->s_free[x][y], 128);
                ptx::mbar_init(&sb->p_full[x][y], 128);
                ptx::mbar_init(&sb->o_full[x][y], 1);
            }
        }
        for (int x = 0; x < kStages; ++x) {
            ptx::mbar_init(&sb->kv_full[x], 1);
            ptx::mbar_init(&sb->kv_empty[x], 1);
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
    for (uint32_t i = kOffOnes / 16 + threadIdx.x; i < kOffBar / 16; i += kThreads)
        reinterpret_cast<uint4*>(smem)[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    ptx::fence_proxy_async_smem();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sb->tmem;
    grid_dependency_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            ptx::tma_prefetch_desc(&tq);
            ptx::tma_prefetch_desc(&tk);
            ptx::tma_prefetch_desc(&tv);
        }
        int my_r0 = 0, my_r1 = 0;  // route ``lane`` of each group's current tile
        for (int s = 0; s < steps; ++s) {
            Step st;
            if (!step_at(p, my_tiles, s, st)) continue;
            const int grp = st.tile & 1, use = st.tile >> 1;  // the group's use-th tile
            int bh = 0, r = 0, part = 0;
            tile_coords(p, g, st.tile, bh, r, part);
            const int b = bh / g.heads, hd = bh - b * g.heads;
            if (st.b == 0) {
                // routes of the tile (lane m < topk holds route m), then its Q box
                if (use > 0 && !wait_or_abort(&sb->q_empty[grp], (use - 1) & 1, sb, status)) break;
                int my_r = lane < g.topk ? __ldg(idx + ((size_t)bh * g.R + r) * g.topk + lane) : 0;
                if (my_r < 0 || my_r >= g.R) my_r = 0;  // the softmax reports and discards the tile
                if (grp) my_r1 = my_r;
                else my_r0 = my_r;
                if (lane == 0) {
                    ptx::mbar_arrive_expect_tx(&sb->q_full[grp], kQBytes);
                    const int ri = r / g.S, rj = r - ri * g.S;
                    ptx::tma_load_4d(sbase + kOffQ + grp * kQBytes, &tq, hd * 32, rj * g.ws,
                                     ri * g.hs + part * p.box_h, b, &sb->q_full[grp]);
                }
            }
            // block st.b: route m = b / kb, rows (b % kb) * box_h of that region
            const int stage = s % kStages;
            if (s >= kStages && !wait_or_abort(&sb->kv_empty[stage], ((s / kStages) - 1) & 1, sb, status)) break;
            const int m = st.b / p.kb, kbi = st.b - m * p.kb;
            const int rr = __shfl_sync(0xffffffffu, grp ? my_r1 : my_r0, m);
            if (lane == 0) {
                const int ri = rr / g.S, rj = rr - ri * g.S;
                const uint32_t kvs = sbase + kOffKv + (uint32_t)stage * 2u * kKvBytes;
                ptx::mbar_arrive_expect_tx(&sb->kv_full[stage], 2u * kKvBytes);
                ptx::tma_load_4d(kvs, &tk, hd * 32, rj * g.ws, ri * g.hs + kbi * p.box_h, b, &sb->kv_full[stage]);
                ptx::tma_load_4d(kvs + kKvBytes, &tv, hd * 32, rj * g.ws, ri * g.hs + kbi * p.box_h, b,
                                 &sb->kv_full[stage]);
            }
            __syncwarp();
        }
    } else if (warp == 1) {
        // ------------------------------------------------------- S = Q K^T issuer
        if (lane == 0) {
            const uint32_t idesc = ptx::idesc_bf16_f32(128, 128, false, false);
            for (int s = 0; s < steps; ++s) {
                Step st;
                if (!step_at(p, my_tiles, s, st)) continue;
                const int grp = st.tile & 1, use = st.tile >> 1;
                const int k = use * p.nb + st.b, buf = k & 1;  // the group's k-th block
                const int stage = s % kStages;
                if (st.b == 0 && !wait_or_abort(&sb->q_full[grp], use & 1, sb, status)) break;
                if (!wait_or_abort(&sb->kv_full[stage], (s / kStages) & 1, sb, status)) break;
                if (k >= 2 && !wait_or_abort(&sb->s_free[grp][buf], ((k >> 1) - 1) & 1, sb, status)) break;
                ptx::tc_fence_after();
                const uint32_t q = sbase + kOffQ + grp * kQBytes;
                const uint32_t kk_base = sbase + kOffKv + (uint32_t)stage * 2u * kKvBytes;
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const uint64_t a = ptx::smem_desc(q + kk * 32, 16, 512, ptx::kSwizzle64B);
                    const uint64_t bd = ptx::smem_desc(kk_base + kk * 32, 16, 512, ptx::kSwizzle64B);
                    ptx::mma_bf16(tmem + (uint32_t)(grp * 2 + buf) * 128u, a, bd, idesc, kk);
                }
                ptx::mma_commit(&sb->s_full[grp][buf]);
                if (st.b == p.nb - 1) ptx::mma_commit(&sb->q_empty[grp]);  // the tile's last use of Q
            }
            ptx::mma_commit(&sb->drain[0]);
            ptx::mbar_wait(&sb->drain[0], 0, kWait);
        }
        __syncwarp();
    } else if (warp == 2) {
        // ---------------------------------------------------- O_blk = P V issuer
        if (lane == 0) {
            // N = 48: columns 0..31 are V, 32..47 the ones block (row sums of P)
            const uint32_t idesc = ptx::idesc_bf16_f32(128, 48, false, true);
            const uint32_t ones = sbase + kOffOnes;
            for (int s = 0; s < steps; ++s) {
                Step st;
                if (!step_at(p, my_tiles, s, st)) continue;
                const int grp = st.tile & 1, use = st.tile >> 1;
                const int k = use * p.nb + st.b, buf = k & 1;
                const int stage = s % kStages;
                if (!wait_or_abort(&sb->p_full[grp][buf], (k >> 1) & 1, sb, status)) break;
                ptx::tc_fence_after();
                const uint32_t vbase = sbase + kOffKv + (uint32_t)stage * 2u * kKvBytes + kKvBytes;
                const uint32_t pbase = sbase + kOffP + (uint32_t)(grp * 2 + buf) * kPBytes;
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t vaddr = vbase + (uint32_t)kk * 1024u;
                    const uint64_t a = ptx::smem_desc(pbase + (uint32_t)(kk >> 2) * 16384u + (kk & 3) * 32, 16, 1024,
                                                      ptx::kSwizzle128B);
                    const uint64_t bd = ptx::smem_desc(vaddr, ones - vaddr, 512, ptx::kSwizzle64B);
                    ptx::mma_bf16(tmem + (uint32_t)(grp * 2 + buf) * 128u, a, bd, idesc, kk);
                }
                ptx::mma_commit(&sb->o_full[grp][buf]);
                ptx::mma_commit(&sb->kv_empty[stage]);
            }
            ptx::mma_commit(&sb->drain[1]);
            ptx::mbar_wait(&sb->drain[1], 0, kWait);
        }
        __syncwarp();
    } else {
        // --------------------------------------------------- softmax + epilogue
        const int grp = (warp - kCtrl) >> 2;
        const int qd = warp & 3;  // TMEM lane quadrant this warp may access
        const int row = 32 * qd + lane;
        const uint32_t lane_addr = (uint32_t)(32 * qd) << 16;
        const float sl = kLog2e * rsqrtf(32.f);
        bool ok = true;
        for (int tile = grp; ok && tile < my_tiles; tile += kGroups) {
            const int use = tile >> 1;
            float acc[32], l_acc = 0.f, m_run = -INFINITY;
#pragma unroll
            for (int c = 0; c < 32; ++c) acc[c] = 0.f;
            float alpha_prev = 0.f;  // rescale of the block whose O is folded next
            int tbh = 0, tr = 0, tpart = 0;
            tile_coords(p, g, tile, tbh, tr, tpart);
            uint32_t live = 0u;
            bool bad = false;
            tile_routes(g, idx, tbh, tr, lane, live, bad);
            if (bad && qd == 0 && lane == 0) raise_status(status, kDevBadRoute);
            // fold O_blk of the group's k-th block into acc (after its P V is done)
            auto fold = [&](int k, float alpha) -> bool {
                const int buf = k & 1;
                if (!wait_or_abort(&sb->o_full[grp][buf], (k >> 1) & 1, sb, status)) return false;
                ptx::tc_fence_after();
                const uint32_t ob = tmem + lane_addr + (uint32_t)(grp * 2 + buf) * 128u;
                uint32_t r[16], r2[16], lw;
                ptx::tmem_ld16(ob, r);
                ptx::tmem_ld16(ob + 16, r2);
                lw = ptx::tmem_ld1(ob + 32);
                ptx::tmem_wait17(r, lw);
                ptx::tmem_wait16(r2);  // no second round trip: the loads above are all complete
#pragma unroll
                for (int c = 0; c < 16; ++c) acc[c] = fmaf(acc[c], alpha, __uint_as_float(r[c]));
#pragma unroll
                for (int c = 0; c < 16; ++c) acc[16 + c] = fmaf(acc[16 + c], alpha, __uint_as_float(r2[c]));
                l_acc = fmaf(l_acc, alpha, __uint_as_float(lw));
                ptx::tc_fence_before();
                ptx::mbar_arrive(&sb->s_free[grp][buf]);
                return true;
            };
            for (int b = 0; b < p.nb && ok; ++b) {
                const int k = use * p.nb + b, buf = k & 1;
                if (!wait_or_abort(&sb->s_full[grp][buf], (k >> 1) & 1, sb, status)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const bool on = (live >> (b / p.kb)) & 1u;  // a repeated listing contributes nothing
                const uint32_t sa = tmem + lane_addr + (uint32_t)(grp * 2 + buf) * 128u;
                float mb = -INFINITY;
                if (on) {
                    // the row's 128 scores, 64 columns per TMEM round trip
                    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int c0 = 0; c0 < 128; c0 += 64) {
                        uint32_t r[4][16];
                        tmem_ld64_grouped(sa + c0, r);
#pragma unroll
                        for (int cc = 0; cc < 4; ++cc)
#pragma unroll
                            for (int e = 0; e < 16; ++e) m4[e & 3] = fmaxf(m4[e & 3], __uint_as_float(r[cc][e]));
                    }
                    mb = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl;
                }
                const float m_new = fmaxf(m_run, mb);
                // rescale of what was accumulated before this block (0 before the first live block)
                const float alpha = m_run == -INFINITY ? 0.f : ptx::ex2(m_run - m_new);
                const uint32_t prow = sbase + kOffP + (uint32_t)(grp * 2 + buf) * kPBytes + (uint32_t)row * 128u;
#pragma unroll
                for (int c0 = 0; c0 < 128; c0 += 64) {
                    uint32_t r[4][16];
                    if (on) tmem_ld64_grouped(sa + c0, r);
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        uint32_t packed[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            packed[e] = on ? ptx::pack_bf16x2(ptx::ex2(fmaf(__uint_as_float(r[cc][2 * e]), sl, -m_new)), ptx::ex2(fmaf(__uint_as_float(r[cc][2 * e + 1]), sl, -m_new)))
                                           : 0u;
                        const int c = c0 + 16 * cc;
                        const uint32_t atom = prow + (uint32_t)(c >> 6) * 16384u;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const int chunk = ((c & 63) >> 3) + h;
                            ptx::st_shared_v4(atom + ((chunk ^ (row & 7)) << 4), packed[4 * h], packed[4 * h + 1],
                                              packed[4 * h + 2], packed[4 * h + 3]);
                        }
                    }
                }
                m_run = m_new;
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                ptx::mbar_arrive(&sb->p_full[grp][buf]);
                // the previous block's O, its P V overlapping this block's softmax
                if (b > 0 && !fold(k - 1, alpha_prev)) {
                    ok = false;
                    break;
                }
                alpha_prev = alpha;
            }
            if (!ok) break;
            // the tile's last block, then O = acc / l
            if (!fold(use * p.nb + p.nb - 1, alpha_prev)) break;
            const int b = tbh / g.heads, hd = tbh - b * g.heads;
            const bool write = !bad && l_acc > 0.f;
            const size_t ooff = token_offset(g, b, tr, tpart * 128 + row) + (size_t)hd * 32;
            if (write && in_bounds(ooff + 31, map_elems(g), status)) {
                const float inv = 1.f / l_acc;
                int4* dst = reinterpret_cast<int4*>(o + ooff);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) w[e] = ptx::pack_bf16x2(acc[8 * c + 2 * e] * inv, acc[8 * c + 2 * e + 1] * inv);
                    __stcs(dst + c, make_int4((int)w[0], (int)w[1], (int)w[2], (int)w[3]));
                }
            }
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

bool make_flash_plan(const Geometry& g, FlashPlan* p) {
    if (g.d != 32 || g.n % 128 != 0 || 128 % g.ws != 0 || g.topk > kMaxRoutes) return false;
    p->box_h = 128 / g.ws;
    if (g.hs % p->box_h != 0) return false;
    p->parts = g.n / 128;
    p->kb = g.n / 128;
    p->nb = g.topk * p->kb;
    const long long tiles = (long long)g.B * g.heads * g.R * p->parts;
    if (tiles > 0x7fffffffLL) return false;
    p->tiles = (int)tiles;
    return kSmemBytes <= 227u * 1024u;
}

}  // namespace

bool attend_flash_covers(const Geometry& g) {
    FlashPlan p;
    return make_flash_plan(g, &p);
}

bra_status attend_flash_launch(const Geometry& g, const void* q, const void* k, const void* v, const int32_t* idx,
                               void* o, int* status, cudaStream_t stream) {
    FlashPlan p;
    if (!make_flash_plan(g, &p)) return BRA_ERR_UNSUPPORTED;
    CUtensorMap tq, tk, tv;
    if (!encode_region_map(&tq, q, g.B, g.H, g.W, g.C, g.ws, p.box_h, 32) ||
        !encode_region_map(&tk, k, g.B, g.H, g.W, g.C, g.ws, p.box_h, 32) ||
        !encode_region_map(&tv, v, g.B, g.H, g.W, g.C, g.ws, p.box_h, 32))
        return BRA_ERR_UNSUPPORTED;
    const int sms = sm_count();
    if (sms <= 0) return BRA_ERR_CUDA;
    const int grid = p.tiles < sms ? p.tiles : sms;
    if (cudaFuncSetAttribute(bra_attend_flash_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes) != cudaSuccess)
        return BRA_ERR_CUDA;
    const cudaError_t e = launch_after_previous(bra_attend_flash_kernel, dim3(grid), dim3(kThreads), kSmemBytes,
                                                stream, tq, tk, tv, idx, static_cast<__nv_bfloat16*>(o), g, p,
                                                status);
    return e == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

}  // namespace bra
