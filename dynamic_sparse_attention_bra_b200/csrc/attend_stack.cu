// Persistent, warp-specialised tcgen05 attention for regions of 16..64 tokens
// (blog "BiFormer Reshapes Visual Attention with Bi-Level Routing", Part 2
// section 2.2, step 4: gather the routed key-value regions, then token
// attention over them).
//
// Tiling.  A tile is two 64-row halves; a half holds Gq whole query regions
// (Gq * n <= 64) of one (batch, head).  With an even number of heads the two
// halves are the heads 2j and 2j + 1 of the same regions (head pairing): the
// query tokens then arrive as one 128-byte-row box per region (both heads'
// 64 channels, 128-byte swizzle) and each half's Q K^T reads its own 64-byte
// column range of those rows; otherwise the halves are consecutive region
// groups of one head with 64-byte query rows.  Each
// query region r brings its own key list: the tokens of its routed regions
// I^r[r][0..topk), kn = topk * n keys, stacked slot after slot, so half h
// multiplies Q_h [64 x 32] by K_h^T [32 x Gq*kn] with one M = 64 tcgen05.mma
// per 16 channels.  The two halves' accumulators share TMEM columns: half 0
// lands in lanes 0-15 of each 32-lane quadrant, half 1 in lanes 16-31.  Row
// m of a half belongs to slot m / n, so its valid scores are exactly the
// window [slot * kn, slot * kn + kn) of its TMEM row -- one 16-row group
// never straddles two slots because n is a multiple of 16, which makes the
// window the same for all lanes of a warp.  No score outside a window is
// ever read, and P is zero outside the windows (each P row only ever writes
// its own window), so O_h = P_h V_h (M = 64, N = 32) needs no masking either.
// With several regions per half and windows of 64 keys or more, P is kept
// compact instead (each row holds only its own window) and P V runs as one
// accumulator per region -- compact P times that region's V window, rows of
// other regions computing values no one reads -- so P is Gq times smaller and
// the dependent 16-key steps of one accumulator are kn / 16, not Gq * kn / 16.
//
// Roles (one CTA per SM, tiles strided by the grid):
//   warps 0-1  producers, tiles alternating between them: read the tile's
//              routes (prefetched into shared memory), then issue TMA box
//              loads of the query regions and of every routed key/value
//              region straight from the [B, H, W, C] maps into a ring of
//              shared-memory stages (64-byte swizzle), completion counted on
//              the stage's mbarrier;
//   warp 2     one lane issues S = Q K^T for every tile as soon as it lands;
//   warp 3     one lane issues O = P V (with the row sums of P) for every tile
//              as soon as its P is written, then releases the stage;
//   then 1, 2 or 4 softmax warp groups, one query row per thread: read the
//              row's window of S, base-2 softmax, P as bf16 into 128-byte
//              swizzled shared memory, then O = (P V) / l to global memory.
// Every mbarrier wait is bounded; on expiry the kernel records
// kDevTimeout, stops all roles, drains its MMAs and frees TMEM.
#include <cuda.h>
#include <stdlib.h>

#include "attend_tc.h"
#include "kernels.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace bra {
namespace {

constexpr int kMaxSlots = 4;    // 64 rows / 16 tokens
constexpr int kMaxRoutes = 16;  // kn <= 256 with n >= 16
constexpr int kMaxStages = 12;
constexpr int kMaxSBuf = 8;
constexpr uint32_t kWait = 1u << 22;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kSmemBudget = 227 * 1024;

struct StackPlan {
    int Gq;                 // query regions per half
    int cp;                 // 1: compact P (each row keeps only its kn-key window; Gq > 1, kn >= 64)
    int kn;                 // keys per query region
    int N;                  // keys per half = Gq * kn (MMA N of Q K^T)
    int hp;                 // 1: halves are a head pair (heads even), 0: region groups of one head
    int halves;             // region groups (of Gq regions) per (batch, head)
    int tiles_bh;           // tiles per (batch, head) or, head-paired, per (batch, head pair)
    int tiles;              // all tiles
    int stages;             // shared-memory ring depth
    int nsb;                // S buffers in TMEM
    int np;                 // P buffers in shared memory
    int items;              // (slot, route) pairs of a tile: 2 * Gq * topk <= 32
    int wgs;                // softmax warp groups (1 or 2)
    int pdepth;             // P buffers per warp group (2: a tile's epilogue waits one tile)
    int nprod;              // producer warps in use: min(kProd, stages)
    uint32_t stage_bytes;   // Q (2 x 64 rows) + K + V of one tile
    uint32_t k_off, v_off;  // offsets inside a stage
    uint32_t p_half;        // one half of a P buffer: ceil(N / 64) atoms of 64 rows x 128 B
    int pin;                // 1: a tile's P is written over its own stage's Q and K (dead once S is done)
    uint32_t p_off;         // offset of the separate P buffers (pin == 0)
    uint32_t ones_off;      // offset of a bf16 ones tile [16][N] (row sums of P by MMA)
    uint32_t bar_off;       // offset of barriers and tile metadata
    uint32_t smem_bytes;    // dynamic shared memory requested (incl. alignment slack)
    uint32_t tmem_cols;     // nsb S buffers of N columns, rounded up to a power of two
    // local context term in the epilogue (8 x 8 regions, head-paired, one region per half)
    int lce;
    uint32_t lce_w_off;     // weights [25][C] fp32 (tap-major), then bias [C]
    uint32_t lce_off;       // per group: V halo | O tile | row flags (kLceGroupBytes)
};

// The local context term fused into the epilogue.  A tile is one 8 x 8 region
// of a head pair (64 channels); its softmax group writes the normalised O
// rows to shared memory, a TMA box brings the region's V with a halo of 2
// (12 x 12 tokens x 64 channels, zero outside the map), and the group's four
// warps apply the 5 x 5 depthwise filter: lane = channel pair, warp = two
// output rows, the five taps of a filter row reused along the halo row.
constexpr int kLceSide = 12;                                      // 8 + 2 * 2
constexpr uint32_t kLceHaloBytes = kLceSide * kLceSide * 128;     // 18 KB, 128-byte token rows
constexpr uint32_t kLceORow = 68;                                 // O tile row stride in floats
constexpr uint32_t kLceOBytes = 64 * kLceORow * 4;                // 17 KB
constexpr uint32_t kLceGroupBytes = kLceHaloBytes + kLceOBytes + 1024;  // + row flags

struct TileMeta {
    int b, h[2];                   // batch, head of each half
    int reg[2][kMaxSlots];         // query region of each slot, -1 if none
    uint32_t live[2][kMaxSlots];   // bit m: route m loaded (in range, first occurrence)
};

constexpr int kProd = 2;   // producer warps (tiles alternate between them)
constexpr int kCtrl = kProd + 2;  // + the S issuer warp and the P V issuer warp
constexpr int kRouteAhead = 4;    // tiles of routes a producer warp has in flight

struct Barriers {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t s_full[kMaxSBuf], o_full[kMaxSBuf], s_free[kMaxSBuf];
    uint64_t p_full[4];
    uint64_t drain[2];
    uint64_t halo_full[4];  // a group's V halo landed
    uint64_t gsync[4];      // the 128 threads of a group meet
    uint64_t wready;        // the filter weights are in shared memory
    TileMeta meta[kMaxStages];
    int32_t routes[kProd][kRouteAhead][32];  // per producer warp: routes of its next tiles
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

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, Barriers* sb,
                                              int* status) {
    for (uint32_t i = 0; i < kWait; ++i) {
        if (ptx::mbar_try_wait(bar, parity)) return true;
        if ((i & 1023) == 1023 && aborted(sb)) return false;
    }
    set_abort(sb, status);
    return false;
}

// Per-row state kept from a tile's softmax until its epilogue.
struct RowState {
    int region, b, h;
};


// WGS softmax warp groups (1, 2 or 4); KN64: every window is exactly 64 keys;
// CP: compact P with one P V accumulator per query region.
// Two fp32 lanes in one 64-bit register (x in the low half); fma.rn.f32x2
// multiplies and adds both, each rounded as fmaf would.
__device__ __forceinline__ uint64_t lce_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void lce_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t lce_fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// LCE: the local context term in the epilogue (th: V halo boxes; lce_weight,
// lce_bias: the filter's weights [C][5][5] and bias [C] or null).
template <int WGS, bool KN64, bool CP, bool LCE>
__global__ void __launch_bounds__(32 * kCtrl + 128 * WGS, 1)
bra_attend_stack_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                        const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap th,
                        const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ o,
                        const float* __restrict__ lce_weight, const float* __restrict__ lce_bias, Geometry g,
                        StackPlan p, int* status) {
    constexpr int kThreads = 32 * kCtrl + 128 * WGS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_addr(smem);
    Barriers* sb = reinterpret_cast<Barriers*>(smem + p.bar_off);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int my_tiles =
        (int)blockIdx.x < p.tiles ? (p.tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.stages; ++s) {
            ptx::mbar_init(&sb->full[s], 1);
            ptx::mbar_init(&sb->empty[s], 1);
        }
        for (int b = 0; b < p.nsb; ++b) {
            ptx::mbar_init(&sb->s_full[b], 1);
            ptx::mbar_init(&sb->o_full[b], 1);
            ptx::mbar_init(&sb->s_free[b], 128);
        }
        for (int b = 0; b < p.np; ++b) ptx::mbar_init(&sb->p_full[b], 128);
        ptx::mbar_init(&sb->drain[0], 1);
        ptx::mbar_init(&sb->drain[1], 1);
        if (LCE) {
            for (int x = 0; x < WGS; ++x) {
                ptx::mbar_init(&sb->halo_full[x], 1);
                ptx::mbar_init(&sb->gsync[x], 128);
            }
            ptx::mbar_init(&sb->wready, 128 * WGS);
        }
        sb->abort = 0;
        ptx::mbar_init_fence();
    }
    if (warp == kProd) {
        ptx::tmem_alloc(&sb->tmem, p.tmem_cols);
        ptx::tmem_relinquish();
        ptx::tc_fence_before();
    }
    // Zero, once, what must not hold stale bits: the V rows of every stage (a
    // dead route's P entries are zero, and 0 times a stale non-finite value
    // would not be) and, when P is block-diagonal, the P buffers (zero outside
    // each row's window).  Stale Q or K rows only reach scores no row reads.
    {
        const uint32_t v_chunks = (p.stage_bytes - p.v_off) / 16;
        for (uint32_t i = threadIdx.x; i < (uint32_t)p.stages * v_chunks; i += kThreads) {
            const uint32_t st = i / v_chunks, c = i - st * v_chunks;
            reinterpret_cast<uint4*>(smem + st * p.stage_bytes + p.v_off)[c] = make_uint4(0, 0, 0, 0);
        }
        if (!CP && p.Gq > 1)
            for (uint32_t i = p.p_off / 16 + threadIdx.x; i < p.ones_off / 16; i += kThreads)
                reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
    }
    // A tile of bf16 ones (same shape as one V half): P times it gives every
    // row's sum of P on the tensor core.
    for (uint32_t i = p.ones_off / 16 + threadIdx.x; i < p.lce_w_off / 16; i += kThreads)
        reinterpret_cast<uint4*>(smem)[i] = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
    ptx::fence_proxy_async_smem();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sb->tmem;
    // Everything above overlaps the routing kernel; from here on the routes
    // are read and O is written.
    grid_dependency_wait();
    if (warp < kProd) {
        // ------------------------------------------------------------ producer
        // Producer warp w loads tiles w, w + kProd, ...  Lane j first owns item
        // j = (half, slot, route m) of the tile (reads its route, checks it),
        // then the tile's boxes -- one query box per slot, one key and one value
        // box per live item -- go out one box per lane in a single TMA
        // instruction (copies from one thread are processed in order, copies
        // from different lanes in parallel), rotated across tiles so that
        // successive tiles use different lanes.  Routes reach shared memory by
        // 4-byte asynchronous copies issued kRouteAhead of the warp's tiles
        // early, so the route latency is paid once, not once per tile.
        if (lane == 0 && warp == 0) {
            ptx::tma_prefetch_desc(&tq);
            ptx::tma_prefetch_desc(&tk);
            ptx::tma_prefetch_desc(&tv);
        }
        const bool item = lane < p.items;
        const int per_half = p.Gq * g.topk;
        const int half = item ? lane / per_half : 0;
        const int slot = item ? (lane / g.topk) % p.Gq : 0;
        const int m = item ? lane % g.topk : 0;
        const int lane0 = lane - m;  // lane of route 0 of this slot
        const uint32_t slot_lanes = (g.topk >= 32 ? 0xffffffffu : ((1u << g.topk) - 1u)) << lane0;
        const uint32_t nbytes_region = (uint32_t)g.n * 64u;        // one head of a region
        const int nq = p.hp ? p.Gq : 2 * p.Gq;                     // query boxes of a tile
        const uint32_t qbytes_box = p.hp ? 2u * nbytes_region : nbytes_region;
        const int nboxes = nq + 2 * p.items;                       // + key and value boxes
        // Region of this lane's item in local tile i (-1: none), and the
        // asynchronous fetch of its route into ring slot (i / kProd) % kRouteAhead;
        // each fetch is one cp.async group, issued kRouteAhead tiles early.
        // (batch, head) slice of half hf of tile t and the tile's region group
        auto tile_slice = [&](int t, int hf, int& ht) -> int {
            const int u = t / p.tiles_bh, tt = t - u * p.tiles_bh;
            if (p.hp) {
                ht = tt;
                return 2 * u + hf;  // u = b * heads / 2 + head pair; b * heads + 2 * pair + hf
            }
            ht = tt * 2 + hf;
            return u;
        };
        auto item_region = [&](int i, int& bh) -> int {
            int ht = 0;
            bh = tile_slice(blockIdx.x + i * gridDim.x, half, ht);
            const int r = ht * p.Gq + slot;
            return (item && ht < p.halves && r < g.R) ? r : -1;
        };
        auto fetch = [&](int i) {
            if (i < my_tiles) {
                int bh = 0;
                const int r = item_region(i, bh);
                const int32_t* src = idx + ((size_t)bh * g.R + (r >= 0 ? r : 0)) * g.topk + m;
                ptx::cp_async4(ptx::smem_addr(&sb->routes[warp][(i / p.nprod) % kRouteAhead][lane]), src,
                               r >= 0 ? 4u : 0u);
            }
            ptx::cp_async_commit();  // an empty group past the last tile keeps the count uniform
        };
        // A stage's release k is awaited only after release k - 1 has happened
        // (the wait is on its parity), which holds when each producer warp's
        // previous tile used a stage released later: hence nprod <= stages.
        if (warp < p.nprod)
            for (int a = 0; a < kRouteAhead; ++a) fetch(warp + a * p.nprod);
        for (int i = warp; warp < p.nprod && i < my_tiles; i += p.nprod) {
            ptx::cp_async_wait_group<kRouteAhead - 1>();  // this tile's routes have landed
            int bh_unused = 0;
            const int cur_reg = item_region(i, bh_unused);
            const int cur = sb->routes[warp][(i / p.nprod) % kRouteAhead][lane];
            fetch(i + kRouteAhead * p.nprod);  // reuses the slot just read
            const int s = i % p.stages;
            if (i >= p.stages && !wait_or_abort(&sb->empty[s], ((i / p.stages) - 1) & 1, sb, status))
                break;
            const int t = blockIdx.x + i * gridDim.x;
            int ht0 = 0;
            const int bh0 = tile_slice(t, 0, ht0);  // half 0; half 1 is the next head or the same
            const int b = bh0 / g.heads, hd0 = bh0 - b * g.heads;
            const int hd1 = p.hp ? hd0 + 1 : hd0;
            const bool valid = cur_reg >= 0;
            const uint32_t bad = __ballot_sync(0xffffffffu, valid && (cur < 0 || cur >= g.R));
            const bool slot_ok = valid && !(bad & slot_lanes);
            if (valid && !slot_ok && m == 0) raise_status(status, kDevBadRoute);
            bool dup = false;
            for (int dd = 1; dd < g.topk; ++dd) {
                const int other = __shfl_up_sync(0xffffffffu, cur, dd);
                if (dd <= m && other == cur) dup = true;
            }
            const bool live = slot_ok && !dup;
            const uint32_t live_lanes = __ballot_sync(0xffffffffu, live);
            const uint32_t ok_lanes = __ballot_sync(0xffffffffu, slot_ok && m == 0);
            // query boxes: per (half, slot) with a usable route set, or, head-paired,
            // per slot whose region exists (one box serves both halves)
            const uint32_t q_lanes = p.hp ? __ballot_sync(0xffffffffu, valid && half == 0 && m == 0) : ok_lanes;
            TileMeta& M = sb->meta[s];
            if (item && m == 0) {
                M.reg[half][slot] = slot_ok ? cur_reg : -1;
                M.live[half][slot] = (live_lanes & slot_lanes) >> lane0;
            }
            if (lane == 0) {
                M.b = b;
                M.h[0] = hd0;
                M.h[1] = hd1;
            }
            const uint32_t bytes = (uint32_t)__popc(q_lanes) * qbytes_box + 2u * __popc(live_lanes) * nbytes_region;
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive_expect_tx(&sb->full[s], bytes);
            __syncwarp();
            const uint32_t stage = sbase + (uint32_t)s * p.stage_bytes;
            const int rot = (i / p.nprod * nboxes) & 31;
            for (int j0 = 0; j0 < nboxes; j0 += 32) {
                const int j = j0 + ((lane - rot) & 31);  // box this lane issues
                // the item behind box j: query box j -> slot lane (j * topk), K/V box -> item
                const int it = j < nq ? j * g.topk : (j - nq) >> 1;
                const int src = it < 32 ? it : 0;
                const int x_cur = __shfl_sync(0xffffffffu, cur, src);
                const int x_reg = __shfl_sync(0xffffffffu, cur_reg, src);
                if (j >= nboxes) continue;
                const int x_half = it / per_half, x_slot = (it / g.topk) % p.Gq, x_m = it % g.topk;
                if (j < nq) {
                    if ((q_lanes >> it) & 1u) {
                        const int ri = x_reg / g.S, rj = x_reg - ri * g.S;
                        // head-paired: 64 channels (heads hd0, hd0 + 1) of the slot's region
                        const uint32_t qoff = p.hp ? (uint32_t)x_slot * qbytes_box
                                                   : (uint32_t)x_half * 4096u + (uint32_t)x_slot * nbytes_region;
                        ptx::tma_load_4d(stage + qoff, &tq, (x_half ? hd1 : hd0) * 32, rj * g.ws, ri * g.hs, b,
                                         &sb->full[s]);
                    }
                } else if ((live_lanes >> it) & 1u) {
                    const int qi = x_cur / g.S, qj = x_cur - qi * g.S;
                    const uint32_t koff = (uint32_t)(x_half * p.N + x_slot * p.kn + x_m * g.n) * 64u;
                    const bool is_v = (j - nq) & 1;
                    ptx::tma_load_4d(stage + (is_v ? p.v_off : p.k_off) + koff, is_v ? (const void*)&tv : (const void*)&tk,
                                     (x_half ? hd1 : hd0) * 32, qj * g.ws, qi * g.hs, b, &sb->full[s]);
                }
            }
        }
        ptx::cp_async_wait_all();
    } else if (warp == kProd) {
        // ------------------------------------------------------- S = Q K^T issuer
        // One lane issues S for every tile in order as soon as the tile's stage
        // is loaded and its TMEM buffer is released; it never waits on P.
        if (lane == 0) {
            const uint32_t idesc_qk = ptx::idesc_bf16_f32(64, p.N, false, false);
            for (int i = 0; i < my_tiles; ++i) {
                const int s = i % p.stages, sbuf = i % p.nsb;
                if (!wait_or_abort(&sb->full[s], (i / p.stages) & 1, sb, status)) break;
                if (i >= p.nsb && !wait_or_abort(&sb->s_free[sbuf], ((i / p.nsb) - 1) & 1, sb, status)) break;
                ptx::tc_fence_after();
                const uint32_t stage = sbase + (uint32_t)s * p.stage_bytes;
                // halves alternate so that consecutive MMAs accumulate into different tiles
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        // A: head-paired, 128-byte rows of both heads (half h at byte 64 h);
                        // otherwise 64-byte rows, one half after the other
                        const uint64_t a = p.hp ? ptx::smem_desc(stage + half * 64 + kk * 32, 16, 1024, ptx::kSwizzle128B)
                                                : ptx::smem_desc(stage + half * 4096 + kk * 32, 16, 512, ptx::kSwizzle64B);
                        const uint64_t bd = ptx::smem_desc(stage + p.k_off + (uint32_t)half * p.N * 64 + kk * 32, 16,
                                                           512, ptx::kSwizzle64B);
                        ptx::mma_bf16(tmem + sbuf * p.N + ((uint32_t)(half * 16) << 16), a, bd, idesc_qk, kk);
                    }
                }
                ptx::mma_commit(&sb->s_full[sbuf]);
            }
            // Let every MMA this thread issued finish before TMEM is freed.
            ptx::mma_commit(&sb->drain[0]);
            ptx::mbar_wait(&sb->drain[0], 0, kWait);
        }
        __syncwarp();
    } else if (warp == kProd + 1) {
        // --------------------------------------------------- O = P V issuer
        // One lane issues P V (and the row sums P x ones) for every tile in
        // order as soon as its P is written, then releases the stage.
        if (lane == 0) {
            // N = 48: columns 0..31 are V, 32..47 come from a tile of ones, so the
            // same MMA leaves the row sums of P next to O.
            const uint32_t idesc_pv = ptx::idesc_bf16_f32(64, 48, false, true);
            const uint32_t ones = sbase + p.ones_off;
            for (int i = 0; i < my_tiles; ++i) {
                const int s = i % p.stages, sbuf = i % p.nsb, pb = i % p.np;
                if (!wait_or_abort(&sb->p_full[pb], (i / p.np) & 1, sb, status)) break;
                ptx::tc_fence_after();
                const uint32_t stage = sbase + (uint32_t)s * p.stage_bytes;
                const uint32_t pbase = p.pin ? stage : sbase + p.p_off + (uint32_t)pb * 2u * p.p_half;
                if constexpr (CP) {
                    // One accumulator per (half, region g) over g's kn-key window, the
                    // O blocks 48 columns apart; steps of all accumulators interleaved.
                    const int steps = p.kn / 16;
                    for (int kk = 0; kk < steps; ++kk) {
                        for (int gg = 0; gg < p.Gq; ++gg) {
                            const int kg = gg * steps + kk;  // 16-key step of the half's stacked keys
#pragma unroll
                            for (int half = 0; half < 2; ++half) {
                                const uint32_t d = tmem + sbuf * p.N + (uint32_t)gg * 48u + ((uint32_t)(half * 16) << 16);
                                const uint64_t a = ptx::smem_desc(pbase + half * p.p_half + (kk >> 2) * 8192 + (kk & 3) * 32,
                                                                  16, 1024, ptx::kSwizzle128B);
                                const uint32_t vaddr = stage + p.v_off + (uint32_t)half * p.N * 64 + kg * 1024;
                                const uint64_t bd = ptx::smem_desc(vaddr, ones + kg * 1024 - vaddr, 512, ptx::kSwizzle64B);
                                ptx::mma_bf16(d, a, bd, idesc_pv, kk);
                            }
                        }
                    }
                } else {
                    // Block-diagonal P: one accumulator per half over all N keys.
                    for (int kk = 0; kk < p.N / 16; ++kk) {
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            const uint32_t d = tmem + sbuf * p.N + ((uint32_t)(half * 16) << 16);
                            const uint64_t a = ptx::smem_desc(pbase + half * p.p_half + (kk >> 2) * 8192 + (kk & 3) * 32,
                                                              16, 1024, ptx::kSwizzle128B);
                            const uint32_t vaddr = stage + p.v_off + (uint32_t)half * p.N * 64 + kk * 1024;
                            const uint64_t bd = ptx::smem_desc(vaddr, ones + kk * 1024 - vaddr, 512, ptx::kSwizzle64B);
                            ptx::mma_bf16(d, a, bd, idesc_pv, kk);
                        }
                    }
                }
                ptx::mma_commit(&sb->o_full[sbuf]);
                ptx::mma_commit(&sb->empty[s]);
            }
            ptx::mma_commit(&sb->drain[1]);
            ptx::mbar_wait(&sb->drain[1], 0, kWait);
        }
        __syncwarp();
    } else {
        // --------------------------------------------------- softmax + epilogue
        // Warp group wg owns tiles wg, wg + WGS, ...; with two groups one
        // group's P V and epilogue overlap the other group's softmax.
        const int wg = (warp - kCtrl) >> 2;
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        const int half = lane >> 4;
        const int m = 16 * q + (lane & 15);  // row within the half
        const int slot = m / g.n;            // same for the whole warp
        const int tok = m - slot * g.n;
        const bool slot_ok = slot < p.Gq;
        const uint32_t lane_addr = (uint32_t)(32 * q) << 16;
        const uint32_t full_live = g.topk >= 32 ? 0xffffffffu : ((1u << g.topk) - 1u);
        const float sl = kLog2e * rsqrtf(32.f);
        // local context term: the filter in shared memory, tap-major ([25][C]
        // fp32, then the bias), staged once by all softmax threads
        float* lce_w = reinterpret_cast<float*>(smem + p.lce_w_off);
        uint8_t* lce_grp = smem + p.lce_off + (uint32_t)wg * kLceGroupBytes;  // halo | O tile | flags
        float* lce_o = reinterpret_cast<float*>(lce_grp + kLceHaloBytes);
        uint8_t* lce_ok = lce_grp + kLceHaloBytes + kLceOBytes;  // [token][half]: the row was written
        uint32_t gsync_phase = 0, halo_phase = 0, halo_issued = 0;
        bool lce_failed = false;
        // the group's 128 threads meet (bounded wait; false once the kernel aborts)
        auto group_sync = [&]() -> bool {
            ptx::mbar_arrive(&sb->gsync[wg]);
            return wait_or_abort(&sb->gsync[wg], (gsync_phase++) & 1, sb, status);
        };
        if (LCE) {
            const int n_st = 128 * WGS, st_i = (int)threadIdx.x - 32 * kCtrl;
            for (int x = st_i; x < 25 * g.C; x += n_st) {
                const int tap = x / g.C, c = x - tap * g.C;
                lce_w[x] = __ldg(lce_weight + c * 25 + tap);
            }
            for (int c = st_i; c < g.C; c += n_st) lce_w[25 * g.C + c] = lce_bias ? __ldg(lce_bias + c) : 0.f;
            ptx::mbar_arrive(&sb->wready);
            if (!wait_or_abort(&sb->wready, 0, sb, status)) lce_failed = true;
        }

        // O = (P V) / l for tile j, then release its TMEM buffer.
        auto epilogue = [&](int j, const RowState& st) -> bool {
            const int sbuf = j % p.nsb;
            if (!wait_or_abort(&sb->o_full[sbuf], (j / p.nsb) & 1, sb, status)) return false;
            ptx::tc_fence_after();
            // l (column 32) with O columns 0-15, then O columns 16-31: no more
            // than 17 accumulator words are held at a time.
            uint32_t r[16], lw = 0;
            const uint32_t o_col = sbuf * p.N + (CP ? (uint32_t)slot * 48u : 0u);  // this row's O block
            if (slot_ok) {
                ptx::tmem_ld16(tmem + lane_addr + o_col, r);
                lw = ptx::tmem_ld1(tmem + lane_addr + o_col + 32);
                ptx::tmem_wait17(r, lw);
            }
            const float l = __uint_as_float(lw);
            const bool write = st.region >= 0 && l > 0.f;
            const float inv = write ? 1.f / l : 0.f;
            if (LCE) {
                // the normalised row (fp32) into the group's O tile; the local
                // context term is added and O stored once, after the whole tile
                float* orow = lce_o + (uint32_t)tok * kLceORow + (uint32_t)half * 32u;
#pragma unroll
                for (int h16 = 0; h16 < 2; ++h16) {
                    if (h16 == 1) {
                        ptx::tmem_ld16(tmem + lane_addr + o_col + 16, r);
                        ptx::tmem_wait16(r);
                    }
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        *reinterpret_cast<float4*>(orow + 16 * h16 + 4 * c) =
                            make_float4(__uint_as_float(r[4 * c]) * inv, __uint_as_float(r[4 * c + 1]) * inv,
                                        __uint_as_float(r[4 * c + 2]) * inv, __uint_as_float(r[4 * c + 3]) * inv);
                }
                lce_ok[tok * 2 + half] = write ? 1 : 0;
                ptx::tc_fence_before();
                ptx::mbar_arrive(&sb->s_free[sbuf]);
                return true;
            }
            const size_t ooff = write ? token_offset(g, st.b, st.region, tok) + (size_t)st.h * 32 : 0;
            int4* dst = write && in_bounds(ooff + 31, map_elems(g), status) ? reinterpret_cast<int4*>(o + ooff) : nullptr;
#pragma unroll
            for (int h16 = 0; h16 < 2; ++h16) {
                if (h16 == 1 && slot_ok) {
                    ptx::tmem_ld16(tmem + lane_addr + o_col + 16, r);
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
                        __stcs(dst + 2 * h16 + c, make_int4((int)w[0], (int)w[1], (int)w[2], (int)w[3]));  // streamed: O is not re-read
                    }
                }
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(&sb->s_free[sbuf]);
            return true;
        };

        // Local context term of tile i (one 8 x 8 region, 64 channels) once its
        // O rows are in the group's O tile: lane = channel pair, this warp's
        // output rows 2q and 2q + 1; halo rows 2q .. 2q + 5 each feed the
        // output rows they are within two rows of, five taps per filter row.
        auto lce_phase = [&](int i) -> bool {
            if (!group_sync()) return false;  // every O row of the tile is in shared memory
            if (!wait_or_abort(&sb->halo_full[wg], (halo_phase++) & 1, sb, status)) return false;
            const int t = blockIdx.x + i * gridDim.x;
            const int u = t / p.tiles_bh, r = t - u * p.tiles_bh;
            const int b = u / (g.heads / 2), hd0 = 2 * (u - b * (g.heads / 2));
            const int ri = r / g.S, rj = r - ri * g.S;
            const int c0 = hd0 * 32 + 2 * lane;  // this lane's channels c0, c0 + 1
            uint64_t acc[2][8];
            {
                const float2 bias = *reinterpret_cast<const float2*>(lce_w + 25 * g.C + c0);
#pragma unroll
                for (int orow = 0; orow < 2; ++orow)
#pragma unroll
                    for (int x = 0; x < 8; ++x) {
                        const float2 ov =
                            *reinterpret_cast<const float2*>(lce_o + (uint32_t)((2 * q + orow) * 8 + x) * kLceORow + 2 * lane);
                        acc[orow][x] = lce_pack(ov.x + bias.x, ov.y + bias.y);
                    }
            }
#pragma unroll
            for (int hr = 0; hr < 6; ++hr) {
                const uint8_t* hrow = lce_grp + (uint32_t)(2 * q + hr) * (kLceSide * 128u) + 4u * lane;
                uint64_t hv[kLceSide];
#pragma unroll
                for (int hx = 0; hx < kLceSide; ++hx) {
                    const uint32_t w2 = *reinterpret_cast<const uint32_t*>(hrow + hx * 128);
                    hv[hx] = lce_pack(__uint_as_float(w2 << 16), __uint_as_float(w2 & 0xffff0000u));
                }
#pragma unroll
                for (int orow = 0; orow < 2; ++orow) {
                    const int dy = hr - orow;  // filter row applied to this halo row for output row 2q + orow
                    if (dy < 0 || dy > 4) continue;
                    uint64_t wv[5];
#pragma unroll
                    for (int dx = 0; dx < 5; ++dx)
                        wv[dx] = *reinterpret_cast<const uint64_t*>(lce_w + (dy * 5 + dx) * g.C + c0);
#pragma unroll
                    for (int x = 0; x < 8; ++x)
#pragma unroll
                        for (int dx = 0; dx < 5; ++dx) acc[orow][x] = lce_fma2(wv[dx], hv[x + dx], acc[orow][x]);
                }
            }
#pragma unroll
            for (int orow = 0; orow < 2; ++orow)
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const int tk = (2 * q + orow) * 8 + x;
                    if (!lce_ok[tk * 2 + (lane >> 4)]) continue;  // the attention row was not written
                    const size_t off = (((size_t)b * g.H + ri * 8 + 2 * q + orow) * g.W + rj * 8 + x) * g.C + c0;
                    if (!in_bounds(off + 1, map_elems(g), status)) continue;
                    float lo, hi;
                    lce_unpack(acc[orow][x], lo, hi);
                    *reinterpret_cast<uint32_t*>(o + off) = ptx::pack_bf16x2(lo, hi);
                }
            return group_sync();  // the tile's O tile and halo are free again
        };

        RowState prev = {-1, 0, 0};
        bool ok = !lce_failed;
        int last = -1;
        for (int i = wg; ok && i < my_tiles; i += WGS) {
            const int s = i % p.stages, sbuf = i % p.nsb, pb = i % p.np;
            if (LCE && q == 0 && lane == 0) {
                // this tile's region with a halo of 2, both heads (the group's
                // previous tile is done with the buffer: its last group_sync)
                const int t = blockIdx.x + i * gridDim.x;
                const int u = t / p.tiles_bh, r = t - u * p.tiles_bh;  // one region per tile
                const int b = u / (g.heads / 2), hd0 = 2 * (u - b * (g.heads / 2));
                const int ri = r / g.S, rj = r - ri * g.S;
                ptx::mbar_arrive_expect_tx(&sb->halo_full[wg], kLceHaloBytes);
                ptx::tma_load_4d(ptx::smem_addr(lce_grp), &th, hd0 * 32, rj * 8 - 2, ri * 8 - 2, b, &sb->halo_full[wg]);
                ++halo_issued;
            }
            if (!wait_or_abort(&sb->full[s], (i / p.stages) & 1, sb, status)) break;
            if (!wait_or_abort(&sb->s_full[sbuf], (i / p.nsb) & 1, sb, status)) break;
            ptx::tc_fence_after();
            const TileMeta& M = sb->meta[s];
            RowState cur;
            cur.region = slot_ok ? M.reg[half][slot] : -1;
            cur.b = M.b;
            cur.h = M.h[half];
            const uint32_t live = slot_ok ? M.live[half][slot] : 0u;
            const bool all_live = live == full_live;
            if (slot_ok) {
                const uint32_t col0 = sbuf * p.N + slot * p.kn;
                const uint32_t pbuf = p.pin ? sbase + (uint32_t)s * p.stage_bytes : sbase + p.p_off + (uint32_t)pb * 2u * p.p_half;
                const uint32_t prow = pbuf + half * p.p_half + m * 128;
                // 16 p values of window columns c .. c + 15 as 8 bf16 pairs: two
                // 16-byte chunks of the row's 128-byte swizzled atom line.
                auto write_p16 = [&](int c, const uint32_t* packed) {
                    const int col = CP ? c : slot * p.kn + c;  // column of the row's P
                    const uint32_t atom = prow + (uint32_t)(col >> 6) * 8192u;
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int chunk = ((col & 63) >> 3) + cc;
                        ptx::st_shared_v4(atom + ((chunk ^ (m & 7)) << 4), packed[4 * cc], packed[4 * cc + 1],
                                          packed[4 * cc + 2], packed[4 * cc + 3]);
                    }
                };
                if (KN64 && __all_sync(0xffffffffu, all_live)) {
                    // Every route of every row of this warp is live: no masks.
                    // TMEM is read 16 columns at a time (max pass, then p pass),
                    // each read waited on before the next is issued.
                    float m8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) m8[e] = -INFINITY;
#pragma unroll
                    for (int c = 0; c < 64; c += 16) {
                        uint32_t r[16];
                        ptx::tmem_ld16(tmem + lane_addr + col0 + c, r);
                        ptx::tmem_wait16(r);
#pragma unroll
                        for (int e = 0; e < 16; ++e) m8[e & 7] = fmaxf(m8[e & 7], __uint_as_float(r[e]));
                    }
                    const float msl = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                                            fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7]))) * sl;
                    // p = 2^(s * sl - max) in fp32, rounded once to bf16: P enters the
                    // MMA as bf16, and the row sums come from the same bf16 values (P x ones).
#pragma unroll
                    for (int c = 0; c < 64; c += 16) {
                        uint32_t r[16];
                        ptx::tmem_ld16(tmem + lane_addr + col0 + c, r);
                        ptx::tmem_wait16(r);
                        uint32_t packed[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            packed[e] = ptx::pack_bf16x2(ptx::ex2(fmaf(__uint_as_float(r[2 * e]), sl, -msl)), ptx::ex2(fmaf(__uint_as_float(r[2 * e + 1]), sl, -msl)));
                        write_p16(c, packed);
                    }
                } else {
                    // 16-column segment c / 16 of the window belongs to route c * 16 / n
                    // (n is a multiple of 16); a dead route's scores are skipped.
                    auto seg_live = [&](int c) -> bool { return (live >> ((c >> 4) * 16 / g.n)) & 1u; };
                    float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                    for (int c = 0; c < p.kn; c += 16) {
                        uint32_t r[16];
                        ptx::tmem_ld16(tmem + lane_addr + col0 + c, r);
                        ptx::tmem_wait16(r);
                        if (seg_live(c)) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) m4[e & 3] = fmaxf(m4[e & 3], __uint_as_float(r[e]));
                        }
                    }
                    const float msl = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl;
                    for (int c = 0; c < p.kn; c += 16) {
                        uint32_t r[16];
                        ptx::tmem_ld16(tmem + lane_addr + col0 + c, r);
                        ptx::tmem_wait16(r);
                        const bool on = seg_live(c);
                        uint32_t packed[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            // fp32 exponentials, rounded to bf16
                            const float p0 = on ? ptx::ex2(fmaf(__uint_as_float(r[2 * e]), sl, -msl)) : 0.f;
                            const float p1 = on ? ptx::ex2(fmaf(__uint_as_float(r[2 * e + 1]), sl, -msl)) : 0.f;
                            packed[e] = ptx::pack_bf16x2(p0, p1);
                        }
                        write_p16(c, packed);
                    }
                }
            }
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            ptx::mbar_arrive(&sb->p_full[pb]);
            if (WGS < 4 && p.pdepth == 2) {  // four groups always run one P buffer each
                // This group's previous tile finishes while this tile's P V runs.
                if (last >= 0) ok = epilogue(last, prev);
                prev = cur;
                last = i;
            } else {
                ok = epilogue(i, cur);
                if (LCE && ok) ok = lce_phase(i);
            }
        }
        if (ok && last >= 0) epilogue(last, prev);
        // a halo load issued for a tile whose filter phase never ran must land
        // before the CTA exits
        if (LCE && q == 0 && lane == 0 && halo_phase < halo_issued)
            ptx::mbar_wait(&sb->halo_full[wg], halo_phase & 1, kWait);
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == kProd) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, p.tmem_cols);
    }
}

bool make_stack_plan(const Geometry& g, int max_groups, bool lce, StackPlan* p) {
    if (g.d != 32 || g.n % 16 != 0 || g.n > 64) return false;
    // the fused local context term: 8 x 8 regions, head pairs, one region per
    // half, the filter of at most 128 channels in shared memory
    if (lce && (g.ws != 8 || g.hs != 8 || g.heads % 2 != 0 || g.C > 128)) return false;
    p->lce = lce ? 1 : 0;
    const int kn = g.topk * g.n;
    if (kn > 256 || kn % 32 != 0 || g.topk > kMaxRoutes) return false;
    p->kn = kn;
    p->Gq = 64 / g.n;
    if (p->Gq * kn > 256) p->Gq = 256 / kn;
    if (p->Gq > g.R) p->Gq = g.R;
    if (p->Gq < 1) return false;
    p->items = 2 * p->Gq * g.topk;
    if (p->items > 32) return false;
    p->N = p->Gq * kn;
    if (p->N < 64) return false;  // the O block (32 columns) and its row sums (16) reuse S
    p->hp = g.heads % 2 == 0 ? 1 : 0;
    p->halves = (g.R + p->Gq - 1) / p->Gq;
    p->tiles_bh = p->hp ? p->halves : (p->halves + 1) / 2;
    const long long tiles = (long long)g.B * (p->hp ? g.heads / 2 : g.heads) * p->tiles_bh;
    if (tiles > 0x7fffffffLL) return false;
    p->tiles = (int)tiles;
    const uint32_t kv = (uint32_t)2 * p->N * 64;  // two halves of N rows of 64 B
    p->k_off = 8192;
    p->v_off = 8192 + kv;
    p->stage_bytes = 8192 + 2 * kv;
    p->cp = (p->Gq > 1 && kn >= 64) ? 1 : 0;  // Gq O blocks of 48 columns fit in the N S columns
    p->p_half = (uint32_t)(((p->cp ? kn : p->N) + 63) / 64) * 8192u;
    const uint32_t misc = (uint32_t)((sizeof(Barriers) + 1023) / 1024 * 1024);
    const uint32_t ones_bytes = (uint32_t)p->N * 64u;  // N keys x 64 B of bf16 ones
    if (512 / p->N < 2) return false;
    p->nsb = 512 / p->N >= kMaxSBuf ? kMaxSBuf : 512 / p->N;
    // Softmax warp groups x P buffers per group, most overlap first, as long
    // as the load ring keeps enough stages to feed that many groups.  Waits
    // on a barrier's parity need the barrier's previous phase complete: a
    // group's earlier tiles must cover the tile `stages` (and `nsb`) before,
    // so groups <= stages and nsb a multiple of the groups.
    // P goes over its own stage's Q and K once S = Q K^T is done reading them,
    // when it fits there and needs no zero fill (a block-diagonal P is zero
    // outside each row's window, which separate buffers keep from the start).
    p->pin = (p->cp || p->Gq == 1) && 2u * p->p_half <= p->v_off ? 1 : 0;
    static const int kOptions[6][3] = {{4, 1, 5}, {2, 2, 3}, {2, 1, 3}, {1, 2, 3}, {2, 1, 2}, {1, 1, 2}};
    // the filter ([25][C] weights and the bias) and, per group, the halo, the O tile and row flags
    const uint32_t lce_w_bytes = lce ? ((26u * (uint32_t)g.C * 4u + 1023u) & ~1023u) : 0u;
    int stages = 0;
    bool found = false;
    for (int o = 0; o < 6 && !found; ++o) {
        // a group holds one S buffer per tile whose epilogue is pending
        if (kOptions[o][0] > max_groups || p->nsb % kOptions[o][0] != 0 ||
            p->nsb < kOptions[o][0] * kOptions[o][1])
            continue;
        if (lce && (kOptions[o][1] != 1 || p->Gq != 1 || !p->hp)) continue;  // the filter phase follows each epilogue
        p->wgs = kOptions[o][0];
        p->pdepth = kOptions[o][1];
        p->np = p->wgs * p->pdepth;
        const uint32_t pbytes = p->pin ? 0u : (uint32_t)p->np * 2u * p->p_half;
        const uint32_t lce_bytes = lce ? lce_w_bytes + (uint32_t)p->wgs * kLceGroupBytes : 0u;
        const uint32_t used = 1024 + misc + ones_bytes + pbytes + lce_bytes;
        stages = used < kSmemBudget ? (int)((kSmemBudget - used) / p->stage_bytes) : 0;
        found = stages >= kOptions[o][2] && stages >= p->wgs;
    }
    if (!found) return false;
    if (stages > kMaxStages) stages = kMaxStages;
    p->stages = stages;
    p->p_off = (uint32_t)stages * p->stage_bytes;
    p->ones_off = p->p_off + (p->pin ? 0u : (uint32_t)p->np * 2u * p->p_half);
    p->lce_w_off = p->ones_off + ones_bytes;
    p->lce_off = p->lce_w_off + lce_w_bytes;
    p->bar_off = p->lce_off + (lce ? (uint32_t)p->wgs * kLceGroupBytes : 0u);
    p->smem_bytes = p->bar_off + (uint32_t)sizeof(Barriers) + 1024;
    p->nprod = stages < kProd ? stages : kProd;
    uint32_t cols = 32;
    while (cols < (uint32_t)(p->nsb * p->N)) cols <<= 1;
    p->tmem_cols = cols;
    return cols <= 512;
}

}  // namespace

namespace {

// One launch of the stack kernel; ``weight`` non-null selects the variant with
// the local context term in the epilogue.
bra_status stack_launch(const Geometry& g, const void* q, const void* k, const void* v, const float* weight,
                        const float* bias, const int32_t* idx, void* o, int* status, cudaStream_t stream) {
    // BRA_STACK_GROUPS caps the softmax warp groups (1, 2 or 4; default 4).
    int max_groups = 4;
    if (const char* env = getenv("BRA_STACK_GROUPS")) {
        const int v = atoi(env);
        if (v >= 1 && v <= 4) max_groups = v;
    }
    const bool lce = weight != nullptr;
    StackPlan p;
    if (!make_stack_plan(g, max_groups, lce, &p)) return BRA_ERR_UNSUPPORTED;
    CUtensorMap tq, tk, tv, th;
    if (!encode_region_map(&tq, q, g.B, g.H, g.W, g.C, g.ws, g.hs, p.hp ? 64 : 32) ||
        !encode_region_map(&tk, k, g.B, g.H, g.W, g.C, g.ws, g.hs, 32) ||
        !encode_region_map(&tv, v, g.B, g.H, g.W, g.C, g.ws, g.hs, 32))
        return BRA_ERR_UNSUPPORTED;
    if (lce) {
        if (!encode_halo_map(&th, v, g.B, g.H, g.W, g.C, kLceSide, kLceSide)) return BRA_ERR_UNSUPPORTED;
    } else {
        th = tv;  // unused
    }
    const int sms = sm_count();
    if (sms <= 0) return BRA_ERR_CUDA;
    const int grid = p.tiles < sms ? p.tiles : sms;
    using KernelFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, const int32_t*, __nv_bfloat16*,
                              const float*, const float*, Geometry, StackPlan, int*);
    // [cp][groups 1, 2, 4][kn == 64]
    static const KernelFn kKernels[2][3][2] = {
        {{bra_attend_stack_kernel<1, false, false, false>, bra_attend_stack_kernel<1, true, false, false>},
         {bra_attend_stack_kernel<2, false, false, false>, bra_attend_stack_kernel<2, true, false, false>},
         {bra_attend_stack_kernel<4, false, false, false>, bra_attend_stack_kernel<4, true, false, false>}},
        {{bra_attend_stack_kernel<1, false, true, false>, bra_attend_stack_kernel<1, true, true, false>},
         {bra_attend_stack_kernel<2, false, true, false>, bra_attend_stack_kernel<2, true, true, false>},
         {bra_attend_stack_kernel<4, false, true, false>, bra_attend_stack_kernel<4, true, true, false>}}};
    // with the local context term: one region per half (no compact P), one or two groups
    static const KernelFn kLceKernels[2][2] = {
        {bra_attend_stack_kernel<1, false, false, true>, bra_attend_stack_kernel<1, true, false, true>},
        {bra_attend_stack_kernel<2, false, false, true>, bra_attend_stack_kernel<2, true, false, true>}};
    KernelFn kernel;
    if (lce) {
        if (p.cp || p.wgs > 2) return BRA_ERR_UNSUPPORTED;
        kernel = kLceKernels[p.wgs - 1][p.kn == 64 ? 1 : 0];
    } else {
        kernel = kKernels[p.cp][p.wgs == 4 ? 2 : p.wgs - 1][p.kn == 64 ? 1 : 0];
    }
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem_bytes) !=
        cudaSuccess)
        return BRA_ERR_CUDA;
    const cudaError_t e = launch_after_previous(kernel, dim3(grid), dim3(32 * kCtrl + 128 * p.wgs), p.smem_bytes,
                                                stream, tq, tk, tv, th, idx, static_cast<__nv_bfloat16*>(o), weight,
                                                bias, g, p, status);
    return e == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

}  // namespace

bra_status attend_stack_launch(const Geometry& g, const void* q, const void* k, const void* v,
                               const int32_t* idx, void* o, int* status, cudaStream_t stream) {
    return stack_launch(g, q, k, v, nullptr, nullptr, idx, o, status, stream);
}

bool attend_stack_lce_covers(const Geometry& g) {
    StackPlan p;
    return make_stack_plan(g, 4, true, &p) && !p.cp && p.wgs <= 2;
}

bra_status attend_stack_lce_launch(const Geometry& g, const void* q, const void* k, const void* v,
                                   const float* weight, const float* bias, const int32_t* idx, void* o, int* status,
                                   cudaStream_t stream) {
    if (!weight) return BRA_ERR_INVALID_ARG;
    return stack_launch(g, q, k, v, weight, bias, idx, o, status, stream);
}

}  // namespace bra
