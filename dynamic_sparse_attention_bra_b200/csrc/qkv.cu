// Q, K, V projection fused with the region means that routing reads (blog
// "BiFormer Reshapes Visual Attention with Bi-Level Routing", Part 2 section
// 2.2 steps 2-3 and pseudocode steps 2-3): [Q | K | V] = X W^T (+ b) on the
// 5th-generation tensor cores, and in the same pass Q^r, K^r = the per-region
// means of the stored (bf16) Q and K.  The separate pooling pass, which reads
// Q and K back from HBM, is not needed after it.
//
// Work unit: a box of whole regions of one image, at most 128 tokens (one
// TMEM lane each):
//   - regions of n <= 128 tokens, kx = 128 / n of them side by side when
//     kx < S (box = kx region columns x one region row), else kb full region
//     rows (box = the full width x kb region rows);
//   - one 4-D TMA box per 64-channel block of X lands in shared memory in the
//     128-byte swizzled K-major layout the MMA reads; boxes that reach past
//     the map are zero-filled on load and clipped on store.
// Per tile, one elected thread issues D = X_tile W^T with M = 128, N = 192
// per MMA, K = 16 per step, into TMEM.  Two warpgroups share the 128 TMEM
// lanes: each reads half of the output columns of its rows, adds the bias
// and rounds to bf16 into swizzled staging buffers (one per output and
// 64-channel block), which TMA stores back; then both sum the staged Q and K
// columns of every region of the tile (deterministic, no atomics: each region
// lies in exactly one tile) and write the means.  The next tile's MMAs are
// issued as soon as this tile's rows have been read from TMEM, so they run
// under the region sums.
//
// The weights (at most 96 KB) stay resident in shared memory for the CTA's
// lifetime.  X tiles go through a ring of two buffers when C = 64 (one when
// C = 128): a buffer is refilled with the tile two (one) ahead as soon as the
// MMAs reading it have completed, so loads overlap the epilogue; two CTAs
// share an SM when C = 64.
//
// Region sums read the staging buffers with 16-byte loads: a thread sums one
// 8-channel chunk of one region over every parts-th token, and the parts
// (lanes 8 apart) are folded with shuffles; when a tile has at most 128 sum
// items the two warpgroups take alternate token parts and add their halves
// through a small shared-memory scratch.
#include "../../include/bra.h"
#include "kernels.h"
#include "qkv.h"
#include "tc_ptx.cuh"
#include "tma_host.h"

namespace bra {
namespace {

constexpr int kThreads = 256;    // two warpgroups over the 128 TMEM lanes
constexpr int kRows = 128;          // MMA M: tokens per tile
constexpr int kNChunk = 192;        // MMA N per instruction
constexpr int kBlockBytes = kRows * 128;  // one 64-channel block of 128 token rows
constexpr uint32_t kWaitLimit = 1u << 22;

struct QkvPlan {
    int bw, bh;            // token box: bw columns x bh rows of one image
    int tiles_x, tiles_y;  // boxes per region-row band, bands per image
    int nrx, nry;          // region columns / rows per box
    int rows;              // bw * bh
    int parts;             // threads that share one (region, 16-byte chunk) sum: 1, 2 or 4
    long long tiles;       // B * tiles_x * tiles_y
};

bool make_qkv_plan(const Geometry& g, QkvPlan* p) {
    if (g.n > kRows) return false;
    const int kmax = kRows / g.n;
    if (kmax >= g.S) {
        const int kb = min(g.S, kmax / g.S);
        p->bw = g.W;
        p->bh = g.hs * kb;
        p->tiles_x = 1;
        p->tiles_y = (g.S + kb - 1) / kb;
        p->nrx = g.S;
        p->nry = kb;
    } else {
        p->bw = g.ws * kmax;
        p->bh = g.hs;
        p->tiles_x = (g.S + kmax - 1) / kmax;
        p->tiles_y = g.S;
        p->nrx = kmax;
        p->nry = 1;
    }
    if (p->bw > 256 || p->bh > 256) return false;  // TMA box extent limit
    p->rows = p->bw * p->bh;
    p->tiles = (long long)g.B * p->tiles_x * p->tiles_y;
    // Pooling items: 8 chunks x parts x (Q and K blocks) x regions per tile.
    const int base = 8 * 2 * (g.C / 64) * p->nrx * p->nry;
    p->parts = 1;
    while (p->parts < 4 && base * p->parts * 2 <= kRows && p->parts * 2 <= g.n) p->parts *= 2;
    return true;
}

template <int KB>
struct Layout {
    static constexpr int C = 64 * KB;
    static constexpr int kWBytes = KB * 3 * C * 128;   // [KB][3C rows][128 B]
    static constexpr int kOffW = 0;
    static constexpr int kAStages = KB == 1 ? 2 : 1;   // X tiles in flight
    static constexpr int kOffA = kOffW + kWBytes;      // [stages][KB][128 rows][128 B]
    static constexpr int kOffOut = kOffA + kAStages * KB * kBlockBytes;  // [3][KB][128 rows][128 B]
    static constexpr int kOffBias = kOffOut + 3 * KB * kBlockBytes;
    static constexpr int kOffScratch = kOffBias + 3 * C * 4;  // [128][8] fp32 partial sums (C = 64 only)
    static constexpr int kOffMisc = kOffScratch + (KB == 1 ? kRows * 8 * 4 : 0);
    static constexpr int kBytes = kOffMisc + 48;  // afull[2], wfull, mma_done, TMEM slot
    static constexpr int kAlloc = kBytes + 1024;       // room to align the base to 1 KB
    static constexpr uint32_t kTmemCols = KB == 1 ? 256 : 512;
    static constexpr int kCtasPerSm = KB == 1 ? 2 : 1;
};

// ---- TMA stores (bulk-group completion) ----------------------------------------
__device__ __forceinline__ void tma_store_4d(const void* tmap, uint32_t src, int c0, int c1, int c2, int c3) {
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// One region-sum item of a thread: 8 channels of one Q or K block of one
// region of the tile, over the tokens first, first + stride, ...
struct SumItem {
    int pp;          // token part
    int blk;         // staging block: 0..KB-1 Q, KB..2KB-1 K
    int i, j;        // region column / row inside the tile
    int ti, xi, t;   // first token: index in the region, column in the region, row in the tile
    int o;           // 0: Q^r, 1: K^r
    int dst_off;     // (head * R) * 32 + channel within the head
    bool valid;      // e < items
};

struct TileCoord {
    int b, x0, y0;
};

__device__ __forceinline__ TileCoord tile_coord(long long t, const QkvPlan& p) {
    const long long per_image = (long long)p.tiles_x * p.tiles_y;
    const int b = (int)(t / per_image);
    const int rem = (int)(t - (long long)b * per_image);
    const int ty = rem / p.tiles_x, tx = rem - ty * p.tiles_x;
    return {b, tx * p.bw, ty * p.bh};
}

// Two fp32 lanes in one 64-bit register (x in the low half), added with one
// add.rn.f32x2 (sm_100a), each lane rounded as a scalar fp32 add would be.
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
    float2 f;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(f.x), "=f"(f.y) : "l"(v));
    return f;
}
// bf16 pair -> packed fp32 pair (a bf16 is the high half of its float)
__device__ __forceinline__ uint64_t f2_from_bf16x2(uint32_t r) {
    return f2_pack(__uint_as_float(r << 16), __uint_as_float(r & 0xffff0000u));
}

template <int KB>
__global__ void __launch_bounds__(kThreads, Layout<KB>::kCtasPerSm)
bra_qkv_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw,
               const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, const float* __restrict__ bias, float* __restrict__ qr,
               float* __restrict__ kr, Geometry g, QkvPlan p, int* status) {
    using L = Layout<KB>;
    constexpr int C = L::C;
    constexpr int kStages = L::kAStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_addr(smem);
    const uint32_t sW = sbase + L::kOffW, sA = sbase + L::kOffA, sOut = sbase + L::kOffOut;
    float* bias_s = reinterpret_cast<float*>(smem + L::kOffBias);
    float* scratch = reinterpret_cast<float*>(smem + L::kOffScratch);  // [128 items][8]
    uint64_t* afull = reinterpret_cast<uint64_t*>(smem + L::kOffMisc);  // [kStages]
    uint64_t* wfull = afull + 2;
    uint64_t* mma_done = afull + 3;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kOffMisc + 32);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, wg = warp >> 2;  // TMEM lane quadrant, warpgroup
    const uint32_t a_bytes = (uint32_t)KB * 64 * p.rows * 2;

    // ---- set-up ------------------------------------------------------------------
    // Rows past the box never receive TMA data: zero the X buffers once,
    // before the async proxy writes there.
    for (int i = tid; i < kStages * KB * kBlockBytes / 16; i += kThreads)
        reinterpret_cast<uint4*>(smem + L::kOffA)[i] = make_uint4(0, 0, 0, 0);
    for (int i = tid; i < 3 * C; i += kThreads) bias_s[i] = bias ? bias[i] : 0.f;
    ptx::fence_proxy_async_smem();
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) ptx::mbar_init(afull + s, 1);
        ptx::mbar_init(wfull, 1);
        ptx::mbar_init(mma_done, 1);
        ptx::mbar_init_fence();
    }
    if (warp == 0) {
        ptx::tmem_alloc(tmem_slot, L::kTmemCols);
        ptx::tmem_relinquish();
        ptx::tc_fence_before();
    }
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // X loads are numbered by the CTA's local tile index j (stage j % kStages,
    // parity (j / kStages) & 1).  Thread 0 alone issues and waits on them.
    uint32_t a_issued = 0, a_done = 0;
    bool w_pending = false;
    auto issue_x = [&](uint32_t j) {
        const long long t = (long long)blockIdx.x + (long long)j * gridDim.x;
        if (t >= p.tiles) return;
        const TileCoord c = tile_coord(t, p);
        const int s = (int)(j % kStages);
        ptx::mbar_arrive_expect_tx(afull + s, a_bytes);
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
            ptx::tma_load_4d(sA + (s * KB + kb) * kBlockBytes, &tx, kb * 64, c.x0, c.y0, c.b, afull + s);
        a_issued = j + 1;
    };
    if (tid == 0) {
        ptx::tma_prefetch_desc(&tx);
        ptx::tma_prefetch_desc(&tq);
        ptx::tma_prefetch_desc(&tk);
        ptx::tma_prefetch_desc(&tv);
        ptx::mbar_arrive_expect_tx(wfull, (uint32_t)(3 * C * C * 2));
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
            for (int nb = 0; nb < 3 * C / kNChunk; ++nb)
                ptx::tma_load_4d(sW + kb * 3 * C * 128 + nb * kNChunk * 128, &tw, kb * 64, nb * kNChunk, 0, 0, wfull);
        w_pending = true;
        for (int j = 0; j < kStages; ++j) issue_x(j);
    }
    bool mma_pending = false;
    // D = X_tile(j) W^T into TMEM; thread 0 only.  False if a wait gave up.
    auto issue_mma = [&](uint32_t j) -> bool {
        if (w_pending) {
            if (!ptx::mbar_wait(wfull, 0, kWaitLimit)) return false;
            w_pending = false;
        }
        const int stage = (int)(j % kStages);
        if (!ptx::mbar_wait(afull + stage, (j / kStages) & 1u, kWaitLimit)) return false;
        a_done = j + 1;
        ptx::tc_fence_after();
        constexpr uint32_t idesc = ptx::idesc_bf16_f32(kRows, kNChunk, false, false);
        const uint32_t sAs = sA + stage * KB * kBlockBytes;
#pragma unroll
        for (int nb = 0; nb < 3 * C / kNChunk; ++nb)
#pragma unroll
            for (int kb = 0; kb < KB; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks) {
                    const uint64_t a = ptx::smem_desc(sAs + kb * kBlockBytes + ks * 32, 16, 1024, ptx::kSwizzle128B);
                    const uint64_t bd = ptx::smem_desc(sW + kb * 3 * C * 128 + nb * kNChunk * 128 + ks * 32, 16, 1024,
                                                       ptx::kSwizzle128B);
                    ptx::mma_bf16(tmem + nb * kNChunk, a, bd, idesc, (kb | ks) != 0);
                }
        ptx::mma_commit(mma_done);
        mma_pending = true;
        return true;
    };
    bool ok = true;
    if (tid == 0 && blockIdx.x < p.tiles) ok = issue_mma(0);

    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const int row = tid & (kRows - 1);
    const float inv_n = 1.f / (float)g.n;
    const int parts = p.parts;
    const int pc = lane & 7;
    const int items = 8 * parts * 2 * KB * p.nrx * p.nry;
    // Tile-invariant part of a region-sum item (see the region sums below).
    auto make_item = [&](int e, int first) {
        SumItem m;
        m.pp = (e >> 3) % parts;
        const int rest = (e >> 3) / parts;
        m.blk = rest % (2 * KB);
        const int reg = rest / (2 * KB);
        m.j = reg / p.nrx;
        m.i = reg - m.j * p.nrx;
        m.valid = e < items;
        m.ti = m.pp + first;
        const int yi = m.ti / g.ws;
        m.xi = m.ti - yi * g.ws;
        m.t = (m.j * g.hs + yi) * p.bw + m.i * g.ws + m.xi;
        m.o = m.blk / KB;
        const int cin = (m.blk - m.o * KB) * 64 + pc * 8;
        m.dst_off = (cin >> 5) * g.R * 32 + (cin & 31);
        return m;
    };
    const SumItem split_item = make_item(quad * 32 + lane, wg * parts);
    uint32_t it = 0;

    for (long long tile = blockIdx.x; tile < p.tiles; tile += gridDim.x, ++it) {
        const TileCoord tc = tile_coord(tile, p);

        // ---- D = X_tile W^T was issued before the previous tile's region sums
        if (__syncthreads_or(!ok)) {
            ok = false;
            break;
        }
        ok = ptx::mbar_wait(mma_done, it & 1u, kWaitLimit);
        if (__syncthreads_or(!ok)) {
            ok = false;
            break;
        }
        ptx::tc_fence_after();
        if (tid == 0) {
            mma_pending = false;
            // This X buffer is free again: fetch the tile kStages ahead.
            issue_x(it + kStages);
            // The previous tile's stores must have read the staging buffers.
            bulk_wait_read();
        }
        __syncthreads();

        // ---- epilogue: row -> +bias -> bf16 -> swizzled staging ---------------
        // Warpgroup wg takes output columns [wg * 3C/2, (wg + 1) * 3C/2) of its
        // rows, 32 columns (four 16-byte chunks of one staging row) at a time.
#pragma unroll
        for (int k32 = 0; k32 < 3 * C / 64; ++k32) {
            const int c0 = wg * (3 * C / 2) + k32 * 32;
            uint32_t r[32];
            ptx::tmem_ld32(tmem + lane_base + c0, r);
            ptx::tmem_ld_wait();
            const int o = c0 / C, cin = c0 - o * C, kb = cin >> 6, ch0 = (cin & 63) >> 3;
            const uint32_t dst = sOut + (o * KB + kb) * kBlockBytes + row * 128;
            const float4* b4 = reinterpret_cast<const float4*>(bias_s + c0);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const float4 ba = b4[2 * cc], bb = b4[2 * cc + 1];
                const uint32_t* q = r + cc * 8;
                const float2 s0 = f2_unpack(f2_add(f2_pack(__uint_as_float(q[0]), __uint_as_float(q[1])), f2_pack(ba.x, ba.y)));
                const float2 s1 = f2_unpack(f2_add(f2_pack(__uint_as_float(q[2]), __uint_as_float(q[3])), f2_pack(ba.z, ba.w)));
                const float2 s2 = f2_unpack(f2_add(f2_pack(__uint_as_float(q[4]), __uint_as_float(q[5])), f2_pack(bb.x, bb.y)));
                const float2 s3 = f2_unpack(f2_add(f2_pack(__uint_as_float(q[6]), __uint_as_float(q[7])), f2_pack(bb.z, bb.w)));
                ptx::st_shared_v4(dst + (((ch0 + cc) ^ (row & 7)) << 4), ptx::pack_bf16x2(s0.x, s0.y),
                                  ptx::pack_bf16x2(s1.x, s1.y), ptx::pack_bf16x2(s2.x, s2.y),
                                  ptx::pack_bf16x2(s3.x, s3.y));
            }
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();
        if (tid == 0) {
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
                tma_store_4d(&tq, sOut + (0 * KB + kb) * kBlockBytes, kb * 64, tc.x0, tc.y0, tc.b);
                tma_store_4d(&tk, sOut + (1 * KB + kb) * kBlockBytes, kb * 64, tc.x0, tc.y0, tc.b);
                tma_store_4d(&tv, sOut + (2 * KB + kb) * kBlockBytes, kb * 64, tc.x0, tc.y0, tc.b);
            }
            bulk_commit();
            // TMEM is free again (every row was read before the barrier): the
            // next tile's MMAs run under this tile's region sums.
            if (tile + gridDim.x < p.tiles) ok = issue_mma(it + 1);
        }

        // ---- region means of the staged Q and K ---------------------------------
        // Item e: chunk pc = e % 8 (8 channels), part pp = (e / 8) % parts,
        // block (Q or K, 64-channel block) and region above.  A thread sums its
        // chunk over tokens first, first + stride, ... of the region; parts are
        // lanes 8 apart and are folded with shuffles (every lane of the warp
        // takes part; items past the end add zeros).  Eight consecutive lanes
        // read the eight chunks of one token row: conflict-free 16-byte loads.
        const int rx0 = tc.x0 / g.ws, ry0 = tc.y0 / g.hs;
        auto region_sum = [&](const SumItem& m, int stride, float (&out)[8], float*& dst) -> bool {
            const int rx = rx0 + m.i, ry = ry0 + m.j;
            const bool live = m.valid && rx < g.S && ry < g.S;
            uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
            int ti = m.ti;
            if (live && ti < g.n) {
                const uint8_t* buf = smem + L::kOffOut + m.blk * kBlockBytes;  // blocks 0..KB-1: Q, then K
                int xi = m.xi, t = m.t;
                for (; ti < g.n; ti += stride) {
                    const uint4 v = *reinterpret_cast<const uint4*>(buf + t * 128 + ((pc ^ (t & 7)) << 4));
                    acc[0] = f2_add(acc[0], f2_from_bf16x2(v.x));
                    acc[1] = f2_add(acc[1], f2_from_bf16x2(v.y));
                    acc[2] = f2_add(acc[2], f2_from_bf16x2(v.z));
                    acc[3] = f2_add(acc[3], f2_from_bf16x2(v.w));
                    t += stride;
                    xi += stride;
                    while (xi >= g.ws) {
                        xi -= g.ws;
                        t += p.bw - g.ws;
                    }
                }
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float2 f = f2_unpack(acc[c]);
                out[2 * c] = f.x;
                out[2 * c + 1] = f.y;
            }
            for (int off = 8; off < 8 * parts; off <<= 1)
#pragma unroll
                for (int c = 0; c < 8; ++c) out[c] += __shfl_xor_sync(0xffffffffu, out[c], off);
            dst = (m.o == 0 ? qr : kr) + ((size_t)tc.b * g.heads * g.R + ry * g.S + rx) * 32 + m.dst_off;
            return live && m.pp == 0;
        };
        auto store_mean = [&](float* dst, const float (&s)[8]) {
            reinterpret_cast<float4*>(dst)[0] = make_float4(s[0] * inv_n, s[1] * inv_n, s[2] * inv_n, s[3] * inv_n);
            reinterpret_cast<float4*>(dst)[1] = make_float4(s[4] * inv_n, s[5] * inv_n, s[6] * inv_n, s[7] * inv_n);
        };
        if (KB == 1 && items <= kRows) {
            // One item per lane of each warpgroup; the two warpgroups take
            // alternate token parts and meet in shared memory.
            const int e = quad * 32 + lane;
            float s[8];
            float* dst;
            const bool head = region_sum(split_item, 2 * parts, s, dst);
            if (wg == 1 && head) {
                reinterpret_cast<float4*>(scratch + e * 8)[0] = make_float4(s[0], s[1], s[2], s[3]);
                reinterpret_cast<float4*>(scratch + e * 8)[1] = make_float4(s[4], s[5], s[6], s[7]);
            }
            __syncthreads();
            if (wg == 0 && head) {
                const float4 u = reinterpret_cast<const float4*>(scratch + e * 8)[0];
                const float4 w = reinterpret_cast<const float4*>(scratch + e * 8)[1];
                s[0] += u.x; s[1] += u.y; s[2] += u.z; s[3] += u.w;
                s[4] += w.x; s[5] += w.y; s[6] += w.z; s[7] += w.w;
                store_mean(dst, s);
            }
        } else {
            for (int e0 = warp * 32; e0 < items; e0 += kThreads) {
                float s[8];
                float* dst;
                if (region_sum(make_item(e0 + lane, 0), parts, s, dst)) store_mean(dst, s);
            }
        }
    }

    // ---- tear-down: no copy or MMA of this CTA may still be in flight ----------
    if (tid == 0) {
        if (!ok && status) raise_status(status, kDevTimeout);
        if (mma_pending) ptx::mbar_wait(mma_done, it & 1u, kWaitLimit);
        if (w_pending) ptx::mbar_wait(wfull, 0, kWaitLimit);
        for (uint32_t j = a_done; j < a_issued; ++j)
            ptx::mbar_wait(afull + j % kStages, (j / kStages) & 1u, kWaitLimit);
        bulk_wait_all();
    }
    allow_dependents();
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, L::kTmemCols);
    }
}

template <int KB>
bra_status launch_kb(const Geometry& g, const QkvPlan& p, const CUtensorMap (&maps)[5], const float* bias, float* qr,
                     float* kr, int* status, cudaStream_t stream) {
    using L = Layout<KB>;
    static_assert(L::kAlloc <= 227 * 1024, "shared memory budget");
    auto kernel = bra_qkv_kernel<KB>;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) != cudaSuccess)
        return BRA_ERR_CUDA;
    const int sms = sm_count();
    if (sms <= 0) return BRA_ERR_CUDA;
    const long long grid = p.tiles < (long long)L::kCtasPerSm * sms ? p.tiles : (long long)L::kCtasPerSm * sms;
    kernel<<<(unsigned)grid, kThreads, L::kAlloc, stream>>>(maps[0], maps[1], maps[2], maps[3], maps[4], bias, qr, kr,
                                                            g, p, status);
    return cudaGetLastError() == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

}  // namespace

bra_status qkv_check(const Geometry& g) {
    if (g.C != 64 && g.C != 128) return BRA_ERR_UNSUPPORTED;
    QkvPlan p;
    if (!make_qkv_plan(g, &p)) return BRA_ERR_UNSUPPORTED;
    return BRA_OK;
}

bra_status qkv_launch(const Geometry& g, const void* x, const void* w, const float* bias, void* q, void* k, void* v,
                      float* qr, float* kr, int* status, cudaStream_t stream) {
    if (qkv_check(g) != BRA_OK) return BRA_ERR_UNSUPPORTED;
    QkvPlan p;
    make_qkv_plan(g, &p);
    if (p.tiles == 0) return BRA_OK;
    CUtensorMap maps[5];
    // X, Q, K, V: [B, H, W, C] boxes of 64 channels x bw x bh tokens; W as a
    // [1, 1, 3C, C] map with boxes of 64 channels x 192 output rows.
    if (!encode_region_map(&maps[0], x, g.B, g.H, g.W, g.C, p.bw, p.bh, 64) ||
        !encode_region_map(&maps[1], w, 1, 1, 3 * g.C, g.C, kNChunk, 1, 64) ||
        !encode_region_map(&maps[2], q, g.B, g.H, g.W, g.C, p.bw, p.bh, 64) ||
        !encode_region_map(&maps[3], k, g.B, g.H, g.W, g.C, p.bw, p.bh, 64) ||
        !encode_region_map(&maps[4], v, g.B, g.H, g.W, g.C, p.bw, p.bh, 64))
        return BRA_ERR_CUDA;
    return g.C == 64 ? launch_kb<1>(g, p, maps, bias, qr, kr, status, stream)
                     : launch_kb<2>(g, p, maps, bias, qr, kr, status, stream);
}

}  // namespace bra
