// Token-to-token attention over routed regions on the 5th-generation tensor
// cores (blog "BiFormer Reshapes Visual Attention with Bi-Level Routing",
// Part 2 section 2.2, step 4): O = softmax(Q K_g^T / sqrt(d)) V_g for bf16,
// head dim 32, with fp32 accumulation in TMEM.
//
// Work unit: one CTA per query tile of one (batch, head): up to 128 query
// rows (one TMEM lane each) made of G whole regions when a region has at
// most 128 tokens, or of a 128-token part of one region otherwise.  The keys
// of a tile are the union U of the routed regions of its query regions.  U
// is walked in key blocks of at most 128 keys (whole regions, or parts of a
// region); for each block
//   1. the block's K and V rows are gathered from HBM/L2 straight into shared
//      memory (cp.async, 16 B per copy) -- the gathered K/V never go back to
//      HBM;
//   2. S = Q K^T runs on tcgen05 (M = 128, N = keys, K = 32) into TMEM;
//   3. each thread reads its query's row of S, keeps only the keys of regions
//      its own region routes to (the others belong to another query region of
//      the tile), and updates a base-2 online softmax; P goes to shared memory
//      as bf16;
//   4. O_blk = P V runs on tcgen05 (M = 128, N = 32, K = keys) into TMEM and
//      is folded into the thread's fp32 output registers.
//
// Shared-memory operand layouts (bf16):
//   Q, K, V  [rows][32]: 64-byte rows, 64-byte swizzle (16-byte chunk c of
//            row r sits at chunk c ^ ((r >> 1) & 3)); Q and K are K-major
//            operands, V is the MN-major B operand of P V.
//   P        [128][keys]: 128-byte swizzled K-major atoms of 64 keys (chunk c
//            of row r at c ^ (r & 7)), one 16 KB atom per 64 keys.
#include "attend_tc.h"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace bra {
namespace {

constexpr int kThreads = 128;       // 4 warps = 128 TMEM lanes = 128 query rows
constexpr int kTileRows = 128;
constexpr int kBlockKeys = 128;
constexpr uint32_t kTmemCols = 128;  // S block (<= 128 fp32 columns); O_blk reuses 0..31
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr float kLog2e = 1.4426950408889634f;

constexpr int kQBytes = kTileRows * 64;
constexpr int kKBytes = kBlockKeys * 64;
constexpr int kPAtomBytes = kTileRows * 128;
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBytes;
constexpr int kOffV = kOffK + kKBytes;
constexpr int kOffP = kOffV + kKBytes;                     // 1024-aligned
constexpr int kOffRmask = kOffP + 2 * kPAtomBytes;         // [128][8] uint32
constexpr int kOffUlist = kOffRmask + kTileRows * 8 * 4;   // [256] int32
constexpr int kOffMisc = kOffUlist + kMaxRegions * 4;
constexpr int kSmemBytes = kOffMisc + 64;
constexpr int kSmemAlloc = kSmemBytes + 1024;              // room to align the base to 1 KB

struct TcPlan {
    int G;       // query regions per tile (1 when a region is split)
    int parts;   // parts per region (1 when n <= 128)
    int unit;    // tokens per part (n when parts == 1)
    int tiles;   // tiles per (batch, head)
    int rpb;     // key regions per block when parts == 1
};

TcPlan make_plan(const Geometry& g) {
    TcPlan p;
    if (g.n <= kTileRows) {
        p.parts = 1;
        p.unit = g.n;
        p.G = kTileRows / g.n;
        if (p.G > g.R) p.G = g.R;
        p.tiles = (g.R + p.G - 1) / p.G;
        p.rpb = kBlockKeys / g.n;
    } else {
        p.parts = (g.n + kTileRows - 1) / kTileRows;
        p.unit = (g.n + p.parts - 1) / p.parts;
        p.G = 1;
        p.tiles = g.R * p.parts;
        p.rpb = 0;
    }
    return p;
}

__device__ __forceinline__ uint32_t swz64(int row, int chunk) {
    return (uint32_t)(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
}

// m |= bits [lo, hi) of a 128-bit mask held in four registers.
__device__ __forceinline__ void set_bits(uint32_t (&m)[4], int lo, int hi) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        const int a = max(lo, 32 * w), e = min(hi, 32 * w + 32);
        if (a < e) {
            const int len = e - a;
            const uint32_t bits = len == 32 ? 0xffffffffu : ((1u << len) - 1u);
            m[w] |= bits << (a - 32 * w);
        }
    }
}

// Copies 64-byte head rows of ``count`` tokens into a swizzled [rows][32]
// buffer; row j is token ``tok`` of region ``reg`` as given by row_of(j).
template <typename RowFn>
__device__ __forceinline__ void gather_rows(uint32_t dst, const __nv_bfloat16* src, int count,
                                            const Geometry& g, int b, int h, RowFn row_of) {
    for (int e = threadIdx.x; e < count * 4; e += kThreads) {
        const int j = e >> 2, c = e & 3;
        int reg, tok;
        row_of(j, reg, tok);
        const __nv_bfloat16* p = src + token_offset(g, b, reg, tok) + (size_t)h * 32 + c * 8;
        ptx::cp_async16(dst + swz64(j, c), p);
    }
}

__global__ void __launch_bounds__(kThreads, 3)
bra_attend_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                     const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ idx,
                     __nv_bfloat16* __restrict__ o, Geometry g, TcPlan plan, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_addr(smem);
    const uint32_t sQ = sbase + kOffQ, sK = sbase + kOffK, sV = sbase + kOffV, sP = sbase + kOffP;
    uint32_t* rmask = reinterpret_cast<uint32_t*>(smem + kOffRmask);
    int* ulist = reinterpret_cast<int*>(smem + kOffUlist);
    uint64_t* mbar = reinterpret_cast<uint64_t*>(smem + kOffMisc);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc + 8);
    int* s_nu = reinterpret_cast<int*>(smem + kOffMisc + 12);
    int* s_bad = reinterpret_cast<int*>(smem + kOffMisc + 16);

    const int tid = threadIdx.x, warp = tid >> 5;
    const int tiles = plan.tiles;
    const int bh = blockIdx.x / tiles, tile = blockIdx.x - bh * tiles;
    const int b = bh / g.heads, h = bh - b * g.heads;

    // Query rows of this tile.
    int r0, nreg, tok0, rows;
    if (plan.parts == 1) {
        r0 = tile * plan.G;
        nreg = min(plan.G, g.R - r0);
        tok0 = 0;
        rows = nreg * g.n;
    } else {
        r0 = tile / plan.parts;
        nreg = 1;
        tok0 = (tile - r0 * plan.parts) * plan.unit;
        rows = min(plan.unit, g.n - tok0);
    }

    // ---- set-up: barrier, TMEM, zeroed operand buffers, route masks --------
    if (tid == 0) {
        ptx::mbar_init(mbar, 1);
        ptx::mbar_init_fence();
        *s_bad = 0;
    }
    if (warp == 0) {
        ptx::tmem_alloc(tmem_slot, kTmemCols);
        ptx::tmem_relinquish();
        ptx::tc_fence_before();
    }
    for (int i = tid; i < (kOffP - kOffQ) / 16; i += kThreads)
        reinterpret_cast<uint4*>(smem + kOffQ)[i] = make_uint4(0, 0, 0, 0);
    for (int i = tid; i < nreg * 8; i += kThreads) rmask[i] = 0;
    __syncthreads();
    for (int e = tid; e < nreg * g.topk; e += kThreads) {
        const int gi = e / g.topk;
        const int rr = idx[((size_t)bh * g.R + r0 + gi) * g.topk + (e - gi * g.topk)];
        if (rr < 0 || rr >= g.R) {
            *s_bad = 1;
        } else {
            atomicOr(&rmask[gi * 8 + (rr >> 5)], 1u << (rr & 31));
        }
    }
    // Q rows of the tile (cp.async) while the union is formed.
    gather_rows(sQ, q, rows, g, b, h, [&](int j, int& reg, int& tok) {
        if (plan.parts == 1) {
            reg = r0 + j / g.n;
            tok = j - (j / g.n) * g.n;
        } else {
            reg = r0;
            tok = tok0 + j;
        }
    });
    __syncthreads();
    if (tid == 0) {
        int nu = 0;
        for (int w = 0; w < 8; ++w) {
            uint32_t m = 0;
            for (int gi = 0; gi < nreg; ++gi) m |= rmask[gi * 8 + w];
            while (m) {
                const int bit = __ffs(m) - 1;
                m &= m - 1;
                ulist[nu++] = w * 32 + bit;
            }
        }
        *s_nu = nu;
    }
    ptx::cp_async_wait_all();
    ptx::fence_proxy_async_smem();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const int nu = *s_nu;
    bool ok = *s_bad == 0;
    if (!ok && tid == 0) raise_status(status, kDevBadRoute);

    // Per-thread query state.
    const int row = tid;
    const int gi = plan.parts == 1 ? row / g.n : 0;
    const bool row_valid = row < rows;
    const uint32_t* my_routes = rmask + min(gi, nreg - 1) * 8;  // route bitmask of the row's region
    const float sl = kLog2e * rsqrtf(32.f);
    float m_run = -INFINITY, l_run = 0.f, acc[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) acc[c] = 0.f;

    const int nblocks = plan.parts == 1 ? (nu + plan.rpb - 1) / plan.rpb : nu * plan.parts;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    uint32_t phase = 0;

    for (int kb = 0; ok && kb < nblocks; ++kb) {
        // ---- 1. gather this block's K and V rows --------------------------
        int keys, ureg0, utok0;
        if (plan.parts == 1) {
            const int u0 = kb * plan.rpb;
            keys = min(plan.rpb, nu - u0) * g.n;
            ureg0 = u0;
            utok0 = 0;
        } else {
            ureg0 = kb / plan.parts;
            utok0 = (kb - ureg0 * plan.parts) * plan.unit;
            keys = min(plan.unit, g.n - utok0);
        }
        auto key_of = [&](int j, int& reg, int& tok) {
            if (plan.parts == 1) {
                const int u = j / g.n;
                reg = ulist[ureg0 + u];
                tok = j - u * g.n;
            } else {
                reg = ulist[ureg0];
                tok = utok0 + j;
            }
        };
        gather_rows(sK, k, keys, g, b, h, key_of);
        gather_rows(sV, v, keys, g, b, h, key_of);
        const int nblk = (keys + 31) & ~31;  // MMA N: multiple of 32, <= 128

        // Valid-key mask of this thread's query row for the block.
        uint32_t kmask[4] = {0u, 0u, 0u, 0u};
        if (row_valid) {
            if (plan.parts == 1) {
                const int units = keys / g.n;
                for (int u = 0; u < units; ++u) {
                    const int reg = ulist[ureg0 + u];
                    if ((my_routes[reg >> 5] >> (reg & 31)) & 1u) set_bits(kmask, u * g.n, (u + 1) * g.n);
                }
            } else {
                const int reg = ulist[ureg0];
                if ((my_routes[reg >> 5] >> (reg & 31)) & 1u) set_bits(kmask, 0, keys);
            }
        }

        ptx::cp_async_wait_all();
        ptx::fence_proxy_async_smem();
        __syncthreads();

        // ---- 2. S = Q K^T ----------------------------------------------------
        if (tid == 0) {
            ptx::tc_fence_after();
            const uint32_t idesc = ptx::idesc_bf16_f32(128, nblk, false, false);
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                const uint64_t a = ptx::smem_desc(sQ + kk * 32, 16, 512, ptx::kSwizzle64B);
                const uint64_t bd = ptx::smem_desc(sK + kk * 32, 16, 512, ptx::kSwizzle64B);
                ptx::mma_bf16(tmem, a, bd, idesc, kk);
            }
            ptx::mma_commit(mbar);
        }
        ok = ptx::mbar_wait(mbar, phase, kWaitLimit);
        phase ^= 1u;
        if (__syncthreads_or(!ok)) {
            ok = false;
            break;
        }
        ptx::tc_fence_after();

        // ---- 3. masked online softmax, P -> shared memory -------------------
        float mloc = -INFINITY;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            if (cb * 32 < nblk) {
                uint32_t r[32];
                ptx::tmem_ld32(tmem + lane_base + cb * 32, r);
                ptx::tmem_ld_wait();
                const uint32_t km = kmask[cb];
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if ((km >> i) & 1u) mloc = fmaxf(mloc, __uint_as_float(r[i]));
            }
        }
        const float m_new = fmaxf(m_run, mloc * sl);
        const float corr = (m_run == -INFINITY) ? 0.f : ptx::ex2(m_run - m_new);
        float lsum = 0.f;
#pragma unroll
        for (int cb = 0; cb < 4; ++cb) {
            if (cb * 32 >= nblk) break;
            const int c0 = cb * 32;
            uint32_t r[32];
            ptx::tmem_ld32(tmem + lane_base + c0, r);
            ptx::tmem_ld_wait();
            const uint32_t km = kmask[cb];
            uint32_t packed[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float p0 = ((km >> (2 * i)) & 1u) ? ptx::ex2(__uint_as_float(r[2 * i]) * sl - m_new) : 0.f;
                float p1 = ((km >> (2 * i + 1)) & 1u) ? ptx::ex2(__uint_as_float(r[2 * i + 1]) * sl - m_new) : 0.f;
                const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                lsum += __low2float(pb) + __high2float(pb);
                packed[i] = *reinterpret_cast<const uint32_t*>(&pb);
            }
            // 32 keys = 4 chunks of 8 keys in the 128-byte swizzled atom c0 / 64.
            const uint32_t atom = sP + (uint32_t)(c0 >> 6) * kPAtomBytes + row * 128;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                const int chunk = ((c0 & 63) >> 3) + cc;
                const uint32_t addr = atom + ((chunk ^ (row & 7)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(packed[4 * cc]),
                             "r"(packed[4 * cc + 1]), "r"(packed[4 * cc + 2]), "r"(packed[4 * cc + 3])
                             : "memory");
            }
        }
        if (mloc != -INFINITY) {
            l_run = l_run * corr + lsum;
            m_run = m_new;
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncthreads();

        // ---- 4. O_blk = P V ---------------------------------------------------
        if (tid == 0) {
            ptx::tc_fence_after();
            const uint32_t idesc = ptx::idesc_bf16_f32(128, 32, false, true);
            for (int kk = 0; kk < nblk / 16; ++kk) {
                const uint64_t a = ptx::smem_desc(sP + (kk >> 2) * kPAtomBytes + (kk & 3) * 32, 16,
                                                  1024, ptx::kSwizzle128B);
                const uint64_t bd = ptx::smem_desc(sV + kk * 1024, 0, 512, ptx::kSwizzle64B);
                ptx::mma_bf16(tmem, a, bd, idesc, kk > 0);
            }
            ptx::mma_commit(mbar);
        }
        ok = ptx::mbar_wait(mbar, phase, kWaitLimit);
        phase ^= 1u;
        if (__syncthreads_or(!ok)) {
            ok = false;
            break;
        }
        ptx::tc_fence_after();
        {
            uint32_t r[32];
            ptx::tmem_ld32(tmem + lane_base, r);
            ptx::tmem_ld_wait();
            if (mloc != -INFINITY) {
#pragma unroll
                for (int c = 0; c < 32; ++c) acc[c] = acc[c] * corr + __uint_as_float(r[c]);
            }
        }
        ptx::tc_fence_before();
        __syncthreads();
    }

    // ---- epilogue: O = acc / l for valid rows --------------------------------
    if (ok && row_valid && l_run > 0.f) {
        int reg, tok;
        if (plan.parts == 1) {
            reg = r0 + gi;
            tok = row - gi * g.n;
        } else {
            reg = r0;
            tok = tok0 + row;
        }
        const float inv = 1.f / l_run;
        const size_t ooff = token_offset(g, b, reg, tok) + (size_t)h * 32;
        uint4* dst = reinterpret_cast<uint4*>(o + ooff);
#pragma unroll
        for (int c = 0; c < 4 && in_bounds(ooff + 31, map_elems(g), status); ++c) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const __nv_bfloat162 pr =
                    __floats2bfloat162_rn(acc[8 * c + 2 * i] * inv, acc[8 * c + 2 * i + 1] * inv);
                w[i] = *reinterpret_cast<const uint32_t*>(&pr);
            }
            dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
    if (!ok && tid == 0 && *s_bad == 0) raise_status(status, kDevTimeout);
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bra_status attend_tc_launch(const Geometry& g, const void* q, const void* k, const void* v,
                            const int32_t* idx, void* o, int* status, cudaStream_t stream) {
    if (g.d != 32) return BRA_ERR_UNSUPPORTED;
    const TcPlan plan = make_plan(g);
    const long long ctas = (long long)g.B * g.heads * plan.tiles;
    if (ctas > 0x7fffffffLL) return BRA_ERR_UNSUPPORTED;
    static_assert(kSmemAlloc <= 227 * 1024, "shared memory budget");
    if (cudaFuncSetAttribute(bra_attend_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemAlloc) != cudaSuccess)
        return BRA_ERR_CUDA;
    bra_attend_tc_kernel<<<(unsigned)ctas, kThreads, kSmemAlloc, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), idx, static_cast<__nv_bfloat16*>(o), g, plan, status);
    return cudaGetLastError() == cudaSuccess ? BRA_OK : BRA_ERR_CUDA;
}

}  // namespace bra
