// Gradients of the token attention on tensor cores (the backward of blog
// "BiFormer Reshapes Visual Attention with Bi-Level Routing", Part 2 section
// 2.2 step 4; top-k has no gradient, so I^r is an input).  With
// s_j = <q_t, k_j> / sqrt(d) over the union of the routed regions' tokens,
//   P = softmax(s),  dP_j = <g_t, v_j>,  D_t = sum_j P_j dP_j,
//   dS_j = P_j (dP_j - D_t),  dq_t = sum_j dS_j k_j / sqrt(d),
//   dk_j += dS_j q_t / sqrt(d),  dv_j += P_j g_t,  g = dL/dO.
//
// bf16 maps, d = 32, regions of 16, 32, 48 or 64 tokens, at most 128 routed
// keys per query.  A team works on one (query region, batch x head): the
// CTA's four warps together for regions of 32 tokens or more, one warp alone
// for 16-token regions (four regions per CTA, each warp with its own slice
// of shared memory, so that no warp idles in phase A).  Per team:
//   staging  Q and G of the region and K, V of its topk route slots (a slot
//            whose region repeats an earlier one is zero-filled and masked)
//            land in shared memory by 16-byte cp.async, 80-byte token rows
//            (64 bytes of the head + 16 of padding, so that the eight rows an
//            ldmatrix reads fall in distinct banks);
//   phase A  the team's warp w takes queries 16 w .. 16 w + 15: S = Q K^T
//            and dP = G V^T as m16n8k16 tiles, the softmax and D_t with quad
//            shuffles (rows live in the four lanes of a fragment group),
//            dS = P (dP - D); P and dS go to shared memory as bf16 (query rows
//            padded by 16 bytes for the same reason), and dq = dS K / sqrt(d)
//            is written straight to global memory (every query of the region
//            is this team's);
//   phase B  the team's warp w takes key tiles 16 w', w' = w, w + (warps of
//            the team), ...: dV = P^T G and
//            dK = dS^T Q / sqrt(d) over the region's queries, the transposed
//            operands read by ldmatrix.trans, then added to dk, dv with
//            16-byte fp32 atomics (other query regions may route to the same
//            keys; the order of the additions varies, so the last bits of dk
//            and dv may differ from run to run).
// Each product rounds its bf16 operands exactly once (P and dS; Q, K, V and
// G are bf16 inputs), accumulating in fp32.
#include "backward.h"
#include "kernels.h"
#include "tc_ptx.cuh"
#include "warp_mma.cuh"

namespace bra {
namespace {

using wmma16::ldsm_x4;
using wmma16::ldsm_x4_t;
using wmma16::mma16816;

constexpr int kWarps = 4;
constexpr int kMaxSlots = 8;        // topk * 16 <= 128
constexpr uint32_t kRowBytes = 80;  // one staged token row: 32 bf16 channels + 16 bytes of padding
constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ constexpr uint32_t p_row_bytes(int kn) { return 2u * (uint32_t)kn + 16u; }

// KN: keys per query region with every route live (topk * n), a multiple of 16, <= 128.
// TW: warps per team (4: one region per CTA; 1: one region per warp, n = 16).
// Five CTAs per SM (96 registers a thread, a few spilled; the shared-memory
// carveout set to its maximum): 20 warps instead of 16, measured 3-8 % faster.
template <int KN, int TW>
__global__ void __launch_bounds__(32 * kWarps, 5)
bra_attend_backward_mma_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                               const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ idx,
                               const __nv_bfloat16* __restrict__ go, float* __restrict__ dq,
                               float* __restrict__ dk, float* __restrict__ dv, Geometry g, int* status) {
    constexpr int NT = KN / 8;  // 8-key column tiles of S
    constexpr uint32_t kPRow = p_row_bytes(KN);
    constexpr int kTeams = kWarps / TW, kTeamThreads = 32 * TW;
    extern __shared__ __align__(16) uint8_t bwd_smem[];
    __shared__ int slot_regions[kTeams][kMaxSlots];
    __shared__ uint32_t live_team[kTeams];
    __shared__ int bad_team[kTeams];
    const int n = g.n;
    const int lane = threadIdx.x & 31, team = (threadIdx.x >> 5) / TW;
    const int warp = (threadIdx.x >> 5) - team * TW;  // the warp's index in its team
    const int ttid = (int)threadIdx.x - team * kTeamThreads;
    const int r = blockIdx.x * kTeams + team, bh = blockIdx.y, b = bh / g.heads, h = bh - b * g.heads;
    if (r >= g.R) return;  // (one-warp teams only: the last CTA's spare warps)
    // the team's barrier: the CTA, or for one-warp teams the warp
    auto team_sync = [&]() {
        if constexpr (TW == 1)
            __syncwarp();
        else
            __syncthreads();
    };
    int* slot_region = slot_regions[team];
    const uint32_t team_bytes = (uint32_t)(2 * n + 2 * KN) * kRowBytes + 2u * (uint32_t)n * kPRow;
    const uint32_t sQ = ptx::smem_addr(bwd_smem) + (uint32_t)team * team_bytes;
    const uint32_t sG = sQ + (uint32_t)n * kRowBytes;
    const uint32_t sK = sG + (uint32_t)n * kRowBytes;
    const uint32_t sV = sK + (uint32_t)KN * kRowBytes;
    const uint32_t sP = sV + (uint32_t)KN * kRowBytes;
    const uint32_t sD = sP + (uint32_t)n * kPRow;
    const size_t elems = map_elems(g);

    // Route slots: lane m < topk reads route m; any out-of-range route skips
    // the region, a repeat of an earlier route is a dead slot.
    if (warp == 0) {
        const int my_r = lane < g.topk ? __ldg(idx + ((size_t)bh * g.R + r) * g.topk + lane) : 0;
        const uint32_t bad = __ballot_sync(0xffffffffu, lane < g.topk && (my_r < 0 || my_r >= g.R));
        bool dup = false;
        for (int dd = 1; dd < g.topk; ++dd) {
            const int other = __shfl_up_sync(0xffffffffu, my_r, dd);
            if (dd <= lane && other == my_r) dup = true;
        }
        const uint32_t live = __ballot_sync(0xffffffffu, lane < g.topk && !dup);
        if (lane < g.topk) slot_region[lane] = my_r;
        if (lane == 0) {
            live_team[team] = live;
            bad_team[team] = bad != 0;
            if (bad) raise_status(status, kDevBadRoute);
        }
    }
    team_sync();
    if (bad_team[team]) {
        // this region's gradients are skipped: its dq rows are zero
        for (int e = ttid; e < n * 8; e += kTeamThreads) {
            const int t = e >> 3, c4 = e & 7;
            const size_t off = token_offset(g, b, r, t) + (size_t)h * 32 + (size_t)c4 * 4;
            if (in_bounds(off + 3, elems, status)) *reinterpret_cast<float4*>(dq + off) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        return;
    }
    const uint32_t live = live_team[team];

    // Staging: 16-byte chunk c of token row t (4 chunks per row).
    for (int e = ttid; e < n * 4; e += kTeamThreads) {
        const int t = e >> 2, c = e & 3;
        const size_t off = token_offset(g, b, r, t) + (size_t)h * 32 + (size_t)c * 8;
        ptx::cp_async16_zfill(sQ + (uint32_t)t * kRowBytes + (uint32_t)c * 16u, q + off, 16u);
        ptx::cp_async16_zfill(sG + (uint32_t)t * kRowBytes + (uint32_t)c * 16u, go + off, 16u);
    }
    for (int e = ttid; e < KN * 4; e += kTeamThreads) {
        const int j = e >> 2, c = e & 3, slot = j / n, t = j - slot * n;
        const bool on = (live >> slot) & 1u;
        const size_t off = on ? token_offset(g, b, slot_region[slot], t) + (size_t)h * 32 + (size_t)c * 8 : 0;
        ptx::cp_async16_zfill(sK + (uint32_t)j * kRowBytes + (uint32_t)c * 16u, k + off, on ? 16u : 0u);
        ptx::cp_async16_zfill(sV + (uint32_t)j * kRowBytes + (uint32_t)c * 16u, v + off, on ? 16u : 0u);
    }
    ptx::cp_async_commit();
    ptx::cp_async_wait_all();
    team_sync();

    const float scale = rsqrtf(32.f), sl = scale * kLog2e;
    const int gq = lane >> 2, tq = lane & 3;  // fragment row group, column pair
    // ldmatrix lane rows: A operand (16 rows x 16 columns, non-transposed) and
    // the transposed 16 x 16 B operands of 8-column n-tiles
    const int a_row = (lane & 7) + ((lane >> 3) & 1) * 8, a_chunk = lane >> 4;
    const int b_row = lane & 7, b_chunk = lane >> 3;
    const int t_row = (lane & 7) + ((lane >> 3) & 1) * 8;  // rows of a transposed B
    // 8-key tiles whose slot is live
    uint32_t tile_live = 0;
#pragma unroll
    for (int j = 0; j < NT; ++j)
        if ((live >> ((8 * j) / n)) & 1u) tile_live |= 1u << j;

    // ---------------------------------------------------------------- phase A
    for (int w = warp; w < n / 16; w += TW) {
        const int q0 = 16 * w;
        uint32_t qa[2][4], ga[2][4];
#pragma unroll
        for (int kc = 0; kc < 2; ++kc) {
            const uint32_t off = (uint32_t)(q0 + a_row) * kRowBytes + (uint32_t)(2 * kc + a_chunk) * 16u;
            ldsm_x4(sQ + off, qa[kc][0], qa[kc][1], qa[kc][2], qa[kc][3]);
            ldsm_x4(sG + off, ga[kc][0], ga[kc][1], ga[kc][2], ga[kc][3]);
        }
        // S = Q K^T, then P (fp32, normalised) in place; rows gq and gq + 8
        float s[NT][4];
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
            uint32_t b0, b1, b2, b3;
            ldsm_x4(sK + (uint32_t)(8 * j + b_row) * kRowBytes + (uint32_t)b_chunk * 16u, b0, b1, b2, b3);
            mma16816(s[j], qa[0][0], qa[0][1], qa[0][2], qa[0][3], b0, b1);
            mma16816(s[j], qa[1][0], qa[1][1], qa[1][2], qa[1][3], b2, b3);
            if (!((tile_live >> j) & 1u)) s[j][0] = s[j][1] = s[j][2] = s[j][3] = -INFINITY;
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
        float l0 = 0.f, l1 = 0.f;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            s[j][0] = ptx::ex2(fmaf(s[j][0], sl, -m0));
            s[j][1] = ptx::ex2(fmaf(s[j][1], sl, -m0));
            s[j][2] = ptx::ex2(fmaf(s[j][2], sl, -m1));
            s[j][3] = ptx::ex2(fmaf(s[j][3], sl, -m1));
            l0 += s[j][0] + s[j][1];
            l1 += s[j][2] + s[j][3];
        }
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        const float i0 = 1.f / l0, i1 = 1.f / l1;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            s[j][0] *= i0;
            s[j][1] *= i0;
            s[j][2] *= i1;
            s[j][3] *= i1;
        }
        // dP = G V^T tile by tile: first for D = sum_j P_j dP_j, then again for dS
        auto dp_tile = [&](int j, float (&dp)[4]) {
            dp[0] = dp[1] = dp[2] = dp[3] = 0.f;
            uint32_t b0, b1, b2, b3;
            ldsm_x4(sV + (uint32_t)(8 * j + b_row) * kRowBytes + (uint32_t)b_chunk * 16u, b0, b1, b2, b3);
            mma16816(dp, ga[0][0], ga[0][1], ga[0][2], ga[0][3], b0, b1);
            mma16816(dp, ga[1][0], ga[1][1], ga[1][2], ga[1][3], b2, b3);
        };
        float d0 = 0.f, d1 = 0.f;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            float dp[4];
            dp_tile(j, dp);
            d0 = fmaf(s[j][0], dp[0], fmaf(s[j][1], dp[1], d0));
            d1 = fmaf(s[j][2], dp[2], fmaf(s[j][3], dp[3], d1));
        }
        d0 += __shfl_xor_sync(0xffffffffu, d0, 1);
        d0 += __shfl_xor_sync(0xffffffffu, d0, 2);
        d1 += __shfl_xor_sync(0xffffffffu, d1, 1);
        d1 += __shfl_xor_sync(0xffffffffu, d1, 2);
        // dS = P (dP - D); P and dS to shared memory (bf16), dS also as the A
        // operand of dQ (the accumulator layout of a tile pair is that operand)
        uint32_t dsa[NT][2];
        const uint32_t prow0 = (uint32_t)(q0 + gq) * kPRow, prow1 = prow0 + 8u * kPRow;
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            float dp[4];
            dp_tile(j, dp);
            const float ds0 = s[j][0] * (dp[0] - d0), ds1 = s[j][1] * (dp[1] - d0);
            const float ds2 = s[j][2] * (dp[2] - d1), ds3 = s[j][3] * (dp[3] - d1);
            dsa[j][0] = ptx::pack_bf16x2(ds0, ds1);
            dsa[j][1] = ptx::pack_bf16x2(ds2, ds3);
            const uint32_t col = (uint32_t)(8 * j + 2 * tq) * 2u;
            ptx::st_shared_u32(sP + prow0 + col, ptx::pack_bf16x2(s[j][0], s[j][1]));
            ptx::st_shared_u32(sP + prow1 + col, ptx::pack_bf16x2(s[j][2], s[j][3]));
            ptx::st_shared_u32(sD + prow0 + col, dsa[j][0]);
            ptx::st_shared_u32(sD + prow1 + col, dsa[j][1]);
        }
        // dQ = dS K / sqrt(d): 16 keys per step, K rows read transposed; 4 tiles of 8 channels
        float acc[4][4];
#pragma unroll
        for (int nn = 0; nn < 4; ++nn) acc[nn][0] = acc[nn][1] = acc[nn][2] = acc[nn][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < NT / 2; ++kk) {
            const uint32_t krow = sK + (uint32_t)(16 * kk + t_row) * kRowBytes;
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(krow + (uint32_t)(0 + a_chunk) * 16u, b0, b1, b2, b3);
            mma16816(acc[0], dsa[2 * kk][0], dsa[2 * kk][1], dsa[2 * kk + 1][0], dsa[2 * kk + 1][1], b0, b1);
            mma16816(acc[1], dsa[2 * kk][0], dsa[2 * kk][1], dsa[2 * kk + 1][0], dsa[2 * kk + 1][1], b2, b3);
            ldsm_x4_t(krow + (uint32_t)(2 + a_chunk) * 16u, b0, b1, b2, b3);
            mma16816(acc[2], dsa[2 * kk][0], dsa[2 * kk][1], dsa[2 * kk + 1][0], dsa[2 * kk + 1][1], b0, b1);
            mma16816(acc[3], dsa[2 * kk][0], dsa[2 * kk][1], dsa[2 * kk + 1][0], dsa[2 * kk + 1][1], b2, b3);
        }
        const size_t o0 = token_offset(g, b, r, q0 + gq) + (size_t)h * 32;
        const size_t o1 = token_offset(g, b, r, q0 + gq + 8) + (size_t)h * 32;
        if (in_bounds((o0 > o1 ? o0 : o1) + 31, elems, status)) {
#pragma unroll
            for (int nn = 0; nn < 4; ++nn) {
                const int c = 8 * nn + 2 * tq;
                *reinterpret_cast<float2*>(dq + o0 + c) = make_float2(acc[nn][0] * scale, acc[nn][1] * scale);
                *reinterpret_cast<float2*>(dq + o1 + c) = make_float2(acc[nn][2] * scale, acc[nn][3] * scale);
            }
        }
    }
    team_sync();

    // ---------------------------------------------------------------- phase B
    // A = P^T (or dS^T): 16 keys x 16 queries from the query-major rows, the
    // four 8 x 8 blocks (keys 0-7 | 8-15) x (queries 0-7 | 8-15) transposed.
    const int pa_query = (lane & 7) + ((lane >> 4) & 1) * 8, pa_key = ((lane >> 3) & 1) * 8;
    for (int mt = warp; mt < KN / 16; mt += TW) {
        const int slot = (16 * mt) / n;
        if (!((live >> slot) & 1u)) continue;  // a repeated route: its P and dS are zero
        float av[4][4], ak[4][4];
#pragma unroll
        for (int nn = 0; nn < 4; ++nn) {
            av[nn][0] = av[nn][1] = av[nn][2] = av[nn][3] = 0.f;
            ak[nn][0] = ak[nn][1] = ak[nn][2] = ak[nn][3] = 0.f;
        }
        for (int ks = 0; ks < n / 16; ++ks) {
            const uint32_t aoff = (uint32_t)(16 * ks + pa_query) * kPRow + (uint32_t)(16 * mt + pa_key) * 2u;
            uint32_t p0, p1, p2, p3, s0, s1, s2, s3;
            ldsm_x4_t(sP + aoff, p0, p1, p2, p3);
            ldsm_x4_t(sD + aoff, s0, s1, s2, s3);
            const uint32_t grow = (uint32_t)(16 * ks + t_row) * kRowBytes;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(sG + grow + (uint32_t)(2 * half + a_chunk) * 16u, b0, b1, b2, b3);
                mma16816(av[2 * half], p0, p1, p2, p3, b0, b1);
                mma16816(av[2 * half + 1], p0, p1, p2, p3, b2, b3);
                ldsm_x4_t(sQ + grow + (uint32_t)(2 * half + a_chunk) * 16u, b0, b1, b2, b3);
                mma16816(ak[2 * half], s0, s1, s2, s3, b0, b1);
                mma16816(ak[2 * half + 1], s0, s1, s2, s3, b2, b3);
            }
        }
        // Rows gq, gq + 8 of the tile, channels 8 nn + 2 tq (+1).  Lanes tq and
        // tq ^ 1 swap halves so that each holds four consecutive channels of
        // one row: even tq row gq, channels 8 nn + 2 tq .. + 3; odd tq row
        // gq + 8, channels 8 nn + 2 tq - 2 .. + 1.
        const bool even = (tq & 1) == 0;
        const int key = 16 * mt + gq + (even ? 0 : 8);
        const size_t base = token_offset(g, b, slot_region[slot], key - slot * n) + (size_t)h * 32;
#pragma unroll
        for (int nn = 0; nn < 4; ++nn) {
            const int c = 8 * nn + 2 * tq - (even ? 0 : 2);
            const float xv = __shfl_xor_sync(0xffffffffu, even ? av[nn][2] : av[nn][0], 1);
            const float yv = __shfl_xor_sync(0xffffffffu, even ? av[nn][3] : av[nn][1], 1);
            const float xk = __shfl_xor_sync(0xffffffffu, even ? ak[nn][2] : ak[nn][0], 1);
            const float yk = __shfl_xor_sync(0xffffffffu, even ? ak[nn][3] : ak[nn][1], 1);
            const float4 gv = even ? make_float4(av[nn][0], av[nn][1], xv, yv) : make_float4(xv, yv, av[nn][2], av[nn][3]);
            const float4 gk = even ? make_float4(ak[nn][0] * scale, ak[nn][1] * scale, xk * scale, yk * scale)
                                   : make_float4(xk * scale, yk * scale, ak[nn][2] * scale, ak[nn][3] * scale);
            if (!in_bounds(base + c + 3, elems, status)) continue;
            atomicAdd(reinterpret_cast<float4*>(dv + base + c), gv);
            atomicAdd(reinterpret_cast<float4*>(dk + base + c), gk);
        }
    }
}

using BwdKernel = void (*)(const __nv_bfloat16*, const __nv_bfloat16*, const __nv_bfloat16*, const int32_t*,
                           const __nv_bfloat16*, float*, float*, float*, Geometry, int*);

// one warp per region for 16-token regions, the CTA per region otherwise
int team_warps(const Geometry& g) { return g.n == 16 ? 1 : kWarps; }

BwdKernel kernel_for(int kn, int tw) {
    if (tw == 1) {
        switch (kn) {
            case 16: return bra_attend_backward_mma_kernel<16, 1>;
            case 32: return bra_attend_backward_mma_kernel<32, 1>;
            case 48: return bra_attend_backward_mma_kernel<48, 1>;
            case 64: return bra_attend_backward_mma_kernel<64, 1>;
            case 80: return bra_attend_backward_mma_kernel<80, 1>;
            case 96: return bra_attend_backward_mma_kernel<96, 1>;
            case 112: return bra_attend_backward_mma_kernel<112, 1>;
            case 128: return bra_attend_backward_mma_kernel<128, 1>;
            default: return nullptr;
        }
    }
    switch (kn) {
        case 32: return bra_attend_backward_mma_kernel<32, kWarps>;
        case 48: return bra_attend_backward_mma_kernel<48, kWarps>;
        case 64: return bra_attend_backward_mma_kernel<64, kWarps>;
        case 96: return bra_attend_backward_mma_kernel<96, kWarps>;
        case 128: return bra_attend_backward_mma_kernel<128, kWarps>;
        default: return nullptr;
    }
}

size_t mma_smem_bytes(const Geometry& g) {
    const int kn = g.topk * g.n, teams = kWarps / team_warps(g);
    return (size_t)teams * ((size_t)(2 * g.n + 2 * kn) * kRowBytes + (size_t)2 * g.n * p_row_bytes(kn));
}

}  // namespace

bool backward_mma_covers(const Geometry& g) {
    const int kn = g.topk * g.n;
    return g.d == 32 && g.n % 16 == 0 && g.n >= 16 && g.n <= 64 && g.topk <= kMaxSlots && kn <= 128 &&
           kernel_for(kn, team_warps(g)) != nullptr && (long long)g.B * g.heads <= 65535 &&
           mma_smem_bytes(g) <= 227u * 1024u;
}

cudaError_t launch_attend_backward_mma(const void* q, const void* k, const void* v, const int32_t* idx,
                                       const void* grad_o, float* dq, float* dk, float* dv, const Geometry& g,
                                       int* status, cudaStream_t stream) {
    if (g.B == 0) return cudaSuccess;
    const int tw = team_warps(g), teams = kWarps / tw;
    const BwdKernel kern = kernel_for(g.topk * g.n, tw);
    if (!kern) return cudaErrorInvalidValue;
    const size_t smem = mma_smem_bytes(g);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return cudaGetLastError();
    if (cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
        return cudaGetLastError();
    kern<<<dim3((unsigned)((g.R + teams - 1) / teams), (unsigned)(g.B * g.heads)), 32 * kWarps, smem, stream>>>(
        static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), idx, static_cast<const __nv_bfloat16*>(grad_o), dq, dk, dv, g,
        status);
    return cudaGetLastError();
}

}  // namespace bra
