// Gradients of the token attention for a fixed routing (the backward of blog
// "BiFormer Reshapes Visual Attention with Bi-Level Routing", Part 2 section
// 2.2 step 4; top-k has no gradient, so I^r is an input).  For query t with
// keys j over the union of its routed regions' tokens,
//   P = softmax(<q_t, k_j> / sqrt(d)),  dP_j = <g_t, v_j>,  D = sum_j P_j dP_j,
//   dS_j = P_j (dP_j - D),  dq_t = sum_j dS_j k_j / sqrt(d),
//   dk_j += dS_j q_t / sqrt(d),  dv_j += P_j g_t,
// with g = dL/dO.  All arithmetic is fp32 on CUDA cores.
//
// One CTA per (query region, batch x head): it takes the union of the region's
// routes (first listing of a repeated region), stages Q, G and the routed K, V
// rows of its head in shared memory as fp32, then one thread per query row
// recomputes P, forms dS and writes dq (each query belongs to one CTA), and
// finally the CTA reduces its contributions to each routed key's dk, dv over
// its queries and adds them to global memory with fp32 atomics (other regions
// may route to the same key region).
#include "backward.h"
#include "kernels.h"

namespace bra {
namespace {

constexpr int kBwdThreads = 256;
constexpr int kD = 32;
constexpr int kLd = kD + 1;  // padded rows: lanes reading different rows hit different banks

template <typename T>
__global__ void __launch_bounds__(kBwdThreads)
bra_attend_backward_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                           const int32_t* __restrict__ idx, const T* __restrict__ go, float* __restrict__ dq,
                           float* __restrict__ dk, float* __restrict__ dv, Geometry g, int* status) {
    extern __shared__ float bwd_smem[];
    __shared__ int live_regions[kMaxRegions];
    __shared__ int n_live;
    const int r = blockIdx.x;
    const int bh = blockIdx.y, b = bh / g.heads, h = bh - b * g.heads;
    const int n = g.n, kn = g.topk * n;
    const float scale = rsqrtf((float)kD);
    float* qs = bwd_smem;                    // [n][kLd]
    float* gs = qs + (size_t)n * kLd;        // [n][kLd]
    float* ks = gs + (size_t)n * kLd;        // [kn][kLd]
    float* vs = ks + (size_t)kn * kLd;       // [kn][kLd]
    float* ps = vs + (size_t)kn * kLd;       // [n][kn + 1]
    float* dss = ps + (size_t)n * (kn + 1);  // [n][kn + 1]

    if (threadIdx.x == 0) {
        const int32_t* route = idx + ((size_t)bh * g.R + r) * g.topk;
        int cnt = 0;
        bool bad = false;
        for (int m = 0; m < g.topk; ++m) {
            const int rr = route[m];
            if (rr < 0 || rr >= g.R) {
                bad = true;
                break;
            }
            bool seen = false;
            for (int mm = 0; mm < cnt; ++mm) seen |= live_regions[mm] == rr;
            if (!seen) live_regions[cnt++] = rr;
        }
        if (bad) raise_status(status, kDevBadRoute);
        n_live = bad ? -1 : cnt;
    }
    __syncthreads();
    const int nl = n_live;
    if (nl < 0) return;  // an out-of-range route: this region's gradients are skipped
    const int nk = nl * n;

    // Stage Q and G of the region and K, V of the live routed regions (fp32).
    for (int e = threadIdx.x; e < n * kD; e += kBwdThreads) {
        const int t = e / kD, c = e - t * kD;
        const size_t off = token_offset(g, b, r, t) + (size_t)h * kD + c;
        qs[t * kLd + c] = to_f32(q[off]);
        gs[t * kLd + c] = to_f32(go[off]);
    }
    for (int e = threadIdx.x; e < nk * kD; e += kBwdThreads) {
        const int j = e / kD, c = e - j * kD;
        const size_t off = token_offset(g, b, live_regions[j / n], j % n) + (size_t)h * kD + c;
        ks[j * kLd + c] = to_f32(k[off]);
        vs[j * kLd + c] = to_f32(v[off]);
    }
    __syncthreads();

    // One thread per query row: P, dS (kept in shared memory) and dq.
    for (int t = threadIdx.x; t < n; t += kBwdThreads) {
        const float* qt = qs + t * kLd;
        const float* gt = gs + t * kLd;
        float* pt = ps + (size_t)t * (kn + 1);
        float* dt = dss + (size_t)t * (kn + 1);
        float mx = -INFINITY;
        for (int j = 0; j < nk; ++j) {
            const float* kj = ks + j * kLd;
            float s = 0.f;
#pragma unroll
            for (int c = 0; c < kD; ++c) s = fmaf(qt[c], kj[c], s);
            s *= scale;
            pt[j] = s;
            mx = fmaxf(mx, s);
        }
        float den = 0.f;
        for (int j = 0; j < nk; ++j) {
            const float p = __expf(pt[j] - mx);
            pt[j] = p;
            den += p;
        }
        const float inv = 1.f / den;
        float dsum = 0.f;
        for (int j = 0; j < nk; ++j) {
            const float* vj = vs + j * kLd;
            float dp = 0.f;
#pragma unroll
            for (int c = 0; c < kD; ++c) dp = fmaf(gt[c], vj[c], dp);
            const float p = pt[j] * inv;
            pt[j] = p;
            dt[j] = dp;
            dsum = fmaf(p, dp, dsum);
        }
        float acc[kD];
#pragma unroll
        for (int c = 0; c < kD; ++c) acc[c] = 0.f;
        for (int j = 0; j < nk; ++j) {
            const float ds = pt[j] * (dt[j] - dsum);
            dt[j] = ds;
            const float* kj = ks + j * kLd;
#pragma unroll
            for (int c = 0; c < kD; ++c) acc[c] = fmaf(ds, kj[c], acc[c]);
        }
        float* out = dq + token_offset(g, b, r, t) + (size_t)h * kD;
#pragma unroll
        for (int c = 0; c < kD; ++c) out[c] = acc[c] * scale;
    }
    __syncthreads();

    // Each routed key's dk, dv contribution from this region's queries.
    for (int e = threadIdx.x; e < nk * kD; e += kBwdThreads) {
        const int j = e / kD, c = e - j * kD;
        float sk = 0.f, sv = 0.f;
        for (int t = 0; t < n; ++t) {
            sk = fmaf(dss[(size_t)t * (kn + 1) + j], qs[t * kLd + c], sk);
            sv = fmaf(ps[(size_t)t * (kn + 1) + j], gs[t * kLd + c], sv);
        }
        const size_t off = token_offset(g, b, live_regions[j / n], j % n) + (size_t)h * kD + c;
        atomicAdd(dk + off, sk * scale);
        atomicAdd(dv + off, sv);
    }
}

}  // namespace

size_t backward_smem_bytes(const Geometry& g) {
    const size_t n = (size_t)g.n, kn = (size_t)g.topk * g.n;
    const size_t bytes = ((2 * n + 2 * kn) * kLd + 2 * n * (kn + 1)) * sizeof(float);
    return bytes <= 227u * 1024u - 2048u ? bytes : 0;
}

cudaError_t launch_attend_backward(bool bf16, const void* q, const void* k, const void* v, const int32_t* idx,
                                   const void* grad_o, float* dq, float* dk, float* dv, const Geometry& g,
                                   int* status, cudaStream_t stream) {
    if (g.B == 0) return cudaSuccess;
    const size_t smem = backward_smem_bytes(g);
    if (smem == 0) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)g.R, (unsigned)(g.B * g.heads));
    if (bf16) {
        auto kern = bra_attend_backward_kernel<__nv_bfloat16>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return cudaGetLastError();
        kern<<<grid, kBwdThreads, smem, stream>>>(
            static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
            static_cast<const __nv_bfloat16*>(v), idx, static_cast<const __nv_bfloat16*>(grad_o), dq, dk, dv, g,
            status);
    } else {
        auto kern = bra_attend_backward_kernel<float>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return cudaGetLastError();
        kern<<<grid, kBwdThreads, smem, stream>>>(static_cast<const float*>(q), static_cast<const float*>(k),
                                                  static_cast<const float*>(v), idx,
                                                  static_cast<const float*>(grad_o), dq, dk, dv, g, status);
    }
    return cudaGetLastError();
}

}  // namespace bra
