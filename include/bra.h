/*
 * bra.h -- C ABI of the B200 (sm_100a) Bi-Level Routing Attention library.
 *
 * Bi-Level Routing Attention (BRA) is the attention of BiFormer ("BiFormer:
 * Vision Transformer with Bi-Level Routing Attention", Zhu et al., CVPR
 * 2023).  The blog page "BiFormer Reshapes Visual Attention with Bi-Level
 * Routing", Part 2 section 2.2 "The Overall BRA Flow", defines the steps this
 * library runs, starting from projected Q, K, V:
 *
 *   region partition  the H x W map is cut into S x S regions of
 *                     n = (H/S)(W/S) tokens (step 1);
 *   region routing    Q^r, K^r = per-region means of Q and K; the region
 *                     affinity A^r = Q^r (K^r)^T; I^r = row-wise top-k of A^r
 *                     (step 3);
 *   token attention   every query token of region r attends, with a
 *                     softmax, over the tokens of the k regions I^r[r] (step 4).
 *
 * Conventions shared by every entry point
 *  - Q, K, V, O are dense channels-last [B, H, W, C] tensors in device
 *    memory, all of the element type ``dtype``; head h owns channels
 *    [h*d, (h+1)*d) with d = C / heads, and every head is routed and attended
 *    on its own.
 *  - Regions are numbered row-major over the S x S grid, tokens row-major
 *    inside a region.
 *  - I^r is int32 [B, heads, S*S, topk] in device memory; each row lists its
 *    regions by (affinity descending, lower index first on ties).
 *  - A^r is computed in fp32 from fp32 region means and is not scaled; the
 *    attention logits are scaled by 1/sqrt(d); the softmax and both products
 *    accumulate in fp32; a bf16 O is rounded to nearest-even from fp32.
 *  - The local-context term of step 4 (a 5x5 depthwise convolution of V) is
 *    not part of these calls.
 *  - Every buffer is owned by the caller.  The library allocates no device or
 *    host memory and keeps no per-call state; its only global state is a
 *    per-device cache of the kernels' launch attributes.
 *  - Every call is asynchronous on ``stream`` (a cudaStream_t; NULL is the
 *    legacy default stream).  Arguments are checked on the host first; an
 *    invalid call returns an error and launches nothing.
 *  - Supported sizes: H % S == 0, W % S == 0, C % heads == 0, 1 <= topk <=
 *    S*S, S*S <= 256, d == 32, C * sizeof(dtype) <= 2048 bytes (up to 32
 *    bf16 or 16 fp32 heads), B >= 0 (B == 0 is a no-op).
 *    Pointers must be 16-byte aligned.  The S constraint is the pages'
 *    own (blog Part 3: S is chosen as a divisor of the map size so that no
 *    padding is needed); d == 32 is the head size of every BiFormer stage.
 *  - Thread safety: calls on different streams may run concurrently as long
 *    as they do not share ``workspace`` or output buffers.
 */
#ifndef BRA_H
#define BRA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BRA_OK = 0,
    BRA_ERR_INVALID_ARG = 1, /* sizes or pointers break the rules above     */
    BRA_ERR_UNSUPPORTED = 2, /* valid BRA problem this build does not cover */
    BRA_ERR_CUDA = 3,        /* a CUDA call or a kernel launch failed       */
    BRA_ERR_TIMEOUT = 4,     /* a device-side bounded wait ran out          */
    BRA_ERR_BAD_ROUTE = 5,   /* bra_attend saw a routing index outside [0, S*S) */
    BRA_ERR_BOUNDS = 6       /* debug build only: a kernel caught an output index
                                outside its buffer and skipped the access      */
} bra_status;

typedef enum { BRA_DTYPE_F32 = 0, BRA_DTYPE_BF16 = 1 } bra_dtype;

/* One problem: feature map [B, H, W, C], heads, S x S regions, topk routes. */
typedef struct {
    int B, H, W, C;
    int heads;
    int S;
    int topk;
    int dtype; /* a bra_dtype */
} bra_shape;

/*
 * Bytes of device workspace the calls below need for ``shape``: the fp32
 * region means Q^r and K^r ([B, heads, S*S, d] each) followed by a 256-byte
 * status block.  Returns 0 when ``shape`` is invalid.  The status block must
 * hold zeros before the first call (zero the whole workspace once after
 * allocating it); kernels only ever set it and bra_device_status clears it.
 * The rest needs no initialisation.  The workspace may be reused by calls
 * that are ordered on the GPU (e.g. one stream).
 */
size_t bra_workspace_bytes(const bra_shape* shape);

/*
 * Region-level routing (blog section 2.2 step 3): pools Q and K per region
 * into the workspace, forms A^r = Q^r (K^r)^T per (batch, head) in fp32 and
 * writes I^r = row-wise top-k to ``idx`` [B, heads, S*S, topk].
 *   q, k       device, [B, H, W, C] of ``shape->dtype``, read only
 *   idx        device int32 [B, heads, S*S, topk], written
 *   workspace  device, bra_workspace_bytes(shape) bytes, scratch
 * Errors: BRA_ERR_INVALID_ARG (bad sizes, NULL or misaligned pointer),
 * BRA_ERR_UNSUPPORTED (d != 32, S*S > 256), BRA_ERR_CUDA (launch failed).
 */
bra_status bra_route(const bra_shape* shape, const void* q, const void* k, int32_t* idx,
                     void* workspace, void* stream);

/*
 * Token-to-token attention over the routed regions (blog section 2.2 step 4):
 * for every query token t of region r and head h,
 *   O[t] = sum_j softmax_j(<q_t, k_j> / sqrt(d)) v_j
 * where j runs over the tokens of the regions idx[b, h, r, 0..topk-1].  The
 * routed K/V tiles are staged in shared memory and never written to HBM.
 *   q, k, v    device, [B, H, W, C] of ``shape->dtype``, read only
 *   idx        device int32 [B, heads, S*S, topk], read only; any routing
 *              (it need not come from bra_route); a region repeated within a
 *              row counts once (attention runs over the union of the routed
 *              regions' tokens); an entry outside [0, S*S)
 *              makes the kernel skip that region's outputs and record
 *              BRA_ERR_BAD_ROUTE in the workspace status block
 *   o          device, [B, H, W, C] of ``shape->dtype``, written
 *   workspace  as for bra_route (only its status block is used)
 * Errors: as bra_route.  Device-side problems are reported by
 * bra_device_status.
 */
bra_status bra_attend(const bra_shape* shape, const void* q, const void* k, const void* v,
                      const int32_t* idx, void* o, void* workspace, void* stream);

/*
 * The whole path: bra_route then bra_attend on the same stream, writing both
 * the routing ``idx`` and the output ``o``.  Arguments as above.
 */
bra_status bra_forward(const bra_shape* shape, const void* q, const void* k, const void* v,
                       void* o, int32_t* idx, void* workspace, void* stream);

/*
 * Local context enhancement, added in place to an attention output (blog
 * "BiFormer Reshapes Visual Attention with Bi-Level Routing", Part 2 section
 * 2.2, step 4 third bullet; pseudocode step 7 adds "dwconv(value)" to the
 * attention result).  For every b, y, x and channel c:
 *   o[b,y,x,c] += bias[c] + sum_{i,j=0..4} weight[c][i][j] * v[b, y+i-2, x+j-2, c]
 * with v = 0 outside the H x W map: a 5x5 depthwise filter, stride 1, zero
 * padding 2, in the cross-correlation orientation of deep-learning
 * convolution layers.  The pages give no weights, bias or padding; the caller
 * supplies the layer's parameters.  Accumulation is fp32; a bf16 ``o`` is
 * read, the term added in fp32 and the sum rounded to nearest-even once.
 *   shape      as for bra_forward (only B, H, W, C and dtype are used by the
 *              filter; the other fields are checked as for bra_forward)
 *   v          device, [B, H, W, C] of ``shape->dtype``, read only
 *   weight     device fp32 [C][5][5] (a [C, 1, 5, 5] layer weight), read only
 *   bias       device fp32 [C], or NULL for no bias
 *   o          device, [B, H, W, C] of ``shape->dtype``, read and written
 * All pointers 16-byte aligned.  Errors: as bra_route (BRA_ERR_INVALID_ARG
 * for a bad shape or a null/misaligned pointer, before any launch;
 * BRA_ERR_CUDA if the launch fails).  Runs on ``stream``; allocates nothing.
 */
bra_status bra_lce(const bra_shape* shape, const void* v, const float* weight, const float* bias, void* o,
                   void* stream);

/*
 * The whole path with the local context term: bra_route, then the token
 * attention with o[b,y,x,c] = attention + bias[c] + sum_{i,j} weight[c][i][j] *
 * v[b, y+i-2, x+j-2, c] (bra_lce's filter) formed in fp32 and rounded once
 * (blog section 2.2 step 4, third bullet; pseudocode step 7).  For bf16 maps
 * of 8 x 8-token regions with an even number of heads and C <= 128 the filter
 * runs in the attention kernel's epilogue (one kernel, V's halo read by TMA,
 * O written once); other shapes run the attention, then the filter as
 * bra_lce does (the attention output rounded before the term is added).
 * Arguments as for bra_forward and bra_lce; a region with an out-of-range
 * route is reported and its outputs are not written (with the fused epilogue,
 * neither the attention nor the filter term).  Errors: as bra_forward.
 */
bra_status bra_forward_lce(const bra_shape* shape, const void* q, const void* k, const void* v, const float* weight,
                           const float* bias, void* o, int32_t* idx, void* workspace, void* stream);

/*
 * Reads (synchronising ``stream``) and clears the device status block in
 * ``workspace``: BRA_OK, BRA_ERR_TIMEOUT (a bounded wait in a kernel gave up;
 * that kernel's outputs are incomplete), BRA_ERR_BAD_ROUTE or, in a library
 * built with -DBRA_DEBUG (libbra_b200_debug.so, which checks the output index
 * of every attention-kernel store against its buffer), BRA_ERR_BOUNDS.
 */
bra_status bra_device_status(const bra_shape* shape, void* workspace, void* stream);

/*
 * Routing without a caller-supplied workspace.  The pages describe nothing
 * like it: it exists for callers that cannot allocate device memory, such as
 * plugins inside a host framework that owns all device memory and hands out
 * none, or loops that must not call cudaMalloc because it can synchronise
 * the whole device.  It writes the same ``idx`` as bra_route.
 *
 * The scratch for Q^r and K^r is a fixed array inside the library (every
 * GPU that loads the library holds it, 2 * BRA_NOALLOC_MAX_MEANS floats =
 * 8 MiB, until the process exits).  Limit: B * heads * S*S * d must not
 * exceed BRA_NOALLOC_MAX_MEANS, else BRA_ERR_UNSUPPORTED (and nothing is
 * launched); other argument errors are those of bra_route.  Every call
 * looks up the array's device address on the caller's current device (so a
 * device reset does not leave a stale address behind); the first call on a
 * device may load the library's module there, so make that first call
 * before any stream capture.  All
 * calls share the array, so calls that overlap on the GPU race: order them
 * (e.g. one stream).  Allocates nothing, host or device.
 */
#define BRA_NOALLOC_MAX_MEANS (1u << 20)
bra_status bra_route_noalloc(const bra_shape* shape, const void* q, const void* k, int32_t* idx,
                             void* stream);

/*
 * Gradients of bra_attend for a fixed routing (the backward of blog section
 * 2.2 step 4; top-k has no gradient, so ``idx`` is an input).  With
 * s_j = <q_t, k_j> / sqrt(d), P = softmax(s) over the union of the routed
 * regions' tokens (a region listed twice counts once), O = P V and
 * G = dL/dO:
 *   dP_j = <G_t, v_j>,  D_t = sum_j P_j dP_j,  dS_j = P_j (dP_j - D_t),
 *   dQ_t = sum_j dS_j k_j / sqrt(d),  dK_j = sum_t dS_tj q_t / sqrt(d),
 *   dV_j = sum_t P_tj G_t.
 * bf16 maps with d = 32, regions of 16, 32, 48 or 64 tokens and at most
 * 128 routed keys per query run on tensor cores: products accumulate in
 * fp32, and P and dS enter them rounded once to bf16 (relative error 2^-8
 * per term).  Other shapes run on CUDA cores in fp32 throughout.  The
 * environment variable BRA_BACKWARD_KERNEL=simt (or =mma) pins one form.
 * dK and dV are accumulated with fp32 atomics, so their last bits may
 * differ from run to run.
 *   shape      as for bra_attend; regions of up to about 64 tokens with up
 *              to 256 routed keys per query fit (staging in shared memory),
 *              larger ones return BRA_ERR_UNSUPPORTED (as does the =mma pin
 *              on a shape the tensor-core form does not cover)
 *   q, k, v    device, [B, H, W, C] of ``shape->dtype``, read only
 *   idx        device int32 [B, heads, S*S, topk], read only; an entry
 *              outside [0, S*S) makes the kernel skip that region's
 *              gradients and record BRA_ERR_BAD_ROUTE in the status block
 *   grad_o     device, [B, H, W, C] of ``shape->dtype``: dL/dO, read only
 *   dq, dk, dv device fp32 [B, H, W, C], every element written (dk, dv
 *              cleared first, then accumulated)
 *   workspace  as for bra_attend (only its status block is used)
 * All pointers 16-byte aligned.  Errors: as bra_attend.  Allocates nothing.
 */
bra_status bra_attend_backward(const bra_shape* shape, const void* q, const void* k, const void* v,
                               const int32_t* idx, const void* grad_o, float* dq, float* dk, float* dv,
                               void* workspace, void* stream);

/*
 * Linear projection fused with the region means (blog "BiFormer Reshapes
 * Visual Attention with Bi-Level Routing", Part 2 section 2.2 step 2 and
 * pseudocode step 2, where query, key and value are the three channel chunks
 * of one linear layer; step 3's Q^r, K^r follow in the same pass).  For every
 * token x (C channels) and output channel o in [0, 3C):
 *   y[o] = bias[o] + sum_c w_qkv[o][c] * x[c],
 * q = y[0, C), k = y[C, 2C), v = y[2C, 3C), each rounded to bf16 from the
 * fp32 accumulator; q_r and k_r are the fp32 means of the stored (bf16) q
 * and k over every region, exactly what bra_route pools from them.
 *   shape      dtype BRA_DTYPE_BF16, C = 64 or 128, regions of at most 128
 *              tokens; other valid shapes return BRA_ERR_UNSUPPORTED (topk
 *              is only checked)
 *   x          device bf16 [B, H, W, C], read only
 *   w_qkv      device bf16 [3C][C] (a linear layer's [out][in] weight), read only
 *   b_qkv      device fp32 [3C], or NULL for no bias
 *   q, k, v    device bf16 [B, H, W, C], written; they must not overlap x
 *   q_r, k_r   device fp32 [B, heads, S*S, d], written
 *   workspace  as for bra_route (only its status block is used: a device
 *              wait that gives up records BRA_ERR_TIMEOUT there)
 * All pointers 16-byte aligned.  Errors: BRA_ERR_INVALID_ARG (bad shape,
 * NULL or misaligned pointer), BRA_ERR_UNSUPPORTED, BRA_ERR_CUDA.
 */
bra_status bra_qkv_project(const bra_shape* shape, const void* x, const void* w_qkv, const float* b_qkv, void* q,
                           void* k, void* v, float* q_r, float* k_r, void* workspace, void* stream);

/*
 * The whole path from the feature map: bra_qkv_project (its region means go
 * to the workspace), the top-k routing of bra_route on those means, then
 * bra_attend.  Writes q, k, v (kept for a backward pass), ``idx`` and ``o``.
 * Arguments and limits as for bra_qkv_project and bra_forward.
 */
bra_status bra_forward_qkv(const bra_shape* shape, const void* x, const void* w_qkv, const float* b_qkv, void* q,
                           void* k, void* v, void* o, int32_t* idx, void* workspace, void* stream);

/*
 * Self-test of the failure-detection path (the pages have no counterpart):
 * every kernel that waits on an mbarrier polls it a bounded number of times
 * and, when the limit runs out, records BRA_ERR_TIMEOUT in the workspace
 * status block and returns instead of hanging.  This call launches one small
 * kernel that waits, with a limit of ``tries`` polls (1 .. 2^24), on an
 * mbarrier that nothing arrives at (``arrive`` = 0; the wait runs out and
 * BRA_ERR_TIMEOUT is recorded) or that it arrives at itself first (``arrive``
 * != 0; the wait succeeds and nothing is recorded).  Read the outcome with
 * bra_device_status.  ``shape`` and ``workspace`` as for bra_route.  Errors:
 * BRA_ERR_INVALID_ARG (bad shape, workspace or ``tries``), BRA_ERR_CUDA.
 */
bra_status bra_selftest_bounded_wait(const bra_shape* shape, void* workspace, unsigned int tries, int arrive,
                                     void* stream);

/* Static English text for a status code. */
const char* bra_status_string(bra_status status);

/* Library version as major * 10000 + minor * 100 + patch. */
int bra_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BRA_H */
