/*
 * moe.h -- C ABI of the B200 (sm_100a) Mixture-of-Experts layer forward.
 *
 * One MoE layer forward on one GPU, in four stages, each a hand-written CUDA
 * kernel (or a short chain of them) behind one entry point:
 *
 *   moe_router_topk        router logits, top-K, softmax over the kept K
 *   moe_permute            expert histogram, prefix scan, stable gather
 *   moe_grouped_ffn        every expert's FFN as one grouped GEMM launch chain
 *   moe_unpermute_combine  y = sum_j g_j * E_j(x)  (or a pure unpermute)
 *   moe_forward            all four, one stream, no host synchronisation
 *
 * Sources (web pages): "Advanced GPU Optimization: How to tech an LLM with
 * CUDA and ROCm? - Part 5" sections 1.1 (router kernel, top-2, sparse softmax)
 * and 1.2 (tokens grouped by destination expert, local expert FFNs);
 * "aclnnQuantGroupedMatMulAlltoAllv" (Ascend CANN) function/formula sections
 * (gmmY = (gmmX @ gmmWeight) * gmmXScale * gmmWeightScale, Unpermute, the
 * parallel shared-expert matmul, quant modes 0 = none / 1 = per-tensor), its
 * return-value section (two-phase interface: validate and size the workspace
 * first, then execute) and constraints (K in [2, 8], e*epWorldSize <= 256,
 * H1, N1 < 65536, deterministic by default); zyxy.net "SpMM ... MoE" MoE
 * structure section (y = sum_i g_i(x) E_i(x), gating (N,E), top-K (N,K)).
 *
 * Conventions for every call
 *  - Pointers named *_host are host memory; every other data pointer is
 *    device memory of the plan's device.  The caller allocates and frees all
 *    of them; the library never frees caller memory.
 *  - Device memory of the library's own: moe_plan_create allocates, once,
 *    plan-owned copies of weight data in the layout the kernels read, and
 *    moe_plan_destroy frees them: the router weights split into three bf16
 *    parts (plans whose router runs on the tensor cores), the MX weight
 *    scales (MOE_QUANT_MX) and the transposed group / block weight scales
 *    (MOE_QUANT_PER_GROUP, MOE_QUANT_PER_BLOCK).  No call allocates device
 *    memory after moe_plan_create.  The only other device memory of the
 *    library is the static scratch array of moe_permute_noalloc.
 *  - Launches are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  Only moe_read_device_status, moe_forward_host and
 *    moe_profile_read synchronise.
 *  - Arguments are validated on the host before anything is launched; a
 *    failed validation returns MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED /
 *    MOE_ERR_WORKSPACE_TOO_SMALL and launches nothing.
 *  - Errors found on the device (an expert id outside [0, E), a permutation
 *    index outside [0, N*K), a pipeline wait that ran out of time) are
 *    recorded in a sticky status word at the start of the workspace; the
 *    kernel skips the offending access and finishes.  Read (and clear) it
 *    with moe_read_device_status.
 *  - Results are deterministic: the same inputs give the same bytes (no
 *    floating-point atomics, fixed summation orders, stable permutation).
 *  - All row pointers must be 16-byte aligned and every row a multiple of
 *    16 bytes (d * sizeof(dtype) % 16 == 0).
 *
 * Layouts (row-major throughout)
 *  x          (N, d)        dtype (fp32, bf16 or e4m3 codes)
 *  w_r        (d, E)        fp32 router weight
 *  router_bias(E)           fp32 or NULL
 *  w1         (E, F, d)     ReLU W1 / SwiGLU gate / the single fp8 matrix;
 *                           each expert output-major (the transpose of the
 *                           Ascend page's logical (e, H1, N1)), like a Linear
 *                           layer's weight
 *  w3         (E, F, d)     SwiGLU up matrix (NULL otherwise)
 *  w2         (E, d, F)     second matrix (NULL for MOE_ACT_NONE)
 *  topk_ids   (N, K) int32, topk_gates (N, K) fp32, slots in descending logit
 *  counts     (E) int32, offsets (E+1) int32 (offsets[E] = N*K)
 *  perm_pos   (N*K) int32: row of x_perm that holds (token t, slot j)
 *  perm_src   (N*K) int32: token of each x_perm row
 *  x_perm     (N*K, d) dtype, expert-contiguous, stable within an expert
 *  y_perm     (N*K, d_out)  d_out = d, or F for MOE_ACT_NONE; dtype = x's
 *                           for fp32/bf16 layers, bf16 for e4m3 layers
 *  y          (N, d_out), or (N*K, F) token-major for the pure unpermute
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* identical to cudaStream_t */

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,         /* bad pointer, size, alignment or limit */
  MOE_ERR_UNSUPPORTED = 2,         /* valid but not built: dtype/act/quant combination */
  MOE_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes below moe_workspace_size */
  MOE_ERR_CUDA = 4,                /* a CUDA runtime/driver call failed */
  MOE_ERR_DEVICE_BAD_INDEX = 5,    /* device: expert id or permutation index out of range */
  MOE_ERR_DEVICE_TIMEOUT = 6       /* device: a bounded pipeline wait gave up */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_E4M3 = 2 } moe_dtype;

/* Expert FFN form.  NONE: one matrix per expert, y = x W1^T (the grouped
 * matmul of the Ascend page).  RELU: y = relu(x W1^T) W2^T.
 * SWIGLU: y = (silu(x W1^T) * (x W3^T)) W2^T, silu(z) = z / (1 + exp(-z)). */
typedef enum { MOE_ACT_NONE = 0, MOE_ACT_RELU = 1, MOE_ACT_SWIGLU = 2 } moe_act;

/* Scale granularity of the expert weights; values equal the Ascend page's
 * quant-mode enumeration (0 = not quantised, 1 = per-tensor, 2 =
 * per-channel: one scale per output column of each expert, 4 = per-group,
 * 5 = per-block, 6 = mx).
 * Per-token activation scales (mode 3) are a per-call argument
 * (x_token_scales); per-token dynamic quantization (mode 7) is
 * moe_permute_quant.  MX is read as OCP MXFP8: e4m3 elements in blocks of
 * 32 consecutive values along the reduction dimension (d), each block with
 * one E8M0 scale byte 2^(s - 127) (255 = NaN), for the weights
 * (w_mx_scales) and the activations (the _mx calls' x_mx_scales); the
 * single-matrix layer only, d a multiple of 32 and at most 32768.
 * PER_GROUP and PER_BLOCK are read as fp32 weight scales per group of 128
 * consecutive elements of d: one per output channel and group (PER_GROUP,
 * w_group_scales (E, F, d/128)) or one per block of 128 output channels x
 * 128 elements (PER_BLOCK, w_group_scales (E, ceil(F/128), d/128)); the
 * activations take a scalar, per-token, or per-token-and-group scales (the
 * _group_scales calls); the single-matrix layer only, d a multiple of 128. */
typedef enum {
  MOE_QUANT_NONE = 0,
  MOE_QUANT_PER_TENSOR = 1,
  MOE_QUANT_PER_CHANNEL = 2,
  MOE_QUANT_PER_GROUP = 4,
  MOE_QUANT_PER_BLOCK = 5,
  MOE_QUANT_MX = 6
} moe_quant;

typedef struct {
  int32_t N;      /* tokens per call, >= 1 */
  int32_t d;      /* token width (H1 of the grouped matmul), < 65536 */
  int32_t E;      /* experts, 1..256 */
  int32_t K;      /* experts kept per token, 1..8 and <= E */
  int32_t F;      /* FFN inner width; for MOE_ACT_NONE the output width N1; < 65536 */
  moe_dtype dtype;/* of x and the expert weights */
  moe_act act;
  moe_quant quant;/* PER_TENSOR, PER_CHANNEL, PER_GROUP, PER_BLOCK or MX for dtype
                     MOE_E4M3; NONE otherwise */
} moe_layer_desc;

typedef struct {
  const float* w_r;         /* (d, E) fp32; NULL if the caller always supplies routing */
  const float* router_bias; /* (E) fp32 added to the logits before top-K, or NULL */
  const void* w1;           /* (E, F, d) */
  const void* w3;           /* (E, F, d) for SWIGLU, else NULL */
  const void* w2;           /* (E, d, F) for RELU / SWIGLU, else NULL */
  float w_scale;            /* per-tensor weight scale (gmmWeightScale), e4m3 PER_TENSOR */
  const float* w_channel_scales; /* (E, F) fp32 per output channel, e4m3 PER_CHANNEL, else NULL */
  const uint8_t* w_mx_scales;    /* (E, F, d/32) E8M0 of w1, MOE_QUANT_MX, else NULL; device
                                    memory (MOE_ERR_INVALID_ARG otherwise), read once by
                                    moe_plan_create (may be freed afterwards) */
  const float* w_group_scales;   /* fp32 of w1: (E, F, d/128) PER_GROUP, (E, ceil(F/128),
                                    d/128) PER_BLOCK, else NULL; device memory, read once by
                                    moe_plan_create */
} moe_layer_weights;

typedef struct moe_plan_s* moe_plan;

/* ---- phase 1: validate, build the executor, size the workspace ---------- */

/* Validates desc and weights, records the weight pointers (not owned: they
 * must stay valid while the plan is used) and encodes the TMA descriptors of
 * the weights for the current CUDA device.  Some plans also hold device
 * copies of weight data in the layout their kernels read, made here
 * (synchronously, on a private stream) and freed by moe_plan_destroy:
 *  - a router on the tensor cores (bf16 x with at most 16 experts, unless
 *    the split-K router applies): w_r split into three bf16 parts, 6*d*E
 *    bytes rounded up to whole 32 x 8 tiles; w_r must be device memory
 *    (MOE_ERR_INVALID_ARG otherwise).  The split is taken from w_r now:
 *    after changing w_r in place call moe_plan_refresh_router;
 *  - MOE_QUANT_MX: the weight scales in the layout of the block-scaled
 *    tensor-core MMA (the same bytes as w_mx_scales, rearranged; about
 *    E*F*d/32 bytes);
 *  - PER_GROUP / PER_BLOCK: a transposed copy of w_group_scales (E, d/128,
 *    columns).
 * With w1, w3 and w2 all NULL (and no per-channel scales) the plan is
 * routing-only: router, permute and unpermute/combine work, the calls that
 * run the experts return MOE_ERR_UNSUPPORTED (an expert-parallel rank's
 * view of a layer whose experts live on several GPUs). */
moe_status moe_plan_create(const moe_layer_desc* desc, const moe_layer_weights* weights,
                           moe_plan* out);
moe_status moe_plan_destroy(moe_plan plan);

/* Re-derives the plan's copy of the router weights from weights.w_r (after
 * the caller changed w_r in place), stream-ordered on `stream`; no-op for
 * plans whose router reads w_r directly.  Not part of the pages' interface:
 * the plan-time copy is this library's choice (the router weights change
 * rarely, the split need not run on every call). */
moe_status moe_plan_refresh_router(moe_plan plan, moe_stream_t stream);

/* Bytes of device workspace that every call below accepts (the largest
 * need, that of moe_forward_host).  Workspace base must be 256-byte aligned. */
moe_status moe_workspace_size(moe_plan plan, size_t* bytes);

/* Clears the device status word of a fresh workspace (stream-ordered). */
moe_status moe_workspace_init(moe_plan plan, void* ws, size_t ws_bytes, moe_stream_t stream);

/* ---- phase 2: execute --------------------------------------------------- */

/* Router (page 1 section 1.1; zyxy MoE expert-selection section).  For each
 * token t: l[e] = sum_k x[t,k] * w_r[k,e] (+ router_bias[e]) with fp32
 * accuracy; keep the K largest (descending, equal logits -> lower expert
 * index); gates = softmax over the kept K only.  margin_or_null (N)
 * receives l_(K) - l_(K+1) (+inf when K == E).  x dtype fp32 or bf16.
 * Needs plan weights.w_r.  bf16 layers with at most 16 experts compute the
 * logits on the warp-level tensor-core MMA from the plan's exact three-part
 * bf16 split of w_r (moe_plan_create, moe_plan_refresh_router); bf16 layers
 * with more than 32 experts on tcgen05 from the same split, written to
 * workspace scratch on every call; the others, and fp32 x, with fp32 FMA. */
moe_status moe_router_topk(moe_plan plan, const void* x, int32_t* topk_ids, float* topk_gates,
                           float* margin_or_null, void* ws, size_t ws_bytes, moe_stream_t stream);

/* Permute / dispatch (page 1 section 1.2 token dispatch, local form; Ascend
 * page sendCounts).  counts[e] = #{(t,j): ids[t,j] = e}; offsets = exclusive
 * scan; perm_pos[t*K+j] = offsets[e] + #{(t',j') before (t,j) in (token,
 * slot) order with the same expert}; perm_src[perm_pos] = t;
 * x_perm[perm_pos[t*K+j]] = x[t] (byte copy).  Ids outside [0, E) set
 * MOE_ERR_DEVICE_BAD_INDEX and are skipped.  Uses workspace scratch. */
moe_status moe_permute(moe_plan plan, const void* x, const int32_t* topk_ids, int32_t* counts,
                       int32_t* offsets, int32_t* perm_pos, int32_t* perm_src, void* x_perm,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

/* moe_permute for callers that cannot allocate device memory: the pages
 * have no counterpart of this entry point.  Some callers cannot call
 * cudaMalloc: code running inside a host framework that owns every device
 * allocation and passes an operator only its inputs and outputs (a plugin
 * of an inference engine), or latency-critical code that must not risk the
 * device-wide synchronisation a cudaMalloc / cudaFree can cause.  This
 * variant takes no workspace and allocates nothing: its scratch (a counter
 * and the per-256-token-block expert counts) is a 1 MiB array in the
 * library's static device memory, held by every GPU that loads the library
 * until the process exits; the counter starts at zero when the library is
 * loaded on a device and every call leaves it at zero.
 * Same outputs as moe_permute.  device_status_or_null (device int32, may be
 * NULL; the caller zeroes it) receives MOE_ERR_DEVICE_BAD_INDEX if an id is
 * outside [0, E).  Limit: 256 + ceil(N/256) * E * 4 bytes <= 1 MiB (e.g.
 * N = 262144 with E = 255, or N = 261888 with E = 256); a larger plan is
 * refused with MOE_ERR_WORKSPACE_TOO_SMALL
 * and nothing is launched.  Every call looks up the array's device address
 * on the current device (cudaGetSymbolAddress, which allocates nothing and
 * is not cached, so it stays valid after a cudaDeviceReset); the first call
 * on a device also loads the library's module there, so make that first
 * call before any stream capture.  Like moe_permute it sets the plan's
 * launch count and stage events.  All calls share the one array: calls
 * whose kernels overlap on the GPU (different streams, or several threads)
 * race on it; serialise them. */
moe_status moe_permute_noalloc(moe_plan plan, const void* x, const int32_t* topk_ids,
                               int32_t* counts, int32_t* offsets, int32_t* perm_pos,
                               int32_t* perm_src, void* x_perm, int32_t* device_status_or_null,
                               moe_stream_t stream);

/* Grouped FFN (page 1 section 1.2 local expert execution; Ascend formula
 * gmmY).  Rows [offsets[e], offsets[e+1]) of x_perm go through expert e; the
 * result goes to the same rows of y_perm.  For e4m3: y_perm[r][n] =
 * (x_perm[r] . W_e[n]) * xs(r) * ws(e, n) in fp32, rounded once to bf16, with
 * xs(r) = x_row_scales[r] (per-token mode: one scale per permuted row) or the
 * per-tensor x_scale when x_row_scales_or_null is NULL, and ws(e, n) the
 * plan's per-channel scale or per-tensor w_scale.  Scales are ignored for
 * bf16/fp32 layers.  offsets must be a valid non-decreasing prefix with
 * offsets[E] = N*K (as moe_permute writes it).  Uses workspace scratch (the
 * SwiGLU/ReLU hidden activations). */
moe_status moe_grouped_ffn(moe_plan plan, const void* x_perm, const int32_t* offsets,
                           float x_scale, const float* x_row_scales_or_null, void* y_perm,
                           void* ws, size_t ws_bytes, moe_stream_t stream);

/* Unpermute + combine (zyxy MoE structure: y = sum_i g_i E_i(x); Ascend
 * Unpermute).  topk_gates != NULL: y[t] = sum_{j<K} gates[t,j] *
 * y_perm[perm_pos[t,j]], fp32 in slot order, one rounding to y's dtype.
 * topk_gates == NULL: y[t*K+j] = y_perm[perm_pos[t*K+j]] (pure reorder,
 * (N*K, d_out)).  Indices outside [0, N*K) set MOE_ERR_DEVICE_BAD_INDEX. */
moe_status moe_unpermute_combine(moe_plan plan, const void* y_perm, const int32_t* perm_pos,
                                 const float* topk_gates_or_null, void* y, void* ws,
                                 size_t ws_bytes, moe_stream_t stream);

/* The three stages above on the first n tokens of the plan's N (0 <= n <= N;
 * rows = n*K), for a batch whose size changes per call, e.g. the rows an
 * expert-parallel rank receives from the others (run with a plan of K = 1
 * and N = the largest possible count; p1 section 1.2, p2 AlltoAllv).
 * Otherwise as moe_permute / moe_grouped_ffn / moe_unpermute_combine. */
moe_status moe_permute_n(moe_plan plan, int32_t n, const void* x, const int32_t* topk_ids,
                         int32_t* counts, int32_t* offsets, int32_t* perm_pos, int32_t* perm_src,
                         void* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream);
moe_status moe_grouped_ffn_n(moe_plan plan, int32_t n, const void* x_perm, const int32_t* offsets,
                             float x_scale, const float* x_row_scales_or_null, void* y_perm,
                             void* ws, size_t ws_bytes, moe_stream_t stream);
moe_status moe_unpermute_combine_n(moe_plan plan, int32_t n, const void* y_perm,
                                   const int32_t* perm_pos, const float* topk_gates_or_null,
                                   void* y, void* ws, size_t ws_bytes, moe_stream_t stream);


/* Shared-expert matmul run beside the routed experts (Ascend formula mmY =
 * (mmX @ mmWeight) * mmXScale * mmWeightScale).  x (M, H) e4m3, w (N2, H)
 * e4m3 output-major, y (M, N2) bf16.  Scales: x_token_scales_or_null (M,
 * per-token) else x_scale; w_channel_scales_or_null (N2, per-channel) else
 * w_scale.  Plan dtype must be e4m3.  Limits: H a multiple of 16 and
 * <= 12288, N2 < 65536. */
moe_status moe_shared_matmul(moe_plan plan, const void* x, int32_t M, int32_t H, const void* w,
                             int32_t N2, float x_scale, const float* x_token_scales_or_null,
                             float w_scale, const float* w_channel_scales_or_null, void* y,
                             moe_stream_t stream);

/* Whole layer: router -> permute -> grouped FFN -> combine, on one stream,
 * with every intermediate in the workspace.  Needs plan weights.w_r (use
 * moe_forward_routed for caller-supplied routing). */
moe_status moe_forward(moe_plan plan, const void* x, void* y, void* ws, size_t ws_bytes,
                       moe_stream_t stream);

/* Layer with caller-supplied routing: permute -> grouped FFN -> unpermute.
 * topk_gates_or_null selects combine (gates) or pure reorder (NULL; y is
 * (N*K, d_out)).  For e4m3: x_token_scales_or_null (N, per-token mode) gives
 * each token's scale (applied to its K permuted rows), else x_scale.  The
 * pure reorder of a single-matrix tensor-core layer (the Ascend page's fused
 * GMM -> Unpermute) is done by the grouped GEMM's stores, row r of the
 * result going straight to row t*K+j of y; rows of invalid (t, j) pairs are
 * left unwritten, as moe_unpermute_combine leaves them. */
moe_status moe_forward_routed(moe_plan plan, const void* x, const int32_t* topk_ids,
                              const float* topk_gates_or_null, float x_scale,
                              const float* x_token_scales_or_null, void* y, void* ws,
                              size_t ws_bytes, moe_stream_t stream);

/* The routed fp8 layer and the shared expert "in parallel" (Ascend page,
 * function section: the shared-expert matmul runs beside the routed grouped
 * matmul): moe_shared_matmul(x, w_sh) on a stream owned by the plan, forked
 * from `stream` at entry, concurrently with moe_forward_routed(...) on
 * `stream`, joined back into `stream` before return (work queued on `stream`
 * afterwards sees both y and y_sh).  x (N, d) e4m3; w_sh (N2, d) e4m3; y_sh
 * (N, N2) bf16; scales as moe_shared_matmul (the activation scales are the
 * routed call's).  The plan's side stream is created on first use. */
moe_status moe_forward_routed_shared(moe_plan plan, const void* x, const int32_t* topk_ids,
                                     const float* topk_gates_or_null, float x_scale,
                                     const float* x_token_scales_or_null, void* y,
                                     const void* w_sh, int32_t N2, float w_sh_scale,
                                     const float* w_sh_channel_scales_or_null, void* y_sh,
                                     void* ws, size_t ws_bytes, moe_stream_t stream);

/* MX layer ("aclnnQuantGroupedMatMulAlltoAllv", parameter section, quant
 * mode 6 "mx", read as OCP MXFP8; the formula section's gmmY with the block
 * scales inside the sum).  MOE_QUANT_MX, act NONE: x (N, d) e4m3 codes with x_mx_scales
 * (N, d/32) E8M0, one per 32 consecutive elements of a row.  Computes, per
 * routed row of expert e,
 *   gmmY[r][n] = sum_k (x[r][k] * 2^(xs[r][k/32] - 127)) * (W[e][n][k] * 2^(ws[e][n][k/32] - 127))
 * in fp32 on the tensor cores (block-scaled tcgen05 MMA), rounded once to
 * bf16.  moe_forward_routed_mx: permute, the scales of every permuted row
 * rearranged for the MMA (in ws), the grouped matmul, then pure unpermute
 * (gates NULL: y (N*K, F), done by the GEMM's stores) or combine (y (N, F)).
 * moe_permute_mx: moe_permute plus x_perm_mx_scales (N*K, d/32), row r the
 * scales of x row perm_src[r].  moe_grouped_ffn_mx: the grouped matmul of
 * permuted rows x_perm with their scales x_perm_mx_scales (N*K, d/32).
 * MOE_ERR_UNSUPPORTED for a plan that is not MX; the other FFN calls return
 * MOE_ERR_UNSUPPORTED for an MX plan.  MOE_ERR_INVALID_ARG for null or
 * misaligned pointers; device errors go to the workspace status word.  All
 * buffers are the caller's. */
moe_status moe_forward_routed_mx(moe_plan plan, const void* x, const uint8_t* x_mx_scales,
                                 const int32_t* topk_ids, const float* topk_gates_or_null,
                                 void* y, void* ws, size_t ws_bytes, moe_stream_t stream);
moe_status moe_permute_mx(moe_plan plan, const void* x, const uint8_t* x_mx_scales,
                          const int32_t* topk_ids, int32_t* counts, int32_t* offsets,
                          int32_t* perm_pos, int32_t* perm_src, void* x_perm,
                          uint8_t* x_perm_mx_scales, void* ws, size_t ws_bytes,
                          moe_stream_t stream);
moe_status moe_grouped_ffn_mx(moe_plan plan, const void* x_perm, const uint8_t* x_perm_mx_scales,
                              const int32_t* offsets, void* y_perm, void* ws, size_t ws_bytes,
                              moe_stream_t stream);

/* Group / block-scaled layer ("aclnnQuantGroupedMatMulAlltoAllv", parameter
 * section, quant modes 4 "pergroup" and 5 "perblock", read as fp32 scales per
 * 128 elements of K; the formula section's gmmY with the scales inside the
 * sum).  MOE_QUANT_PER_GROUP or PER_BLOCK, act NONE:
 *   gmmY[r][n] = sum_g xs[r][g] * ws[e][n][g] * (sum_{k in group g} x[r][k] * W[e][n][k])
 * groups of 128 elements of d; ws the plan's weight scales (for PER_BLOCK
 * the scale of channel n's block n/128); xs per row and group from
 * x_group_scales (N, d/128), else per token from x_token_scales (N), else
 * x_scale.  Every K stage of 128 is accumulated alone on the tensor cores
 * (fp32) and added to fp32 sums with its scales; the result is rounded
 * once to bf16.  moe_forward_routed_group_scales: permute, the grouped
 * matmul, pure unpermute by its stores (gates NULL, y (N*K, F)) or combine
 * (y (N, F)); the activation scales are indexed by token.
 * moe_grouped_ffn_group_scales: permuted rows, their scales per permuted
 * row (x_row_scales (N*K) or x_group_scales (N*K, d/128)).
 * MOE_ERR_UNSUPPORTED for other plans; MOE_ERR_INVALID_ARG for null or
 * misaligned pointers (x, y, x_perm, y_perm: 16-byte aligned rows); device
 * errors (bad expert ids, a pipeline wait that ran out) go to the workspace
 * status word.  All buffers are the caller's. */
moe_status moe_forward_routed_group_scales(moe_plan plan, const void* x, float x_scale,
                                           const float* x_token_scales_or_null,
                                           const float* x_group_scales_or_null,
                                           const int32_t* topk_ids,
                                           const float* topk_gates_or_null, void* y, void* ws,
                                           size_t ws_bytes, moe_stream_t stream);
moe_status moe_grouped_ffn_group_scales(moe_plan plan, const void* x_perm, float x_scale,
                                        const float* x_row_scales_or_null,
                                        const float* x_group_scales_or_null,
                                        const int32_t* offsets, void* y_perm, void* ws,
                                        size_t ws_bytes, moe_stream_t stream);

/* Permute with per-token dynamic quantization (Ascend quant mode 7,
 * "pertoken dynamic quantization", parameter section): for an e4m3 plan, x is
 * the bf16 activations (N, d) (16-byte aligned rows; d a multiple of 16).
 * Each token row t gets token_scales[t] = amax(|x[t]|) / 448 (1 for an
 * all-zero row, fp32) and its codes e4m3(x / scale) (fp32 division, round to
 * nearest even, saturated to +-448) are written to its K destination rows of
 * x_perm (N*K, d) e4m3.  counts, offsets, perm_pos, perm_src as moe_permute.
 * MOE_ERR_UNSUPPORTED unless the plan dtype is e4m3. */
moe_status moe_permute_quant(moe_plan plan, const void* x_bf16, const int32_t* topk_ids,
                             int32_t* counts, int32_t* offsets, int32_t* perm_pos,
                             int32_t* perm_src, void* x_perm, float* token_scales, void* ws,
                             size_t ws_bytes, moe_stream_t stream);

/* moe_forward_routed for bf16 activations of an e4m3 layer: permute with
 * per-token dynamic quantization (as moe_permute_quant), the grouped fp8
 * GEMM with each row's token scale (and the plan's weight scales), then
 * unpermute (gates NULL, y (N*K, d_out), done by the GEMM's stores) or
 * combine (y (N, d_out)). */
moe_status moe_forward_routed_dynamic(moe_plan plan, const void* x_bf16, const int32_t* topk_ids,
                                      const float* topk_gates_or_null, void* y, void* ws,
                                      size_t ws_bytes, moe_stream_t stream);

/* moe_forward from host buffers: copies x_host (N, d) in, runs the layer,
 * copies y back to y_host (N, d_out) and synchronises the stream.  Pinned
 * host memory gives asynchronous copies; pageable memory works too. */
moe_status moe_forward_host(moe_plan plan, const void* x_host, void* y_host, void* ws,
                            size_t ws_bytes, moe_stream_t stream);

/* Asynchronous moe_forward_host for a stream of batches: returns once the
 * work is queued.  The H2D copy of x_host and the D2H copy into y_host run
 * on two copy streams owned by the plan, the layer on `stream`; two staging
 * slots in the workspace alternate between calls, so the copies of one
 * batch overlap the compute of its neighbours.  x_host must stay unchanged
 * and y_host unread until the copies finish: after moe_host_join(plan, s)
 * work queued on s runs after them (synchronise s to wait on the host).
 * Use one stream per plan for these calls.  x_host / y_host should be pinned
 * for the copies to overlap. */
moe_status moe_forward_host_async(moe_plan plan, const void* x_host, void* y_host, void* ws,
                                  size_t ws_bytes, moe_stream_t stream);

/* Makes `stream` wait for every host-buffer copy queued so far on this plan. */
moe_status moe_host_join(moe_plan plan, moe_stream_t stream);

/* Synchronises `stream`, returns the sticky device status of the workspace
 * (MOE_OK if clean) and clears it. */
moe_status moe_read_device_status(moe_plan plan, void* ws, moe_stream_t stream);

/* Diagnostic of the device-side failure path (the pages have no counterpart):
 * launches one CTA that waits, with the same bounded mbarrier wait the
 * tensor-core kernels use but a limit of limit_us microseconds (1..1e6), on
 * a barrier nothing arrives at, while a second warp waits on it with the
 * kernels' default limit.  The first wait gives up and records
 * MOE_ERR_DEVICE_TIMEOUT in the status word at the start of `ws` (read it
 * with moe_read_device_status); the second leaves through the shared abort
 * flag.  leave_order_or_null (device int32[2], caller-initialised) receives
 * the order in which the two warps left.  No trap, fault or hang: the
 * context stays usable. */
moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes, int32_t limit_us,
                                     int32_t* leave_order_or_null, moe_stream_t stream);

/* Stage timing: when enabled, moe_forward / moe_forward_routed record CUDA
 * events between their kernels.  moe_profile_read synchronises the last
 * recorded forward and writes per-kernel milliseconds in launch order;
 * names_or_null receives static kernel names. */
moe_status moe_profile_enable(moe_plan plan, int enable);
moe_status moe_profile_read(moe_plan plan, float* ms, const char** names_or_null, int capacity,
                            int* count);

/* Number of kernels the last moe_forward / moe_forward_routed launched. */
int moe_last_launch_count(moe_plan plan);

const char* moe_status_string(moe_status status);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
