// Internal launchers of the MoE layer kernels.  Host-side C++ only; the
// public surface is the C ABI in include/moe.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

struct moe_plan_s;  // the C ABI's plan (include/moe.h)

namespace moe {

// Launch with programmatic stream serialization (the kernel must call
// griddep_wait before reading its predecessor's output).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

enum DType { kF32 = 0, kBF16 = 1, kE4M3 = 2 };
enum Act { kActNone = 0, kActRelu = 1, kActSwiglu = 2 };

inline int dtype_bytes(int dt) { return dt == kF32 ? 4 : dt == kBF16 ? 2 : 1; }

// ---- router -----------------------------------------------------------------
// SIMT router (fp32 logits, any E <= 256).  Few tokens with long rows
// (router_uses_splitk) take the split-K form, which needs `scratch` of
// router_splitk_scratch_bytes for its partial logits; otherwise scratch may
// be NULL.
cudaError_t launch_router(const void* x, int x_dtype, const float* w_r, const float* bias, int N,
                          int d, int E, int K, int32_t* ids, float* gates, float* margin,
                          void* scratch, cudaStream_t stream);
constexpr int kRouterSplitkMaxTokens = 512;
constexpr size_t kRouterSplitkSmemMax = 96 * 1024;
bool router_uses_splitk(int N, int d);
int router_splitk_rows(int d, int E);
size_t router_splitk_scratch_bytes(int N, int d, int E);

// bf16 tokens and at most kRouterMmaMaxExperts experts (and not split-K):
// logits on the warp-level tensor-core MMA from a fragment-ordered three-part
// bf16 split of w_r made once per plan (launch_router_mma_frag, into
// router_mma_frag_bytes of device memory).
constexpr int kRouterMmaMaxExperts = 16;
bool router_uses_mma(int N, int d, int E, int x_dtype);
size_t router_mma_frag_bytes(int d, int E);
cudaError_t launch_router_mma_frag(const float* w_r, int d, int E, void* frag, cudaStream_t stream);
// Split weights up to this size are staged in shared memory by each CTA.
constexpr size_t kRouterMmaSmemMax = 96 * 1024;
cudaError_t launch_router_mma(const void* x, const void* frag, const float* bias, int N, int d,
                              int E, int K, int32_t* ids, float* gates, float* margin, int* status,
                              cudaStream_t stream);

// Top-K, softmax and margin of fp32 logits (N, E) in memory, plus bias.
cudaError_t launch_logits_topk(const float* logits, const float* bias, int N, int E, int K,
                              int32_t* ids, float* gates, float* margin, cudaStream_t stream);

// Tensor-core router (bf16 x): splits w_r into three bf16 parts in `scratch`
// (router_tc_scratch_bytes), runs the logits on tcgen05 into fp32 logits in
// the same scratch, then the top-K and softmax (launch_logits_topk).
size_t router_tc_scratch_bytes(int N, int d, int E);
cudaError_t launch_router_tc(const void* x, const float* w_r, const float* bias, int N, int d,
                             int E, int K, int32_t* ids, float* gates, float* margin,
                             void* scratch, int* status, cudaStream_t stream);
// Experts above which bf16 routers run on the tensor cores.
constexpr int kRouterTcMinExperts = 33;
// bf16 tokens with 33..kRouterFusedMaxExperts experts (and not split-K): one
// kernel computes the logits on tcgen05 from the plan's split router weights
// (launch_router_fused_split into router_fused_weight_bytes of device memory,
// TMA map from encode_router_fused_weights) and takes the top-K in its
// epilogue.  More experts use launch_router_tc.
constexpr int kRouterFusedMaxExperts = 128;
bool router_uses_fused_tc(int N, int d, int E, int x_dtype);
size_t router_fused_weight_bytes(int d, int E);
cudaError_t launch_router_fused_split(const float* w_r, int d, int E, void* out,
                                      cudaStream_t stream);
bool encode_router_fused_weights(CUtensorMap* map, const void* split, int d, int E);
cudaError_t launch_router_fused(const void* x, const CUtensorMap& tmW, const float* bias, int N,
                                int d, int E, int K, int32_t* ids, float* gates, float* margin,
                                int* status, cudaStream_t stream);

// ---- permute ----------------------------------------------------------------
constexpr int kPermuteChunk = 32;   // tokens ranked by one warp (lane = token)
constexpr int kPermuteBlock = 256;  // tokens per rank CTA: its expert histogram is one row
inline int permute_blocks(int N) { return (N + kPermuteBlock - 1) / kPermuteBlock; }
// Device scratch of the rank pass: the block histograms (then bases) and the
// last-CTA counter (one unsigned, zero between calls).
inline size_t permute_block_counts_bytes(int N, int E) {
  return static_cast<size_t>(permute_blocks(N) > 0 ? permute_blocks(N) : 1) * E * 4;
}

// Writes each (t, j)'s rank within its 256-token block to local_rank (the
// perm_pos buffer; the gather turns it into the final position), the blocks'
// expert histograms to block_counts, and -- in the last CTA to finish, found
// through *counter, which must be zero on entry and is zero again on exit --
// the per-(block, expert) first destination rows (over block_counts), the
// expert counts and the offsets (E + 1).
// With src non-null (N*K <= kRankPositionsMaxRows) the last CTA also makes
// the final positions (local_rank -> pos, src[pos] = t), as the gather would.
constexpr long long kRankPositionsMaxRows = 8192;
cudaError_t launch_permute_rank(const int32_t* ids, int N, int K, int E, int32_t* block_counts,
                                unsigned* counter, int32_t* local_rank, int32_t* counts,
                                int32_t* offsets, int* status, cudaStream_t stream,
                                int32_t* src = nullptr);
// pos holds the ranks from launch_permute_rank on entry, the final
// positions on exit; src[pos] = t and, when slot is non-null,
// slot[pos] = t*K + j.  chunk_base = the block bases from the rank pass; a
// position outside [0, N*K) is recorded in status and skipped.  With x_perm
// NULL only the positions are made (no row is copied).
cudaError_t launch_permute_gather(const void* x, int row_bytes, const int32_t* ids, int N, int K,
                                  int E, const int32_t* chunk_base, int32_t* pos, int32_t* src,
                                  int32_t* slot, void* x_perm, int* status, cudaStream_t stream);

// The same with per-token dynamic quantization: x_bf16 (N, d) rows,
// d % 16 == 0; x_perm gets e4m3 codes (N*K, d), token_scale (N) the scales.
cudaError_t launch_permute_quant(const void* x_bf16, int d, const int32_t* ids, int N, int K,
                                 int E, const int32_t* chunk_base, int32_t* pos, int32_t* src,
                                 int32_t* slot, void* x_perm_e4m3, float* token_scale, int* status,
                                 cudaStream_t stream);

// ---- combine / unpermute ----------------------------------------------------
// y_dtype: kF32 or kBF16 (the dtype of y_perm and y).
cudaError_t launch_combine(const void* y_perm, int y_dtype, int dout, const int32_t* pos,
                           const float* gates, int N, int K, void* y, int* status,
                           cudaStream_t stream);

// ---- grouped FFN, fp32 SIMT path --------------------------------------------
// C[r, n] for rows of expert e: act(A[r,:] . W[e][n,:]) with A (R, kdim),
// W (E, ncols, kdim); SwiGLU uses W3 as the up matrix.  out (R, ncols) fp32.
// partial: split-K scratch of simt_f32_partial_bytes (NULL: no split).
cudaError_t launch_gemm_simt_f32(const float* A, int kdim, const float* W, const float* W3,
                                 int ncols, int act, float scale, const int32_t* offsets, int E,
                                 int R, float* out, float* partial, cudaStream_t stream);
int simt_f32_splits(int kdim, int ncols, int R, int E);
size_t simt_f32_partial_bytes(int kdim, int ncols, int R, int E, int act);

// ---- grouped GEMM on tcgen05 tensor cores -----------------------------------
// kEpiRouter: fp32 logits from the three-part split router weights (bf16,
// single-CTA tiles only).
// kEpiGroupScale: e4m3 store epilogue with fp32 scales per 128-element K
// stage (group / block quantization): every stage is accumulated alone and
// the epilogue adds it to fp32 registers times the stage's scales.
// kEpiGroupScale takes one weight scale per output column and stage,
// kEpiBlockScale one per 128 x 128 weight block.
enum TcEpilogue { kEpiStore = 0, kEpiSwiglu = 1, kEpiRouter = 2, kEpiGroupScale = 3,
                  kEpiBlockScale = 4 };

struct TcGemmArgs {
  CUtensorMap tmA;   // activations: rows (R), cols kdim
  CUtensorMap tmB0;  // weights: rows (groups * n_out), cols kdim (gate / single matrix)
  CUtensorMap tmB1;  // SwiGLU up matrix, same shape as tmB0
  const int32_t* offsets;  // (groups + 1) row offsets of A, device; NULL: one group of m_total
  int groups;              // experts (1 for a plain matmul)
  int m_total;             // rows of A and out; rows at or past it are never stored
  int kdim;
  int n_out;               // output columns per group
  int n_tiles;             // output column tiles per group
  void* out;               // bf16 (rows, ldo); fp32 for kEpiRouter
  long long ldo;           // elements
  float scale;             // multiplies the fp32 accumulator before rounding
  // finer scales (store epilogue): out = acc * scale * row_scale[row'] *
  // col_scale[g * n_out + col], row' = row_index[row] (or row); NULL = 1
  const float* row_scale;
  const int32_t* row_index;
  const float* col_scale;
  int* status;
  // Row scatter (unpermute fused into the store): when set, row r of the
  // result is stored at row out_rows[r] of out.
  const int32_t* out_rows;
  // MX block scales (GEMM dtype kGemmMxE4M3), in the tensor-core scale
  // layout below: sfa per 128-row tile of A counted over the groups' padded
  // tiles (group g's tiles follow those of groups < g, each group starting
  // a new tile), sfb per (group, 256-row weight tile).
  const uint8_t* sfa;
  const uint8_t* sfb;
  // Group scales (kEpiGroupScale, kEpiBlockScale), one per 128-element K
  // stage kb:
  //   out = sum_kb (xgs[row'][kb] (1 if NULL) * w) * acc_kb, then * scale * row_scale
  // w = wgs[(g * num_kb + kb) * n_out + col] (kEpiGroupScale, per output
  // column; the buffer holds 256 floats of slack past its end), or
  // wgs[(g * num_kb + kb) * ceil(n_out / 128) + col / 128] (kEpiBlockScale,
  // 128 x 128 weight blocks).  row' = row_index[row] (or row); num_kb =
  // kdim / 128.
  const float* xgs;
  const float* wgs;
  // Gathered A (bf16 SwiGLU gate/up GEMM, single CTA): when a_rows is set,
  // row r of A is row a_rows[r] of the matrix under tmAg (a box one row
  // high, 128 bytes of K); tmA is not read.
  const int32_t* a_rows;
  CUtensorMap tmAg;
  // Tile stores by TMA (bf16 out with contiguous rows, out_rows NULL): when
  // out_tma is set, tmOut covers out as m_total rows of n_out columns, ldo
  // apart (encode_out_map: 32 x 32 boxes, 64-byte swizzle); a warp whose 32
  // rows are all stored hands each 32-column chunk to the TMA engine.
  CUtensorMap tmOut;
  int out_tma;
};

// Host: the tile-store map of a bf16 (rows, cols) matrix, ld elements apart.
bool encode_out_map(CUtensorMap* map, void* base, long long rows, long long cols, long long ld);

// Host: encode a 2-D K-major tile map over a (rows, kdim) row-major matrix of
// elem_bytes-wide elements; box = (128 bytes of K) x box_rows, 128-B swizzle.
bool encode_kmajor_map(CUtensorMap* map, const void* base, int elem_bytes, long long rows,
                       long long kdim, int box_rows);

// dtype kBF16 or kE4M3.  offsets on device; rows_upper = upper bound of the
// number of A rows (to size the grid).  pair: 256-row tiles on CTA pairs
// (tcgen05 cta_group::2); the B maps then have 128-row boxes for the store
// epilogue (each CTA loads half of the 256 weight rows).
// dtype kGemmMxE4M3: e4m3 operands with MX block scales (args.sfa, args.sfb),
// single CTA, store epilogue only.
cudaError_t launch_gemm_tc(const TcGemmArgs& args, int dtype, int epilogue, int rows_upper,
                           bool pair, cudaStream_t stream);
constexpr int kTcBlockM = 128;
constexpr int kTcBlockN = 256;  // accumulator columns; SwiGLU: 128 gate + 128 up

// e4m3 GEMM with per-column group scales (the kEpiGroupScale arithmetic;
// launch_gemm_tc refuses that epilogue): 128 x 128 tiles, so args.n_tiles =
// ceil(n_out / kGsTileN) and tmB0 has 128-row boxes; the other fields as for
// launch_gemm_tc's block-scaled epilogue.
constexpr int kGsTileN = 128;
cudaError_t launch_gemm_gs(const TcGemmArgs& args, int rows_upper, cudaStream_t stream);
constexpr int kGemmMxE4M3 = 3;

// ---- MX (OCP MXFP8) block scales in the tensor-core layout ----------------
// One E8M0 byte scales 32 consecutive elements of K.  The GEMM consumes them
// per 128-element K stage as 512-byte atoms of 128 rows x 4 scales: the
// scale j (0..3) of row i (0..127) sits at byte (i % 32) * 16 + (i / 32) * 4
// + j, the order in which tcgen05.cp 32x128b.warpx4 fills the scale columns
// of the block-scaled MMA.  Scales past the end of K or of the rows are 127
// (1.0; their operands are zero or never stored).
//   weights: atom ((g * n_tiles + nt) * num_kb + kb) * 2 + h covers weight
//            rows nt * 256 + h * 128 + i of group g, n_tiles = ceil(n_out / 256)
//   activations: atom (pt * num_kb + kb) covers padded row 128 * pt + i
// with num_kb = ceil(kdim / 128).
constexpr int kMxBlock = 32;
constexpr int kMxMaxKdim = 32768;  // MX layers: d <= 32768 (one 128-row tile's scales in 128 KB)
constexpr int kMxAtomBytes = 512;
__host__ __device__ inline int mx_num_kb(int kdim) { return (kdim + 127) / 128; }
inline size_t mx_weight_sf_bytes(int groups, int n_out, int kdim) {
  return static_cast<size_t>(groups) * ((n_out + kTcBlockN - 1) / kTcBlockN) * mx_num_kb(kdim) * 2 *
         kMxAtomBytes;
}
// upper bound of the padded activation tiles of `rows` rows over `groups`
inline size_t mx_act_sf_bytes(long long rows, int groups, int kdim) {
  return static_cast<size_t>(rows / kTcBlockM + groups + 1) * mx_num_kb(kdim) * kMxAtomBytes;
}
// w_sf (groups, n_out, kdim / 32) row-major -> the weight atoms.
cudaError_t launch_mx_weight_sf(const uint8_t* w_sf, int groups, int n_out, int kdim, uint8_t* out,
                                cudaStream_t stream);
// Activation atoms of the permuted rows r < offsets[groups] (at most
// rows_upper): the scales of row r are row src_rows[r] (or r when NULL) of
// x_sf (*, kdim / 32) row-major.
cudaError_t launch_mx_act_sf(const uint8_t* x_sf, const int32_t* src_rows, const int32_t* offsets,
                             int groups, int rows_upper, int kdim, uint8_t* out,
                             cudaStream_t stream);
// Group / block scales of the weights, (E, rows, ng) fp32 -> the kernel's
// (E, ng, rows) layout (rows = F per output column, or ceil(F / 128) blocks).
cudaError_t launch_group_scales_t(const float* src, int groups, int rows, int ng, float* dst,
                                  cudaStream_t stream);
// Row gather of scales: out row r = x_sf row src_rows[r], for r <
// offsets[groups] (at most rows_upper); nsf bytes per row.
cudaError_t launch_mx_sf_gather(const uint8_t* x_sf, const int32_t* src_rows,
                                const int32_t* offsets, int groups, int rows_upper, int nsf,
                                uint8_t* out, cudaStream_t stream);

int device_sm_count();

// Warps per token row for the row-copy kernels (gather, combine): the
// smallest of 1, 2, 4, 8 that puts about 16 warps per SM in flight.
inline int warps_per_token(int N) {
  const long long want = 16LL * device_sm_count();
  if (N >= want) return 1;
  if (2LL * N >= want) return 2;
  if (4LL * N >= want) return 4;
  return 8;
}

// Shape of a plan for code outside the plan's translation unit: tokens,
// token width, experts, experts per token and bytes per token row of x.
// Returns false for a null plan.
bool plan_permute_shape(const ::moe_plan_s* plan, int* N, int* d, int* E, int* K,
                        int* row_bytes);

// Per-call bookkeeping of a plan for entry points outside the plan's
// translation unit: begin() clears the launch count and the stage events,
// mark() records the boundary before the named stage (when per-stage timing
// is on), end() records the last boundary and adds the call's launches to
// the count that moe_last_launch_count reports.
void plan_call_begin(::moe_plan_s* plan);
void plan_call_mark(::moe_plan_s* plan, cudaStream_t s, const char* name_of_next);
void plan_call_end(::moe_plan_s* plan, cudaStream_t s, int launches);

}  // namespace moe
