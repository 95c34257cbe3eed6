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

// ---- permute ----------------------------------------------------------------
constexpr int kPermuteChunk = 32;  // tokens per chunk of the stable counting pass
inline int permute_chunks(int N) { return (N + kPermuteChunk - 1) / kPermuteChunk; }

// Writes each (t, j)'s rank within its 32-token chunk to local_rank (the
// perm_pos buffer; the gather turns it into the final position) and the
// chunk's expert histogram to chunk_counts.
cudaError_t launch_permute_count(const int32_t* ids, int N, int K, int E, int32_t* chunk_counts,
                                 int32_t* local_rank, int* status, cudaStream_t stream);
cudaError_t launch_permute_scan(int32_t* chunk_counts, int nchunks, int E, int32_t* counts,
                                int32_t* offsets, cudaStream_t stream);
// pos holds the ranks from launch_permute_count on entry, the final
// positions on exit; src[pos] = t and, when slot is non-null,
// slot[pos] = t*K + j.
cudaError_t launch_permute_gather(const void* x, int row_bytes, const int32_t* ids, int N, int K,
                                  int E, const int32_t* chunk_base, int32_t* pos, int32_t* src,
                                  int32_t* slot, void* x_perm, int* status, cudaStream_t stream);

// The same with per-token dynamic quantization: x_bf16 (N, d) rows,
// d % 16 == 0; x_perm gets e4m3 codes (N*K, d), token_scale (N) the scales.
cudaError_t launch_permute_quant(const void* x_bf16, int d, const int32_t* ids, int N, int K,
                                 int E, const int32_t* chunk_base, int32_t* pos, int32_t* src,
                                 int32_t* slot, void* x_perm_e4m3, float* token_scale,
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
enum TcEpilogue { kEpiStore = 0, kEpiSwiglu = 1, kEpiRouter = 2 };

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
};

// Host: encode a 2-D K-major tile map over a (rows, kdim) row-major matrix of
// elem_bytes-wide elements; box = (128 bytes of K) x box_rows, 128-B swizzle.
bool encode_kmajor_map(CUtensorMap* map, const void* base, int elem_bytes, long long rows,
                       long long kdim, int box_rows);

// dtype kBF16 or kE4M3.  offsets on device; rows_upper = upper bound of the
// number of A rows (to size the grid).  pair: 256-row tiles on CTA pairs
// (tcgen05 cta_group::2); the B maps then have 128-row boxes for the store
// epilogue (each CTA loads half of the 256 weight rows).
cudaError_t launch_gemm_tc(const TcGemmArgs& args, int dtype, int epilogue, int rows_upper,
                           bool pair, cudaStream_t stream);
constexpr int kTcBlockM = 128;
constexpr int kTcBlockN = 256;  // accumulator columns; SwiGLU: 128 gate + 128 up

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

}  // namespace moe
