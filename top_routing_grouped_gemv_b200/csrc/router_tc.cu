// Router on the 5th-generation tensor cores, for bf16 tokens and many
// experts ("Advanced GPU Optimization ... Part 5", section 1.1 The Router
// Kernel: expert scores from the router weights, the best experts tracked,
// softmax over the kept scores; zyxy.net MoE page, expert selection).
//
// The logits x . W_r are a dense (N x d) x (d x E) contraction, so they run
// on tcgen05 like the expert GEMMs, with fp32-level accuracy kept by an exact
// split of the fp32 router weights into three bf16 parts:
//   w = hi + mid + lo,  hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid)
// (each difference is exact in fp32; the three parts carry 24 significant
// bits).  bf16 x times a bf16 part is exact in the fp32 accumulator, so
//   logit[t, e] = (x.hi)[t, e] + (x.mid)[t, e] + (x.lo)[t, e]
// matches the fp32 dot product to within fp32 accumulation error.
//
// The split weights are laid out per chunk of 64 experts as 256 K-major rows
// [hi(64) | mid(64) | lo(64) | zero(64)], so one M=128, N=256, K=16 MMA per
// k-step yields all three partial logits of 64 experts for 128 tokens.  The
// contraction runs on the persistent grouped-GEMM kernel (one group, rows =
// tokens, one column tile per chunk) with its router epilogue, which adds
// the three parts and stores fp32 logits; a warp-per-token kernel shared
// with the SIMT routers then takes the top-K (value desc, index asc), the
// softmax over the kept K and the margin.
// (A dedicated kernel with one CTA per 128-token tile that kept a running
// top-9 list per thread in its epilogue was bound by that epilogue: 116 us
// against 44 us without it for 16384 tokens x 128 experts.)
#include <string.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int REC = 64;    // experts per chunk
constexpr int RN = 256;    // rows per chunk: hi | mid | lo | zero

// w_r (d, E) fp32 row-major -> per 64-expert chunk the 256 rows
// [hi | mid | lo | zero] of length d (bf16, K-major): a transpose, through a
// 32 x 32 shared tile so that both the reads (along e) and the writes (along
// k) are coalesced.  Block (32, 8); grid (chunk rows / 32, d / 32).
__global__ void __launch_bounds__(256)
router_split_kernel(const float* __restrict__ w_r, int d, int E, __nv_bfloat16* __restrict__ w3) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  __shared__ float tile[32][33];
  const int e0 = blockIdx.x * 32, k0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int r = ty; r < 32; r += 8) {
    const int k = k0 + r, e = e0 + tx;
    tile[r][tx] = (k < d && e < E) ? w_r[static_cast<long long>(k) * E + e] : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int e = e0 + r, k = k0 + tx;
    if (k >= d) continue;
    const float w = tile[tx][r];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
    const long long row = static_cast<long long>(e / REC) * RN + (e % REC);
    w3[row * d + k] = hi;
    w3[(row + REC) * d + k] = mid;
    w3[(row + 2 * REC) * d + k] = lo;
    w3[(row + 3 * REC) * d + k] = __float2bfloat16_rn(0.f);
  }
}

}  // namespace

// scratch: the split weights (nchunks * 256 rows of d bf16), then the fp32
// logits (N, E)
static size_t split_weight_bytes(int d, int E) {
  const int nchunks = (E + REC - 1) / REC;
  return static_cast<size_t>(nchunks) * RN * d * sizeof(__nv_bfloat16);
}

size_t router_tc_scratch_bytes(int N, int d, int E) {
  return split_weight_bytes(d, E) + static_cast<size_t>(N) * E * sizeof(float);
}

cudaError_t launch_router_tc(const void* x, const float* w_r, const float* bias, int N, int d,
                             int E, int K, int32_t* ids, float* gates, float* margin,
                             void* scratch, int* status, cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  const int nchunks = (E + REC - 1) / REC;
  auto* w3 = static_cast<__nv_bfloat16*>(scratch);
  {
    const dim3 grid(static_cast<unsigned>(nchunks * REC / 32), static_cast<unsigned>((d + 31) / 32));
    cudaError_t e = launch_pdl(router_split_kernel, grid, dim3(32, 8), 0, stream, w_r, d, E, w3);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  float* logits = reinterpret_cast<float*>(static_cast<char*>(scratch) + split_weight_bytes(d, E));
  TcGemmArgs a;
  memset(&a, 0, sizeof(a));
  if (!encode_kmajor_map(&a.tmA, x, 2, N, d, kTcBlockM) ||
      !encode_kmajor_map(&a.tmB0, w3, 2, static_cast<long long>(nchunks) * RN, d, RN))
    return cudaErrorInvalidValue;
  a.tmB1 = a.tmB0;
  a.offsets = nullptr;  // one group: all tokens
  a.groups = 1;
  a.m_total = N;
  a.kdim = d;
  a.n_out = E;          // logit columns
  a.n_tiles = nchunks;  // one column tile of 64 experts per chunk
  a.out = logits;
  a.ldo = E;
  a.scale = 1.f;
  a.status = status;
  cudaError_t e = launch_gemm_tc(a, kBF16, kEpiRouter, N, false, stream);
  if (e != cudaSuccess) return e;
  return launch_logits_topk(logits, bias, N, E, K, ids, gates, margin, stream);
}

}  // namespace moe
