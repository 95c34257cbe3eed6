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
// k-step yields all three partial logits of 64 experts for 128 tokens.
// Structure: one CTA per 128-token tile (persistent), warp 0 streams x and
// weight tiles with TMA into a 4-stage ring, warp 1 issues the MMAs into two
// TMEM accumulators (one per expert chunk, double-buffered), warps 2..5 (one
// token row per thread) add the three parts and store the fp32 logits.  A
// warp-per-token kernel then takes the top-K (value desc, index asc), the
// softmax over the kept K and the margin, shared with the SIMT routers.
// (Keeping a running top-(K+1) list per thread in the epilogue instead made
// the epilogue, one warp per SM sub-partition on serial compare chains, the
// bound: 116 us against 44 us without it on the 16384-token, 128-expert
// workload.)
#include <float.h>
#include <limits.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace tc;

constexpr int RM = 128;    // tokens per tile
constexpr int REC = 64;    // experts per chunk
constexpr int RN = 256;    // MMA N: hi | mid | lo | zero rows of a chunk
constexpr int RROWB = 128;
constexpr int RSTAGES = 4;
constexpr int RA_BYTES = RM * RROWB;
constexpr int RB_BYTES = RN * RROWB;
constexpr int RSTAGE_BYTES = RA_BYTES + RB_BYTES;
constexpr int kRThreads = 192;
constexpr uint32_t kRTmemCols = 2 * RN;
constexpr int kRBarFull = 0, kRBarEmpty = RSTAGES, kRBarTFull = 2 * RSTAGES,
              kRBarTEmpty = 2 * RSTAGES + 2, kRNumBars = 2 * RSTAGES + 4;
constexpr int kRSmemBytes = 1024 + RSTAGES * RSTAGE_BYTES + kRNumBars * 8 + 16;

// fp32 accumulator, bf16 A and B, both K-major, N = 256, M = 128
constexpr uint32_t kRouterIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                  (static_cast<uint32_t>(RN >> 3) << 17) |
                                  (static_cast<uint32_t>(RM >> 4) << 24);

__global__ void __launch_bounds__(256)
router_split_kernel(const float* __restrict__ w_r, int d, int E, int nchunks,
                    __nv_bfloat16* __restrict__ w3) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  const long long total = static_cast<long long>(nchunks) * REC * d;
  for (long long idx = blockIdx.x * 256ll + threadIdx.x; idx < total; idx += 256ll * gridDim.x) {
    const int e = static_cast<int>(idx / d), k = static_cast<int>(idx % d);
    const float w = e < E ? w_r[static_cast<long long>(k) * E + e] : 0.f;
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

struct RouterTcArgs {
  CUtensorMap tmX;  // x: rows N, cols d, 128-row boxes
  CUtensorMap tmW;  // split weights: rows nchunks*256, cols d, 256-row boxes
  int N, d, E, nchunks;
  float* logits;  // (N, E) fp32
  int* status;
};

__global__ void __launch_bounds__(kRThreads, 1) router_tc_kernel(const __grid_constant__ RouterTcArgs args) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + RSTAGES * RA_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + RSTAGES * RSTAGE_BYTES);
  const uint32_t bar0 = smem_u32(bars);
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kRNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 32) {
    for (int s = 0; s < RSTAGES; ++s) {
      mbar_init(bar(kRBarFull + s), 1);
      mbar_init(bar(kRBarEmpty + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(kRBarTFull + a), 1);
      mbar_init(bar(kRBarTEmpty + a), 4);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&args.tmX);
    tma_prefetch_desc(&args.tmW);
  }
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kRTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int ntiles = (args.N + RM - 1) / RM;
  const int num_kb = (args.d + 63) / 64;
  const int nchunks = args.nchunks;
  // Every CTA reads the same split-weight tiles; starting each CTA's k loop
  // at a different block (rotated order) spreads those reads over the L2
  // instead of sending all CTAs to the same lines at once.
  const int kb_first = static_cast<int>(blockIdx.x % static_cast<unsigned>(num_kb));

  if (warp == 0) {
    if (lane == 0) {  // ---- TMA producer ----
      int s = 0;
      uint32_t ph = 0;
      bool aborted = false;
      for (int t = blockIdx.x; t < ntiles && !aborted; t += gridDim.x)
        for (int c = 0; c < nchunks && !aborted; ++c)
          for (int j = 0; j < num_kb; ++j) {
            const int kb = kb_first + j < num_kb ? kb_first + j : kb_first + j - num_kb;
            if (!mbar_wait(bar(kRBarEmpty + s), ph ^ 1u, abort_flag)) { aborted = true; break; }
            mbar_expect_tx(bar(kRBarFull + s), RSTAGE_BYTES);
            tma_load_2d(sA + s * RA_BYTES, &args.tmX, kb * 64, t * RM, bar(kRBarFull + s));
            tma_load_2d(sB + s * RB_BYTES, &args.tmW, kb * 64, c * RN, bar(kRBarFull + s));
            if (++s == RSTAGES) { s = 0; ph ^= 1u; }
          }
      if (aborted) set_status(args.status, kStatusTimeout);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer ----
      int s = 0;
      uint32_t ph = 0;
      bool aborted = false;
      int i = 0;
      for (int t = blockIdx.x; t < ntiles && !aborted; t += gridDim.x)
        for (int c = 0; c < nchunks; ++c, ++i) {
          const int acc = i & 1;
          const uint32_t aph = (i >> 1) & 1;
          if (!mbar_wait(bar(kRBarTEmpty + acc), aph ^ 1u, abort_flag)) { aborted = true; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * RN);
          for (int j = 0; j < num_kb; ++j) {  // k blocks in the producer's rotated order
            if (!mbar_wait(bar(kRBarFull + s), ph, abort_flag)) { aborted = true; break; }
            tc_fence_after();
            const uint32_t a0 = sA + s * RA_BYTES, b0 = sB + s * RB_BYTES;
#pragma unroll
            for (int k = 0; k < 4; ++k)
              tc_mma<false>(d_tmem, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), kRouterIdesc,
                            (j | k) != 0 ? 1u : 0u);
            tc_commit(bar(kRBarEmpty + s));
            if (++s == RSTAGES) { s = 0; ph ^= 1u; }
          }
          if (aborted) break;
          tc_commit(bar(kRBarTFull + acc));
        }
      if (aborted) set_status(args.status, kStatusTimeout);
    }
    __syncwarp();
  } else {
    // ---- epilogue: one token row per thread ----
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int E = args.E;
    const bool vec = (E & 3) == 0;
    int i = 0;
    bool aborted = false;
    for (int t = blockIdx.x; t < ntiles && !aborted; t += gridDim.x) {
      const long long tok = static_cast<long long>(t) * RM + row;
      float* lrow = args.logits + tok * E;
      for (int c = 0; c < nchunks; ++c, ++i) {
        const int acc = i & 1;
        const uint32_t aph = (i >> 1) & 1;
        const bool ok =
            __shfl_sync(0xffffffffu, mbar_wait(bar(kRBarTFull + acc), aph, abort_flag), 0);
        if (!ok) {
          set_status(args.status, kStatusTimeout);
          aborted = true;
          break;
        }
        tc_fence_after();
        const uint32_t tb =
            tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * RN);
#pragma unroll 1
        for (int h = 0; h < REC; h += 32) {
          uint32_t vh[32], vm[32], vl[32];
          __syncwarp();
          tmem_ld32(tb + h, vh);
          tmem_ld32(tb + REC + h, vm);
          tmem_ld32(tb + 2 * REC + h, vl);
          tmem_ld_wait();
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j)
            v[j] = (__uint_as_float(vh[j]) + __uint_as_float(vm[j])) + __uint_as_float(vl[j]);
          const int e0 = c * REC + h;
          if (tok < args.N && e0 < E) {
            if (vec && e0 + 32 <= E) {
              float4* dst = reinterpret_cast<float4*>(lrow + e0);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (e0 + j < E) lrow[e0 + j] = v[j];
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kRBarTEmpty + acc));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kRTmemCols)
                 : "memory");
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
    const long long total = static_cast<long long>(nchunks) * REC * d;
    long long blocks = (total + 255) / 256;
    if (blocks > 4LL * device_sm_count()) blocks = 4LL * device_sm_count();
    cudaError_t e = launch_pdl(router_split_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                               stream, w_r, d, E, nchunks, w3);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  RouterTcArgs a;
  memset(&a, 0, sizeof(a));
  if (!encode_kmajor_map(&a.tmX, x, 2, N, d, RM) ||
      !encode_kmajor_map(&a.tmW, w3, 2, static_cast<long long>(nchunks) * RN, d, RN))
    return cudaErrorInvalidValue;
  a.N = N;
  a.d = d;
  a.E = E;
  a.nchunks = nchunks;
  a.logits = reinterpret_cast<float*>(static_cast<char*>(scratch) + split_weight_bytes(d, E));
  a.status = status;
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kRSmemBytes);
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  const int ntiles = (N + RM - 1) / RM;
  const int grid = ntiles < device_sm_count() ? ntiles : device_sm_count();
  cudaError_t e = launch_pdl(router_tc_kernel, dim3(grid), dim3(kRThreads), kRSmemBytes, stream, a);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_logits_topk(a.logits, bias, N, E, K, ids, gates, margin, stream);
}

}  // namespace moe
