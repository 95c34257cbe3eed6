// Grouped e4m3 GEMM with fp32 scales per output column and 128-element group
// of K, on tcgen05.
//
// What it computes (aclnnQuantGroupedMatMulAlltoAllv, parameter section:
// quantisation mode 4, per-group; the formula section's gmmY with the scales
// taken per group of the reduction): for every expert g and row r of its
// rows, every output column n,
//   out[r][n] = scale * row_scale[r'] * sum_kb xgs[r'][kb] * w[kb][n] * acc_kb[r][n]
// where acc_kb is the fp32 product of the 128 K elements of group kb (e4m3 x
// e4m3, exact products summed by the tensor core), w[kb][n] =
// wgs[(g*num_kb + kb) * n_out + n], and r' = row_index[r] (or r).
//
// A scale that changes every 128 elements of K cannot ride in the tensor
// core's accumulator: every K group lands in a fresh accumulator, which the
// CUDA cores scale and add to fp32 sums in registers.  With a scale per
// column that is two operations per element on the CUDA cores, as long as
// the K group's MMAs, and the accumulator hand-off (MMA done -> epilogue
// reads it -> MMA may overwrite it) has a long round trip.  So the tile is
// 128 x 128 and TMEM holds four accumulators of 128 columns: the MMAs run up
// to three K groups ahead of the epilogue, and the epilogue gives an
// accumulator back as soon as its columns are in registers and scales and
// adds them while the next MMAs run (3.3 -> 2.8 ms on the full fp8 layer
// against the 128 x 256 tile with two accumulators; with one scale per
// 128 x 128 weight block, whose epilogue is one multiply-add per element,
// the 128 x 256 tile stays faster, 1.45 against 2.35 ms, and runs in
// gemm_tc.cu).
//
// Structure (one persistent CTA per SM, 10 warps):
//   warp 0      TMA producer: 128 rows of A and 128 weight rows per 128-element
//               K stage (128-byte swizzle) into a 6-stage ring
//   warp 1      TMEM owner; lane 0 issues tcgen05.mma kind::f8f6f4 (M=128,
//               N=128, K=32) into accumulator (stage mod 4)
//   warps 2..9  epilogue: two warps per TMEM lane quadrant, 64 columns each;
//               row scales read three stages ahead (registers), column
//               scales by cp.async into a four-slot ring of the warp's
//               shared memory
// The tile list is the grouped one of the other tensor-core GEMMs
// (grouped_tiles.cuh).  Every mbarrier wait is bounded (1 s): on expiry the
// CTA records MOE_ERR_DEVICE_TIMEOUT, the roles leave their loops, copies and
// MMAs in flight are drained (bounded) and TMEM is freed before exit.
#include <cuda.h>

#include "common.cuh"
#include "grouped_tiles.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace tc;

constexpr int kGsBM = 128;             // rows per tile
constexpr int kGsBN = 128;             // columns per tile
constexpr int kGsRowB = 128;           // bytes of K per row per stage (128 e4m3)
constexpr int kGsStages = 6;           // smem ring
constexpr int kGsAcc = 4;              // TMEM accumulators of kGsBN columns
constexpr int kGsEpiWarps = 8;         // two per lane quadrant
constexpr int kGsCols = kGsBN / 2;     // columns per epilogue warp
constexpr int kGsAhead = 3;            // scale prefetch distance (stages)
constexpr int kGsRing = kGsAhead + 1;  // per-column scale slots per warp
constexpr int kGsThreads = 32 * (2 + kGsEpiWarps);
constexpr int kGsMaxGroups = 256;

struct GsGeo {
  static constexpr int A_BYTES = kGsBM * kGsRowB;
  static constexpr int B_BYTES = kGsBN * kGsRowB;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int kBarFull = 0, kBarEmpty = kGsStages, kBarTFull = 2 * kGsStages,
                       kBarTEmpty = 2 * kGsStages + kGsAcc, kBarDrain = 2 * kGsStages + 2 * kGsAcc,
                       kNumBars = 2 * kGsStages + 2 * kGsAcc + 1;
  // ring | barriers | TMEM slot + abort flag (16 B) | tile prefix and group
  // offsets | per-column scale rings (16-byte aligned)
  static constexpr int kRingFloats = kGsEpiWarps * kGsRing * kGsCols;
  static constexpr int kSmemBytes = 1024 /*alignment slack*/ + kGsStages * STAGE_BYTES +
                                    kNumBars * 8 + 16 + 2 * (kGsMaxGroups + 1) * 4 + 16 +
                                    kRingFloats * 4;
};

// fp8 e4m3 x e4m3 -> fp32, M = 128, N = 128, both operands K-major.
constexpr uint32_t kGsIdesc = (1u << 4) | (static_cast<uint32_t>(kGsBN >> 3) << 17) |
                              (static_cast<uint32_t>(kGsBM >> 4) << 24);

__global__ void __launch_bounds__(kGsThreads, 1)
gemm_gs_kernel(const __grid_constant__ TcGemmArgs args) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  using Gm = GsGeo;
  extern __shared__ uint8_t gs_smem_raw[];
  const uint32_t raw = smem_u32(gs_smem_raw);
  uint8_t* smem = gs_smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + kGsStages * Gm::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kGsStages * Gm::STAGE_BYTES);
  const uint32_t bar0 = smem_u32(bars);
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Gm::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_pref = reinterpret_cast<int*>(tmem_slot + 4);
  int* s_off = s_pref + (kGsMaxGroups + 1);
  float* s_wring = reinterpret_cast<float*>(
      (reinterpret_cast<uintptr_t>(s_off + kGsMaxGroups + 1) + 15) & ~static_cast<uintptr_t>(15));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = args.groups;
  const int unit = static_cast<int>(blockIdx.x), nunits = static_cast<int>(gridDim.x);

  if (warp == 0)
    build_tile_prefix<kGsBM>(args.offsets, G, args.m_total, args.n_tiles, lane, s_pref, s_off);
  if (threadIdx.x == 32) {
    for (int s = 0; s < kGsStages; ++s) {
      mbar_init(bar(Gm::kBarFull + s), 1);
      mbar_init(bar(Gm::kBarEmpty + s), 1);
    }
    for (int a = 0; a < kGsAcc; ++a) {
      mbar_init(bar(Gm::kBarTFull + a), 1);
      mbar_init(bar(Gm::kBarTEmpty + a), kGsEpiWarps);
    }
    mbar_init(bar(Gm::kBarDrain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&args.tmA);
    tma_prefetch_desc(&args.tmB0);
  }
  if (warp == 1) {
    __syncwarp();  // tcgen05.alloc is .sync.aligned: converge after thread 32's branch
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kGsAcc * kGsBN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_pref[G];
  const int num_kb = args.kdim / kGsRowB;  // K groups of 128 (kdim % 128 == 0)

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_ph = 0;
      bool aborted = false;
      for (int T = unit; T < total && !aborted; T += nunits) {
        const TileCoord c = decode_tile<kGsBM>(T, s_pref, s_off, G, args.n_tiles);
        const int brow = c.g * args.n_out + c.n_tile * kGsBN;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(bar(Gm::kBarEmpty + s), ph ^ 1u, abort_flag)) { aborted = true; break; }
          const int kx = kb * kGsRowB;
          mbar_expect_tx(bar(Gm::kBarFull + s), Gm::STAGE_BYTES);
          tma_load_2d(sA + s * Gm::A_BYTES, &args.tmA, kx, c.m_row0, bar(Gm::kBarFull + s));
          tma_load_2d(sB + s * Gm::B_BYTES, &args.tmB0, kx, brow, bar(Gm::kBarFull + s));
          issued |= 1u << s;
          issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
          if (++s == kGsStages) { s = 0; ph ^= 1u; }
        }
      }
      if (aborted) {
        set_status(args.status, kStatusTimeout);
        // let copies already in flight land before the CTA's memory is reused
        for (int i = 0; i < kGsStages; ++i)
          if ((issued >> i) & 1u) mbar_wait_drain(bar(Gm::kBarFull + i), (issued_ph >> i) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer: K group j into accumulator j mod 4 ----------------
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0, j = 0;
      bool aborted = false;
      for (int T = unit; T < total && !aborted; T += nunits) {
        for (int kb = 0; kb < num_kb; ++kb, ++j) {
          const uint32_t acc = j % kGsAcc, aph = (j / kGsAcc) & 1u;
          if (!mbar_wait(bar(Gm::kBarTEmpty + acc), aph ^ 1u, abort_flag)) { aborted = true; break; }
          if (!mbar_wait(bar(Gm::kBarFull + s), ph, abort_flag)) { aborted = true; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + acc * static_cast<uint32_t>(kGsBN);
          const uint32_t a0 = sA + s * Gm::A_BYTES, b0 = sB + s * Gm::B_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma<true>(d_tmem, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), kGsIdesc,
                         k != 0 ? 1u : 0u);
          tc_commit(bar(Gm::kBarEmpty + s));
          tc_commit(bar(Gm::kBarTFull + acc));
          if (++s == kGsStages) { s = 0; ph ^= 1u; }
        }
      }
      if (aborted) {
        set_status(args.status, kStatusTimeout);
        // every MMA issued so far has finished before TMEM is freed
        tc_commit(bar(Gm::kBarDrain));
        mbar_wait_drain(bar(Gm::kBarDrain), 0);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue ----------------
    const int q = warp & 3;            // TMEM lane quadrant this warp may access
    const int half = (warp - 2) >> 2;  // its 64 columns of the tile
    float* wring = s_wring + (warp - 2) * (kGsRing * kGsCols);
    uint32_t j = 0;
    bool ok = true;
    for (int T = unit; T < total && ok; T += nunits) {
      const TileCoord c = decode_tile<kGsBM>(T, s_pref, s_off, G, args.n_tiles);
      const int row = q * 32 + lane;
      const long long grow = static_cast<long long>(c.m_row0) + row;
      const bool valid = grow < s_off[c.g + 1] && grow < args.m_total && grow >= 0;
      const long long srow = valid && args.row_index != nullptr ? args.row_index[grow] : grow;
      const int col0 = c.n_tile * kGsBN + half * kGsCols;
      const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(half * kGsCols);
      // the stage's row scale, kGsAhead stages ahead
      const float* xrow = valid && args.xgs != nullptr ? args.xgs + srow * num_kb : nullptr;
      float f_q[kGsAhead];
#pragma unroll
      for (int u = 0; u < kGsAhead; ++u) f_q[u] = xrow != nullptr && u < num_kb ? xrow[u] : 1.f;
      // per-column scales: lane l copies those of columns 4l..4l+3 from col0
      // (lanes 0..15), stage kb into slot kb % kGsRing of this warp's ring;
      // the buffer has 256 floats of slack past its last column
      const float* wcol = args.wgs + static_cast<long long>(c.g) * num_kb * args.n_out + col0 +
                          4 * lane;
      __syncwarp();  // the previous tile's reads of the ring are done
#pragma unroll
      for (int u = 0; u < kGsAhead; ++u) {
        if (lane < kGsCols / 4 && u < num_kb)
          cp_async16(smem_u32(wring + (u % kGsRing) * kGsCols + 4 * lane),
                     wcol + static_cast<long long>(u) * args.n_out);
        cp_async_commit();
      }
      float sum[kGsCols];
#pragma unroll
      for (int cc = 0; cc < kGsCols; ++cc) sum[cc] = 0.f;
      for (int kb = 0; kb < num_kb; ++kb, ++j) {
        const uint32_t acc = j % kGsAcc, aph = (j / kGsAcc) & 1u;
        const float sx = f_q[0];
#pragma unroll
        for (int u = 0; u + 1 < kGsAhead; ++u) f_q[u] = f_q[u + 1];
        const int kn = kb + kGsAhead;
        if (kn < num_kb && xrow != nullptr) f_q[kGsAhead - 1] = xrow[kn];
        __syncwarp();  // every lane is done with the slot refilled now (stage kb - 1's)
        if (lane < kGsCols / 4 && kn < num_kb)
          cp_async16(smem_u32(wring + (kn % kGsRing) * kGsCols + 4 * lane),
                     wcol + static_cast<long long>(kn) * args.n_out);
        cp_async_commit();
        ok = __shfl_sync(0xffffffffu, mbar_wait(bar(Gm::kBarTFull + acc), aph, abort_flag), 0);
        if (!ok) break;
        tc_fence_after();
        uint32_t v0[32], v1[32];
        __syncwarp();
        tmem_ld32(tq + acc * kGsBN, v0);
        tmem_ld32(tq + acc * kGsBN + 32, v1);
        tmem_ld_wait();
        // the accumulator is in registers: a later K group's MMAs may overwrite it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(Gm::kBarTEmpty + acc));
        {
          // the stage's column scales, read four at a time by every lane (one
          // broadcast load), times this lane's row scale
          cp_async_wait<kGsAhead>();  // this lane's copy of stage kb has landed
          __syncwarp();               // and every lane's
          const float4* wsm = reinterpret_cast<const float4*>(wring + (kb % kGsRing) * kGsCols);
#pragma unroll
          for (int jj = 0; jj < 32; jj += 4) {
            const float4 wa = wsm[jj >> 2], wb = wsm[(32 + jj) >> 2];
            sum[jj] = fmaf(__uint_as_float(v0[jj]), wa.x * sx, sum[jj]);
            sum[jj + 1] = fmaf(__uint_as_float(v0[jj + 1]), wa.y * sx, sum[jj + 1]);
            sum[jj + 2] = fmaf(__uint_as_float(v0[jj + 2]), wa.z * sx, sum[jj + 2]);
            sum[jj + 3] = fmaf(__uint_as_float(v0[jj + 3]), wa.w * sx, sum[jj + 3]);
            sum[32 + jj] = fmaf(__uint_as_float(v1[jj]), wb.x * sx, sum[32 + jj]);
            sum[33 + jj] = fmaf(__uint_as_float(v1[jj + 1]), wb.y * sx, sum[33 + jj]);
            sum[34 + jj] = fmaf(__uint_as_float(v1[jj + 2]), wb.z * sx, sum[34 + jj]);
            sum[35 + jj] = fmaf(__uint_as_float(v1[jj + 3]), wb.w * sx, sum[35 + jj]);
          }
        }
      }
      if (!ok) {
        set_status(args.status, kStatusTimeout);
        cp_async_wait<0>();  // no copy outlives the CTA
        break;
      }
      if (valid) {
        float sc = args.scale;
        if (args.row_scale != nullptr)
          sc *= args.row_scale[args.row_index != nullptr ? args.row_index[grow] : grow];
        const long long orow_i = args.out_rows != nullptr ? args.out_rows[grow] : grow;
        __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(args.out) + orow_i * args.ldo;
#pragma unroll
        for (int cc = 0; cc < kGsCols; cc += 32) {
          const int col = col0 + cc;
          if (col + 32 <= args.n_out) {
            uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              dst[q4] = make_uint4(pack_bf16x2(sum[cc + 8 * q4] * sc, sum[cc + 8 * q4 + 1] * sc),
                                   pack_bf16x2(sum[cc + 8 * q4 + 2] * sc, sum[cc + 8 * q4 + 3] * sc),
                                   pack_bf16x2(sum[cc + 8 * q4 + 4] * sc, sum[cc + 8 * q4 + 5] * sc),
                                   pack_bf16x2(sum[cc + 8 * q4 + 6] * sc, sum[cc + 8 * q4 + 7] * sc));
          } else if (col < args.n_out) {
#pragma unroll
            for (int jj = 0; jj < 32; ++jj)
              if (col + jj < args.n_out) orow[col + jj] = __float2bfloat16_rn(sum[cc + jj] * sc);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(kGsAcc * kGsBN)
                 : "memory");
  }
}

cudaError_t launch_gs(const TcGemmArgs& args, long long max_units, cudaStream_t stream) {
  auto kern = gemm_gs_kernel;
  static int configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    const cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, GsGeo::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured[dev] = 1;
  }
  long long units = device_sm_count();
  if (max_units < units) units = max_units;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(static_cast<unsigned>(units), 1, 1);
  cfg.blockDim = dim3(kGsThreads, 1, 1);
  cfg.dynamicSmemBytes = GsGeo::kSmemBytes;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args);
}

}  // namespace

cudaError_t launch_gemm_gs(const TcGemmArgs& args, int rows_upper, cudaStream_t stream) {
  if (args.groups < 1 || args.groups > kGsMaxGroups || args.wgs == nullptr || args.kdim % 128 ||
      args.kdim <= 0)
    return cudaErrorInvalidValue;
  const long long max_units =
      (static_cast<long long>(rows_upper) / kGsBM + args.groups) * args.n_tiles;
  if (max_units <= 0) return cudaSuccess;
  return launch_gs(args, max_units, stream);
}

}  // namespace moe
