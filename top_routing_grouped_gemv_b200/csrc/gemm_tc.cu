// Grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// What it computes ("Advanced GPU Optimization ... Part 5", section 1.2
// step 2, local expert FFNs; aclnnQuantGroupedMatMulAlltoAllv formula:
// gmmY = (gmmX @ gmmWeight) * gmmXScale * gmmWeightScale, and the shared
// expert mmY = (mmX @ mmWeight) * ...): for every group g (expert), the rows
// [offsets[g], offsets[g+1]) of A times the transpose of the group's
// weight block W_g (n_out x kdim, K-major), fp32 accumulation, then either
//   kEpiStore : out = bf16(acc * scale)
//   kEpiSwiglu: out = bf16(silu(acc_gate) * acc_up)  (the weight tile holds
//               128 gate rows followed by 128 up rows of the same outputs)
//   kEpiRouter: out = fp32 router logits (hi + mid) + lo  (the weight tile
//               holds three bf16 parts of 64 experts' fp32 router weights
//               and 64 zero rows: columns [0,64) hi, [64,128) mid,
//               [128,192) lo; one group, rows = tokens)
//
// Structure (one persistent CTA per SM, 10 warps):
//   warp 0      TMA producer: 128-byte-swizzled K-major tiles of A (128 rows)
//               and W (256 rows) into a 4-stage shared-memory ring (6
//               stages of 128 + 128 rows per CTA in the CTA-pair mode)
//   warp 1      owns the 512 TMEM columns; lane 0 issues tcgen05.mma
//               (M=128, N=256, K=16 bf16 / K=32 e4m3 per instruction) into
//               one of two fp32 accumulators, and tcgen05.commit releases
//               ring slots and hands finished accumulators to the epilogue
//   warps 2..9  epilogue, two per TMEM lane quadrant, each taking half of
//               the tile's columns: tcgen05.ld of the accumulator rows of
//               their quadrant, activation/scale, bf16, 16-byte stores;
//               overlaps the next tile's MMAs (double-buffered TMEM)
// The tile list (group, row tile, column tile) is derived on the device
// from the offsets, so no host synchronisation is needed; empty groups own
// no tiles, and rows past a group's end are computed but never stored.
//
// Optional row scatter: result row r is stored at row out_rows[r] (the pure
// unpermute of the single-matrix layer done by the stores).
//
// MX variant (Ascend quant mode 6, read as OCP MXFP8: e4m3 operands, one
// E8M0 scale per 32 elements of K for every row of A and of W): each stage
// also brings the stage's scale atoms (512 bytes per 128 rows) by untiled
// bulk copies; the MMA thread copies them into TMEM (tcgen05.cp, four scale
// columns for A, eight for the 256 weight rows) ahead of the stage's four
// block-scaled MMAs (tcgen05.mma kind::mxf8f6f4.block_scale, scale byte k
// for the k-th MMA).  The scale columns take the place of the second
// accumulator, so the MX kernel has one accumulator and its epilogue does
// not overlap the next tile's MMAs.
//
// Gathered A (kGather, bf16 SwiGLU gate/up GEMM on single CTAs): instead of
// a 128-row box of the permuted rows, each stage's A tile is gathered from the
// token rows themselves (args.tmAg over x, a box one row high;
// args.a_rows[r] = the token of permuted row r) by TMA tile::gather4, four
// rows per instruction and only as many as the tile has rows of its expert;
// the tile's other rows keep stale data, are computed and never stored.  It
// lets small batches skip the permute's row copy: with a few rows per expert
// the A tile is a sliver of the stage next to the 256 weight rows.
//
// Every mbarrier wait is bounded (1 s): on expiry the CTA records
// MOE_ERR_DEVICE_TIMEOUT, the other roles leave their loops, in-flight
// copies and MMAs are drained (bounded) and TMEM is freed before exit.
#include <cuda.h>

#include "common.cuh"
#include "grouped_tiles.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace tc;

constexpr int BM = kTcBlockM;     // 128 rows per CTA (256 per CTA pair)
constexpr int BN = kTcBlockN;     // 256 accumulator columns per tile
constexpr int ROWB = 128;         // bytes of K per row per stage (one swizzle atom)
constexpr int A_BYTES = BM * ROWB;
// producer warp, MMA warp, eight epilogue warps: two per TMEM lane
// quadrant, each draining half of the tile's columns (with one warp per
// quadrant the epilogue's stores held back the next tiles' MMAs: the
// fine-grained workload's down GEMM ran 420 us with its stores, 320 us
// without).  The block-scaled epilogue, whose fp32 sums live in
// registers, splits the columns the same way (sixteen warps ran 1.6 ->
// 2.6 ms on the full fp8 workload).
constexpr int kEpiWarps = 8;
constexpr int kBsEpiWarps = kEpiWarps;
template <int kEpi>
constexpr int threads_of() {
  return 32 * (2 + kEpiWarps);
}
constexpr uint32_t kTmemCols = 2 * BN;
constexpr int kMaxGroups = 256;

// Per-mode geometry.  Single CTA: B tile 256 rows, 4 stages of 48 KB.  CTA
// pair (tcgen05 cta_group::2): each CTA holds its 128 A rows and half of the
// 256 B rows, 6 stages of 32 KB.
template <bool kPair, bool kMx = false>
struct Geo {
  static constexpr int B_ROWS = kPair ? BN / 2 : BN;
  static constexpr int B_BYTES = B_ROWS * ROWB;
  static constexpr int SF_BYTES = kMx ? 3 * kMxAtomBytes : 0;  // A atom + two B atoms
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SF_BYTES;
  static constexpr int STAGES = kPair ? 6 : 4;
  static constexpr int TILE_M = kPair ? 2 * BM : BM;
  static constexpr int kBarFull = 0, kBarEmpty = STAGES, kBarTFull = 2 * STAGES,
                       kBarTEmpty = 2 * STAGES + 2, kBarDrain = 2 * STAGES + 4,
                       kNumBars = 2 * STAGES + 5;
  // ring | barriers | TMEM slot + abort flag | tile prefix and group offsets |
  // the epilogue warps' 2 KB staging buffers for their stores (1024-byte
  // aligned: a buffer is also a TMA store's 64-byte-swizzled source)
  static constexpr int kSmemBytes = 1024 /*alignment slack*/ + STAGES * STAGE_BYTES +
                                    kNumBars * 8 + 16 + 2 * (kMaxGroups + 1) * 4 + 1024 +
                                    kEpiWarps * 2048;
};

__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.f + __expf(-g)) * u; }

// Stores a warp's chunk of 32 rows x 32 bf16 columns (lane l holds row l's
// 16 packed words; dst: this lane's row at the chunk's first column, or
// nullptr when the row is not stored) through the warp's 2 KB of shared
// memory: lane l writes its row's four 16-byte units (unit u to slot
// u ^ ((l >> 1) & 3): conflict-free), then each store instruction writes
// 64 contiguous bytes into each of 8 rows -- whole 32-byte sectors, where a
// store straight from the row-per-lane registers writes 16 bytes into each
// of 32 rows 4 KB apart.
__device__ __forceinline__ void store_chunk_rows(uint8_t* stage, int lane, const uint32_t (&pk)[16],
                                                 __nv_bfloat16* dst) {
  uint4* srow = reinterpret_cast<uint4*>(stage + lane * 64);
  const int f = (lane >> 1) & 3;
  if (lane == 0) tc::bulk_wait_read0();  // a TMA store of the buffer has read it
  __syncwarp();  // the previous chunk's reads are done
#pragma unroll
  for (int u = 0; u < 4; ++u)
    srow[u ^ f] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
  __syncwarp();
  const int U = lane & 3;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int R = 8 * i + (lane >> 2);
    const uint4 v = reinterpret_cast<const uint4*>(stage + R * 64)[U ^ ((R >> 1) & 3)];
    const unsigned long long p =
        __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(dst), R);
    if (p != 0ull) reinterpret_cast<uint4*>(p)[U] = v;
  }
}

// The same chunk when all 32 rows are stored and are consecutive rows of
// out: written to the buffer in the layout of a 32 x 32 box with 64-byte
// swizzle (16-byte unit u of row r at unit u ^ ((r >> 1) & 3), the layout
// above), then stored by one TMA instruction; the warp goes on without
// waiting for the store.
__device__ __forceinline__ void store_chunk_tma(uint8_t* stage, int lane, const uint32_t (&pk)[16],
                                                const CUtensorMap* map, int col, int row) {
  uint4* srow = reinterpret_cast<uint4*>(stage + lane * 64);
  const int f = (lane >> 1) & 3;
  if (lane == 0) tc::bulk_wait_read0();  // the previous store has read the buffer
  __syncwarp();
#pragma unroll
  for (int u = 0; u < 4; ++u)
    srow[u ^ f] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
  tc::fence_proxy_async_smem();  // this lane's writes, visible to the TMA engine
  __syncwarp();
  if (lane == 0) {
    tc::tma_store_2d(map, tc::smem_u32(stage), col, row);
    tc::bulk_commit();
  }
}

template <bool kFp8, bool kPair>
constexpr uint32_t make_idesc_mode() {
  return (1u << 4) | ((kFp8 ? 0u : 1u) << 7) | ((kFp8 ? 0u : 1u) << 10) |
         (static_cast<uint32_t>(BN >> 3) << 17) |
         (static_cast<uint32_t>((kPair ? 2 * BM : BM) >> 4) << 24);
}

// Block-scaled (MX) instruction descriptor: e4m3 A and B (format 0), E8M0
// scales (bit 23), N >> 3 at [17,23), M >> 4 at [24,29); the scale byte of
// B goes to [4,6) and of A to [29,31) per MMA (mx_sf_ids).
constexpr uint32_t make_idesc_mx() {
  return (1u << 23) | (static_cast<uint32_t>(BN >> 3) << 17) | (static_cast<uint32_t>(BM >> 4) << 24);
}
__device__ __forceinline__ uint32_t mx_sf_ids(uint32_t k) { return (k << 29) | (k << 4); }

// kPair: a cluster of 2 CTAs computes 256-row tiles with tcgen05 cta_group::2;
// CTA rank r holds rows [128r, 128r+128) of the tile and B rows [128r, 128r+128)
// of the 256-row weight tile; the leader (rank 0) issues the MMAs.
template <bool kFp8, int kEpi, bool kPair, bool kMx, bool kGather = false>
__global__ void __launch_bounds__(threads_of<kEpi>(), 1) gemm_tc_kernel(const __grid_constant__ TcGemmArgs args) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  static_assert(!kMx || (kFp8 && !kPair && kEpi == kEpiStore), "MX: e4m3, single CTA, store");
  static_assert(!kGather || (!kFp8 && !kPair && !kMx && kEpi == kEpiSwiglu),
                "gathered A: bf16 SwiGLU, single CTA");
  // per-column group scales run in gemm_gs.cu; block scales here
  constexpr bool kGs = kEpi == kEpiBlockScale;
  static_assert(kEpi != kEpiGroupScale, "per-column group scales: gemm_gs_kernel");
  static_assert(!kGs || (kFp8 && !kPair && !kMx), "block scales: e4m3, single CTA");
  using Gm = Geo<kPair, kMx>;
  constexpr int STAGES = Gm::STAGES;
  constexpr int kAcc = kMx ? 1 : 2;  // accumulators in TMEM
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + STAGES * A_BYTES;
  const uint32_t sSF = sB + STAGES * Gm::B_BYTES;  // MX scale atoms (kMx only)
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * Gm::STAGE_BYTES);
  const uint32_t bar0 = smem_u32(bars);
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Gm::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_pref = reinterpret_cast<int*>(tmem_slot + 4);
  int* s_off = s_pref + (kMaxGroups + 1);
  uint8_t* s_ostage = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(s_off + kMaxGroups + 1) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = args.groups;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int nunits = kPair ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  // Per-group tile counts -> exclusive prefix (warp 0), group row offsets.
  if (warp == 0)
    build_tile_prefix<Gm::TILE_M>(args.offsets, G, args.m_total, args.n_tiles, lane, s_pref, s_off);
  if (threadIdx.x == 32) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar(Gm::kBarFull + s), 1);
      mbar_init(bar(Gm::kBarEmpty + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar(Gm::kBarTFull + a), 1);
      mbar_init(bar(Gm::kBarTEmpty + a), kPair ? 2 * kEpiWarps : kEpiWarps);
    }
    mbar_init(bar(Gm::kBarDrain), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    if constexpr (kGather) tma_prefetch_desc(&args.tmAg);
    else tma_prefetch_desc(&args.tmA);
    tma_prefetch_desc(&args.tmB0);
    if (kEpi == kEpiSwiglu) tma_prefetch_desc(&args.tmB1);
  }
  if (warp == 1) {
    __syncwarp();  // tcgen05.alloc is .sync.aligned: converge after thread 32's branch
    if constexpr (kPair) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(kTmemCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                       smem_u32(tmem_slot)),
                   "r"(kTmemCols)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync();  // the leader's barriers exist before the peer signals them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_pref[G];
  constexpr int kElems = kFp8 ? 128 : 64;  // K elements per stage
  const int num_kb = (args.kdim + kElems - 1) / kElems;

  if (warp == 0) {
    // ---------------- TMA producer (every CTA fills its own ring) ----------------
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool aborted = false;
      uint32_t issued = 0, issued_ph = 0;  // per-stage bits: loaded at least once / its parity
      const CUtensorMap* mapB = (kEpi == kEpiSwiglu && kPair && rank == 1) ? &args.tmB1 : &args.tmB0;
      for (int T = unit; T < total && !aborted; T += nunits) {
        const TileCoord c = decode_tile<Gm::TILE_M>(T, s_pref, s_off, G, args.n_tiles);
        const int arow = c.m_row0 + static_cast<int>(rank) * BM;
        // gathered A: the tile's rows of its expert and, for a tile of at most
        // 16 rows, their token indices once for all its stages
        int g_rows = 0, g_idx[16];
        if constexpr (kGather) {
          g_rows = min(BM, s_off[c.g + 1] - c.m_row0);
          if (g_rows <= 16) {
#pragma unroll
            for (int u = 0; u < 16; ++u) g_idx[u] = args.a_rows[c.m_row0 + min(u, g_rows - 1)];
          }
        }
        int brow;
        if constexpr (kEpi == kEpiSwiglu)
          brow = c.g * args.n_out + c.n_tile * (BN / 2);  // gate (and up) rows of 128 outputs
        else
          brow = c.g * args.n_out + c.n_tile * BN + static_cast<int>(rank) * Gm::B_ROWS;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(bar(Gm::kBarEmpty + s), ph ^ 1u, abort_flag)) { aborted = true; break; }
          const int kx = kb * kElems;
          if constexpr (kPair) {
            const uint32_t full_leader = map_to_rank(bar(Gm::kBarFull + s), 0);
            if (leader) mbar_expect_tx(bar(Gm::kBarFull + s), 2 * Gm::STAGE_BYTES);
            tma_load_2d_pair(sA + s * A_BYTES, &args.tmA, kx, arow, full_leader);
            tma_load_2d_pair(sB + s * Gm::B_BYTES, mapB, kx, brow, full_leader);
          } else {
            if constexpr (kGather) {
              // the tile's rows of its expert, four per gather (the last
              // group padded with the last row)
              const int rows = g_rows;
              const int ng4 = (rows + 3) >> 2;
              mbar_expect_tx(bar(Gm::kBarFull + s), ng4 * 512 + Gm::B_BYTES);
              if (rows <= 16) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  if (q < ng4)
                    tma_gather4(sA + s * A_BYTES + 512 * q, &args.tmAg, kx, g_idx[4 * q],
                                g_idx[4 * q + 1], g_idx[4 * q + 2], g_idx[4 * q + 3],
                                bar(Gm::kBarFull + s));
              } else {
                const int32_t* src = args.a_rows + c.m_row0;
                for (int q = 0; q < ng4; ++q) {
                  const int i = 4 * q;
                  tma_gather4(sA + s * A_BYTES + 512 * q, &args.tmAg, kx, src[i],
                              src[min(i + 1, rows - 1)], src[min(i + 2, rows - 1)],
                              src[min(i + 3, rows - 1)], bar(Gm::kBarFull + s));
                }
              }
            } else {
              mbar_expect_tx(bar(Gm::kBarFull + s), Gm::STAGE_BYTES);
              tma_load_2d(sA + s * A_BYTES, &args.tmA, kx, arow, bar(Gm::kBarFull + s));
            }
            if (kEpi == kEpiSwiglu) {
              tma_load_2d(sB + s * Gm::B_BYTES, &args.tmB0, kx, brow, bar(Gm::kBarFull + s));
              tma_load_2d(sB + s * Gm::B_BYTES + (BN / 2) * ROWB, &args.tmB1, kx, brow,
                          bar(Gm::kBarFull + s));
            } else {
              tma_load_2d(sB + s * Gm::B_BYTES, &args.tmB0, kx, brow, bar(Gm::kBarFull + s));
            }
            if constexpr (kMx) {
              const uint32_t sf = sSF + s * Gm::SF_BYTES;
              bulk_load(sf, args.sfa + (static_cast<size_t>(c.m_tile) * num_kb + kb) * kMxAtomBytes,
                        kMxAtomBytes, bar(Gm::kBarFull + s));
              bulk_load(sf + kMxAtomBytes,
                        args.sfb + ((static_cast<size_t>(c.g) * args.n_tiles + c.n_tile) * num_kb + kb) *
                                       (2 * kMxAtomBytes),
                        2 * kMxAtomBytes, bar(Gm::kBarFull + s));
            }
          }
          issued |= 1u << s;
          issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      if (aborted) {
        set_status(args.status, kStatusTimeout);
        // let copies already in flight land before the CTA's memory is reused
        if (leader)
          for (int i = 0; i < STAGES; ++i)
            if ((issued >> i) & 1u) mbar_wait_drain(bar(Gm::kBarFull + i), (issued_ph >> i) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (the pair leader issues for both CTAs) ----------------
    if (kGs && lane == 0) {
      // every K stage into a fresh accumulator (the two alternate); the
      // epilogue adds it to its fp32 sums with the stage's scales
      constexpr uint32_t idesc = make_idesc_mode<true, false>();
      int s = 0;
      uint32_t ph = 0, j = 0;
      bool aborted = false;
      for (int T = unit; T < total && !aborted; T += nunits) {
        for (int kb = 0; kb < num_kb; ++kb, ++j) {
          const uint32_t acc = j & 1u, aph = (j >> 1) & 1u;
          if (!mbar_wait(bar(Gm::kBarTEmpty + acc), aph ^ 1u, abort_flag)) { aborted = true; break; }
          if (!mbar_wait(bar(Gm::kBarFull + s), ph, abort_flag)) { aborted = true; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + acc * static_cast<uint32_t>(BN);
          const uint32_t a0 = sA + s * A_BYTES, b0 = sB + s * Gm::B_BYTES;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc_mma<true>(d_tmem, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), idesc,
                         k != 0 ? 1u : 0u);
          tc_commit(bar(Gm::kBarEmpty + s));
          tc_commit(bar(Gm::kBarTFull + acc));
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      if (aborted) {
        set_status(args.status, kStatusTimeout);
        tc_commit(bar(Gm::kBarDrain));
        mbar_wait_drain(bar(Gm::kBarDrain), 0);
      }
    } else if (!kGs && lane == 0 && leader) {
      constexpr uint32_t idesc = kMx ? make_idesc_mx() : make_idesc_mode<kFp8, kPair>();
      // MX scale columns (after the single accumulator): A at BN, B at BN + 4
      const uint32_t sfa_t = tmem_base + static_cast<uint32_t>(BN);
      const uint32_t sfb_t = sfa_t + 4u;
      int s = 0;
      uint32_t ph = 0;
      bool aborted = false;
      int i = 0;
      for (int T = unit; T < total; T += nunits, ++i) {
        const int acc = i % kAcc;
        const uint32_t aph = (i / kAcc) & 1;
        if (!mbar_wait(bar(Gm::kBarTEmpty + acc), aph ^ 1u, abort_flag)) { aborted = true; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(bar(Gm::kBarFull + s), ph, abort_flag)) { aborted = true; break; }
          tc_fence_after();
          const uint32_t a0 = sA + s * A_BYTES, b0 = sB + s * Gm::B_BYTES;
          if constexpr (kMx) {
            // the stage's scales into TMEM; tcgen05 operations of this thread
            // run in issue order, so the MMAs below read them, and the next
            // stage's copies wait for those MMAs
            const uint32_t sf = sSF + s * Gm::SF_BYTES;
            tc_cp_32x128b_x4(sfa_t, rows16_desc(sf));
            tc_cp_32x128b_x4(sfb_t, rows16_desc(sf + kMxAtomBytes));
            tc_cp_32x128b_x4(sfb_t + 4u, rows16_desc(sf + 2 * kMxAtomBytes));
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t accum = (kb | k) != 0 ? 1u : 0u;
            if constexpr (kMx)
              tc_mma_mx(d_tmem, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k),
                        idesc | mx_sf_ids(k), sfa_t | (static_cast<uint32_t>(k) << 30),
                        sfb_t | (static_cast<uint32_t>(k) << 30), accum);
            else if constexpr (kPair)
              tc_mma_pair<kFp8>(d_tmem, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), idesc, accum);
            else
              tc_mma<kFp8>(d_tmem, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), idesc, accum);
          }
          if constexpr (kPair) tc_commit_pair_both(bar(Gm::kBarEmpty + s));
          else tc_commit(bar(Gm::kBarEmpty + s));
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
        if (aborted) break;
        if constexpr (kPair) tc_commit_pair_both(bar(Gm::kBarTFull + acc));
        else tc_commit(bar(Gm::kBarTFull + acc));
      }
      if (aborted) {
        set_status(args.status, kStatusTimeout);
        // arrives once every MMA issued so far has finished
        if constexpr (kPair) tc_commit_pair_self(bar(Gm::kBarDrain));
        else tc_commit(bar(Gm::kBarDrain));
        mbar_wait_drain(bar(Gm::kBarDrain), 0);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2..9, two per TMEM lane quadrant) ----------------
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    int i = 0;
    if constexpr (kGs) {
      constexpr int kCols = BN / (kBsEpiWarps / 4);  // columns of this warp
      const int half = (warp - 2) >> 2;               // its column slice
      const int nblk = (args.n_out + 127) / 128;
      uint32_t j = 0;
      for (int T = unit; T < total; T += nunits) {
        const TileCoord c = decode_tile<Gm::TILE_M>(T, s_pref, s_off, G, args.n_tiles);
        const int row = q * 32 + lane;
        const long long grow = static_cast<long long>(c.m_row0) + row;
        const bool valid = grow < s_off[c.g + 1] && grow < args.m_total && grow >= 0;
        const long long srow = valid && args.row_index != nullptr ? args.row_index[grow] : grow;
        const int col0 = c.n_tile * BN + half * kCols;
        const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                            static_cast<uint32_t>(half * kCols);
        float sum[kCols];
#pragma unroll
        for (int cc = 0; cc < kCols; ++cc) sum[cc] = 0.f;
        // the stage's row scale and block scale are loaded one stage ahead,
        // so their latency is not on the path from TFull to TEmpty
        const float* xrow = valid && args.xgs != nullptr ? args.xgs + srow * num_kb : nullptr;
        const float* wblk = args.wgs + static_cast<long long>(c.g) * num_kb * nblk + col0 / 128;
        float sx_next = xrow ? xrow[0] : 1.f;
        float wb_next = wblk[0];
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb, ++j) {
          const uint32_t a = j & 1u, aph = (j >> 1) & 1u;
          const float sx = sx_next, wb = wb_next;
          if (kb + 1 < num_kb) {
            if (xrow) sx_next = xrow[kb + 1];
            wb_next = wblk[static_cast<long long>(kb + 1) * nblk];
          }
          ok = __shfl_sync(0xffffffffu, mbar_wait(bar(Gm::kBarTFull + a), aph, abort_flag), 0);
          if (!ok) break;
          tc_fence_after();
          {
            // one 128 x 128 weight block covers this warp's columns
            const float f = sx * wb;
#pragma unroll
            for (int cc = 0; cc < kCols; cc += 16) {
              uint32_t v[16];
              __syncwarp();
              tmem_ld16(tq + a * BN + cc, v);
              tmem_ld_wait();
#pragma unroll
              for (int jj = 0; jj < 16; jj += 2)
                fma_f32x2(sum[cc + jj], sum[cc + jj + 1], __uint_as_float(v[jj]),
                          __uint_as_float(v[jj + 1]), f, f);
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(Gm::kBarTEmpty + a));
        }
        if (!ok) {
          set_status(args.status, kStatusTimeout);
          break;
        }
        if (valid) {
          float sc = args.scale;
          if (args.row_scale != nullptr)
            sc *= args.row_scale[args.row_index != nullptr ? args.row_index[grow] : grow];
          const long long orow_i = args.out_rows != nullptr ? args.out_rows[grow] : grow;
          __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(args.out) + orow_i * args.ldo;
#pragma unroll
          for (int cc = 0; cc < kCols; cc += 32) {
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
    for (int T = unit; !kGs && T < total; T += nunits, ++i) {
      const int acc = i % kAcc;
      const uint32_t aph = (i / kAcc) & 1;
      // every lane polls; lane 0's answer is taken by all (and converges the warp
      // before the .sync.aligned TMEM loads)
      const bool ok = __shfl_sync(0xffffffffu, mbar_wait(bar(Gm::kBarTFull + acc), aph, abort_flag), 0);
      if (!ok) {
        set_status(args.status, kStatusTimeout);
        break;
      }
      tc_fence_after();
      const TileCoord c = decode_tile<Gm::TILE_M>(T, s_pref, s_off, G, args.n_tiles);
      // lane quadrant q holds rows 32q.. of this CTA's 128 rows of the tile
      const int row = static_cast<int>(rank) * BM + q * 32 + lane;
      // output columns of the tile, and this warp's half of them
      constexpr int span = kEpi == kEpiSwiglu ? BN / 2 : kEpi == kEpiRouter ? BN / 4 : BN;
      constexpr int hspan = span / 2;
      const int hh = (warp - 2) >> 2;
      const int col0 = c.n_tile * span + hh * hspan;
      const long long grow = static_cast<long long>(c.m_row0) + row;
      const bool valid = grow < s_off[c.g + 1] && grow < args.m_total && grow >= 0;
      // TMEM columns of the accumulator (and of its gate / up or hi / mid /
      // lo parts) from this warp's first column
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * BN + hh * hspan);
      long long orow_i = grow;
      if (valid && args.out_rows != nullptr) orow_i = args.out_rows[grow];
      // staged stores where the warp stores most of its 32 rows; a warp of a
      // short tile (an expert's last rows, decode-shaped batches) stores
      // its few rows directly
      const unsigned vmask = __ballot_sync(0xffffffffu, valid);
      const bool staged = __popc(vmask) > 16;
      // all 32 rows stored, consecutive in out: TMA tile stores
      const bool tma_rows = args.out_tma != 0 && vmask == 0xffffffffu;
      const int warp_row0 = static_cast<int>(c.m_row0) + static_cast<int>(rank) * BM + q * 32;
      __nv_bfloat16* orow = static_cast<__nv_bfloat16*>(args.out) + orow_i * args.ldo;
      if constexpr (kEpi == kEpiRouter) {
        float* frow = static_cast<float*>(args.out) + orow_i * args.ldo;
        const bool vec4 = (args.ldo & 3) == 0;
#pragma unroll 1
        for (int cc = 0; cc < hspan; cc += 32) {
          uint32_t vh[32], vm[32], vl[32];
          __syncwarp();
          tmem_ld32(tbase + cc, vh);             // hi part
          tmem_ld32(tbase + span + cc, vm);      // mid part
          tmem_ld32(tbase + 2 * span + cc, vl);  // lo part
          tmem_ld_wait();
          const int col = col0 + cc;
          if (valid && col < args.n_out) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
              v[j] = (__uint_as_float(vh[j]) + __uint_as_float(vm[j])) + __uint_as_float(vl[j]);
            if (vec4 && col + 32 <= args.n_out) {
              float4* dst = reinterpret_cast<float4*>(frow + col);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                dst[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col + j < args.n_out) frow[col + j] = v[j];
            }
          }
        }
      } else if (kEpi == kEpiSwiglu) {
#pragma unroll 1
        for (int cc = 0; cc < hspan; cc += 32) {
          uint32_t gr[32], ur[32];
          __syncwarp();
          tmem_ld32(tbase + cc, gr);          // gate columns
          tmem_ld32(tbase + span + cc, ur);   // up columns of the same outputs
          tmem_ld_wait();
          const int col = col0 + cc;
          const bool whole = col + 32 <= args.n_out;  // the same for the whole warp
          if (whole && (staged || valid)) {
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              pk[j] = pack_bf16x2(silu_mul(__uint_as_float(gr[2 * j]), __uint_as_float(ur[2 * j])),
                                  silu_mul(__uint_as_float(gr[2 * j + 1]),
                                           __uint_as_float(ur[2 * j + 1])));
            if (staged) {
              if (tma_rows)
                store_chunk_tma(s_ostage + (warp - 2) * 2048, lane, pk, &args.tmOut, col, warp_row0);
              else
                store_chunk_rows(s_ostage + (warp - 2) * 2048, lane, pk, valid ? orow + col : nullptr);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            }
          } else if (!whole && valid && col < args.n_out) {
            {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col + j < args.n_out)
                  orow[col + j] = __float2bfloat16_rn(
                      silu_mul(__uint_as_float(gr[j]), __uint_as_float(ur[j])));
            }
          }
        }
      } else {
        float rsc = args.scale;
        if (valid && args.row_scale != nullptr)
          rsc *= args.row_scale[args.row_index != nullptr ? args.row_index[grow] : grow];
#pragma unroll 1
        for (int cc = 0; cc < hspan; cc += 32) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld32(tbase + cc, v);
          tmem_ld_wait();
          const int col = col0 + cc;
          const float sc = rsc;
          const bool whole = col + 32 <= args.n_out;  // the same for the whole warp
          if (whole && (staged || valid)) {
            if (args.col_scale != nullptr) {
              // per output channel: fold the channel scale into the values
              const float* cs = args.col_scale + static_cast<long long>(c.g) * args.n_out + col;
#pragma unroll
              for (int j = 0; j < 32; ++j) v[j] = __float_as_uint(__uint_as_float(v[j]) * cs[j]);
            }
            uint32_t pk[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              pk[j] = pack_bf16x2(__uint_as_float(v[2 * j]) * sc, __uint_as_float(v[2 * j + 1]) * sc);
            if (staged) {
              if (tma_rows)
                store_chunk_tma(s_ostage + (warp - 2) * 2048, lane, pk, &args.tmOut, col, warp_row0);
              else
                store_chunk_rows(s_ostage + (warp - 2) * 2048, lane, pk, valid ? orow + col : nullptr);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(orow + col);
#pragma unroll
              for (int j = 0; j < 4; ++j)
                dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            }
          } else if (!whole && valid && col < args.n_out) {
            if (args.col_scale != nullptr) {
              const float* cs = args.col_scale + static_cast<long long>(c.g) * args.n_out + col;
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col + j < args.n_out) v[j] = __float_as_uint(__uint_as_float(v[j]) * cs[j]);
            }
            {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col + j < args.n_out) orow[col + j] = __float2bfloat16_rn(__uint_as_float(v[j]) * sc);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if constexpr (kPair) mbar_arrive_cluster(map_to_rank(bar(Gm::kBarTEmpty + acc), 0));
        else mbar_arrive(bar(Gm::kBarTEmpty + acc));
      }
    }
    if (lane == 0) bulk_wait0();  // the warp's TMA tile stores have completed
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (kPair) cluster_sync();  // the peer is done with this CTA's memory and TMEM
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (kPair)
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(kTmemCols)
                   : "memory");
    else
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"(kTmemCols)
                   : "memory");
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

template <bool kFp8, int kEpi, bool kPair, bool kMx = false, bool kGather = false>
cudaError_t launch_t(const TcGemmArgs& args, long long max_units, cudaStream_t stream) {
  using Gm = Geo<kPair, kMx>;
  auto kern = gemm_tc_kernel<kFp8, kEpi, kPair, kMx, kGather>;
  static int configured[64] = {0};
  static int max_clusters[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.blockDim = dim3(threads_of<kEpi>(), 1, 1);
  cfg.dynamicSmemBytes = Gm::kSmemBytes;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if constexpr (kPair) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Gm::kSmemBytes);
    if (e != cudaSuccess) return e;
    if constexpr (kPair) {
      int n = 0;
      cfg.gridDim = dim3(2 * (device_sm_count() / 2), 1, 1);
      e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
      if (e != cudaSuccess) return e;
      max_clusters[dev] = n > 0 ? n : 1;
    }
    configured[dev] = 1;
  }
  long long units = kPair ? max_clusters[dev] : device_sm_count();
  if (max_units < units) units = max_units;
  cfg.gridDim = dim3(static_cast<unsigned>((kPair ? 2 : 1) * units), 1, 1);
  return cudaLaunchKernelEx(&cfg, kern, args);
}

}  // namespace

bool encode_out_map(CUtensorMap* map, void* base, long long rows, long long cols, long long ld) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows <= 0 || cols <= 0 || (ld * 2) % 16 != 0) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  cuuint32_t box[2] = {32, 32};  // 64 bytes x 32 rows: one warp's chunk
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_kmajor_map(CUtensorMap* map, const void* base, int elem_bytes, long long rows,
                       long long kdim, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rows <= 0 || kdim <= 0) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kdim), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kdim * elem_bytes)};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(ROWB / elem_bytes), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUtensorMapDataType dt =
      elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8;
  CUresult r = fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t launch_gemm_tc(const TcGemmArgs& args, int dtype, int epilogue, int rows_upper,
                           bool pair, cudaStream_t stream) {
  if (args.groups < 1 || args.groups > kMaxGroups) return cudaErrorInvalidValue;
  const int tile_m = pair ? 2 * BM : BM;
  const long long max_units =
      (static_cast<long long>(rows_upper) / tile_m + args.groups) * args.n_tiles;
  if (max_units <= 0) return cudaSuccess;
  if (dtype == kGemmMxE4M3) {
    if (pair || epilogue != kEpiStore || !args.sfa || !args.sfb) return cudaErrorInvalidValue;
    return launch_t<true, kEpiStore, false, true>(args, max_units, stream);
  }
  if (epilogue == kEpiGroupScale) return cudaErrorInvalidValue;  // launch_gemm_gs
  if (epilogue == kEpiBlockScale) {
    if (pair || dtype != kE4M3 || !args.wgs || args.kdim % 128) return cudaErrorInvalidValue;
    return launch_t<true, kEpiBlockScale, false>(args, max_units, stream);
  }
  const bool fp8 = dtype == kE4M3;
  const bool sw = epilogue == kEpiSwiglu;
  if (args.a_rows != nullptr) {
    if (pair || fp8 || !sw) return cudaErrorInvalidValue;
    return launch_t<false, kEpiSwiglu, false, false, true>(args, max_units, stream);
  }
  if (epilogue == kEpiRouter) {
    if (pair || fp8) return cudaErrorInvalidValue;
    return launch_t<false, kEpiRouter, false>(args, max_units, stream);
  }
  if (pair) {
    if (fp8) return sw ? launch_t<true, kEpiSwiglu, true>(args, max_units, stream)
                       : launch_t<true, kEpiStore, true>(args, max_units, stream);
    return sw ? launch_t<false, kEpiSwiglu, true>(args, max_units, stream)
              : launch_t<false, kEpiStore, true>(args, max_units, stream);
  }
  if (fp8) return sw ? launch_t<true, kEpiSwiglu, false>(args, max_units, stream)
                     : launch_t<true, kEpiStore, false>(args, max_units, stream);
  return sw ? launch_t<false, kEpiSwiglu, false>(args, max_units, stream)
            : launch_t<false, kEpiStore, false>(args, max_units, stream);
}

int device_sm_count() {
  static int count[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (count[dev] == 0) {
    int c = 0;
    cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev);
    count[dev] = c > 0 ? c : 148;
  }
  return count[dev];
}

}  // namespace moe
