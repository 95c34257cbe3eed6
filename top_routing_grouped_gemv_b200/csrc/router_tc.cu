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
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

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


// ---- fused router: logits on tcgen05, top-K in the epilogue (33..128 experts) ----
//
// One CTA pair (a cluster of two, tcgen05 cta_group::2) per 256-token tile:
// each CTA loads its 128 token rows and half of the weight rows, the leader
// issues M=256 MMAs over both CTAs' shared memory, and each CTA's
// accumulators hold its own 128 tokens -- half the weight bytes per CTA and
// stage of a single-CTA tile (the weights are read by every tile).  The
// plan holds w_r split into its three bf16 parts as 3*EP K-major rows
// [hi(EP) | mid(EP) | lo(EP)] (EP = E rounded up to 32, rows past E zero),
// made once (router_split3_kernel).  Per 64-element K stage each CTA loads
// its 128 token rows and its half of the weight rows by TMA (128-byte
// swizzle); the leader's MMA thread issues, per K=16 step, one M=256 MMA of
// N = 3*EP (EP = 64) or two, of N = 2*EP and N = EP (FrGeo), whose output
// columns are the parts' fp32 accumulators (TMEM columns [0,EP) hi,
// [EP,2EP) mid, [2EP,3EP) lo: bf16 x bf16 products are exact in fp32, each
// part keeps its own rounding scale).  Wide MMAs matter: with one N=EP MMA
// per part the MMAs alone took 37 us for a tile's 32 stages, three times
// their tensor-pipe time.  The four
// epilogue warps then own one token row each per lane (TMEM lane = token):
//   logit[e] = ((hi + mid) + lo) + bias[e]
// and the top-K (value descending, equal values to the lower expert) in
// three passes over the row:
//   1. the logits go to shared memory (the pipeline buffers, free once the
//      accumulators are final), and tau = min over KMAX+1 disjoint expert
//      groups (group (e mod 32) mod (KMAX+1)) of the group maximum: at
//      least KMAX+1 logits are >= tau, so every member of the top K+1 is;
//   2. a bit per expert marks the logits >= tau (usually a dozen or two);
//   3. the marked ones are inserted, in expert order, into a sorted K+1
//      list held in registers (an unrolled compare-and-shift; ties keep the
//      earlier, lower expert).
// This touches each logit with a few instructions instead of a full
// insertion, which matters because the four epilogue warps have the SM to
// themselves (one tile per CTA) and are bound by instruction issue.  An
// earlier pass 2 appended each candidate to a per-thread list in shared
// memory: its data-dependent store per logit cost ~7 us of the tile.
// Softmax over the kept K, margin = K-th minus (K+1)-th logit.

constexpr int kFrBM = 128;      // tokens per tile
constexpr int kFrKE = 64;       // K elements per stage (128 bytes of bf16)

template <int EP>
struct FrGeo {
  // The 3*EP weight rows [hi | mid | lo] go to the tensor core as one MMA
  // of N = 3*EP columns when that fits (N <= 256: EP = 64), else as one of
  // the first two parts (N = 2*EP) and one of the third (N = EP): few wide
  // MMAs, each reading the token tile once, instead of one narrow MMA per
  // part.  In a CTA pair each MMA's weight rows are split in halves, the
  // first half in the leader's shared memory and the second in the peer's;
  // a CTA's halves of the chunks sit back to back, as PARTS0 + (PARTS0 ==
  // 2) boxes of EP/2 rows.
  static constexpr int PARTS0 = 3 * EP <= 256 ? 3 : 2;  // parts in the first MMA
  static constexpr int A_BYTES = kFrBM * 128;
  static constexpr int B_BYTES = 3 * (EP / 2) * 128;  // this CTA's halves of the chunks
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = EP <= 64 ? 7 : EP <= 96 ? 6 : 5;
  static constexpr int kBarFull = 0, kBarEmpty = STAGES, kBarTFull = 2 * STAGES,
                       kNumBars = 2 * STAGES + 1;
  // ring | barriers | TMEM slot + abort flag (16 B) | bias (EP floats) |
  // the epilogue warp pairs' go-ahead flags (8 ints)
  static constexpr int kSmemBytes = 1024 + STAGES * STAGE_BYTES + kNumBars * 8 + 16 + EP * 4 + 32;
  // the epilogue's logits (EP floats per token), the exchanged group maxima
  // (2 * (KMAX + 1) floats per token) and half lists ((KMAX + 1) float2)
  static_assert(kFrBM * (EP + 4 * 9) * 4 <= STAGES * STAGE_BYTES, "the epilogue's data fit the ring");
};

// Inserts (v, e) into a descending list of L entries held in registers (L
// a compile-time size, every index a constant); v goes after entries equal
// to it, so with e ascending equal values keep the lower expert first.
template <int L>
__device__ __forceinline__ void fr_insert(float v, int e, float (&val)[L], int (&idx)[L]) {
#pragma unroll
  for (int j = L - 1; j > 0; --j) {
    const bool up = v > val[j - 1];
    const bool here = v > val[j];
    val[j] = up ? val[j - 1] : (here ? v : val[j]);
    idx[j] = up ? idx[j - 1] : (here ? e : idx[j]);
  }
  if (v > val[0]) {
    val[0] = v;
    idx[0] = e;
  }
}

// Threads: warp 0 TMA producer, warp 1 MMA issuer, warps 2..9 epilogue (two
// per TMEM lane quadrant, each selecting over half of the experts).
constexpr int kFrThreads = 320;

__device__ __forceinline__ void fr_pair_bar(int q) {
  // the two epilogue warps of lane quadrant q (named barrier 1 + q)
  asm volatile("bar.sync %0, %1;" ::"r"(1 + q), "r"(64) : "memory");
}

template <int EP, int KMAX>
__global__ void __launch_bounds__(kFrThreads, 1)
router_fused_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    const float* __restrict__ bias, int N, int d, int E, int K,
                    int32_t* __restrict__ ids, float* __restrict__ gates,
                    float* __restrict__ margin, int* status) {
  using namespace tc;
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  using Gm = FrGeo<EP>;
  constexpr int STAGES = Gm::STAGES;
  extern __shared__ uint8_t fr_smem_raw[];
  const uint32_t raw = smem_u32(fr_smem_raw);
  uint8_t* smem = fr_smem_raw + ((1024u - (raw & 1023u)) & 1023u);
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = sA + STAGES * Gm::A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * Gm::STAGE_BYTES);
  const uint32_t bar0 = smem_u32(bars);
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + Gm::kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_bias = reinterpret_cast<float*>(tmem_slot + 4);
  int* s_pair_ok = reinterpret_cast<int*>(s_bias + EP);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int row0 = pair * 2 * kFrBM + static_cast<int>(rank) * kFrBM;
  for (int e = threadIdx.x; e < EP; e += blockDim.x)
    s_bias[e] = (bias != nullptr && e < E) ? bias[e] : 0.f;
  const int num_kb = (d + kFrKE - 1) / kFrKE;
  // Every tile reads the same router weights; each pair starts its k loop
  // at a different stage (the same in both CTAs), so the weight tiles in
  // flight differ between pairs.  Only the order of the fp32 accumulation
  // over k changes, fixed per pair.
  const int kb0 = static_cast<int>(static_cast<unsigned>(pair) % static_cast<unsigned>(num_kb));

  if (threadIdx.x == 32) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(bar(Gm::kBarFull + s), 1);
      mbar_init(bar(Gm::kBarEmpty + s), 1);
    }
    mbar_init(bar(Gm::kBarTFull), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    __syncwarp();
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(512)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the leader's barriers exist before the peer's copies signal them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---- TMA producer ----
      int s = 0;
      uint32_t ph = 0, issued = 0, issued_ph = 0;
      bool aborted = false;
      auto kb_of = [&](int it) { return it + kb0 < num_kb ? it + kb0 : it + kb0 - num_kb; };
      for (int it = 0; it < num_kb; ++it) {
        if (!mbar_wait(bar(Gm::kBarEmpty + s), ph ^ 1u, abort_flag)) { aborted = true; break; }
        const int kb = kb_of(it);
        const int kx = kb * kFrKE;
        // both CTAs' copies complete on the leader's barrier
        const uint32_t full_leader = map_to_rank(bar(Gm::kBarFull + s), 0);
        if (leader) mbar_expect_tx(bar(Gm::kBarFull + s), 2 * Gm::STAGE_BYTES);
        tma_load_2d_pair(sA + s * Gm::A_BYTES, &tmX, kx, row0, full_leader);
#pragma unroll
        for (int b = 0; b < 3; ++b) {
          // box b: weight rows of the first MMA's half (b < PARTS0) or of
          // the second's
          const int wrow = b < Gm::PARTS0
                               ? static_cast<int>(rank) * (Gm::PARTS0 * EP / 2) + b * (EP / 2)
                               : Gm::PARTS0 * EP + static_cast<int>(rank) * (EP / 2);
          tma_load_2d_pair(sB + s * Gm::B_BYTES + b * (EP / 2) * 128, &tmW, kx, wrow, full_leader);
        }
        issued |= 1u << s;
        issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
        if (++s == STAGES) { s = 0; ph ^= 1u; }
      }
      if (aborted) {
        set_status(status, kStatusTimeout);
        // let copies already in flight land before the CTA pair's memory is reused
        if (leader)
          for (int i = 0; i < STAGES; ++i)
            if ((issued >> i) & 1u) mbar_wait_drain(bar(Gm::kBarFull + i), (issued_ph >> i) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---- MMA issuer (the pair's leader): each part into its own TMEM columns ----
      // bf16 x bf16 -> fp32, M = 256 (the pair), N = the chunk's rows
      constexpr uint32_t idesc_base = (1u << 4) | (1u << 7) | (1u << 10) |
                                      (static_cast<uint32_t>((2 * kFrBM) >> 4) << 24);
      constexpr uint32_t idesc0 = idesc_base | (static_cast<uint32_t>((Gm::PARTS0 * EP) >> 3) << 17);
      constexpr uint32_t idesc1 = idesc_base | (static_cast<uint32_t>(EP >> 3) << 17);
      int s = 0;
      uint32_t ph = 0;
      bool aborted = false;
      for (int it = 0; it < num_kb; ++it) {
        if (!mbar_wait(bar(Gm::kBarFull + s), ph, abort_flag)) { aborted = true; break; }
        tc_fence_after();
        const uint32_t a0 = sA + s * Gm::A_BYTES, b0 = sB + s * Gm::B_BYTES;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t acc = (it | k) != 0 ? 1u : 0u;
          tc_mma_pair<false>(tmem_base, sw128_desc(a0 + 32 * k), sw128_desc(b0 + 32 * k), idesc0,
                             acc);
          if constexpr (Gm::PARTS0 == 2)
            tc_mma_pair<false>(tmem_base + static_cast<uint32_t>(2 * EP), sw128_desc(a0 + 32 * k),
                               sw128_desc(b0 + 2 * (EP / 2) * 128 + 32 * k), idesc1, acc);
        }
        tc_commit_pair_both(bar(Gm::kBarEmpty + s));  // frees the stage in both CTAs
        if (++s == STAGES) { s = 0; ph ^= 1u; }
      }
      if (aborted) set_status(status, kStatusTimeout);
      // arrives (in both CTAs) once every MMA issued so far has finished;
      // the epilogues leave through the abort flag when the loop gave up
      tc_commit_pair_both(bar(Gm::kBarTFull));
      if (aborted) mbar_wait_drain(bar(Gm::kBarTFull), 0);
    }
    __syncwarp();
  } else {
    // ---- epilogue: one token per lane, two warps per token row ----
    const int q = warp & 3;            // TMEM lane quadrant of this warp
    const int h = (warp - 2) >> 2;     // its half of the experts
    const bool ok_self =
        __shfl_sync(0xffffffffu, mbar_wait(bar(Gm::kBarTFull), 0, abort_flag), 0);
    // the pair goes on only if both of its warps saw the accumulators final
    // (every barrier below is shared by the pair)
    if (lane == 0) s_pair_ok[2 * q + h] = ok_self ? 1 : 0;
    fr_pair_bar(q);
    const bool ok = ok_self && s_pair_ok[2 * q + (1 - h)] != 0;
    if (!ok) {
      if (!ok_self) set_status(status, kStatusTimeout);
    } else {
      tc_fence_after();
      const int r = q * 32 + lane;  // row of the tile
      const long long t = static_cast<long long>(row0) + r;
      const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      constexpr int G = KMAX + 1;   // disjoint expert groups for the threshold
      constexpr int HALF = EP / 2;  // experts per warp of the pair
      const int e0 = h * HALF;
      // Per 16-expert chunk (the chunks in a loop: fully unrolled over the
      // experts the epilogue is thousands of instructions executed once,
      // and fetching them cost more than running them).
      // pass 1: this half's logits, into the ring (logit e of row r at float
      // index e * 128 + r: a warp's 32 rows are 32 consecutive words), and
      // its group maxima (group = position in the chunk mod G)
      float* lg = reinterpret_cast<float*>(smem);
      float gmax[G];
#pragma unroll
      for (int g = 0; g < G; ++g) gmax[g] = -INFINITY;
#pragma unroll 1
      for (int cc = 0; cc < HALF; cc += 16) {
        uint32_t vh[16], vm[16], vl[16];
        __syncwarp();
        tmem_ld16(tq + e0 + cc, vh);
        tmem_ld16(tq + EP + e0 + cc, vm);
        tmem_ld16(tq + 2 * EP + e0 + cc, vl);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int e = e0 + cc + j;
          if (e < E) {
            const float v = ((__uint_as_float(vh[j]) + __uint_as_float(vm[j])) +
                             __uint_as_float(vl[j])) + s_bias[e];
            lg[e * kFrBM + r] = v;
            gmax[j % G] = fmaxf(gmax[j % G], v);  // a constant index
          }
        }
      }
      // the pair's group maxima -> tau: at least KMAX+1 logits (one per
      // group; experts 0..31 fill every position, so no group is empty) are
      // >= tau, so every member of the top K+1 is
      float* xg = lg + EP * kFrBM;
#pragma unroll
      for (int g = 0; g < G; ++g) xg[(h * G + g) * kFrBM + r] = gmax[g];
      fr_pair_bar(q);
      float tau = INFINITY;
#pragma unroll
      for (int g = 0; g < G; ++g)
        tau = fminf(tau, fmaxf(gmax[g], xg[((1 - h) * G + g) * kFrBM + r]));
      // passes 2 and 3, per chunk: a bit per expert whose logit is >= tau
      // (no branches, no data-dependent addresses), then those inserted in
      // expert order into a sorted top KMAX+1 of this half (K <= KMAX reads
      // the first K+1: the list keeps a superset of what it needs)
      float val[G];
      int idx[G];
#pragma unroll
      for (int j = 0; j < G; ++j) {
        val[j] = -INFINITY;
        idx[j] = 0x7fffffff;
      }
#pragma unroll 1
      for (int cc = 0; cc < HALF; cc += 16) {
        uint32_t m = 0u;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int e = e0 + cc + j;
          if (e < E) m |= static_cast<uint32_t>(lg[e * kFrBM + r] >= tau) << j;
        }
        while (m != 0u) {
          const int e = e0 + cc + __ffs(m) - 1;
          m &= m - 1u;
          fr_insert<G>(lg[e * kFrBM + r], e, val, idx);
        }
      }
      // merge: the upper half's list into the lower half's; its experts are
      // all higher, so inserting after equal values keeps ties on the lower
      // expert
      float2* xl = reinterpret_cast<float2*>(xg + 2 * G * kFrBM);
      if (h == 1) {
#pragma unroll
        for (int j = 0; j < G; ++j) xl[j * kFrBM + r] = make_float2(val[j], __int_as_float(idx[j]));
      }
      fr_pair_bar(q);
      if (h == 0) {
#pragma unroll
        for (int j = 0; j < G; ++j) {
          const float2 c = xl[j * kFrBM + r];
          fr_insert<G>(c.x, __float_as_int(c.y), val, idx);
        }
      }
      if (h == 0 && t < N) {
        // every index below is a constant within the list (j < KMAX < G), so
        // the list stays in registers
        float z = 0.f;
        float p[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          p[j] = 0.f;
          if (j < K) {
            p[j] = expf(val[j] - val[0]);
            z += p[j];
          }
        }
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
          if (j < K) {
            ids[t * K + j] = idx[j];
            gates[t * K + j] = p[j] / z;
          }
        if (margin != nullptr) {
          float kth = val[0], next = val[0];
#pragma unroll
          for (int j = 0; j < G; ++j) {
            kth = sel_f(j == K - 1, val[j], kth);
            next = sel_f(j == K, val[j], next);
          }
          margin[t] = (K == E) ? INFINITY : kth - next;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer is done with this CTA's shared memory and TMEM
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(512)
                 : "memory");
  }
}

// w_r (d, E) fp32 -> out (3 * EP, d) bf16 rows [hi | mid | lo], rows e >= E
// zero; through a 32 x 32 shared tile (reads along e, writes along k).
// Block (32, 8); grid (EP / 32, ceil(d / 32)).
__global__ void __launch_bounds__(256)
router_split3_kernel(const float* __restrict__ w_r, int d, int E, int EP,
                     __nv_bfloat16* __restrict__ out) {
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
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    out[static_cast<long long>(e) * d + k] = hi;
    out[static_cast<long long>(EP + e) * d + k] = mid;
    out[static_cast<long long>(2 * EP + e) * d + k] = lo;
  }
}

template <int EP, int KMAX>
cudaError_t launch_fused_t(const CUtensorMap& tmX, const CUtensorMap& tmW, const float* bias,
                           int N, int d, int E, int K, int32_t* ids, float* gates, float* margin,
                           int* status, cudaStream_t stream) {
  auto kern = router_fused_kernel<EP, KMAX>;
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         FrGeo<EP>::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  // a cluster of two CTAs per 256 tokens
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  cfg.gridDim = dim3(static_cast<unsigned>(2 * ((N + 2 * kFrBM - 1) / (2 * kFrBM))));
  cfg.blockDim = dim3(kFrThreads);
  cfg.dynamicSmemBytes = FrGeo<EP>::kSmemBytes;
  cfg.stream = stream;
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, tmX, tmW, bias, N, d, E, K, ids, gates, margin, status);
}

template <int EP>
cudaError_t launch_fused_k(const CUtensorMap& tmX, const CUtensorMap& tmW, const float* bias,
                           int N, int d, int E, int K, int32_t* ids, float* gates, float* margin,
                           int* status, cudaStream_t stream) {
  if (K <= 2)
    return launch_fused_t<EP, 2>(tmX, tmW, bias, N, d, E, K, ids, gates, margin, status, stream);
  if (K <= 4)
    return launch_fused_t<EP, 4>(tmX, tmW, bias, N, d, E, K, ids, gates, margin, status, stream);
  return launch_fused_t<EP, 8>(tmX, tmW, bias, N, d, E, K, ids, gates, margin, status, stream);
}

int fused_ep(int E) { return (E + 31) / 32 * 32; }
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

namespace moe {

bool router_uses_fused_tc(int N, int d, int E, int x_dtype) {
  return x_dtype == kBF16 && E >= kRouterTcMinExperts && E <= kRouterFusedMaxExperts &&
         !router_uses_splitk(N, d);
}

size_t router_fused_weight_bytes(int d, int E) {
  return static_cast<size_t>(3) * fused_ep(E) * d * sizeof(__nv_bfloat16);
}

cudaError_t launch_router_fused_split(const float* w_r, int d, int E, void* out,
                                      cudaStream_t stream) {
  const int EP = fused_ep(E);
  const dim3 grid(static_cast<unsigned>(EP / 32), static_cast<unsigned>((d + 31) / 32));
  router_split3_kernel<<<grid, dim3(32, 8), 0, stream>>>(w_r, d, E, EP,
                                                          static_cast<__nv_bfloat16*>(out));
  return cudaGetLastError();
}

bool encode_router_fused_weights(CUtensorMap* map, const void* split, int d, int E) {
  const int EP = fused_ep(E);
  return encode_kmajor_map(map, split, 2, 3LL * EP, d, EP / 2);  // a CTA's half of a part
}

cudaError_t launch_router_fused(const void* x, const CUtensorMap& tmW, const float* bias, int N,
                                int d, int E, int K, int32_t* ids, float* gates, float* margin,
                                int* status, cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  CUtensorMap tmX;
  if (!encode_kmajor_map(&tmX, x, 2, N, d, kFrBM)) return cudaErrorInvalidValue;
  switch (fused_ep(E)) {
    case 64:
      return launch_fused_k<64>(tmX, tmW, bias, N, d, E, K, ids, gates, margin, status, stream);
    case 96:
      return launch_fused_k<96>(tmX, tmW, bias, N, d, E, K, ids, gates, margin, status, stream);
    case 128:
      return launch_fused_k<128>(tmX, tmW, bias, N, d, E, K, ids, gates, margin, status, stream);
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace moe
