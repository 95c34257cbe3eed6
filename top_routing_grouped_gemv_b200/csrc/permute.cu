// Permute / dispatch: expert histogram, prefix scan and a stable gather of
// token rows into expert-contiguous order ("Advanced GPU Optimization ...
// Part 5", section 1.2 step 1, token dispatch: a buffer per destination built
// from the routing decisions, here local; aclnnQuantGroupedMatMulAlltoAllv
// constraints: sendCounts per expert; determinism by default).
//
// Stable order: within expert e the rows appear in (token, slot) order, so
//   pos[t,j] = offsets[e] + #{(t',j') before (t,j) with ids[t',j'] = e}.
// Tokens are cut into chunks of kPermuteChunk (32) and blocks of
// kPermuteBlock (256 = eight chunks).  Two launches:
//   1. rank:   one CTA of eight warps per block, one warp per chunk: each
//              lane (token) sets its bit in a per-expert 32-bit mask of its
//              warp, and the rank of (t, j) within the chunk is the number of
//              lower lanes in the mask of its expert (a token whose K experts
//              are not distinct takes a shuffle-based count instead); the
//              chunks' histograms are scanned over the block's eight chunks,
//              so each pair's rank within its block goes to perm_pos and the
//              block's expert histogram to block_counts.  The last CTA to
//              finish (an atomic counter, reset for the next call) scans the
//              block histograms into per-(block, expert) bases (offsets[e] +
//              rows of e in earlier blocks), counts and offsets.  Either way
//              the order is fixed.
//   2. gather: one warp per token turns its ranks into final positions
//              (checked against N*K) and copies the token row once from HBM
//              into its K destination rows with 16-byte vector loads/stores
//              (and, on request, notes each position's flat slot t*K + j for
//              an unpermute done by the grouped GEMM's stores).
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int CH = kPermuteChunk;
constexpr int BT = kPermuteBlock;
constexpr int kRankWarps = BT / CH;  // chunks (warps) per block
static_assert(kRankWarps * 32 == 256, "one rank CTA = 256 threads");

// Exclusive scan of the block histograms bc (nblk, E) over blocks, per
// expert, by the 256 threads of one CTA; afterwards bc[b][e] holds the first
// destination row of block b's rows of expert e, and counts / offsets the
// expert totals and their exclusive scan (offsets[E] = the rows).  Thread
// (e, s) owns expert e and a contiguous slice s of the blocks; part and
// total are 256 and 257 ints of shared memory.  bc is read through L2 (it
// was written by other CTAs).
__device__ __forceinline__ void scan_block_counts(int32_t* __restrict__ bc, int nblk, int E,
                                                  int32_t* __restrict__ counts,
                                                  int32_t* __restrict__ offsets, int* part,
                                                  int* total) {
  int Ep = 1;
  while (Ep < E) Ep <<= 1;
  const int S = 256 / Ep;  // slices per expert (>= 1 for E <= 256)
  const int e = threadIdx.x % Ep, sl = threadIdx.x / Ep;
  const int cs = (nblk + S - 1) / S;
  const int c0 = sl * cs, c1 = min(nblk, c0 + cs);
  int sum = 0;
  if (e < E) {
    int c = c0;
    for (; c + 8 <= c1; c += 8) {  // eight loads in flight
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldcg(bc + (long long)(c + u) * E + e);
#pragma unroll
      for (int u = 0; u < 8; ++u) sum += v[u];
    }
    for (; c < c1; ++c) sum += __ldcg(bc + (long long)c * E + e);
  }
  part[threadIdx.x] = sum;
  __syncthreads();
  if (threadIdx.x < E) {  // over the slices of each expert
    int run = 0;
    for (int q = 0; q < S; ++q) {
      const int v = part[q * Ep + threadIdx.x];
      part[q * Ep + threadIdx.x] = run;
      run += v;
    }
    total[threadIdx.x] = run;
  }
  __syncthreads();
  if (threadIdx.x < 32) {  // over the experts (E <= 256: up to 8 per lane)
    const int lane = threadIdx.x;
    const int per = (E + 31) / 32;
    const int b0 = min(E, lane * per), b1 = min(E, b0 + per);
    int local = 0;
    for (int q = b0; q < b1; ++q) local += total[q];
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    int run = incl - local;
    for (int q = b0; q < b1; ++q) {
      const int c = total[q];
      counts[q] = c;
      offsets[q] = run;
      total[q] = run;
      run += c;
    }
    if (lane == 31) offsets[E] = incl;
  }
  __syncthreads();
  if (e < E) {
    int run = total[e] + part[sl * Ep + e];
    int c = c0;
    for (; c + 8 <= c1; c += 8) {  // eight loads in flight, then the eight bases
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = __ldcg(bc + (long long)(c + u) * E + e);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        bc[(long long)(c + u) * E + e] = run;
        run += v[u];
      }
    }
    for (; c < c1; ++c) {
      int32_t* q = bc + (long long)c * E + e;
      const int v = __ldcg(q);
      *q = run;
      run += v;
    }
  }
}

// One CTA per block of 256 tokens, one warp per 32-token chunk (lane =
// token); the last CTA also runs the scan.  At most 40 registers a thread:
// a CTA (8 warps, 10 K registers, 18 KB of shared memory) then fits on an SM
// beside one CTA of a persistent tensor-core GEMM (the shared expert running
// on a forked stream) instead of waiting for that GEMM to end.
//
// With src non-null (small batches) the last CTA also turns every rank into
// its final position (pos = block base + rank, src[pos] = t), so that a
// permute that copies no rows needs no second launch.
template <int KMAX>
__global__ void __maxnreg__(40)
permute_rank_kernel(const int32_t* __restrict__ ids, int N, int K, int E,
                    int32_t* __restrict__ block_counts, unsigned* __restrict__ counter,
                    int32_t* __restrict__ local_rank, int32_t* __restrict__ counts,
                    int32_t* __restrict__ offsets, int32_t* __restrict__ src, int* status) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  __shared__ int hist[kRankWarps][256];
  __shared__ unsigned lanes_of[kRankWarps][256];  // bit l: lane (token) l routes to the expert
  __shared__ int s_part[256];
  __shared__ int s_total[257];
  __shared__ int s_last;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int e = lane; e < E; e += 32) {
    hist[warp][e] = 0;
    lanes_of[warp][e] = 0u;
  }
  __syncwarp();
  const long long t = (static_cast<long long>(blockIdx.x) * kRankWarps + warp) * CH + lane;
  int my[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    my[j] = -1;
    if (j < K && t < N) {
      const int e = ids[t * K + j];
      if (e >= 0 && e < E) my[j] = e;
      else set_status(status, kStatusBadIndex);
    }
  }
  // rank of (t, j) in its chunk: earlier slots of t with the same expert ...
  int rank[KMAX];
  bool repeated = false;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    rank[j] = 0;
#pragma unroll
    for (int jj = 0; jj < KMAX; ++jj)
      if (jj < j && my[jj] == my[j] && my[j] >= 0) {
        rank[j]++;
        repeated = true;
      }
  }
  // ... plus every slot of the earlier tokens of this chunk with that expert
  if (!__any_sync(0xffffffffu, repeated)) {
    // K distinct experts per token: one bit per (token, expert)
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (my[j] >= 0) atomicOr(&lanes_of[warp][my[j]], 1u << lane);
    __syncwarp();
    const unsigned below = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (my[j] >= 0) rank[j] = __popc(lanes_of[warp][my[j]] & below);
  } else {
#pragma unroll
    for (int jj = 0; jj < KMAX; ++jj) {
      if (jj >= K) break;
      for (int sl = 0; sl < 31; ++sl) {
        const int v = __shfl_sync(0xffffffffu, my[jj], sl);
        if (sl < lane) {
#pragma unroll
          for (int j = 0; j < KMAX; ++j)
            if (v == my[j] && v >= 0) rank[j]++;
        }
      }
    }
  }
#pragma unroll
  for (int j = 0; j < KMAX; ++j)
    if (j < K && my[j] >= 0) atomicAdd(&hist[warp][my[j]], 1);  // integer counts: order-independent
  __syncthreads();
  // the chunks' histograms -> exclusive prefix over the block's chunks
  for (int e = threadIdx.x; e < E; e += 256) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kRankWarps; ++w) {
      const int v = hist[w][e];
      hist[w][e] = run;
      run += v;
    }
    block_counts[static_cast<long long>(blockIdx.x) * E + e] = run;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j >= K) break;
    if (t < N) local_rank[t * K + j] = my[j] >= 0 ? hist[warp][my[j]] + rank[j] : -1;
  }
  // the last CTA to get here scans every block's histogram
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(counter, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  scan_block_counts(block_counts, static_cast<int>(gridDim.x), E, counts, offsets, s_part, s_total);
  if (threadIdx.x == 0) *counter = 0u;  // ready for the next call (stream-ordered)
  if (src != nullptr) {
    __syncthreads();  // the block bases are in block_counts
    const long long R = static_cast<long long>(N) * K;
    for (long long i = threadIdx.x; i < R; i += blockDim.x) {
      const long long tt = i / K;
      const int e = __ldcg(ids + i);
      const int r = __ldcg(local_rank + i);  // written by every CTA
      int mine = -1;
      if (r >= 0 && e >= 0 && e < E) {
        mine = __ldcg(block_counts + (tt / BT) * E + e) + r;
        if (mine < 0 || mine >= R) {  // only a damaged workspace gets here
          set_status(status, kStatusBadIndex);
          mine = -1;
        } else {
          src[mine] = static_cast<int32_t>(tt);
        }
      }
      local_rank[i] = mine;
    }
  }
}

// WPT warps per token (8 / WPT tokens per CTA): final positions from the
// chunk bases and the ranks (the token's first warp, shared through shared
// memory), then one read of the token row and K writes, the row's 16-byte
// vectors split over the token's warps.  WPT > 1 spreads a small batch over
// more SMs.
template <int KMAX, int WPT>
__global__ void __launch_bounds__(256)
permute_gather_kernel(const uint4* __restrict__ x, int row_vecs, const int32_t* __restrict__ ids,
                      int N, int K, int E, const int32_t* __restrict__ chunk_base,
                      int32_t* __restrict__ pos, int32_t* __restrict__ src,
                      int32_t* __restrict__ slot, uint4* __restrict__ x_perm, int* status) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  __shared__ int sp[8 / WPT][KMAX];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tl = warp / WPT, sub = warp % WPT;
  const int t = blockIdx.x * (8 / WPT) + tl;
  if (t < N && sub == 0 && lane < KMAX) {
    int mine = -1;
    if (lane < K) {
      const long long i = (long long)t * K + lane;
      const int e = ids[i];
      const int r = pos[i];  // rank within the block (written by the rank pass)
      if (r >= 0 && e >= 0 && e < E) {
        mine = chunk_base[(long long)(t / BT) * E + e] + r;
        if (mine < 0 || mine >= N * K) {  // only a damaged workspace gets here
          set_status(status, kStatusBadIndex);
          mine = -1;
        } else {
          src[mine] = t;
          if (slot) slot[mine] = static_cast<int32_t>(i);
        }
      }
      pos[i] = mine;
    }
    sp[tl][lane] = mine;
  }
  if constexpr (WPT > 1) __syncthreads();
  else __syncwarp();
  if (t >= N || x_perm == nullptr) return;  // no x_perm: positions only
  int p[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) p[j] = sp[tl][j];
  const uint4* srow = x + (long long)t * row_vecs;
  constexpr int STEP = 32 * WPT;
  int v = sub * 32 + lane;
  // eight 16-byte loads in flight per lane where the row allows, then four
  for (; v + 7 * STEP < row_vecs; v += 8 * STEP) {
    uint4 a[8];
#pragma unroll
    for (int b = 0; b < 8; ++b) a[b] = srow[v + b * STEP];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j >= K || p[j] < 0) continue;
      uint4* drow = x_perm + (long long)p[j] * row_vecs;
#pragma unroll
      for (int b = 0; b < 8; ++b) drow[v + b * STEP] = a[b];
    }
  }
  for (; v + 3 * STEP < row_vecs; v += 4 * STEP) {
    const uint4 a0 = srow[v], a1 = srow[v + STEP], a2 = srow[v + 2 * STEP], a3 = srow[v + 3 * STEP];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j >= K || p[j] < 0) continue;
      uint4* drow = x_perm + (long long)p[j] * row_vecs;
      drow[v] = a0; drow[v + STEP] = a1; drow[v + 2 * STEP] = a2; drow[v + 3 * STEP] = a3;
    }
  }
  for (; v < row_vecs; v += STEP) {
    const uint4 a0 = srow[v];
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < K && p[j] >= 0) x_perm[(long long)p[j] * row_vecs + v] = a0;
  }
}

// Per-token dynamic quantization fused into the gather (Ascend quant mode 7,
// per-token dynamic): a bf16 token row gets the scale amax(|row|) / 448 (1
// for an all-zero row) and e4m3 codes of x / scale (fp32 division, round to
// nearest even, saturated to 448), written once per destination row; the
// scale goes to token_scale[t].  WPT warps per token as in the gather; a lane
// handles 16 elements (32 bytes in, 16 bytes out) at a time.
template <int KMAX, int WPT>
__global__ void __launch_bounds__(256)
permute_quant_kernel(const uint4* __restrict__ x, int d, const int32_t* __restrict__ ids, int N,
                     int K, int E, const int32_t* __restrict__ chunk_base,
                     int32_t* __restrict__ pos, int32_t* __restrict__ src,
                     int32_t* __restrict__ slot, uint4* __restrict__ x_perm,
                     float* __restrict__ token_scale, int* status) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  __shared__ int sp[8 / WPT][KMAX];
  __shared__ float wmax[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tl = warp / WPT, sub = warp % WPT;
  const int t = blockIdx.x * (8 / WPT) + tl;
  const bool active = t < N;
  if (active && sub == 0 && lane < KMAX) {
    int mine = -1;
    if (lane < K) {
      const long long i = (long long)t * K + lane;
      const int e = ids[i];
      const int r = pos[i];  // rank within the block (written by the rank pass)
      if (r >= 0 && e >= 0 && e < E) {
        mine = chunk_base[(long long)(t / BT) * E + e] + r;
        if (mine < 0 || mine >= N * K) {  // only a damaged workspace gets here
          set_status(status, kStatusBadIndex);
          mine = -1;
        } else {
          src[mine] = t;
          if (slot) slot[mine] = static_cast<int32_t>(i);
        }
      }
      pos[i] = mine;
    }
    sp[tl][lane] = mine;
  }
  const int units = d / 16;               // 16 elements per unit
  const uint4* srow = x + (long long)(active ? t : 0) * (d / 8);
  constexpr int STEP = 32 * WPT;
  float am = 0.f;
  if (active)
    for (int u = sub * 32 + lane; u < units; u += STEP) {
      const uint4 a = srow[2 * u], b = srow[2 * u + 1];
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
        am = fmaxf(am, fmaxf(fabsf(bf16lo(w[i])), fabsf(bf16hi(w[i]))));
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  if (lane == 0) wmax[warp] = am;
  if constexpr (WPT > 1) __syncthreads();
  else __syncwarp();
  if (!active) return;
  am = 0.f;
#pragma unroll
  for (int q = 0; q < WPT; ++q) am = fmaxf(am, wmax[tl * WPT + q]);
  const float scale = am > 0.f ? am / 448.f : 1.f;
  if (sub == 0 && lane == 0) token_scale[t] = scale;
  int p[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) p[j] = sp[tl][j];
  for (int u = sub * 32 + lane; u < units; u += STEP) {
    const uint4 a = srow[2 * u], b = srow[2 * u + 1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    uint32_t packed[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t c0 = __nv_cvt_float_to_fp8(bf16lo(w[2 * i]) / scale, __NV_SATFINITE, __NV_E4M3);
      const uint32_t c1 = __nv_cvt_float_to_fp8(bf16hi(w[2 * i]) / scale, __NV_SATFINITE, __NV_E4M3);
      const uint32_t c2 = __nv_cvt_float_to_fp8(bf16lo(w[2 * i + 1]) / scale, __NV_SATFINITE, __NV_E4M3);
      const uint32_t c3 = __nv_cvt_float_to_fp8(bf16hi(w[2 * i + 1]) / scale, __NV_SATFINITE, __NV_E4M3);
      packed[i] = c0 | (c1 << 8) | (c2 << 16) | (c3 << 24);
    }
    const uint4 out = make_uint4(packed[0], packed[1], packed[2], packed[3]);
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < K && p[j] >= 0) x_perm[(long long)p[j] * units + u] = out;
  }
}

template <int KMAX>
void launch_quant_k(const uint4* xv, int d, const int32_t* ids, int N, int K, int E,
                    const int32_t* chunk_base, int32_t* pos, int32_t* src, int32_t* slot, uint4* xp,
                    float* scales, int* status, cudaStream_t stream) {
  const int wpt = warps_per_token(N);
  const dim3 grid((N + 8 / wpt - 1) / (8 / wpt));
  if (wpt == 1)
    launch_pdl(permute_quant_kernel<KMAX, 1>, grid, dim3(256), 0, stream, xv, d, ids, N, K, E, chunk_base, pos, src, slot, xp, scales, status);
  else if (wpt == 2)
    launch_pdl(permute_quant_kernel<KMAX, 2>, grid, dim3(256), 0, stream, xv, d, ids, N, K, E, chunk_base, pos, src, slot, xp, scales, status);
  else if (wpt == 4)
    launch_pdl(permute_quant_kernel<KMAX, 4>, grid, dim3(256), 0, stream, xv, d, ids, N, K, E, chunk_base, pos, src, slot, xp, scales, status);
  else
    launch_pdl(permute_quant_kernel<KMAX, 8>, grid, dim3(256), 0, stream, xv, d, ids, N, K, E, chunk_base, pos, src, slot, xp, scales, status);
}

template <int KMAX>
void launch_gather_k(const uint4* xv, int row_vecs, const int32_t* ids, int N, int K, int E,
                     const int32_t* chunk_base, int32_t* pos, int32_t* src, int32_t* slot,
                     uint4* xp, int* status, cudaStream_t stream) {
  const int wpt = warps_per_token(N);
  const int tpc = 8 / wpt;
  const dim3 grid((N + tpc - 1) / tpc);
  if (wpt == 1)
    launch_pdl(permute_gather_kernel<KMAX, 1>, grid, dim3(256), 0, stream, xv, row_vecs, ids, N, K, E, chunk_base, pos, src, slot, xp, status);
  else if (wpt == 2)
    launch_pdl(permute_gather_kernel<KMAX, 2>, grid, dim3(256), 0, stream, xv, row_vecs, ids, N, K, E, chunk_base, pos, src, slot, xp, status);
  else if (wpt == 4)
    launch_pdl(permute_gather_kernel<KMAX, 4>, grid, dim3(256), 0, stream, xv, row_vecs, ids, N, K, E, chunk_base, pos, src, slot, xp, status);
  else
    launch_pdl(permute_gather_kernel<KMAX, 8>, grid, dim3(256), 0, stream, xv, row_vecs, ids, N, K, E, chunk_base, pos, src, slot, xp, status);
}

}  // namespace

cudaError_t launch_permute_rank(const int32_t* ids, int N, int K, int E, int32_t* block_counts,
                                unsigned* counter, int32_t* local_rank, int32_t* counts,
                                int32_t* offsets, int* status, cudaStream_t stream,
                                int32_t* src) {
  if (src != nullptr && static_cast<long long>(N) * K > kRankPositionsMaxRows)
    return cudaErrorInvalidValue;
  // at least one CTA, so that counts and offsets are written for zero tokens
  const int grid = permute_blocks(N) > 0 ? permute_blocks(N) : 1;
  if (K <= 2)
    return launch_pdl(permute_rank_kernel<2>, dim3(grid), dim3(256), 0, stream, ids, N, K, E,
                      block_counts, counter, local_rank, counts, offsets, src, status);
  if (K <= 4)
    return launch_pdl(permute_rank_kernel<4>, dim3(grid), dim3(256), 0, stream, ids, N, K, E,
                      block_counts, counter, local_rank, counts, offsets, src, status);
  return launch_pdl(permute_rank_kernel<8>, dim3(grid), dim3(256), 0, stream, ids, N, K, E,
                    block_counts, counter, local_rank, counts, offsets, src, status);
}

cudaError_t launch_permute_gather(const void* x, int row_bytes, const int32_t* ids, int N, int K,
                                  int E, const int32_t* chunk_base, int32_t* pos, int32_t* src,
                                  int32_t* slot, void* x_perm, int* status, cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  const int row_vecs = row_bytes / 16;
  auto xv = static_cast<const uint4*>(x);
  auto xp = static_cast<uint4*>(x_perm);
  if (K <= 2)
    launch_gather_k<2>(xv, row_vecs, ids, N, K, E, chunk_base, pos, src, slot, xp, status, stream);
  else if (K <= 4)
    launch_gather_k<4>(xv, row_vecs, ids, N, K, E, chunk_base, pos, src, slot, xp, status, stream);
  else
    launch_gather_k<8>(xv, row_vecs, ids, N, K, E, chunk_base, pos, src, slot, xp, status, stream);
  return cudaGetLastError();
}

cudaError_t launch_permute_quant(const void* x_bf16, int d, const int32_t* ids, int N, int K,
                                 int E, const int32_t* chunk_base, int32_t* pos, int32_t* src,
                                 int32_t* slot, void* x_perm_e4m3, float* token_scale, int* status,
                                 cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  if (d % 16) return cudaErrorInvalidValue;
  auto xv = static_cast<const uint4*>(x_bf16);
  auto xp = static_cast<uint4*>(x_perm_e4m3);
  if (K <= 2)
    launch_quant_k<2>(xv, d, ids, N, K, E, chunk_base, pos, src, slot, xp, token_scale, status, stream);
  else if (K <= 4)
    launch_quant_k<4>(xv, d, ids, N, K, E, chunk_base, pos, src, slot, xp, token_scale, status, stream);
  else
    launch_quant_k<8>(xv, d, ids, N, K, E, chunk_base, pos, src, slot, xp, token_scale, status, stream);
  return cudaGetLastError();
}

}  // namespace moe
