// Router: per-token expert logits in fp32, top-K with lower-index tie break,
// softmax over the kept K ("Advanced GPU Optimization ... Part 5", section
// 1.1 The Router Kernel: scores from the router weights, the best experts
// tracked by a manual reduction, softmax only over the kept scores; zyxy.net
// MoE page, expert selection: gating (N, E) -> top-K index matrix (N, K)).
//
// Layout of the work: a CTA of 8 warps owns 8*TPW tokens.  The reduction
// dimension d is staged through shared memory in chunks of kKC: the token
// chunk transposed to [k][token] (fp32) and the router-weight rows
// W_r[k][0..E) (fp32).  Lane l of a warp accumulates the logits of experts
// l, l+32, ... (EPL of them) for the warp's TPW tokens, in registers, adding
// k in ascending order with fp32 FMA.  The top-K is then chosen per token by
// K rounds of a warp-wide (value desc, index asc) argmax over shuffles, so
// every lane holds the kept logits and the softmax needs no shared memory.
#include <float.h>
#include <limits.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kKC = 32;       // k rows per shared-memory chunk
constexpr int kWarps = 8;

// One round of the warp-wide argmax over the still-available logits of a
// token (lane l holds experts l, l+32, ...): the larger value wins, equal
// values go to the lower expert index.  Every lane returns the winner.
template <int EPL>
__device__ __forceinline__ void warp_argmax(const float (&v)[EPL], const bool (&avail)[EPL],
                                            int lane, float& bv, int& be) {
  bv = -FLT_MAX;
  be = INT_MAX;
#pragma unroll
  for (int q = 0; q < EPL; ++q) {
    const int e = lane + 32 * q;
    if (avail[q] && (be == INT_MAX || v[q] > bv || (v[q] == bv && e < be))) {
      bv = v[q];
      be = e;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
    const int oe = __shfl_xor_sync(0xffffffffu, be, off);
    if (oe != INT_MAX && (be == INT_MAX || ov > bv || (ov == bv && oe < be))) {
      bv = ov;
      be = oe;
    }
  }
}

template <typename TX, int EPL, int TPW>
__global__ void __launch_bounds__(kWarps * 32)
router_kernel(const TX* __restrict__ x, const float* __restrict__ w_r,
              const float* __restrict__ bias, int N, int d, int E, int K,
              int32_t* __restrict__ ids, float* __restrict__ gates, float* __restrict__ margin) {
  constexpr int TM = kWarps * TPW;  // tokens per CTA
  constexpr int EP = EPL * 32;      // padded experts
  __shared__ float xs[kKC][TM + 1];  // +1: conflict-free transposed stores
  __shared__ __align__(16) float ws[kKC][EP];

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tok0 = blockIdx.x * TM;

  float acc[TPW][EPL];
#pragma unroll
  for (int i = 0; i < TPW; ++i)
#pragma unroll
    for (int q = 0; q < EPL; ++q) acc[i][q] = 0.f;

  for (int k0 = 0; k0 < d; k0 += kKC) {
    // stage x[tok0 .. tok0+TM)[k0 .. k0+kKC) transposed, zero outside
    for (int idx = threadIdx.x; idx < TM * kKC; idx += kWarps * 32) {
      int t = idx / kKC, kk = idx % kKC;
      int gt = tok0 + t, gk = k0 + kk;
      xs[kk][t] = (gt < N && gk < d) ? to_f32(x[(long long)gt * d + gk]) : 0.f;
    }
    for (int idx = threadIdx.x; idx < kKC * EP; idx += kWarps * 32) {
      int kk = idx / EP, e = idx % EP;
      int gk = k0 + kk;
      ws[kk][e] = (gk < d && e < E) ? w_r[(long long)gk * E + e] : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < kKC; ++kk) {
      float wv[EPL];
#pragma unroll
      for (int q = 0; q < EPL; ++q) wv[q] = ws[kk][lane + 32 * q];
#pragma unroll
      for (int i = 0; i < TPW; ++i) {
        float xv = xs[kk][warp * TPW + i];
#pragma unroll
        for (int q = 0; q < EPL; ++q) acc[i][q] = fmaf(xv, wv[q], acc[i][q]);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < TPW; ++i) {
    const int t = tok0 + warp * TPW + i;
    if (t >= N) break;  // warp-uniform
    float v[EPL];
    bool avail[EPL];
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
      int e = lane + 32 * q;
      avail[q] = e < E;
      v[q] = acc[i][q] + ((bias != nullptr && e < E) ? bias[e] : 0.f);
    }
    float sel_v[8];
    int sel_e[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j >= K) break;  // warp-uniform
      warp_argmax<EPL>(v, avail, lane, sel_v[j], sel_e[j]);
#pragma unroll
      for (int q = 0; q < EPL; ++q)
        if (lane + 32 * q == sel_e[j]) avail[q] = false;
    }
    float next_v = 0.f;
    if (K < E) {
      int next_e;
      warp_argmax<EPL>(v, avail, lane, next_v, next_e);
    }
    // softmax over the kept logits, largest first (sel_v[0] is the max)
    float z = 0.f, my_g = 0.f;
    int my_e = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < K) {
        float p = expf(sel_v[j] - sel_v[0]);
        z += p;
        if (j == lane) { my_g = p; my_e = sel_e[j]; }
      }
    }
    if (lane < K) {
      ids[(long long)t * K + lane] = my_e;
      gates[(long long)t * K + lane] = my_g / z;
    }
    if (margin != nullptr && lane == 0) {
      float kth = sel_v[0];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j == K - 1) kth = sel_v[j];
      margin[t] = (K == E) ? __int_as_float(0x7f800000) : kth - next_v;
    }
  }
}

// Small d*E (d*E <= 256 threads * 64 weights): every thread keeps the
// router weights of its k-slice [tid*KPT, tid*KPT+KPT) for all experts in
// registers, so the weights are read from memory once per CTA.  A CTA takes
// TB = 32/ET tokens at a time: each thread forms its partial logits for
// them (k ascending inside the slice), a warp reduce-scatter (31 shuffles)
// leaves lane l with the warp's sum of value l = (token l/ET, expert l%ET),
// and the eight warp sums are added in warp order.  Warp j then picks the
// top-K of token j.
template <int V>
__device__ __forceinline__ float warp_reduce_scatter(float (&v)[V], int lane) {
  static_assert(V == 32, "one value per lane after the reduction");
#pragma unroll
  for (int o = 16, n = 32; o >= 1; o >>= 1, n >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float send = upper ? v[i] : v[i + n / 2];
      const float keep = upper ? v[i + n / 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  return v[0];
}

template <typename TX, int ET, int KPT>
__global__ void __launch_bounds__(256)
router_regw_kernel(const TX* __restrict__ x, const float* __restrict__ w_r,
                   const float* __restrict__ bias, int N, int d, int E, int K,
                   int32_t* __restrict__ ids, float* __restrict__ gates, float* __restrict__ margin) {
  constexpr int TB = 32 / ET;  // tokens per pass
  __shared__ float red[8][32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k0 = tid * KPT;
  float w[KPT][ET];
#pragma unroll
  for (int i = 0; i < KPT; ++i)
#pragma unroll
    for (int e = 0; e < ET; ++e)
      w[i][e] = (k0 + i < d && e < E) ? w_r[(long long)(k0 + i) * E + e] : 0.f;

  for (int t0 = blockIdx.x * TB; t0 < N; t0 += gridDim.x * TB) {
    float part[32];
#pragma unroll
    for (int j = 0; j < TB; ++j) {
      float xv[KPT];
      const int t = t0 + j;
#pragma unroll
      for (int i = 0; i < KPT; ++i)
        xv[i] = (t < N && k0 + i < d) ? to_f32(x[(long long)t * d + k0 + i]) : 0.f;
#pragma unroll
      for (int e = 0; e < ET; ++e) {
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < KPT; ++i) a = fmaf(xv[i], w[i][e], a);
        part[j * ET + e] = a;
      }
    }
    red[warp][lane] = warp_reduce_scatter<32>(part, lane);
    __syncthreads();
    if (warp < TB) {
      const int t = t0 + warp;
      float v[1];
      bool avail[1];
      v[0] = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) v[0] += red[q][warp * ET + (lane % ET)];
      avail[0] = lane < E;
      if (avail[0] && bias != nullptr) v[0] += bias[lane];
      if (t < N) {
        float sel_v[8];
        int sel_e[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j >= K) break;
          warp_argmax<1>(v, avail, lane, sel_v[j], sel_e[j]);
          if (lane == sel_e[j]) avail[0] = false;
        }
        float next_v = 0.f;
        if (K < E) {
          int next_e;
          warp_argmax<1>(v, avail, lane, next_v, next_e);
        }
        float z = 0.f, my_g = 0.f;
        int my_e = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (j < K) {
            const float p = expf(sel_v[j] - sel_v[0]);
            z += p;
            if (j == lane) { my_g = p; my_e = sel_e[j]; }
          }
        }
        if (lane < K) {
          ids[(long long)t * K + lane] = my_e;
          gates[(long long)t * K + lane] = my_g / z;
        }
        if (margin != nullptr && lane == 0) {
          float kth = sel_v[0];
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (j == K - 1) kth = sel_v[j];
          margin[t] = (K == E) ? __int_as_float(0x7f800000) : kth - next_v;
        }
      }
    }
    __syncthreads();
  }
}

template <typename TX, int ET, int KPT>
void launch_regw_kpt(const TX* x, const float* w_r, const float* bias, int N, int d, int E, int K,
                     int32_t* ids, float* gates, float* margin, int grid, cudaStream_t stream) {
  router_regw_kernel<TX, ET, KPT><<<grid, 256, 0, stream>>>(x, w_r, bias, N, d, E, K, ids, gates,
                                                            margin);
}

// Picks the k-slice per thread (KPT = 1, 2, 4, 8: d <= 256*KPT) with at most
// 64 weights per thread; false if d*E is too large for this kernel.
template <typename TX, int ET>
bool launch_regw(const TX* x, const float* w_r, const float* bias, int N, int d, int E, int K,
                 int32_t* ids, float* gates, float* margin, cudaStream_t stream) {
  constexpr int TB = 32 / ET;
  const int grid = min((N + TB - 1) / TB, 2 * device_sm_count());
  if (d <= 256) {
    launch_regw_kpt<TX, ET, 1>(x, w_r, bias, N, d, E, K, ids, gates, margin, grid, stream);
    return true;
  }
  if constexpr (2 * ET <= 64) {
    if (d <= 512) {
      launch_regw_kpt<TX, ET, 2>(x, w_r, bias, N, d, E, K, ids, gates, margin, grid, stream);
      return true;
    }
  }
  if constexpr (4 * ET <= 64) {
    if (d <= 1024) {
      launch_regw_kpt<TX, ET, 4>(x, w_r, bias, N, d, E, K, ids, gates, margin, grid, stream);
      return true;
    }
  }
  if constexpr (8 * ET <= 64) {
    if (d <= 2048) {
      launch_regw_kpt<TX, ET, 8>(x, w_r, bias, N, d, E, K, ids, gates, margin, grid, stream);
      return true;
    }
  }
  return false;
}

template <typename TX, int EPL>
cudaError_t launch_epl(const TX* x, const float* w_r, const float* bias, int N, int d, int E,
                       int K, int32_t* ids, float* gates, float* margin, cudaStream_t stream) {
  // Many tokens: 8 per warp reuse each staged weight row 8 times.  Few
  // tokens: 2 per warp spread the CTAs over more SMs.
  int sms = device_sm_count();
  if ((long long)N >= 64LL * 2 * sms) {
    int grid = (N + 63) / 64;
    router_kernel<TX, EPL, 8><<<grid, kWarps * 32, 0, stream>>>(x, w_r, bias, N, d, E, K, ids,
                                                                 gates, margin);
  } else {
    int grid = (N + 15) / 16;
    router_kernel<TX, EPL, 2><<<grid, kWarps * 32, 0, stream>>>(x, w_r, bias, N, d, E, K, ids,
                                                                 gates, margin);
  }
  return cudaGetLastError();
}

template <typename TX>
cudaError_t launch_t(const TX* x, const float* w_r, const float* bias, int N, int d, int E, int K,
                     int32_t* ids, float* gates, float* margin, cudaStream_t stream) {
  if (E <= 8 && launch_regw<TX, 8>(x, w_r, bias, N, d, E, K, ids, gates, margin, stream))
    return cudaGetLastError();
  if (E <= 16 && launch_regw<TX, 16>(x, w_r, bias, N, d, E, K, ids, gates, margin, stream))
    return cudaGetLastError();
  if (E <= 32 && launch_regw<TX, 32>(x, w_r, bias, N, d, E, K, ids, gates, margin, stream))
    return cudaGetLastError();
  if (E <= 32) return launch_epl<TX, 1>(x, w_r, bias, N, d, E, K, ids, gates, margin, stream);
  if (E <= 64) return launch_epl<TX, 2>(x, w_r, bias, N, d, E, K, ids, gates, margin, stream);
  if (E <= 128) return launch_epl<TX, 4>(x, w_r, bias, N, d, E, K, ids, gates, margin, stream);
  return launch_epl<TX, 8>(x, w_r, bias, N, d, E, K, ids, gates, margin, stream);
}

}  // namespace

cudaError_t launch_router(const void* x, int x_dtype, const float* w_r, const float* bias, int N,
                          int d, int E, int K, int32_t* ids, float* gates, float* margin,
                          cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  if (x_dtype == kF32)
    return launch_t(static_cast<const float*>(x), w_r, bias, N, d, E, K, ids, gates, margin,
                    stream);
  return launch_t(static_cast<const __nv_bfloat16*>(x), w_r, bias, N, d, E, K, ids, gates, margin,
                  stream);
}

}  // namespace moe
