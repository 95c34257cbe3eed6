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
#include "tc_ptx.cuh"

namespace moe {
namespace {

constexpr int kKC = 32;       // k rows per shared-memory chunk
constexpr int kWarps = 8;

// Order-preserving 32-bit key of a float (larger float -> larger key; -0
// and +0 share the key of +0) and its inverse.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  if ((b & 0x7fffffffu) == 0u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// One round of the warp-wide argmax over the still-available logits of a
// token (lane l holds experts l, l+32, ...): the larger value wins, equal
// values go to the lower expert index.  Every lane returns the winner.  Two
// warp reductions (redux.sync): the largest key, then the smallest expert
// index among the lanes whose best entry carries that key.
template <int EPL>
__device__ __forceinline__ void warp_argmax(const float (&v)[EPL], const bool (&avail)[EPL],
                                            int lane, float& bv, int& be) {
  uint32_t mk = 0u;
  int mi = INT_MAX;
#pragma unroll
  for (int q = 0; q < EPL; ++q) {
    const uint32_t k = order_key(v[q]);
    if (avail[q] && (mi == INT_MAX || k > mk)) {  // q ascending: ties keep the lower index
      mk = k;
      mi = lane + 32 * q;
    }
  }
  const uint32_t wk = __reduce_max_sync(0xffffffffu, mi != INT_MAX ? mk : 0u);
  const uint32_t wi =
      __reduce_min_sync(0xffffffffu, (mi != INT_MAX && mk == wk) ? static_cast<uint32_t>(mi)
                                                                 : 0xffffffffu);
  be = wi == 0xffffffffu ? INT_MAX : static_cast<int>(wi);
  bv = key_value(wk);
}

// Top-K of one token's logits held by a warp (lane l: experts l, l+32, ...;
// avail marks the real experts), softmax over the kept K, margin = K-th
// minus (K+1)-th logit (+inf when K = E).  Warp-uniform; writes slot j from
// lane j.
template <int EPL>
__device__ __forceinline__ void write_topk(const float (&v)[EPL], bool (&avail)[EPL], int lane,
                                           int K, int E, long long t, int32_t* __restrict__ ids,
                                           float* __restrict__ gates, float* __restrict__ margin) {
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
  // (selections by sel_f / sel_i: sel_v and sel_e stay in registers)
  float z = 0.f, my_g = 0.f;
  int my_e = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < K) {
      const float p = expf(sel_v[j] - sel_v[0]);
      z += p;
      my_g = sel_f(j == lane, p, my_g);
      my_e = sel_i(j == lane, sel_e[j], my_e);
    }
  }
  if (lane < K) {
    ids[t * K + lane] = my_e;
    gates[t * K + lane] = my_g / z;
  }
  if (margin != nullptr && lane == 0) {
    float kth = sel_v[0];
#pragma unroll
    for (int j = 0; j < 8; ++j) kth = sel_f(j == K - 1, sel_v[j], kth);
    margin[t] = (K == E) ? __int_as_float(0x7f800000) : kth - next_v;
  }
}

template <typename TX, int EPL, int TPW>
__global__ void __launch_bounds__(kWarps * 32)
router_kernel(const TX* __restrict__ x, const float* __restrict__ w_r,
              const float* __restrict__ bias, int N, int d, int E, int K,
              int32_t* __restrict__ ids, float* __restrict__ gates, float* __restrict__ margin) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

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
    write_topk<EPL>(v, avail, lane, K, E, t, ids, gates, margin);
  }
}

// Small E (<= 32) with W_r fitting in shared memory: the whole router
// weight is staged once per CTA; warps then stream tokens.  Lane l of a warp
// reads 16-byte vectors v = l, l+32, ... of a token row (VEC consecutive k)
// and accumulates all E logits of TPW tokens in registers (k ascending
// within each vector), so every weight read from shared memory feeds TPW
// tokens.  The E partial sums are then added across the 32 lanes by an XOR
// butterfly (fixed order), after which lane e holds logit e and the top-K is
// taken by K rounds of the warp-shuffle argmax.
//
// Shared layout: block m holds the VEC rows k = m*VEC .. m*VEC+VEC-1 as
// [e][VEC] floats, i.e. 16-byte chunks c = e*VEC/4 + h.  Chunk c of block m
// sits at position c ^ (m & 7): the lanes of a warp read consecutive blocks,
// so the XOR spreads one logical chunk over 8 bank groups (conflict-free
// 128-bit reads).
template <typename TX, int E_T, int TPW>
__global__ void __launch_bounds__(256, E_T <= 8 ? 2 : 1)
router_smem_kernel(const TX* __restrict__ x, const float* __restrict__ w_r,
                   const float* __restrict__ bias, int N, int d, int E, int K,
                   int32_t* __restrict__ ids, float* __restrict__ gates, float* __restrict__ margin) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  constexpr int VEC = 16 / sizeof(TX);        // k per 16-byte vector of x
  constexpr int CPB = E_T * VEC / 4;          // 16-byte chunks per block
  extern __shared__ float4 wsm[];
  const int nvec = d / VEC;                   // d is a multiple of VEC
  // stage W_r: block m, expert e, row i -> chunk (e*VEC + i)/4 ^ (m & 7), lane (i % 4)
  float* wf = reinterpret_cast<float*>(wsm);
  auto put = [&](int k, int e, float v) {
    const int m = k / VEC, i = k % VEC;
    const int c = (e * VEC + i) >> 2;
    wf[((long long)m * CPB + (c ^ (m & 7))) * 4 + (i & 3)] = v;
  };
  // eight loads in flight per thread before their shared-memory stores
  constexpr int kBatch = 8;
  if (E == E_T && (E & 3) == 0) {  // whole rows, 16-byte loads
    const float4* w4 = reinterpret_cast<const float4*>(w_r);
    const int n4 = d * E / 4;
    for (int base = threadIdx.x; base < n4; base += kBatch * blockDim.x) {
      float4 v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int idx = base + u * blockDim.x;
        if (idx < n4) v[u] = w4[idx];
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int idx = base + u * blockDim.x;
        if (idx < n4) {
          const int k = idx * 4 / E, e = idx * 4 % E;
          put(k, e, v[u].x); put(k, e + 1, v[u].y); put(k, e + 2, v[u].z); put(k, e + 3, v[u].w);
        }
      }
    }
  } else {
    const int n = d * E_T;
    for (int base = threadIdx.x; base < n; base += kBatch * blockDim.x) {
      float v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int idx = base + u * blockDim.x;
        const int k = idx / E_T, e = idx % E_T;
        v[u] = (idx < n && e < E) ? w_r[(long long)k * E + e] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int idx = base + u * blockDim.x;
        if (idx < n) put(idx / E_T, idx % E_T, v[u]);
      }
    }
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int gwarp = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int nwarps = gridDim.x * (blockDim.x >> 5);
  for (int t0 = gwarp * TPW; t0 < N; t0 += nwarps * TPW) {
    float acc[TPW][E_T];
#pragma unroll
    for (int j = 0; j < TPW; ++j)
#pragma unroll
      for (int e = 0; e < E_T; ++e) acc[j][e] = 0.f;
    // four vectors per token in flight per lane before the FMAs
    for (int mb = lane; mb < nvec; mb += 128) {
      uint4 u[4][TPW];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int j = 0; j < TPW; ++j) {
          const int m = mb + 32 * q;
          const int t = min(t0 + j, N - 1);
          u[q][j] = m < nvec ? reinterpret_cast<const uint4*>(x + (long long)t * d)[m]
                             : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int m = mb + 32 * q;
        if (m >= nvec) break;
        float xv[TPW][VEC];
#pragma unroll
        for (int j = 0; j < TPW; ++j) {
          if constexpr (VEC == 8) {
            xv[j][0] = bf16lo(u[q][j].x); xv[j][1] = bf16hi(u[q][j].x);
            xv[j][2] = bf16lo(u[q][j].y); xv[j][3] = bf16hi(u[q][j].y);
            xv[j][4] = bf16lo(u[q][j].z); xv[j][5] = bf16hi(u[q][j].z);
            xv[j][6] = bf16lo(u[q][j].w); xv[j][7] = bf16hi(u[q][j].w);
          } else {
            xv[j][0] = __uint_as_float(u[q][j].x); xv[j][1] = __uint_as_float(u[q][j].y);
            xv[j][2] = __uint_as_float(u[q][j].z); xv[j][3] = __uint_as_float(u[q][j].w);
          }
        }
        const float4* blk = wsm + (long long)m * CPB;
#pragma unroll
        for (int e = 0; e < E_T; ++e) {
#pragma unroll
          for (int h = 0; h < VEC / 4; ++h) {
            const float4 w4 = blk[(e * (VEC / 4) + h) ^ (m & 7)];
            const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
              for (int j = 0; j < TPW; ++j) acc[j][e] = fmaf(xv[j][h * 4 + i], wv[i], acc[j][e]);
          }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < TPW; ++j)
#pragma unroll
      for (int e = 0; e < E_T; ++e)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[j][e] += __shfl_xor_sync(0xffffffffu, acc[j][e], o);

#pragma unroll
    for (int j = 0; j < TPW; ++j) {
      const int t = t0 + j;
      if (t >= N) break;  // warp-uniform
      float v[1];
      bool avail[1];
      v[0] = 0.f;
#pragma unroll
      for (int e = 0; e < E_T; ++e)
        if (e == lane) v[0] = acc[j][e];
      avail[0] = lane < E;
      if (avail[0] && bias != nullptr) v[0] += bias[lane];
      write_topk<1>(v, avail, lane, K, E, t, ids, gates, margin);
    }
  }
}

// Split-K router for few tokens and long rows (decode-shaped batches): the
// per-token kernels above give one warp (or one 128-token tile) per token
// group and so leave most SMs idle, each streaming the whole of W_r.  Here
// the reduction dimension is cut into S slices of ks rows: CTA (s, b) stages
// W_r[ks*s .. ks*s+ks) and the matching x columns of 32 tokens in shared
// memory and writes their partial logits (k ascending) to part[s][t][e];
// a second kernel adds the S partials of each (t, e) in slice order (fixed,
// so results are deterministic) and takes the top-K.
constexpr int kSkTokens = 32;  // tokens per CTA of the partial kernel

template <typename TX, int EPL>
__global__ void __launch_bounds__(256)
router_splitk_kernel(const TX* __restrict__ x, const float* __restrict__ w_r, int N, int d, int E,
                     int ks, float* __restrict__ part) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  constexpr int EP = EPL * 32;
  extern __shared__ float sk_smem[];
  float* ws = sk_smem;                 // [ks][EP]
  float* xs = sk_smem + ks * EP;       // [ks][kSkTokens + 1]
  const int k0 = blockIdx.x * ks, kn = min(ks, d - k0);
  const int t0 = blockIdx.y * kSkTokens;
  for (int idx = threadIdx.x; idx < kn * EP; idx += 256) {
    const int kk = idx / EP, e = idx % EP;
    ws[idx] = e < E ? w_r[static_cast<long long>(k0 + kk) * E + e] : 0.f;
  }
  for (int idx = threadIdx.x; idx < kSkTokens * kn; idx += 256) {
    const int t = idx / kn, kk = idx % kn;
    const int gt = t0 + t;
    xs[kk * (kSkTokens + 1) + t] = gt < N ? to_f32(x[static_cast<long long>(gt) * d + k0 + kk]) : 0.f;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int TPW = kSkTokens / 8;  // tokens per warp
  float acc[TPW][EPL];
#pragma unroll
  for (int i = 0; i < TPW; ++i)
#pragma unroll
    for (int q = 0; q < EPL; ++q) acc[i][q] = 0.f;
#pragma unroll 4
  for (int kk = 0; kk < kn; ++kk) {
    float wv[EPL];
#pragma unroll
    for (int q = 0; q < EPL; ++q) wv[q] = ws[kk * EP + lane + 32 * q];
#pragma unroll
    for (int i = 0; i < TPW; ++i) {
      const float xv = xs[kk * (kSkTokens + 1) + warp * TPW + i];
#pragma unroll
      for (int q = 0; q < EPL; ++q) acc[i][q] = fmaf(xv, wv[q], acc[i][q]);
    }
  }
#pragma unroll
  for (int i = 0; i < TPW; ++i) {
    const int t = t0 + warp * TPW + i;
    if (t >= N) break;  // warp-uniform
    float* prow = part + (static_cast<long long>(blockIdx.x) * N + t) * E;
#pragma unroll
    for (int q = 0; q < EPL; ++q)
      if (lane + 32 * q < E) prow[lane + 32 * q] = acc[i][q];
  }
}

// One CTA of 256 threads per token: thread (g, e) adds the partials of
// expert e over its share of the slices (slice order), the G shares are
// added in share order, then warp 0 takes the top-K.
template <int EPL>
__global__ void __launch_bounds__(256)
router_splitk_reduce_kernel(const float* __restrict__ part, const float* __restrict__ bias, int N,
                            int E, int K, int S, int32_t* __restrict__ ids,
                            float* __restrict__ gates, float* __restrict__ margin) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  constexpr int EP = EPL * 32;
  constexpr int G = 256 / EP;  // slice shares per expert
  __shared__ float sums[G][EP];
  const int t = blockIdx.x;
  const int e = threadIdx.x % EP, g = threadIdx.x / EP;
  const int per = (S + G - 1) / G;
  const int s0 = g * per, s1 = min(S, s0 + per);
  float a = 0.f;
  if (e < E) {
    const float* p = part + static_cast<long long>(t) * E + e;
    const long long stride = static_cast<long long>(N) * E;
    int s = s0;
    for (; s + 4 <= s1; s += 4) {
      const float v0 = p[s * stride], v1 = p[(s + 1) * stride], v2 = p[(s + 2) * stride],
                  v3 = p[(s + 3) * stride];
      a += v0; a += v1; a += v2; a += v3;
    }
    for (; s < s1; ++s) a += p[s * stride];
  }
  sums[g][e] = a;
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    float v[EPL];
    bool avail[EPL];
#pragma unroll
    for (int q = 0; q < EPL; ++q) {
      const int ee = lane + 32 * q;
      float tot = 0.f;
#pragma unroll
      for (int gg = 0; gg < G; ++gg) tot += sums[gg][ee];
      avail[q] = ee < E;
      v[q] = tot + ((bias != nullptr && ee < E) ? bias[ee] : 0.f);
    }
    write_topk<EPL>(v, avail, lane, K, E, t, ids, gates, margin);
  }
}

// Top-K of logits already in memory (the tensor-core router's output): one
// warp per token, lane l reads experts l, l+32, ...
template <int EPL>
__global__ void __launch_bounds__(256)
logits_topk_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int N, int E,
                   int K, int32_t* __restrict__ ids, float* __restrict__ gates,
                   float* __restrict__ margin) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (t >= N) return;  // whole warp
  const float* row = logits + static_cast<long long>(t) * E;
  float v[EPL];
  bool avail[EPL];
#pragma unroll
  for (int q = 0; q < EPL; ++q) {
    const int e = lane + 32 * q;
    avail[q] = e < E;
    v[q] = avail[q] ? row[e] + (bias != nullptr ? bias[e] : 0.f) : 0.f;
  }
  write_topk<EPL>(v, avail, lane, K, E, t, ids, gates, margin);
}

template <typename TX, int EPL>
cudaError_t launch_splitk(const TX* x, const float* w_r, const float* bias, int N, int d, int E,
                          int K, int32_t* ids, float* gates, float* margin, float* part,
                          cudaStream_t stream) {
  constexpr int EP = EPL * 32;
  const int ks = router_splitk_rows(d, E);
  const int S = (d + ks - 1) / ks;
  const size_t smem = static_cast<size_t>(ks) * (EP + kSkTokens + 1) * sizeof(float);
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(router_splitk_kernel<TX, EPL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kRouterSplitkSmemMax));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  if (smem > kRouterSplitkSmemMax) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(S), static_cast<unsigned>((N + kSkTokens - 1) / kSkTokens));
  cudaError_t e = launch_pdl(router_splitk_kernel<TX, EPL>, grid, dim3(256), smem, stream, x, w_r,
                             N, d, E, ks, part);
  if (e != cudaSuccess) return e;
  return launch_pdl(router_splitk_reduce_kernel<EPL>, dim3(static_cast<unsigned>(N)), dim3(256), 0,
                    stream, part, bias, N, E, K, S, ids, gates, margin);
}

template <typename TX>
cudaError_t launch_splitk_t(const TX* x, const float* w_r, const float* bias, int N, int d, int E,
                            int K, int32_t* ids, float* gates, float* margin, float* part,
                            cudaStream_t stream) {
  if (E <= 32) return launch_splitk<TX, 1>(x, w_r, bias, N, d, E, K, ids, gates, margin, part, stream);
  if (E <= 64) return launch_splitk<TX, 2>(x, w_r, bias, N, d, E, K, ids, gates, margin, part, stream);
  if (E <= 128) return launch_splitk<TX, 4>(x, w_r, bias, N, d, E, K, ids, gates, margin, part, stream);
  return launch_splitk<TX, 8>(x, w_r, bias, N, d, E, K, ids, gates, margin, part, stream);
}

constexpr size_t kRouterSmemMax = 160 * 1024;

template <typename TX, int E_T>
bool launch_smem(const TX* x, const float* w_r, const float* bias, int N, int d, int E, int K,
                 int32_t* ids, float* gates, float* margin, cudaStream_t stream) {
  constexpr int VEC = 16 / sizeof(TX);
  const size_t smem = static_cast<size_t>(d) * E_T * sizeof(float);
  if (d % VEC != 0 || smem > kRouterSmemMax) return false;
  constexpr int TPW = E_T <= 8 ? 2 : 1;
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    if (cudaFuncSetAttribute(router_smem_kernel<TX, E_T, TPW>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kRouterSmemMax)) != cudaSuccess)
      return false;
    configured[dev] = true;
  }
  // up to two CTAs per SM (shared memory permitting): the weights are staged
  // once per CTA, then every warp streams tokens
  const int per_sm = (E_T <= 8 && smem <= 100 * 1024) ? 2 : 1;
  const long long need = (static_cast<long long>(N) + 8 * TPW - 1) / (8 * TPW);
  const long long cap = static_cast<long long>(per_sm) * device_sm_count();
  const int grid = static_cast<int>(need < cap ? need : cap);
  launch_pdl(router_smem_kernel<TX, E_T, TPW>, dim3(grid), dim3(256), smem, stream, x, w_r, bias, N, d, E, K, ids,
                                                                gates, margin);
  return true;
}

template <typename TX, int EPL>
cudaError_t launch_epl(const TX* x, const float* w_r, const float* bias, int N, int d, int E,
                       int K, int32_t* ids, float* gates, float* margin, cudaStream_t stream) {
  // Many tokens: 8 per warp reuse each staged weight row 8 times.  Few
  // tokens: 2 per warp spread the CTAs over more SMs.
  int sms = device_sm_count();
  if ((long long)N >= 64LL * 2 * sms) {
    int grid = (N + 63) / 64;
    launch_pdl(router_kernel<TX, EPL, 8>, dim3(grid), dim3(kWarps * 32), 0, stream, x, w_r, bias, N, d, E, K, ids,
                                                                 gates, margin);
  } else {
    int grid = (N + 15) / 16;
    launch_pdl(router_kernel<TX, EPL, 2>, dim3(grid), dim3(kWarps * 32), 0, stream, x, w_r, bias, N, d, E, K, ids,
                                                                 gates, margin);
  }
  return cudaGetLastError();
}

template <typename TX>
cudaError_t launch_t(const TX* x, const float* w_r, const float* bias, int N, int d, int E, int K,
                     int32_t* ids, float* gates, float* margin, cudaStream_t stream) {
  if (E <= 8 && launch_smem<TX, 8>(x, w_r, bias, N, d, E, K, ids, gates, margin, stream))
    return cudaGetLastError();
  if (E <= 16 && launch_smem<TX, 16>(x, w_r, bias, N, d, E, K, ids, gates, margin, stream))
    return cudaGetLastError();
  if (E <= 32 && launch_smem<TX, 32>(x, w_r, bias, N, d, E, K, ids, gates, margin, stream))
    return cudaGetLastError();
  if (E <= 32) return launch_epl<TX, 1>(x, w_r, bias, N, d, E, K, ids, gates, margin, stream);
  if (E <= 64) return launch_epl<TX, 2>(x, w_r, bias, N, d, E, K, ids, gates, margin, stream);
  if (E <= 128) return launch_epl<TX, 4>(x, w_r, bias, N, d, E, K, ids, gates, margin, stream);
  return launch_epl<TX, 8>(x, w_r, bias, N, d, E, K, ids, gates, margin, stream);
}

// ---- bf16 tokens, few experts: the logits on the warp-level tensor-core MMA ----
//
// For a handful of experts (E <= 16) the router reads N*d*2 bytes of tokens
// and does 8 FLOP per byte: the fp32 FMA form above spends more issue slots
// on its multiply-adds and weight loads than the tokens take to stream from
// HBM.  Here the contraction runs on mma.sync m16n8k16 (bf16 in, fp32
// accumulate), one instruction per 16 tokens x 8 experts x 16 k, so the
// kernel is bound by the token stream.  fp32-level logits come from the same
// exact three-part split as the tcgen05 router:
//   w = hi + mid + lo,  hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid),
// each part in its own fp32 accumulator (bf16 x bf16 products are exact in
// fp32), logit = (hi + mid) + lo.
//
// Work split: a CTA owns G groups of 16 tokens; its 8G warps are (group,
// k-slice) pairs, the reduction dimension cut into 8 slices of 32-element
// blocks, so every warp issues all the 16-byte token loads of its slice at
// once (16 rows x 256 elements for d = 2048).  The slices' partial logits
// meet in shared memory and are added in slice order (fixed: deterministic);
// then one warp per token takes the top-K as in the other routers.
//
// k order inside a 32-element block.  Thread (g, c) of a warp (g = lane / 4,
// c = lane % 4) loads 8 consecutive elements 8c..8c+7 of token rows g and
// g+8 as one 16-byte vector each.  The MMA's A fragment wants that thread to
// hold logical k positions {2c, 2c+1, 2c+8, 2c+9}; the sum over k does not
// depend on which physical k sits at which logical position as long as A and
// B agree, so the first MMA of a block takes physical k = 8c + {0,1,2,3} and
// the second 8c + {4,5,6,7}.  The weights are stored in exactly that order
// (router_frag_kernel): entry ((b * NT + nt) * 3 + part) * 32 + lane is the
// 16-byte vector W_part[32b + 8c + i][8nt + g], i = 0..7.

constexpr int kMmaSlices = 8;   // warps (k slices) per 16-token group

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Token rows are read once: keep them out of L1 so the weights stay there.
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// w_r (d, E) fp32 -> fragment-ordered three-part bf16 split (see above), for
// nb = ceil(d / 32) blocks and NT = ceil(E / 8) expert tiles; entries past d
// or E are zero.  One thread per 16-byte entry.
__global__ void __launch_bounds__(256)
router_frag_kernel(const float* __restrict__ w_r, int d, int E, int nb, int NT,
                   uint4* __restrict__ frag) {
  const long long n = static_cast<long long>(nb) * NT * 3 * 32;
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int lane = static_cast<int>(i % 32);
  const int part = static_cast<int>((i / 32) % 3);
  const int nt = static_cast<int>((i / 96) % NT);
  const int b = static_cast<int>(i / (96LL * NT));
  const int g = lane >> 2, c = lane & 3;
  const int e = 8 * nt + g;
  uint32_t h[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int k = 32 * b + 8 * c + q;
    const float w = (k < d && e < E) ? w_r[static_cast<long long>(k) * E + e] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    const __nv_bfloat16 v = part == 0 ? hi : part == 1 ? mid : lo;
    h[q] = static_cast<uint32_t>(__bfloat16_as_ushort(v));
  }
  frag[i] = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                       h[6] | (h[7] << 16));
}

// XB: 32-element blocks whose token vectors are loaded before their MMAs
// (2 * XB 16-byte loads in flight per thread; fewer for two expert tiles,
// whose accumulators take the registers).
//
// kSmemW: the CTA first copies the split weights into shared memory, one
// bulk copy (cp.async.bulk, no multicast) per k slice onto that slice's
// mbarrier, issued in an order rotated by the CTA index; each warp issues its
// token loads, then waits for its own slice only.  Every CTA reads the same
// weights: rotating the order spreads those reads over the weight lines
// instead of every SM asking for the same lines at once.  Without kSmemW
// (weights too large for shared memory) the fragments are read straight
// from global memory, the slice's blocks in the same rotated order.
template <int NT, int G, bool kSmemW, int XB = (NT == 1 ? 8 : 4)>
__global__ void __launch_bounds__(32 * kMmaSlices * G)
router_mma_kernel(const __nv_bfloat16* __restrict__ x, const uint4* __restrict__ frag,
                  const float* __restrict__ bias, int N, int d, int E, int K, int nb, int bps,
                  int32_t* __restrict__ ids, float* __restrict__ gates,
                  float* __restrict__ margin, int* status) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  constexpr int EW = 8 * NT;  // expert columns
  constexpr int kBlockU4 = NT * 96;  // 16-byte entries of one 32-element block
  __shared__ float part_s[G][kMmaSlices][16][EW];
  __shared__ __align__(8) uint64_t wbar[kMmaSlices];
  __shared__ int abort_s;
  extern __shared__ uint4 mma_wsm[];  // kSmemW: the split weights, nb blocks
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int gi = warp / kMmaSlices, ks = warp % kMmaSlices;
  const int g = lane >> 2, c = lane & 3;
  const long long t0 = (static_cast<long long>(blockIdx.x) * G + gi) * 16;
  const long long ta = t0 + g, tb = t0 + g + 8;
  const int rv = d / 8;  // 16-byte vectors per token row (d % 8 == 0)
  const uint4* xa = reinterpret_cast<const uint4*>(x) + (ta < N ? ta : 0) * rv;
  const uint4* xb = reinterpret_cast<const uint4*>(x) + (tb < N ? tb : 0) * rv;
  const int b0 = ks * bps, b1 = min(nb, b0 + bps);

  if constexpr (kSmemW) {
    if (threadIdx.x == 0) {
      for (int q = 0; q < kMmaSlices; ++q) tc::mbar_init(tc::smem_u32(&wbar[q]), 1);
      abort_s = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int i = 0; i < kMmaSlices; ++i) {
        const int q = static_cast<int>((i + blockIdx.x) % kMmaSlices);
        const int q0 = q * bps, q1 = min(nb, q0 + bps);
        const uint32_t bar = tc::smem_u32(&wbar[q]);
        if (q1 > q0) {
          const uint32_t bytes = static_cast<uint32_t>((q1 - q0) * kBlockU4 * 16);
          tc::mbar_expect_tx(bar, bytes);
          tc::bulk_load(tc::smem_u32(mma_wsm + static_cast<long long>(q0) * kBlockU4),
                        frag + static_cast<long long>(q0) * kBlockU4, bytes, bar);
        } else {
          tc::mbar_arrive(bar);  // an empty slice: its phase completes at once
        }
      }
    }
  }

  float acc[3][NT][4];
#pragma unroll
  for (int p = 0; p < 3; ++p)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[p][nt][q] = 0.f;

  bool waited = !kSmemW;
  const int nblk = b1 > b0 ? b1 - b0 : 0;
  const int rot = kSmemW ? 0 : static_cast<int>(blockIdx.x % static_cast<unsigned>(nblk > 0 ? nblk : 1));
  for (int bb = 0; bb < nblk; bb += XB) {
    // the token vectors of up to XB blocks in flight before any MMA
    uint4 ua[XB], ub[XB];
#pragma unroll
    for (int i = 0; i < XB; ++i) {
      const int bi = bb + i < nblk ? b0 + (bb + i + rot) % nblk : b0;
      const int v = 4 * bi + c;  // vector index of elements 32 bi + 8c ..
      const bool in = bb + i < nblk && v < rv;
      ua[i] = (in && ta < N) ? ld_stream(xa + v) : make_uint4(0u, 0u, 0u, 0u);
      ub[i] = (in && tb < N) ? ld_stream(xb + v) : make_uint4(0u, 0u, 0u, 0u);
    }
    if (!waited) {  // this slice's weights in shared memory
      waited = true;
      const bool ok = tc::mbar_wait(tc::smem_u32(&wbar[ks]), 0, &abort_s);
      if (!ok) set_status(status, kStatusTimeout);
    }
#pragma unroll
    for (int i = 0; i < XB; ++i) {
      if (bb + i >= nblk) break;  // warp-uniform
      const int b = b0 + (bb + i + rot) % nblk;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const long long wi = static_cast<long long>(b) * kBlockU4 + nt * 96 + lane;
#pragma unroll
        for (int p = 0; p < 3; ++p) {
          const uint4 w = kSmemW ? mma_wsm[wi + 32 * p] : __ldg(frag + wi + 32 * p);
          mma_bf16_16816(acc[p][nt], ua[i].x, ub[i].x, ua[i].y, ub[i].y, w.x, w.y);
          mma_bf16_16816(acc[p][nt], ua[i].z, ub[i].z, ua[i].w, ub[i].w, w.z, w.w);
        }
      }
    }
  }
  if (kSmemW && !waited) {  // a slice with no blocks still consumes its phase
    if (!tc::mbar_wait(tc::smem_u32(&wbar[ks]), 0, &abort_s)) set_status(status, kStatusTimeout);
  }
  // this slice's partial logits: rows g, g+8; columns 8nt + 2c, 2c+1
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int row = g + (q >> 1) * 8, col = 8 * nt + 2 * c + (q & 1);
      part_s[gi][ks][row][col] = (acc[0][nt][q] + acc[1][nt][q]) + acc[2][nt][q];
    }
  __syncthreads();
  // top-K: one warp per token, lane e holds expert e's logit (slices added in order)
  for (int tl = warp; tl < 16 * G; tl += kMmaSlices * G) {
    const long long t = static_cast<long long>(blockIdx.x) * 16 * G + tl;
    if (t >= N) break;  // warp-uniform
    float v[1];
    bool avail[1];
    float sum = 0.f;
    if (lane < EW) {
#pragma unroll
      for (int s = 0; s < kMmaSlices; ++s) sum += part_s[tl / 16][s][tl % 16][lane];
    }
    avail[0] = lane < E;
    v[0] = avail[0] ? sum + (bias != nullptr ? bias[lane] : 0.f) : 0.f;
    write_topk<1>(v, avail, lane, K, E, t, ids, gates, margin);
  }
}

}  // namespace

cudaError_t launch_logits_topk(const float* logits, const float* bias, int N, int E, int K,
                              int32_t* ids, float* gates, float* margin, cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((N + 7) / 8));
  if (E <= 32)
    return launch_pdl(logits_topk_kernel<1>, grid, dim3(256), 0, stream, logits, bias, N, E, K, ids, gates, margin);
  if (E <= 64)
    return launch_pdl(logits_topk_kernel<2>, grid, dim3(256), 0, stream, logits, bias, N, E, K, ids, gates, margin);
  if (E <= 128)
    return launch_pdl(logits_topk_kernel<4>, grid, dim3(256), 0, stream, logits, bias, N, E, K, ids, gates, margin);
  return launch_pdl(logits_topk_kernel<8>, grid, dim3(256), 0, stream, logits, bias, N, E, K, ids, gates, margin);
}

int router_splitk_rows(int d, int E) {
  // about 64 slices, each staging at most kRouterSplitkSmemMax of weights and
  // token columns; a multiple of 4 rows
  const int ep = (E + 31) / 32 * 32;
  const int cap = static_cast<int>(kRouterSplitkSmemMax / ((ep + kSkTokens + 1) * sizeof(float)));
  int ks = (d + 63) / 64;
  ks = (ks + 3) / 4 * 4;
  if (ks > cap) ks = cap / 4 * 4;
  return ks < 4 ? 4 : ks;
}

bool router_uses_splitk(int N, int d) { return N <= kRouterSplitkMaxTokens && d >= 1024; }

size_t router_splitk_scratch_bytes(int N, int d, int E) {
  const int ks = router_splitk_rows(d, E);
  const long long S = (d + ks - 1) / ks;
  return static_cast<size_t>(S) * N * E * sizeof(float);
}

cudaError_t launch_router(const void* x, int x_dtype, const float* w_r, const float* bias, int N,
                          int d, int E, int K, int32_t* ids, float* gates, float* margin,
                          void* scratch, cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  if (router_uses_splitk(N, d)) {
    if (scratch == nullptr) return cudaErrorInvalidValue;
    float* part = static_cast<float*>(scratch);
    if (x_dtype == kF32)
      return launch_splitk_t(static_cast<const float*>(x), w_r, bias, N, d, E, K, ids, gates,
                             margin, part, stream);
    return launch_splitk_t(static_cast<const __nv_bfloat16*>(x), w_r, bias, N, d, E, K, ids, gates,
                           margin, part, stream);
  }
  if (x_dtype == kF32)
    return launch_t(static_cast<const float*>(x), w_r, bias, N, d, E, K, ids, gates, margin,
                    stream);
  return launch_t(static_cast<const __nv_bfloat16*>(x), w_r, bias, N, d, E, K, ids, gates, margin,
                  stream);
}


// ---- the warp-MMA router (bf16 tokens, E <= 16) ----------------------------

bool router_uses_mma(int N, int d, int E, int x_dtype) {
  return x_dtype == kBF16 && E <= kRouterMmaMaxExperts && !router_uses_splitk(N, d);
}

size_t router_mma_frag_bytes(int d, int E) {
  const int nb = (d + 31) / 32, NT = (E + 7) / 8;
  return static_cast<size_t>(nb) * NT * 3 * 32 * sizeof(uint4);
}

cudaError_t launch_router_mma_frag(const float* w_r, int d, int E, void* frag, cudaStream_t stream) {
  const int nb = (d + 31) / 32, NT = (E + 7) / 8;
  const long long n = static_cast<long long>(nb) * NT * 96;
  router_frag_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, stream>>>(
      w_r, d, E, nb, NT, static_cast<uint4*>(frag));
  return cudaGetLastError();
}

cudaError_t launch_router_mma(const void* x, const void* frag, const float* bias, int N, int d,
                              int E, int K, int32_t* ids, float* gates, float* margin, int* status,
                              cudaStream_t stream) {
  if (N == 0) return cudaSuccess;
  if (E > kRouterMmaMaxExperts || d % 8) return cudaErrorInvalidValue;
  const int nb = (d + 31) / 32;
  const int bps = (nb + kMmaSlices - 1) / kMmaSlices;  // 32-element blocks per slice
  auto xb = static_cast<const __nv_bfloat16*>(x);
  auto fr = static_cast<const uint4*>(frag);
  // two 16-token groups per CTA (sixteen warps) once there are more groups
  // than SMs: the same per-SM work as two one-group CTAs, half the weight reads
  const long long groups = (N + 15) / 16;
  const bool two = groups > device_sm_count();
  const unsigned grid = static_cast<unsigned>(two ? (groups + 1) / 2 : groups);
  const size_t wbytes = router_mma_frag_bytes(d, E);
  const bool smem_w = wbytes <= kRouterMmaSmemMax;
  const size_t smem = smem_w ? wbytes : 0;
  const dim3 block(two ? 512 : 256);
#define MOE_ROUTER_MMA_LAUNCH(NT_, G_, S_)                                                       \
  do {                                                                                           \
    auto kern = router_mma_kernel<NT_, G_, S_>;                                                  \
    if (S_) {                                                                                    \
      static bool configured[64] = {false};                                                      \
      int dev = 0;                                                                               \
      cudaGetDevice(&dev);                                                                       \
      if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;                                   \
      if (!configured[dev]) {                                                                    \
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,  \
                                             static_cast<int>(kRouterMmaSmemMax));               \
        if (e != cudaSuccess) return e;                                                          \
        configured[dev] = true;                                                                  \
      }                                                                                          \
    }                                                                                            \
    return launch_pdl(kern, dim3(grid), block, smem, stream, xb, fr, bias, N, d, E, K, nb, bps,  \
                      ids, gates, margin, status);                                               \
  } while (0)
  if (E <= 8) {
    if (two) {
      if (smem_w) MOE_ROUTER_MMA_LAUNCH(1, 2, true);
      MOE_ROUTER_MMA_LAUNCH(1, 2, false);
    }
    if (smem_w) MOE_ROUTER_MMA_LAUNCH(1, 1, true);
    MOE_ROUTER_MMA_LAUNCH(1, 1, false);
  }
  if (two) {
    if (smem_w) MOE_ROUTER_MMA_LAUNCH(2, 2, true);
    MOE_ROUTER_MMA_LAUNCH(2, 2, false);
  }
  if (smem_w) MOE_ROUTER_MMA_LAUNCH(2, 1, true);
  MOE_ROUTER_MMA_LAUNCH(2, 1, false);
#undef MOE_ROUTER_MMA_LAUNCH
}

}  // namespace moe
