// Unpermute + combine: y[t] = sum_j g[t,j] * y_perm[pos[t,j]] (zyxy.net MoE
// page, MoE structure: y = sum_i g_i(x) E_i(x)), or the pure reorder
// y[t*K+j] = y_perm[pos[t,j]] (aclnnQuantGroupedMatMulAlltoAllv formula:
// unpermuteOut = Unpermute(gmmY), output (BSK, N1)).
//
// WPT warps per output token (gated; more than one for small batches, the
// row's 16-byte vectors split between them) or one warp per output row
// (reorder).  The K source rows of a token are read with coalesced 512-byte
// warp accesses and accumulated in fp32 in slot order j = 0..K-1, then
// rounded once to the output dtype.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

// 16 bytes of T as fp32 lanes
template <typename T> struct Vec;
template <> struct Vec<float> {
  static constexpr int n = 4;
  __device__ static void load(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
  __device__ static uint4 store(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};
template <> struct Vec<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ static void load(const uint4& u, float* f) {
    f[0] = bf16lo(u.x); f[1] = bf16hi(u.x); f[2] = bf16lo(u.y); f[3] = bf16hi(u.y);
    f[4] = bf16lo(u.z); f[5] = bf16hi(u.z); f[6] = bf16lo(u.w); f[7] = bf16hi(u.w);
  }
  __device__ static uint4 store(const float* f) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
  }
};

template <typename T, int KMAX, int WPT>
__global__ void __launch_bounds__(256)
combine_kernel(const uint4* __restrict__ y_perm, int row_vecs, const int32_t* __restrict__ pos,
               const float* __restrict__ gates, int N, int K, int R, uint4* __restrict__ y,
               int* status) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.x * (8 / WPT) + warp / WPT;
  const int sub = warp % WPT;
  if (t >= N) return;
  int p[KMAX];
  float g[KMAX];
  int mine_p = -1;
  float mine_g = 0.f;
  if (lane < K) {
    mine_p = pos[(long long)t * K + lane];
    mine_g = gates[(long long)t * K + lane];
    if (mine_p < 0 || mine_p >= R) {
      set_status(status, kStatusBadIndex);
      mine_p = -1;
    }
  }
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    p[j] = __shfl_sync(0xffffffffu, mine_p, j);
    g[j] = __shfl_sync(0xffffffffu, mine_g, j);
  }
  constexpr int n = Vec<T>::n;
  constexpr int STEP = 32 * WPT;
  // several vectors of the row per lane at once (about eight 16-byte loads
  // in flight per lane: KMAX rows x kBatch vectors)
  constexpr int kBatch = KMAX <= 2 ? 4 : KMAX <= 4 ? 2 : 1;
  int v = sub * 32 + lane;
  if constexpr (kBatch > 1) {
    for (; v + (kBatch - 1) * STEP < row_vecs; v += kBatch * STEP) {
      uint4 raw[kBatch][KMAX];
#pragma unroll
      for (int b = 0; b < kBatch; ++b)
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
          if (j < K && p[j] >= 0) raw[b][j] = y_perm[(long long)p[j] * row_vecs + v + b * STEP];
#pragma unroll
      for (int b = 0; b < kBatch; ++b) {
        float acc[n];
#pragma unroll
        for (int i = 0; i < n; ++i) acc[i] = 0.f;
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          if (j < K && p[j] >= 0) {
            float f[n];
            Vec<T>::load(raw[b][j], f);
#pragma unroll
            for (int i = 0; i < n; ++i) acc[i] = fmaf(g[j], f[i], acc[i]);
          }
        }
        y[(long long)t * row_vecs + v + b * STEP] = Vec<T>::store(acc);
      }
    }
  }
  for (; v < row_vecs; v += STEP) {
    float acc[n];
#pragma unroll
    for (int i = 0; i < n; ++i) acc[i] = 0.f;
    uint4 raw[KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
      if (j < K && p[j] >= 0) raw[j] = y_perm[(long long)p[j] * row_vecs + v];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < K && p[j] >= 0) {
        float f[n];
        Vec<T>::load(raw[j], f);
#pragma unroll
        for (int i = 0; i < n; ++i) acc[i] = fmaf(g[j], f[i], acc[i]);
      }
    }
    y[(long long)t * row_vecs + v] = Vec<T>::store(acc);
  }
}

__global__ void __launch_bounds__(256)
unpermute_kernel(const uint4* __restrict__ y_perm, int row_vecs, const int32_t* __restrict__ pos,
                 int R, uint4* __restrict__ y, int* status) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  const int lane = threadIdx.x & 31;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= R) return;
  int p = pos[r];
  if (p < 0 || p >= R) {
    if (lane == 0) set_status(status, kStatusBadIndex);
    return;
  }
  const uint4* s = y_perm + (long long)p * row_vecs;
  uint4* d = y + (long long)r * row_vecs;
  int v = lane;
  for (; v + 96 < row_vecs; v += 128) {
    uint4 a0 = s[v], a1 = s[v + 32], a2 = s[v + 64], a3 = s[v + 96];
    d[v] = a0; d[v + 32] = a1; d[v + 64] = a2; d[v + 96] = a3;
  }
  for (; v < row_vecs; v += 32) d[v] = s[v];
}

template <typename T, int KMAX>
void launch_gated_k(const uint4* yp, int row_vecs, const int32_t* pos, const float* gates, int N,
                    int K, int R, uint4* y, int* status, cudaStream_t stream) {
  const int wpt = warps_per_token(N);
  const dim3 grid((N + 8 / wpt - 1) / (8 / wpt));
  if (wpt == 1)
    launch_pdl(combine_kernel<T, KMAX, 1>, grid, dim3(256), 0, stream, yp, row_vecs, pos, gates, N, K, R, y, status);
  else if (wpt == 2)
    launch_pdl(combine_kernel<T, KMAX, 2>, grid, dim3(256), 0, stream, yp, row_vecs, pos, gates, N, K, R, y, status);
  else if (wpt == 4)
    launch_pdl(combine_kernel<T, KMAX, 4>, grid, dim3(256), 0, stream, yp, row_vecs, pos, gates, N, K, R, y, status);
  else
    launch_pdl(combine_kernel<T, KMAX, 8>, grid, dim3(256), 0, stream, yp, row_vecs, pos, gates, N, K, R, y, status);
}

template <typename T>
void launch_gated(const uint4* yp, int row_vecs, const int32_t* pos, const float* gates, int N,
                  int K, int R, uint4* y, int* status, cudaStream_t stream) {
  if (K <= 2) launch_gated_k<T, 2>(yp, row_vecs, pos, gates, N, K, R, y, status, stream);
  else if (K <= 4) launch_gated_k<T, 4>(yp, row_vecs, pos, gates, N, K, R, y, status, stream);
  else launch_gated_k<T, 8>(yp, row_vecs, pos, gates, N, K, R, y, status, stream);
}

}  // namespace

cudaError_t launch_combine(const void* y_perm, int y_dtype, int dout, const int32_t* pos,
                           const float* gates, int N, int K, void* y, int* status,
                           cudaStream_t stream) {
  const int R = N * K;
  if (R == 0) return cudaSuccess;
  const int row_vecs = dout * dtype_bytes(y_dtype) / 16;
  auto yp = static_cast<const uint4*>(y_perm);
  auto yo = static_cast<uint4*>(y);
  if (gates == nullptr) {
    launch_pdl(unpermute_kernel, dim3((R + 7) / 8), dim3(256), 0, stream, yp, row_vecs, pos, R, yo, status);
  } else if (y_dtype == kF32) {
    launch_gated<float>(yp, row_vecs, pos, gates, N, K, R, yo, status, stream);
  } else {
    launch_gated<__nv_bfloat16>(yp, row_vecs, pos, gates, N, K, R, yo, status, stream);
  }
  return cudaGetLastError();
}

}  // namespace moe
