// Grouped expert GEMM for fp32 layers on the FP32 FMA pipes ("Advanced GPU
// Optimization ... Part 5", section 1.2 step 2: every expert's FFN on the
// tokens routed to it).  The fp32 path needs fp32-exact products (tf32
// tensor cores round the operands to 10 mantissa bits), so it runs on the
// SIMT pipes: 64x64 output tiles, k staged through shared memory in slices
// of 16 (the next slice prefetched into registers), a 4x4 register
// micro-tile per thread, k summed in ascending order.
//
// Tile schedule: blockIdx.y enumerates the 64-row tiles of all experts in
// expert order (empty experts own none); the CTA finds its expert from the
// device-side offsets, so no host round trip is needed.
//
// Split-K (small grids): blockIdx.z takes k slice z of a fixed partition; the
// CTA writes its raw sums to partial[z] and a second kernel adds the slices
// in order (deterministic) and applies the activation.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <int ACT>
__global__ void __launch_bounds__(256)
gemm_simt_f32_kernel(const float* __restrict__ A, int kdim, const float* __restrict__ W,
                     const float* __restrict__ W3, int ncols, float scale,
                     const int32_t* __restrict__ offsets, int E, float* __restrict__ out,
                     int kchunk, float* __restrict__ partial, long long part_stride) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  __shared__ __align__(16) float As[BK][BM + 4];
  __shared__ __align__(16) float Bs[BK][BN + 4];
  __shared__ __align__(16) float Us[BK][BN + 4];
  __shared__ int s_e, s_row0, s_row1;

  if (threadIdx.x == 0) {
    int tile = blockIdx.y, run = 0, found = -1;
    for (int e = 0; e < E; ++e) {
      int r0 = offsets[e], r1 = offsets[e + 1];
      int mt = (r1 - r0 + BM - 1) / BM;
      if (tile < run + mt) {
        found = e;
        s_row0 = r0 + (tile - run) * BM;
        s_row1 = r1;
        break;
      }
      run += mt;
    }
    s_e = found;
  }
  __syncthreads();
  const int e = s_e;
  if (e < 0) return;  // fewer tiles than the grid's upper bound
  const int row0 = s_row0, row1 = s_row1;
  const int col0 = blockIdx.x * BN;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  const float* We = W + (long long)e * ncols * kdim;
  const float* Ue = ACT == kActSwiglu ? W3 + (long long)e * ncols * kdim : nullptr;
  // k range of this CTA (the whole row without split-K)
  const int kb = blockIdx.z * kchunk, ke = min(kdim, kb + kchunk);

  float acc[4][4], accu[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = accu[i][j] = 0.f;

  const int lr = tid / 4, lk = (tid % 4) * 4;  // loader: row/col within tile, k offset
  // the next k-slice is fetched into registers while the current one is
  // multiplied out of shared memory
  float4 na, nb, nu;
  auto fetch = [&](int k0) {
    const int r = row0 + lr, k = k0 + lk, n = col0 + lr;
    na = (r < row1 && k < ke) ? *reinterpret_cast<const float4*>(A + (long long)r * kdim + k)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    nb = (n < ncols && k < ke) ? *reinterpret_cast<const float4*>(We + (long long)n * kdim + k)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
    if (ACT == kActSwiglu)
      nu = (n < ncols && k < ke) ? *reinterpret_cast<const float4*>(Ue + (long long)n * kdim + k)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  fetch(kb);
  for (int k0 = kb; k0 < ke; k0 += BK) {
    As[lk + 0][lr] = na.x; As[lk + 1][lr] = na.y; As[lk + 2][lr] = na.z; As[lk + 3][lr] = na.w;
    Bs[lk + 0][lr] = nb.x; Bs[lk + 1][lr] = nb.y; Bs[lk + 2][lr] = nb.z; Bs[lk + 3][lr] = nb.w;
    if (ACT == kActSwiglu) {
      Us[lk + 0][lr] = nu.x; Us[lk + 1][lr] = nu.y; Us[lk + 2][lr] = nu.z; Us[lk + 3][lr] = nu.w;
    }
    __syncthreads();
    if (k0 + BK < ke) fetch(k0 + BK);
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float4 a = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      float4 b = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      if (ACT == kActSwiglu) {
        float4 u = *reinterpret_cast<const float4*>(&Us[kk][tx * 4]);
        float uv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) accu[i][j] = fmaf(av[i], uv[j], accu[i][j]);
      }
    }
    __syncthreads();
  }

  if (partial != nullptr) {
    // split-K: raw sums of this k slice (gate in partial, up after it)
    float* pg = partial + blockIdx.z * part_stride;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = row0 + ty * 4 + i;
      if (r >= row1 || r >= row0 + BM) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = col0 + tx * 4 + j;
        if (n >= ncols) continue;
        pg[(long long)r * ncols + n] = acc[i][j];
        if (ACT == kActSwiglu) pg[part_stride / 2 + (long long)r * ncols + n] = accu[i][j];
      }
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int r = row0 + ty * 4 + i;
    if (r >= row1 || r >= row0 + BM) continue;
    float o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float v = acc[i][j];
      if (ACT == kActRelu) v = fmaxf(v, 0.f);
      else if (ACT == kActSwiglu) v = (v / (1.f + expf(-v))) * accu[i][j];
      else v *= scale;
      o[j] = v;
    }
    int n = col0 + tx * 4;
    if (n + 3 < ncols) {
      *reinterpret_cast<float4*>(out + (long long)r * ncols + n) = make_float4(o[0], o[1], o[2], o[3]);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (n + j < ncols) out[(long long)r * ncols + n + j] = o[j];
    }
  }
}

// Adds the S k-slice partials of every routed row in slice order and applies
// the activation: out[r][n] = act(sum_z partial[z][r][n]).
template <int ACT>
__global__ void __launch_bounds__(256)
simt_splitk_reduce_kernel(const float* __restrict__ partial, long long part_stride, int S,
                          const int32_t* __restrict__ offsets, int E, int ncols, float scale,
                          float* __restrict__ out) {
  griddep_trigger();  // let the next kernel of the stream start launching
  griddep_wait();     // inputs written by the previous kernel are visible

  const long long nvalid = static_cast<long long>(offsets[E]) * ncols;  // rows of real experts
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < nvalid; i += 256ll * gridDim.x) {
    float g = 0.f, u = 0.f;
    for (int z = 0; z < S; ++z) {
      g += partial[z * part_stride + i];
      if (ACT == kActSwiglu) u += partial[z * part_stride + part_stride / 2 + i];
    }
    float v;
    if (ACT == kActRelu) v = fmaxf(g, 0.f);
    else if (ACT == kActSwiglu) v = (g / (1.f + expf(-g))) * u;
    else v = g * scale;
    out[i] = v;
  }
}

template <int ACT>
void launch_act(dim3 grid, const float* A, int kdim, const float* W, const float* W3, int ncols,
                float scale, const int32_t* offsets, int E, float* out, int kchunk, float* partial,
                long long part_stride, cudaStream_t stream) {
  launch_pdl(gemm_simt_f32_kernel<ACT>, grid, dim3(256), 0, stream, A, kdim, W, W3, ncols, scale,
             offsets, E, out, kchunk, partial, part_stride);
  if (partial != nullptr) {
    const long long n = static_cast<long long>(grid.y) * BM * ncols;  // upper bound of rows*cols
    const long long blocks = std::min<long long>((n + 255) / 256, 4LL * device_sm_count());
    launch_pdl(simt_splitk_reduce_kernel<ACT>, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
               stream, partial, part_stride, static_cast<int>(grid.z), offsets, E, ncols, scale, out);
  }
}

}  // namespace

int simt_f32_splits(int kdim, int ncols, int R, int E) {
  const long long ctas = static_cast<long long>((ncols + BN - 1) / BN) * ((R + BM - 1) / BM + E);
  int s = 1;
  // about two CTAs per SM, slices of at least 64 k, at most 8 slices
  while (s < 8 && ctas * s * 2 <= 2LL * device_sm_count() && kdim / (2 * s) >= 64) s *= 2;
  return s;
}

size_t simt_f32_partial_bytes(int kdim, int ncols, int R, int E, int act) {
  const int s = simt_f32_splits(kdim, ncols, R, E);
  if (s == 1) return 0;
  return static_cast<size_t>(s) * (act == kActSwiglu ? 2 : 1) * R * ncols * sizeof(float);
}

cudaError_t launch_gemm_simt_f32(const float* A, int kdim, const float* W, const float* W3,
                                 int ncols, int act, float scale, const int32_t* offsets, int E,
                                 int R, float* out, float* partial, cudaStream_t stream) {
  if (R == 0) return cudaSuccess;
  const int S = partial != nullptr ? simt_f32_splits(kdim, ncols, R, E) : 1;
  const int kchunk = S == 1 ? kdim : ((kdim + S - 1) / S + BK - 1) / BK * BK;
  const long long part_stride =
      static_cast<long long>(act == kActSwiglu ? 2 : 1) * R * ncols;
  float* part = S == 1 ? nullptr : partial;
  dim3 grid((ncols + BN - 1) / BN, (R + BM - 1) / BM + E, S);
  if (act == kActRelu)
    launch_act<kActRelu>(grid, A, kdim, W, W3, ncols, scale, offsets, E, out, kchunk, part, part_stride, stream);
  else if (act == kActSwiglu)
    launch_act<kActSwiglu>(grid, A, kdim, W, W3, ncols, scale, offsets, E, out, kchunk, part, part_stride, stream);
  else
    launch_act<kActNone>(grid, A, kdim, W, W3, ncols, scale, offsets, E, out, kchunk, part, part_stride, stream);
  return cudaGetLastError();
}

}  // namespace moe
