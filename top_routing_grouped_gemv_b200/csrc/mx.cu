// MX block scales: from the row-major E8M0 scale matrices the caller holds
// to the 512-byte atoms the block-scaled grouped GEMM reads (layout in
// kernels.h), and the row gather of scales that goes with the permute; the
// transposition of fp32 group / block weight scales for the group-scaled
// GEMM (quant modes 4 and 5).
//
// Quant mode 6 ("mx") of the Ascend grouped-matmul page
// ("aclnnQuantGroupedMatMulAlltoAllv", parameter section, quant-mode
// enumeration), read as OCP MXFP8: one E8M0 scale per 32 consecutive
// elements of a row along the reduction dimension.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr uint32_t kUnitScales = 0x7F7F7F7Fu;  // four scales of 1.0

__device__ __forceinline__ int atom_offset(int i) { return (i & 31) * 16 + (i >> 5) * 4; }

// Four scales of K stage kb of one row: bytes [4 kb, 4 kb + 4) of the row,
// 127 past its end.
__device__ __forceinline__ uint32_t stage_scales(const uint8_t* row, int nsf, int kb) {
  uint32_t v = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int s = 4 * kb + j;
    const uint32_t b = s < nsf ? row[s] : 0x7Fu;
    v |= b << (8 * j);
  }
  return v;
}

// One thread per (weight row slot, K stage): grid covers
// groups * n_tiles * 256 rows x num_kb stages.
__global__ void mx_weight_sf_kernel(const uint8_t* __restrict__ w_sf, int groups, int n_out,
                                    int kdim, uint8_t* __restrict__ out) {
  const int nsf = kdim / kMxBlock;
  const int num_kb = mx_num_kb(kdim);
  const int n_tiles = (n_out + kTcBlockN - 1) / kTcBlockN;
  const long long total = static_cast<long long>(groups) * n_tiles * kTcBlockN * num_kb;
  for (long long t = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int kb = static_cast<int>(t % num_kb);
    const long long rs = t / num_kb;          // (g, nt, row in 256)
    const int r256 = static_cast<int>(rs % kTcBlockN);
    const long long gt = rs / kTcBlockN;      // g * n_tiles + nt
    const int nt = static_cast<int>(gt % n_tiles);
    const int g = static_cast<int>(gt / n_tiles);
    const int n = nt * kTcBlockN + r256;
    const uint32_t v = n < n_out
                           ? stage_scales(w_sf + (static_cast<long long>(g) * n_out + n) * nsf, nsf, kb)
                           : kUnitScales;
    const int h = r256 >> 7, i = r256 & 127;
    uint8_t* atom = out + ((gt * num_kb + kb) * 2 + h) * kMxAtomBytes;
    *reinterpret_cast<uint32_t*>(atom + atom_offset(i)) = v;
  }
}

// Per-group padded tile prefix (tiles of 128 rows) in shared memory: tp[g] =
// sum over g' < g of ceil(rows of g' / 128).  One warp; G <= 256.
__device__ void tile_prefix(const int32_t* offsets, int G, int* s_off, int* s_tp) {
  const int lane = threadIdx.x & 31;
  const int per = (G + 31) / 32;
  const int b0 = min(G, lane * per), b1 = min(G, b0 + per);
  int local = 0;
  for (int q = b0; q < b1; ++q) {
    const int o0 = offsets[q], o1 = offsets[q + 1];
    s_off[q] = o0;
    const int t = (max(0, o1 - o0) + kTcBlockM - 1) / kTcBlockM;
    s_tp[q] = t;
    local += t;
  }
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  int run = incl - local;
  for (int q = b0; q < b1; ++q) {
    const int t = s_tp[q];
    s_tp[q] = run;
    run += t;
  }
  if (lane == 31) {
    s_tp[G] = incl;
    s_off[G] = offsets[G];
  }
}

// One block per padded 128-row tile: the scale rows of the tile's permuted
// rows are gathered into shared memory, then the tile's num_kb atoms (one
// contiguous region) are written with 16-byte stores.  Rows past the
// group's end and scales past the end of K get 127.
constexpr int kActThreads = 256;

__global__ void __launch_bounds__(kActThreads) mx_act_sf_kernel(
    const uint8_t* __restrict__ x_sf, const int32_t* __restrict__ src,
    const int32_t* __restrict__ offsets, int G, int kdim, uint8_t* __restrict__ out) {
  extern __shared__ uint8_t s_rows[];  // (128, row_bytes): the tile's scale rows
  __shared__ int s_off[257], s_tp[257];
  griddep_trigger();
  griddep_wait();
  if (threadIdx.x < 32) tile_prefix(offsets, G, s_off, s_tp);
  __syncthreads();
  const int pt = blockIdx.x;
  if (pt >= s_tp[G]) return;
  int lo = 0, hi = G - 1;  // the group owning padded tile pt: last g with s_tp[g] <= pt
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_tp[mid] <= pt) lo = mid; else hi = mid - 1;
  }
  const int r0 = s_off[lo] + (pt - s_tp[lo]) * kTcBlockM;  // first permuted row of the tile
  const int nrow = min(kTcBlockM, s_off[lo + 1] - r0);
  const int nsf = kdim / kMxBlock;
  const int num_kb = mx_num_kb(kdim);
  const int row_bytes = num_kb * 4;
  // gather: row i of the tile <- scale row src[r0 + i] (127 past the end)
  if (nsf % 16 == 0 && (reinterpret_cast<uintptr_t>(x_sf) & 15) == 0) {
    // rows of whole, aligned 16-byte chunks (row_bytes == nsf): unrolled vector loads
    const int vpr = nsf / 16;
    const uint4 unit = make_uint4(kUnitScales, kUnitScales, kUnitScales, kUnitScales);
#pragma unroll 8
    for (int t = threadIdx.x; t < kTcBlockM * vpr; t += kActThreads) {
      const int i = t / vpr, v = t - i * vpr;
      uint4 val = unit;
      if (i < nrow) {
        const long long sr = src ? src[r0 + i] : r0 + i;
        val = reinterpret_cast<const uint4*>(x_sf + sr * nsf)[v];
      }
      reinterpret_cast<uint4*>(s_rows)[t] = val;
    }
  } else {
#pragma unroll 8
    for (int t = threadIdx.x; t < kTcBlockM * row_bytes; t += kActThreads) {
      const int i = t / row_bytes, b = t - i * row_bytes;
      uint8_t v = 0x7F;
      if (i < nrow && b < nsf) {
        const long long sr = src ? src[r0 + i] : r0 + i;
        v = x_sf[sr * nsf + b];
      }
      s_rows[t] = v;
    }
  }
  __syncthreads();
  // atoms: line m of atom kb = scales 4kb..4kb+3 of rows m, m+32, m+64, m+96
  uint4* dst = reinterpret_cast<uint4*>(out + static_cast<long long>(pt) * num_kb * kMxAtomBytes);
  for (int t = threadIdx.x; t < num_kb * 32; t += kActThreads) {
    const int kb = t >> 5, m = t & 31;
    uint32_t w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      w[q] = *reinterpret_cast<const uint32_t*>(s_rows + (m + 32 * q) * row_bytes + 4 * kb);
    dst[t] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// One thread per (row, scale byte).
__global__ void mx_sf_gather_kernel(const uint8_t* __restrict__ x_sf, const int32_t* __restrict__ src,
                                    const int32_t* __restrict__ offsets, int G, int rows_upper,
                                    int nsf, uint8_t* __restrict__ out) {
  griddep_trigger();
  griddep_wait();
  const int rows = min(offsets[G], rows_upper);
  const long long total = static_cast<long long>(rows) * nsf;
  for (long long t = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>(t % nsf);
    const long long r = t / nsf;
    out[t] = x_sf[static_cast<long long>(src[r]) * nsf + j];
  }
}

__global__ void group_scales_t_kernel(const float* __restrict__ src, int groups, int rows, int ng,
                                      float* __restrict__ dst) {
  const long long total = static_cast<long long>(groups) * rows * ng;
  for (long long t = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; t < total;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int n = static_cast<int>(t % rows);          // destination order: (g, kb, n)
    const long long gk = t / rows;
    const int kb = static_cast<int>(gk % ng);
    const long long g = gk / ng;
    dst[t] = src[(g * rows + n) * ng + kb];
  }
}

int grid_for(long long work, int threads) {
  const long long b = (work + threads - 1) / threads;
  const long long cap = 8LL * device_sm_count();
  return static_cast<int>(b < 1 ? 1 : (b > cap ? cap : b));
}

}  // namespace

cudaError_t launch_mx_weight_sf(const uint8_t* w_sf, int groups, int n_out, int kdim, uint8_t* out,
                                cudaStream_t stream) {
  if (groups < 1 || n_out < 1 || kdim < kMxBlock || kdim % kMxBlock) return cudaErrorInvalidValue;
  const long long work = static_cast<long long>(groups) * ((n_out + kTcBlockN - 1) / kTcBlockN) *
                         kTcBlockN * mx_num_kb(kdim);
  mx_weight_sf_kernel<<<grid_for(work, 256), 256, 0, stream>>>(w_sf, groups, n_out, kdim, out);
  return cudaGetLastError();
}

cudaError_t launch_group_scales_t(const float* src, int groups, int rows, int ng, float* dst,
                                  cudaStream_t stream) {
  if (groups < 1 || rows < 1 || ng < 1) return cudaErrorInvalidValue;
  const long long work = static_cast<long long>(groups) * rows * ng;
  group_scales_t_kernel<<<grid_for(work, 256), 256, 0, stream>>>(src, groups, rows, ng, dst);
  return cudaGetLastError();
}

cudaError_t launch_mx_act_sf(const uint8_t* x_sf, const int32_t* src_rows, const int32_t* offsets,
                             int groups, int rows_upper, int kdim, uint8_t* out,
                             cudaStream_t stream) {
  if (groups < 1 || groups > 256 || kdim < kMxBlock || kdim % kMxBlock || kdim > kMxMaxKdim)
    return cudaErrorInvalidValue;
  if (rows_upper <= 0) return cudaSuccess;
  // one block per padded tile; at most rows_upper / 128 + groups tiles exist
  const int tiles = rows_upper / kTcBlockM + groups;
  const size_t smem = static_cast<size_t>(kTcBlockM) * mx_num_kb(kdim) * 4;
  // the shared-memory opt-in is a per-device function attribute
  static bool configured[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(mx_act_sf_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kTcBlockM * mx_num_kb(kMxMaxKdim) * 4);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  return launch_pdl(mx_act_sf_kernel, dim3(tiles), dim3(kActThreads), smem, stream, x_sf, src_rows,
                    offsets, groups, kdim, out);
}

cudaError_t launch_mx_sf_gather(const uint8_t* x_sf, const int32_t* src_rows,
                                const int32_t* offsets, int groups, int rows_upper, int nsf,
                                uint8_t* out, cudaStream_t stream) {
  if (groups < 1 || nsf < 1 || !src_rows) return cudaErrorInvalidValue;
  if (rows_upper <= 0) return cudaSuccess;
  const long long work = static_cast<long long>(rows_upper) * nsf;
  return launch_pdl(mx_sf_gather_kernel, dim3(grid_for(work, 256)), dim3(256), 0, stream, x_sf,
                    src_rows, offsets, groups, rows_upper, nsf, out);
}

}  // namespace moe
