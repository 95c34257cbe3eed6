// moe_permute_noalloc: the permute stage for callers that cannot allocate
// device memory.  Such callers run inside a host framework that owns every
// device allocation and hands a kernel only its inputs and outputs (an
// operator plugin of an inference engine, for example), or sit on a
// latency-critical path where a cudaMalloc / cudaFree, which can synchronise
// the whole device, is not acceptable.  The per-chunk expert counts that
// moe_permute keeps in the caller's workspace live here in a file-scope
// device array instead; nothing is allocated by this entry point.
//
// The array is a module-scope __device__ variable: every GPU that loads the
// library holds its 1 MiB until the process exits.  Its host-side name is
// only a stand-in for the symbol, so every call looks the device address up
// with cudaGetSymbolAddress on the current device (a host-side query that
// allocates nothing; on a device's first call it also loads the module
// there).  Nothing is cached, so the address stays right after a
// cudaDeviceReset or a reload of the library.
#include <cuda_runtime.h>

#include "moe.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = size_t(1) << 20;

constexpr size_t kCounterBytes = 256;  // the counter, alone in the array's first 256 bytes

// First 256 bytes: the rank pass's last-CTA counter, which must be zero when
// a call starts.  A __device__ array starts zeroed when the module loads, and
// every call's last CTA sets the counter back to zero.  Then the per-block
// expert counts, and after the scan the per-block expert bases: every call
// writes all ceil(N/256)*E entries that it later reads, so these need no
// clearing.
static __device__ __align__(256) int32_t g_permute_scratch[kScratchBytes / sizeof(int32_t)];

// Device address of g_permute_scratch on the current device.
moe_status scratch_on_current_device(int32_t** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr) {
    cudaGetLastError();  // leave no sticky error behind for the caller
    return MOE_ERR_CUDA;
  }
  *out = static_cast<int32_t*>(p);
  return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" moe_status moe_permute_noalloc(moe_plan plan, const void* x, const int32_t* topk_ids,
                                          int32_t* counts, int32_t* offsets, int32_t* perm_pos,
                                          int32_t* perm_src, void* x_perm,
                                          int32_t* device_status_or_null, moe_stream_t stream) {
  int N = 0, d = 0, E = 0, K = 0, row_bytes = 0;
  if (!moe::plan_permute_shape(plan, &N, &d, &E, &K, &row_bytes)) return MOE_ERR_INVALID_ARG;
  if (!x || !topk_ids || !counts || !offsets || !perm_pos || !perm_src || !x_perm)
    return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(x_perm)) return MOE_ERR_INVALID_ARG;
  if (kCounterBytes + moe::permute_block_counts_bytes(N, E) > kScratchBytes)
    return MOE_ERR_WORKSPACE_TOO_SMALL;
  int32_t* scratch = nullptr;
  moe_status st = scratch_on_current_device(&scratch);
  if (st != MOE_OK) return st;
  cudaStream_t s = stream;
  int* status = device_status_or_null;
  // the same two kernels as moe_permute, recorded in the plan's launch count
  // and stage events like that call
  unsigned* counter = reinterpret_cast<unsigned*>(scratch);
  int32_t* block_counts = scratch + kCounterBytes / sizeof(int32_t);
  moe::plan_call_begin(plan);
  moe::plan_call_mark(plan, s, "permute_rank");
  bool ok = moe::launch_permute_rank(topk_ids, N, K, E, block_counts, counter, perm_pos, counts,
                                     offsets, status, s) == cudaSuccess;
  moe::plan_call_mark(plan, s, "permute_gather");
  ok = ok && moe::launch_permute_gather(x, row_bytes, topk_ids, N, K, E, block_counts, perm_pos,
                                        perm_src, nullptr, x_perm, status, s) == cudaSuccess;
  moe::plan_call_end(plan, s, 2);
  return ok ? MOE_OK : MOE_ERR_CUDA;
}
