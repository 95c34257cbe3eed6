// Self-test of the device-side failure path: the bounded mbarrier wait that
// every tensor-core kernel uses gives up after its limit, raises the CTA's
// abort flag so the other waiting roles leave too, and records
// MOE_ERR_DEVICE_TIMEOUT in the workspace status word -- without a trap,
// a fault or a hang, so the context stays usable.
#include "common.cuh"
#include "kernels.h"
#include "moe.h"
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace tc;

// One CTA, two warps.  Warp 0 waits with the short limit on a barrier that
// nothing arrives at; warp 1 waits on the same barrier with the default
// (long) limit and must leave through the abort flag that warp 0 raises.
__global__ void __launch_bounds__(64) wait_timeout_kernel(int* status, uint64_t limit_ns,
                                                          int* leave_order) {
  griddep_trigger();
  griddep_wait();
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag, order;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);  // expects one arrival that never comes
    abort_flag = 0;
    order = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  bool ok = true;
  if (lane == 0) {
    ok = warp == 0 ? mbar_wait(smem_u32(&bar), 0, &abort_flag, limit_ns)
                   : mbar_wait(smem_u32(&bar), 0, &abort_flag);
    if (!ok && leave_order != nullptr) leave_order[warp] = atomicAdd(&order, 1);
    if (!ok && warp == 0) set_status(status, kStatusTimeout);
  }
  __syncthreads();
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_selftest_wait_timeout(void* ws, size_t ws_bytes, int32_t limit_us,
                                                int32_t* leave_order_or_null, moe_stream_t stream) {
  if (!ws || ws_bytes < 4 || limit_us < 1 || limit_us > 1000000) return MOE_ERR_INVALID_ARG;
  cudaError_t e = moe::launch_pdl(moe::wait_timeout_kernel, dim3(1), dim3(64), 0, stream,
                                  static_cast<int*>(ws), static_cast<uint64_t>(limit_us) * 1000ull,
                                  leave_order_or_null);
  if (e == cudaSuccess) e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
