// Diagnostic kernel for the bounded waits: one CTA allocates TMEM, then two warps wait on an
// mbarrier that nothing arrives at.  The first to pass ``timeout_ns`` raises the CTA's abort
// flag and STARKV_DEV_TIMEOUT; the other sees the flag and gives up; the CTA frees TMEM and
// returns.  This is the same wait/abort/teardown code the pipelines use, driven to expiry
// without any fault.
#include "internal.cuh"

namespace starkv {
namespace {

__global__ void __launch_bounds__(64) bounded_wait_kernel(int* status, unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t misc[2];  // [0] TMEM base, [1] abort flag
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    misc[1] = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(misc), 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  WaitCtl wc{reinterpret_cast<volatile int*>(misc + 1), status, timeout_ns};
  // warp 1 waits with the timeout; warp 0 with ten times more, so it only returns through
  // the abort flag that warp 1 raises
  WaitCtl w = wc;
  if (warp == 0) w.timeout_ns = timeout_ns * 10;
  const bool ok = __all_sync(0xffffffffu, wait_bounded(smem_u32(&bar), 0, w));
  (void)ok;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(misc[0], 32);
}

}  // namespace

cudaError_t launch_bounded_wait(int* status, unsigned long long timeout_ns, cudaStream_t s) {
  bounded_wait_kernel<<<1, 64, 0, s>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace starkv
