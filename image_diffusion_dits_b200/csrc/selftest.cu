// rf2_selftest_wait_timeout: a device-side check of the bounded waits every kernel of the
// library relies on, without provoking a fault.  Two one-warp CTAs each wait, through the
// same bounded mbarrier wait the kernels use, on a barrier that nothing ever arrives at:
// CTA 0 gives up after the short limit and raises RF2_ERR_TIMEOUT in the status word;
// CTA 1 (long limit) gives up as soon as it sees that word, as the CTAs of a kernel do
// when one of them times out.  Both waits end by the clock, so the launch always ends.
#include "rf2_common.cuh"
#include "sm100_ptx.cuh"

namespace {

__global__ void wait_timeout_kernel(int* status, unsigned long long short_ns, unsigned long long long_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_s;
  if (threadIdx.x == 0) {
    const uint32_t b = rf2::ptx::smem_u32(&bar);
    rf2::ptx::mbar_init(b, 1);
    abort_s = 0;
    rf2::ptx::fence_mbar_init();
    rf2::ptx::mbar_wait(b, 0, &abort_s, status, blockIdx.x == 0 ? short_ns : long_ns, rf2::kStatusTimeout);
  }
}

}  // namespace

extern "C" int rf2_selftest_wait_timeout(int32_t* status, double short_s, double long_s, void* stream) {
  if (status == nullptr || ((uintptr_t)status & 3u)) return RF2_ERR_INVALID_ARG;
  if (!(short_s > 0.0 && short_s <= long_s && long_s <= 5.0)) return RF2_ERR_INVALID_ARG;
  wait_timeout_kernel<<<2, 32, 0, (cudaStream_t)stream>>>(status, (unsigned long long)(short_s * 1e9),
                                                          (unsigned long long)(long_s * 1e9));
  return cudaGetLastError() == cudaSuccess ? RF2_OK : RF2_ERR_CUDA;
}
