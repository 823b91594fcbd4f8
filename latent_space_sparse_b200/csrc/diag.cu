// diag.cu -- a check of the failure path every pipeline wait of the decode
// kernels shares: a bounded wait on an mbarrier phase that never completes
// gives up after its limit, records FLAG_WAIT_TIMEOUT in the workspace's
// anomaly word and returns, so that the kernel ends and the context stays
// usable.  Nothing is copied and nothing else runs while the wait spins.
#include "tc.cuh"

namespace salsc {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_kernel(uint32_t* flags, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = tc::smem_u32(&bar);
  if (threadIdx.x == 0) {
    tc::mbar_init(b, 1);  // one arrival expected; none is ever made
    tc::mbar_fence_init();
  }
  __syncwarp();
  // the same bounded wait as the decode pipelines, with the caller's limit
  const bool ok = tc::mbar_wait_limit(b, 0u, threadIdx.x == 0 ? flags : nullptr, limit_ns);
  (void)ok;
}

}  // namespace
}  // namespace salsc

extern "C" salsc_status salsc_check_wait_timeout(uint64_t limit_ns, void* ws, size_t ws_bytes,
                                                 salsc_stream stream) {
  if (limit_ns == 0 || limit_ns > 1000000000ull) return SALSC_ERR_INVALID_ARG;
  if (!ws || ((uintptr_t)ws % salsc::kWsAlign) != 0 || ws_bytes < 16) return SALSC_ERR_WORKSPACE;
  salsc::wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint32_t*)ws, limit_ns);
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? SALSC_OK : salsc::record_cuda_error(e);
}
