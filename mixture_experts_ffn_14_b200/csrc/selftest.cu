// selftest.cu — a check of the library's failure path that faults nothing:
// one thread waits, with the same bounded mbarrier wait the GEMM pipelines use,
// on a barrier that nothing arrives on. The wait gives up after the given limit,
// the kernel records kStatusSelftestTimeout in the status word and returns, so
// the context stays usable and moe_device_status() reports the failure.
#include <cuda_runtime.h>

#include <cstdint>

#include "moe_internal.cuh"
#include "sm100.cuh"

namespace moe {
namespace {

__global__ void moe_selftest_wait_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  sm100::mbar_init(&bar, 1);
  sm100::fence_mbar_init();
  // Phase 0 never completes: nobody arrives.
  if (!sm100::mbar_wait(&bar, 0, limit_ns)) atomicOr(status, kStatusSelftestTimeout);
}

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_selftest_bounded_wait(void* workspace, uint32_t limit_us, moe_stream_t stream) {
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MOE_ERR_WORKSPACE;
  if (limit_us == 0 || limit_us > 10000000u) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(uint32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  moe::moe_selftest_wait_kernel<<<1, 32, 0, s>>>(status, static_cast<uint64_t>(limit_us) * 1000u);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
