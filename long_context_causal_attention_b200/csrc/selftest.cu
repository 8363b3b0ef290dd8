// Self-test of the failure path every tensor-core kernel relies on: a
// bounded mbarrier wait that runs out raises the CTA's abort flag and leaves
// LWM_ERR_TIMEOUT (with the wait's tag) in the workspace status word, and the
// kernel returns normally, so the CUDA context stays usable.  No counterpart
// on the pages; it lets a test make a wait run out on purpose (a barrier
// nothing arrives on) without faulting or hanging the GPU.
#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"

namespace lwm {
namespace {

constexpr int kSelftestTag = 99;

__global__ void selftest_wait_kernel(DeviceStatus* status, long long limit_cycles, int arrive) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    sm100::mbar_init(smem_u32(&bar), 1);
    sm100::fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && arrive) sm100::mbar_arrive(smem_u32(&bar));
  __syncthreads();
  const sm100::Abort ab{&abort_flag, status};
  if (threadIdx.x == 0) sm100::mbar_wait_limit(smem_u32(&bar), 0, ab, kSelftestTag, limit_cycles);
}

}  // namespace

cudaError_t launch_selftest_wait(DeviceStatus* status, long long limit_cycles, int arrive,
                                 cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(DeviceStatus), st);
  if (e != cudaSuccess) return e;
  selftest_wait_kernel<<<1, 32, 0, st>>>(status, limit_cycles, arrive);
  note_launches(1);
  return cudaGetLastError();
}

}  // namespace lwm
