// Failure-path check without a fault: one thread waits, through the same
// bounded mbarrier wait every tensor-core kernel uses, on a barrier that
// nothing arrives at.  After the wait's limit (~2 s of SM clocks) it sets the
// CTA's abort flag and the library's device error word and returns, so the
// host sees FSDIT_E_TIMEOUT from fsdit_device_error() and the context stays
// usable.
#include "tc_ptx.cuh"

namespace fsdit {

__global__ void bounded_wait_check_kernel(int* __restrict__ result) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  abort_flag = 0;
  const uint32_t b = ptx::smem_u32(&bar);
  ptx::mbar_init(b, 1);
  ptx::fence_mbar_init();
  // phase 0 of a fresh barrier completes only when one arrival lands: none does
  const bool completed = ptx::mbar_wait(b, 0, reinterpret_cast<volatile int*>(&abort_flag));
  result[0] = completed ? 1 : 0;
  result[1] = abort_flag;
}

}  // namespace fsdit

extern "C" fsdit_status fsdit_check_bounded_wait(int* result, fsdit_stream_t stream) {
  using namespace fsdit;
  if (result == nullptr) {
    set_error("check_bounded_wait: result (device, int[2]) is required");
    return FSDIT_E_NULL;
  }
  bounded_wait_check_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(result);
  return cuda_check(cudaGetLastError(), "bounded_wait_check_kernel");
}
