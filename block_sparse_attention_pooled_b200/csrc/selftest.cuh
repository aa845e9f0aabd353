// Self-test of the bounded device waits that every kernel of the library
// uses. One CTA of 128 threads sets up what the real kernels set up (an
// mbarrier, an abort flag shared by the roles, 32 TMEM columns owned by
// warp 0), then all four warps wait on the barrier, which nothing ever
// arrives on, through the same role_wait the kernels use, with a limit of a
// few milliseconds. The first warp to give up records kErrSelfTest in the
// device error word and raises the abort flag; the others see the flag and
// stop waiting. Warp 0 then frees its TMEM and the kernel returns, so the
// context stays usable and the host reads the site code through
// sparge_device_status.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace sparge {

enum : unsigned int { kErrSelfTest = 0xF00 };

__global__ void __launch_bounds__(128) selftest_wait_kernel(unsigned long long limit_ns, int* waited_out) {
  __shared__ __align__(8) unsigned long long bar_storage;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const int warp = threadIdx.x / 32;
  const uint32_t bar = smem_u32(&bar_storage);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&tmem_slot), 32);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  // Nothing arrives on `bar`: every role gives up, the first after limit_ns.
  const bool got = role_wait(bar, 0, kErrSelfTest, &abort_flag, limit_ns);
  const bool all_gave_up = __syncthreads_and(!got);
  if (threadIdx.x == 0 && waited_out != nullptr) *waited_out = all_gave_up ? 1 : 0;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 32);
  }
}

}  // namespace sparge
