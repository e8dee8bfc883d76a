// A self-test of the bounded waits: a kernel whose wait can never succeed must give up, report
// SEMKV_STATUS_TIMEOUT in the device status word and leave the device usable.
//
// Every wait in the library's kernels (copies landing, tensor-core products finishing) is bounded
// (mbar_wait gives up after a fixed number of tests) and a kernel that gives up still frees its
// tensor memory and returns with the status bit set.  Those waits cannot be made to fail on
// purpose without breaking a copy or a product, so this kernel exercises the same path on a wait
// that nothing completes: one thread arrives on an mbarrier that expects two arrivals and then
// waits for the phase with a short test bound; optionally the warp holds tensor memory meanwhile
// and frees it after the wait, as the decode kernels do.  No memory access is out of bounds and
// no wait is unbounded.
#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace semkv {
namespace {

__global__ void __launch_bounds__(32) k_selftest_wait_timeout(int32_t* status, uint32_t tests, int use_tmem)
{
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_slot;
    if (use_tmem) {
        tmem_alloc(&tmem_slot, 32);
        tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        mbar_init(&bar, 2);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    bool ok = true;
    if (threadIdx.x == 0) {
        mbar_arrive(&bar);                 // the second arrival never comes
        ok = mbar_wait(&bar, 0u, tests);   // so this gives up after `tests` tests
    }
    tc_fence_before();
    __syncthreads();
    if (use_tmem) {
        tc_fence_after();
        tmem_dealloc(tmem_slot, 32);
    }
    if (!ok) atomicOr(status, SEMKV_STATUS_TIMEOUT);
}

}  // namespace
}  // namespace semkv

extern "C" int semkv_selftest_wait_timeout(int32_t* status, int32_t tests, int32_t use_tmem, void* stream)
{
    if (!status || tests < 1 || tests > (1 << 16) || (use_tmem != 0 && use_tmem != 1)) return SEMKV_ERR_INVALID_ARG;
    semkv::k_selftest_wait_timeout<<<1, 32, 0, (cudaStream_t)stream>>>(status, (uint32_t)tests, use_tmem);
    if (cudaGetLastError() != cudaSuccess) return SEMKV_ERR_CUDA;
    return SEMKV_OK;
}
