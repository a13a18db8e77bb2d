// sol_selftest.cu -- sol_selftest_wait_timeout: exercises the failure path of the bounded
// waits on the device without any fault.
//
// Every libsol kernel that waits on an mbarrier (for its own bulk copies, or between the
// roles of the linear-layer kernels) bounds the wait, and on give-up records a bit in a
// device error word that sol_device_errors reads, and returns; the context stays usable.
// This entry point runs that path on purpose: one CTA initialises an mbarrier that expects
// two arrivals, arrives once, so its phase can never complete, waits on it with the same
// bounded helper (mbar_wait_bounded) for `polls` polls -- each suspends for at most about a
// millisecond -- and, when the wait gives up, records bit 2 of the device error flags.
#include "common.cuh"
#include "launch.h"
#include "sol.h"

namespace sol {

static __device__ unsigned int g_selftest_error;

__global__ void k_selftest_wait_timeout(uint32_t polls)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(smem_u32(&bar), 2);
    mbar_fence_init();
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(&bar)) : "memory");
    if (!mbar_wait_bounded(smem_u32(&bar), 0, polls)) atomicOr(&g_selftest_error, 4u);
}

uint32_t selftest_device_error(bool clear)
{
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_selftest_error, sizeof v) != cudaSuccess) return 0xffffffffu;
    if (clear && v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_selftest_error, &zero, sizeof zero);
    }
    return v;
}

}  // namespace sol

extern "C" sol_status sol_selftest_wait_timeout(int32_t polls, sol_stream_t stream)
{
    if (polls < 1 || polls > 1000) {
        sol::record_error("polls must be in [1, 1000]");
        return SOL_ERR_INVALID_ARGUMENT;
    }
    sol::k_selftest_wait_timeout<<<1, 32, 0, (cudaStream_t)stream>>>((uint32_t)polls);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        sol::record_error(cudaGetErrorString(e));
        return SOL_ERR_CUDA;
    }
    return SOL_OK;
}
