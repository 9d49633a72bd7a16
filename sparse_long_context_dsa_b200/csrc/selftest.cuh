// Self-test of the failure-detection path: a kernel whose mbarrier wait can never complete.
// Every mbarrier wait in the library's kernels is bounded and, when its bound runs out, sets
// the timeout bit of the per-device error word and lets the kernel return, so a logic error
// shows up as a status on the host instead of a hung GPU.  This kernel exercises exactly that
// path with a short bound chosen by the caller: one barrier is initialised for one arrival
// that nobody makes; one thread spins on it (mbar_wait) and one suspends on it
// (mbar_wait_sleep).  It issues no copy, no MMA and allocates no tensor memory, so nothing is
// in flight when it gives up.
#pragma once

#include "common.cuh"

namespace dsa {

__global__ void __launch_bounds__(64) wait_timeout_kernel(long long limit_cycles)
{
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    pdl_wait();
    // phase 0 of a fresh barrier completes only after one arrival: never, here
    if (threadIdx.x == 0) mbar_wait(&bar, 0, limit_cycles);
    if (threadIdx.x == 32) mbar_wait_sleep(&bar, 0, limit_cycles);
    __syncthreads();
}

}  // namespace dsa
