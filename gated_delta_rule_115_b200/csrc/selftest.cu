// selftest.cu -- self-test of the bounded device waits.  The chunk kernels
// wait on shared-memory barriers (mbarrier) with a time limit; a wait that
// runs out is recorded and the kernel finishes instead of hanging the GPU.
// This kernel makes one such wait run out on purpose, on a barrier nothing
// arrives on and with no copy or tensor-core operation in flight, so the
// recording path can be tested without a fault.
#include <cuda_runtime.h>
#include <stdint.h>

#include "profile.h"
#include "tc2.cuh"

namespace muir {

__device__ unsigned int g_selftest_timeouts;

namespace {

__global__ void k_expired_wait(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        t2::mbar_init(&bar, 1);  // one arrival expected; none is ever made
        t2::fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !t2::mbar_wait(&bar, 0, limit_ns)) atomicAdd(&g_selftest_timeouts, 1u);
}

}  // namespace

cudaError_t launch_expired_wait(int limit_us, cudaStream_t st) {
    MUIR_TIMED("k_expired_wait", st, k_expired_wait<<<1, 32, 0, st>>>((uint64_t)limit_us * 1000u));
    return cudaGetLastError();
}

unsigned int timeouts_selftest() {
    unsigned int n = 0;
    cudaMemcpyFromSymbol(&n, g_selftest_timeouts, sizeof(n));
    const unsigned int z = 0;
    cudaMemcpyToSymbol(g_selftest_timeouts, &z, sizeof(z));
    return n;
}

}  // namespace muir
