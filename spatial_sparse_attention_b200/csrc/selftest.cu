// Failure detection without a fault: every wait of the library's kernels on an mbarrier is
// bounded, and a wait that runs out records DEV_TIMEOUT in the plan's status word, which the host
// returns as SSA_ERR_DEVICE_TIMEOUT. ssa_debug_wait_timeout drives that path on purpose: one warp
// initialises an mbarrier that nothing ever arrives at and waits on it with the same bounded wait
// (tc::mbar_wait) the kernels use. No copy or tensor-core operation is in flight, so the kernel
// simply records the timeout and ends; the context stays usable.
#include "common.cuh"
#include "tc.cuh"

namespace ssa {

namespace {

__global__ void k_wait_timeout(int32_t* __restrict__ status, long long max_cycles) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1u);
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !tc::mbar_wait(&bar, 0u, max_cycles)) atomicOr(status, DEV_TIMEOUT);
}

}  // namespace

ssa_status_t launch_wait_timeout(Plan* p, int64_t max_cycles, cudaStream_t st) {
    k_wait_timeout<<<1, 32, 0, st>>>(p->d_status, (long long)max_cycles);
    note_launch();
    return cudaGetLastError() == cudaSuccess ? SSA_OK : SSA_ERR_CUDA;
}

}  // namespace ssa
