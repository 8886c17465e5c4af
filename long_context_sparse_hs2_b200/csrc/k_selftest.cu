// Self-test of the bounded waits (failure detection without a GPU fault).
//
// Every pipeline wait in the library's kernels (mbarrier phases of the TMA rings, the tensor-core
// hand-offs, the decode tail's logit stream) gives up after a bound, flags HS2_DEV_TIMEOUT in the
// workspace status word and lets the kernel return, so a pipeline that stalls leaves an error the
// host can read instead of a hung GPU.  This kernel runs exactly that wait on an mbarrier nothing
// ever arrives on, with a short bound, so a test can watch the bound run out and the context stay
// usable.
#include "hs2_device.cuh"

namespace hs2 {

namespace {

__global__ void __launch_bounds__(32) wait_bound_kernel(unsigned* status, uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncwarp();
    const bool completed = mbar_wait(&bar, 0, status, limit_ns);  // no arrival: runs out after limit_ns
    __syncwarp();
    if (threadIdx.x == 0) {
        if (completed) set_status(status, HS2_DEV_BAD_INDEX);  // cannot happen: nothing arrived
        mbar_inval(&bar);
    }
}

}  // namespace

}  // namespace hs2

using namespace hs2;

extern "C" hs2_status hs2_selftest_wait_bound(void* ws, size_t ws_bytes, uint64_t limit_ns, void* stream) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) % 256) != 0 || ws_bytes < 256) return HS2_ERR_WORKSPACE;
    if (limit_ns < 1000 || limit_ns > kWaitLimitNs) return HS2_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    trace_call_begin(st);
    if (launch_init(ws, 256, st) != cudaSuccess) return HS2_ERR_CUDA;
    wait_bound_kernel<<<1, 32, 0, st>>>(static_cast<unsigned*>(ws), limit_ns);
    trace_mark("wait_bound_selftest", st);
    return cudaGetLastError() == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
}
