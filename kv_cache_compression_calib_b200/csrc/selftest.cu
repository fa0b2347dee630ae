// Self-test of the bounded wait the staged kernels use on their copy barriers.
//
// One warp initialises a barrier that expects one arrival, never arrives on
// it, and waits on it with mbar_wait and the caller's limit - the same wait,
// running out the same way as when a staged copy never lands.  The warp then
// sets TRI_FLAG_STAGE_TIMEOUT in the workspace flag word and returns: nothing
// is in flight, so the context stays usable.  No fault is involved.
#include "stage.cuh"

namespace tri {

__global__ void __launch_bounds__(32) wait_selftest_kernel(unsigned *flags, unsigned long long limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_init_fence();
    }
    __syncwarp();
    const bool landed = __all_sync(0xffffffffu, mbar_wait(&bar, 0u, limit_ns));
    if (!landed && threadIdx.x == 0) atomicOr(flags, TRI_FLAG_STAGE_TIMEOUT);
}

}  // namespace tri

extern "C" tri_status tri_selftest_wait_timeout(void *ws, size_t ws_bytes, uint64_t limit_ns, tri_stream_t stream) {
    if (!ws || ws_bytes < 256) return ws ? TRI_ERR_WORKSPACE_TOO_SMALL : TRI_ERR_INVALID_ARG;
    if ((uintptr_t)ws % 256) return TRI_ERR_ALIGNMENT;
    if (limit_ns < 1000ull || limit_ns > 10000000000ull) return TRI_ERR_INVALID_ARG;
    tri::wait_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((unsigned *)ws, (unsigned long long)limit_ns);
    return cudaGetLastError() == cudaSuccess ? TRI_OK : TRI_ERR_CUDA;
}
