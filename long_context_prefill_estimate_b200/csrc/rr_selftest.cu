// Self-test of the bounded mbarrier wait that every kernel of the library uses instead of an
// unbounded spin: a wait on a phase that nothing completes must give up after its limit and
// leave the GPU usable, and a completed phase must still be seen.
#include "rr_common.cuh"
#include "rr_sm100.cuh"

namespace rr {

namespace {

__device__ uint32_t g_selftest[3];

__global__ void wait_timeout_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    const uint32_t b = smem_u32(&bar);
    sm100::mbar_init(b, 1);
    sm100::fence_mbar_init();
    const uint64_t t0 = sm100::globaltimer();
    const bool first = sm100::mbar_wait(b, 0, limit_ns);  // nothing arrives: must give up
    const uint64_t t1 = sm100::globaltimer();
    sm100::mbar_arrive(b);                                 // complete phase 0 ourselves
    const bool second = sm100::mbar_wait(b, 0, limit_ns);  // must see it
    g_selftest[0] = first ? 0u : 1u;
    g_selftest[1] = second ? 1u : 0u;
    g_selftest[2] = (uint32_t)((t1 - t0) / 1000u);
}

}  // namespace

rr_status_t selftest_wait(uint32_t timeout_us, uint32_t *result) {
    const uint32_t zero[3] = {0, 0, 0};
    cudaError_t e = cudaMemcpyToSymbol(g_selftest, zero, sizeof(zero));
    if (e == cudaSuccess) {
        wait_timeout_kernel<<<1, 32>>>((uint64_t)timeout_us * 1000u);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) e = cudaMemcpyFromSymbol(result, g_selftest, sizeof(zero));
    if (e != cudaSuccess) return set_error(RR_ERR_CUDA, "rr_selftest_wait: %s", cudaGetErrorString(e));
    return RR_OK;
}

}  // namespace rr
