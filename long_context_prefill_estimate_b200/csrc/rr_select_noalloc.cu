// rr_select_noalloc: the Top-tau selection of rr_select for callers that cannot allocate
// device memory.
//
// Some callers have no way to hand this library a workspace: a plugin inside a host
// application whose own allocator owns every byte of device memory and gives plugins no
// allocation hook, or a latency-critical path that must never call cudaMalloc/cudaFree
// because those calls can synchronise the whole device.  For them the per-row counts and
// selection bitmaps that rr_select keeps in its caller-provided workspace live instead in a
// fixed array compiled into this library (kNoAllocScratchBytes = 8 MiB, enough for 32 heads
// x 1024 blocks, i.e. a 128K-token layer at B = 128).  Every GPU that loads the library keeps
// that array for the life of the process.
//
// Set-up: the first call on a device, with that device current, looks up the array's device
// address with cudaGetSymbolAddress (a host-side name of a __device__ array is only a stand-in,
// never a usable device pointer) and caches it for that device.  Make that first call on each
// device before any stream capture begins.  Only a successful lookup is cached: a failed one
// returns RR_ERR_CUDA and the next call on that device tries again.
//
// Sharing: all calls on a device use the same array and it keeps whatever the last call left.
// Every word a call reads is first written by the same call (each row writes its count and all
// of its bitmap words), so nothing needs clearing.  Calls that overlap on the GPU (different
// streams, or different host threads, without ordering between them) race on the array; order
// them on one stream or with events.
#include <mutex>

#include "rr_common.cuh"

namespace rr {
size_t select_workspace_bytes(int H, int Nb);
rr_status_t launch_select(const float *A, int H, int Nb, double tau, int protect_last,
                          int32_t *row_ptr, int32_t *col_idx, int64_t *nnz_out, void *ws,
                          cudaStream_t st);
}  // namespace rr

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mutex;
void *g_scratch_addr[kMaxDevices];  // the array's device address per device, once looked up

// Device address of the scratch array on the current device `dev` (cached after the first
// successful lookup), or the CUDA error of the lookup.
cudaError_t scratch_address(int dev, void **addr) {
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_select_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

using namespace rr;

extern "C" rr_status_t rr_select_noalloc(const float *block_scores, int H, int Nb, double tau,
                                         int protect_last, int32_t *row_ptr, int32_t *col_idx,
                                         int64_t col_capacity, int64_t *nnz_out,
                                         rr_stream_t stream) {
    static const char *fn = "rr_select_noalloc";
    clear_error();
    const rr_status_t st = check_select_args(fn, block_scores, H, Nb, tau, row_ptr, col_idx,
                                             col_capacity, nnz_out);
    if (st != RR_OK) return st;
    if (Nb == 0) return RR_OK;
    const size_t need = select_workspace_bytes(H, Nb);
    if (need > kNoAllocScratchBytes)
        return set_error(RR_ERR_UNSUPPORTED,
                         "%s: H=%d, Nb=%d needs %zu bytes of scratch but the built-in array holds "
                         "%zu; use rr_select with a caller-provided workspace", fn, H, Nb, need,
                         kNoAllocScratchBytes);
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return set_error(RR_ERR_CUDA, "%s: cudaGetDevice: %s", fn, cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDevices)
        return set_error(RR_ERR_UNSUPPORTED, "%s: device index %d out of range", fn, dev);
    void *scratch = nullptr;
    e = scratch_address(dev, &scratch);
    if (e != cudaSuccess)
        return set_error(RR_ERR_CUDA, "%s: cudaGetSymbolAddress of the scratch array: %s", fn,
                         cudaGetErrorString(e));
    return launch_select(block_scores, H, Nb, tau, protect_last, row_ptr, col_idx, nnz_out,
                         scratch, static_cast<cudaStream_t>(stream));
}
