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
// device before any stream capture begins.
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

void *g_scratch_addr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];

}  // namespace

using namespace rr;

extern "C" rr_status_t rr_select_noalloc(const float *block_scores, int H, int Nb, double tau,
                                         int protect_last, int32_t *row_ptr, int32_t *col_idx,
                                         int64_t col_capacity, int64_t *nnz_out,
                                         rr_stream_t stream) {
    static const char *fn = "rr_select_noalloc";
    if (H <= 0 || Nb < 0 || H > 256 || Nb > (1 << 20) / 64)
        return set_error(RR_ERR_INVALID_ARG, "%s: bad sizes H=%d Nb=%d", fn, H, Nb);
    if (!(tau > 0.0 && tau <= 1.0))
        return set_error(RR_ERR_INVALID_ARG, "%s: tau=%g must be in (0, 1]", fn, tau);
    if (Nb == 0) return RR_OK;
    const int64_t worst = (int64_t)H * Nb * (Nb + 1) / 2;
    if (worst > INT32_MAX)
        return set_error(RR_ERR_UNSUPPORTED, "%s: worst-case nnz %lld exceeds int32", fn,
                         (long long)worst);
    if (col_capacity < worst)
        return set_error(RR_ERR_INVALID_ARG, "%s: col_capacity %lld < worst case %lld", fn,
                         (long long)col_capacity, (long long)worst);
    if (!block_scores || !aligned16(block_scores) || !row_ptr || !aligned16(row_ptr) || !col_idx ||
        !aligned16(col_idx))
        return set_error(RR_ERR_INVALID_ARG, "%s: block_scores, row_ptr and col_idx must be "
                                             "non-null and 16-byte aligned", fn);
    if (nnz_out && (reinterpret_cast<uintptr_t>(nnz_out) & 7))
        return set_error(RR_ERR_INVALID_ARG, "%s: nnz_out is not 8-byte aligned", fn);
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
    std::call_once(g_scratch_once[dev], [dev] {
        g_scratch_err[dev] = cudaGetSymbolAddress(&g_scratch_addr[dev], g_select_scratch);
    });
    if (g_scratch_err[dev] != cudaSuccess || !g_scratch_addr[dev])
        return set_error(RR_ERR_CUDA, "%s: cudaGetSymbolAddress of the scratch array: %s", fn,
                         cudaGetErrorString(g_scratch_err[dev]));
    return launch_select(block_scores, H, Nb, tau, protect_last, row_ptr, col_idx, nnz_out,
                         g_scratch_addr[dev], static_cast<cudaStream_t>(stream));
}
