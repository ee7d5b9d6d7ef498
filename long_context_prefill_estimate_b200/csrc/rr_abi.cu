// C ABI of librrattn: argument validation on the host, then kernel launches on the caller's
// stream.  Nothing here allocates device memory or synchronises.
#include <stdarg.h>
#include <stdio.h>

#include <cmath>

#include "rr_common.cuh"

// NVTX ranges around the entry points (header-only NVTX 3; a profiler that injects NVTX, such
// as Nsight Systems, shows them on the host timeline, otherwise they cost a branch each).
#if __has_include(<nvtx3/nvToolsExt.h>)
#include <nvtx3/nvToolsExt.h>
#define RR_NVTX 1
#endif

namespace rr {

size_t estimate_workspace_bytes(int Hkv, int L, int d, int S);
bool estimate_supported(int H, int Hkv, int d, int S, int B, int L);
rr_status_t launch_estimate(const uint16_t *Q, const uint16_t *K, int H, int Hkv, int L, int d,
                            int S, int B, int mode, int layer, int head_base, float *A, void *ws,
                            cudaStream_t st);
size_t select_workspace_bytes(int H, int Nb);
rr_status_t launch_select(const float *A, int H, int Nb, double tau, int protect_last,
                          int32_t *row_ptr, int32_t *col_idx, int64_t *nnz_out, void *ws,
                          cudaStream_t st);
rr_status_t launch_validate_csr(const int32_t *row_ptr, const int32_t *col_idx, int H, int Nb,
                                int64_t nnz_cap, int32_t *bad, cudaStream_t st);
rr_status_t launch_prefill_tc(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int H, int Hkv,
                              int L, int d, int B, const int32_t *row_ptr, const int32_t *col_idx,
                              float scale, uint16_t *O, cudaStream_t st);
rr_status_t read_device_errors(unsigned *out, bool reset);
rr_status_t read_estimate_errors(unsigned *out, bool reset);
rr_status_t read_pp_errors(unsigned *out, bool reset);
rr_status_t read_xattn_errors(unsigned *out, bool reset);
bool xattn_supported(int d, int S, int B);
rr_status_t launch_xattn(const uint16_t *Q, const uint16_t *K, int H, int Hkv, int L, int d, int S, int B,
                         float *A, cudaStream_t st);
rr_status_t selftest_wait(uint32_t timeout_us, uint32_t *result);

#define RR_TRY(x)                       \
    do {                                \
        const rr_status_t s_ = (x);     \
        if (s_ != RR_OK) return s_;     \
    } while (0)

static thread_local char g_last_error[512] = "";

rr_status_t set_error(rr_status_t s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
    va_end(ap);
    return s;
}

void clear_error() { g_last_error[0] = 0; }

rr_status_t check_ptr(const char *fn, const char *name, const void *p) {
    if (!p) return set_error(RR_ERR_INVALID_ARG, "%s: %s is NULL", fn, name);
    if (!aligned16(p)) return set_error(RR_ERR_INVALID_ARG, "%s: %s is not 16-byte aligned", fn, name);
    return RR_OK;
}

rr_status_t check_launch(const char *what) {
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return set_error(RR_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
    return RR_OK;
}

rr_status_t check_select_args(const char *fn, const float *block_scores, int H, int Nb, double tau,
                              const int32_t *row_ptr, const int32_t *col_idx, int64_t col_capacity,
                              const int64_t *nnz_out) {
    if (H <= 0 || Nb < 0 || H > kMaxH || Nb > kMaxL / 64)
        return set_error(RR_ERR_INVALID_ARG, "%s: bad sizes H=%d Nb=%d", fn, H, Nb);
    if (!(tau > 0.0 && tau <= 1.0) || std::isnan(tau))
        return set_error(RR_ERR_INVALID_ARG, "%s: tau=%g must be in (0, 1]", fn, tau);
    if (Nb == 0) return RR_OK;
    const int64_t worst = (int64_t)H * Nb * (Nb + 1) / 2;
    if (worst > INT32_MAX)
        return set_error(RR_ERR_UNSUPPORTED, "%s: worst-case nnz %lld exceeds int32", fn, (long long)worst);
    if (col_capacity < worst)
        return set_error(RR_ERR_INVALID_ARG, "%s: col_capacity %lld < worst case %lld", fn,
                         (long long)col_capacity, (long long)worst);
    RR_TRY(check_ptr(fn, "block_scores", block_scores));
    RR_TRY(check_ptr(fn, "row_ptr", row_ptr));
    RR_TRY(check_ptr(fn, "col_idx", col_idx));
    if (nnz_out && (reinterpret_cast<uintptr_t>(nnz_out) & 7))
        return set_error(RR_ERR_INVALID_ARG, "%s: nnz_out is not 8-byte aligned", fn);
    return RR_OK;
}

namespace {

// Scoped NVTX range named after the entry point.
struct NvtxRange {
    explicit NvtxRange(const char *name) {
#ifdef RR_NVTX
        nvtxRangePushA(name);
#else
        (void)name;
#endif
    }
    ~NvtxRange() {
#ifdef RR_NVTX
        nvtxRangePop();
#endif
    }
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

rr_status_t check_common(const char *fn, int H, int Hkv, int L, int d, int B) {
    if (H <= 0 || Hkv <= 0 || L < 0 || d <= 0 || B <= 0)
        return set_error(RR_ERR_INVALID_ARG, "%s: sizes must be positive (H=%d Hkv=%d L=%d d=%d B=%d)",
                         fn, H, Hkv, L, d, B);
    if (H % Hkv)
        return set_error(RR_ERR_INVALID_ARG, "%s: H=%d is not a multiple of Hkv=%d", fn, H, Hkv);
    if (d != 64 && d != 128)
        return set_error(RR_ERR_UNSUPPORTED, "%s: head dim d=%d not in {64, 128}", fn, d);
    if (B != 64 && B != 128)
        return set_error(RR_ERR_UNSUPPORTED, "%s: block size B=%d not in {64, 128}", fn, B);
    if (L % B)
        return set_error(RR_ERR_UNSUPPORTED, "%s: L=%d is not a multiple of B=%d", fn, L, B);
    if (L > kMaxL || H > kMaxH)
        return set_error(RR_ERR_UNSUPPORTED, "%s: L=%d or H=%d above the supported maximum", fn, L, H);
    return RR_OK;
}

}  // namespace
}  // namespace rr

using namespace rr;

extern "C" {

int rr_version(void) { return 100; }

const char *rr_status_string(rr_status_t s) {
    switch (s) {
    case RR_OK: return "RR_OK";
    case RR_ERR_INVALID_ARG: return "RR_ERR_INVALID_ARG";
    case RR_ERR_UNSUPPORTED: return "RR_ERR_UNSUPPORTED";
    case RR_ERR_CUDA: return "RR_ERR_CUDA";
    case RR_ERR_WORKSPACE: return "RR_ERR_WORKSPACE";
    default: return "RR_ERR_UNKNOWN";
    }
}

const char *rr_last_error(void) { return g_last_error; }

rr_status_t rr_device_errors(uint32_t *flags, int reset) {
    clear_error();
    if (!flags) return set_error(RR_ERR_INVALID_ARG, "rr_device_errors: flags is NULL");
    unsigned v = 0, ve = 0, vp = 0, vx = 0;
    rr_status_t s = read_device_errors(&v, reset != 0);
    if (s == RR_OK) s = read_estimate_errors(&ve, reset != 0);
    if (s == RR_OK) s = read_pp_errors(&vp, reset != 0);
    if (s == RR_OK) s = read_xattn_errors(&vx, reset != 0);
    *flags = v | ve | vp | vx;
    return s;
}

rr_status_t rr_selftest_wait(uint32_t timeout_us, uint32_t *result) {
    clear_error();
    if (!result) return set_error(RR_ERR_INVALID_ARG, "rr_selftest_wait: result is NULL");
    if (timeout_us == 0 || timeout_us > 2000000u)
        return set_error(RR_ERR_INVALID_ARG, "rr_selftest_wait: timeout_us=%u outside (0, 2e6]",
                         timeout_us);
    return selftest_wait(timeout_us, result);
}

size_t rr_estimate_workspace_bytes(int H, int Hkv, int L, int d, int S, int B) {
    (void)H;
    (void)B;
    if (Hkv <= 0 || L <= 0 || S <= 0 || d <= 0) return 0;
    return estimate_workspace_bytes(Hkv, L, d, S);
}

rr_status_t rr_estimate_heads(const rr_bf16_t *Q, const rr_bf16_t *K, int H, int Hkv, int L, int d,
                              int S, int B, rr_strategy_t strategy, int layer, int head_base,
                              float *block_scores, void *workspace, size_t workspace_bytes,
                              rr_stream_t stream) {
    static const char *fn = "rr_estimate";
    const NvtxRange range(fn);
    clear_error();
    RR_TRY(check_common(fn, H, Hkv, L, d, B));
    if (S <= 0 || S > B || B % S)
        return set_error(RR_ERR_INVALID_ARG, "%s: stride S=%d must divide B=%d", fn, S, B);
    if ((B / S) % 8 && B / S != 4)
        return set_error(RR_ERR_UNSUPPORTED, "%s: B/S=%d must be 4 or a multiple of 8", fn, B / S);
    if ((L / S) % 8)
        return set_error(RR_ERR_UNSUPPORTED, "%s: L/S=%d strides must be a multiple of 8", fn, L / S);
    if ((int)strategy < RR_HEAD || (int)strategy > RR_HYBRID || layer < 0 || head_base < 0 ||
        head_base > (1 << 20))
        return set_error(RR_ERR_INVALID_ARG, "%s: bad strategy %d / layer %d / head_base %d", fn,
                         (int)strategy, layer, head_base);
    if (L == 0) return RR_OK;
    RR_TRY(check_ptr(fn, "Q", Q));
    RR_TRY(check_ptr(fn, "K", K));
    RR_TRY(check_ptr(fn, "block_scores", block_scores));
    const size_t need = estimate_workspace_bytes(Hkv, L, d, S);
    if (!workspace || workspace_bytes < need)
        return set_error(RR_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need,
                         workspace ? workspace_bytes : (size_t)0);
    RR_TRY(check_ptr(fn, "workspace", workspace));
    if (!estimate_supported(H, Hkv, d, S, B, L))
        return set_error(RR_ERR_UNSUPPORTED, "%s: no kernel for d=%d B/S=%d", fn, d, B / S);
    return launch_estimate(Q, K, H, Hkv, L, d, S, B, (int)strategy, layer, head_base, block_scores,
                           workspace, static_cast<cudaStream_t>(stream));
}

rr_status_t rr_estimate_strategy(const rr_bf16_t *Q, const rr_bf16_t *K, int H, int Hkv, int L,
                                 int d, int S, int B, rr_strategy_t strategy, int layer,
                                 float *block_scores, void *workspace, size_t workspace_bytes,
                                 rr_stream_t stream) {
    return rr_estimate_heads(Q, K, H, Hkv, L, d, S, B, strategy, layer, 0, block_scores, workspace,
                             workspace_bytes, stream);
}

rr_status_t rr_estimate(const rr_bf16_t *Q, const rr_bf16_t *K, int H, int Hkv, int L, int d,
                        int S, int B, float *block_scores, void *workspace,
                        size_t workspace_bytes, rr_stream_t stream) {
    return rr_estimate_strategy(Q, K, H, Hkv, L, d, S, B, RR_HEAD, 0, block_scores, workspace,
                                workspace_bytes, stream);
}

rr_status_t rr_xattn_estimate(const rr_bf16_t *Q, const rr_bf16_t *K, int H, int Hkv, int L, int d,
                              int S, int B, float *block_scores, rr_stream_t stream) {
    static const char *fn = "rr_xattn_estimate";
    const NvtxRange range(fn);
    clear_error();
    RR_TRY(check_common(fn, H, Hkv, L, d, B));
    if (S <= 0 || S > B || B % S)
        return set_error(RR_ERR_INVALID_ARG, "%s: stride S=%d must divide B=%d", fn, S, B);
    if (!xattn_supported(d, S, B))
        return set_error(RR_ERR_UNSUPPORTED, "%s: no kernel for d=%d B/S=%d", fn, d, B / S);
    if ((L / S) % 8)
        return set_error(RR_ERR_UNSUPPORTED, "%s: L/S=%d strides must be a multiple of 8", fn, L / S);
    if (L == 0) return RR_OK;
    RR_TRY(check_ptr(fn, "Q", Q));
    RR_TRY(check_ptr(fn, "K", K));
    RR_TRY(check_ptr(fn, "block_scores", block_scores));
    return launch_xattn(Q, K, H, Hkv, L, d, S, B, block_scores, static_cast<cudaStream_t>(stream));
}

size_t rr_select_workspace_bytes(int H, int Nb) { return select_workspace_bytes(H, Nb); }

rr_status_t rr_select(const float *block_scores, int H, int Nb, double tau, int protect_last,
                      int32_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                      int64_t *nnz_out, void *workspace, size_t workspace_bytes,
                      rr_stream_t stream) {
    static const char *fn = "rr_select";
    const NvtxRange range(fn);
    clear_error();
    RR_TRY(check_select_args(fn, block_scores, H, Nb, tau, row_ptr, col_idx, col_capacity, nnz_out));
    if (Nb == 0) return RR_OK;
    const size_t need = select_workspace_bytes(H, Nb);
    if (!workspace || workspace_bytes < need)
        return set_error(RR_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need,
                         workspace ? workspace_bytes : (size_t)0);
    RR_TRY(check_ptr(fn, "workspace", workspace));
    return launch_select(block_scores, H, Nb, tau, protect_last, row_ptr, col_idx, nnz_out,
                         workspace, static_cast<cudaStream_t>(stream));
}

rr_status_t rr_sparse_prefill(const rr_bf16_t *Q, const rr_bf16_t *K, const rr_bf16_t *V,
                              int H, int Hkv, int L, int d, int B, const int32_t *row_ptr,
                              const int32_t *col_idx, float softmax_scale, rr_bf16_t *O,
                              rr_stream_t stream) {
    static const char *fn = "rr_sparse_prefill";
    const NvtxRange range(fn);
    clear_error();
    RR_TRY(check_common(fn, H, Hkv, L, d, B));
    if (std::isnan(softmax_scale) || std::isinf(softmax_scale))
        return set_error(RR_ERR_INVALID_ARG, "%s: softmax_scale is not finite", fn);
    if (L == 0) return RR_OK;
    RR_TRY(check_ptr(fn, "Q", Q));
    RR_TRY(check_ptr(fn, "K", K));
    RR_TRY(check_ptr(fn, "V", V));
    RR_TRY(check_ptr(fn, "O", O));
    RR_TRY(check_ptr(fn, "row_ptr", row_ptr));
    RR_TRY(check_ptr(fn, "col_idx", col_idx));
    const float scale = softmax_scale > 0.f ? softmax_scale : (float)(1.0 / std::sqrt((double)d));
    return launch_prefill_tc(Q, K, V, H, Hkv, L, d, B, row_ptr, col_idx, scale, O,
                             static_cast<cudaStream_t>(stream));
}

rr_status_t rr_validate_csr(const int32_t *row_ptr, const int32_t *col_idx, int H, int Nb,
                            int64_t nnz_cap, int32_t *bad_rows, rr_stream_t stream) {
    static const char *fn = "rr_validate_csr";
    clear_error();
    if (H <= 0 || Nb <= 0 || nnz_cap < 0)
        return set_error(RR_ERR_INVALID_ARG, "%s: bad sizes", fn);
    RR_TRY(check_ptr(fn, "row_ptr", row_ptr));
    RR_TRY(check_ptr(fn, "col_idx", col_idx));
    if (!bad_rows || (reinterpret_cast<uintptr_t>(bad_rows) & 3))
        return set_error(RR_ERR_INVALID_ARG, "%s: bad_rows is NULL or misaligned", fn);
    return launch_validate_csr(row_ptr, col_idx, H, Nb, nnz_cap, bad_rows,
                               static_cast<cudaStream_t>(stream));
}

}  // extern "C"
