// Shared helpers of librrattn: status/error plumbing and small PTX wrappers.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "rr_attn.h"

namespace rr {

// ---------------------------------------------------------------- host-side errors
rr_status_t set_error(rr_status_t s, const char *fmt, ...);
rr_status_t check_launch(const char *what);
// Empties the calling thread's last-error text; every entry point calls it first.
void clear_error();

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Largest sizes any entry point accepts.
constexpr int kMaxL = 1 << 20;
constexpr int kMaxH = 256;

// Non-null and 16-byte aligned, else RR_ERR_INVALID_ARG with the argument's name.
rr_status_t check_ptr(const char *fn, const char *name, const void *p);

// The host-side checks of rr_select's arguments other than its workspace (sizes, tau, the
// output capacity, pointers), shared by every selection entry point.
rr_status_t check_select_args(const char *fn, const float *block_scores, int H, int Nb, double tau,
                              const int32_t *row_ptr, const int32_t *col_idx, int64_t col_capacity,
                              const int64_t *nnz_out);

// TMA descriptor (a CUtensorMap, 128 bytes, 64-byte aligned) of a 2-D row-major bf16 tensor
// [rows][cols]: boxes of 64 columns x box_rows rows, 128-byte swizzle.  False when the
// driver entry point is missing or the driver rejects the layout.
bool make_tmap_bf16(void *tmap, const void *ptr, uint64_t rows, int cols, uint32_t box_rows);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------- device helpers
// Offset inside stride i of the query sampled for query head h (round-robin strategies of
// Sec. 4.3 Table 6: head h mod S, none S-1, layer l mod S, hybrid (h+l) mod S).
__device__ __forceinline__ int rr_offset(int h, int S, int mode, int layer) {
    switch (mode) {
    case RR_NONE: return S - 1;
    case RR_LAYER: return layer % S;
    case RR_HYBRID: return (h + layer) % S;
    default: return h % S;
    }
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 2^x on the SFU (ex2.approx: relative error about 2^-22, flushes denormals; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float bf16_lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

}  // namespace rr
