// Adaptive Top-tau block selection of RRAttention ("RRAttention: Dynamic Block Sparse
// Attention via Per-Head Round-Robin Shifts for Long-Context Inference", Sec. 1 contribution
// (iii), Sec. 3.3 heading; the rule as the XAttention card states it: the smallest set of
// blocks whose cumulative score reaches tau) with last-query-block protection (Sec. 4.3).
//
//   select_rows_warp_kernel  one warp per row of up to 1024 causal blocks: the cut score by a
//                       binary search over float bit patterns with exact 64-bit fixed-point
//                       sums, ties at the cut taken in ascending J; selected blocks as a bitmap.
//   select_rows_kernel  one CTA per longer row: bitonic sort of the row's causal scores on the
//                       key (score desc, J asc), float64 inclusive scan,
//                       k* = 1 + #{k : cum_k < tau*T}, selected blocks as a bitmap.
//   scan_counts_kernel  exclusive scan of the per-row counts -> row_ptr, nnz.
//   emit_csr_kernel     one warp per row: bitmap -> ascending block indices in col_idx, one
//                       coalesced store per 32 blocks.
//   validate_csr_kernel debug check of a CSR, counts bad rows, never traps.
#include "rr_common.cuh"

namespace rr {

namespace {

constexpr int kSelThreads = 256;
// rows of up to 32*32 blocks go to the warp-per-row kernel, longer ones to the sorting kernel
constexpr int kWarpRowSlots = 32;

__device__ __forceinline__ uint64_t sort_key(float a, int J) {
    uint32_t bits = __float_as_uint(a);
    if (a == 0.f) bits = 0;  // -0 sorts as +0
    return ((uint64_t)(~bits) << 32) | (uint32_t)J;
}

__device__ __forceinline__ double key_value(uint64_t k) {
    return (double)__uint_as_float(~(uint32_t)(k >> 32));
}

// Block-wide exclusive scan of one value per thread (double), returns the exclusive prefix
// and writes the block total to *total.
__device__ double block_exclusive_scan(double v, double *warp_tot, double *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    double x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
        double t = lane < nw ? warp_tot[lane] : 0.0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const double y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        if (lane < nw) warp_tot[lane] = t;  // inclusive per warp
        if (lane == nw - 1) *total = t;
    }
    __syncthreads();
    const double before = warp ? warp_tot[warp - 1] : 0.0;
    return before + x - v;
}

__global__ void __launch_bounds__(kSelThreads)
    select_rows_kernel(const float *__restrict__ A, int Nb, long row_base, double tau,
                       int protect_last, int P, int W, int *__restrict__ counts,
                       uint32_t *__restrict__ bitmap) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem_raw);
    uint32_t *bm = reinterpret_cast<uint32_t *>(smem_raw + (size_t)P * 8);
    __shared__ double warp_tot[32];
    __shared__ double s_total;
    __shared__ int s_below;

    const long row = (long)blockIdx.x + row_base;
    const int I = (int)(row % Nb), n = I + 1, tid = threadIdx.x;
    if (n <= 32 * kWarpRowSlots) return;  // handled by select_rows_warp_kernel
    uint32_t *out_bm = bitmap + row * W;
    const bool keep_all = (tau >= 1.0) || (protect_last && I == Nb - 1);
    if (keep_all) {
        for (int w = tid; w < W; w += kSelThreads) {
            const int lo = w * 32;
            uint32_t m = 0;
            if (n >= lo + 32) m = 0xffffffffu;
            else if (n > lo) m = (1u << (n - lo)) - 1u;
            out_bm[w] = m;
        }
        if (tid == 0) counts[row] = n;
        return;
    }
    const float *a = A + row * (long)Nb;
    for (int k = tid; k < P; k += kSelThreads) keys[k] = (k < n) ? sort_key(__ldg(a + k), k) : ~0ull;
    for (int w = tid; w < W; w += kSelThreads) bm[w] = 0;
    if (tid == 0) s_below = 0;
    __syncthreads();
    // bitonic sort, ascending keys
    for (int size = 2; size <= P; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = tid; t < P / 2; t += kSelThreads) {
                const int lo = 2 * t - (t & (stride - 1));
                const int hi = lo + stride;
                const bool up = ((lo & size) == 0);
                const uint64_t x = keys[lo], y = keys[hi];
                if ((x > y) == up) {
                    keys[lo] = y;
                    keys[hi] = x;
                }
            }
            __syncthreads();
        }
    }
    // each thread owns a contiguous chunk of the sorted order
    const int per = (P + kSelThreads - 1) / kSelThreads;
    const int k0 = tid * per, k1 = min(k0 + per, n);
    double local = 0.0;
    for (int k = k0; k < k1; ++k) local += key_value(keys[k]);
    const double base = block_exclusive_scan(local, warp_tot, &s_total);
    const double T = s_total;  // all n values summed (pads excluded)
    const double thr = tau * T;
    int below = 0;
    double cum = base;
    for (int k = k0; k < k1; ++k) {
        cum += key_value(keys[k]);
        below += (cum < thr);
    }
    if (below) atomicAdd(&s_below, below);
    __syncthreads();
    const int kstar = min(s_below + 1, n);
    for (int k = tid; k < kstar; k += kSelThreads) {
        const int J = (int)(keys[k] & 0xffffffffu);
        atomicOr(&bm[J >> 5], 1u << (J & 31));
    }
    __syncthreads();
    for (int w = tid; w < W; w += kSelThreads) out_bm[w] = bm[w];
    if (tid == 0) counts[row] = kstar;
}

// Warp per row for rows of at most 32*32 blocks (values held in registers, lane l owns blocks
// J = l + 32*k).  The selected set is the first k* keys in (score desc, J asc) order; it is
// found without sorting: s* = the largest score with sum_{a >= s*} a >= tau*T (a binary search
// over the bit patterns, which order non-negative floats), then all scores above s* plus the
// ties at s* in ascending J until the sum reaches tau*T.
//
// The decision is exact on a 64-bit fixed-point grid: a score is worth its value times
// 2^(176 - E), E the biased exponent of the row maximum, truncated (a score keeps all 24 bits
// of its significand when it is within 2^-26 of the maximum, and everything down to 2^-50 of
// it; the row total stays below 2^60).  T is summed exactly on that grid, tau*T is formed in
// float64 and rounded up to it, so "cum >= tau*T" is decided exactly, with no dependence on
// summation order.  Each round of the search first sums in fp32 (one compare and one add per
// score) and settles the comparison from that sum whenever it is further from tau*T than the
// fp32 rounding error can reach (37 roundings of 2^-24 relative each; the bound used is 4e-6);
// only rounds that land closer are re-summed exactly on the grid.  A warp holds its row in
// NS registers per lane, NS the row's 32-block slots rounded up to a multiple of 4, so short
// rows do not pay for the longest row's slots.
__device__ __forceinline__ long long warp_sum_ll(long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// acc += x when the bit pattern of x is >= mid: one compare and one predicated add (the add
// on the FMA pipe, not a select on the integer pipe, which the search otherwise saturates).
__device__ __forceinline__ void add_if_at_least(float &acc, float x, uint32_t mid) {
    asm("{\n\t.reg .pred p;\n\tsetp.ge.u32 p, %1, %2;\n\t@p add.f32 %0, %0, %3;\n\t}"
        : "+f"(acc)
        : "r"(__float_as_uint(x)), "r"(mid), "f"(x));
}

// Fixed-point value of a non-negative float with bit pattern b, on the grid of a row whose
// maximum has biased exponent E (E >= 1): b's value times 2^(176 - E), truncated.
__device__ __forceinline__ long long to_fixed(uint32_t b, int E) {
    const int e = (int)(b >> 23);
    const uint32_t m = e ? ((b & 0x7fffffu) | 0x800000u) : (b & 0x7fffffu);
    const int sh = (e ? e : 1) + 26 - E;  // <= 26: the row maximum's significand lands below 2^50
    if (sh >= 0) return (long long)m << sh;
    return sh > -24 ? (long long)(m >> -sh) : 0ll;
}

template <int NS>
__device__ __forceinline__ void select_row_warp(const float *__restrict__ a, int n, double tau, int lane,
                                                uint32_t *__restrict__ out_bm, int W, int *__restrict__ count) {
    float v[NS];  // scores (-0 as +0); 0 beyond the row
    uint32_t vmax = 0;
#pragma unroll
    for (int k = 0; k < NS; ++k) {
        const int J = k * 32 + lane;
        const float x = J < n ? __ldg(a + J) : 0.f;
        v[k] = (x == 0.f) ? 0.f : x;
        vmax = max(vmax, __float_as_uint(v[k]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) vmax = max(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    const int E = max((int)(vmax >> 23), 1);
    long long tot = 0;
#pragma unroll
    for (int k = 0; k < NS; ++k) tot += to_fixed(__float_as_uint(v[k]), E);
    const long long T = warp_sum_ll(tot);
    // tau*T rounded up to the grid: for an integer sum c, c >= tau*T <=> c >= thr
    const long long thr = __double2ll_ru(tau * (double)T);
    // the same threshold in value units, widened by the fp32 error bound on both sides.  Rows
    // whose maximum is below 2^-87 (where fp32 sums lose their relative accuracy) and tau below
    // 1e-4 (where the grid's truncation, up to 2^-39 of the maximum, is no longer far below
    // the margin) always take the exact sums.
    const bool fast = E > 40 && tau >= 1e-4;
    const double thr_val = ldexp((double)thr, E - 176);
    const float thr_hi = (float)(thr_val * (1.0 + 4e-6)), thr_lo = (float)(thr_val * (1.0 - 4e-6));
    // largest u in [0, vmax] with sum_{bits(a) >= u} a >= thr (true at u = 0)
    uint32_t lo = 0, hi = vmax;
    while (lo < hi) {
        const uint32_t mid = lo + (hi - lo + 1) / 2;
        float p0 = 0.f, p1 = 0.f;
#pragma unroll
        for (int k = 0; k < NS; k += 2) {
            add_if_at_least(p0, v[k], mid);
            add_if_at_least(p1, v[k + 1], mid);
        }
        const float p = warp_sum_f(p0 + p1);
        bool ge;
        if (fast && p >= thr_hi) ge = true;
        else if (fast && p < thr_lo) ge = false;
        else {
            long long q = 0;
#pragma unroll
            for (int k = 0; k < NS; ++k)
                if (__float_as_uint(v[k]) >= mid) q += to_fixed(__float_as_uint(v[k]), E);
            ge = warp_sum_ll(q) >= thr;
        }
        if (ge) lo = mid;
        else hi = mid - 1;
    }
    const uint32_t sbits = lo;
    long long gt = 0;
    int cnt_gt = 0;
#pragma unroll
    for (int k = 0; k < NS; ++k)
        if (__float_as_uint(v[k]) > sbits) {
            gt += to_fixed(__float_as_uint(v[k]), E);
            ++cnt_gt;
        }
    gt = warp_sum_ll(gt);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt_gt += __shfl_xor_sync(0xffffffffu, cnt_gt, o);
    // ties at s*, ascending J: the smallest t >= 1 with gt + t*s >= thr (gt < thr because s*
    // is the largest score that reaches the threshold; a zero s* can only mean thr <= gt,
    // which happens for an all-zero row, where the first block is kept)
    const long long sfx = to_fixed(sbits, E);
    long long need_ll = 1;
    if (sfx > 0 && thr > gt) need_ll = (thr - gt + sfx - 1) / sfx;
    const int need_ties = (int)min(max(need_ll, 1ll), (long long)(32 * kWarpRowSlots));
    // emit the bitmap: blocks above s*, plus the first need_ties ties by ascending J
    int taken = 0;
    for (int w = NS + lane; w < W; w += 32) out_bm[w] = 0u;
#pragma unroll
    for (int k = 0; k < NS; ++k) {
        const int J = k * 32 + lane;
        const bool valid = J < n;
        const uint32_t b = __float_as_uint(v[k]);
        const bool above = valid && b > sbits;
        const bool tie = valid && b == sbits;
        const uint32_t tb = __ballot_sync(0xffffffffu, tie);
        const int before = __popc(tb & ((1u << lane) - 1u));
        const bool take_tie = tie && (taken + before < need_ties);
        taken += __popc(tb);
        const uint32_t sel = __ballot_sync(0xffffffffu, above || take_tie);
        if (lane == 0 && k < W) out_bm[k] = sel;  // word k covers blocks 32k..32k+31
    }
    if (lane == 0) *count = cnt_gt + min(need_ties, taken);
}

__global__ void __launch_bounds__(256, 4)
    select_rows_warp_kernel(const float *__restrict__ A, int Nb, long nrows, double tau,
                            int protect_last, int W, int *__restrict__ counts,
                            uint32_t *__restrict__ bitmap) {
    const long row = blockIdx.x * 8L + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= nrows) return;
    const int I = (int)(row % Nb), n = I + 1;
    if (n > 32 * kWarpRowSlots) return;  // long rows: select_rows_kernel
    uint32_t *out_bm = bitmap + row * W;
    const bool keep_all = (tau >= 1.0) || (protect_last && I == Nb - 1);
    if (keep_all) {
        for (int w = lane; w < W; w += 32) {
            const int lo = w * 32;
            uint32_t m = 0;
            if (n >= lo + 32) m = 0xffffffffu;
            else if (n > lo) m = (1u << (n - lo)) - 1u;
            out_bm[w] = m;
        }
        if (lane == 0) counts[row] = n;
        return;
    }
    const float *a = A + row * (long)Nb;
    int *cnt = counts + row;
    switch ((n + 127) >> 7) {  // 32-block slots per lane, rounded up to a multiple of 4
    case 1: select_row_warp<4>(a, n, tau, lane, out_bm, W, cnt); break;
    case 2: select_row_warp<8>(a, n, tau, lane, out_bm, W, cnt); break;
    case 3: select_row_warp<12>(a, n, tau, lane, out_bm, W, cnt); break;
    case 4: select_row_warp<16>(a, n, tau, lane, out_bm, W, cnt); break;
    case 5: select_row_warp<20>(a, n, tau, lane, out_bm, W, cnt); break;
    case 6: select_row_warp<24>(a, n, tau, lane, out_bm, W, cnt); break;
    case 7: select_row_warp<28>(a, n, tau, lane, out_bm, W, cnt); break;
    default: select_row_warp<32>(a, n, tau, lane, out_bm, W, cnt); break;
    }
}

// One CTA: the counts in chunks of 4096 (four consecutive rows per thread, one 16-byte load when
// aligned), a block-wide exclusive scan per chunk, a running carry between chunks.
__global__ void __launch_bounds__(1024)
    scan_counts_kernel(const int *__restrict__ counts, long nrows, int32_t *__restrict__ row_ptr,
                       int64_t *__restrict__ nnz_out) {
    __shared__ long warp_tot[32];
    __shared__ long s_carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) s_carry = 0;
    __syncthreads();
    for (long c0 = 0; c0 < nrows; c0 += 4096) {
        const long r0 = c0 + 4L * tid;
        int cv[4];
        if (r0 + 3 < nrows && (r0 & 3) == 0) {
            const int4 q = *reinterpret_cast<const int4 *>(counts + r0);
            cv[0] = q.x, cv[1] = q.y, cv[2] = q.z, cv[3] = q.w;
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) cv[k] = r0 + k < nrows ? counts[r0 + k] : 0;
        }
        const long local = (long)cv[0] + cv[1] + cv[2] + cv[3];
        long x = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (lane == 31) warp_tot[warp] = x;
        __syncthreads();
        if (warp == 0) {
            long t = warp_tot[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const long y = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += y;
            }
            warp_tot[lane] = t;
        }
        __syncthreads();
        const long carry = s_carry;
        long at = carry + (warp ? warp_tot[warp - 1] : 0) + x - local;
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (r0 + k < nrows) {
                row_ptr[r0 + k] = (int32_t)at;
                at += cv[k];
            }
        __syncthreads();  // every thread has read s_carry and warp_tot
        if (tid == 1023) s_carry = carry + warp_tot[31];
        __syncthreads();
    }
    if (tid == 0) {
        row_ptr[nrows] = (int32_t)s_carry;
        if (nnz_out) *nnz_out = s_carry;
    }
}

__global__ void __launch_bounds__(256)
    emit_csr_kernel(const uint32_t *__restrict__ bitmap, const int32_t *__restrict__ row_ptr,
                    long nrows, int W, int32_t *__restrict__ col_idx) {
    const long row = blockIdx.x * 8L + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= nrows) return;
    const uint32_t *bm = bitmap + row * W;
    const uint32_t below = (1u << lane) - 1u;
    int at = row_ptr[row];
    for (int w0 = 0; w0 < W; w0 += 32) {
        const uint32_t mine = (w0 + lane < W) ? bm[w0 + lane] : 0u;
        const int nw = min(32, W - w0);
        // word k covers blocks 32(w0+k) .. +31: lane l stores block 32(w0+k)+l if its bit is set,
        // at the position counted by the set bits below it, so the warp's stores are contiguous
        for (int k = 0; k < nw; ++k) {
            const uint32_t m = __shfl_sync(0xffffffffu, mine, k);
            if (m >> lane & 1u) col_idx[at + __popc(m & below)] = (w0 + k) * 32 + lane;
            at += __popc(m);
        }
    }
}

__global__ void __launch_bounds__(256)
    validate_csr_kernel(const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                        int Nb, long nrows, long nnz_cap, int32_t *__restrict__ bad) {
    for (long row = blockIdx.x * (long)blockDim.x + threadIdx.x; row < nrows;
         row += (long)gridDim.x * blockDim.x) {
        const int I = (int)(row % Nb);
        const long b = row_ptr[row], e = row_ptr[row + 1];
        bool ok = (row != 0 || b == 0) && b >= 0 && e > b && e <= nnz_cap;
        if (ok) {
            int prev = -1;
            for (long c = b; c < e && ok; ++c) {
                const int J = col_idx[c];
                ok = (J > prev) && (J <= I);
                prev = J;
            }
        }
        if (!ok) atomicAdd(bad, 1);
    }
}

}  // namespace

static int pow2_at_least(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

size_t select_workspace_bytes(int H, int Nb) {
    if (H <= 0 || Nb <= 0) return 0;
    const size_t nrows = (size_t)H * Nb, W = (Nb + 31) / 32;
    return align_up(nrows * 4, 256) + nrows * W * 4;
}

size_t select_smem_bytes(int Nb) {
    const int P = pow2_at_least(Nb < 2 ? 2 : Nb);
    return (size_t)P * 8 + (size_t)((P + 31) / 32) * 4;
}

rr_status_t launch_select(const float *A, int H, int Nb, double tau, int protect_last,
                          int32_t *row_ptr, int32_t *col_idx, int64_t *nnz_out, void *ws,
                          cudaStream_t st) {
    const long nrows = (long)H * Nb;
    const int W = (Nb + 31) / 32;
    const int P = pow2_at_least(Nb < 2 ? 2 : Nb);
    int *counts = static_cast<int *>(ws);
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(static_cast<char *>(ws) + align_up(nrows * 4, 256));
    select_rows_warp_kernel<<<(unsigned)((nrows + 7) / 8), 256, 0, st>>>(A, Nb, nrows, tau, protect_last,
                                                                        W, counts, bitmap);
    rr_status_t s = check_launch("rr_select: select_rows_warp_kernel");
    if (s != RR_OK) return s;
    if (Nb > 32 * kWarpRowSlots) {  // rows I >= 1024 of every head: sort-based kernel
        const size_t smem = select_smem_bytes(Nb);
        cudaError_t e = cudaFuncSetAttribute(select_rows_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return set_error(RR_ERR_CUDA, "rr_select: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
        select_rows_kernel<<<(unsigned)nrows, kSelThreads, smem, st>>>(A, Nb, 0L, tau, protect_last, P,
                                                                       W, counts, bitmap);
        s = check_launch("rr_select: select_rows_kernel");
        if (s != RR_OK) return s;
    }
    scan_counts_kernel<<<1, 1024, 0, st>>>(counts, nrows, row_ptr, nnz_out);
    s = check_launch("rr_select: scan_counts_kernel");
    if (s != RR_OK) return s;
    emit_csr_kernel<<<(unsigned)((nrows + 7) / 8), 256, 0, st>>>(bitmap, row_ptr, nrows, W, col_idx);
    return check_launch("rr_select: emit_csr_kernel");
}

rr_status_t launch_validate_csr(const int32_t *row_ptr, const int32_t *col_idx, int H, int Nb,
                                int64_t nnz_cap, int32_t *bad, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(bad, 0, sizeof(int32_t), st);
    if (e != cudaSuccess)
        return set_error(RR_ERR_CUDA, "rr_validate_csr: memset: %s", cudaGetErrorString(e));
    const long nrows = (long)H * Nb;
    const long want = (nrows + 255) / 256;
    validate_csr_kernel<<<(unsigned)(want < 4096 ? want : 4096), 256, 0, st>>>(row_ptr, col_idx, Nb,
                                                                               nrows, nnz_cap, bad);
    return check_launch("rr_validate_csr");
}

}  // namespace rr
