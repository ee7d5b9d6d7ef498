// Causal block-sparse attention over the selected blocks ("RRAttention: Dynamic Block Sparse
// Attention via Per-Head Round-Robin Shifts for Long-Context Inference", Sec. 2.1 with the
// per-head CSR block lists as the block selection matrix).
//
// Warp-level tensor-core kernel (mma.sync m16n8k16, bf16 in, fp32 accumulate): one CTA per
// (query block I, query head h), B/16 warps with 16 query rows each.  It walks only the CSR
// entries of row h*Nb + I, in 64-key sub-tiles streamed through shared memory with cp.async
// (double-buffered, XOR-swizzled 16-byte chunks), with an online softmax in registers and
// the causal mask applied only inside the diagonal block.  K and V come from KV head
// h / (H/Hkv).
#include <cuda_bf16.h>

#include "rr_common.cuh"

namespace rr {

namespace {

constexpr int kKT = 64;  // keys per sub-tile

template <int D>
__device__ __forceinline__ int swz(int row, int chunk) {  // element offset of a 16-byte chunk
    return row * D + ((chunk ^ (row & 7)) << 3);
}

template <int D, int BQ>
__global__ void __launch_bounds__(BQ * 2)
    prefill_mma_kernel(const uint16_t *__restrict__ Q, const uint16_t *__restrict__ K,
                       const uint16_t *__restrict__ V, int H, int Hkv, int L, int Nb,
                       const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                       float scale_log2, uint16_t *__restrict__ O) {
    constexpr int NW = BQ / 16, NTH = NW * 32, CH = D / 8, KSQ = D / 16, NTO = D / 8;
    constexpr int SUB = BQ / kKT;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    uint16_t *qs = reinterpret_cast<uint16_t *>(smem_raw);
    uint16_t *ks = qs + BQ * D;          // [2][kKT][D]
    uint16_t *vs = ks + 2 * kKT * D;     // [2][kKT][D]

    const int I = Nb - 1 - (int)blockIdx.x;
    const int h = blockIdx.y;
    const int g = h / (H / Hkv);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gq = lane >> 2, tq = lane & 3;
    const long q0 = (long)I * BQ;
    const uint16_t *Qh = Q + ((long)h * L + q0) * D;
    const uint16_t *Kg = K + (long)g * L * D;
    const uint16_t *Vg = V + (long)g * L * D;
    const long rrow = (long)h * Nb + I;
    const int e0 = row_ptr[rrow], e1 = row_ptr[rrow + 1];
    const int nunits = (e1 - e0) * SUB;

    for (int x = tid; x < BQ * CH; x += NTH) {
        const int row = x / CH, c = x % CH;
        cp_async_16(smem_u32(qs + swz<D>(row, c)), Qh + (long)row * D + c * 8);
    }
    cp_async_commit();
    auto load_unit = [&](int u, int buf) {
        const int J = col_idx[e0 + u / SUB];
        const long k0 = (long)J * BQ + (u % SUB) * kKT;
        uint16_t *kd = ks + buf * kKT * D, *vd = vs + buf * kKT * D;
        for (int x = tid; x < kKT * CH; x += NTH) {
            const int row = x / CH, c = x % CH;
            cp_async_16(smem_u32(kd + swz<D>(row, c)), Kg + (k0 + row) * D + c * 8);
            cp_async_16(smem_u32(vd + swz<D>(row, c)), Vg + (k0 + row) * D + c * 8);
        }
    };
    if (nunits > 0) load_unit(0, 0);
    cp_async_commit();

    uint32_t qf[KSQ][4];
    float o[NTO][4];
#pragma unroll
    for (int n = 0; n < NTO; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
    const long qrow0 = q0 + warp * 16 + gq;  // rows qrow0 and qrow0 + 8

    for (int u = 0; u < nunits; ++u) {
        if (u + 1 < nunits) load_unit(u + 1, (u + 1) & 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        if (u == 0) {
#pragma unroll
            for (int kk = 0; kk < KSQ; ++kk) {
                const int row = warp * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
                ldmatrix_x4(qf[kk], smem_u32(qs + swz<D>(row, kk * 2 + (lane >> 4))));
            }
        }
        const int J = col_idx[e0 + u / SUB];
        const long k0 = (long)J * BQ + (u % SUB) * kKT;
        const bool diag = (J == I);
        // rows of this warp all precede the sub-tile: nothing to attend here
        if (!(diag && q0 + warp * 16 + 15 < k0)) {
            const uint16_t *kb = ks + (u & 1) * kKT * D;
            const uint16_t *vb = vs + (u & 1) * kKT * D;
            float s[kKT / 8][4];
#pragma unroll
            for (int n = 0; n < kKT / 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < KSQ; ++kk) {
#pragma unroll
                for (int np = 0; np < kKT / 16; ++np) {
                    uint32_t b[4];
                    const int key = np * 16 + (lane >> 4) * 8 + (lane & 7);
                    ldmatrix_x4(b, smem_u32(kb + swz<D>(key, kk * 2 + ((lane >> 3) & 1))));
                    mma_16816(s[2 * np], qf[kk], b[0], b[1]);
                    mma_16816(s[2 * np + 1], qf[kk], b[2], b[3]);
                }
            }
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int n = 0; n < kKT / 8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const long key = k0 + n * 8 + 2 * tq + (e & 1);
                    const long qr = qrow0 + 8 * (e >> 1);
                    float v = s[n][e] * scale_log2;
                    if (diag && key > qr) v = -INFINITY;
                    s[n][e] = v;
                    mx[e >> 1] = fmaxf(mx[e >> 1], v);
                }
            float alpha[2];
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const float mnew = fmaxf(mrow[x], quad_max(mx[x]));
                alpha[x] = (mrow[x] == -INFINITY) ? 0.f : exp2f(mrow[x] - mnew);
                mrow[x] = mnew;
            }
            float rs[2] = {0.f, 0.f};
#pragma unroll
            for (int n = 0; n < kKT / 8; ++n)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float m = mrow[e >> 1];
                    const float pv = (m == -INFINITY) ? 0.f : exp2f(s[n][e] - m);
                    s[n][e] = pv;
                    rs[e >> 1] += pv;
                }
#pragma unroll
            for (int x = 0; x < 2; ++x) lrow[x] = lrow[x] * alpha[x] + rs[x];
#pragma unroll
            for (int n = 0; n < NTO; ++n) {
                o[n][0] *= alpha[0];
                o[n][1] *= alpha[0];
                o[n][2] *= alpha[1];
                o[n][3] *= alpha[1];
            }
#pragma unroll
            for (int kk = 0; kk < kKT / 16; ++kk) {
                uint32_t pa[4];
                pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
                pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
                pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
                pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
                for (int nd = 0; nd < NTO; nd += 2) {
                    uint32_t b[4];
                    const int key = kk * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
                    ldmatrix_x4_trans(b, smem_u32(vb + swz<D>(key, nd + (lane >> 4))));
                    mma_16816(o[nd], pa, b[0], b[1]);
                    mma_16816(o[nd + 1], pa, b[2], b[3]);
                }
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();

    float inv[2];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        const float l = quad_sum(lrow[x]);
        inv[x] = (l > 0.f) ? 1.f / l : 0.f;
    }
    uint16_t *Oh = O + ((long)h * L + q0 + warp * 16 + gq) * D;
#pragma unroll
    for (int n = 0; n < NTO; ++n) {
        const int col = n * 8 + 2 * tq;
        *reinterpret_cast<uint32_t *>(Oh + col) = pack_bf16(o[n][0] * inv[0], o[n][1] * inv[0]);
        *reinterpret_cast<uint32_t *>(Oh + 8L * D + col) =
            pack_bf16(o[n][2] * inv[1], o[n][3] * inv[1]);
    }
}

}  // namespace

rr_status_t launch_prefill_mma(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int H,
                               int Hkv, int L, int d, int B, const int32_t *row_ptr,
                               const int32_t *col_idx, float scale, uint16_t *O,
                               cudaStream_t st) {
    const int Nb = L / B;
    const float scale_log2 = scale * 1.4426950408889634f;
    dim3 grid(Nb, H);
    auto launch = [&](auto kern, int D, int BQ) -> rr_status_t {
        const size_t smem = (size_t)(BQ * D + 4 * kKT * D) * 2;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return set_error(RR_ERR_CUDA, "rr_sparse_prefill: cudaFuncSetAttribute: %s",
                             cudaGetErrorString(e));
        kern<<<grid, BQ * 2, smem, st>>>(Q, K, V, H, Hkv, L, Nb, row_ptr, col_idx, scale_log2, O);
        return check_launch("rr_sparse_prefill: prefill_mma_kernel");
    };
    if (d == 128 && B == 128) return launch(prefill_mma_kernel<128, 128>, 128, 128);
    if (d == 128 && B == 64) return launch(prefill_mma_kernel<128, 64>, 128, 64);
    if (d == 64 && B == 128) return launch(prefill_mma_kernel<64, 128>, 64, 128);
    return launch(prefill_mma_kernel<64, 64>, 64, 64);
}

}  // namespace rr
