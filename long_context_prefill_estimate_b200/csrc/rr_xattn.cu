// XAttention's antidiagonal block importance on the 5th-generation tensor cores: the estimator
// the pattern-discovery timing compares against ("RRAttention: Dynamic Block Sparse Attention
// via Per-Head Round-Robin Shifts for Long-Context Inference", Sec. 2.2 and Sec. 4.2 "Runtime
// Efficiency", Fig. 3(b); the XAttention card, "Summary" and "Key points").
//
// Inside every S x S sub-block of the attention logits (query stride i, key stride j) the
// antidiagonal from lower-left (query iS+S-1, key jS) to upper-right (query iS, key jS+S-1) is
// summed:  a(i,j) = sum_u Q[iS+S-1-u] . K[jS+u] = sum_v Q[iS+v] . K[jS+S-1-v].  Viewed as rows
// of S*d elements, Qt_i = Q[iS .. iS+S-1] and Kt_j = K[jS .. jS+S-1] are contiguous; the second
// form pairs the 64-element chunk c of Qt_i (sub-row v = 64c / d, columns 64c % d ..) with the
// same columns of sub-row S-1-v of Kt_j, so the reversal costs nothing: it is the B operand's
// TMA coordinate.  Scores z = a / (S sqrt d) are softmax-normalised over the key strides j <= i
// and summed into blocks, times S/B, as the round-robin estimate's are.
//
//   xattn_tc_kernel  one CTA per (query head, 128 consecutive query strides).  Key strides come
//                    in tiles of 128; for each tile the 128 x 128 S tile accumulates S*d/64
//                    chunk products (A = 128 x 64 of Qt, B = 128 x 64 of Kt, both by TMA into a
//                    ring of stages) in one of two TMEM buffers.  Two passes over the tiles, as
//                    in the round-robin estimator: the first finds each row's max and sum of
//                    exp2, the second recomputes S, normalises exactly, sums each key block's
//                    B/S strides and reduces over the B/S rows of each query block with warp
//                    shuffles.
// Warp roles: 0 TMA producer and TMEM allocation, 1 MMA issuer, 2-3 idle, 4-7 softmax (thread
// = row = TMEM lane).  Every wait is bounded; a timeout sets a device error bit.
#include <cuda.h>
#include <cuda_bf16.h>

#include "rr_common.cuh"
#include "rr_sm100.cuh"

namespace rr {

namespace {

__device__ unsigned int g_xattn_errors;
constexpr unsigned kErrTimeoutXattn = 16u;

constexpr int kXRows = 128;  // query strides per CTA (tensor-core M)
constexpr int kXTile = 128;  // key strides per tile (tensor-core N)
constexpr int kXStages = 3;  // ring of (A chunk, B chunk) stages

struct XattnParams {
    float *A;
    int H, Hkv, G, Ns, Nb, S, D, nchunks;
    float c_log2;  // log2(e) / (S * sqrt(d))
};

struct XattnCfg {
    static constexpr uint32_t A_BYTES = kXRows * 64 * 2;   // 16 KB
    static constexpr uint32_t B_BYTES = kXTile * 64 * 2;   // 16 KB
    static constexpr uint32_t STAGE = A_BYTES + B_BYTES;
    static constexpr uint32_t BAR_OFF = kXStages * STAGE;
    // full[NS], empty[NS], s_full[2], s_free[2], fin
    static constexpr uint32_t NBAR = 2 * kXStages + 5;
    static constexpr uint32_t SMEM = BAR_OFF + NBAR * 8 + 16;
    static constexpr uint32_t IDESC = sm100::idesc_bf16(kXRows, kXTile, false);
    static_assert(SMEM + 1024 <= 113u * 1024u, "two CTAs per SM");
};

template <int R>
__global__ void __launch_bounds__(256, 2)
    xattn_tc_kernel(const __grid_constant__ CUtensorMap tmQt, const __grid_constant__ CUtensorMap tmKt,
                    const XattnParams p) {
    using C = XattnCfg;
    constexpr int NS = kXStages;
    constexpr int HALF = 64;          // S columns a softmax step holds in registers
    constexpr int NBH = HALF / R;     // key blocks per half tile
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t s0 = smem_u32(base);
    auto sA = [&](int s) { return s0 + s * C::STAGE; };
    auto sB = [&](int s) { return s0 + s * C::STAGE + C::A_BYTES; };
    const uint32_t sBar = s0 + C::BAR_OFF;
    auto full = [&](int s) { return sBar + 8u * s; };
    auto empty = [&](int s) { return sBar + 8u * (NS + s); };
    auto s_full = [&](int b) { return sBar + 8u * (2 * NS + b); };
    auto s_free = [&](int b) { return sBar + 8u * (2 * NS + 2 + b); };
    const uint32_t fin_bar = sBar + 8u * (2 * NS + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + C::BAR_OFF + C::NBAR * 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // CTA -> (row group, query head), longest rows first, the heads of a KV group adjacent
    const int nRG = (p.Ns + kXRows - 1) / kXRows;
    const int rg = nRG - 1 - (int)(blockIdx.x / p.H);
    const int h = (int)(blockIdx.x % p.H);
    const int g = h / p.G;
    const int i0 = rg * kXRows;
    const int nT = rg + 1;              // key tiles covering strides < i0 + 128 (i0 is a tile multiple)
    const int nq = 2 * nT;              // tile visits over both passes

    if (tid == 32) {
        for (int s = 0; s < NS; ++s) {
            sm100::mbar_init(full(s), 1);
            sm100::mbar_init(empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            sm100::mbar_init(s_full(b), 1);
            sm100::mbar_init(s_free(b), 128);
        }
        sm100::mbar_init(fin_bar, 1);
        sm100::fence_mbar_init();
    }
    if (warp == 0) {
        sm100::tmem_alloc(smem_u32(tmem_slot), 2 * kXTile);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------------- producer
            sm100::prefetch_tmap(&tmQt);
            sm100::prefetch_tmap(&tmKt);
            int k = 0;  // chunk loads issued
            bool ok = true;
            for (int qv = 0; qv < nq && ok; ++qv) {
                const int j0 = (qv % nT) * kXTile;
                for (int c = 0; c < p.nchunks; ++c, ++k) {
                    const int s = k % NS;
                    if (!sm100::mbar_wait(empty(s), ((k / NS) & 1) ^ 1)) {
                        ok = false;
                        break;
                    }
                    // chunk c of Qt: sub-row v, columns dc..dc+63; of Kt: sub-row S-1-v
                    const int v = (c * 64) / p.D, dc = (c * 64) % p.D;
                    sm100::mbar_arrive_expect_tx(full(s), C::STAGE);
                    sm100::tma_load_2d(sA(s), &tmQt, c * 64, h * p.Ns + i0, full(s));
                    sm100::tma_load_2d(sB(s), &tmKt, (p.S - 1 - v) * p.D + dc, g * p.Ns + j0, full(s));
                }
            }
            if (!ok) {
                atomicOr(&g_xattn_errors, kErrTimeoutXattn);
                for (int t = k > NS ? k - NS : 0; t < k; ++t) sm100::mbar_wait(full(t % NS), (t / NS) & 1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            bool ok = true;
            int k = 0;
            for (int qv = 0; qv < nq && ok; ++qv) {
                const int b = qv & 1;
                // buffer b is free once the softmax has loaded the tile two visits back
                if (!sm100::mbar_wait(s_free(b), ((qv >> 1) & 1) ^ 1)) {
                    ok = false;
                    break;
                }
                for (int c = 0; c < p.nchunks; ++c, ++k) {
                    const int s = k % NS;
                    if (!sm100::mbar_wait(full(s), (k / NS) & 1)) {
                        ok = false;
                        break;
                    }
                    sm100::tc_fence_after();
#pragma unroll
                    for (int w4 = 0; w4 < 4; ++w4) {
                        const uint64_t ad = sm100::smem_desc_sw128(sA(s) + w4 * 32, 16, 1024);
                        const uint64_t bd = sm100::smem_desc_sw128(sB(s) + w4 * 32, 16, 1024);
                        sm100::mma_ss(tmem + b * kXTile, ad, bd, C::IDESC, (c > 0 || w4 > 0) ? 1u : 0u);
                    }
                    sm100::mma_commit(empty(s));
                }
                if (ok) sm100::mma_commit(s_full(b));
            }
            sm100::mma_commit(fin_bar);
            if (!sm100::mbar_wait(fin_bar, 0)) ok = false;
            if (!ok) atomicOr(&g_xattn_errors, kErrTimeoutXattn);
        }
    } else if (warp >= 4) {
        // -------------------------------------------------------------------- softmax
        const int row = (warp & 3) * 32 + lane;  // = TMEM lane
        const int irow = i0 + row;                // the row's query stride
        const bool valid = irow < p.Ns;
        const int I = irow / R, ii = irow % R;
        float *arow = p.A + ((long)h * p.Nb + (valid ? I : 0)) * p.Nb;
        const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const float c = p.c_log2;
        float m = -INFINITY, l = 0.f, mL = 0.f;
        bool ok = true;
        for (int qv = 0; qv < nq; ++qv) {
            const int b = qv & 1;
            ok = __all_sync(0xffffffffu, sm100::mbar_wait(s_full(b), (qv >> 1) & 1));
            if (!ok) break;
            sm100::tc_fence_after();
            const int j0 = (qv % nT) * kXTile;
            const bool pass1 = qv < nT;
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t sr[HALF];
                sm100::tmem_ld32(trow + b * kXTile + hf * HALF, *reinterpret_cast<uint32_t(*)[32]>(sr));
                sm100::tmem_ld32(trow + b * kXTile + hf * HALF + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
                sm100::tmem_wait_ld();
                if (hf == 1) {  // both halves read: the MMA warp may refill this buffer
                    sm100::tc_fence_before();
                    sm100::mbar_arrive(s_free(b));
                }
                const int jh = j0 + hf * HALF;
                // strides j > i are outside the stride-level causal mask
                const int nvis = max(0, min(HALF, irow - jh + 1));
                if (pass1) {
                    float mx = -INFINITY;
#pragma unroll
                    for (int j = 0; j < HALF; ++j)
                        if (j < nvis) mx = fmaxf(mx, __uint_as_float(sr[j]) * c);
                    if (mx > m + 8.f) {
                        l *= ex2_approx(m - mx);  // 0 while nothing was seen
                        m = mx;
                    }
                    float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int j = 0; j < HALF; ++j)
                        s4[j & 3] += (j < nvis) ? ex2_approx(fmaf(__uint_as_float(sr[j]), c, -m)) : 0.f;
                    l += (s4[0] + s4[1]) + (s4[2] + s4[3]);
                    if (qv == nT - 1 && hf == 1) mL = (l > 0.f) ? m + log2f(l) : INFINITY;  // p = 2^(s*c - mL)
                } else {
                    float bs[NBH];
#pragma unroll
                    for (int kb = 0; kb < NBH; ++kb) {
                        float acc = 0.f;
#pragma unroll
                        for (int jj = 0; jj < R; ++jj) {
                            const int j = kb * R + jj;
                            acc += (j < nvis) ? ex2_approx(fmaf(__uint_as_float(sr[j]), c, -mL)) : 0.f;
                        }
                        bs[kb] = valid ? acc : 0.f;
                    }
#pragma unroll
                    for (int o = 1; o < R; o <<= 1)
#pragma unroll
                        for (int kb = 0; kb < NBH; ++kb) bs[kb] += __shfl_xor_sync(0xffffffffu, bs[kb], o);
                    const int J0 = jh / R;
                    if (valid) {
#pragma unroll
                        for (int kb = 0; kb < NBH; ++kb)
                            if (kb % R == ii && J0 + kb < p.Nb) arow[J0 + kb] = bs[kb] * (1.f / R);
                    }
                }
            }
        }
        if (!ok) {
            if (lane == 0) atomicOr(&g_xattn_errors, kErrTimeoutXattn);
        } else if (valid) {
            // blocks past the last tile are above the diagonal: zero
            for (int J = nT * kXTile / R + ii; J < p.Nb; J += R) arow[J] = 0.f;
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();  // lane 0 ran the producer; dealloc is warp-collective
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, 2 * kXTile);
    }
}

template <int R>
rr_status_t launch_xattn_r(const CUtensorMap &mq, const CUtensorMap &mk, const XattnParams &p, cudaStream_t st) {
    using C = XattnCfg;
    auto kern = xattn_tc_kernel<R>;
    const size_t smem = C::SMEM + 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return set_error(RR_ERR_CUDA, "rr_xattn_estimate: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    const long ctas = (long)p.H * ((p.Ns + kXRows - 1) / kXRows);
    kern<<<(unsigned)ctas, 256, smem, st>>>(mq, mk, p);
    return check_launch("rr_xattn_estimate: xattn_tc_kernel");
}

}  // namespace

// Sizes with a kernel: d in {64, 128}, B/S in {4, 8, 16, 32}, S*d a multiple of 64.
bool xattn_supported(int d, int S, int B) {
    const int r = B / S;
    return (d == 64 || d == 128) && (r == 4 || r == 8 || r == 16 || r == 32) && (S * d) % 64 == 0;
}

rr_status_t launch_xattn(const uint16_t *Q, const uint16_t *K, int H, int Hkv, int L, int d, int S, int B,
                         float *A, cudaStream_t st) {
    const int Ns = L / S;
    alignas(64) CUtensorMap mq, mk;
    // Q and K viewed as rows of S*d elements: row i of head h is the stride Q[h][iS .. iS+S-1]
    if (!make_tmap_bf16(&mq, Q, (uint64_t)H * Ns, S * d, kXRows) ||
        !make_tmap_bf16(&mk, K, (uint64_t)Hkv * Ns, S * d, kXTile))
        return set_error(RR_ERR_CUDA, "rr_xattn_estimate: cuTensorMapEncodeTiled failed");
    XattnParams p;
    p.A = A;
    p.H = H;
    p.Hkv = Hkv;
    p.G = H / Hkv;
    p.Ns = Ns;
    p.Nb = L / B;
    p.S = S;
    p.D = d;
    p.nchunks = S * d / 64;
    p.c_log2 = (float)(1.4426950408889634 / ((double)S * sqrt((double)d)));
    switch (B / S) {
    case 4: return launch_xattn_r<4>(mq, mk, p, st);
    case 8: return launch_xattn_r<8>(mq, mk, p, st);
    case 16: return launch_xattn_r<16>(mq, mk, p, st);
    default: return launch_xattn_r<32>(mq, mk, p, st);
    }
}

rr_status_t read_xattn_errors(unsigned *out, bool reset) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_xattn_errors, sizeof(unsigned));
    if (e == cudaSuccess && reset) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_xattn_errors, &zero, sizeof(unsigned));
    }
    if (e != cudaSuccess) return set_error(RR_ERR_CUDA, "rr_device_errors: %s", cudaGetErrorString(e));
    return RR_OK;
}

}  // namespace rr
