// Stride-level block importance of RRAttention on the 5th-generation tensor cores
// ("RRAttention: Dynamic Block Sparse Attention via Per-Head Round-Robin Shifts for
// Long-Context Inference", Sec. 3.1 heading, Sec. 3.2, Sec. 3.3 heading).
//
//   pool_keys_rows_kernel  Kbar_j = sum of the S keys of stride j (fp32), split into bf16
//                          hi + lo, stored row-major: hi [Hkv][Ns][d], then lo [Hkv][Ns][d].
//   estimate_tc_kernel     one CTA per (KV head g, chunk of hc of g's query heads, group of
//                          QB consecutive query blocks).  Its 128 rows are the sampled
//                          queries Q[h][i*S + off(h)] of those heads and blocks (QB * hc * r
//                          of them, r = B/S), staged once into TMEM (the MMA's A operand, read
//                          from tensor memory, so shared memory feeds only the key tiles).
//                          Pooled keys arrive by TMA in tiles of 64 strides (a ring of three);
//                          S = Qhat (Kbar_hi + Kbar_lo)^T (fp32-grade logits) goes to one of
//                          two TMEM buffers.  96 KB of shared memory and 256 TMEM columns per
//                          CTA: two CTAs share an SM, so the softmax of one overlaps the MMAs
//                          and loads of the other.  Two passes over the
//                          tiles: the first finds each row's max and sum of exp2 over the
//                          causal strides j <= i; the second recomputes S, normalises exactly,
//                          sums each key block's r strides and reduces over the r rows of each
//                          (head, query block) with warp shuffles; times S/B that is the block
//                          score, written straight to A.
// For r <= 32 the r rows of a (head, query block) lie in one warp and are reduced with
// shuffles; for r = 64 or 128 they span r/32 warps, whose sums meet in shared memory behind
// bounded mbarrier waits (a fixed summation order, so the result is deterministic).
// Warp roles: 0 TMA producer and TMEM allocation, 1 MMA issuer, 2-3 idle, 4-7 staging of the
// sampled rows, then softmax (thread = row = TMEM lane).  Every wait is bounded; a timeout sets a device error bit.
#include <cuda.h>
#include <cuda_bf16.h>

#include "rr_common.cuh"
#include "rr_sm100.cuh"

namespace rr {

namespace {

__device__ unsigned int g_est_errors;
constexpr unsigned kErrTimeoutEstimate = 8u;

constexpr int kRows = 128;   // sampled rows per CTA (tensor-core M)
constexpr int kTileN = 64;   // strides per key tile (tensor-core N)

template <int D>
__global__ void __launch_bounds__(256) pool_keys_rows_kernel(const uint16_t *__restrict__ K, int L, int S,
                                                             int Ns, int Hkv, uint16_t *__restrict__ hi,
                                                             uint16_t *__restrict__ lo) {
    constexpr int C = D / 8;  // 16-byte chunks per key row
    const long total = (long)Hkv * Ns * C;
    for (long idx = blockIdx.x * (long)blockDim.x + threadIdx.x; idx < total;
         idx += (long)gridDim.x * blockDim.x) {
        const int c = (int)(idx % C);
        const long row = idx / C;  // g * Ns + j
        const int g = (int)(row / Ns);
        const long j = row % Ns;
        const uint4 *src = reinterpret_cast<const uint4 *>(K + ((long)g * L + j * S) * D) + c;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        for (int u = 0; u < S; ++u) {
            const uint4 v = __ldg(src + (long)u * C);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[2 * e] += bf16_lo_to_f32(w[e]);
                acc[2 * e + 1] += bf16_hi_to_f32(w[e]);
            }
        }
        uint32_t h4[4], l4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float x0 = acc[2 * e], x1 = acc[2 * e + 1];
            const float h0 = __bfloat162float(__float2bfloat16_rn(x0));
            const float h1 = __bfloat162float(__float2bfloat16_rn(x1));
            h4[e] = pack_bf16(h0, h1);
            l4[e] = pack_bf16(x0 - h0, x1 - h1);
        }
        reinterpret_cast<uint4 *>(hi + row * D)[c] = make_uint4(h4[0], h4[1], h4[2], h4[3]);
        reinterpret_cast<uint4 *>(lo + row * D)[c] = make_uint4(l4[0], l4[1], l4[2], l4[3]);
    }
}

struct EstTcParams {
    const uint16_t *Q;
    float *A;
    int H, L, S, Nb, Ns, G, hc, nHC, Hkv, QB, RB;
    int head_base, mode, layer;
    float c_log2;  // log2(e) / (S * sqrt(d))
};

template <int D>
struct EstTcCfg {
    static constexpr int DC = D / 64;
    static constexpr uint32_t T_BYTES = kTileN * D * 2;  // one hi or lo key tile
    static constexpr int NS = D == 128 ? 3 : 6;          // stages of (hi, lo) tiles
    static constexpr uint32_t BAR_OFF = NS * 2 * T_BYTES;  // the sampled rows live in TMEM
    // k_full[NS], k_empty[NS], s_full[2], s_free[2], fin, red_full[2], red_empty[2]
    static constexpr uint32_t NBAR = 2 * NS + 9;
    static constexpr uint32_t SMEM = BAR_OFF + NBAR * 8 + 16;
    static constexpr uint32_t IDESC = sm100::idesc_bf16(kRows, kTileN, false);
    static_assert(SMEM + 1024 <= 113u * 1024u, "two CTAs per SM");
};

template <int D, int R>
__global__ void __launch_bounds__(256, 2)
    estimate_tc_kernel(const __grid_constant__ CUtensorMap tmHi, const __grid_constant__ CUtensorMap tmLo,
                       const EstTcParams p) {
    using C = EstTcCfg<D>;
    constexpr int NS = C::NS;
    constexpr int NBT = kTileN / R;  // key blocks per tile
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sK = smem_u32(base);  // ring of (hi, lo) key tiles
    auto sHi = [&](int s) { return sK + s * 2 * C::T_BYTES; };
    auto sLo = [&](int s) { return sK + s * 2 * C::T_BYTES + C::T_BYTES; };
    constexpr uint32_t Q_COL = 2 * kTileN;  // TMEM columns of the sampled rows (bf16 pairs)
    const uint32_t sBar = sK + C::BAR_OFF;
    auto k_full = [&](int s) { return sBar + 8u * s; };
    auto k_empty = [&](int s) { return sBar + 8u * (NS + s); };
    auto s_full = [&](int b) { return sBar + 8u * (2 * NS + b); };
    auto s_free = [&](int b) { return sBar + 8u * (2 * NS + 2 + b); };
    const uint32_t fin_bar = sBar + 8u * (2 * NS + 4);
    // B/S > 32: a (head, query block)'s rows span B/S/32 warps, whose partial block sums meet
    // in red[tile parity][warp] (lane 0 of each warp writes, the group's first warp reads)
    auto red_full = [&](int b) { return sBar + 8u * (2 * NS + 5 + b); };
    auto red_empty = [&](int b) { return sBar + 8u * (2 * NS + 7 + b); };
    __shared__ float red[2][4];
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + C::BAR_OFF + C::NBAR * 8);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // CTA -> (query-block group, KV head, head chunk), longest rows first
    const int nQG = (p.Nb + p.QB - 1) / p.QB;
    const int lin = blockIdx.x;
    const int qg = nQG - 1 - lin / (p.Hkv * p.nHC);
    const int rem = lin % (p.Hkv * p.nHC);
    const int g = rem / p.nHC, hci = rem % p.nHC;
    const int I0 = qg * p.QB;
    const int nqb = min(p.QB, p.Nb - I0);
    const int nrows = nqb * p.RB;
    const int nT = ((I0 + nqb) * R + kTileN - 1) / kTileN;  // tiles covering strides < (I0+nqb)*r

    if (tid == 32) {
        for (int s = 0; s < NS; ++s) {
            sm100::mbar_init(k_full(s), 1);
            sm100::mbar_init(k_empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            sm100::mbar_init(s_full(b), 1);
            sm100::mbar_init(s_free(b), 128);
        }
        sm100::mbar_init(fin_bar, 1);
        for (int b = 0; b < 2; ++b) {
            sm100::mbar_init(red_full(b), 4);
            sm100::mbar_init(red_empty(b), R > 32 ? kRows / R : 1);
        }
        sm100::fence_mbar_init();
    }
    if (warp == 0) {
        sm100::tmem_alloc(smem_u32(tmem_slot), 4 * kTileN);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // Stage the sampled rows into TMEM (the MMA's A operand): row rho = qb*RB + hh*r + ii, the
    // sample of stride i = (I0+qb)*r + ii of head g*G + hci*hc + hh, in lane rho, two bf16 per
    // column.  Warps 4-7 own the four lane quadrants.
    if (warp >= 4) {
        const int rho = (warp & 3) * 32 + lane;
        uint32_t w[D / 2];
        if (rho < nrows) {
            const int qb = rho / p.RB, rr_ = rho % p.RB, hh = rr_ / R, ii = rr_ % R;
            const int h = g * p.G + hci * p.hc + hh;
            const long i = (long)(I0 + qb) * R + ii;
            const long pos = i * p.S + rr_offset(p.head_base + h, p.S, p.mode, p.layer);
            const uint4 *src = reinterpret_cast<const uint4 *>(p.Q + ((long)h * p.L + pos) * D);
#pragma unroll
            for (int u = 0; u < D / 8; ++u) {
                const uint4 v = __ldg(src + u);
                w[4 * u] = v.x, w[4 * u + 1] = v.y, w[4 * u + 2] = v.z, w[4 * u + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < D / 2; ++k) w[k] = 0u;
        }
        const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
#pragma unroll
        for (int cc = 0; cc < D / 64; ++cc)
            sm100::tmem_st32(trow + Q_COL + cc * 32, *reinterpret_cast<const uint32_t(*)[32]>(w + cc * 32));
        sm100::tmem_wait_st();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const int nq = 2 * nT;  // tile visits over both passes

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------------- producer
            sm100::prefetch_tmap(&tmHi);
            sm100::prefetch_tmap(&tmLo);
            int q = 0;
            bool ok = true;
            for (; q < nq; ++q) {
                const int s = q % NS;
                if (!sm100::mbar_wait(k_empty(s), ((q / NS) & 1) ^ 1)) {
                    ok = false;
                    break;
                }
                const int row0 = g * p.Ns + (q % nT) * kTileN;
                sm100::mbar_arrive_expect_tx(k_full(s), 2 * C::T_BYTES);
                for (int c = 0; c < C::DC; ++c) {
                    sm100::tma_load_2d(sHi(s) + c * kTileN * 128, &tmHi, c * 64, row0, k_full(s));
                    sm100::tma_load_2d(sLo(s) + c * kTileN * 128, &tmLo, c * 64, row0, k_full(s));
                }
            }
            if (!ok) {
                atomicOr(&g_est_errors, kErrTimeoutEstimate);
                for (int t = q > NS ? q - NS : 0; t < q; ++t) sm100::mbar_wait(k_full(t % NS), (t / NS) & 1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            bool ok = true;
            for (int q = 0; q < nq; ++q) {
                const int s = q % NS, b = q & 1;
                // buffer b is free once the softmax has loaded the tile two visits back
                if (!sm100::mbar_wait(s_free(b), ((q >> 1) & 1) ^ 1) ||
                    !sm100::mbar_wait(k_full(s), (q / NS) & 1)) {
                    ok = false;
                    break;
                }
                sm100::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int c = kk >> 2, w4 = kk & 3;
                    const uint64_t bd = sm100::smem_desc_sw128(sHi(s) + c * kTileN * 128 + w4 * 32, 16, 1024);
                    sm100::mma_ts(tmem + b * kTileN, tmem + Q_COL + kk * 8, bd, C::IDESC, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int c = kk >> 2, w4 = kk & 3;
                    const uint64_t bd = sm100::smem_desc_sw128(sLo(s) + c * kTileN * 128 + w4 * 32, 16, 1024);
                    sm100::mma_ts(tmem + b * kTileN, tmem + Q_COL + kk * 8, bd, C::IDESC, 1);
                }
                sm100::mma_commit(k_empty(s));
                sm100::mma_commit(s_full(b));
            }
            sm100::mma_commit(fin_bar);
            if (!sm100::mbar_wait(fin_bar, 0)) ok = false;
            if (!ok) atomicOr(&g_est_errors, kErrTimeoutEstimate);
        }
    } else if (warp >= 4) {
        // -------------------------------------------------------------------- softmax
        const int row = (warp & 3) * 32 + lane;  // = TMEM lane
        const bool valid = row < nrows;
        const int qb = row / p.RB, rr_ = row % p.RB, hh = rr_ / R, ii = rr_ % R;
        const int I = I0 + qb;
        const long irow = (long)I * R + ii;  // the row's stride index
        const int h = g * p.G + hci * p.hc + hh;
        float *arow = p.A + ((long)h * p.Nb + I) * p.Nb;
        const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const float c = p.c_log2;
        float m = -INFINITY, l = 0.f, mL = 0.f;
        float blk = 0.f;  // r > 32: a key block's sum over its tiles (the group's first warp)
        bool ok = true;
        for (int q = 0; q < nq; ++q) {
            const int b = q & 1;
            ok = __all_sync(0xffffffffu, sm100::mbar_wait(s_full(b), (q >> 1) & 1));
            if (!ok) break;
            sm100::tc_fence_after();
            uint32_t sr[kTileN];
#pragma unroll
            for (int cc = 0; cc < kTileN / 32; ++cc)
                sm100::tmem_ld32(trow + b * kTileN + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(sr + cc * 32));
            sm100::tmem_wait_ld();
            sm100::tc_fence_before();
            sm100::mbar_arrive(s_free(b));
            const long j0 = (long)(q % nT) * kTileN;
            // strides j > i are outside the stride-level causal mask
            const int nvis = (int)max(0L, min((long)kTileN, irow - j0 + 1));
            if (q < nT) {
                // pass 1: running max and sum of exp2 (the sum is rescaled only when the max
                // grows by more than 2^8)
                float mx = -INFINITY;
#pragma unroll
                for (int j = 0; j < kTileN; ++j)
                    if (j < nvis) mx = fmaxf(mx, __uint_as_float(sr[j]) * c);
                if (mx > m + 8.f) {
                    l *= ex2_approx(m - mx);  // 0 while nothing was seen
                    m = mx;
                }
                float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int j = 0; j < kTileN; ++j)
                    s4[j & 3] += (j < nvis) ? ex2_approx(fmaf(__uint_as_float(sr[j]), c, -m)) : 0.f;
                l += (s4[0] + s4[1]) + (s4[2] + s4[3]);
                if (q == nT - 1) mL = (l > 0.f) ? m + log2f(l) : INFINITY;  // p = 2^(s*c - mL)
            } else if constexpr (R <= 32) {
                // pass 2: exact probabilities summed per key block, reduced over the r rows of
                // the (head, query block) -- r lanes of one warp -- times S/B
                float bs[NBT];
#pragma unroll
                for (int k = 0; k < NBT; ++k) {
                    float acc = 0.f;
#pragma unroll
                    for (int jj = 0; jj < R; ++jj) {
                        const int j = k * R + jj;
                        acc += (j < nvis) ? ex2_approx(fmaf(__uint_as_float(sr[j]), c, -mL)) : 0.f;
                    }
                    bs[k] = valid ? acc : 0.f;
                }
#pragma unroll
                for (int o = 1; o < R; o <<= 1)
#pragma unroll
                    for (int k = 0; k < NBT; ++k) bs[k] += __shfl_xor_sync(0xffffffffu, bs[k], o);
                const int J0 = (q - nT) * NBT;
                if (valid) {
#pragma unroll
                    for (int k = 0; k < NBT; ++k)
                        if (k % R == ii && J0 + k < p.Nb) arow[J0 + k] = bs[k] * (1.f / R);
                }
            } else {
                // pass 2 for r = 64 or 128: the tile lies inside one key block (r/64 tiles per
                // block) and the block's r rows span r/32 warps; each warp reduces its 32
                // rows, the group's first warp adds the warps' sums in a fixed order
                constexpr int TPB = R / kTileN, WPG = R / 32;
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < kTileN; ++j)
                    acc += (j < nvis) ? ex2_approx(fmaf(__uint_as_float(sr[j]), c, -mL)) : 0.f;
                acc = valid ? acc : 0.f;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                const int u = q - nT, par = u & 1, use = u >> 1, wq = warp & 3;
                if (lane == 0) {
                    // the slot's previous use has been read
                    if (sm100::mbar_wait(red_empty(par), (use & 1) ^ 1)) {
                        red[par][wq] = acc;
                        sm100::mbar_arrive(red_full(par));
                    } else {
                        atomicOr(&g_est_errors, kErrTimeoutEstimate);
                    }
                    if (wq % WPG == 0) {  // the group's first warp
                        if (sm100::mbar_wait(red_full(par), use & 1)) {
                            float tot = 0.f;
#pragma unroll
                            for (int w = 0; w < WPG; ++w) tot += red[par][wq + w];
                            sm100::mbar_arrive(red_empty(par));
                            blk += tot;
                            if (u % TPB == TPB - 1) {
                                const int J = u / TPB;
                                if (valid && J < p.Nb) arow[J] = blk * (1.f / R);
                                blk = 0.f;
                            }
                        } else {
                            atomicOr(&g_est_errors, kErrTimeoutEstimate);
                        }
                    }
                }
            }
        }
        if (!ok) {
            if (lane == 0) atomicOr(&g_est_errors, kErrTimeoutEstimate);
        } else if (valid) {
            // blocks past the last tile are above the diagonal: zero
            for (int J = nT * kTileN / R + ii; J < p.Nb; J += R) arow[J] = 0.f;
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();  // lane 0 ran the producer; dealloc is warp-collective
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, 4 * kTileN);
    }
}

// Rows per CTA: QB query blocks of hc heads each, hc the largest divisor of G with
// hc * r <= 128.
void plan_tc(int G, int r, int *hc, int *QB) {
    int best = 1;
    for (int c = 1; c <= G; ++c)
        if (G % c == 0 && c * r <= kRows) best = c;
    *hc = best;
    *QB = kRows / (best * r);
}

template <int D, int R>
rr_status_t launch_tc_r(const CUtensorMap &mhi, const CUtensorMap &mlo, const EstTcParams &p,
                        cudaStream_t st) {
    using C = EstTcCfg<D>;
    auto kern = estimate_tc_kernel<D, R>;
    const size_t smem = C::SMEM + 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return set_error(RR_ERR_CUDA, "rr_estimate: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    const long ctas = (long)p.Hkv * p.nHC * ((p.Nb + p.QB - 1) / p.QB);
    kern<<<(unsigned)ctas, 256, smem, st>>>(mhi, mlo, p);
    return check_launch("rr_estimate: estimate_tc_kernel");
}

}  // namespace

size_t estimate_workspace_bytes(int Hkv, int L, int d, int S) {
    if (L <= 0) return 0;
    return (size_t)Hkv * (L / S) * d * 4;  // bf16 hi + lo per pooled element
}

// Every size the ABI accepts (d in {64, 128}, B/S in {4, 8, 16, 32, 64, 128}) has a kernel.
bool estimate_supported(int H, int Hkv, int d, int S, int B, int L) {
    (void)H, (void)Hkv, (void)L;
    const int r = B / S;
    return (d == 64 || d == 128) && (r == 4 || r == 8 || r == 16 || r == 32 || r == 64 || r == 128);
}

rr_status_t launch_estimate(const uint16_t *Q, const uint16_t *K, int H, int Hkv, int L, int d,
                            int S, int B, int mode, int layer, int head_base, float *A, void *ws,
                            cudaStream_t st) {
    const int Ns = L / S, Nb = L / B, r = B / S, G = H / Hkv;
    uint16_t *hi = static_cast<uint16_t *>(ws);
    uint16_t *lo = hi + (size_t)Hkv * Ns * d;
    {
        const long total = (long)Hkv * Ns * (d / 8);
        const long want = (total + 255) / 256;
        const int blocks = (int)(want < 148L * 16 ? want : 148L * 16);
        if (d == 128)
            pool_keys_rows_kernel<128><<<blocks, 256, 0, st>>>(K, L, S, Ns, Hkv, hi, lo);
        else
            pool_keys_rows_kernel<64><<<blocks, 256, 0, st>>>(K, L, S, Ns, Hkv, hi, lo);
        const rr_status_t s = check_launch("rr_estimate: pool_keys_rows_kernel");
        if (s != RR_OK) return s;
    }
    alignas(64) CUtensorMap mhi, mlo;
    if (!make_tmap_bf16(&mhi, hi, (uint64_t)Hkv * Ns, d, kTileN) ||
        !make_tmap_bf16(&mlo, lo, (uint64_t)Hkv * Ns, d, kTileN))
        return set_error(RR_ERR_CUDA, "rr_estimate: cuTensorMapEncodeTiled failed");
    EstTcParams p;
    p.Q = Q;
    p.A = A;
    p.H = H;
    p.L = L;
    p.S = S;
    p.Nb = Nb;
    p.Ns = Ns;
    p.G = G;
    p.Hkv = Hkv;
    plan_tc(G, r, &p.hc, &p.QB);
    p.nHC = G / p.hc;
    p.RB = p.hc * r;
    p.head_base = head_base;
    p.mode = mode;
    p.layer = layer;
    p.c_log2 = (float)(1.4426950408889634 / ((double)S * sqrt((double)d)));
    if (d == 128) {
        switch (r) {
        case 4: return launch_tc_r<128, 4>(mhi, mlo, p, st);
        case 8: return launch_tc_r<128, 8>(mhi, mlo, p, st);
        case 16: return launch_tc_r<128, 16>(mhi, mlo, p, st);
        case 32: return launch_tc_r<128, 32>(mhi, mlo, p, st);
        case 64: return launch_tc_r<128, 64>(mhi, mlo, p, st);
        default: return launch_tc_r<128, 128>(mhi, mlo, p, st);
        }
    }
    switch (r) {
    case 4: return launch_tc_r<64, 4>(mhi, mlo, p, st);
    case 8: return launch_tc_r<64, 8>(mhi, mlo, p, st);
    case 16: return launch_tc_r<64, 16>(mhi, mlo, p, st);
    case 32: return launch_tc_r<64, 32>(mhi, mlo, p, st);
    case 64: return launch_tc_r<64, 64>(mhi, mlo, p, st);
    default: return launch_tc_r<64, 128>(mhi, mlo, p, st);
    }
}

rr_status_t read_estimate_errors(unsigned *out, bool reset) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_est_errors, sizeof(unsigned));
    if (e == cudaSuccess && reset) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_est_errors, &zero, sizeof(unsigned));
    }
    if (e != cudaSuccess) return set_error(RR_ERR_CUDA, "rr_device_errors: %s", cudaGetErrorString(e));
    return RR_OK;
}

}  // namespace rr
