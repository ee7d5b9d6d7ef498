// Causal block-sparse attention over the selected blocks on the 5th-generation tensor cores
// ("RRAttention: Dynamic Block Sparse Attention via Per-Head Round-Robin Shifts for
// Long-Context Inference", Sec. 2.1 with the per-head CSR block lists as the block selection
// matrix; Sec. 4.1: sparsity in prefill only).
//
// B = 64 layers.  One CTA per (query head h, pair of query blocks 2p and 2p+1): a 128-row
// query tile whose rows 0-63 are block 2p and rows 64-127 block 2p+1, so no tensor-core row
// is padding.  The CTA walks the ascending union of the two blocks' CSR lists, one 64-key
// block per step; each softmax warp's 32 rows lie in one half, and a warp whose block's list
// lacks the step's key block masks that whole block (P = 0 for its rows).
// Two CTAs share an SM, so each SM sub-partition runs two independent softmax streams.
// Warp roles (224 threads):
//   warp 0      TMA producer of Q (once) and of the K tiles, into a ring of two or more
//               (128-byte swizzle, mbarrier transaction counts); L2 prefetch of upcoming
//               tiles; TMEM allocation / release.
//   warp 1      TMA producer of the V tiles (its own ring, so K loads never queue behind a V
//               slot that is still being read).
//   warp 2      MMA issuer (one thread): S_t = Q K_t^T (both operands in shared memory) into
//               the single S buffer as soon as the softmax has loaded S_{t-1}, so S_t is
//               computed while the softmax works on S_{t-1}; then O += P_t V_t with P_t read
//               from TMEM (the A-from-tensor-memory form).  Completion is signalled by
//               tcgen05.commit.
//   warps 3-6   softmax: one thread per query row (TMEM lane).  Online softmax in fp32 with a
//               lazily rescaled running max (O is rescaled in TMEM only when a row's max grows
//               by more than 2^8), P packed to bf16 pairs and stored into one of two TMEM P
//               buffers, final normalisation and bf16 store of O.
// TMEM columns (256 per CTA): S [0, 64) fp32, P0 and P1 [64, 128) bf16 pairs, O [128, 128+d).
// K and V come from KV head h / (H/Hkv); the heads of a KV group run as adjacent CTAs so
// their K/V tiles are served from L2.  Every wait is bounded (about one second of
// %globaltimer); a timeout sets a device error bit and the CTA drains and exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include "rr_common.cuh"
#include "rr_sm100.cuh"

namespace rr {

namespace {

__device__ unsigned int g_device_errors;

constexpr unsigned kErrTimeoutProducer = 1u, kErrTimeoutMma = 2u, kErrTimeoutSoftmax = 4u;

// max(a, b, c) in one instruction (sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float y;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
    return y;
}

// Packed pairs of fp32 (one 64-bit register, two lanes of the FMA pipe per instruction).
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 f2_pack(float lo, float hi) {
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(f32x2 v, float &lo, float &hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 f2_fma(f32x2 a, f32x2 b, f32x2 c) {
    f32x2 r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ f32x2 f2_add(f32x2 a, f32x2 b) {
    f32x2 r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

constexpr int kBM = 128;  // query rows per CTA
constexpr int kSub = 64;  // keys per sub-block: the unit of S, P and the K/V pipeline

// The two query blocks' CSR lists as bitmaps over the key blocks (shared memory, filled once):
// the steps of the CTA are the set bits of their union in ascending order.
constexpr int kBmWords = kMaxL / 64 / 32;  // bitmap words per list, enough for any layer B = 64 allows

// The union block after `cur` (-1 when there is none).
__device__ __forceinline__ int next_block(const uint32_t *bmL, const uint32_t *bmH, int W, int cur) {
    int w = (cur + 1) >> 5;
    if (w >= W) return -1;
    uint32_t m = (bmL[w] | bmH[w]) & (~0u << ((cur + 1) & 31));
    while (m == 0) {
        if (++w >= W) return -1;
        m = bmL[w] | bmH[w];
    }
    return (w << 5) + __ffs(m) - 1;
}

template <int D, int BN>
struct TcCfg {
    static constexpr int DC = D / 64;       // 64-element (128-byte) column chunks
    static constexpr uint32_t Q_BYTES = kBM * D * 2;
    static constexpr uint32_t SUB_BYTES = kSub * D * 2;  // one K or V sub-tile
    // Two CTAs per SM: each may use 113 KB of shared memory (1024 bytes of that are
    // alignment slack, 256 barriers); the rest holds K and V sub-tile rings.
    static constexpr int SLOTS = (int)((113u * 1024u - 1024u - 256u - 8u * kBmWords - Q_BYTES) / SUB_BYTES);
    static constexpr int NK = SLOTS / 2 > 4 ? 4 : SLOTS / 2;
    static constexpr int NV = NK;
    static constexpr int PF = 8;  // sub-blocks prefetched into L2 ahead of the shared-memory loads
    static constexpr uint32_t BAR_OFF = Q_BYTES + (NK + NV) * SUB_BYTES;
    // q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], s_full, s_free, p_full[2],
    // o_bar, fin
    static constexpr uint32_t NBAR = 1 + 2 * NK + 2 * NV + 6;
    static constexpr uint32_t BM_OFF = BAR_OFF + NBAR * 8 + 16;  // the two list bitmaps
    static constexpr uint32_t SMEM = BM_OFF + 8 * kBmWords;
    // at least 80 KB so that a third CTA never fits on an SM (3 x 80 KB > 228 KB): with two
    // CTAs of 256 TMEM columns each, a TMEM allocation never waits
    static constexpr uint32_t SMEM_LAUNCH = SMEM + 1024 > 80u * 1024u ? SMEM + 1024 : 80u * 1024u;
    // TMEM columns: S [0, 64) fp32 (one sub-block), P0 and P1 [64, 128) (bf16 pairs, 32 columns
    // each), O [128, 128 + D) fp32
    static constexpr uint32_t S_COL = 0, P_COL = kSub, O_COL = 2 * kSub;
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr uint32_t IDESC_S = sm100::idesc_bf16(kBM, kSub, false);
    static constexpr uint32_t IDESC_PV = sm100::idesc_bf16(kBM, D, true);
    static_assert(BN == kSub && 2 * BN == kBM, "two 64-row query blocks per tile, one 64-key block per step");
    static_assert(NK >= 2, "need at least two K and two V sub-tiles");
    static_assert(O_COL + D <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM + 1024 <= 113u * 1024u, "two CTAs per SM");
};

template <int D, int BN>
__global__ void __launch_bounds__(224, 2)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, uint16_t *__restrict__ O,
                      const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                      int H, int Hkv, int L, int Nb, float scale_log2) {
    using C = TcCfg<D, BN>;
    constexpr int NK = C::NK, NV = C::NV;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sQ = smem_u32(base);
    const uint32_t sK = sQ + C::Q_BYTES;
    const uint32_t sV = sK + NK * C::SUB_BYTES;
    const uint32_t sBar = sQ + C::BAR_OFF;
    const uint32_t q_full = sBar;
    auto k_full = [&](int s) { return sBar + 8u * (1 + s); };
    auto k_empty = [&](int s) { return sBar + 8u * (1 + NK + s); };
    auto v_full = [&](int s) { return sBar + 8u * (1 + 2 * NK + s); };
    auto v_empty = [&](int s) { return sBar + 8u * (1 + 2 * NK + NV + s); };
    const uint32_t s_full = sBar + 8u * (1 + 2 * NK + 2 * NV);
    const uint32_t s_free = s_full + 8;
    auto p_full = [&](int t) { return s_full + 16u + 8u * (t & 1); };
    const uint32_t o_bar = s_full + 32;
    const uint32_t fin_bar = s_full + 40;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + C::BAR_OFF + C::NBAR * 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Launch order: KV group by KV group, and inside a group pairs of query blocks from the
    // longest CSR rows down with the group's heads adjacent.  CTAs resident at the same time
    // then stream one KV head's K/V, which stays in L2.
    const int G = H / Hkv, NPR = (Nb + 1) / 2;
    const long lin = blockIdx.x;
    const int g = (int)(lin / ((long)G * NPR));
    const int within = (int)(lin % ((long)G * NPR));
    const int I_lo = 2 * (NPR - 1 - within / G), I_hi = I_lo + 1;  // I_hi == Nb: no upper block
    const int h = g * G + within % G;
    const long crow = (long)h * Nb + I_lo;
    const int eL = row_ptr[crow], nL = row_ptr[crow + 1] - eL;
    const int eH = I_hi < Nb ? row_ptr[crow + 1] : 0;
    const int nH = I_hi < Nb ? row_ptr[crow + 2] - eH : 0;
    const int32_t *listL = col_idx + eL, *listH = col_idx + eH;
    uint32_t *bmL = reinterpret_cast<uint32_t *>(base + C::BM_OFF), *bmH = bmL + kBmWords;
    const int W = (Nb + 31) / 32;
    for (int w = threadIdx.x; w < 2 * W; w += blockDim.x) (w < W ? bmL[w] : bmH[w - W]) = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < nL + nH; i += blockDim.x) {
        const int J = i < nL ? __ldg(listL + i) : __ldg(listH + i - nL);
        atomicOr((i < nL ? bmL : bmH) + (J >> 5), 1u << (J & 31));
    }

    if (threadIdx.x == 64) {
        sm100::mbar_init(q_full, 1);
        for (int s = 0; s < NK; ++s) {
            sm100::mbar_init(k_full(s), 1);
            sm100::mbar_init(k_empty(s), 1);
        }
        for (int s = 0; s < NV; ++s) {
            sm100::mbar_init(v_full(s), 1);
            sm100::mbar_init(v_empty(s), 1);
        }
        sm100::mbar_init(s_full, 1);
        sm100::mbar_init(s_free, 128);
        sm100::mbar_init(p_full(0), 128);
        sm100::mbar_init(p_full(1), 128);
        sm100::mbar_init(o_bar, 1);
        sm100::mbar_init(fin_bar, 1);
        sm100::fence_mbar_init();
    }
    if (warp == 0) {
        sm100::tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // steps: the blocks of the union (every warp counts them, 32 bitmap words per lane step)
    int nsub = 0;
    for (int w = lane; w < W; w += 32) nsub += __popc(bmL[w] | bmH[w]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) nsub += __shfl_xor_sync(0xffffffffu, nsub, o);

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------- K producer (and Q)
            sm100::prefetch_tmap(&tmQ);
            sm100::prefetch_tmap(&tmK);
            sm100::prefetch_tmap(&tmV);
            sm100::mbar_arrive_expect_tx(q_full, C::Q_BYTES);
            for (int c = 0; c < C::DC; ++c)
                sm100::tma_load_2d(sQ + c * kBM * 128, &tmQ, c * 64, h * L + I_lo * BN, q_full);
            int ja = -1, J = -1;  // prefetch cursor (PF blocks ahead) and load cursor
            for (int t = 0; t < C::PF && (ja = next_block(bmL, bmH, W, ja)) >= 0; ++t)
                for (int c = 0; c < C::DC; ++c) {
                    sm100::tma_prefetch_2d(&tmK, c * 64, g * L + ja * BN);
                    sm100::tma_prefetch_2d(&tmV, c * 64, g * L + ja * BN);
                }
            int issued = 0;
            bool ok = true;
            for (int t = 0; t < nsub; ++t) {
                if (ja >= 0 && (ja = next_block(bmL, bmH, W, ja)) >= 0)
                    for (int c = 0; c < C::DC; ++c) {
                        sm100::tma_prefetch_2d(&tmK, c * 64, g * L + ja * BN);
                        sm100::tma_prefetch_2d(&tmV, c * 64, g * L + ja * BN);
                    }
                const int s = t % NK;
                J = next_block(bmL, bmH, W, J);
                const int y = g * L + J * BN;
                if (!sm100::mbar_wait(k_empty(s), ((t / NK) & 1) ^ 1)) {  // S_{t-NK} has completed
                    ok = false;
                    break;
                }
                sm100::mbar_arrive_expect_tx(k_full(s), C::SUB_BYTES);
                for (int c = 0; c < C::DC; ++c)
                    sm100::tma_load_2d(sK + s * C::SUB_BYTES + c * kSub * 128, &tmK, c * 64, y, k_full(s));
                issued = t + 1;
            }
            if (!ok) {
                atomicOr(&g_device_errors, kErrTimeoutProducer);
                // let the copies already in flight land before the CTA's memory is released
                sm100::mbar_wait(q_full, 0);
                for (int t = issued > NK ? issued - NK : 0; t < issued; ++t)
                    sm100::mbar_wait(k_full(t % NK), (t / NK) & 1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------- V producer
            int issued = 0, J = -1;
            bool ok = true;
            for (int t = 0; t < nsub; ++t) {
                const int s = t % NV;
                J = next_block(bmL, bmH, W, J);
                const int y = g * L + J * BN;
                if (!sm100::mbar_wait(v_empty(s), ((t / NV) & 1) ^ 1)) {  // P_{t-NV} V_{t-NV} has completed
                    ok = false;
                    break;
                }
                sm100::mbar_arrive_expect_tx(v_full(s), C::SUB_BYTES);
                for (int c = 0; c < C::DC; ++c)
                    sm100::tma_load_2d(sV + s * C::SUB_BYTES + c * kSub * 128, &tmV, c * 64, y, v_full(s));
                issued = t + 1;
            }
            if (!ok) {
                atomicOr(&g_device_errors, kErrTimeoutProducer);
                for (int t = issued > NV ? issued - NV : 0; t < issued; ++t)
                    sm100::mbar_wait(v_full(t % NV), (t / NV) & 1);
            }
        }
    } else if (warp == 2) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            bool ok = sm100::mbar_wait(q_full, 0);
            sm100::tc_fence_after();
            auto issue_s = [&](int t) -> bool {
                const int s = t % NK;
                if (!sm100::mbar_wait(k_full(s), (t / NK) & 1)) return false;
                sm100::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int c = kk >> 2, w = kk & 3;
                    const uint64_t ad = sm100::smem_desc_sw128(sQ + c * kBM * 128 + w * 32, 16, 1024);
                    const uint64_t bd =
                        sm100::smem_desc_sw128(sK + s * C::SUB_BYTES + c * kSub * 128 + w * 32, 16, 1024);
                    sm100::mma_ss(tmem + C::S_COL, ad, bd, C::IDESC_S, kk > 0);
                }
                sm100::mma_commit(k_empty(s));
                sm100::mma_commit(s_full);
                return true;
            };
            if (ok && nsub > 0) ok = issue_s(0);
            for (int t = 0; ok && t < nsub; ++t) {
                // S_{t+1} goes into the S columns once every softmax thread has loaded S_t
                if (t + 1 < nsub && !(sm100::mbar_wait(s_free, t & 1) && issue_s(t + 1))) {
                    ok = false;
                    break;
                }
                if (!sm100::mbar_wait(p_full(t), (t >> 1) & 1) || !sm100::mbar_wait(v_full(t % NV), (t / NV) & 1)) {
                    ok = false;
                    break;
                }
                sm100::tc_fence_after();
                const int s = t % NV;
#pragma unroll
                for (int kk = 0; kk < kSub / 16; ++kk) {
                    const uint64_t bd =
                        sm100::smem_desc_sw128(sV + s * C::SUB_BYTES + kk * 16 * 128, kSub * 128, 1024);
                    sm100::mma_ts(tmem + C::O_COL, tmem + C::P_COL + (t & 1) * (kSub / 2) + kk * 8, bd,
                                  C::IDESC_PV, (t > 0 || kk > 0));
                }
                sm100::mma_commit(o_bar);
                sm100::mma_commit(v_empty(s));
            }
            // fin_bar: every MMA has completed (the epilogue reads O, then the TMEM is released)
            sm100::mma_commit(fin_bar);
            if (!sm100::mbar_wait(fin_bar, 0)) ok = false;
            if (!ok) atomicOr(&g_device_errors, kErrTimeoutMma);
        }
    } else {
        // -------------------------------------------------------------------- softmax
        // warps 3-6; a warp may only touch TMEM lanes 32*(warp % 4) .. +31
        const int r = (warp & 3) * 32 + lane;  // query row within the tile = TMEM lane
        const bool upper = r >= BN;             // the warp's rows are all in one half
        const int Iown = upper ? I_hi : I_lo, rb = r - (upper ? BN : 0);
        const long qpos = (long)I_lo * BN + r;
        const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        const uint32_t *bmOwn = upper ? bmH : bmL;
        int J = -1;
        for (int t = 0; t < nsub; ++t) {
            J = next_block(bmL, bmH, W, J);
            const bool mine = (bmOwn[J >> 5] >> (J & 31)) & 1u;  // warp-uniform
            ok = __all_sync(0xffffffffu, sm100::mbar_wait(s_full, t & 1));
            if (!ok) break;
            sm100::tc_fence_after();
            uint32_t sr[kSub];
            sm100::tmem_ld32(trow + C::S_COL, *reinterpret_cast<uint32_t(*)[32]>(sr));
            sm100::tmem_ld32(trow + C::S_COL + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
            sm100::tmem_wait_ld();
            // S_t is in registers: the MMA warp may write S_{t+1}
            sm100::tc_fence_before();
            sm100::mbar_arrive(s_free);
            // keys i > lim are masked: none (lim = 63), those after the row on its diagonal block,
            // or all of a block this half's list does not hold (lim = -1)
            const int lim = !mine ? -1 : (J == Iown ? rb : kSub - 1);
            if (lim < kSub - 1) {
#pragma unroll
                for (int i = 0; i < kSub; ++i)
                    if (i > lim) sr[i] = __float_as_uint(-INFINITY);
            }
            // row max: four chains of three-input maxima
            float mq[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) mq[k] = __uint_as_float(sr[k]);
#pragma unroll
            for (int i = 4; i + 8 <= kSub; i += 8)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    mq[k] = fmax3(mq[k], __uint_as_float(sr[i + 2 * k]), __uint_as_float(sr[i + 2 * k + 1]));
            mq[0] = fmax3(mq[0], __uint_as_float(sr[kSub - 4]), __uint_as_float(sr[kSub - 3]));
            mq[1] = fmax3(mq[1], __uint_as_float(sr[kSub - 2]), __uint_as_float(sr[kSub - 1]));
            const float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])) * scale_log2;  // scale > 0
            // Lazy rescale: a row keeps its stale max while p <= 2^8.  The decision is per row,
            // but tcgen05.ld/st are warp-collective, so the O rescale (after the exponentials,
            // below) runs for the whole warp whenever any of its rows needs it (alpha = 1 on
            // the others), once P_{t-1} V_{t-1} is complete.
            const bool need = mx > m + 8.f;
            float alpha = 1.f;
            if (need) {
                alpha = ex2_approx(m - mx);  // 0 on a row's first sub-block
                l *= alpha;
                m = mx;
            }
            // P_t goes to the buffer P_{t-2} used.  Its P*V product is complete: S_t was issued
            // after P_{t-2} V_{t-2}, and the commit behind S_t (waited for above) fires only
            // once every earlier MMA of the issuing thread is done.
            const float nm = (m == -INFINITY) ? 0.f : -m;  // a row with nothing attended yet
            const f32x2 sc2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(nm, nm);
            f32x2 rs2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
            uint32_t pk[kSub / 2];
#pragma unroll
            for (int e = 0; e < kSub / 2; ++e) {
                const f32x2 x2 = f2_fma(f2_pack(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])),
                                        sc2, nm2);
                float x0, x1;
                f2_unpack(x2, x0, x1);
                const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                rs2[e & 1] = f2_add(rs2[e & 1], f2_pack(p0, p1));
                pk[e] = pack_bf16(p0, p1);
            }
            sm100::tmem_st32(trow + C::P_COL + (t & 1) * (kSub / 2), pk);
            float ra, rb, rc, rd;
            f2_unpack(rs2[0], ra, rb);
            f2_unpack(rs2[1], rc, rd);
            l += (ra + rb) + (rc + rd);
            if (t > 0 && __any_sync(0xffffffffu, need)) {
                ok = __all_sync(0xffffffffu, sm100::mbar_wait(o_bar, (t - 1) & 1));
                if (!ok) break;
                sm100::tc_fence_after();
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t rg[32];
                    sm100::tmem_ld32(trow + C::O_COL + cc * 32, rg);
                    sm100::tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) rg[i] = __float_as_uint(__uint_as_float(rg[i]) * alpha);
                    sm100::tmem_st32(trow + C::O_COL + cc * 32, rg);
                }
            }
            sm100::tmem_wait_st();
            sm100::tc_fence_before();
            sm100::mbar_arrive(p_full(t));
        }
        // O is final once every MMA has completed.  (o_bar cannot say so: when the last
        // softmax step ends, only the P*V of two steps earlier is known to be complete, so the
        // barrier may still be two phases short and a parity wait on it would alias.)
        if (ok) {
            ok = __all_sync(0xffffffffu, sm100::mbar_wait(fin_bar, 0));
            sm100::tc_fence_after();
        }
        if (!ok) {
            if (lane == 0) atomicOr(&g_device_errors, kErrTimeoutSoftmax);
        } else {
            // a row that attended nothing (an empty CSR row) is written as zeros: its O columns
            // in TMEM were never written
            const float inv = (l > 0.f) ? 1.f / l : 0.f;
            uint16_t *orow = O + ((long)h * L + qpos) * D;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t rg[32];
                if (nsub > 0) {
                    sm100::tmem_ld32(trow + C::O_COL + cc * 32, rg);
                    sm100::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) rg[i] = 0u;
                }
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16(__uint_as_float(rg[2 * i]) * inv, __uint_as_float(rg[2 * i + 1]) * inv);
                if (!upper || I_hi < Nb) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + cc * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                }
            }
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();  // lane 0 ran the producer; dealloc is warp-collective
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <int D, int BN>
rr_status_t launch_tc(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int H, int Hkv, int L,
                      const int32_t *row_ptr, const int32_t *col_idx, float scale, uint16_t *O,
                      cudaStream_t st) {
    using C = TcCfg<D, BN>;
    CUtensorMap mq, mk, mv;
    if (!make_tmap_bf16(&mq, Q, (uint64_t)H * L, D, kBM) || !make_tmap_bf16(&mk, K, (uint64_t)Hkv * L, D, kSub) ||
        !make_tmap_bf16(&mv, V, (uint64_t)Hkv * L, D, kSub))
        return set_error(RR_ERR_CUDA, "rr_sparse_prefill: cuTensorMapEncodeTiled failed");
    const size_t smem = C::SMEM_LAUNCH;
    auto kern = prefill_tc_kernel<D, BN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return set_error(RR_ERR_CUDA, "rr_sparse_prefill: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    const int Nb = L / BN;
    dim3 grid((unsigned)((long)H * ((Nb + 1) / 2)));
    kern<<<grid, 224, smem, st>>>(mq, mk, mv, O, row_ptr, col_idx, H, Hkv, L, Nb,
                                  scale * 1.4426950408889634f);
    return check_launch("rr_sparse_prefill: prefill_tc_kernel");
}

}  // namespace

rr_status_t launch_prefill_pp(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int H, int Hkv,
                              int L, int d, const int32_t *row_ptr, const int32_t *col_idx, float scale,
                              uint16_t *O, cudaStream_t st);

// B = 128: two query tiles per CTA (rr_prefill_pp.cu); B = 64: this file's one-tile kernel.
rr_status_t launch_prefill_tc(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int H, int Hkv,
                              int L, int d, int B, const int32_t *row_ptr, const int32_t *col_idx,
                              float scale, uint16_t *O, cudaStream_t st) {
    if (B == 128) return launch_prefill_pp(Q, K, V, H, Hkv, L, d, row_ptr, col_idx, scale, O, st);
    if (d == 128) return launch_tc<128, 64>(Q, K, V, H, Hkv, L, row_ptr, col_idx, scale, O, st);
    return launch_tc<64, 64>(Q, K, V, H, Hkv, L, row_ptr, col_idx, scale, O, st);
}

rr_status_t read_device_errors(unsigned *out, bool reset) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_device_errors, sizeof(unsigned));
    if (e == cudaSuccess && reset) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_device_errors, &zero, sizeof(unsigned));
    }
    if (e != cudaSuccess)
        return set_error(RR_ERR_CUDA, "rr_device_errors: %s", cudaGetErrorString(e));
    return RR_OK;
}

}  // namespace rr
