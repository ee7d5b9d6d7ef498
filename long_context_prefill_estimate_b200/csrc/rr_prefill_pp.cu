// Causal block-sparse attention over the selected blocks, two query tiles per CTA
// ("RRAttention: Dynamic Block Sparse Attention via Per-Head Round-Robin Shifts for
// Long-Context Inference", Sec. 2.1 with the per-head CSR block lists as the block selection
// matrix; Sec. 4.1: sparsity in prefill only).
//
// Work unit: two query tiles of one query head, query blocks I and I-1 (128 rows each, B =
// 128), one CTA per SM (the whole 512-column tensor memory).  Both tiles read the same KV head,
// and their block lists are walked as one merged, ascending union: every key block of the
// union is loaded into shared memory once and serves each tile whose list holds it.
//
// Per tile the chain is serial: S = Q K^T into the tile's S columns, softmax, P (bf16) written
// over the first half of those columns, O += P V with P read from tensor memory, then the next
// S into the same columns (the MMAs of one thread execute in order, so it never overwrites P
// before the P V product has read it).  While one tile's softmax runs, the tensor core can
// compute the other tile's P V and next S.
//
// Warp roles (384 threads):
//   warp 0      TMA producer of Q (both tiles, once) and of the K tiles of the union (ring of
//               NK), L2 prefetch of upcoming tiles, TMEM allocation / release.
//   warp 1      TMA producer of the V tiles of the union (ring of NV).
//   warp 2      MMA issuer (one thread).  For each union block u, for tile A then tile B:
//               first the P V of the tile's previous block (once its softmax published P),
//               then, if the tile's list holds u, its S for u.  The commit behind a tile's S
//               tells its softmax that S is ready and that every earlier MMA of the tile
//               (the P V that last wrote O) has completed.
//   warp 3      idle after set-up.
//   warps 4-7   softmax of tile A, warps 8-11 softmax of tile B: one thread per query row
//               (TMEM lane), online softmax in fp32 with a lazily rescaled running max (O is
//               rescaled in TMEM only when a row's max grows by more than 2^8), final
//               normalisation and bf16 store of O.
// TMEM columns (512): S/P of tile A [0, 128), S/P of tile B [128, 256), O_A [256, 256 + d),
// O_B [256 + d, 256 + 2d).  Every wait is bounded (about one second of %globaltimer); a
// timeout sets a device error bit and the CTA drains and exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include <climits>

#include "rr_common.cuh"
#include "rr_sm100.cuh"

namespace rr {

namespace {

__device__ unsigned int g_pp_errors;

constexpr unsigned kErrTimeoutProducer = 1u, kErrTimeoutMma = 2u, kErrTimeoutSoftmax = 4u;

constexpr int kRowsPP = 128;  // query rows per tile
constexpr int kBlk = 128;     // keys per block: one S tile
constexpr int kThreadsPP = 384;

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float y;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(y) : "f"(a), "f"(b), "f"(c));
    return y;
}

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

// The merged, ascending union of two ascending block lists; next() yields each block once
// with the lists that hold it.  Each list's next two entries are held in registers and the
// entry after them is loaded when one is consumed, so a load is issued a union step before
// its value is needed and the MMA issuer does not wait on global memory between steps.
struct UnionWalk {
    const int32_t *a, *b;
    int na, nb, ia, ib;
    int a0, a1, b0, b1;  // a[ia], a[ia+1], b[ib], b[ib+1]; INT_MAX past the end
    __device__ UnionWalk(const int32_t *a_, int na_, const int32_t *b_, int nb_)
        : a(a_), b(b_), na(na_), nb(nb_), ia(0), ib(0) {
        a0 = na > 0 ? __ldg(a) : INT_MAX;
        a1 = na > 1 ? __ldg(a + 1) : INT_MAX;
        b0 = nb > 0 ? __ldg(b) : INT_MAX;
        b1 = nb > 1 ? __ldg(b + 1) : INT_MAX;
    }
    __device__ __forceinline__ bool next(int &J, bool &inA, bool &inB) {
        if (a0 == INT_MAX && b0 == INT_MAX) return false;
        J = min(a0, b0);
        inA = a0 == J;
        inB = b0 == J;
        if (inA) {
            ++ia;
            a0 = a1;
            a1 = ia + 1 < na ? __ldg(a + ia + 1) : INT_MAX;
        }
        if (inB) {
            ++ib;
            b0 = b1;
            b1 = ib + 1 < nb ? __ldg(b + ib + 1) : INT_MAX;
        }
        return true;
    }
};

template <int D>
struct PpCfg {
    static constexpr int DC = D / 64;  // 64-element (128-byte) column chunks
    static constexpr uint32_t Q_BYTES = kRowsPP * D * 2;
    static constexpr uint32_t T_BYTES = kBlk * D * 2;  // one K or V tile
    static constexpr int NK = 2, NV = 2;
    static constexpr int PF = 4;  // union blocks prefetched into L2 ahead of the loads
    static constexpr uint32_t K_OFF = 2 * Q_BYTES;
    static constexpr uint32_t V_OFF = K_OFF + NK * T_BYTES;
    static constexpr uint32_t BAR_OFF = V_OFF + NV * T_BYTES;
    // q_full, k_full[NK], k_empty[NK], v_full[NV], v_empty[NV], s_full[2], p_full[2], fin
    static constexpr uint32_t NBAR = 1 + 2 * NK + 2 * NV + 5;
    static constexpr uint32_t SMEM = BAR_OFF + NBAR * 8 + 16;
    // more than half of an SM's shared memory, so that a second CTA never fits: the CTA holds
    // all 512 TMEM columns
    static constexpr uint32_t SMEM_LAUNCH = SMEM + 1024 > 116u * 1024u ? SMEM + 1024 : 116u * 1024u;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t O_COL = 2 * kBlk;
    static constexpr uint32_t IDESC_S = sm100::idesc_bf16(kRowsPP, kBlk, false);
    static constexpr uint32_t IDESC_PV = sm100::idesc_bf16(kRowsPP, D, true);
    static_assert(O_COL + 2 * D <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM_LAUNCH <= 227u * 1024u, "shared memory budget");
    static_assert(SMEM_LAUNCH > 114u * 1024u, "one CTA per SM (the CTA holds all 512 TMEM columns)");
};

template <int D>
__global__ void __launch_bounds__(kThreadsPP, 1)
    prefill_pp_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, uint16_t *__restrict__ O,
                      const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                      int H, int Hkv, int L, int Nb, float scale_log2) {
    using C = PpCfg<D>;
    constexpr int NK = C::NK, NV = C::NV;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sQ = smem_u32(base);  // Q_A, then Q_B
    const uint32_t sK = sQ + C::K_OFF;
    const uint32_t sV = sQ + C::V_OFF;
    const uint32_t sBar = sQ + C::BAR_OFF;
    const uint32_t q_full = sBar;
    auto k_full = [&](int s) { return sBar + 8u * (1 + s); };
    auto k_empty = [&](int s) { return sBar + 8u * (1 + NK + s); };
    auto v_full = [&](int s) { return sBar + 8u * (1 + 2 * NK + s); };
    auto v_empty = [&](int s) { return sBar + 8u * (1 + 2 * NK + NV + s); };
    auto s_full = [&](int x) { return sBar + 8u * (1 + 2 * NK + 2 * NV + x); };
    auto p_full = [&](int x) { return sBar + 8u * (3 + 2 * NK + 2 * NV + x); };
    const uint32_t fin_bar = sBar + 8u * (5 + 2 * NK + 2 * NV);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + C::BAR_OFF + C::NBAR * 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Work order: KV group by KV group; inside a group, pairs of query blocks from the longest
    // rows down with the group's heads adjacent, so resident CTAs stream one KV head's K/V,
    // which stays in L2.
    const int G = H / Hkv, NP = (Nb + 1) / 2;
    const long lin = blockIdx.x;
    const int g = (int)(lin / ((long)G * NP));
    const int within = (int)(lin % ((long)G * NP));
    const int pair = within / G;
    const int h = g * G + within % G;
    const int I_A = Nb - 1 - 2 * pair, I_B = I_A - 1;  // I_B < 0: the CTA has one tile
    const bool hasB = I_B >= 0;
    const long rA = (long)h * Nb + I_A;
    const int eA = row_ptr[rA], nA = row_ptr[rA + 1] - eA;
    const int eB = hasB ? row_ptr[rA - 1] : 0;
    const int nB = hasB ? row_ptr[rA] - eB : 0;

    if (threadIdx.x == 96) {
        sm100::mbar_init(q_full, 1);
        for (int s = 0; s < NK; ++s) {
            sm100::mbar_init(k_full(s), 1);
            sm100::mbar_init(k_empty(s), 1);
        }
        for (int s = 0; s < NV; ++s) {
            sm100::mbar_init(v_full(s), 1);
            sm100::mbar_init(v_empty(s), 1);
        }
        for (int x = 0; x < 2; ++x) {
            sm100::mbar_init(s_full(x), 1);
            sm100::mbar_init(p_full(x), 128);
        }
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
    const int32_t *listA = col_idx + eA, *listB = col_idx + eB;

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------------- K producer (and Q)
            sm100::prefetch_tmap(&tmQ);
            sm100::prefetch_tmap(&tmK);
            sm100::prefetch_tmap(&tmV);
            sm100::mbar_arrive_expect_tx(q_full, (hasB ? 2 : 1) * C::Q_BYTES);
            for (int c = 0; c < C::DC; ++c) {
                sm100::tma_load_2d(sQ + c * kRowsPP * 128, &tmQ, c * 64, h * L + I_A * kRowsPP, q_full);
                if (hasB)
                    sm100::tma_load_2d(sQ + C::Q_BYTES + c * kRowsPP * 128, &tmQ, c * 64,
                                       h * L + I_B * kRowsPP, q_full);
            }
            UnionWalk ahead(listA, nA, listB, nB);
            int J, pj = 0;
            bool ia, ib;
            for (; pj < C::PF && ahead.next(J, ia, ib); ++pj)
                for (int c = 0; c < C::DC; ++c) {
                    sm100::tma_prefetch_2d(&tmK, c * 64, g * L + J * kBlk);
                    sm100::tma_prefetch_2d(&tmV, c * 64, g * L + J * kBlk);
                }
            UnionWalk walk(listA, nA, listB, nB);
            int u = 0;
            bool ok = true;
            while (walk.next(J, ia, ib)) {
                if (ahead.next(pj, ia, ib))
                    for (int c = 0; c < C::DC; ++c) {
                        sm100::tma_prefetch_2d(&tmK, c * 64, g * L + pj * kBlk);
                        sm100::tma_prefetch_2d(&tmV, c * 64, g * L + pj * kBlk);
                    }
                const int s = u % NK;
                if (!sm100::mbar_wait(k_empty(s), ((u / NK) & 1) ^ 1)) {  // S of block u-NK issued and done
                    ok = false;
                    break;
                }
                sm100::mbar_arrive_expect_tx(k_full(s), C::T_BYTES);
                for (int c = 0; c < C::DC; ++c)
                    sm100::tma_load_2d(sK + s * C::T_BYTES + c * kBlk * 128, &tmK, c * 64, g * L + J * kBlk,
                                       k_full(s));
                ++u;
            }
            if (!ok) {
                atomicOr(&g_pp_errors, kErrTimeoutProducer);
                // let the copies already in flight land before the CTA's memory is released
                sm100::mbar_wait(q_full, 0);
                for (int t = u > NK ? u - NK : 0; t < u; ++t) sm100::mbar_wait(k_full(t % NK), (t / NK) & 1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------------------- V producer
            UnionWalk walk(listA, nA, listB, nB);
            int J, u = 0;
            bool ia, ib, ok = true;
            while (walk.next(J, ia, ib)) {
                const int s = u % NV;
                if (!sm100::mbar_wait(v_empty(s), ((u / NV) & 1) ^ 1)) {  // P V of block u-NV done
                    ok = false;
                    break;
                }
                sm100::mbar_arrive_expect_tx(v_full(s), C::T_BYTES);
                for (int c = 0; c < C::DC; ++c)
                    sm100::tma_load_2d(sV + s * C::T_BYTES + c * kBlk * 128, &tmV, c * 64, g * L + J * kBlk,
                                       v_full(s));
                ++u;
            }
            if (!ok) {
                atomicOr(&g_pp_errors, kErrTimeoutProducer);
                for (int t = u > NV ? u - NV : 0; t < u; ++t) sm100::mbar_wait(v_full(t % NV), (t / NV) & 1);
            }
        }
    } else if (warp == 2) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            bool ok = sm100::mbar_wait(q_full, 0);
            sm100::tc_fence_after();
            // shared-memory descriptors of the operand bases, built once: an MMA step only adds
            // the step's byte offset >> 4 to the start-address field (every address is below
            // 256 KB, so the 14-bit field never carries into the next one).  The issuing thread
            // runs only a few instructions between MMAs: the tensor core queues almost nothing
            // ahead of the MMA it executes, so every instruction in between can leave it idle.
            const uint64_t dQ0 = sm100::smem_desc_sw128(sQ, 16, 1024);
            const uint64_t dQ1 = sm100::smem_desc_sw128(sQ + C::Q_BYTES, 16, 1024);
            const uint64_t dK0 = sm100::smem_desc_sw128(sK, 16, 1024);
            const uint64_t dV0 = sm100::smem_desc_sw128(sV, kBlk * 128, 1024);
            // P V of tile x for the union block held in V slot vs; n = blocks of x done so far
            auto issue_pv = [&](int x, int vs, int n) -> bool {
                if (!sm100::mbar_wait(p_full(x), n & 1)) return false;
                sm100::tc_fence_after();
                const uint64_t bd0 = dV0 + ((vs * C::T_BYTES) >> 4);
                const uint32_t dcol = tmem + C::O_COL + x * D, acol = tmem + x * kBlk;
#pragma unroll
                for (int kk = 0; kk < kBlk / 16; ++kk)
                    sm100::mma_ts(dcol, acol + kk * 8, bd0 + ((kk * 16 * 128) >> 4), C::IDESC_PV,
                                  (n > 0 || kk > 0));
                return true;
            };
            auto issue_s = [&](int x, int ks) {
                const uint64_t ad0 = x ? dQ1 : dQ0;
                const uint64_t bd0 = dK0 + ((ks * C::T_BYTES) >> 4);
                const uint32_t dcol = tmem + x * kBlk;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int c = kk >> 2, w = kk & 3;
                    sm100::mma_ss(dcol, ad0 + ((c * kRowsPP * 128 + w * 32) >> 4),
                                  bd0 + ((c * kBlk * 128 + w * 32) >> 4), C::IDESC_S, kk > 0);
                }
                sm100::mma_commit(s_full(x));
            };
            UnionWalk walk(listA, nA, listB, nB);
            int J, u = 0;
            bool in[2];
            bool pend[2] = {false, false};  // tile x's S for block u-1 is out, its P V is not
            int done[2] = {0, 0};           // blocks whose P V tile x has issued
            while (ok && walk.next(J, in[0], in[1])) {
                const int ks = u % NK;
                // the P V products of block u-1 need V(u-1); the S products of block u need K(u)
                if ((pend[0] || pend[1]) && !sm100::mbar_wait(v_full((u - 1) % NV), ((u - 1) / NV) & 1)) {
                    ok = false;
                    break;
                }
                bool have_k = false;
                for (int x = 0; x < 2 && ok; ++x) {
                    if (pend[x]) {
                        ok = issue_pv(x, (u - 1) % NV, done[x]);
                        ++done[x];
                        pend[x] = false;
                    }
                    if (ok && in[x]) {
                        if (!have_k) {
                            ok = sm100::mbar_wait(k_full(ks), (u / NK) & 1);
                            sm100::tc_fence_after();
                            have_k = true;
                        }
                        if (ok) {
                            issue_s(x, ks);
                            pend[x] = true;
                        }
                    }
                }
                if (!ok) break;
                sm100::mma_commit(k_empty(ks));                       // K of block u read
                if (u > 0) sm100::mma_commit(v_empty((u - 1) % NV));  // V of block u-1 read
                ++u;
            }
            if (ok && (pend[0] || pend[1])) {
                if (!sm100::mbar_wait(v_full((u - 1) % NV), ((u - 1) / NV) & 1)) ok = false;
                sm100::tc_fence_after();
                for (int x = 0; x < 2 && ok; ++x)
                    if (pend[x]) {
                        ok = issue_pv(x, (u - 1) % NV, done[x]);
                        ++done[x];
                    }
                if (ok) sm100::mma_commit(v_empty((u - 1) % NV));
            }
            // fin_bar: every MMA has completed (the epilogue reads O, then the TMEM is released)
            sm100::mma_commit(fin_bar);
            if (!sm100::mbar_wait(fin_bar, 0)) ok = false;
            if (!ok) atomicOr(&g_pp_errors, kErrTimeoutMma);
        }
    } else if (warp >= 4) {
        // -------------------------------------------------------------------- softmax
        const int x = (warp - 4) >> 2;  // tile: warps 4-7 -> A, 8-11 -> B
        const int I = x ? I_B : I_A;
        const int n = x ? nB : nA;
        const int32_t *list = x ? listB : listA;
        if (x == 0 || hasB) {
            const int r = (warp & 3) * 32 + lane;  // query row within the tile = TMEM lane
            const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
            const uint32_t sc = x * kBlk, oc = C::O_COL + x * D;
            float m = -INFINITY, l = 0.f;
            bool ok = true;
            // A CSR row is ascending with J <= I, so only its last block can be the diagonal one.
            const bool diag_last = n > 0 && __ldg(list + n - 1) == I;
            for (int t = 0; t < n; ++t) {
                ok = __all_sync(0xffffffffu, sm100::mbar_wait(s_full(x), t & 1));
                if (!ok) break;
                sm100::tc_fence_after();
                uint32_t sr[kBlk];
#pragma unroll
                for (int cc = 0; cc < kBlk / 32; ++cc)
                    sm100::tmem_ld32(trow + sc + cc * 32, *reinterpret_cast<uint32_t(*)[32]>(sr + cc * 32));
                sm100::tmem_wait_ld();
                if (diag_last && t == n - 1) {  // key i of the diagonal block is visible iff i <= r
#pragma unroll
                    for (int i = 0; i < kBlk; ++i)
                        if (i > r) sr[i] = __float_as_uint(-INFINITY);
                }
                // row max: four chains of three-input maxima
                float mq[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) mq[k] = __uint_as_float(sr[k]);
#pragma unroll
                for (int i = 4; i + 8 <= kBlk; i += 8)
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        mq[k] = fmax3(mq[k], __uint_as_float(sr[i + 2 * k]), __uint_as_float(sr[i + 2 * k + 1]));
                mq[0] = fmax3(mq[0], __uint_as_float(sr[kBlk - 4]), __uint_as_float(sr[kBlk - 3]));
                mq[1] = fmax3(mq[1], __uint_as_float(sr[kBlk - 2]), __uint_as_float(sr[kBlk - 1]));
                const float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])) * scale_log2;  // scale > 0
                // Lazy rescale: a row keeps its stale max while p <= 2^8.  tcgen05.ld/st are
                // warp-collective, so the O rescale (after the exponentials, below) runs for the
                // whole warp whenever any of its rows needs it (alpha = 1 on the others).  O is
                // stable here: the commit behind this S fired after the tile's previous P V
                // completed, and the next P V waits for this step's P.
                const bool need = mx > m + 8.f;
                float alpha = 1.f;
                if (need) {
                    alpha = ex2_approx(m - mx);  // 0 on a row's first block
                    l *= alpha;
                    m = mx;
                }
                const float nm = (m == -INFINITY) ? 0.f : -m;  // a row with nothing attended yet
                const f32x2 sc2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(nm, nm);
                f32x2 rs2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
                for (int hh = 0; hh < 4; ++hh) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int i = hh * 32 + 2 * e;
                        const f32x2 x2 = f2_fma(f2_pack(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])), sc2, nm2);
                        float x0, x1;
                        f2_unpack(x2, x0, x1);
                        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                        rs2[e & 1] = f2_add(rs2[e & 1], f2_pack(p0, p1));
                        pk[e] = pack_bf16(p0, p1);
                    }
                    // P (keys 32hh .. 32hh+31, bf16 pairs) over S columns [16hh, 16hh + 16),
                    // which this thread has already loaded
                    sm100::tmem_st16(trow + sc + hh * 16, pk);
                }
                float ra, rb, rc, rd;
                f2_unpack(rs2[0], ra, rb);
                f2_unpack(rs2[1], rc, rd);
                l += (ra + rb) + (rc + rd);
                if (t > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t rg[32];
                        sm100::tmem_ld32(trow + oc + cc * 32, rg);
                        sm100::tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) rg[i] = __float_as_uint(__uint_as_float(rg[i]) * alpha);
                        sm100::tmem_st32(trow + oc + cc * 32, rg);
                    }
                }
                sm100::tmem_wait_st();
                sm100::tc_fence_before();
                sm100::mbar_arrive(p_full(x));
            }
            // O is final once every MMA has completed
            if (ok) {
                ok = __all_sync(0xffffffffu, sm100::mbar_wait(fin_bar, 0));
                sm100::tc_fence_after();
            }
            if (!ok) {
                if (lane == 0) atomicOr(&g_pp_errors, kErrTimeoutSoftmax);
            } else {
                // a row that attended nothing (an empty CSR row) is written as zeros: its O
                // columns in TMEM were never written
                const float inv = (l > 0.f) ? 1.f / l : 0.f;
                uint16_t *orow = O + ((long)h * L + (long)I * kRowsPP + r) * D;
#pragma unroll
                for (int cc = 0; cc < D / 32; ++cc) {
                    uint32_t rg[32];
                    if (n > 0) {
                        sm100::tmem_ld32(trow + oc + cc * 32, rg);
                        sm100::tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) rg[i] = 0u;
                    }
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        pk[i] = pack_bf16(__uint_as_float(rg[2 * i]) * inv, __uint_as_float(rg[2 * i + 1]) * inv);
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

template <int D>
rr_status_t launch_pp(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int H, int Hkv, int L,
                      const int32_t *row_ptr, const int32_t *col_idx, float scale, uint16_t *O,
                      cudaStream_t st) {
    using C = PpCfg<D>;
    alignas(64) CUtensorMap mq, mk, mv;
    if (!make_tmap_bf16(&mq, Q, (uint64_t)H * L, D, kRowsPP) || !make_tmap_bf16(&mk, K, (uint64_t)Hkv * L, D, kBlk) ||
        !make_tmap_bf16(&mv, V, (uint64_t)Hkv * L, D, kBlk))
        return set_error(RR_ERR_CUDA, "rr_sparse_prefill: cuTensorMapEncodeTiled failed");
    auto kern = prefill_pp_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM_LAUNCH);
    if (e != cudaSuccess)
        return set_error(RR_ERR_CUDA, "rr_sparse_prefill: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    const int Nb = L / kBlk, G = H / Hkv;
    dim3 grid((unsigned)((long)Hkv * G * ((Nb + 1) / 2)));
    kern<<<grid, kThreadsPP, C::SMEM_LAUNCH, st>>>(mq, mk, mv, O, row_ptr, col_idx, H, Hkv, L, Nb,
                                                    scale * 1.4426950408889634f);
    return check_launch("rr_sparse_prefill: prefill_pp_kernel");
}

}  // namespace

// B = 128 layers: two query tiles per CTA (d = 64 or 128).
rr_status_t launch_prefill_pp(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int H, int Hkv,
                              int L, int d, const int32_t *row_ptr, const int32_t *col_idx, float scale,
                              uint16_t *O, cudaStream_t st) {
    if (d == 128) return launch_pp<128>(Q, K, V, H, Hkv, L, row_ptr, col_idx, scale, O, st);
    return launch_pp<64>(Q, K, V, H, Hkv, L, row_ptr, col_idx, scale, O, st);
}

rr_status_t read_pp_errors(unsigned *out, bool reset) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_pp_errors, sizeof(unsigned));
    if (e == cudaSuccess && reset) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_pp_errors, &zero, sizeof(unsigned));
    }
    if (e != cudaSuccess) return set_error(RR_ERR_CUDA, "rr_device_errors: %s", cudaGetErrorString(e));
    return RR_OK;
}

}  // namespace rr
