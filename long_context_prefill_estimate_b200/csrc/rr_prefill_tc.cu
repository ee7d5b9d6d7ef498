// Causal block-sparse attention over the selected blocks on the 5th-generation tensor cores
// ("RRAttention: Dynamic Block Sparse Attention via Per-Head Round-Robin Shifts for
// Long-Context Inference", Sec. 2.1 with the per-head CSR block lists as the block selection
// matrix; Sec. 4.1: sparsity in prefill only).
//
// One CTA per (query head h, query block I): a 128-row query tile (for B = 64 the upper 64
// rows are padding that is computed and never stored).  The CTA walks only the CSR entries
// of row h*Nb + I.  Warp roles:
//   warp 0      TMA producer: Q tile once, then K and V tiles of each selected block into a
//               ring of 3-4 stages (128-byte swizzle, mbarrier transaction counts).
//   warp 1      MMA issuer (one thread): S_j = Q K_j^T (both operands in shared memory) into
//               one of two TMEM buffers, then O += P_j V_j with P_j read from TMEM (the
//               A-from-tensor-memory form) and V_j from shared memory; completion is signalled
//               by tcgen05.commit.
//   warp 2      TMEM allocation / release.
//   warps 4-7   softmax: one thread per query row (TMEM lane).  Online softmax in fp32 with a
//               lazily rescaled running max (O is rescaled in TMEM only when a row's max grows
//               by more than 2^8), P packed to bf16 pairs and stored back into TMEM (two
//               buffers, so block j's softmax never waits for block j-1's P*V), final
//               normalisation and bf16 store of O.
// TMEM columns: S0, S1 (fp32, B each), O (fp32, d), P0, P1 (bf16 pairs, B/2 each).
// The producer also prefetches the K/V tiles of the next few selected blocks into L2.
// K and V come from KV head h / (H/Hkv); the heads of a KV group run as adjacent CTAs so
// their K/V tiles are served from L2.  Every wait is bounded (about one second of
// %globaltimer); a timeout sets a device error bit and the CTA drains and exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

#include "rr_common.cuh"
#include "rr_sm100.cuh"

namespace rr {

namespace {

__device__ unsigned int g_device_errors;

constexpr unsigned kErrTimeoutProducer = 1u, kErrTimeoutMma = 2u, kErrTimeoutSoftmax = 4u;

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase of `parity` to complete, for at most ~1 s.
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity) {
    if (sm100::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    for (uint32_t i = 1;; ++i) {
        if (sm100::mbar_try_wait(bar, parity)) return true;
        if ((i & 1023u) == 0 && globaltimer() - t0 > 1000000000ull) return false;
    }
}

// 2^x on the SFU (approximate, flushes denormals; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
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

template <int D, int BN>
struct TcCfg {
    static constexpr int DC = D / 64;  // 64-element (128-byte) column chunks
    static constexpr uint32_t Q_BYTES = kBM * D * 2;
    static constexpr uint32_t KV_BYTES = BN * D * 2;
    // as many K/V stages (up to 4) as fit next to Q in the 227 KB a CTA may use (1024 bytes
    // of alignment slack, 256 for barriers)
    static constexpr int PF = 4;  // K/V blocks prefetched into L2 ahead of the shared-memory loads
    static constexpr int NS_FIT = (int)((227u * 1024u - Q_BYTES - 1024u - 256u) / (2u * KV_BYTES));
    static constexpr int NS = NS_FIT > 4 ? 4 : NS_FIT;
    static constexpr uint32_t BAR_OFF = Q_BYTES + 2 * NS * KV_BYTES;
    static constexpr uint32_t NBAR = 1 + 2 * NS + 2 + 1 + 1 + 1;
    static constexpr uint32_t SMEM = BAR_OFF + NBAR * 8 + 16;
    // TMEM columns: S0 [0,BN) S1 [BN,2BN) O [2BN,2BN+D) P0, P1 [2BN+D, 2BN+D+BN) (bf16 pairs,
    // BN/2 columns each)
    static constexpr uint32_t S_COL = 0, O_COL = 2 * BN, P_COL = 2 * BN + D;
    static constexpr uint32_t TMEM_NEED = 2 * BN + D + BN;
    static constexpr uint32_t TMEM_COLS = TMEM_NEED <= 256 ? 256 : 512;
    static constexpr uint32_t IDESC_S = sm100::idesc_bf16(kBM, BN, false);
    static constexpr uint32_t IDESC_PV = sm100::idesc_bf16(kBM, D, true);
    static_assert(NS >= 2, "need at least two K/V stages");
    static_assert(SMEM + 1024 <= 227u * 1024u, "shared memory budget");
    static_assert(TMEM_NEED <= 512, "TMEM budget");
};

template <int D, int BN>
__global__ void __launch_bounds__(256, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, uint16_t *__restrict__ O,
                      const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col_idx,
                      int H, int Hkv, int L, int Nb, float scale_log2) {
    using C = TcCfg<D, BN>;
    constexpr int kNS = C::NS;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sQ = smem_u32(base);
    const uint32_t sK = sQ + C::Q_BYTES;
    const uint32_t sV = sK + kNS * C::KV_BYTES;
    const uint32_t sBar = sQ + C::BAR_OFF;
    const uint32_t q_full = sBar;
    auto kv_full = [&](int s) { return sBar + 8u * (1 + s); };
    auto kv_empty = [&](int s) { return sBar + 8u * (1 + kNS + s); };
    auto s_full = [&](int b) { return sBar + 8u * (1 + 2 * kNS + b); };
    const uint32_t p_full = sBar + 8u * (3 + 2 * kNS);
    const uint32_t o_bar = sBar + 8u * (4 + 2 * kNS);
    const uint32_t fin_bar = sBar + 8u * (5 + 2 * kNS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base + C::BAR_OFF + C::NBAR * 8);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Launch order: KV group by KV group, and inside a group query blocks from the longest
    // CSR rows down with the group's heads adjacent.  CTAs resident at the same time then
    // stream one KV head's K/V, which stays in L2.
    const int G = H / Hkv;
    const long lin = blockIdx.x;
    const int g = (int)(lin / ((long)G * Nb));
    const int within = (int)(lin % ((long)G * Nb));
    const int I = Nb - 1 - within / G;
    const int h = g * G + within % G;
    const long crow = (long)h * Nb + I;
    const int e0 = row_ptr[crow];
    const int n = row_ptr[crow + 1] - e0;

    if (threadIdx.x == 0) {
        sm100::mbar_init(q_full, 1);
        for (int s = 0; s < kNS; ++s) {
            sm100::mbar_init(kv_full(s), 1);
            sm100::mbar_init(kv_empty(s), 1);
        }
        sm100::mbar_init(s_full(0), 1);
        sm100::mbar_init(s_full(1), 1);
        sm100::mbar_init(p_full, 128);
        sm100::mbar_init(o_bar, 1);
        sm100::mbar_init(fin_bar, 1);
        sm100::fence_mbar_init();
    }
    if (warp == 2) {
        sm100::tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        sm100::tmem_relinquish();
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------------- producer
            sm100::prefetch_tmap(&tmQ);
            sm100::prefetch_tmap(&tmK);
            sm100::prefetch_tmap(&tmV);
            sm100::mbar_arrive_expect_tx(q_full, C::Q_BYTES);
            for (int c = 0; c < C::DC; ++c)
                sm100::tma_load_2d(sQ + c * kBM * 128, &tmQ, c * 64, h * L + I * BN, q_full);
            int issued = 0;
            bool ok = true;
            for (int j = 0; j < n && j < C::PF; ++j) {
                const int Jp = __ldg(col_idx + e0 + j);
                for (int c = 0; c < C::DC; ++c) {
                    sm100::tma_prefetch_2d(&tmK, c * 64, g * L + Jp * BN);
                    sm100::tma_prefetch_2d(&tmV, c * 64, g * L + Jp * BN);
                }
            }
            for (int j = 0; j < n; ++j) {
                if (j + C::PF < n) {
                    const int Jp = __ldg(col_idx + e0 + j + C::PF);
                    for (int c = 0; c < C::DC; ++c) {
                        sm100::tma_prefetch_2d(&tmK, c * 64, g * L + Jp * BN);
                        sm100::tma_prefetch_2d(&tmV, c * 64, g * L + Jp * BN);
                    }
                }
                const int s = j % kNS;
                if (!wait_bar(kv_empty(s), ((j / kNS) & 1) ^ 1)) {
                    ok = false;
                    break;
                }
                const int J = __ldg(col_idx + e0 + j);
                sm100::mbar_arrive_expect_tx(kv_full(s), 2 * C::KV_BYTES);
                for (int c = 0; c < C::DC; ++c) {
                    sm100::tma_load_2d(sK + s * C::KV_BYTES + c * BN * 128, &tmK, c * 64, g * L + J * BN,
                                       kv_full(s));
                    sm100::tma_load_2d(sV + s * C::KV_BYTES + c * BN * 128, &tmV, c * 64, g * L + J * BN,
                                       kv_full(s));
                }
                issued = j + 1;
            }
            if (!ok) {
                atomicOr(&g_device_errors, kErrTimeoutProducer);
                // let the copies already in flight land before the CTA's memory is released
                wait_bar(q_full, 0);
                for (int j = issued > kNS ? issued - kNS : 0; j < issued; ++j)
                    wait_bar(kv_full(j % kNS), (j / kNS) & 1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------------- MMA issuer
            bool ok = wait_bar(q_full, 0);
            sm100::tc_fence_after();
            auto issue_s = [&](int j) -> bool {
                const int s = j % kNS, b = j & 1;
                if (!wait_bar(kv_full(s), (j / kNS) & 1)) return false;
                sm100::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const int c = kk >> 2, w = kk & 3;
                    const uint64_t ad = sm100::smem_desc_sw128(sQ + c * kBM * 128 + w * 32, 16, 1024);
                    const uint64_t bd =
                        sm100::smem_desc_sw128(sK + s * C::KV_BYTES + c * BN * 128 + w * 32, 16, 1024);
                    sm100::mma_ss(tmem + C::S_COL + b * BN, ad, bd, C::IDESC_S, kk > 0);
                }
                sm100::mma_commit(s_full(b));
                return true;
            };
            if (ok && n > 0) ok = issue_s(0);
            for (int j = 0; ok && j < n; ++j) {
                if (j + 1 < n && !issue_s(j + 1)) {
                    ok = false;
                    break;
                }
                if (!wait_bar(p_full, j & 1)) {
                    ok = false;
                    break;
                }
                sm100::tc_fence_after();
                const int s = j % kNS;
#pragma unroll
                for (int kk = 0; kk < BN / 16; ++kk) {
                    const uint64_t bd =
                        sm100::smem_desc_sw128(sV + s * C::KV_BYTES + kk * 16 * 128, BN * 128, 1024);
                    sm100::mma_ts(tmem + C::O_COL, tmem + C::P_COL + (j & 1) * (BN / 2) + kk * 8, bd,
                                  C::IDESC_PV, (j > 0 || kk > 0));
                }
                sm100::mma_commit(o_bar);
                sm100::mma_commit(kv_empty(s));
            }
            // every MMA issued must complete before the TMEM is released
            sm100::mma_commit(fin_bar);
            if (!wait_bar(fin_bar, 0)) ok = false;
            if (!ok) atomicOr(&g_device_errors, kErrTimeoutMma);
        }
    } else if (warp >= 4) {
        // -------------------------------------------------------------------- softmax
        const int r = threadIdx.x - 128;  // query row within the tile = TMEM lane
        const long qpos = (long)I * BN + r;
        const uint32_t trow = tmem + ((uint32_t)((warp - 4) * 32) << 16);
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            const int b = j & 1;
            ok = __all_sync(0xffffffffu, wait_bar(s_full(b), (j >> 1) & 1));
            if (!ok) break;
            sm100::tc_fence_after();
            const int J = __ldg(col_idx + e0 + j);
            uint32_t sr[BN];
#pragma unroll
            for (int cc = 0; cc < BN / 32; ++cc)
                sm100::tmem_ld32(trow + C::S_COL + b * BN + cc * 32,
                                 *reinterpret_cast<uint32_t(*)[32]>(sr + cc * 32));
            sm100::tmem_wait_ld();
            const bool diag = (J == I);
            if (diag) {  // diagonal block: key i of the block is visible iff i <= r
#pragma unroll
                for (int i = 0; i < BN; ++i)
                    if (i > r) sr[i] = __float_as_uint(-INFINITY);
            }
            float mq[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) mq[k] = __uint_as_float(sr[k]);
#pragma unroll
            for (int i = 8; i < BN; ++i) mq[i & 7] = fmaxf(mq[i & 7], __uint_as_float(sr[i]));
            const float mraw = fmaxf(fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])),
                                     fmaxf(fmaxf(mq[4], mq[5]), fmaxf(mq[6], mq[7])));
            const float mx = mraw * scale_log2;  // scale > 0 keeps the order
            // Lazy rescale: a row keeps its stale max while p <= 2^8.  The decision is per row,
            // but tcgen05.ld/st are warp-collective, so the O rescale runs for the whole warp
            // whenever any of its rows needs it (alpha = 1 on the others).  Only then must the
            // previous block's P*V be complete; P itself is double-buffered.
            const bool need = mx > m + 8.f;
            float alpha = 1.f;
            if (need) {
                alpha = ex2_approx(m - mx);  // 0 on a row's first block
                l *= alpha;
            }
            if (j > 0 && __any_sync(0xffffffffu, need)) {
                ok = __all_sync(0xffffffffu, wait_bar(o_bar, (j - 1) & 1));
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
            if (need) m = mx;
            // P_j goes to the buffer P_{j-2} used.  Its P*V product is complete: S_j was issued
            // after P_{j-2} V_{j-2}, and the commit behind S_j (which this warpgroup waited for
            // before reading S_j) fires only once every earlier MMA of the issuing thread is done.
            const float nm = (m == -INFINITY) ? 0.f : -m;  // a row with nothing attended yet
            const f32x2 sc2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(nm, nm);
            f32x2 rs2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
            for (int hc = 0; hc < BN / 64; ++hc) {
                uint32_t pk[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const f32x2 x2 = f2_fma(f2_pack(__uint_as_float(sr[hc * 64 + 2 * e]),
                                                    __uint_as_float(sr[hc * 64 + 2 * e + 1])),
                                            sc2, nm2);
                    float x0, x1;
                    f2_unpack(x2, x0, x1);
                    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                    rs2[e & 1] = f2_add(rs2[e & 1], f2_pack(p0, p1));
                    pk[e] = pack_bf16(p0, p1);
                }
                sm100::tmem_st32(trow + C::P_COL + (j & 1) * (BN / 2) + hc * 32, pk);
            }
            float ra, rb, rc, rd;
            f2_unpack(rs2[0], ra, rb);
            f2_unpack(rs2[1], rc, rd);
            const float rs = (ra + rb) + (rc + rd);
            sm100::tmem_wait_st();
            l += rs;
            sm100::tc_fence_before();
            sm100::mbar_arrive(p_full);
        }
        if (ok && n > 0) {
            ok = __all_sync(0xffffffffu, wait_bar(o_bar, (n - 1) & 1));
            sm100::tc_fence_after();
        }
        if (!ok) {
            if (lane == 0) atomicOr(&g_device_errors, kErrTimeoutSoftmax);
        } else {
            const float inv = (l > 0.f) ? 1.f / l : 0.f;
            uint16_t *orow = O + ((long)h * L + qpos) * D;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t rg[32];
                sm100::tmem_ld32(trow + C::O_COL + cc * 32, rg);
                sm100::tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16(__uint_as_float(rg[2 * i]) * inv, __uint_as_float(rg[2 * i + 1]) * inv);
                if (r < BN) {
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
    if (warp == 2) {
        sm100::tc_fence_after();
        sm100::tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D bf16 view [rows][d] of a row-major tensor, boxes of 64 columns x box_rows rows,
// 128-byte swizzle.
bool make_map(CUtensorMap *m, const void *ptr, uint64_t rows, int d, uint32_t box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)d, rows};
    const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int BN>
rr_status_t launch_tc(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int H, int Hkv, int L,
                      const int32_t *row_ptr, const int32_t *col_idx, float scale, uint16_t *O,
                      cudaStream_t st) {
    using C = TcCfg<D, BN>;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, Q, (uint64_t)H * L, D, kBM) || !make_map(&mk, K, (uint64_t)Hkv * L, D, BN) ||
        !make_map(&mv, V, (uint64_t)Hkv * L, D, BN))
        return set_error(RR_ERR_CUDA, "rr_sparse_prefill: cuTensorMapEncodeTiled failed");
    // at least 116 KB of shared memory: one CTA per SM, so TMEM allocation never contends
    size_t smem = C::SMEM + 1024;
    if (smem < 116 * 1024) smem = 116 * 1024;
    auto kern = prefill_tc_kernel<D, BN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
        return set_error(RR_ERR_CUDA, "rr_sparse_prefill: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    const int Nb = L / BN;
    dim3 grid((unsigned)((long)H * Nb));
    kern<<<grid, 256, smem, st>>>(mq, mk, mv, O, row_ptr, col_idx, H, Hkv, L, Nb,
                                  scale * 1.4426950408889634f);
    return check_launch("rr_sparse_prefill: prefill_tc_kernel");
}

}  // namespace

rr_status_t launch_prefill_tc(const uint16_t *Q, const uint16_t *K, const uint16_t *V, int H, int Hkv,
                              int L, int d, int B, const int32_t *row_ptr, const int32_t *col_idx,
                              float scale, uint16_t *O, cudaStream_t st) {
    if (d == 128 && B == 128) return launch_tc<128, 128>(Q, K, V, H, Hkv, L, row_ptr, col_idx, scale, O, st);
    if (d == 128 && B == 64) return launch_tc<128, 64>(Q, K, V, H, Hkv, L, row_ptr, col_idx, scale, O, st);
    if (d == 64 && B == 128) return launch_tc<64, 128>(Q, K, V, H, Hkv, L, row_ptr, col_idx, scale, O, st);
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
