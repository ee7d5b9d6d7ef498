// Stride-level block importance of RRAttention ("RRAttention: Dynamic Block Sparse Attention
// via Per-Head Round-Robin Shifts for Long-Context Inference", Sec. 3.1 heading, Sec. 3.2,
// Sec. 3.3 heading).
//
// launch_estimate sends B/S in {4, 8, 16, 32} to the tensor-core (tcgen05) estimator of
// rr_estimate_tc.cu.  This file holds the launch planning and, for B/S = 64 or 128 (S = 1,
// the exact mode), a register-fragment estimator whose rows of a query block span several
// warps:
//   pool_keys_kernel  Kbar_j = sum of the S keys of stride j (fp32), split into bf16 hi + lo
//                     and stored directly in the register order of the m16n8k16 B operand.
//                     HBM bound: reads K once, writes Hkv*Ns*d*4 bytes.
//   estimate_kernel   one CTA per (query block I, KV head g, chunk of the g's query heads).
//                     Rows = sampled queries Q[h][i*S + off(h)] of the chunk's heads for the
//                     B/S strides i of block I.  Tensor-core logits (Q exact in bf16, Kbar as
//                     hi + lo => fp32-grade products), stride-level softmax with a lazily
//                     rescaled running max (rescale only when the max grows by > 2^8), per
//                     (row, key block) partial sums kept in shared memory, then one exact
//                     normalisation per row and the (S/B)-weighted block sums.
#include <cuda_bf16.h>

#include "rr_common.cuh"

namespace rr {

namespace {

constexpr int kEstThreads = 256;
constexpr int kEstWarps = kEstThreads / 32;

// Fragment layout of the pooled keys: index ((g*NT + tile)*KS + ks)*32 + lane holds, for
// stride tile*8 + lane/4 and dims ks*16 + 2*(lane%4) + {0,1} (b0) and + 8 (b1):
// uint4 {b0_hi, b1_hi, b0_lo, b1_lo}.
template <int D>
__global__ void __launch_bounds__(256)
    pool_keys_kernel(const uint16_t *__restrict__ K, int L, int S, int Ns, int Hkv,
                     uint32_t *__restrict__ frag) {
    constexpr int C = D / 8;  // 16-byte chunks per key row
    constexpr int KS = D / 16;
    const long total = (long)Hkv * Ns * C;
    const int NT = Ns / 8;
    for (long idx = blockIdx.x * (long)blockDim.x + threadIdx.x; idx < total;
         idx += (long)gridDim.x * blockDim.x) {
        const int c = (int)(idx % C);
        const long j = (idx / C) % Ns;
        const int g = (int)(idx / ((long)C * Ns));
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
        const int ks = c >> 1, half = c & 1;
        const long base = (((long)g * NT + j / 8) * KS + ks) * 32;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const float x0 = acc[2 * t], x1 = acc[2 * t + 1];
            const float h0 = __bfloat162float(__float2bfloat16_rn(x0));
            const float h1 = __bfloat162float(__float2bfloat16_rn(x1));
            const uint32_t hi = pack_bf16(h0, h1);
            const uint32_t lo = pack_bf16(x0 - h0, x1 - h1);
            uint32_t *dst = frag + (base + (j % 8) * 4 + t) * 4;
            dst[half] = hi;
            dst[2 + half] = lo;
        }
    }
}

struct EstParams {
    const uint16_t *Q;
    const uint4 *frag;
    float *A;
    int H, L, S, r, Nb, NT, NTB, BPT;  // NTB: 8-stride tiles per work group, BPT: blocks per group
    int G, hc, nHC, R, MT, MTW, NG, WJ;
    int mode, layer;
    int head_base;  // layer-wide index of query head 0 of this call (round-robin offset only)
    float c_log2;  // log2(e) / (S * sqrt(d))
};

template <int D, int MTW, int BPT>
__global__ void __launch_bounds__(kEstThreads, MTW == 1 ? 2 : 1) estimate_kernel(const EstParams p) {
    constexpr int KS = D / 16;
    constexpr int QSTRIDE = D + 8;  // bf16 elements per staged query row (16-byte pad)
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int R = p.R, Rpad = p.MT * 16, Nb = p.Nb, r = p.r;
    uint16_t *qs = reinterpret_cast<uint16_t *>(smem_raw);
    float *sst = reinterpret_cast<float *>(smem_raw + Rpad * QSTRIDE * 2);  // multiple of 16 B
    float *stat_m = sst + (long)R * Nb;
    float *stat_l = stat_m + p.WJ * Rpad;
    float *fac = stat_l + p.WJ * Rpad;

    const int I = Nb - 1 - (int)blockIdx.x;  // longest rows first
    const int g = blockIdx.y / p.nHC;
    const int h0 = g * p.G + (blockIdx.y % p.nHC) * p.hc;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // ---- stage the sampled query rows (16-byte coalesced loads)
    constexpr int CH = D / 8;
    for (int x = tid; x < Rpad * CH; x += kEstThreads) {
        const int rho = x / CH, c = x % CH;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (rho < R) {
            const int h = h0 + rho / r;
            const long i = (long)I * r + rho % r;
            const long pos = i * p.S + rr_offset(p.head_base + h, p.S, p.mode, p.layer);
            v = __ldg(reinterpret_cast<const uint4 *>(p.Q + ((long)h * p.L + pos) * D) + c);
        }
        *reinterpret_cast<uint4 *>(qs + rho * QSTRIDE + c * 8) = v;
    }
    __syncthreads();

    const int grp = warp % p.NG, jw = warp / p.NG, WJ = p.WJ;
    const int gq = lane >> 2, tq = lane & 3;

    uint32_t a[MTW][KS][4];
#pragma unroll
    for (int mm = 0; mm < MTW; ++mm)
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            const int row = (grp * MTW + mm) * 16 + ((lane >> 3) & 1) * 8 + (lane & 7);
            const int col = ks * 16 + (lane >> 4) * 8;
            ldmatrix_x4(a[mm][ks], smem_u32(qs + row * QSTRIDE + col));
        }

    int rho[MTW][2];
    long irow[MTW][2];
    bool valid[MTW][2];
    float mref[MTW][2], lsum[MTW][2], bs[MTW][2];
#pragma unroll
    for (int mm = 0; mm < MTW; ++mm)
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            rho[mm][x] = (grp * MTW + mm) * 16 + gq + 8 * x;
            valid[mm][x] = rho[mm][x] < R;
            irow[mm][x] = (long)I * r + rho[mm][x] % r;
            mref[mm][x] = -INFINITY;
            lsum[mm][x] = 0.f;
            bs[mm][x] = 0.f;
        }

    // Work groups: for r >= 8 a group is one key block (r/8 stride tiles); for r = 4 it is one
    // stride tile spanning two key blocks.  Warp jw takes groups jw, jw+WJ, ...
    const int ngroups = (I + BPT) / BPT;  // groups covering blocks 0..I
    const int nJ = (ngroups > jw) ? (ngroups - 1 - jw) / WJ + 1 : 0;
    const int nunits = nJ * p.NTB;
    const uint4 *fragg = p.frag + (long)g * p.NT * KS * 32 + lane;
    uint4 b[KS], bn[KS];
    if (nunits > 0) {
        const uint4 *src = fragg + (long)(jw * p.NTB) * KS * 32;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) bn[ks] = __ldg(src + ks * 32);
    }
    for (int u = 0; u < nunits; ++u) {
        const int grpi = jw + (u / p.NTB) * WJ, nt = u % p.NTB;
        const int tile = grpi * p.NTB + nt;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) b[ks] = bn[ks];
        if (u + 1 < nunits) {
            const int g2 = jw + ((u + 1) / p.NTB) * WJ, nt2 = (u + 1) % p.NTB;
            const uint4 *src = fragg + (long)(g2 * p.NTB + nt2) * KS * 32;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) bn[ks] = __ldg(src + ks * 32);
        }
        const long col0 = (long)tile * 8 + 2 * tq;
#pragma unroll
        for (int mm = 0; mm < MTW; ++mm) {
            // four independent accumulation chains (hi/lo x two halves of the k-steps), summed
            // afterwards, so consecutive MMAs do not wait on each other
            float cq[4][4];
#pragma unroll
            for (int q = 0; q < 4; ++q) cq[q][0] = cq[q][1] = cq[q][2] = cq[q][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                const int hk = (2 * ks) / KS;
                mma_16816(cq[2 * hk], a[mm][ks], b[ks].x, b[ks].y);
                mma_16816(cq[2 * hk + 1], a[mm][ks], b[ks].z, b[ks].w);
            }
            float c[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) c[e] = (cq[0][e] + cq[1][e]) + (cq[2][e] + cq[3][e]);
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const float s0 = (col0 <= irow[mm][x]) ? c[2 * x] * p.c_log2 : -INFINITY;
                const float s1 = (col0 + 1 <= irow[mm][x]) ? c[2 * x + 1] * p.c_log2 : -INFINITY;
                const float mx = quad_max(fmaxf(s0, s1));
                if (mx > mref[mm][x] + 8.f) {  // lazy rescale: stored sums stay <= r*2^8
                    const float f = ex2_approx(mref[mm][x] - mx);  // 0 on the first block
                    lsum[mm][x] *= f;
                    bs[mm][x] *= f;
                    if (valid[mm][x]) {
                        float *row = sst + (long)rho[mm][x] * Nb;
                        const int done = u / p.NTB;  // this warp's groups already stored
                        for (int k = tq; k < done * BPT; k += 4) {
                            const int J = (jw + (k / BPT) * WJ) * BPT + k % BPT;
                            if (J < Nb) row[J] *= f;
                        }
                    }
                    mref[mm][x] = mx;
                }
                bs[mm][x] += ex2_approx(s0 - mref[mm][x]) + ex2_approx(s1 - mref[mm][x]);
            }
        }
        if (nt == p.NTB - 1) {
            __syncwarp();
#pragma unroll
            for (int mm = 0; mm < MTW; ++mm)
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    float tot;
                    int J;
                    bool writer;
                    if constexpr (BPT == 1) {  // the quad's 8 columns are one block
                        tot = quad_sum(bs[mm][x]);
                        J = grpi;
                        writer = (tq == 0);
                    } else {  // columns 0-3 (lanes 0,1) and 4-7 (lanes 2,3) are two blocks
                        tot = bs[mm][x] + __shfl_xor_sync(0xffffffffu, bs[mm][x], 1);
                        J = grpi * 2 + (tq >> 1);
                        writer = ((tq & 1) == 0);
                    }
                    bs[mm][x] = 0.f;
                    // the row sum takes each block once: add the other half's share too
                    if constexpr (BPT == 1) lsum[mm][x] += tot;
                    else lsum[mm][x] += tot + __shfl_xor_sync(0xffffffffu, tot, 2);
                    if (writer && valid[mm][x] && J <= I) sst[(long)rho[mm][x] * Nb + J] = tot;
                }
            __syncwarp();
        }
    }
    if (tq == 0) {
#pragma unroll
        for (int mm = 0; mm < MTW; ++mm)
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                stat_m[jw * Rpad + rho[mm][x]] = mref[mm][x];
                stat_l[jw * Rpad + rho[mm][x]] = lsum[mm][x];
            }
    }
    __syncthreads();

    // ---- exact per-row normalisation across the warps that shared the row
    const float inv_r = 1.f / (float)r;
    for (int x = tid; x < R; x += kEstThreads) {
        float M = -INFINITY;
        for (int w = 0; w < WJ; ++w) M = fmaxf(M, stat_m[w * Rpad + x]);
        float l = 0.f;
        for (int w = 0; w < WJ; ++w) {
            const float m = stat_m[w * Rpad + x];
            if (m != -INFINITY) l += stat_l[w * Rpad + x] * ex2_approx(m - M);
        }
        for (int w = 0; w < WJ; ++w) {
            const float m = stat_m[w * Rpad + x];
            fac[w * Rpad + x] = (m != -INFINITY) ? ex2_approx(m - M) / l * inv_r : 0.f;
        }
    }
    __syncthreads();

    // ---- block scores of the chunk's heads: row I, all Nb columns (zeros above the diagonal)
    for (int hh = 0; hh < p.hc; ++hh) {
        float *out = p.A + ((long)(h0 + hh) * Nb + I) * Nb;
        for (int J = tid; J < Nb; J += kEstThreads) {
            float v = 0.f;
            if (J <= I) {
                const int w = (J / BPT) % WJ;
                for (int ii = 0; ii < r; ++ii) {
                    const int x = hh * r + ii;
                    v += sst[(long)x * Nb + J] * fac[w * Rpad + x];
                }
            }
            out[J] = v;
        }
    }
}

struct EstPlan {
    int hc, nHC, R, MT, MTW, NG, WJ;
    size_t smem;
};

size_t est_smem(int R, int MT, int WJ, int Nb, int d) {
    const int Rpad = MT * 16;
    return align_up((size_t)Rpad * (d + 8) * 2, 16) + (size_t)R * Nb * 4 +
           (size_t)3 * WJ * Rpad * 4;
}

bool plan_estimate(int H, int Hkv, int d, int S, int B, int Nb, EstPlan *pl) {
    const int G = H / Hkv, r = B / S;
    // Rows per CTA: exactly 16 (one m16 tile per warp, two CTAs per SM) when a whole number
    // of heads gives 16 and it fits, else the largest chunk that fits (one CTA per SM).
    for (int pass = 0; pass < 2; ++pass) {
        for (int hc = G; hc >= 1; --hc) {
            if (G % hc) continue;
            const int R = hc * r;
            if (R > 128 || (pass == 0 && R != 16)) continue;
            int MT = 1;
            while (MT * 16 < R) MT *= 2;
            const int MTW = MT < 2 ? MT : 2;
            const int NG = MT / MTW, WJ = kEstWarps / NG;
            const size_t sm = est_smem(R, MT, WJ, Nb, d);
            if (sm > 200 * 1024) continue;
            *pl = EstPlan{hc, G / hc, R, MT, MTW, NG, WJ, sm};
            return true;
        }
    }
    return false;
}

}  // namespace

size_t estimate_workspace_bytes(int Hkv, int L, int d, int S) {
    if (L <= 0) return 0;
    return (size_t)Hkv * (L / S) * d * 4;  // bf16 hi + lo per pooled element
}

bool estimate_tc_eligible(int d, int S, int B);
rr_status_t launch_estimate_tc(const uint16_t *Q, const uint16_t *K, int H, int Hkv, int L, int d,
                               int S, int B, int mode, int layer, int head_base, float *A, void *ws,
                               cudaStream_t st);

bool estimate_supported(int H, int Hkv, int d, int S, int B, int L) {
    if (estimate_tc_eligible(d, S, B)) return true;
    EstPlan pl;
    return plan_estimate(H, Hkv, d, S, B, L / B, &pl);
}

rr_status_t launch_estimate(const uint16_t *Q, const uint16_t *K, int H, int Hkv, int L, int d,
                            int S, int B, int mode, int layer, int head_base, float *A, void *ws,
                            cudaStream_t st) {
    // B/S in {4, 8, 16, 32}: the tensor-core (tcgen05) estimator; otherwise (B/S = 64 or
    // 128, the S = 1 exact mode) the register-fragment kernel below
    if (estimate_tc_eligible(d, S, B))
        return launch_estimate_tc(Q, K, H, Hkv, L, d, S, B, mode, layer, head_base, A, ws, st);
    const int Ns = L / S, Nb = L / B;
    EstPlan pl;
    if (!plan_estimate(H, Hkv, d, S, B, Nb, &pl))
        return set_error(RR_ERR_UNSUPPORTED, "rr_estimate: no launch plan fits shared memory "
                                             "(H=%d Hkv=%d d=%d S=%d B=%d L=%d)", H, Hkv, d, S, B, L);
    uint32_t *frag = static_cast<uint32_t *>(ws);
    {
        const long total = (long)Hkv * Ns * (d / 8);
        const int threads = 256;
        const long want = (total + threads - 1) / threads;
        const int blocks = (int)(want < 148L * 16 ? want : 148L * 16);
        if (d == 128)
            pool_keys_kernel<128><<<blocks, threads, 0, st>>>(K, L, S, Ns, Hkv, frag);
        else
            pool_keys_kernel<64><<<blocks, threads, 0, st>>>(K, L, S, Ns, Hkv, frag);
        rr_status_t s = check_launch("rr_estimate: pool_keys_kernel");
        if (s != RR_OK) return s;
    }
    EstParams p;
    p.Q = Q;
    p.frag = reinterpret_cast<const uint4 *>(frag);
    p.A = A;
    p.H = H;
    p.L = L;
    p.S = S;
    p.r = B / S;
    p.Nb = Nb;
    p.NT = Ns / 8;
    p.NTB = p.r >= 8 ? p.r / 8 : 1;
    p.BPT = p.r >= 8 ? 1 : 8 / p.r;
    p.G = H / Hkv;
    p.hc = pl.hc;
    p.nHC = pl.nHC;
    p.R = pl.R;
    p.MT = pl.MT;
    p.MTW = pl.MTW;
    p.NG = pl.NG;
    p.WJ = pl.WJ;
    p.mode = mode;
    p.layer = layer;
    p.head_base = head_base;
    p.c_log2 = (float)(1.4426950408889634 / ((double)S * sqrt((double)d)));
    dim3 grid(Nb, Hkv * pl.nHC);
    auto launch = [&](auto kern) -> rr_status_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)pl.smem);
        if (e != cudaSuccess)
            return set_error(RR_ERR_CUDA, "rr_estimate: cudaFuncSetAttribute: %s",
                             cudaGetErrorString(e));
        kern<<<grid, kEstThreads, pl.smem, st>>>(p);
        return check_launch("rr_estimate: estimate_kernel");
    };
    if (p.BPT == 1) {
        if (d == 128)
            return pl.MTW == 2 ? launch(estimate_kernel<128, 2, 1>) : launch(estimate_kernel<128, 1, 1>);
        return pl.MTW == 2 ? launch(estimate_kernel<64, 2, 1>) : launch(estimate_kernel<64, 1, 1>);
    }
    if (d == 128)
        return pl.MTW == 2 ? launch(estimate_kernel<128, 2, 2>) : launch(estimate_kernel<128, 1, 2>);
    return pl.MTW == 2 ? launch(estimate_kernel<64, 2, 2>) : launch(estimate_kernel<64, 1, 2>);
}

}  // namespace rr
