/*
 * rr_attn.h -- C ABI of librrattn.so: the prefill hot path of RRAttention
 * ("RRAttention: Dynamic Block Sparse Attention via Per-Head Round-Robin Shifts for
 * Long-Context Inference", paperpeel.com/paper/2602.05853) on NVIDIA B200 (sm_100a).
 *
 * Three calls, in the order the paper's pipeline runs them (Sec. 1 contributions (i)-(iii)):
 *   rr_estimate        round-robin query sampling + stride-level importance -> block scores
 *   rr_select          adaptive Top-tau block selection -> per-head CSR block lists
 *   rr_sparse_prefill  causal block-sparse attention over the selected blocks -> O
 *
 * Conventions shared by every call
 *   - Batch 1.  Q and O are [H][L][d], K and V are [Hkv][L][d], all contiguous row-major
 *     bfloat16 (rr_bf16_t holds the raw bit pattern).  Query head h reads KV head
 *     h / (H / Hkv) (grouped-query attention, contiguous groups).
 *   - Every pointer is a DEVICE pointer owned by the caller; the library allocates no
 *     device memory.  Every pointer must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *     Calls only enqueue work on it: they never synchronise the device or the stream.
 *   - Arguments are validated on the host before anything is launched.  A rejected call
 *     returns RR_ERR_INVALID_ARG / RR_ERR_UNSUPPORTED / RR_ERR_WORKSPACE and launches
 *     nothing; a failed launch returns RR_ERR_CUDA.  rr_last_error() then holds a
 *     human-readable reason (per calling thread).  No kernel traps or asserts.
 *   - L = 0 is accepted by every call as an empty problem: nothing is launched.
 *   - Supported: d in {64, 128}; B in {64, 128}; 1 <= S <= B with B % S == 0 and B/S = 4
 *     or a multiple of 8; (L/S) % 8 == 0; L % B == 0; H % Hkv == 0; L <= 2^20; H <= 256.
 */
#ifndef RR_ATTN_H
#define RR_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RR_OK = 0,
    RR_ERR_INVALID_ARG = 1, /* null/misaligned pointer, inconsistent sizes, bad tau */
    RR_ERR_UNSUPPORTED = 2, /* a size outside the supported set above */
    RR_ERR_CUDA = 3,        /* a CUDA launch or runtime call failed */
    RR_ERR_WORKSPACE = 4    /* workspace missing or smaller than *_workspace_bytes() */
} rr_status_t;

typedef uint16_t rr_bf16_t;
typedef void *rr_stream_t;

/* Round-robin strategies (Sec. 4.3, Table 6).  The offset of the sampled query inside
 * stride i is: HEAD -> h mod S (the method's default), NONE -> S-1 for every head,
 * LAYER -> layer mod S, HYBRID -> (h + layer) mod S. */
typedef enum { RR_HEAD = 0, RR_NONE = 1, RR_LAYER = 2, RR_HYBRID = 3 } rr_strategy_t;

/* Bytes of device workspace rr_estimate needs for these sizes (0 when L = 0). */
size_t rr_estimate_workspace_bytes(int H, int Hkv, int L, int d, int S, int B);

/*
 * rr_estimate -- stride-level block importance (Sec. 3.1 heading, Sec. 3.2, Sec. 3.3 heading).
 *
 * For each query head h and stride i (Ns = L/S strides of S tokens) one query is sampled,
 * at position P(i,h) = i*S + (h mod S) (head round-robin).  Keys are pooled per stride,
 * Kbar_j = sum of the S keys of stride j, and the stride-level scores
 *     z(h,i,j) = Q[h][P(i,h)] . Kbar[g(h)][j] / (S * sqrt(d)),   j <= i,
 * are normalised by a softmax over j (stride-level softmax).  The probabilities are summed
 * over the (B/S) x (B/S) strides of each block pair and scaled by S/B:
 *     block_scores[h][I][J] = (S/B) * sum_{i in I} sum_{j in J, j <= i} p(h,i,j),
 * so every row sums to 1.  block_scores is [H][L/B][L/B] float32 and is fully written:
 * entries with J > I are 0.
 *
 * Arithmetic: pooled keys are summed in fp32 and split into two bf16 terms (hi + lo);
 * logits come from bf16 tensor-core products with fp32 accumulation; softmax and block
 * sums in fp32.  workspace: at least rr_estimate_workspace_bytes(...) bytes, caller-owned,
 * contents undefined on entry and exit.
 */
rr_status_t rr_estimate(const rr_bf16_t *Q, const rr_bf16_t *K, int H, int Hkv, int L, int d,
                        int S, int B, float *block_scores, void *workspace,
                        size_t workspace_bytes, rr_stream_t stream);

/* rr_estimate with an explicit round-robin strategy and layer index (Sec. 4.3 Table 6). */
rr_status_t rr_estimate_strategy(const rr_bf16_t *Q, const rr_bf16_t *K, int H, int Hkv, int L,
                                 int d, int S, int B, rr_strategy_t strategy, int layer,
                                 float *block_scores, void *workspace, size_t workspace_bytes,
                                 rr_stream_t stream);

/*
 * rr_estimate_heads -- rr_estimate_strategy for a slice of whole KV groups of a layer.
 *
 * Every step of the estimate is independent per query head, so a layer may be processed in
 * slices (a pipeline over host copies, or KV groups sharded across GPUs).  Q points at the
 * slice's first query head and K at its first KV head; H and Hkv are the slice's counts (the
 * slice must hold whole KV groups, so the GQA mapping inside it is the layer's).  head_base is
 * the layer-wide index of the slice's first query head: the round-robin offset of local head h
 * is that of head head_base + h (HEAD: (head_base + h) mod S; HYBRID: (head_base + h + layer)
 * mod S), so the slice's block_scores equal rows [head_base, head_base + H) of the whole
 * layer's.  0 <= head_base <= 2^20, else RR_ERR_INVALID_ARG.  The page defines no slicing;
 * this entry point only carries the head index across the cut.
 */
rr_status_t rr_estimate_heads(const rr_bf16_t *Q, const rr_bf16_t *K, int H, int Hkv, int L, int d,
                              int S, int B, rr_strategy_t strategy, int layer, int head_base,
                              float *block_scores, void *workspace, size_t workspace_bytes,
                              rr_stream_t stream);

/*
 * rr_xattn_estimate -- XAttention's antidiagonal block importance, the estimator the paper
 * compares pattern-discovery time against (Sec. 2.2; Sec. 4.2 "Runtime Efficiency", Fig. 3(b);
 * the XAttention card, "Summary" and "Key points").  Not part of the RRAttention path.
 *
 * Inside every S x S sub-block of the logits (query stride i, key stride j) the antidiagonal
 * from lower-left to upper-right is summed and scaled like the round-robin score:
 *     z(h,i,j) = (1 / (S sqrt(d))) * sum_{u<S} Q[h][iS+S-1-u] . K[g(h)][jS+u],   j <= i,
 * normalised by a softmax over j and aggregated exactly like rr_estimate's scores:
 *     block_scores[h][I][J] = (S/B) * sum_{i in I} sum_{j in J, j <= i} p(h,i,j)
 * ([H][L/B][L/B] float32, fully written, J > I entries 0), so rr_select applies unchanged.
 * bf16 tensor-core products with fp32 accumulation over the S*d-long antidiagonal sums; softmax
 * and block sums in fp32.  No workspace.  Supported: d in {64, 128}; B/S in {4, 8, 16, 32};
 * (L/S) % 8 == 0; the common size rules above.
 */
rr_status_t rr_xattn_estimate(const rr_bf16_t *Q, const rr_bf16_t *K, int H, int Hkv, int L, int d,
                              int S, int B, float *block_scores, rr_stream_t stream);

/* Bytes of device workspace rr_select needs for H heads and Nb blocks per row. */
size_t rr_select_workspace_bytes(int H, int Nb);

/*
 * rr_select -- adaptive Top-tau block selection (Sec. 1 contribution (iii), Sec. 3.3
 * heading; the selection rule as stated for XAttention: the smallest set of blocks whose
 * cumulative score reaches tau) with last-query-block protection (Sec. 4.3).
 *
 * For every head h and query block I (row r = h*Nb + I) the causal scores
 * block_scores[h][I][0..I] are ordered by (score descending, J ascending); with T the row
 * total and cum_k the sum of the first k, the row keeps the first k* blocks where k* is the
 * smallest k with cum_k >= tau * T.  Precision of the decision: for rows of up to 1024
 * blocks the sums are exact integers on a fixed-point grid set by the row maximum (every
 * score keeps its bits down to 2^-50 of the maximum) and tau * T is formed in float64 and
 * rounded up to that grid; longer rows sum in float64.  tau >= 1, or protect_last != 0 and
 * I = Nb-1, keeps all I+1 blocks.  Every row keeps at least 1 block.
 *
 * Output (device, caller-owned): row_ptr int32 [H*Nb + 1] (row_ptr[0] = 0) and col_idx
 * int32 [col_capacity]; row r's blocks are col_idx[row_ptr[r] .. row_ptr[r+1]) in strictly
 * ascending order, every J <= I.  *nnz_out (device int64) = row_ptr[H*Nb].
 * col_capacity must be >= H*Nb*(Nb+1)/2 (the all-blocks worst case) or the call is
 * rejected before any launch.  tau must be in (0, 1]; block_scores entries must be finite
 * and >= 0 (as rr_estimate writes them).
 */
rr_status_t rr_select(const float *block_scores, int H, int Nb, double tau, int protect_last,
                      int32_t *row_ptr, int32_t *col_idx, int64_t col_capacity,
                      int64_t *nnz_out, void *workspace, size_t workspace_bytes,
                      rr_stream_t stream);

/*
 * rr_select_noalloc -- rr_select without a caller-provided workspace.  The paper has no
 * counterpart to this call: it exists for callers that cannot allocate device memory (a
 * plugin whose host application owns all device memory and offers no allocation hook, or a
 * latency-critical path that must not call cudaMalloc/cudaFree).  Same arguments, results
 * and validation as rr_select, minus workspace/workspace_bytes; the library allocates
 * nothing and calls no allocating routine.
 *
 * Scratch: a fixed 8 MiB array compiled into the library (held by every GPU that loads it
 * until the process exits).  Sizes with rr_select_workspace_bytes(H, Nb) > 8 MiB are rejected
 * with RR_ERR_UNSUPPORTED before any launch.  The first call on a device (with that device
 * current) looks up the array's device address and keeps it; make it before any stream
 * capture.  If that lookup fails the call returns RR_ERR_CUDA and the next call retries it.
 * All calls share the array: calls that overlap on the GPU (unordered streams or threads)
 * race; each call writes every scratch word it reads, so no clearing is needed.
 */
rr_status_t rr_select_noalloc(const float *block_scores, int H, int Nb, double tau,
                              int protect_last, int32_t *row_ptr, int32_t *col_idx,
                              int64_t col_capacity, int64_t *nnz_out, rr_stream_t stream);

/*
 * rr_sparse_prefill -- causal block-sparse attention over the selected blocks (Sec. 2.1
 * with the CSR as the block selection matrix).  For query row t of head h, in block
 * I = t / B, key k of KV head g(h) is attended iff k <= t and k / B is listed in row
 * h*Nb + I of the CSR:
 *     O[h][t] = sum_k softmax_k(scale * Q[h][t] . K[g][k]) V[g][k]   over those keys.
 * softmax_scale <= 0 selects 1/sqrt(d).  bf16 inputs, fp32 accumulation and softmax, bf16
 * output.  The CSR must be well formed (as rr_select writes it): ascending, J <= I, at least
 * one block per row; rr_validate_csr checks a CSR on the device.
 */
rr_status_t rr_sparse_prefill(const rr_bf16_t *Q, const rr_bf16_t *K, const rr_bf16_t *V,
                              int H, int Hkv, int L, int d, int B, const int32_t *row_ptr,
                              const int32_t *col_idx, float softmax_scale, rr_bf16_t *O,
                              rr_stream_t stream);

/*
 * rr_validate_csr -- counts malformed CSR rows on the device without trapping.  A row is
 * malformed if its range is negative, empty or out of [0, nnz_cap], or an entry is out of
 * [0, I] or not strictly ascending.  *bad_rows (device int32) is overwritten with the count.
 */
rr_status_t rr_validate_csr(const int32_t *row_ptr, const int32_t *col_idx, int H, int Nb,
                            int64_t nnz_cap, int32_t *bad_rows, rr_stream_t stream);

/*
 * rr_device_errors -- error bits the kernels recorded on the current device instead of
 * trapping: bit 0 producer, bit 1 MMA issuer, bit 2 softmax warps of rr_sparse_prefill, bit 3
 * a warp of rr_estimate's tensor-core kernel gave up a wait after about one second, bit 4 one of
 * rr_xattn_estimate's.  *flags
 * (host) receives the bits; reset != 0 clears them.
 * Synchronous: waits for the device's preceding work.
 */
rr_status_t rr_device_errors(uint32_t *flags, int reset);

/*
 * rr_selftest_wait -- exercises the bounded wait the kernels use in place of an unbounded
 * spin (no counterpart in the paper).  A one-thread kernel waits on an mbarrier phase that
 * nothing completes; after timeout_us (1 .. 2,000,000) it must give up; it then completes the
 * phase itself and waits again, which must succeed.  result (host, 3 elements): [0] = 1 if
 * the first wait gave up, [1] = 1 if the second saw the phase, [2] = microseconds the first
 * wait took.  Synchronous on the legacy default stream; touches no other library state.
 */
rr_status_t rr_selftest_wait(uint32_t timeout_us, uint32_t *result);

/* Static text for a status code. */
const char *rr_status_string(rr_status_t s);

/* Text of the last failure on the calling thread ("" if none). */
const char *rr_last_error(void);

/* Library version: major*10000 + minor*100 + patch. */
int rr_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RR_ATTN_H */
