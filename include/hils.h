/*
 * hils.h — C ABI of the HiLS-Attention hot path on NVIDIA B200 (sm_100a).
 *
 * Method: "Hierarchical Sparse Attention Done Right: Toward Infinite Context Modeling"
 * (arXiv 2607.02980). Four stages: (a) landmark chunk summaries (Eq. 8), (b) retrieval scores
 * (Eq. 7) and GQA-shared top-k chunk selection (Sec. 3 RQ1, Sec. 4 "GQA"), (c) softmax attention of
 * each query within each selected chunk and within its chunk-aligned causal sliding window
 * (Sec. 2), (d) fusion of the per-chunk outputs by softmax(s^) over the selected chunks plus the
 * window (Eq. 10), in prefill, decode (one or up to 8 query tokens) and backward forms. Beside them:
 * stage (a) with one shared landmark query per head (Sec. 4), stage (b) with the Q-Cal projection
 * fused in (Sec. 4), and the naive block-sparse selection on exact chunk masses (Sec. 2) as the
 * reference for selection quality.
 *
 * Conventions shared by every call
 * --------------------------------
 * Sizes (hils_params): B batch, T query rows, L KV length, Hq query heads, Hkv KV heads
 * (G = Hq/Hkv heads share one KV head: query head h reads KV head h/G), d head dim, S chunk size,
 * topk chunks kept per query, window W, q_pos0 = absolute position of query row 0 (row i sits at
 * p = q_pos0 + i and attends keys at positions <= p), scale tau (0 => 1/sqrt(d)).
 * Nc = floor(L/S) complete chunks; chunk c holds tokens [c*S, (c+1)*S).
 * Window of position p: tokens [l_p, p] with l_p = S*floor(max(0, p-W+1)/S); its candidate chunks
 * are c < n_p = l_p/S (the chunks wholly left of the window; all complete).
 *
 * Tensors are dense, row-major, contiguous, 16-byte aligned device pointers:
 *   q, q_hat, out, dout, dq, dq_hat        [B, Hq, T, d]   element type = params.dtype
 *   k, v, dk, dv (prefill) / k_cache, v_cache [B, Hkv, L, d]   params.dtype
 *   q_land, dq_land                         [B, Hq, Nc, d]  params.dtype (one landmark query per chunk)
 *   k_sum                                   [B, Hq, Nc, d]  params.dtype (summary key k')
 *   b_sum                                   [B, Hq, Nc]     float32      (entropy bias b')
 *   idx                                     [B, Hkv, T, topk] int32 (ascending chunk ids, -1 padded)
 *   lse                                     [B, Hq, T]      float32 (natural-log log Z^_i)
 * An idx row is read as a set: entries outside [0, n_p) are ignored and a repeated id counts once.
 *
 * Ownership: the caller owns every buffer, including the workspace (size from
 * hils_workspace_size). The library keeps no state between calls. Every compute call is
 * asynchronous on `stream` and returns after enqueueing its kernels.
 * Errors: shapes, pointers, alignment and workspace size are checked before any launch
 * (HILS_ERR_INVALID_ARG / HILS_ERR_UNSUPPORTED / HILS_ERR_WORKSPACE, nothing enqueued); a failed
 * launch returns HILS_ERR_CUDA. hils_last_error() gives a thread-local message. No C++ exception
 * crosses this boundary.
 */
#ifndef HILS_H_
#define HILS_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HILS_API __attribute__((visibility("default")))
#else
#define HILS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *hils_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
    HILS_OK = 0,
    HILS_ERR_INVALID_ARG = 1, /* bad size, null or misaligned pointer */
    HILS_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels implement (e.g. d not 64/128) */
    HILS_ERR_WORKSPACE = 3,   /* workspace missing or smaller than hils_workspace_size() */
    HILS_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
    HILS_ERR_TIMEOUT = 5      /* a bounded device-side wait expired (reported by hils_check) */
} hils_status;

typedef enum { HILS_BF16 = 0, HILS_FP32 = 1 } hils_dtype;

typedef struct {
    int32_t B, T, L, Hq, Hkv, d, S, topk, window;
    int32_t q_pos0;   /* absolute position of query row 0: 0 for prefill, L-1 for decode */
    float scale;      /* tau; 0 => 1/sqrt(d) */
    int32_t dtype;    /* hils_dtype of q, k, v, q_hat, q_land, k_sum, out and the gradients */
} hils_params;

/* Operation ids for hils_workspace_size. */
enum { HILS_OP_SUMMARY = 0, HILS_OP_SELECT = 1, HILS_OP_ATTN_FWD = 2, HILS_OP_DECODE = 3, HILS_OP_ATTN_BWD = 4 };

/* Supported ranges (HILS_ERR_UNSUPPORTED outside them). */
#define HILS_MAX_S 128
#define HILS_MAX_TOPK 64

/*
 * Bytes of device workspace `op` needs for these sizes (0 = none; the pointer may then be NULL).
 * Returns (size_t)-1 if the sizes are invalid. Host-only, no CUDA call.
 */
HILS_API size_t hils_workspace_size(const hils_params *p, int op);

/*
 * Stage (a), Eq. 8 (Prop. 3.1, the landmark summary): for every b, query head h and complete chunk
 * c in [c_begin, c_end):  u_j = tau * q_land[b,h,c] . k[b,h/G,c*S+j],  p = softmax_j(u),
 *   k_sum[b,h,c] = sum_j p_j k_j  (stored in params.dtype),  b_sum[b,h,c] = -sum_j p_j log p_j.
 * Chunks outside the range are not touched, so a decode cache can be extended as chunks complete.
 * Uses q_land/k_sum/b_sum sized by Nc = floor(L/S); 0 <= c_begin <= c_end <= Nc. T, topk, window
 * and q_pos0 are not read. An empty range returns HILS_OK without reading any pointer. No workspace.
 */
HILS_API hils_status hils_chunk_summary(const hils_params *p, const void *k, const void *q_land, int32_t c_begin,
                               int32_t c_end, void *k_sum, float *b_sum, hils_stream_t stream);

/*
 * Stage (a) with the shared landmark query (Sec. 4, the alternative to landmark tokens: one learned
 * query vector per head and layer instead of one per chunk): exactly hils_chunk_summary with
 * q_land[b,h,c] := q_shared[h] for every b and c. q_shared [Hq, d] in params.dtype (16-byte aligned
 * for the bf16 fast path); every other argument, layout, range rule and error as hils_chunk_summary.
 * Forward only: the gradient for q_shared is the sum over (b, c) of hils_attn_bwd's dq_land.
 */
HILS_API hils_status hils_chunk_summary_shared_query(const hils_params *p, const void *k, const void *q_shared,
                                                     int32_t c_begin, int32_t c_end, void *k_sum, float *b_sum,
                                                     hils_stream_t stream);

/*
 * Stage (b), Eq. 7 + Sec. 3 RQ1 + Sec. 4 "GQA": for every (b, KV group g, row i) with n = n_p
 * candidates:  s^_{h,c} = tau * q_hat[b,h,i] . k_sum[b,h,c] + b_sum[b,h,c]  for c < n and each head h
 * of the group; group score g_c = max_h (s^_{h,c} - LSE_{c'<n} s^_{h,c'}); keep the min(topk, n)
 * largest by (g_c desc, c asc). idx[b,g,i,:] = those ids ascending, then -1.
 * gap (nullable, float32 [B, Hkv, T]) = g_(topk) - g_(topk+1), +inf when n <= topk.
 * shat (nullable, float32 [B, Hq, T, topk]): shat[b,h,i,t] = s^_{h, idx[b,g,i,t]} for each head h of
 * group g, -inf where idx is -1: the retrieval scores hils_attn_fwd_shat takes with idx.
 * Scores in fp32. On the tensor-core path (bf16, d 128, G <= 4, topk <= 32, 1..128 candidates per row)
 * the top-k compares keys that keep 16 mantissa bits of g_c, so two candidates whose scores are within
 * |g_c| * 2^-16 of each other order by chunk id. Otherwise supports G * Nc * 4 + next_pow2(Nc) * 8 <= 200
 * KiB of shared memory per row (Nc <= 8192 at G = 4); longer contexts use hils_decode. Outputs 16-byte
 * aligned. Workspace: none.
 */
HILS_API hils_status hils_select_topk(const hils_params *p, const void *q_hat, const void *k_sum, const float *b_sum,
                             int32_t *idx, float *gap, float *shat, void *workspace, size_t workspace_bytes,
                             hils_stream_t stream);

/*
 * hils_select_topk with the Q-Cal projection (Sec. 4) fused into the score kernel: the retrieval query
 * is q^ = q + W_up (W_down q) (rank 32, the token's own query as h, one pair shared by all heads), formed
 * tile by tile in shared memory; no q^ tensor is read or written. q [B, Hq, T, d]; w_down [32, d] and
 * w_up [d, 32] row-major, params.dtype, 16-byte aligned. Outputs (idx, gap, shat), layouts and errors as
 * hils_select_topk; with shat, a Q-Cal model reaches hils_attn_fwd_shat without ever forming q^.
 * Only the tensor-core shapes (bf16, d 128, G <= 4, topk <= 32, 1..128 candidates per row) and rank 32
 * are taken (HILS_ERR_UNSUPPORTED otherwise: form q^ and call hils_select_topk). No workspace.
 */
HILS_API hils_status hils_select_topk_qcal(const hils_params *p, const void *q, const void *w_down, const void *w_up,
                                           int32_t rank, const void *k_sum, const float *b_sum, int32_t *idx,
                                           float *gap, float *shat, hils_stream_t stream);

/*
 * Naive block-sparse attention selection (Sec. 2), the exact counterpart of hils_select_topk: for every
 * (b, query head h, row i) at position p with n = n_p candidates, the exact chunk mass
 *   mass[b,h,i,c] = LSE_{j in chunk c} tau q[b,h,i].k[b,h/G,j]   for c < n (entries c >= n untouched),
 * then the group rule of hils_select_topk with mass in place of s^: per-head normalisation over the
 * candidates, max over the group's heads, the min(topk, n) largest by (score desc, c asc).
 * idx [B, Hkv, T, topk] int32 (ascending ids, -1 padded); gap (nullable) [B, Hkv, T] as in
 * hils_select_topk; mass [B, Hq, T, Nc] fp32 (nullable when Nc = 0). q [B, Hq, T, d], k [B, Hkv, L, d].
 * Reads every pre-window key once per query row (O(T * L) work): a reference for selection quality,
 * not a step of the HiLS path. Needs topk <= 32 and at most 1024 candidates per row
 * (HILS_ERR_UNSUPPORTED otherwise). Tensor cores for bf16, d 128, S 64, G in {1, 2, 4, 8}.
 * No workspace.
 */
HILS_API hils_status hils_bsa_select_topk(const hils_params *p, const void *q, const void *k, int32_t *idx, float *gap,
                                          float *mass, hils_stream_t stream);

/*
 * Stages (c)+(d), Eq. 10 (chunked prefill form): for every (b, h, row i) at position p:
 *   window logits s_j = tau q.k_j, j in [l_p, p];  for each selected chunk c (idx, as a set):
 *   s^_c (as above), L_c = LSE_{j in c} s_j, o_c = sum_j exp(s_j - L_c) v_j;
 *   lse = log Z^ = LSE({s_j}_window U {s^_c}_selected);
 *   out = sum_window exp(s_j - lse) v_j + sum_c exp(s^_c - lse) o_c.
 * The per-chunk outputs o_c never reach memory: each chunk's weights are scaled by
 * exp(s^_c - L_c) before its value product. fp32 accumulation.
 * Workspace: hils_workspace_size(p, HILS_OP_ATTN_FWD) bytes (non-zero on the tensor-core path:
 * bf16, d 128, S 64, G <= 4, topk <= 32, at most 128 candidate chunks per row).
 */
HILS_API hils_status hils_attn_fwd(const hils_params *p, const void *q, const void *k, const void *v, const void *q_hat,
                          const void *k_sum, const float *b_sum, const int32_t *idx, void *out, float *lse,
                          void *workspace, size_t workspace_bytes, hils_stream_t stream);

/*
 * hils_attn_fwd given the selection's retrieval scores instead of recomputing them: the same Eq. 10
 * (out, lse) with s^_c read from shat [B, Hq, T, topk] fp32 (slot t of row (b, h, i) scores chunk
 * idx[b, h/G, i, t], as hils_select_topk writes it). q_hat, k_sum and b_sum are not needed.
 * idx must be in the canonical form hils_select_topk writes: per row, candidate ids (c < n_p) strictly
 * ascending, then -1. A row that is not raises a device error word (hils_check then returns
 * HILS_ERR_INVALID_ARG) and that call's output is invalid; no memory outside the arguments is touched.
 * Tensor-core shapes only: bf16, d 128, S 64, 128 % G == 0, topk <= 32, at most 8192 chunks
 * (HILS_ERR_UNSUPPORTED otherwise: call hils_attn_fwd). Pointers 16-byte aligned. No workspace.
 */
HILS_API hils_status hils_attn_fwd_shat(const hils_params *p, const void *q, const void *k, const void *v,
                                        const int32_t *idx, const float *shat, void *out, float *lse,
                                        hils_stream_t stream);

/*
 * One decode step (stages b-d) for T = M query tokens per sequence at positions q_pos0 .. L-1 with
 * q_pos0 = L-M (M = 1: the usual single-token step; 2 <= M <= 8: multi-token decode, e.g. verifying M
 * speculated tokens, each query with its own window and selection) over a KV cache of L tokens that
 * already holds them: scores every candidate chunk's summary (each summary row read once for all M
 * queries), selects topk chunks per KV group and query as hils_select_topk does, attends, and fuses
 * as hils_attn_fwd does. q, q_hat [B, Hq, M, d]; out [B, Hq, M, d]; lse [B, Hq, M]; idx_out (nullable)
 * [B, Hkv, M, topk]. M > 1 needs bf16, d 128, S 64, G <= 8, topk <= 32 and 16-byte aligned q, q_hat,
 * caches and k_sum (HILS_ERR_UNSUPPORTED otherwise).
 * Workspace: hils_workspace_size(p, HILS_OP_DECODE) bytes.
 */
HILS_API hils_status hils_decode(const hils_params *p, const void *q, const void *q_hat, const void *k_cache,
                        const void *v_cache, const void *k_sum, const float *b_sum, void *out, float *lse,
                        int32_t *idx_out, void *workspace, size_t workspace_bytes, hils_stream_t stream);

/*
 * Backward of hils_chunk_summary + hils_attn_fwd for loss = sum(dout * out), idx held fixed (the
 * hard top-k is not differentiable; gradients reach q_land through s^ -> k_sum, b_sum -> Eq. 8):
 *   window: ds_j = a_j (dout.v_j - D), dv_j += a_j dout,  a_j = exp(s_j - lse), D = dout.out
 *   chunk:  ds^_c = b_c (dout.o_c - D), ds_j = b_c pi_cj (dout.v_j - dout.o_c), dv_j += b_c pi_cj dout
 *   dq = tau sum ds_j k_j, dk_j += tau ds_j q, dq_hat = tau sum ds^_c k_sum_c,
 *   dk_sum_c += tau ds^_c q_hat, db_sum_c += ds^_c;  Eq. 8 backward:
 *   du_j = p_j (dk_sum.(k_j - k_sum) - db_sum (log p_j + b_sum)), dq_land = tau sum du_j k_j,
 *   dk_j += p_j dk_sum + tau du_j q_land.
 * out and lse must be this forward's outputs. Every gradient is fully overwritten (fp32
 * accumulation, stored in params.dtype). Requires q_pos0 == 0 and T == L (self-attention prefill).
 * Workspace: hils_workspace_size(p, HILS_OP_ATTN_BWD) bytes.
 */
HILS_API hils_status hils_attn_bwd(const hils_params *p, const void *q, const void *k, const void *v, const void *q_hat,
                          const void *q_land, const void *k_sum, const float *b_sum, const int32_t *idx,
                          const void *out, const float *lse, const void *dout, void *dq, void *dk, void *dv,
                          void *dq_hat, void *dq_land, void *workspace, size_t workspace_bytes,
                          hils_stream_t stream);

/*
 * A decode step that allocates nothing. The paper has no counterpart: this exists for callers that
 * cannot hand the library a workspace (a serving engine whose memory planner owns the whole device
 * and forbids library-side allocation, a foreign-language binding that passes tensor pointers but
 * has no device allocator, a latency-critical loop that cannot afford cudaMalloc's implicit
 * synchronisation). Same inputs, outputs, rules and results as hils_decode; the scratch lives in a
 * static __device__ array of HILS_DECODE_NOALLOC_MAX_BYTES that every GPU loading this library
 * holds until the process exits.
 *  - Sizes whose decode workspace (hils_workspace_size(p, HILS_OP_DECODE)) exceeds the array are
 *    rejected with HILS_ERR_UNSUPPORTED before anything is enqueued.
 *  - The first call on a device (with that device current) looks up the array's device address
 *    with cudaGetSymbolAddress; make that first call before any stream capture. Later calls reuse it
 *    for the life of the process, so a cudaDeviceReset (or anything else that destroys the device's
 *    primary context) invalidates it: do not call this entry point on that device afterwards.
 *  - All calls on a device share the one array and it keeps the previous call's contents: calls
 *    whose GPU work overlaps (e.g. on two streams without ordering between them) race and corrupt
 *    each other's results; order them on one stream or with events. Every scratch byte a call reads
 *    is written earlier in the same call, so nothing needs clearing between calls.
 *  - No cudaMalloc, cudaFree or allocating library routine is called.
 */
#define HILS_DECODE_NOALLOC_MAX_BYTES (32u << 20)
HILS_API hils_status hils_decode_noalloc(const hils_params *p, const void *q, const void *q_hat,
                                         const void *k_cache, const void *v_cache, const void *k_sum,
                                         const float *b_sum, void *out, float *lse, int32_t *idx_out,
                                         hils_stream_t stream);

/*
 * Test hook of the failure detection; the paper has no counterpart. Every kernel of this library waits on
 * its copies and tensor-core operations with a bounded mbarrier wait; when a wait runs out the kernel
 * records it in a device error word and leaves, and the next hils_check returns HILS_ERR_TIMEOUT. This call
 * runs that same wait in one CTA on a barrier that nothing arrives at (arrive_first = 0), with a limit of
 * max_polls polls (1 .. HILS_TEST_WAIT_MAX_POLLS), so the wait expires and is
 * recorded; with arrive_first != 0 the CTA arrives first and the wait completes (a control). The barrier
 * is fed by no copy and no tensor-core operation, so nothing is left in flight and the context stays
 * usable. Returns after enqueueing; the outcome is read with hils_check. HILS_ERR_INVALID_ARG for a
 * max_polls outside the range.
 */
#define HILS_TEST_WAIT_MAX_POLLS (1u << 20)
HILS_API hils_status hils_test_wait_expiry(uint32_t max_polls, int32_t arrive_first, hils_stream_t stream);

/* Waits for `stream`, then reports a device-side error word (HILS_ERR_TIMEOUT) or a CUDA error. */
HILS_API hils_status hils_check(hils_stream_t stream);

HILS_API const char *hils_status_string(hils_status s);
HILS_API const char *hils_last_error(void); /* thread-local message for the last failing call */
HILS_API const char *hils_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HILS_H_ */
