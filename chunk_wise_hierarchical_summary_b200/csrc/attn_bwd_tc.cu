// Backward of summaries + Eq. 10 attention on the tensor cores (bf16, d 128, S 64, G <= 4), selection
// held fixed ("Hierarchical Sparse Attention Done Right", Sec. 3 RQ2: the LM-loss gradient reaches the
// landmark summaries through s^ in Z^; Eq. 8 / Prop. 3.1 for the summaries).
//
// Per row r = (query i, head h), with lse = log Z^ and D_r = dout_r . out_r saved by the forward:
//   window token j:          P_j = exp(s_j - lse),                     ds_j = P_j (dP_j - D_r)
//   token j of a selected c: P_j = beta_c pi_cj, beta_c = exp(s^_c - lse), pi_c = softmax_j(s_cj),
//                            ds_j = P_j (dP_j - doo_c), doo_c = sum_j pi_cj dP_j,  ds^_c = beta_c (doo_c - D_r)
//   (dP_j = dout_r . v_j; s already includes tau). Then dq = tau sum_j ds_j k_j, dk_j = tau sum_r ds_j q_r,
//   dv_j = sum_r P_j dout_r, dq^ = tau sum_c ds^_c k'_c, dk'_c = tau sum_r ds^_c q^_r, db'_c = sum_r ds^_c,
//   and the Eq. 8 backward turns (dk'_c, db'_c) into dq'_c and a second share of dk_j.
//
// Launches (all deterministic, no floating-point atomics):
//   gather   canonical ids + s^ per (row, slot)                          (select_tc.cu, GATHER mode)
//   delta    D_r
//   bq       query-major, tcgen05: CTA = 128 rows (128/G queries x G heads) over the union of their
//            chunks (as the forward): S = Q K^T and dP = dO V^T into TMEM, ds written over S in TMEM as
//            bf16 pairs, dQ += ds K with ds read from TMEM. Two groups of four row warps take alternate
//            tiles (rows need no running state in the backward). ds^ goes to a dense [rows x Nc] bf16
//            matrix and beta = exp(s^ - lse) to a dense fp32 one (both zero where a chunk is not
//            selected).
//   dqhat    dq^ = tau ds^ K'  (warp per row, the head's summaries in shared memory)
//   dksum    dk'^T, db' = the dense ds^ matrix contracted with q^ over the rows (mma.sync), split in
//            sixteen row ranges whose partials the next launch sums in a fixed order
//   eq8      per (b, KV group, chunk): the Eq. 8 backward: dq' and an fp32 share of dk
//   bkv      KV-major, tcgen05: CTA = one chunk (64 keys, K and V resident) streaming the query tiles
//            that can reach it (a row's beta for the chunk, lse and D fetched one tile ahead); S, dP as in
//            bq, then P and ds (bf16, 128-byte swizzled, MN-major) in
//            shared memory feed dV^T += dO^T P and dK^T += Q^T ds with both operands read transposed.
#include <algorithm>

#include "internal.h"
#include "mma_sync.cuh"
#include "tcgen05.cuh"

namespace hils {

bool make_tmap_bf16_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint64_t ld,
                       uint32_t box_rows);
bool make_tmap_bf16_3d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1_bytes,
                       uint64_t s2_bytes, uint32_t b1, uint32_t b2);
cudaError_t launch_gather_shat_tc(const Dims &D, const void *q_hat, const void *k_sum, const float *b_sum,
                                  const int *idx, int *ws_idx, float *ws_shat, cudaStream_t stream);
bool attn_fwd_tc_supported(const Dims &D, int dtype);

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kHalf = 16384;     // one 64-column half of a 128-row tile
constexpr uint32_t kRowTile = 32768;  // 128 rows x 128 columns bf16
constexpr uint32_t kKvTile = 16384;   // 64 tokens x 128 columns bf16
constexpr int kListCap = 1024;
constexpr int kBitmapWords = 256;
constexpr int kMaxK = 32;
constexpr int kTcThreads = 320;  // producer, MMA issuer, two groups of four row warps
constexpr int kBqStages = 3;
constexpr int kDkSplit = 16;  // row ranges of the dk'/db' reduction (partials summed in order)
constexpr int kPartStride = 129;  // dk'(128) + db'(1) per (b, h, split, chunk)

__device__ unsigned int g_bwd_tc_errors = 0;

// ------------------------------------------------------------------------------------------ delta

__global__ void bwd_delta_kernel(const __nv_bfloat16 *__restrict__ out, const __nv_bfloat16 *__restrict__ dout,
                                 float *__restrict__ Dbuf, long long rows) {
    const long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 4;
    const int l = threadIdx.x & 15;
    float s = 0.f;
    if (r < rows) {
        float a[8], c[8];
        load8(out + r * 128 + 8 * l, a);
        load8(dout + r * 128 + 8 * l, c);
#pragma unroll
        for (int e = 0; e < 8; ++e) s = fmaf(a[e], c[e], s);
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (l == 0 && r < rows) Dbuf[r] = s;
}

// One row's ds over a 64-token tile, shared by bq and bkv, in two phases so that the dP load from TMEM
// overlaps the exponentials. kind: 1 selected chunk, 2 window, 0 neither.
// Phase A: s = the row's raw logits (q . k) in, e_j out (window rows: e_j = P_j; others relative to the
// tile max); returns z = sum e_j.
__device__ __forceinline__ float row_grad_a(float (&s)[64], int kind, int lo, int hi, float sc2, float lse2,
                                            bool warp_needs_mask) {
    if (warp_needs_mask) {
        const int mlo = kind == 2 ? lo : 0, mhi = kind == 2 ? hi : 63;
#pragma unroll
        for (int e = 0; e < 64; ++e) s[e] = (e >= mlo && e <= mhi) ? s[e] : -INFINITY;
    }
    float mx[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) mx[e] = s[e];
#pragma unroll
    for (int e = 8; e < 64; ++e) mx[e & 7] = fmaxf(mx[e & 7], s[e]);
    const float m2 = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                     sc2;
    // window rows: e_j = P_j directly (base lse); other rows: base = the tile max (e_j <= 1)
    const float base = kind == 2 ? lse2 : m2;
    const float2 sc = make_float2(sc2, sc2), nb = make_float2(-base, -base);
    float2 za[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        float2 t = __ffma2_rn(make_float2(s[2 * e], s[2 * e + 1]), sc, nb);
        t.x = ex2_approx(t.x);
        t.y = ex2_approx(t.y);
        s[2 * e] = t.x;
        s[2 * e + 1] = t.y;
        za[e & 1] = __fadd2_rn(za[e & 1], t);
    }
    return (za[0].x + za[0].y) + (za[1].x + za[1].y);
}
// Phase B: dp = dout . v_j in, ds_j out; s: e_j in, P_j out. beta = exp(s^_c - lse) of a selected chunk.
// Returns ds^ of a selected chunk.
__device__ __forceinline__ float row_grad_b(float (&s)[64], float (&dp)[64], int kind, float z, float beta,
                                           float Dr) {
    float2 zo[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
    for (int e = 0; e < 32; ++e)
        zo[e & 1] = __ffma2_rn(make_float2(s[2 * e], s[2 * e + 1]), make_float2(dp[2 * e], dp[2 * e + 1]), zo[e & 1]);
    const float eo = (zo[0].x + zo[0].y) + (zo[1].x + zo[1].y);
    float f = 0.f, delta = 0.f, dshat = 0.f;
    if (kind == 1) {
        const float iz = 1.f / z;
        const float doo = eo * iz;
        f = beta * iz;
        delta = doo;
        dshat = beta * (doo - Dr);
    } else if (kind == 2) {
        f = 1.f;
        delta = Dr;
    }
    const float2 f2 = make_float2(f, f), nd = make_float2(-delta, -delta);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const float2 p = __fmul2_rn(make_float2(s[2 * e], s[2 * e + 1]), f2);
        const float2 g = __fmul2_rn(p, __fadd2_rn(make_float2(dp[2 * e], dp[2 * e + 1]), nd));
        s[2 * e] = p.x;
        s[2 * e + 1] = p.y;
        dp[2 * e] = g.x;
        dp[2 * e + 1] = g.y;
    }
    return dshat;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// ------------------------------------------------------------------------------------------ bq

struct BqBars {
    uint64_t q_full, k_full[kBqStages], k_empty[kBqStages], v_full[kBqStages], v_empty[kBqStages], s_full[2],
        ds_full[2], buf_free[2], dq_final;
};

__global__ void __launch_bounds__(kTcThreads, 1)
bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap domap,
                 const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap, Dims D,
                 const int *__restrict__ ws_idx, const float *__restrict__ ws_shat, const float *__restrict__ lse,
                 const float *__restrict__ Dbuf, __nv_bfloat16 *__restrict__ dS, float *__restrict__ betas, int ncp,
                 __nv_bfloat16 *__restrict__ dq) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) BqBars bar;
    __shared__ uint32_t s_tmem;
    __shared__ uint32_t bitmap[kBitmapWords];
    __shared__ int list[kListCap];
    __shared__ int s_ntiles;
    __shared__ int lc[128][kMaxK];    // per query of the tile (128/G of them): selected chunks ascending, -1 padded
    __shared__ float lsh[128][kMaxK];  // per row: the matching s^ in log2 units
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = D.G, QT = 128 / G;
    // late query tiles visit the most chunks: launch them first, across all (b, group), so that short CTAs
    // make the grid's tail
    const XSlowest blk = x_slowest_block();
    const int i0 = (gridDim.x - 1 - blk.x) * QT, g = blk.y, b = blk.z;
    const int S = D.S, K = D.topk;
    unsigned char *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    unsigned char *Qs = base, *DOs = base + kRowTile;
    unsigned char *Ks = base + 2 * kRowTile;
    unsigned char *Vs = Ks + kBqStages * kKvTile;
    const int nchunks = (D.L + S - 1) / S, nwords = (nchunks + 31) / 32;

    if (warp == 1) {
        tmem_alloc(&s_tmem, 512);  // buffers b = 0,1: S [128b, 128b+64), dP [128b+64, 128b+128); dQ [256, 384)
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bar.q_full, 1);
        for (int s = 0; s < kBqStages; ++s) {
            mbar_init(&bar.k_full[s], 1);
            mbar_init(&bar.k_empty[s], 1);
            mbar_init(&bar.v_full[s], 1);
            mbar_init(&bar.v_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar.s_full[s], 1);
            mbar_init(&bar.ds_full[s], 128);
            mbar_init(&bar.buf_free[s], 1);
        }
        mbar_init(&bar.dq_final, 1);
        fence_mbar_init();
    }
    for (int w = tid; w < nwords; w += blockDim.x) bitmap[w] = 0;
    for (int e = tid; e < QT * K; e += blockDim.x) {
        const int qi = e / K, t = e % K, i = i0 + qi;
        lc[qi][t] = (i < D.T) ? ws_idx[(((size_t)b * D.Hkv + g) * D.T + i) * K + t] : -1;
    }
    for (int e = tid; e < 128 * K; e += blockDim.x) {
        const int r = e / K, t = e % K, i = i0 + r / G;
        lsh[r][t] = (i < D.T) ? ws_shat[(((size_t)b * D.Hq + g * G + r % G) * D.T + i) * K + t] * kLog2e : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    for (int e = tid; e < QT * K; e += blockDim.x) {
        const int c = lc[e / K][e % K];
        if (c >= 0) atomicOr(&bitmap[c >> 5], 1u << (c & 31));
    }
    if (tid == 0) {
        const int ilast = min(D.T, i0 + QT) - 1;
        const int c_lo = window_left(D.q_pos0 + i0, D.W, S) / S, c_hi = (D.q_pos0 + ilast) / S;
        for (int c = c_lo; c <= c_hi; ++c) atomicOr(&bitmap[c >> 5], 1u << (c & 31));
    }
    __syncthreads();
    if (tid == 0) {
        int n = 0;
        for (int w = nwords - 1; w >= 0 && n < kListCap; --w) {
            uint32_t bits = bitmap[w];
            while (bits && n < kListCap) {
                const int hi = 31 - __clz(bits);
                list[n++] = 32 * w + hi;
                bits &= ~(1u << hi);
            }
        }
        s_ntiles = n;
    }
    __syncthreads();
    const int ntiles = s_ntiles;
    bool ok = true;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            const int head0 = b * D.Hq + g * G;
            mbar_arrive_expect_tx(&bar.q_full, 2 * kRowTile);
            tma_load_3d(Qs, &qmap, 0, head0, i0, &bar.q_full);
            tma_load_3d(Qs + kHalf, &qmap, 64, head0, i0, &bar.q_full);
            tma_load_3d(DOs, &domap, 0, head0, i0, &bar.q_full);
            tma_load_3d(DOs + kHalf, &domap, 64, head0, i0, &bar.q_full);
            const int kvrow0 = (b * D.Hkv + g) * D.L;
            for (int n = 0; n < ntiles; ++n) {
                const int st = n % kBqStages;
                const uint32_t ph = ((n / kBqStages) - 1) & 1;
                const int y = kvrow0 + list[n] * S;
                if (n >= kBqStages && !mbar_wait_bounded(&bar.k_empty[st], ph)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&bar.k_full[st], kKvTile);
                tma_load_2d(Ks + st * kKvTile, &kmap, 0, y, &bar.k_full[st]);
                tma_load_2d(Ks + st * kKvTile + 8192, &kmap, 64, y, &bar.k_full[st]);
                if (n >= kBqStages && !mbar_wait_bounded(&bar.v_empty[st], ph)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&bar.v_full[st], kKvTile);
                tma_load_2d(Vs + st * kKvTile, &vmap, 0, y, &bar.v_full[st]);
                tma_load_2d(Vs + st * kKvTile + 8192, &vmap, 64, y, &bar.v_full[st]);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);
            const uint32_t idesc_dq = idesc_bf16_f32(128, 128, 0, 1);
            const uint32_t qa = smem_u32(Qs), da = smem_u32(DOs);
            ok = mbar_wait_bounded(&bar.q_full, 0);
            auto issue_dq = [&](int m) -> bool {
                const int bm = m & 1, stm = m % kBqStages;
                if (!mbar_wait_bounded(&bar.ds_full[bm], (m >> 1) & 1)) return false;
                tc_fence_after();
                const uint32_t ka = smem_u32(Ks + stm * kKvTile);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16_tmem_a(tmem + 256, tmem + bm * 128 + ks * 8, sdesc_sw128(ka + ks * 2048, 8192, 1024),
                                     idesc_dq, (m > 0 || ks > 0) ? 1u : 0u);
                umma_commit(&bar.buf_free[bm]);
                umma_commit(&bar.k_empty[stm]);
                return true;
            };
            for (int n = 0; n < ntiles && ok; ++n) {
                const int st = n % kBqStages, bb = n & 1;
                const uint32_t ph = (n / kBqStages) & 1;
                if (!mbar_wait_bounded(&bar.k_full[st], ph) || !mbar_wait_bounded(&bar.v_full[st], ph)) {
                    ok = false;
                    break;
                }
                // buffer bb held tile n-2: its ds has been consumed once that tile's dQ product completed
                if (n >= 2 && !mbar_wait_bounded(&bar.buf_free[bb], ((n - 2) >> 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t ka = smem_u32(Ks + st * kKvTile), va = smem_u32(Vs + st * kKvTile);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (ks >> 2) * 8192 + (ks & 3) * 32;
                    const uint32_t qoff = (ks >> 2) * kHalf + (ks & 3) * 32;
                    umma_bf16(tmem + bb * 128, sdesc_sw128(qa + qoff, 16, 1024), sdesc_sw128(ka + off, 16, 1024),
                              idesc_s, ks > 0 ? 1u : 0u);
                    umma_bf16(tmem + bb * 128 + 64, sdesc_sw128(da + qoff, 16, 1024), sdesc_sw128(va + off, 16, 1024),
                              idesc_s, ks > 0 ? 1u : 0u);
                }
                umma_commit(&bar.s_full[bb]);
                umma_commit(&bar.v_empty[st]);
                if (n >= 1 && !issue_dq(n - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok && ntiles > 0 && !issue_dq(ntiles - 1)) ok = false;
            umma_commit(&bar.dq_final);  // arrives once every MMA above has completed (also on error paths)
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- row warps
        const int grp = (warp - 2) >> 2;
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;
        const int qi = r / G, hh = r % G;
        const int i = i0 + qi;
        const bool valid = i < D.T;
        const int pos = D.q_pos0 + i;
        const int lpos = valid ? window_left(pos, D.W, S) : 0;
        const size_t row = ((size_t)b * D.Hq + g * G + hh) * D.T + (valid ? i : 0);
        const float lse2 = valid ? lse[row] * kLog2e : 0.f;
        const float Dr = valid ? Dbuf[row] : 0.f;
        const float sc2 = D.tau * kLog2e;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
        int u = -1;
        if (valid)
            for (int t = 0; t < K; ++t)
                if (lc[qi][t] >= 0) u = t;
        __nv_bfloat16 *dS_row = dS + row * ncp;
        float *beta_row = betas + row * ncp;
        for (int n = grp; n < ntiles; n += 2) {
            const int bb = n & 1;
            const int c = list[n];
            const int j0 = c * S;
            while (u >= 0 && lc[qi][u] > c) --u;
            const bool sel = valid && u >= 0 && lc[qi][u] == c;
            int lo = 0, hi = S - 1;
            if (valid && !sel) {
                lo = max(lpos - j0, 0);
                hi = min(pos - j0, S - 1);
            }
            const bool win = valid && !sel && lo <= hi;
            const int kind = sel ? 1 : (win ? 2 : 0);
            const float sh2 = sel ? lsh[r][u] : 0.f;
            if (__any_sync(0xffffffffu, !mbar_wait_bounded(&bar.s_full[bb], (n >> 1) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t pk[32];
            if (__any_sync(0xffffffffu, kind != 0)) {
                float s[64], dp[64];
                tmem_ld32(lane_base + bb * 128, *reinterpret_cast<float(*)[32]>(&s[0]));
                tmem_ld32(lane_base + bb * 128 + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
                tmem_wait_ld();
                // dP is loaded during the exponentials of S
                tmem_ld32(lane_base + bb * 128 + 64, *reinterpret_cast<float(*)[32]>(&dp[0]));
                tmem_ld32(lane_base + bb * 128 + 96, *reinterpret_cast<float(*)[32]>(&dp[32]));
                const bool mask = __any_sync(0xffffffffu, kind == 2 && (lo > 0 || hi < S - 1));
                const float z = row_grad_a(s, kind, lo, hi, sc2, lse2, mask);
                tmem_wait_ld();
                const float beta = kind == 1 ? ex2_approx(sh2 - lse2) : 0.f;
                const float dshat = row_grad_b(s, dp, kind, z, beta, Dr);
                if (kind == 1) {
                    dS_row[c] = __float2bfloat16_rn(dshat);
                    beta_row[c] = beta;  // for the KV-major kernel
                }
#pragma unroll
                for (int e = 0; e < 32; ++e) pk[e] = pack_bf16(dp[2 * e], dp[2 * e + 1]);
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) pk[e] = 0u;
            }
            // ds over S in TMEM (S and dP have been read); the dQ product reads it from there
            tmem_st32u(lane_base + bb * 128, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bar.ds_full[bb]);
        }
        // epilogue: group grp writes dQ columns [64 grp, 64 grp + 64)
        if (__any_sync(0xffffffffu, !mbar_wait_bounded(&bar.dq_final, 0))) ok = false;
        tc_fence_after();
#pragma unroll 1
        for (int t = 0; t < 2; ++t) {
            float o[32];
            tmem_ld32(lane_base + 256 + 64 * grp + 32 * t, o);
            tmem_wait_ld();
            if (valid) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint4 w4;
                    w4.x = pack_bf16(o[8 * k] * D.tau, o[8 * k + 1] * D.tau);
                    w4.y = pack_bf16(o[8 * k + 2] * D.tau, o[8 * k + 3] * D.tau);
                    w4.z = pack_bf16(o[8 * k + 4] * D.tau, o[8 * k + 5] * D.tau);
                    w4.w = pack_bf16(o[8 * k + 6] * D.tau, o[8 * k + 7] * D.tau);
                    *reinterpret_cast<uint4 *>(dq + row * 128 + 64 * grp + 32 * t + 8 * k) = w4;
                }
            }
        }
    }
    if (!ok) atomicOr(&g_bwd_tc_errors, 1u);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------------------------------ dqhat

// dq^_r = tau sum_t ds^_{r, c_t} k'_{h, c_t}. CTA = (256 queries, head h, b); the head's summaries
// (Nc <= 128 rows) in shared memory; warp per query, lane owns 4 columns.
__global__ void __launch_bounds__(256)
bwd_dqhat_kernel(Dims D, const int *__restrict__ ws_idx, const __nv_bfloat16 *__restrict__ dS, int ncp,
                 const __nv_bfloat16 *__restrict__ k_sum, __nv_bfloat16 *__restrict__ dq_hat) {
    __shared__ __align__(16) __nv_bfloat16 ks[128 * 128];
    const int h = blockIdx.y, b = blockIdx.z, g = h / D.G, K = D.topk;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t bh = (size_t)b * D.Hq + h;
    for (int e = threadIdx.x; e < D.Nc * 16; e += blockDim.x)
        reinterpret_cast<uint4 *>(ks)[e] = reinterpret_cast<const uint4 *>(k_sum + bh * D.Nc * 128)[e];
    __syncthreads();
    for (int qi = warp; qi < 256; qi += 8) {
        const int i = blockIdx.x * 256 + qi;
        if (i >= D.T) break;
        const int *irow = ws_idx + (((size_t)b * D.Hkv + g) * D.T + i) * K;
        const __nv_bfloat16 *drow = dS + (bh * D.T + i) * ncp;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
        // lane t < K fetches slot t's id and its ds^ at once (one round trip each for the whole row),
        // then the warp walks the slots with the values broadcast from their lanes
        const int cl = lane < K ? irow[lane] : -1;
        const float wl = cl >= 0 ? __bfloat162float(drow[cl]) : 0.f;
        for (int t = 0; t < K; ++t) {
            const int c = __shfl_sync(0xffffffffu, cl, t);
            if (c < 0) break;
            const float w = __shfl_sync(0xffffffffu, wl, t);
            const uint2 raw = *reinterpret_cast<const uint2 *>(ks + c * 128 + 4 * lane);
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
            const float2 bq = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
            acc[0] = fmaf(w, a.x, acc[0]);
            acc[1] = fmaf(w, a.y, acc[1]);
            acc[2] = fmaf(w, bq.x, acc[2]);
            acc[3] = fmaf(w, bq.y, acc[3]);
        }
        uint2 o;
        o.x = pack_bf16(acc[0] * D.tau, acc[1] * D.tau);
        o.y = pack_bf16(acc[2] * D.tau, acc[3] * D.tau);
        *reinterpret_cast<uint2 *>(dq_hat + (bh * D.T + i) * 128 + 4 * lane) = o;
    }
}

// ------------------------------------------------------------------------------------------ dksum

// Partial sums over one of kDkSplit row ranges of dk'[c][t] = sum_i ds^[i][c] q^[i][t] and db'[c] =
// sum_i ds^[i][c] for 64 chunks x 128 columns of one (b, h): four warps, 16 chunks each, mma.sync with
// the dense ds^ matrix read transposed (A) and q^ read transposed (B); db' comes from a product with a
// column of ones. ds^ rows have stride ncp (columns Nc..ncp-1 are zero). Partials:
// part[((bh * kDkSplit + split) * Nc + c) * 129 + (t, or 128 for db')].
__global__ void __launch_bounds__(128)
bwd_dksum_kernel(Dims D, const __nv_bfloat16 *__restrict__ dS, int ncp, const __nv_bfloat16 *__restrict__ q_hat,
                 float *__restrict__ part) {
    constexpr int kDsStride = 72, kQStride = 136;  // padded rows (bf16 elements): conflict-free ldmatrix
    __shared__ __align__(16) __nv_bfloat16 ds_t[64 * kDsStride];
    __shared__ __align__(16) __nv_bfloat16 qh_t[64 * kQStride];
    const int cb = blockIdx.x, split = blockIdx.y, bh = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g8 = lane >> 2, t4 = lane & 3, mi = lane >> 3, r8 = lane & 7;
    const int Nc = D.Nc, T = D.T;
    const int rows_per = (T + kDkSplit - 1) / kDkSplit;
    const int rb = split * rows_per, re = min(T, rb + rows_per);
    const __nv_bfloat16 *dsb = dS + (size_t)bh * T * ncp;
    const __nv_bfloat16 *qhb = q_hat + (size_t)bh * T * 128;
    float acc[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
    float ones[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t kOnes = 0x3F803F80u;  // two bf16 1.0
    for (int i0 = rb; i0 < re; i0 += 64) {
        __syncthreads();
        for (int e = tid; e < 64 * 8; e += 128) {  // ds^ rows: 64 chunks = 8 x 16 bytes
            const int rr = e >> 3, ch = e & 7, i = i0 + rr, c = cb * 64 + ch * 8;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (i < re && c < ncp) v = *reinterpret_cast<const uint4 *>(dsb + (size_t)i * ncp + c);
            *reinterpret_cast<uint4 *>(ds_t + rr * kDsStride + ch * 8) = v;
        }
        for (int e = tid; e < 64 * 16; e += 128) {  // q^ rows: 128 columns = 16 x 16 bytes
            const int rr = e >> 4, ch = e & 15, i = i0 + rr;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (i < re) v = *reinterpret_cast<const uint4 *>(qhb + (size_t)i * 128 + ch * 8);
            *reinterpret_cast<uint4 *>(qh_t + rr * kQStride + ch * 8) = v;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t a[4];
            {
                const int rr = kk * 16 + r8 + (mi >> 1) * 8, cc = 16 * warp + (mi & 1) * 8;
                ldsm_x4_trans(smem_u32(ds_t + rr * kDsStride + cc), a);
            }
            mma_16816(ones, a, kOnes, kOnes);
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                uint32_t bb[4];
                const int rr = kk * 16 + r8 + (mi & 1) * 8, cc = 16 * nt + (mi >> 1) * 8;
                ldsm_x4_trans(smem_u32(qh_t + rr * kQStride + cc), bb);
                mma_16816(acc[2 * nt], a, bb[0], bb[1]);
                mma_16816(acc[2 * nt + 1], a, bb[2], bb[3]);
            }
        }
    }
    const int c0 = cb * 64 + 16 * warp + g8;
    float *pb = part + ((size_t)bh * kDkSplit + split) * Nc * kPartStride;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        const int t = 8 * n + 2 * t4;
        if (c0 < Nc) {
            pb[(size_t)c0 * kPartStride + t] = acc[n][0];
            pb[(size_t)c0 * kPartStride + t + 1] = acc[n][1];
        }
        if (c0 + 8 < Nc) {
            pb[(size_t)(c0 + 8) * kPartStride + t] = acc[n][2];
            pb[(size_t)(c0 + 8) * kPartStride + t + 1] = acc[n][3];
        }
    }
    if (t4 == 0) {
        if (c0 < Nc) pb[(size_t)c0 * kPartStride + 128] = ones[0];
        if (c0 + 8 < Nc) pb[(size_t)(c0 + 8) * kPartStride + 128] = ones[2];
    }
}

// ------------------------------------------------------------------------------------------ eq8

// Eq. 8 backward for one (b, KV group, chunk c): per head, u_j = tau q'.k_j, p = softmax(u),
// k' = sum p_j k_j, b' = -sum p log p; with dk' (tau folded) and db' summed from the partials:
//   du_j = p_j (dk'.(k_j - k') - db' (log p_j + b')), dq' = tau sum_j du_j k_j,
//   dk_extra_j = sum_h p_hj dk'_h + tau du_hj q'_h   (fp32, added to dk by bkv).
__global__ void __launch_bounds__(256)
bwd_eq8_kernel(Dims D, const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ q_land,
               const float *__restrict__ part, __nv_bfloat16 *__restrict__ dq_land, float *__restrict__ dk_extra) {
    __shared__ float Kf[64][129];
    __shared__ float ql[4][128], dks[4][128];
    __shared__ float uu[4][64], pp[4][64], du[4][64];
    __shared__ float db[4];
    const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int G = D.G, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t bg = (size_t)b * D.Hkv + g;
    const __nv_bfloat16 *kc = k + (bg * D.L + (size_t)c * 64) * 128;
    for (int e = tid; e < 64 * 16; e += blockDim.x) {
        float f[8];
        load8(kc + e * 8, f);
        const int j = e >> 4, t = (e & 15) * 8;
#pragma unroll
        for (int x = 0; x < 8; ++x) Kf[j][t + x] = f[x];
    }
    for (int e = tid; e < G * 128; e += blockDim.x) {
        const int hh = e >> 7, t = e & 127;
        const size_t bh = (size_t)b * D.Hq + g * G + hh;
        ql[hh][t] = __bfloat162float(q_land[(bh * D.Nc + c) * 128 + t]);
        float s = 0.f;
        for (int sp = 0; sp < kDkSplit; ++sp) s += part[((bh * kDkSplit + sp) * D.Nc + c) * kPartStride + t];
        dks[hh][t] = s * D.tau;
        if (t == 0) {
            float s2 = 0.f;
            for (int sp = 0; sp < kDkSplit; ++sp) s2 += part[((bh * kDkSplit + sp) * D.Nc + c) * kPartStride + 128];
            db[hh] = s2;
        }
    }
    __syncthreads();
    if (warp < G) {
        const int hh = warp;
        float mx = -INFINITY;
        for (int j = lane; j < 64; j += 32) {
            float s = 0.f;
            for (int t = 0; t < 128; ++t) s = fmaf(ql[hh][t], Kf[j][t], s);
            s *= D.tau;
            uu[hh][j] = s;
            mx = fmaxf(mx, s);
        }
        mx = warp_max(mx);
        float z = 0.f;
        for (int j = lane; j < 64; j += 32) z += __expf(uu[hh][j] - mx);
        z = warp_sum(z);
        const float lu = mx + logf(z);
        float ent = 0.f;
        for (int j = lane; j < 64; j += 32) {
            const float lp = uu[hh][j] - lu;
            const float pj = __expf(lp);
            pp[hh][j] = pj;
            ent -= pj * lp;
        }
        ent = warp_sum(ent);
        __syncwarp();
        float kk = 0.f;
        for (int t = lane; t < 128; t += 32) {
            float a = 0.f;
            for (int j = 0; j < 64; ++j) a = fmaf(pp[hh][j], Kf[j][t], a);  // k'_t in fp32
            kk = fmaf(dks[hh][t], a, kk);
        }
        kk = warp_sum(kk);
        for (int j = lane; j < 64; j += 32) {
            float a = 0.f;
            for (int t = 0; t < 128; ++t) a = fmaf(dks[hh][t], Kf[j][t], a);
            du[hh][j] = pp[hh][j] * (a - kk - db[hh] * ((uu[hh][j] - lu) + ent));
        }
        __syncwarp();
        const size_t bh = (size_t)b * D.Hq + g * G + hh;
        for (int t = lane; t < 128; t += 32) {
            float a = 0.f;
            for (int j = 0; j < 64; ++j) a = fmaf(du[hh][j], Kf[j][t], a);
            dq_land[(bh * D.Nc + c) * 128 + t] = __float2bfloat16_rn(D.tau * a);
        }
    }
    __syncthreads();
    float *dx = dk_extra + (bg * D.L + (size_t)c * 64) * 128;
    for (int e = tid; e < 64 * 128; e += blockDim.x) {
        const int j = e >> 7, t = e & 127;
        float a = 0.f;
        for (int hh = 0; hh < G; ++hh) a = fmaf(pp[hh][j], dks[hh][t], fmaf(D.tau * du[hh][j], ql[hh][t], a));
        dx[e] = a;
    }
}

// ------------------------------------------------------------------------------------------ bkv

struct KvBars {
    uint64_t kv_full, qd_full[2], qd_empty[2], s_full[2], pds_full, pds_free, kv_final;
};

__global__ void __launch_bounds__(kTcThreads, 1)
bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap domap,
                   const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap, Dims D,
                   const float *__restrict__ betas, int ncp, const float *__restrict__ lse,
                   const float *__restrict__ Dbuf, const float *__restrict__ dk_extra, __nv_bfloat16 *__restrict__ dk,
                   __nv_bfloat16 *__restrict__ dv) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) KvBars bar;
    __shared__ uint32_t s_tmem;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = D.G, QT = 128 / G;
    // chunks in launch order within each (b, group): the concurrently running CTAs share that group's
    // query and dO tiles in L2 (chunk-major order across the groups measured slower)
    const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int S = D.S;
    unsigned char *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    unsigned char *Kc = base, *Vc = base + kKvTile;
    unsigned char *QD = base + 2 * kKvTile;       // 2 stages x (Q tile, dO tile)
    unsigned char *Ps = QD + 4 * kRowTile;        // P  [128 rows x 64 tokens] bf16, MN-major, 128-byte swizzle
    unsigned char *DSs = Ps + kKvTile;            // ds, same layout
    const int j0 = c * S, jn = min(S, D.L - j0);
    const int nqt = (D.T + QT - 1) / QT;
    const int qt0 = min(nqt, j0 / QT);  // earlier tiles hold only queries before the chunk
    const int nq = nqt - qt0;
    const size_t bg = (size_t)b * D.Hkv + g;

    if (warp == 1) {
        tmem_alloc(&s_tmem, 512);  // S/dP buffers as in bq; dK^T [256, 320), dV^T [320, 384)
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bar.kv_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar.qd_full[s], 1);
            mbar_init(&bar.qd_empty[s], 1);
            mbar_init(&bar.s_full[s], 1);
        }
        mbar_init(&bar.pds_full, 128);
        mbar_init(&bar.pds_free, 1);
        mbar_init(&bar.kv_final, 1);
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;
    bool ok = true;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            const int y = (int)(bg * D.L) + j0;
            mbar_arrive_expect_tx(&bar.kv_full, 2 * kKvTile);
            tma_load_2d(Kc, &kmap, 0, y, &bar.kv_full);
            tma_load_2d(Kc + 8192, &kmap, 64, y, &bar.kv_full);
            tma_load_2d(Vc, &vmap, 0, y, &bar.kv_full);
            tma_load_2d(Vc + 8192, &vmap, 64, y, &bar.kv_full);
            const int head0 = b * D.Hq + g * G;
            for (int m = 0; m < nq; ++m) {
                const int st = m & 1;
                if (m >= 2 && !mbar_wait_bounded(&bar.qd_empty[st], ((m >> 1) - 1) & 1)) {
                    ok = false;
                    break;
                }
                unsigned char *Qt = QD + st * 2 * kRowTile;
                const int i0 = (qt0 + m) * QT;
                mbar_arrive_expect_tx(&bar.qd_full[st], 2 * kRowTile);
                tma_load_3d(Qt, &qmap, 0, head0, i0, &bar.qd_full[st]);
                tma_load_3d(Qt + kHalf, &qmap, 64, head0, i0, &bar.qd_full[st]);
                tma_load_3d(Qt + kRowTile, &domap, 0, head0, i0, &bar.qd_full[st]);
                tma_load_3d(Qt + kRowTile + kHalf, &domap, 64, head0, i0, &bar.qd_full[st]);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);
            const uint32_t idesc_t = idesc_bf16_f32(128, 64, 1, 1);  // A and B both read transposed
            const uint32_t ka = smem_u32(Kc), va = smem_u32(Vc), pa = smem_u32(Ps), sa = smem_u32(DSs);
            ok = mbar_wait_bounded(&bar.kv_full, 0);
            auto issue_kv = [&](int p) -> bool {
                if (!mbar_wait_bounded(&bar.pds_full, p & 1)) return false;
                tc_fence_after();
                const uint32_t qa = smem_u32(QD + (p & 1) * 2 * kRowTile), da = qa + kRowTile;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {  // K = the 128 rows of the query tile, 16 per step
                    const uint32_t acc = (p > 0 || ks > 0) ? 1u : 0u;
                    umma_bf16(tmem + 320, sdesc_sw128(da + ks * 2048, kHalf, 1024), sdesc_sw128(pa + ks * 2048, 8192, 1024),
                              idesc_t, acc);
                    umma_bf16(tmem + 256, sdesc_sw128(qa + ks * 2048, kHalf, 1024), sdesc_sw128(sa + ks * 2048, 8192, 1024),
                              idesc_t, acc);
                }
                umma_commit(&bar.pds_free);
                umma_commit(&bar.qd_empty[p & 1]);
                return true;
            };
            for (int m = 0; m < nq && ok; ++m) {
                const int st = m & 1;
                if (!mbar_wait_bounded(&bar.qd_full[st], (m >> 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t qa = smem_u32(QD + st * 2 * kRowTile), da = qa + kRowTile;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (ks >> 2) * 8192 + (ks & 3) * 32;
                    const uint32_t qoff = (ks >> 2) * kHalf + (ks & 3) * 32;
                    umma_bf16(tmem + st * 128, sdesc_sw128(qa + qoff, 16, 1024), sdesc_sw128(ka + off, 16, 1024),
                              idesc_s, ks > 0 ? 1u : 0u);
                    umma_bf16(tmem + st * 128 + 64, sdesc_sw128(da + qoff, 16, 1024), sdesc_sw128(va + off, 16, 1024),
                              idesc_s, ks > 0 ? 1u : 0u);
                }
                umma_commit(&bar.s_full[st]);
                if (m >= 1 && !issue_kv(m - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok && nq > 0 && !issue_kv(nq - 1)) ok = false;
            umma_commit(&bar.kv_final);
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- row warps
        const int grp = (warp - 2) >> 2;
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;
        const int qi = r / G, hh = r % G;
        const float sc2 = D.tau * kLog2e;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
        // (beta of this chunk, lse in log2 units, D) of the row in query tile m: three independent loads,
        // fetched one iteration ahead (beta = 0 where the row did not select the chunk)
        auto fetch = [&](int m, float &beta, float &lse2, float &Dr) {
            const int i = (qt0 + m) * QT + qi;
            beta = 0.f;
            lse2 = 0.f;
            Dr = 0.f;
            if (m < nq && i < D.T) {
                const size_t row = ((size_t)b * D.Hq + g * G + hh) * D.T + i;
                if (c < D.Nc) beta = betas[row * ncp + c];
                lse2 = lse[row] * kLog2e;
                Dr = Dbuf[row];
            }
        };
        float nbeta, nlse2, nDr;
        fetch(grp, nbeta, nlse2, nDr);
        for (int m = grp; m < nq; m += 2) {
            const int bb = m & 1;
            const float beta = nbeta, lse2 = nlse2, Dr = nDr;
            fetch(m + 2, nbeta, nlse2, nDr);
            const int i = (qt0 + m) * QT + qi;
            const bool valid = i < D.T;
            const int pos = D.q_pos0 + i;
            const int lpos = valid ? window_left(pos, D.W, S) : 0;
            const bool sel = valid && beta > 0.f;
            int lo = 0, hi = S - 1;
            if (valid && !sel) {
                lo = max(lpos - j0, 0);
                hi = min(pos - j0, S - 1);
            }
            const bool win = valid && !sel && lo <= hi;
            const int kind = sel ? 1 : (win ? 2 : 0);
            if (__any_sync(0xffffffffu, !mbar_wait_bounded(&bar.s_full[bb], (m >> 1) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint4 pw[8], dw[8];
            if (__any_sync(0xffffffffu, kind != 0)) {
                float s[64], dp[64];
                tmem_ld32(lane_base + bb * 128, *reinterpret_cast<float(*)[32]>(&s[0]));
                tmem_ld32(lane_base + bb * 128 + 32, *reinterpret_cast<float(*)[32]>(&s[32]));
                tmem_wait_ld();
                // dP is loaded during the exponentials of S
                tmem_ld32(lane_base + bb * 128 + 64, *reinterpret_cast<float(*)[32]>(&dp[0]));
                tmem_ld32(lane_base + bb * 128 + 96, *reinterpret_cast<float(*)[32]>(&dp[32]));
                const bool mask = __any_sync(0xffffffffu, kind == 2 && (lo > 0 || hi < S - 1));
                const float z = row_grad_a(s, kind, lo, hi, sc2, lse2, mask);
                tmem_wait_ld();
                row_grad_b(s, dp, kind, z, beta, Dr);
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    pw[x] = make_uint4(pack_bf16(s[8 * x], s[8 * x + 1]), pack_bf16(s[8 * x + 2], s[8 * x + 3]),
                                       pack_bf16(s[8 * x + 4], s[8 * x + 5]), pack_bf16(s[8 * x + 6], s[8 * x + 7]));
                    dw[x] = make_uint4(pack_bf16(dp[8 * x], dp[8 * x + 1]), pack_bf16(dp[8 * x + 2], dp[8 * x + 3]),
                                       pack_bf16(dp[8 * x + 4], dp[8 * x + 5]), pack_bf16(dp[8 * x + 6], dp[8 * x + 7]));
                }
            } else {
#pragma unroll
                for (int x = 0; x < 8; ++x) pw[x] = dw[x] = make_uint4(0u, 0u, 0u, 0u);
            }
            // this group's S/dP buffer has been read; the shared P/ds tiles are free once the previous
            // query tile's products have completed
            tc_fence_before();
            if (m >= 1 && __any_sync(0xffffffffu, !mbar_wait_bounded(&bar.pds_free, (m - 1) & 1))) {
                ok = false;
                break;
            }
#pragma unroll
            for (int x = 0; x < 8; ++x) {
                const uint32_t off = (uint32_t)r * 128 + (((uint32_t)x ^ (uint32_t)(r & 7)) << 4);
                *reinterpret_cast<uint4 *>(Ps + off) = pw[x];
                *reinterpret_cast<uint4 *>(DSs + off) = dw[x];
            }
            fence_async_smem();
            mbar_arrive(&bar.pds_full);
        }
        // epilogue: group 0 writes dV, group 1 dK (TMEM lanes = columns t of the head dim, cols = tokens)
        if (__any_sync(0xffffffffu, !mbar_wait_bounded(&bar.kv_final, 0))) ok = false;
        tc_fence_after();
        const int t = 32 * q4 + lane;
        const bool is_k = grp == 1;
        const bool extra = is_k && c < D.Nc;
#pragma unroll 1
        for (int h2 = 0; h2 < 2; ++h2) {
            float o[32];
            tmem_ld32(lane_base + (is_k ? 256 : 320) + 32 * h2, o);
            tmem_wait_ld();
#pragma unroll 4
            for (int e = 0; e < 32; ++e) {
                const int j = 32 * h2 + e;
                if (j < jn) {
                    const size_t at = (bg * D.L + j0 + j) * 128 + t;
                    if (is_k) {
                        const float v = o[e] * D.tau + (extra ? dk_extra[at] : 0.f);
                        dk[at] = __float2bfloat16_rn(v);
                    } else {
                        dv[at] = __float2bfloat16_rn(o[e]);
                    }
                }
            }
        }
    }
    if (!ok) atomicOr(&g_bwd_tc_errors, 1u);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// Row stride (elements) of the dense ds^ matrix: Nc rounded up to 8, so rows start 16-byte aligned.
int ds_stride(const Dims &D) { return (std::max(D.Nc, 1) + 7) & ~7; }

struct BwdLayout {
    size_t idx, shat, dbuf, ds, beta, part, dkx, total;
};

BwdLayout bwd_layout(const Dims &D) {
    BwdLayout L{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t at = off;
        off += (bytes + 255) & ~(size_t)255;
        return at;
    };
    L.idx = take((size_t)D.B * D.Hkv * D.T * D.topk * sizeof(int));
    L.shat = take((size_t)D.B * D.Hq * D.T * D.topk * sizeof(float));
    L.dbuf = take((size_t)D.B * D.Hq * D.T * sizeof(float));
    L.ds = take((size_t)D.B * D.Hq * D.T * ds_stride(D) * sizeof(__nv_bfloat16));
    L.beta = take((size_t)D.B * D.Hq * D.T * ds_stride(D) * sizeof(float));
    L.part = take((size_t)D.B * D.Hq * kDkSplit * std::max(D.Nc, 1) * kPartStride * sizeof(float));
    L.dkx = take((size_t)D.B * D.Hkv * D.L * 128 * sizeof(float));
    L.total = off;
    return L;
}

}  // namespace

bool attn_bwd_tc_supported(const Dims &D, int dtype) {
    // the forward's tensor-core conditions (bf16, d 128, S 64, G <= 4, topk <= 32, <= 128 chunks, tile
    // list bounds) plus a self-attention prefill
    return attn_fwd_tc_supported(D, dtype) && D.q_pos0 == 0 && D.T == D.L && D.Nc <= 128 && D.topk <= kMaxK;
}

size_t attn_bwd_tc_workspace(const Dims &D) { return bwd_layout(D).total; }

unsigned int attn_bwd_tc_error_flags(bool clear) {
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_bwd_tc_errors, sizeof(v));
    if (clear && v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_bwd_tc_errors, &zero, sizeof(zero));
    }
    return v;
}

cudaError_t launch_attn_bwd_tc(const Dims &D, const void *q, const void *k, const void *v, const void *q_hat,
                               const void *q_land, const void *k_sum, const float *b_sum, const int *idx,
                               const void *out, const float *lse, const void *dout, void *dq, void *dk, void *dv,
                               void *dq_hat, void *dq_land, void *ws, cudaStream_t stream) {
    const BwdLayout L = bwd_layout(D);
    unsigned char *w = (unsigned char *)ws;
    int *ws_idx = (int *)(w + L.idx);
    float *ws_shat = (float *)(w + L.shat);
    float *Dbuf = (float *)(w + L.dbuf);
    __nv_bfloat16 *dS = (__nv_bfloat16 *)(w + L.ds);
    float *betas = (float *)(w + L.beta);
    float *part = (float *)(w + L.part);
    float *dkx = (float *)(w + L.dkx);
    cudaError_t e = launch_gather_shat_tc(D, q_hat, k_sum, b_sum, idx, ws_idx, ws_shat, stream);
    if (e != cudaSuccess) return e;
    const long long rows = (long long)D.B * D.Hq * D.T;
    bwd_delta_kernel<<<(unsigned)((rows * 16 + 255) / 256), 256, 0, stream>>>(
        (const __nv_bfloat16 *)out, (const __nv_bfloat16 *)dout, Dbuf, rows);
    const int ncp = ds_stride(D);
    e = cudaMemsetAsync(dS, 0, (size_t)rows * ncp * sizeof(__nv_bfloat16), stream);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(betas, 0, (size_t)rows * ncp * sizeof(float), stream);
    if (e != cudaSuccess) return e;
    const int QT = 128 / D.G;
    CUtensorMap qmap, domap, kmap, vmap;
    if (!make_tmap_bf16_3d(&qmap, q, 128, (uint64_t)D.B * D.Hq, (uint64_t)D.T, (uint64_t)D.T * 256, 256, D.G, QT) ||
        !make_tmap_bf16_3d(&domap, dout, 128, (uint64_t)D.B * D.Hq, (uint64_t)D.T, (uint64_t)D.T * 256, 256, D.G,
                           QT) ||
        !make_tmap_bf16_2d(&kmap, k, (uint64_t)D.B * D.Hkv * D.L, 128, 128, 64) ||
        !make_tmap_bf16_2d(&vmap, v, (uint64_t)D.B * D.Hkv * D.L, 128, 128, 64))
        return cudaErrorInvalidValue;
    {
        const size_t smem = 1024 + 2 * kRowTile + 2 * kBqStages * kKvTile;
        cudaFuncSetAttribute(bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        bwd_dq_tc_kernel<<<dim3((D.T + QT - 1) / QT, D.Hkv, D.B), kTcThreads, smem, stream>>>(
            qmap, domap, kmap, vmap, D, ws_idx, ws_shat, lse, Dbuf, dS, betas, ncp, (__nv_bfloat16 *)dq);
    }
    if (D.Nc > 0) {
        bwd_dqhat_kernel<<<dim3((D.T + 255) / 256, D.Hq, D.B), 256, 0, stream>>>(
            D, ws_idx, dS, ncp, (const __nv_bfloat16 *)k_sum, (__nv_bfloat16 *)dq_hat);
        bwd_dksum_kernel<<<dim3((D.Nc + 63) / 64, kDkSplit, D.B * D.Hq), 128, 0, stream>>>(
            D, dS, ncp, (const __nv_bfloat16 *)q_hat, part);
        bwd_eq8_kernel<<<dim3(D.Nc, D.Hkv, D.B), 256, 0, stream>>>(D, (const __nv_bfloat16 *)k,
                                                                    (const __nv_bfloat16 *)q_land, part,
                                                                    (__nv_bfloat16 *)dq_land, dkx);
    } else {
        e = cudaMemsetAsync(dq_hat, 0, (size_t)rows * 128 * sizeof(__nv_bfloat16), stream);
        if (e != cudaSuccess) return e;
    }
    {
        const size_t smem = 1024 + 2 * kKvTile + 4 * kRowTile + 2 * kKvTile;
        cudaFuncSetAttribute(bwd_dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        bwd_dkdv_tc_kernel<<<dim3((D.L + D.S - 1) / D.S, D.Hkv, D.B), kTcThreads, smem, stream>>>(
            qmap, domap, kmap, vmap, D, betas, ncp, lse, Dbuf, dkx, (__nv_bfloat16 *)dk, (__nv_bfloat16 *)dv);
    }
    return cudaGetLastError();
}

}  // namespace hils
