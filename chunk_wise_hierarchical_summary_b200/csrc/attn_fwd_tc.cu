// Stages (c)+(d) on the tensor cores: per-chunk attention and Eq. 10 fusion, prefill form, bf16, d 128,
// chunk size 64 ("Hierarchical Sparse Attention Done Right", Sec. 3 RQ2 / Eq. 10; Sec. 4 kernel).
//
// Launches: hils_attn_fwd first runs a gather (select_tc.cu, the selection's tcgen05 GEMM) that writes
// each row's ids in canonical form (valid, distinct, ascending) and their retrieval scores s^ to the
// workspace; hils_attn_fwd_shat is given both by the selection and launches this kernel alone.
//  CTA = 128 rows = 128/G queries x G heads of one KV group (row = query*G + head), so the heads of a
//  group share every K/V tile. The tiles it visits are the union of the queries' window chunks and
//  selected chunks (the paper's query packing over the union, Fig. 4b), in descending chunk order so
//  that window tiles come first.
//    warp 0     TMA producer: Q once (3-D map, rows query-major), then K and V tiles (2-D maps, 128-byte
//               swizzle) into two-stage K and V rings.
//    warp 1     MMA issuer: S = Q K^T (M 128, N 64, K 128) into one of two TMEM S buffers, then
//               O += P V (M 128, N 128, K 64) with P read from TMEM and V MN-major from shared memory;
//               O lives in TMEM throughout.
//    warps 2-5  one row each (the row's TMEM lane): per tile the row is a window row (logits masked to
//               its window), a selecting row (logits s_j - L_c + s^_c with L_c the intra-chunk LSE, so
//               the chunk carries mass exp(s^_c)), or neither (P = 0). P (bf16) overwrites its S buffer
//               in TMEM. The running max starts at max s^ over the row's chunks, which no chunk tile can
//               exceed; only a window logit more than 8 above it rescales the row of O in TMEM.
//  Epilogue: O / l to bf16, lse = m + log l.
#include "internal.h"
#include "tcgen05.cuh"

namespace hils {

bool make_tmap_bf16_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint64_t ld,
                       uint32_t box_rows);
bool make_tmap_bf16_3d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1_bytes,
                       uint64_t s2_bytes, uint32_t b1, uint32_t b2);
cudaError_t launch_gather_shat_tc(const Dims &D, const void *q_hat, const void *k_sum, const float *b_sum,
                                  const int *idx, int *ws_idx, float *ws_shat, cudaStream_t stream);
bool select_tc_supported(const Dims &D, int dtype);

namespace {

constexpr int kThreads = 192;
constexpr int kStages = 2;           // K ring and V ring, each kStages deep
constexpr int kListCap = 1024;
constexpr int kBitmapWords = 256;    // chunks per sequence <= 8192
constexpr uint32_t kQBytes = 32768;
constexpr uint32_t kTileBytes = 16384;  // one K or V tile: 64 tokens x 128 d bf16
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleSlack2 = 11.5f;  // log2 units (about 8 in natural units)

__device__ unsigned int g_attn_tc_errors = 0;

struct Bars {
    // p_full is per S/P buffer: a row warp may run one tile ahead (its next S is ready before every warp
    // has written this tile's P), so one shared barrier would let an early arrival complete a phase.
    // o_final completes once, after the last value product: the row warps' epilogue cannot wait on a
    // pv_done parity, because a warp that skipped per-tile waits may see pv_done several phases behind.
    // With two stages and two S buffers, stage n % 2 and buffer n & 1 coincide: s_full[b] also frees K stage
    // b (the QK product read it) and pv_done[b] frees V stage b, so each MMA group needs one commit.
    uint64_t q_full, k_full[kStages], v_full[kStages], s_full[2], p_full[2], pv_done[2], o_final;
};

__global__ void __launch_bounds__(kThreads, 2)
attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
               const __grid_constant__ CUtensorMap vmap, Dims D, const int *__restrict__ ws_idx,
               const float *__restrict__ ws_shat, __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) Bars bar;
    __shared__ uint32_t s_tmem;
    __shared__ uint32_t bitmap[kBitmapWords];
    __shared__ int list[kListCap];
    __shared__ int s_ntiles;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = D.G, QT = 128 / G;
    // Late query tiles visit the most chunks (every earlier candidate): launch them first so that the
    // grid's tail is made of short CTAs.
    const XSlowest blk = x_slowest_block();  // across all (b, group), not within each
    const int i0 = (gridDim.x - 1 - blk.x) * QT, g = blk.y, b = blk.z;
    const int S = D.S, K = D.topk;
    unsigned char *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    unsigned char *Qs = base;
    unsigned char *Ks = base + kQBytes;                    // kStages K tiles
    unsigned char *Vs = Ks + kStages * kTileBytes;         // kStages V tiles
    const int nchunks = (D.L + S - 1) / S;
    const int nwords = (nchunks + 31) / 32;
    const float scale2 = D.tau * kLog2e;

    if (warp == 1) {
        tmem_alloc(&s_tmem, 256);  // S/P buffers: columns [0,64) and [64,128); O: [128,256)
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bar.q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bar.k_full[s], 1);
            mbar_init(&bar.v_full[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar.s_full[s], 1);
            mbar_init(&bar.p_full[s], 128);
            mbar_init(&bar.pv_done[s], 1);
        }
        mbar_init(&bar.o_final, 1);
        fence_mbar_init();
    }
    for (int w = tid; w < nwords; w += blockDim.x) bitmap[w] = 0;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    // ---- per-row data (softmax warps) and the CTA's tile list
    const bool softmax = warp >= 2;
    const int q4 = warp & 3;
    const int r = 32 * q4 + lane;  // row = TMEM lane
    const int qi = r / G, hh = r % G;
    const int i = i0 + qi;
    const bool valid = softmax && i < D.T;
    const int pos = D.q_pos0 + i;
    const int lpos = valid ? window_left(pos, D.W, S) : 0;
    const int *row_idx = ws_idx + (((size_t)b * D.Hkv + g) * D.T + (valid ? i : 0)) * K;
    const float *row_sh = ws_shat + (((size_t)b * D.Hq + g * G + hh) * D.T + (valid ? i : 0)) * K;
    int ns = 0;
    float m2 = -INFINITY;  // running max, log2 units
    if (valid) {
        // The ids must be in canonical form: candidates (c < lpos / S) strictly ascending, then -1. A row
        // that is not keeps its canonical prefix and raises the call's error word.
        const int n_r = lpos / S;
        bool canon = true;
        int prev = -1;
        for (int t = 0; t < K; ++t) {
            const int c = row_idx[t];
            if (c == -1) {
                for (int t2 = t + 1; t2 < K; ++t2) canon = canon && row_idx[t2] == -1;
                break;
            }
            if (c <= prev || c >= n_r) {
                canon = false;
                break;
            }
            prev = c;
            ++ns;
            m2 = fmaxf(m2, row_sh[t] * kLog2e);
            atomicOr(&bitmap[c >> 5], 1u << (c & 31));
        }
        if (!canon) atomicOr(&g_attn_tc_errors, 2u);
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
        // K of tile n and V of tile n-1 per step, so K loads run ahead of the value products.
        if (lane == 0) {
            const int head0 = b * D.Hq + g * G;
            mbar_arrive_expect_tx(&bar.q_full, kQBytes);
            tma_load_3d(Qs, &qmap, 0, head0, i0, &bar.q_full);
            tma_load_3d(Qs + 16384, &qmap, 64, head0, i0, &bar.q_full);
            const int kvrow0 = (b * D.Hkv + g) * D.L;
            auto load_k = [&](int n) {
                const int st = n % kStages;
                if (n >= kStages && !mbar_wait_bounded(&bar.s_full[st], ((n / kStages) - 1) & 1)) return false;
                unsigned char *Kt = Ks + st * kTileBytes;
                const int y = kvrow0 + list[n] * S;
                mbar_arrive_expect_tx(&bar.k_full[st], kTileBytes);
                tma_load_2d(Kt, &kmap, 0, y, &bar.k_full[st]);
                tma_load_2d(Kt + 8192, &kmap, 64, y, &bar.k_full[st]);
                return true;
            };
            auto load_v = [&](int n) {
                const int st = n % kStages;
                if (n >= kStages && !mbar_wait_bounded(&bar.pv_done[st], ((n / kStages) - 1) & 1)) return false;
                unsigned char *Vt = Vs + st * kTileBytes;
                const int y = kvrow0 + list[n] * S;
                mbar_arrive_expect_tx(&bar.v_full[st], kTileBytes);
                tma_load_2d(Vt, &vmap, 0, y, &bar.v_full[st]);
                tma_load_2d(Vt + 8192, &vmap, 64, y, &bar.v_full[st]);
                return true;
            };
            for (int n = 0; n <= ntiles && ok; ++n) {
                if (n < ntiles && !load_k(n)) ok = false;
                if (ok && n >= 1 && !load_v(n - 1)) ok = false;
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc_qk = idesc_bf16_f32(128, 64, 0, 0);
            const uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
            const uint32_t qa = smem_u32(Qs);
            ok = mbar_wait_bounded(&bar.q_full, 0);
            auto issue_pv = [&](int n) {
                const int st = n % kStages;
                if (!mbar_wait_bounded(&bar.v_full[st], (n / kStages) & 1)) return false;
                tc_fence_after();
                const uint32_t va = smem_u32(Vs + st * kTileBytes);
                const uint32_t pa = tmem + (n & 1) * 64;  // P(n) aliases S(n): 32 columns of bf16 pairs
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16_tmem_a(tmem + 128, pa + ks * 8, sdesc_sw128(va + ks * 2048, 8192, 1024), idesc_pv,
                                     (n > 0 || ks > 0) ? 1u : 0u);
                umma_commit(&bar.pv_done[n & 1]);
                return true;
            };
            for (int n = 0; n < ntiles && ok; ++n) {
                const int st = n % kStages, sb = n & 1;
                if (!mbar_wait_bounded(&bar.k_full[st], (n / kStages) & 1)) { ok = false; break; }
                // S/P buffer sb held P(n-2): reuse it only after PV(n-2) has completed
                if (n >= 2 && !mbar_wait_bounded(&bar.pv_done[sb], ((n - 2) >> 1) & 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t ka = smem_u32(Ks + st * kTileBytes);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (ks >> 2) * 8192 + (ks & 3) * 32;
                    const uint32_t qoff = (ks >> 2) * 16384 + (ks & 3) * 32;
                    umma_bf16(tmem + sb * 64, sdesc_sw128(qa + qoff, 16, 1024), sdesc_sw128(ka + off, 16, 1024),
                              idesc_qk, ks > 0 ? 1u : 0u);
                }
                umma_commit(&bar.s_full[sb]);
                if (n >= 1) {
                    if (!mbar_wait_bounded(&bar.p_full[(n - 1) & 1], ((n - 1) >> 1) & 1)) { ok = false; break; }
                    tc_fence_after();
                    if (!issue_pv(n - 1)) { ok = false; break; }
                }
            }
            if (ok && ntiles > 0) {
                if (mbar_wait_bounded(&bar.p_full[(ntiles - 1) & 1], ((ntiles - 1) >> 1) & 1)) {
                    tc_fence_after();
                    if (!issue_pv(ntiles - 1)) ok = false;
                } else {
                    ok = false;
                }
            }
            umma_commit(&bar.o_final);  // arrives once every MMA above has completed (also on error paths)
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- one row per thread
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
        const float2 sc2 = make_float2(scale2, scale2);
        float l_run = 0.f;
        // Cursor into the row's ascending chunk list, walked from the top because tiles arrive in
        // descending order. Every selected chunk is in the tile list, so the current entry is matched by
        // equality; the entry after it is loaded one match ahead, off the critical path.
        int u = ns - 1;
        int cur_c = (valid && u >= 0) ? row_idx[u] : -1;
        float cur_sh2 = (valid && u >= 0) ? row_sh[u] * kLog2e : 0.f;
        int nxt_c = (valid && u >= 1) ? row_idx[u - 1] : -1;
        float nxt_sh2 = (valid && u >= 1) ? row_sh[u - 1] * kLog2e : 0.f;
        for (int n = 0; n < ntiles; ++n) {
            const int sb = n & 1;
            const int c = list[n];
            const int j0 = c * S;
            const bool sel = valid && cur_c == c;
            int lo = 0, hi = S - 1;
            if (valid && !sel) {
                lo = max(lpos - j0, 0);
                hi = min(pos - j0, S - 1);
            }
            const bool win = valid && !sel && lo <= hi;
            const float sh2 = cur_sh2;
            if (sel) {
                cur_c = nxt_c;
                cur_sh2 = nxt_sh2;
                --u;
                nxt_c = u >= 1 ? row_idx[u - 1] : -1;
                nxt_sh2 = u >= 1 ? row_sh[u - 1] * kLog2e : 0.f;
            }
            if (__any_sync(0xffffffffu, !mbar_wait_bounded(&bar.s_full[sb], (n >> 1) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t pk[32];
            float factor = 1.f;
            if (__any_sync(0xffffffffu, sel || win)) {
                float v[64];
                {
                    float a[32];
                    tmem_ld32(lane_base + sb * 64, a);
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[e] = a[e];
                    tmem_ld32(lane_base + sb * 64 + 32, a);
#pragma unroll
                    for (int e = 0; e < 32; ++e) v[32 + e] = a[e];
                    tmem_wait_ld();
                }
                // only a window row whose window starts or ends inside this tile needs a mask
                if (__any_sync(0xffffffffu, win && (lo > 0 || hi < S - 1))) {
                    const int mlo = win ? lo : 0, mhi = win ? hi : S - 1;
#pragma unroll
                    for (int e = 0; e < 64; ++e) v[e] = (e >= mlo && e <= mhi) ? v[e] : -INFINITY;
                }
                float mx[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) mx[e] = v[e];
#pragma unroll
                for (int e = 8; e < 64; ++e) mx[e & 7] = fmaxf(mx[e & 7], v[e]);
                const float mraw = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                         fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
                const float tmax = mraw * scale2;  // tau > 0: the max commutes with the scale
                if (win && tmax > m2 + kRescaleSlack2) {
                    // a row with no mass yet (m2 = -inf) has O = 0 and l = 0: no rescale needed
                    if (m2 != -INFINITY) factor = ex2_approx(m2 - tmax);
                    l_run *= factor;
                    m2 = tmax;
                }
                // e_j = 2^(t_j - base): window rows use the running max, all others their tile max
                const float basev = win ? m2 : tmax;
                const float2 nb2 = make_float2(-basev, -basev);
                float2 zacc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                  make_float2(0.f, 0.f)};
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    float2 t = __ffma2_rn(make_float2(v[2 * e], v[2 * e + 1]), sc2, nb2);
                    t.x = ex2_approx(t.x);
                    t.y = ex2_approx(t.y);
                    v[2 * e] = t.x;
                    v[2 * e + 1] = t.y;
                    zacc[e & 3] = __fadd2_rn(zacc[e & 3], t);
                }
                const float2 zz = __fadd2_rn(__fadd2_rn(zacc[0], zacc[1]), __fadd2_rn(zacc[2], zacc[3]));
                const float z = zz.x + zz.y;
                // selected chunk: total mass 2^(s^2 - m2), split by the intra-chunk softmax e_j / z;
                // a row that neither selects nor windows this tile contributes P = 0
                const float mass = sel ? ex2_approx(sh2 - m2) : 0.f;
                const float f = sel ? mass / z : (win ? 1.f : 0.f);
                l_run += win ? z : mass;
                const float2 f2 = make_float2(f, f);
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float2 pr = __fmul2_rn(make_float2(v[2 * e], v[2 * e + 1]), f2);
                    const __nv_bfloat162 h2 = __floats2bfloat162_rn(pr.x, pr.y);
                    pk[e] = *reinterpret_cast<const uint32_t *>(&h2);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) pk[e] = 0u;
            }
            // O rescale (rare; warp-collective TMEM access) once PV(n-1) has completed
            const unsigned need = __ballot_sync(0xffffffffu, factor != 1.f && n >= 1);
            if (need) {
                if (__any_sync(0xffffffffu, !mbar_wait_bounded(&bar.pv_done[(n - 1) & 1], ((n - 1) >> 1) & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll 1
                for (int t = 0; t < 4; ++t) {
                    float o[32];
                    tmem_ld32(lane_base + 128 + 32 * t, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] *= factor;
                    tmem_st32(lane_base + 128 + 32 * t, o);
                }
            }
            // P(n) over S(n) in TMEM (S(n) is read; PV(n-2), the last reader of these columns, completed
            // before QK(n) was issued)
            tmem_st32u(lane_base + sb * 64, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bar.p_full[sb]);
        }
        // epilogue
        if (__any_sync(0xffffffffu, !mbar_wait_bounded(&bar.o_final, 0))) ok = false;
        tc_fence_after();
        const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
        __nv_bfloat16 *orow = out + (((size_t)b * D.Hq + g * G + hh) * D.T + (valid ? i : 0)) * 128;
#pragma unroll 1
        for (int t = 0; t < 4; ++t) {
            float o[32];
            tmem_ld32(lane_base + 128 + 32 * t, o);
            tmem_wait_ld();
            if (valid) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint32_t w[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(o[8 * k + 2 * e] * inv, o[8 * k + 2 * e + 1] * inv);
                        w[e] = *reinterpret_cast<const uint32_t *>(&h2);
                    }
                    *reinterpret_cast<uint4 *>(orow + 32 * t + 8 * k) = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
        if (valid) lse[((size_t)b * D.Hq + g * G + hh) * D.T + i] = (m2 + log2f(l_run)) * (1.f / kLog2e);
    }
    if (!ok) atomicOr(&g_attn_tc_errors, 1u);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

size_t workspace_bytes(const Dims &D) {
    const size_t a = ((size_t)D.B * D.Hkv * D.T * D.topk * sizeof(int) + 255) & ~(size_t)255;
    const size_t s = ((size_t)D.B * D.Hq * D.T * D.topk * sizeof(float) + 255) & ~(size_t)255;
    return a + s;
}

}  // namespace

bool attn_fwd_tc_supported(const Dims &D, int dtype) {
    if (!select_tc_supported(D, dtype)) return false;  // the gather GEMM: bf16, d 128, G <= 4, <= 128 candidates
    if (D.S != 64 || D.topk > 32 || (128 % D.G) != 0) return false;
    const int QT = 128 / D.G;
    const int nchunks = (D.L + D.S - 1) / D.S;
    const int max_list = (D.W + 2 * D.S + QT) / D.S + 2 + QT * D.topk;
    return nchunks <= 32 * kBitmapWords && max_list <= kListCap;
}

size_t attn_fwd_tc_workspace(const Dims &D) { return workspace_bytes(D); }

unsigned int attn_tc_error_flags(bool clear) {
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_attn_tc_errors, sizeof(v));
    if (clear && v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_attn_tc_errors, &zero, sizeof(zero));
    }
    return v;
}

namespace {

cudaError_t launch_attn_tc(const Dims &D, const void *q, const void *k, const void *v, const int *ids,
                           const float *shat, void *out, float *lse, cudaStream_t stream) {
    CUtensorMap qmap, kmap, vmap;
    const int QT = 128 / D.G;
    if (!make_tmap_bf16_3d(&qmap, q, 128, (uint64_t)D.B * D.Hq, (uint64_t)D.T, (uint64_t)D.T * 128 * 2, 128 * 2, D.G,
                           QT) ||
        !make_tmap_bf16_2d(&kmap, k, (uint64_t)D.B * D.Hkv * D.L, 128, 128, 64) ||
        !make_tmap_bf16_2d(&vmap, v, (uint64_t)D.B * D.Hkv * D.L, 128, 128, 64))
        return cudaErrorInvalidValue;
    const size_t smem = 1024 + kQBytes + 2 * kStages * kTileBytes;
    cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 grid((D.T + QT - 1) / QT, D.Hkv, D.B);
    attn_tc_kernel<<<grid, kThreads, smem, stream>>>(qmap, kmap, vmap, D, ids, shat, (__nv_bfloat16 *)out, lse);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_tc(const Dims &D, const void *q, const void *k, const void *v, const void *q_hat,
                               const void *k_sum, const float *b_sum, const int *idx, void *out, float *lse,
                               void *ws, cudaStream_t stream) {
    unsigned char *w = (unsigned char *)ws;
    int *ws_idx = (int *)w;
    float *ws_shat = (float *)(w + (((size_t)D.B * D.Hkv * D.T * D.topk * sizeof(int) + 255) & ~(size_t)255));
    cudaError_t e = launch_gather_shat_tc(D, q_hat, k_sum, b_sum, idx, ws_idx, ws_shat, stream);
    if (e != cudaSuccess) return e;
    return launch_attn_tc(D, q, k, v, ws_idx, ws_shat, out, lse, stream);
}

// Ids in canonical form with their retrieval scores given (as hils_select_topk writes them with shat):
// no gather, and no limit of 128 candidates per row.
bool attn_fwd_shat_supported(const Dims &D, int dtype) {
    if (dtype != HILS_BF16 || D.d != 128 || D.S != 64 || D.topk > 32 || (128 % D.G) != 0 || D.G > 128) return false;
    const int QT = 128 / D.G;
    const int nchunks = (D.L + D.S - 1) / D.S;
    const int max_list = (D.W + 2 * D.S + QT) / D.S + 2 + QT * D.topk;
    return nchunks <= 32 * kBitmapWords && max_list <= kListCap;
}

cudaError_t launch_attn_fwd_tc_shat(const Dims &D, const void *q, const void *k, const void *v, const int *idx,
                                    const float *shat, void *out, float *lse, cudaStream_t stream) {
    return launch_attn_tc(D, q, k, v, idx, shat, out, lse, stream);
}

}  // namespace hils
