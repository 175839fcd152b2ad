// Stages (c)+(d) on the tensor cores: per-chunk attention and Eq. 10 fusion, prefill form, bf16, d 128,
// chunk size 64 ("Hierarchical Sparse Attention Done Right", Sec. 3 RQ2 / Eq. 10; Sec. 4 kernel).
//
// Two launches:
//  1. gather (select_tc.cu, same tcgen05 GEMM as the selection): each row's ids canonicalised (valid,
//     distinct, ascending) and their retrieval scores s^ written to the workspace.
//  2. this kernel. CTA = 128 rows = 128/G queries x G heads of one KV group (row = query*G + head), so
//     the heads of a group share every K/V tile. The tiles it visits are the union of the queries'
//     window chunks and selected chunks (the paper's query packing over the union, Fig. 4b), in
//     descending chunk order so that window tiles come first.
//       warp 0     TMA producer: Q once (3-D map, rows query-major), then K and V tiles (2-D maps,
//                  128-byte swizzle) into a 3-stage ring.
//       warp 1     MMA issuer: S = Q K^T (M 128, N 64, K 128) into one of two TMEM S buffers, then
//                  O += P V (M 128, N 128, K 64) with V read MN-major; O lives in TMEM throughout.
//       warps 2-5  one row each (the row's TMEM lane): per tile the row is a window row (logits
//                  masked to its window), a selecting row (logits s_j - L_c + s^_c with L_c the
//                  intra-chunk LSE, so the chunk carries mass exp(s^_c)), or neither (P = 0).
//                  P is written to shared memory in the swizzled K-major layout. The running max
//                  starts at max s^ over the row's chunks, which no chunk tile can exceed; only a
//                  window logit more than 8 above it rescales the row of O in TMEM.
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
constexpr int kStages = 3;
constexpr int kListCap = 1024;
constexpr int kBitmapWords = 2048;  // chunks per sequence <= 65536
constexpr uint32_t kQBytes = 32768;
constexpr uint32_t kKVBytes = 32768;  // K tile 16 KiB + V tile 16 KiB
constexpr uint32_t kPBytes = 16384;
constexpr float kRescaleSlack = 8.f;

__device__ unsigned int g_attn_tc_errors = 0;

struct Bars {
    uint64_t q_full, kv_full[kStages], kv_empty[kStages], s_full[2], s_free[2], p_full, pv_done;
};

__global__ void __launch_bounds__(kThreads, 1)
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
    const int i0 = blockIdx.x * QT, g = blockIdx.y, b = blockIdx.z;
    const int S = D.S, K = D.topk;
    unsigned char *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    unsigned char *Qs = base;
    unsigned char *KV = base + kQBytes;
    unsigned char *Ps = KV + kStages * kKVBytes;
    const int nchunks = (D.L + S - 1) / S;
    const int nwords = (nchunks + 31) / 32;

    if (warp == 1) {
        tmem_alloc(&s_tmem, 256);
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bar.q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bar.kv_full[s], 1);
            mbar_init(&bar.kv_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar.s_full[s], 1);
            mbar_init(&bar.s_free[s], 128);
        }
        mbar_init(&bar.p_full, 128);
        mbar_init(&bar.pv_done, 1);
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
    float m_run = -INFINITY;
    if (valid) {
        for (int t = 0; t < K; ++t) {
            const int c = row_idx[t];
            if (c < 0) break;
            ++ns;
            m_run = fmaxf(m_run, row_sh[t]);
            atomicOr(&bitmap[c >> 5], 1u << (c & 31));
        }
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
            mbar_arrive_expect_tx(&bar.q_full, kQBytes);
            tma_load_3d(Qs, &qmap, 0, head0, i0, &bar.q_full);
            tma_load_3d(Qs + 16384, &qmap, 64, head0, i0, &bar.q_full);
            const int kvrow0 = (b * D.Hkv + g) * D.L;
            for (int n = 0; n < ntiles && ok; ++n) {
                const int st = n % kStages;
                if (n >= kStages && !mbar_wait_bounded(&bar.kv_empty[st], ((n / kStages) - 1) & 1)) {
                    ok = false;
                    break;
                }
                unsigned char *Kt = KV + st * kKVBytes, *Vt = Kt + 16384;
                const int y = kvrow0 + list[n] * S;
                mbar_arrive_expect_tx(&bar.kv_full[st], kKVBytes);
                tma_load_2d(Kt, &kmap, 0, y, &bar.kv_full[st]);
                tma_load_2d(Kt + 8192, &kmap, 64, y, &bar.kv_full[st]);
                tma_load_2d(Vt, &vmap, 0, y, &bar.kv_full[st]);
                tma_load_2d(Vt + 8192, &vmap, 64, y, &bar.kv_full[st]);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc_qk = idesc_bf16_f32(128, 64, 0, 0);
            const uint32_t idesc_pv = idesc_bf16_f32(128, 128, 0, 1);
            const uint32_t qa = smem_u32(Qs), pa = smem_u32(Ps);
            ok = mbar_wait_bounded(&bar.q_full, 0);
            auto issue_pv = [&](int n) {
                const int st = n % kStages;
                const uint32_t va = smem_u32(KV + st * kKVBytes + 16384);
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(tmem + 128, sdesc_sw128(pa + ks * 32, 16, 1024), sdesc_sw128(va + ks * 2048, 8192, 1024),
                              idesc_pv, (n > 0 || ks > 0) ? 1u : 0u);
                umma_commit(&bar.pv_done);
                umma_commit(&bar.kv_empty[st]);
            };
            for (int n = 0; n < ntiles && ok; ++n) {
                const int st = n % kStages, sb = n & 1;
                if (!mbar_wait_bounded(&bar.kv_full[st], (n / kStages) & 1)) { ok = false; break; }
                if (n >= 2 && !mbar_wait_bounded(&bar.s_free[sb], ((n >> 1) - 1) & 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t ka = smem_u32(KV + st * kKVBytes);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (ks >> 2) * 8192 + (ks & 3) * 32;
                    const uint32_t qoff = (ks >> 2) * 16384 + (ks & 3) * 32;
                    umma_bf16(tmem + sb * 64, sdesc_sw128(qa + qoff, 16, 1024), sdesc_sw128(ka + off, 16, 1024),
                              idesc_qk, ks > 0 ? 1u : 0u);
                }
                umma_commit(&bar.s_full[sb]);
                if (n >= 1) {
                    if (!mbar_wait_bounded(&bar.p_full, (n - 1) & 1)) { ok = false; break; }
                    tc_fence_after();
                    issue_pv(n - 1);
                }
            }
            if (ok && ntiles > 0) {
                if (mbar_wait_bounded(&bar.p_full, (ntiles - 1) & 1)) {
                    tc_fence_after();
                    issue_pv(ntiles - 1);
                } else {
                    ok = false;
                }
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- one row per thread
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
        float l_run = 0.f;
        int u = ns - 1;  // cursor into the row's ascending chunk list (tiles arrive descending)
        for (int n = 0; n < ntiles; ++n) {
            const int sb = n & 1;
            const int c = list[n];
            float v[64];
            // a failed wait ends the row loop of the whole warp (the wait result is warp-uniform in practice,
            // and the ballot makes it so)
            if (__any_sync(0xffffffffu, !mbar_wait_bounded(&bar.s_full[sb], (n >> 1) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
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
            tc_fence_before();
            mbar_arrive(&bar.s_free[sb]);
            // role of this row for chunk c
            while (u >= 0 && row_idx[u] > c) --u;
            const bool sel = valid && u >= 0 && row_idx[u] == c;
            const int j0 = c * S;
            const bool win = valid && !sel && j0 <= pos && j0 + S - 1 >= lpos;
            float tmax = -INFINITY;
            if (sel) {
                float mx = -INFINITY;
#pragma unroll
                for (int e = 0; e < 64; ++e) {
                    v[e] *= D.tau;
                    mx = fmaxf(mx, v[e]);
                }
                float z = 0.f;
#pragma unroll
                for (int e = 0; e < 64; ++e) z += __expf(v[e] - mx);
                const float off = row_sh[u] - (mx + logf(z));
#pragma unroll
                for (int e = 0; e < 64; ++e) v[e] += off;
                tmax = mx + off;
            } else if (win) {
#pragma unroll
                for (int e = 0; e < 64; ++e) {
                    const int jj = j0 + e;
                    v[e] = (jj >= lpos && jj <= pos) ? v[e] * D.tau : -INFINITY;
                    tmax = fmaxf(tmax, v[e]);
                }
            }
            float factor = 1.f;
            if (tmax > m_run + kRescaleSlack || (m_run == -INFINITY && tmax > -INFINITY)) {
                const float m_new = fmaxf(tmax, m_run);
                factor = (m_run == -INFINITY) ? 0.f : __expf(m_run - m_new);
                l_run *= factor;
                m_run = m_new;
            }
            // P in bf16; row sum in fp32
            uint32_t pk[32];
            float psum = 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float p0 = (sel || win) ? __expf(v[2 * e] - m_run) : 0.f;
                const float p1 = (sel || win) ? __expf(v[2 * e + 1] - m_run) : 0.f;
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                pk[e] = *reinterpret_cast<const uint32_t *>(&h2);
                psum += p0 + p1;
            }
            l_run += psum;
            // P buffer and O are free once PV(n-1) has completed
            if (n >= 1) {
                if (__any_sync(0xffffffffu, !mbar_wait_bounded(&bar.pv_done, (n - 1) & 1))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
            }
            {
                // TMEM loads/stores are warp-collective: the whole warp rescales if any of its rows needs it
                // (rows that do not need it multiply by 1).
                const unsigned need = __ballot_sync(0xffffffffu, factor != 1.f && n >= 1);
                if (need) {
#pragma unroll 1
                    for (int t = 0; t < 4; ++t) {
                        float o[32];
                        tmem_ld32(lane_base + 128 + 32 * t, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] *= factor;
                        tmem_st32(lane_base + 128 + 32 * t, o);
                    }
                    tmem_wait_st();
                }
            }
            // P row r, 128 bytes, 16-byte chunk k stored at chunk k ^ (r % 8)
            unsigned char *prow = Ps + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                uint4 w4 = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
                *reinterpret_cast<uint4 *>(prow + ((k ^ (r & 7)) << 4)) = w4;
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&bar.p_full);
        }
        // epilogue
        if (ok && ntiles > 0) {
            if (__any_sync(0xffffffffu, !mbar_wait_bounded(&bar.pv_done, (ntiles - 1) & 1))) ok = false;
            tc_fence_after();
        }
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
        if (valid) lse[((size_t)b * D.Hq + g * G + hh) * D.T + i] = m_run + logf(l_run);
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

cudaError_t launch_attn_fwd_tc(const Dims &D, const void *q, const void *k, const void *v, const void *q_hat,
                               const void *k_sum, const float *b_sum, const int *idx, void *out, float *lse,
                               void *ws, cudaStream_t stream) {
    unsigned char *w = (unsigned char *)ws;
    int *ws_idx = (int *)w;
    float *ws_shat = (float *)(w + (((size_t)D.B * D.Hkv * D.T * D.topk * sizeof(int) + 255) & ~(size_t)255));
    cudaError_t e = launch_gather_shat_tc(D, q_hat, k_sum, b_sum, idx, ws_idx, ws_shat, stream);
    if (e != cudaSuccess) return e;
    CUtensorMap qmap, kmap, vmap;
    const int QT = 128 / D.G;
    if (!make_tmap_bf16_3d(&qmap, q, 128, (uint64_t)D.B * D.Hq, (uint64_t)D.T, (uint64_t)D.T * 128 * 2, 128 * 2, D.G,
                           QT) ||
        !make_tmap_bf16_2d(&kmap, k, (uint64_t)D.B * D.Hkv * D.L, 128, 128, 64) ||
        !make_tmap_bf16_2d(&vmap, v, (uint64_t)D.B * D.Hkv * D.L, 128, 128, 64))
        return cudaErrorInvalidValue;
    const size_t smem = 1024 + kQBytes + kStages * kKVBytes + kPBytes;
    cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    dim3 grid((D.T + QT - 1) / QT, D.Hkv, D.B);
    attn_tc_kernel<<<grid, kThreads, smem, stream>>>(qmap, kmap, vmap, D, ws_idx, ws_shat, (__nv_bfloat16 *)out, lse);
    return cudaGetLastError();
}

}  // namespace hils
