// Naive block-sparse attention selection ("Hierarchical Sparse Attention Done Right", Sec. 2): the exact
// mass of every candidate chunk, M_{h,i,c} = LSE_{j in c} tau q_i.k_j, then the same GQA top-k rule the
// HiLS selection applies to its surrogate s^ (Sec. 4 "GQA": per-head normalisation over the candidates,
// max over the group's heads, top-k by (score desc, id asc)). It is the selection the landmark summary
// approximates (Prop. 3.1), so it serves as the exact reference for selection quality; it costs a
// dense O(T^2) pass over all pre-window tokens.
//
// Two launches:
//  1. masses, [B, Hq, T, Nc] fp32, written for c < n_i only:
//     bsa_mass_tc_kernel (bf16, d 128, S 64): CTA = 128 rows = 128/G queries x G heads of one KV
//       group; every candidate chunk of the tile's last query is one K tile. Warp 0 loads Q once and
//       K tiles into a two-stage TMA ring; warp 1 issues S = Q K^T (M 128, N 64, K 128) into two TMEM
//       buffers; warps 2-5 own one row each and reduce the 64 logits of their row to the chunk's LSE.
//     bsa_mass_kernel (any dtype and shape): one warp per (b, h, i), lanes split d.
//  2. bsa_select_kernel: one warp per (b, g, i) reads the G heads' masses of its row and runs the
//     group top-k with (score desc, id asc) 64-bit keys.
#include "internal.h"
#include "tcgen05.cuh"

namespace hils {

bool make_tmap_bf16_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint64_t ld,
                       uint32_t box_rows);
bool make_tmap_bf16_3d(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1_bytes,
                       uint64_t s2_bytes, uint32_t b1, uint32_t b2);

namespace {

constexpr int kThreads = 192;
constexpr int kStages = 2;
constexpr int kCtasPerSm = 3;
constexpr uint32_t kQBytes = 32768;     // 128 rows x 128 d bf16
constexpr uint32_t kTileBytes = 16384;  // 64 tokens x 128 d bf16
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kSelWarps = 8;

__device__ unsigned int g_bsa_errors = 0;

struct Bars {
    // With two K stages and two S buffers, s_full[b] (the QK product of tile n, n % 2 == b, completed)
    // also frees K stage b; s_free[b] (all 128 rows have read S buffer b) lets the next QK overwrite it.
    uint64_t q_full, k_full[kStages], s_full[2], s_free[2], done;
};

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
bsa_mass_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap, Dims D,
                   float *__restrict__ mass) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) Bars bar;
    __shared__ uint32_t s_tmem;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = D.G, QT = 128 / G, S = D.S;
    // late query tiles have the most candidates: launch them first
    const int i0 = (gridDim.x - 1 - blockIdx.x) * QT, g = blockIdx.y, b = blockIdx.z;
    const int ilast = min(D.T, i0 + QT) - 1;
    const int ntiles = window_left(D.q_pos0 + ilast, D.W, S) / S;
    if (ntiles == 0) return;  // no row of the tile has a candidate (uniform over the CTA)
    unsigned char *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    unsigned char *Qs = base;
    unsigned char *Ks = base + kQBytes;

    if (warp == 1) {
        tmem_alloc(&s_tmem, 128);  // S buffers: columns [0, 64) and [64, 128)
        tmem_relinquish();
    }
    if (tid == 0) {
        mbar_init(&bar.q_full, 1);
        for (int s = 0; s < kStages; ++s) mbar_init(&bar.k_full[s], 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar.s_full[s], 1);
            mbar_init(&bar.s_free[s], 128);
        }
        mbar_init(&bar.done, 1);
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
            const int head0 = b * D.Hq + g * G;
            mbar_arrive_expect_tx(&bar.q_full, kQBytes);
            tma_load_3d(Qs, &qmap, 0, head0, i0, &bar.q_full);
            tma_load_3d(Qs + 16384, &qmap, 64, head0, i0, &bar.q_full);
            const int kvrow0 = (b * D.Hkv + g) * D.L;
            for (int n = 0; n < ntiles; ++n) {
                const int st = n % kStages;
                if (n >= kStages && !mbar_wait_bounded(&bar.s_full[st], ((n / kStages) - 1) & 1)) {
                    ok = false;
                    break;
                }
                unsigned char *Kt = Ks + st * kTileBytes;
                mbar_arrive_expect_tx(&bar.k_full[st], kTileBytes);
                tma_load_2d(Kt, &kmap, 0, kvrow0 + n * S, &bar.k_full[st]);
                tma_load_2d(Kt + 8192, &kmap, 64, kvrow0 + n * S, &bar.k_full[st]);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(128, 64, 0, 0);
            const uint32_t qa = smem_u32(Qs);
            ok = mbar_wait_bounded(&bar.q_full, 0);
            for (int n = 0; n < ntiles && ok; ++n) {
                const int st = n % kStages, sb = n & 1;
                if (!mbar_wait_bounded(&bar.k_full[st], (n / kStages) & 1)) { ok = false; break; }
                if (n >= 2 && !mbar_wait_bounded(&bar.s_free[sb], ((n - 2) >> 1) & 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t ka = smem_u32(Ks + st * kTileBytes);
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (ks >> 2) * 8192 + (ks & 3) * 32;
                    const uint32_t qoff = (ks >> 2) * 16384 + (ks & 3) * 32;
                    umma_bf16(tmem + sb * 64, sdesc_sw128(qa + qoff, 16, 1024), sdesc_sw128(ka + off, 16, 1024),
                              idesc, ks > 0 ? 1u : 0u);
                }
                umma_commit(&bar.s_full[sb]);
            }
            // every MMA above has completed once `done` fires (error paths included): TMEM can be freed
            umma_commit(&bar.done);
            if (!mbar_wait_bounded(&bar.done, 0)) ok = false;
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- one row per thread
        const int q4 = warp & 3;
        const int r = 32 * q4 + lane;  // row = TMEM lane = query * G + head
        const int qi = r / G, hh = r % G;
        const int i = i0 + qi;
        const bool valid = i < D.T;
        const int nrow = valid ? window_left(D.q_pos0 + i, D.W, S) / S : 0;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q4) << 16);
        float *mrow = mass + (((size_t)b * D.Hq + g * G + hh) * D.T + (valid ? i : 0)) * D.Nc;
        const float scale2 = D.tau * kLog2e;
        const float2 sc2 = make_float2(scale2, scale2);
        for (int n = 0; n < ntiles; ++n) {
            const int sb = n & 1;
            if (__any_sync(0xffffffffu, !mbar_wait_bounded(&bar.s_full[sb], (n >> 1) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const bool live = __any_sync(0xffffffffu, n < nrow);
            float v[64];
            if (live) {
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
            if (live) {
                float mx[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) mx[e] = v[e];
#pragma unroll
                for (int e = 8; e < 64; ++e) mx[e & 7] = fmaxf(mx[e & 7], v[e]);
                const float m = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                      fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
                const float m2 = m * scale2;  // tau > 0: the max commutes with the scale
                const float2 nb2 = make_float2(-m2, -m2);
                float2 z4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                make_float2(0.f, 0.f)};
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    float2 t = __ffma2_rn(make_float2(v[2 * e], v[2 * e + 1]), sc2, nb2);
                    t.x = ex2_approx(t.x);
                    t.y = ex2_approx(t.y);
                    z4[e & 3] = __fadd2_rn(z4[e & 3], t);
                }
                const float2 zz = __fadd2_rn(__fadd2_rn(z4[0], z4[1]), __fadd2_rn(z4[2], z4[3]));
                if (n < nrow) mrow[n] = (m2 + log2f(zz.x + zz.y)) * (1.f / kLog2e);
            }
        }
    }
    if (!ok) atomicOr(&g_bsa_errors, 1u);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 128);
    }
}

// Any dtype / shape: one warp per (b, h, i); lane t holds q elements t, t+32, ... (d <= 128).
template <typename T>
__global__ void __launch_bounds__(256)
bsa_mass_kernel(Dims D, const T *__restrict__ q, const T *__restrict__ k, float *__restrict__ mass) {
    const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= (long long)D.B * D.Hq * D.T) return;
    const int i = (int)(w % D.T);
    const int h = (int)((w / D.T) % D.Hq), b = (int)(w / ((long long)D.T * D.Hq));
    const int n = window_left(D.q_pos0 + i, D.W, D.S) / D.S;
    const int d = D.d, per = (d + 31) / 32;
    float qv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) qv[e] = (e < per && lane + 32 * e < d) ? to_f(q[(size_t)w * d + lane + 32 * e]) : 0.f;
    const T *kb = k + ((size_t)b * D.Hkv + h / D.G) * D.L * d;
    float *mrow = mass + (size_t)w * D.Nc;
    for (int c = 0; c < n; ++c) {
        float m = -INFINITY, z = 0.f;
        for (int j = c * D.S; j < (c + 1) * D.S; ++j) {
            float part = 0.f;
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (e < per && lane + 32 * e < d) part = fmaf(qv[e], to_f(kb[(size_t)j * d + lane + 32 * e]), part);
            const float s = warp_sum(part) * D.tau;  // every lane holds the full dot product
            if (s > m) {
                z = z * __expf(m - s) + 1.f;
                m = s;
            } else {
                z += __expf(s - m);
            }
        }
        if (lane == 0) mrow[c] = m + __logf(z);
    }
}

// Group top-k from the masses: one warp per (b, g, i); lane t holds candidates t, t+32, ... (VPL per lane).
// Warp-wide minima of the 64-bit (score desc, id asc) keys use two 32-bit redux steps (high word, then
// the low word among the lanes holding that high word).
template <int VPL>
__global__ void __launch_bounds__(32 * kSelWarps)
bsa_select_kernel(Dims D, const float *__restrict__ mass, int *__restrict__ idx, float *__restrict__ gap) {
    const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (w >= (long long)D.B * D.Hkv * D.T) return;
    const int i = (int)(w % D.T);
    const int g = (int)((w / D.T) % D.Hkv), b = (int)(w / ((long long)D.T * D.Hkv));
    const int n = window_left(D.q_pos0 + i, D.W, D.S) / D.S;
    const int K = D.topk, G = D.G;
    int *out = idx + (size_t)w * K;
    if (n == 0) {
        if (lane < K) out[lane] = -1;
        if (gap != nullptr && lane == 0) gap[w] = INFINITY;
        return;
    }
    float gs[VPL];
#pragma unroll
    for (int t = 0; t < VPL; ++t) gs[t] = -INFINITY;
    // four heads at a time: their loads are in flight together and their reductions interleave
    for (int h0 = 0; h0 < G; h0 += 4) {
        float v[4][VPL], mx[4], z[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const bool live = h0 + u < G;
            const float *mr = mass + (((size_t)b * D.Hq + g * G + h0 + (live ? u : 0)) * D.T + i) * D.Nc;
            mx[u] = -INFINITY;
#pragma unroll
            for (int t = 0; t < VPL; ++t) {
                const int c = lane + 32 * t;
                v[u][t] = (live && c < n) ? __ldg(mr + c) : -INFINITY;
            }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
#pragma unroll
            for (int t = 0; t < VPL; ++t) mx[u] = fmaxf(mx[u], v[u][t]);
            mx[u] = float_from_order_key(__reduce_max_sync(0xffffffffu, float_order_key(mx[u])));
            z[u] = 0.f;
#pragma unroll
            for (int t = 0; t < VPL; ++t) z[u] += (v[u][t] > -INFINITY) ? __expf(v[u][t] - mx[u]) : 0.f;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int u = 0; u < 4; ++u) z[u] += __shfl_xor_sync(0xffffffffu, z[u], o);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (h0 + u >= G) break;
            const float lse = mx[u] + __logf(z[u]);
#pragma unroll
            for (int t = 0; t < VPL; ++t)
                if (lane + 32 * t < n) gs[t] = fmaxf(gs[t], v[u][t] - lse);
        }
    }
    uint64_t key[VPL];
#pragma unroll
    for (int t = 0; t < VPL; ++t) {
        const int c = lane + 32 * t;
        key[t] = c < n ? desc_value_key(gs[t], (uint32_t)c) : ~0ull;
    }
    const int kk = min(K, n);
    const int rounds = kk + (n > K ? 1 : 0);
    int my_id = -1;
    float s_k = 0.f, s_k1 = 0.f;
    for (int rd = 0; rd < rounds; ++rd) {
        uint64_t best = key[0];
#pragma unroll
        for (int t = 1; t < VPL; ++t) best = key[t] < best ? key[t] : best;
        const uint32_t hi = (uint32_t)(best >> 32);
        const uint32_t bh = __reduce_min_sync(0xffffffffu, hi);
        const uint32_t bl = __reduce_min_sync(0xffffffffu, hi == bh ? (uint32_t)best : 0xffffffffu);
        const int c = (int)bl;
        const float sv = float_from_order_key(~bh);
        if (rd < kk && lane == rd) my_id = c;
        if (rd == kk - 1) s_k = sv;
        if (rd == kk) s_k1 = sv;
        if ((c & 31) == lane) {
#pragma unroll
            for (int t = 0; t < VPL; ++t)
                if (t == (c >> 5)) key[t] = ~0ull;
        }
    }
    // ids ascending: the lane holding the r-th winner finds its rank among the kk winners
    int rank = 0;
    for (int s2 = 0; s2 < kk; ++s2) {
        const int o = __shfl_sync(0xffffffffu, my_id, s2);
        rank += (lane < kk && o < my_id) ? 1 : 0;
    }
    if (lane < kk) out[rank] = my_id;
    else if (lane < K) out[lane] = -1;
    if (gap != nullptr && lane == 0) gap[w] = n > K ? s_k - s_k1 : INFINITY;
}

template <int VPL>
cudaError_t launch_select(const Dims &D, const float *mass, int *idx, float *gap, cudaStream_t stream) {
    const long long warps = (long long)D.B * D.Hkv * D.T;
    const int grid = (int)((warps + kSelWarps - 1) / kSelWarps);
    bsa_select_kernel<VPL><<<grid, 32 * kSelWarps, 0, stream>>>(D, mass, idx, gap);
    return cudaGetLastError();
}

}  // namespace

int bsa_max_candidates(const Dims &D) { return window_left(D.q_pos0 + D.T - 1, D.W, D.S) / D.S; }

bool bsa_tc_supported(const Dims &D, int dtype, const void *q, const void *k) {
    auto al16 = [](const void *p) { return ((uintptr_t)p & 15u) == 0; };
    return dtype == HILS_BF16 && D.d == 128 && D.S == 64 && D.G <= 8 && (128 % D.G) == 0 && al16(q) && al16(k) &&
           (long long)D.B * D.Hkv * D.L < (1ll << 31) && (long long)D.B * D.Hq * D.T < (1ll << 31);
}

unsigned int bsa_error_flags(bool clear) {
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_bsa_errors, sizeof(v));
    if (clear && v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_bsa_errors, &zero, sizeof(zero));
    }
    return v;
}

// Masses [B, Hq, T, Nc] (c < n_i written), then the group top-k. Needs topk <= 32 and at most 1024
// candidates per row (checked by the caller).
cudaError_t launch_bsa_select_topk(const Dims &D, int dtype, const void *q, const void *k, int *idx, float *gap,
                                   float *mass, cudaStream_t stream) {
    if (bsa_tc_supported(D, dtype, q, k)) {
        CUtensorMap qmap, kmap;
        const int QT = 128 / D.G;
        if (!make_tmap_bf16_3d(&qmap, q, 128, (uint64_t)D.B * D.Hq, (uint64_t)D.T, (uint64_t)D.T * 128 * 2, 128 * 2,
                               D.G, QT) ||
            !make_tmap_bf16_2d(&kmap, k, (uint64_t)D.B * D.Hkv * D.L, 128, 128, 64))
            return cudaErrorInvalidValue;
        const size_t smem = 1024 + kQBytes + kStages * kTileBytes;
        cudaFuncSetAttribute(bsa_mass_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        dim3 grid((D.T + QT - 1) / QT, D.Hkv, D.B);
        bsa_mass_tc_kernel<<<grid, kThreads, smem, stream>>>(qmap, kmap, D, mass);
    } else {
        const long long warps = (long long)D.B * D.Hq * D.T;
        const int grid = (int)((warps + 7) / 8);
        if (dtype == HILS_BF16)
            bsa_mass_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(D, (const __nv_bfloat16 *)q,
                                                                     (const __nv_bfloat16 *)k, mass);
        else
            bsa_mass_kernel<float><<<grid, 256, 0, stream>>>(D, (const float *)q, (const float *)k, mass);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int n = bsa_max_candidates(D);
    if (n <= 32) return launch_select<1>(D, mass, idx, gap, stream);
    if (n <= 128) return launch_select<4>(D, mass, idx, gap, stream);
    if (n <= 512) return launch_select<16>(D, mass, idx, gap, stream);
    return launch_select<32>(D, mass, idx, gap, stream);
}

}  // namespace hils
