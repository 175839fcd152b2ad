// Single-token decode over a long KV cache: stages (b)-(d) for one query at position L-1
// ("Hierarchical Sparse Attention Done Right", Eq. 7, Sec. 4 "GQA", Eq. 10).
//
// Four launches, all HBM-streaming CUDA-core kernels (one query row per head: no dense contraction):
//  1. score   grid (slices, Hkv, B): streams the summaries k'/b' of a slice of candidate chunks once,
//             s^_{h,c} = tau q^_h . k'_{h,c} + b'_{h,c}; writes per (slice, head) the partial
//             (max, sum exp) and the slice's top-(k+1) chunks by s^ (value desc, id asc).
//  2. select  grid (Hkv, B): per-head LSE from the partials; group score g_c = max_h (s^_{h,c} - LSE_h)
//             over the union of the lists; top-k by (g desc, c asc).
//             Exactness: if c is in the group's top-(k+1), the head h* attaining g_c ranks c in its own
//             top-(k+1) by s^ (any chunk above c there has a larger g), hence in its slice's list; and
//             g_c is recovered from h*'s entry. So the union of per-slice per-head top-(k+1) lists holds
//             the group's top-(k+1) with exact scores, and ranking the union by the per-entry maximum
//             reproduces the full selection.
//  3. attend  grid (tiles, Hkv, B): one S-token tile (a selected chunk or a window tile) per CTA, all G
//             heads; writes a partial (max, sum, acc[d]) of the Eq. 10 online softmax over adjusted
//             logits (chunk tokens carry s_j - L_c + s^_c).
//  4. combine grid over (b, h): merges the tiles' partials into out and lse.
#include "internal.h"

namespace hils {
namespace {

constexpr int kScoreThreads = 256;
constexpr int kSelThreads = 512;
constexpr int kAttnThreads = 128;
constexpr int kMaxSliceChunks = 8192;
constexpr int kMaxListEntries = 8192;

struct DecodePlan {
    int n;        // candidate chunks
    int nslices;  // score slices per (b, g)
    int per;      // chunks per slice
    int K1;       // list length per (slice, head) = topk + 1
    int wtiles;   // window tiles
    int ntiles;   // topk + wtiles
    size_t off_part, off_list, off_sel, off_attn, total;
};

DecodePlan make_plan(const Dims &D) {
    DecodePlan P{};
    const int pos = D.L - 1;
    const int l = window_left(pos, D.W, D.S);
    P.n = l / D.S;
    P.K1 = D.topk + 1;
    int max_slices = kMaxListEntries / (D.G * P.K1);
    if (max_slices < 1) max_slices = 1;
    int want = (P.n + 255) / 256;
    P.nslices = want < 1 ? 1 : (want > max_slices ? max_slices : want);
    P.per = P.n > 0 ? (P.n + P.nslices - 1) / P.nslices : 0;
    P.wtiles = (pos - l + 1 + D.S - 1) / D.S;
    P.ntiles = D.topk + P.wtiles;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t at = off;
        off += (bytes + 255) & ~(size_t)255;
        return at;
    };
    const size_t BG = (size_t)D.B * D.Hkv;
    P.off_part = take(BG * P.nslices * D.G * 2 * sizeof(float));
    P.off_list = take(BG * P.nslices * D.G * P.K1 * sizeof(uint64_t));
    P.off_sel = take(BG * D.topk * sizeof(int));
    P.off_attn = take((size_t)D.B * D.Hq * P.ntiles * (D.d + 2) * sizeof(float));
    P.total = off;
    return P;
}

template <typename T>
__global__ void __launch_bounds__(kScoreThreads)
decode_score_kernel(Dims D, DecodePlan P, const T *__restrict__ q_hat, const T *__restrict__ k_sum,
                    const float *__restrict__ b_sum, float *__restrict__ part, uint64_t *__restrict__ lists) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int d = D.d, G = D.G;
    const int c0 = s * P.per;
    const int c1 = min(P.n, c0 + P.per);
    const int R = max(0, c1 - c0);
    const int rpad = next_pow2(max(R, 1));
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem_raw);  // [rpad]
    float *qs = reinterpret_cast<float *>(keys + rpad);        // [G][d]
    __shared__ float red[kScoreThreads / 32][2];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;

    for (int e = threadIdx.x; e < G * d; e += blockDim.x) {
        const int hh = e / d, t = e % d;
        qs[e] = to_f(q_hat[((size_t)b * D.Hq + g * G + hh) * d + t]) * D.tau;
    }
    __syncthreads();

    const int lanes_per_row = d / 8;
    const int rows_per_warp = 32 / lanes_per_row;
    const int sub = lane / lanes_per_row, sl = lane % lanes_per_row;
    const size_t bg = (size_t)b * D.Hkv + g;
    for (int hh = 0; hh < G; ++hh) {
        const int h = g * G + hh;
        const T *ksh = k_sum + ((size_t)b * D.Hq + h) * D.Nc * d;
        const float *bsh = b_sum + ((size_t)b * D.Hq + h) * D.Nc;
        const float *qq = qs + hh * d + sl * 8;
        constexpr int U = 4;
        for (int r0 = warp * rows_per_warp * U; r0 < rpad; r0 += nwarps * rows_per_warp * U) {
            float f[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int r = r0 + u * rows_per_warp + sub;
                if (r < R) load8(ksh + (size_t)(c0 + r) * d + sl * 8, f[u]);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int r = r0 + u * rows_per_warp + sub;
                float part_dot = 0.f;
                if (r < R) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) part_dot = fmaf(f[u][e], qq[e], part_dot);
                }
                for (int o = lanes_per_row / 2; o > 0; o >>= 1) part_dot += __shfl_xor_sync(0xffffffffu, part_dot, o);
                if (sl == 0 && r < rpad)
                    keys[r] = (r < R) ? desc_value_key(part_dot + bsh[c0 + r], (uint32_t)(c0 + r)) : ~0ull;
            }
        }
        __syncthreads();
        // Partial (max, sum exp) of this head's slice.
        float mx = -INFINITY;
        for (int r = threadIdx.x; r < R; r += blockDim.x) mx = fmaxf(mx, desc_key_value(keys[r]));
        mx = warp_max(mx);
        if (lane == 0) red[warp][0] = mx;
        __syncthreads();
        mx = -INFINITY;
        for (int w = 0; w < nwarps; ++w) mx = fmaxf(mx, red[w][0]);
        float z = 0.f;
        for (int r = threadIdx.x; r < R; r += blockDim.x) z += __expf(desc_key_value(keys[r]) - mx);
        z = warp_sum(z);
        if (lane == 0) red[warp][1] = z;
        __syncthreads();
        if (threadIdx.x == 0) {
            float zz = 0.f;
            for (int w = 0; w < nwarps; ++w) zz += red[w][1];
            float *pp = part + ((bg * P.nslices + s) * G + hh) * 2;
            pp[0] = mx;
            pp[1] = zz;
        }
        block_bitonic_sort(keys, rpad);
        uint64_t *lst = lists + ((bg * P.nslices + s) * G + hh) * P.K1;
        for (int t = threadIdx.x; t < P.K1; t += blockDim.x) lst[t] = (t < R) ? keys[t] : ~0ull;
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kSelThreads)
decode_select_kernel(Dims D, DecodePlan P, const float *__restrict__ part, const uint64_t *__restrict__ lists,
                     int *__restrict__ sel, int *__restrict__ idx_out) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int g = blockIdx.x, b = blockIdx.y;
    const int G = D.G, K = D.topk;
    const size_t bg = (size_t)b * D.Hkv + g;
    const int E = P.nslices * G * P.K1;
    const int epad = next_pow2(max(E, 1));
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem_raw);  // [epad]
    float *lse = reinterpret_cast<float *>(keys + epad);       // [G]
    int *out = sel + bg * K;
    int *out2 = idx_out ? idx_out + bg * K : nullptr;
    if (P.n == 0) {
        for (int t = threadIdx.x; t < K; t += blockDim.x) {
            out[t] = -1;
            if (out2) out2[t] = -1;
        }
        return;
    }
    for (int hh = threadIdx.x; hh < G; hh += blockDim.x) {
        float M = -INFINITY;
        for (int s = 0; s < P.nslices; ++s) M = fmaxf(M, part[((bg * P.nslices + s) * G + hh) * 2]);
        float Z = 0.f;
        for (int s = 0; s < P.nslices; ++s) {
            const float *pp = part + ((bg * P.nslices + s) * G + hh) * 2;
            if (pp[0] > -INFINITY) Z += pp[1] * __expf(pp[0] - M);
        }
        lse[hh] = M + logf(Z);
    }
    __syncthreads();
    // Pass 1: order the entries by (chunk asc, normalised score desc).
    for (int e = threadIdx.x; e < epad; e += blockDim.x) {
        uint64_t key = ~0ull;
        if (e < E) {
            const uint64_t raw = lists[bg * (size_t)P.nslices * G * P.K1 + e];
            if (raw != ~0ull) {
                const int hh = (e / P.K1) % G;
                const float val = desc_key_value(raw) - lse[hh];
                key = ((uint64_t)desc_key_index(raw) << 32) | (uint64_t)(~float_order_key(val));
            }
        }
        keys[e] = key;
    }
    block_bitonic_sort(keys, epad);
    // Keep the first (largest) entry of each chunk, re-keyed by (value desc, chunk asc).
    uint64_t mine[16];
    int cnt = 0;
    for (int e = threadIdx.x; e < epad; e += blockDim.x) {
        const uint64_t k0 = keys[e];
        uint64_t nk = ~0ull;
        if (k0 != ~0ull && (e == 0 || (keys[e - 1] >> 32) != (k0 >> 32))) {
            const float val = float_from_order_key(~(uint32_t)k0);
            nk = desc_value_key(val, (uint32_t)(k0 >> 32));
        }
        mine[cnt++] = nk;
    }
    __syncthreads();
    cnt = 0;
    for (int e = threadIdx.x; e < epad; e += blockDim.x) keys[e] = mine[cnt++];
    block_bitonic_sort(keys, epad);
    const int kk = min(K, P.n);
    for (int t = threadIdx.x; t < K; t += blockDim.x) {
        if (t < kk) {
            const uint32_t me = desc_key_index(keys[t]);
            int rank = 0;
            for (int u = 0; u < kk; ++u) rank += desc_key_index(keys[u]) < me;
            out[rank] = (int)me;
            if (out2) out2[rank] = (int)me;
        } else {
            out[t] = -1;
            if (out2) out2[t] = -1;
        }
    }
}

template <typename T, int DPL>
__global__ void __launch_bounds__(kAttnThreads)
decode_attn_kernel(Dims D, DecodePlan P, const T *__restrict__ q, const T *__restrict__ q_hat,
                   const T *__restrict__ kc, const T *__restrict__ vc, const T *__restrict__ k_sum,
                   const float *__restrict__ b_sum, const int *__restrict__ sel, float *__restrict__ partial) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int t = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int d = D.d, S = D.S, G = D.G;
    const int ld = d + 1;
    float *ks = reinterpret_cast<float *>(smem_raw);  // [S][d+1]
    float *vs = ks + S * ld;                          // [S][d]
    float *qs = vs + S * d;                           // [G][d]
    float *ls = qs + G * d;                           // [warps][S]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    const size_t bg = (size_t)b * D.Hkv + g;
    const int pos = D.L - 1;
    const int l = window_left(pos, D.W, S);

    int c = -1, j0 = 0, jn = 0;  // tile tokens [j0, j0 + jn)
    if (t < D.topk) {
        c = sel[bg * D.topk + t];
        if (c >= 0) { j0 = c * S; jn = S; }
    } else {
        j0 = l + (t - D.topk) * S;
        jn = min(S, pos + 1 - j0);
    }
    if (jn <= 0) {
        for (int hh = warp; hh < G; hh += nwarps) {
            float *pp = partial + (((size_t)b * D.Hq + g * G + hh) * P.ntiles + t) * (d + 2);
            if (lane == 0) { pp[0] = -INFINITY; pp[1] = 0.f; }
        }
        return;
    }
    const T *kb = kc + (bg * D.L + j0) * d;
    const T *vb = vc + (bg * D.L + j0) * d;
    for (int e = threadIdx.x * 8; e < jn * d; e += blockDim.x * 8) {
        float f[8];
        load8(kb + e, f);
        const int j = e / d, tt = e % d;
#pragma unroll
        for (int u = 0; u < 8; ++u) ks[j * ld + tt + u] = f[u];
        load8(vb + e, f);
#pragma unroll
        for (int u = 0; u < 8; ++u) vs[e + u] = f[u];
    }
    for (int e = threadIdx.x; e < G * d; e += blockDim.x)
        qs[e] = to_f(q[((size_t)b * D.Hq + g * G) * d + e]) * D.tau;
    __syncthreads();

    float *lw = ls + warp * S;
    for (int hh = warp; hh < G; hh += nwarps) {
        const int h = g * G + hh;
        const float *qq = qs + hh * d;
        float mx = -INFINITY;
        for (int j = lane; j < jn; j += 32) {
            const float *kj = ks + j * ld;
            float s = 0.f;
            for (int u = 0; u < d; ++u) s = fmaf(qq[u], kj[u], s);
            lw[j] = s;
            mx = fmaxf(mx, s);
        }
        mx = warp_max(mx);
        float offset = 0.f;
        if (c >= 0) {
            float zc = 0.f;
            for (int j = lane; j < jn; j += 32) zc += __expf(lw[j] - mx);
            zc = warp_sum(zc);
            const size_t srow = ((size_t)b * D.Hq + h) * D.Nc + c;
            float sh = 0.f;
#pragma unroll
            for (int u = 0; u < DPL; ++u)
                sh = fmaf(to_f(q_hat[((size_t)b * D.Hq + h) * d + lane + 32 * u]), to_f(k_sum[srow * d + lane + 32 * u]),
                          sh);
            sh = warp_sum(sh) * D.tau + b_sum[srow];
            offset = sh - (mx + logf(zc));
        }
        const float m = mx + offset;
        float z = 0.f;
        __syncwarp();
        for (int j = lane; j < jn; j += 32) {
            const float w = __expf(lw[j] + offset - m);
            lw[j] = w;
            z += w;
        }
        z = warp_sum(z);
        __syncwarp();
        float *pp = partial + (((size_t)b * D.Hq + h) * P.ntiles + t) * (d + 2);
        for (int u = lane; u < d; u += 32) {
            float acc = 0.f;
            for (int j = 0; j < jn; ++j) acc = fmaf(lw[j], vs[j * d + u], acc);
            pp[2 + u] = acc;
        }
        if (lane == 0) { pp[0] = m; pp[1] = z; }
        __syncwarp();
    }
}

template <typename T>
__global__ void decode_combine_kernel(Dims D, DecodePlan P, const float *__restrict__ partial, T *__restrict__ out,
                                      float *__restrict__ lse) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x * (blockDim.x >> 5) + warp;
    if (bh >= D.B * D.Hq) return;
    const int d = D.d;
    const float *pp = partial + (size_t)bh * P.ntiles * (d + 2);
    float M = -INFINITY;
    for (int t = 0; t < P.ntiles; ++t) M = fmaxf(M, pp[t * (d + 2)]);
    float Z = 0.f;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int t = 0; t < P.ntiles; ++t) {
        const float m = pp[t * (d + 2)];
        if (!(m > -INFINITY)) continue;
        const float r = __expf(m - M);
        Z = fmaf(pp[t * (d + 2) + 1], r, Z);
        for (int u = 0; u < d / 32; ++u) acc[u] = fmaf(pp[t * (d + 2) + 2 + lane + 32 * u], r, acc[u]);
    }
    const float inv = 1.f / Z;
    for (int u = 0; u < d / 32; ++u) out[(size_t)bh * d + lane + 32 * u] = from_f<T>(acc[u] * inv);
    if (lane == 0) lse[bh] = M + logf(Z);
}

template <typename T>
cudaError_t launch_t(const Dims &D, const void *q, const void *q_hat, const void *k_cache, const void *v_cache,
                     const void *k_sum, const float *b_sum, void *out, float *lse, int *idx_out, void *ws,
                     cudaStream_t stream) {
    const DecodePlan P = make_plan(D);
    unsigned char *w = (unsigned char *)ws;
    float *part = (float *)(w + P.off_part);
    uint64_t *lists = (uint64_t *)(w + P.off_list);
    int *sel = (int *)(w + P.off_sel);
    float *partial = (float *)(w + P.off_attn);
    if (P.n > 0) {
        const size_t smem1 = (size_t)next_pow2(max(P.per, 1)) * 8 + (size_t)D.G * D.d * 4;
        auto k1 = decode_score_kernel<T>;
        cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
        k1<<<dim3(P.nslices, D.Hkv, D.B), kScoreThreads, smem1, stream>>>(D, P, (const T *)q_hat, (const T *)k_sum,
                                                                           b_sum, part, lists);
    }
    const int E = P.nslices * D.G * P.K1;
    const size_t smem2 = (size_t)next_pow2(max(E, 1)) * 8 + (size_t)D.G * 4 + 16;
    cudaFuncSetAttribute(decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2);
    decode_select_kernel<<<dim3(D.Hkv, D.B), kSelThreads, smem2, stream>>>(D, P, part, lists, sel, idx_out);
    const size_t smem3 = sizeof(float) * ((size_t)D.S * (D.d + 1) + (size_t)D.S * D.d + (size_t)D.G * D.d +
                                          (size_t)(kAttnThreads / 32) * D.S);
    auto k3 = (D.d == 128) ? decode_attn_kernel<T, 4> : decode_attn_kernel<T, 2>;
    cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem3);
    k3<<<dim3(P.ntiles, D.Hkv, D.B), kAttnThreads, smem3, stream>>>(D, P, (const T *)q, (const T *)q_hat,
                                                                     (const T *)k_cache, (const T *)v_cache,
                                                                     (const T *)k_sum, b_sum, sel, partial);
    const int rows = D.B * D.Hq;
    decode_combine_kernel<T><<<(rows + 3) / 4, 128, 0, stream>>>(D, P, partial, (T *)out, lse);
    return cudaGetLastError();
}

}  // namespace

size_t decode_workspace_bytes(const Dims &D) { return make_plan(D).total; }

bool decode_supported(const Dims &D) {
    const DecodePlan P = make_plan(D);
    return P.per <= kMaxSliceChunks && P.nslices * D.G * P.K1 <= 2 * kMaxListEntries;
}

cudaError_t launch_decode(const Dims &D, int dtype, const void *q, const void *q_hat, const void *k_cache,
                          const void *v_cache, const void *k_sum, const float *b_sum, void *out, float *lse,
                          int *idx_out, void *ws, cudaStream_t stream) {
    if (dtype == HILS_BF16)
        return launch_t<__nv_bfloat16>(D, q, q_hat, k_cache, v_cache, k_sum, b_sum, out, lse, idx_out, ws, stream);
    return launch_t<float>(D, q, q_hat, k_cache, v_cache, k_sum, b_sum, out, lse, idx_out, ws, stream);
}

}  // namespace hils
