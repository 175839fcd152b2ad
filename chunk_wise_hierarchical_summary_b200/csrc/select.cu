// Stage (b): retrieval scores (Eq. 7) and GQA-shared top-k chunk selection
// ("Hierarchical Sparse Attention Done Right", Sec. 3 RQ1 and Sec. 4 "GQA").
//
// One CTA per (b, KV group g, query row i). For the n = n_p candidate chunks of the row:
//   s^_{h,c} = tau * q^_{h,i} . k'_{h,c} + b'_{h,c}          (each head h of the group; fp32)
//   g_c = max_h (s^_{h,c} - LSE_{c'<n} s^_{h,c'})            (per-head normalised weight, max over heads)
// then a block-wide bitonic sort of the keys (g desc, c asc) gives the top-min(k, n) and the gap
// g_(k) - g_(k+1); optionally each head's s^ of the kept ids. The summary rows are read with
// half-warp-per-row 16-byte loads.
#include "internal.h"

namespace hils {
namespace {

constexpr int kSelectThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kSelectThreads)
select_kernel(Dims D, const T *__restrict__ q_hat, const T *__restrict__ k_sum, const float *__restrict__ b_sum,
              int *__restrict__ idx, float *__restrict__ gap, float *__restrict__ shat) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int i = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int d = D.d, G = D.G, K = D.topk;
    const int pos = D.q_pos0 + i;
    const int n = window_left(pos, D.W, D.S) / D.S;
    int *row = idx + (((size_t)b * D.Hkv + g) * D.T + i) * K;
    float *gp = gap ? gap + ((size_t)b * D.Hkv + g) * D.T + i : nullptr;
    // shat (nullable): each head's s^ of the kept ids, in the order of row; -inf in the unused slots
    auto shat_row = [&](int hh) { return shat + (((size_t)b * D.Hq + g * G + hh) * D.T + i) * K; };
    if (n == 0) {
        for (int t = threadIdx.x; t < K; t += blockDim.x) {
            row[t] = -1;
            if (shat)
                for (int hh = 0; hh < G; ++hh) shat_row(hh)[t] = -INFINITY;
        }
        if (gp && threadIdx.x == 0) *gp = INFINITY;
        return;
    }
    const int npad = next_pow2(n);
    uint64_t *keys = reinterpret_cast<uint64_t *>(smem_raw);    // [npad]
    float *sc = reinterpret_cast<float *>(keys + npad);         // [G][n]
    float *qs = sc + (size_t)G * n;                             // [G][d]
    float *lse = qs + (size_t)G * d;                            // [G]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;

    for (int e = threadIdx.x; e < G * d; e += blockDim.x) {
        const int hh = e / d, t = e % d;
        qs[e] = to_f(q_hat[(((size_t)b * D.Hq + g * G + hh) * D.T + i) * d + t]);
    }
    __syncthreads();

    // Scores: each row (h, c) is d elements; lanes_per_row lanes x 8 elements.
    const int lanes_per_row = d / 8;  // 8 (d=64) or 16 (d=128)
    const int rows_per_warp = 32 / lanes_per_row;
    const int sub = lane / lanes_per_row, sl = lane % lanes_per_row;
    for (int r0 = warp * rows_per_warp; r0 < G * n; r0 += nwarps * rows_per_warp) {
        const int r = r0 + sub;
        float part = 0.f;
        int hh = 0, c = 0;
        if (r < G * n) {
            hh = r / n;
            c = r % n;
            float f[8];
            load8(k_sum + (((size_t)b * D.Hq + g * G + hh) * D.Nc + c) * d + sl * 8, f);
            const float *qq = qs + hh * d + sl * 8;
#pragma unroll
            for (int u = 0; u < 8; ++u) part = fmaf(f[u], qq[u], part);
        }
        for (int o = lanes_per_row / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        if (r < G * n && sl == 0)
            sc[hh * n + c] = fmaf(D.tau, part, b_sum[((size_t)b * D.Hq + g * G + hh) * D.Nc + c]);
    }
    __syncthreads();

    // Per-head log-partition over the candidates.
    for (int hh = warp; hh < G; hh += nwarps) {
        float mx = -INFINITY;
        for (int c = lane; c < n; c += 32) mx = fmaxf(mx, sc[hh * n + c]);
        mx = warp_max(mx);
        float z = 0.f;
        for (int c = lane; c < n; c += 32) z += __expf(sc[hh * n + c] - mx);
        z = warp_sum(z);
        if (lane == 0) lse[hh] = mx + logf(z);
    }
    __syncthreads();

    for (int c = threadIdx.x; c < npad; c += blockDim.x) {
        if (c < n) {
            float gv = -INFINITY;
            for (int hh = 0; hh < G; ++hh) gv = fmaxf(gv, sc[hh * n + c] - lse[hh]);
            keys[c] = desc_value_key(gv, (uint32_t)c);
        } else {
            keys[c] = ~0ull;
        }
    }
    block_bitonic_sort(keys, npad);

    const int kk = n < K ? n : K;
    if (threadIdx.x == 0) {
        if (gp) *gp = (n > K) ? desc_key_value(keys[K - 1]) - desc_key_value(keys[K]) : INFINITY;
    }
    __syncthreads();
    // Write the kept ids ascending: rank each kept id among the kept ids.
    for (int t = threadIdx.x; t < K; t += blockDim.x) {
        if (t < kk) {
            const uint32_t me = desc_key_index(keys[t]);
            int rank = 0;
            for (int u = 0; u < kk; ++u) rank += desc_key_index(keys[u]) < me;
            row[rank] = (int)me;
            if (shat)
                for (int hh = 0; hh < G; ++hh) shat_row(hh)[rank] = sc[hh * n + me];
        } else {
            row[t] = -1;
            if (shat)
                for (int hh = 0; hh < G; ++hh) shat_row(hh)[t] = -INFINITY;
        }
    }
}

}  // namespace

size_t select_smem_bytes(const Dims &D) {
    const int n = D.Nc;  // upper bound on candidates of any row
    if (n == 0) return 0;
    return (size_t)next_pow2(n) * 8 + (size_t)D.G * n * 4 + (size_t)D.G * D.d * 4 + (size_t)D.G * 4 + 16;
}

cudaError_t launch_select_topk(const Dims &D, int dtype, const void *q_hat, const void *k_sum, const float *b_sum,
                               int *idx, float *gap, float *shat, cudaStream_t stream) {
    const size_t smem = select_smem_bytes(D);
    dim3 grid(D.T, D.Hkv, D.B);
    if (dtype == HILS_BF16) {
        auto kern = select_kernel<__nv_bfloat16>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<grid, kSelectThreads, smem, stream>>>(D, (const __nv_bfloat16 *)q_hat, (const __nv_bfloat16 *)k_sum,
                                                     b_sum, idx, gap, shat);
    } else {
        auto kern = select_kernel<float>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<grid, kSelectThreads, smem, stream>>>(D, (const float *)q_hat, (const float *)k_sum, b_sum, idx, gap,
                                                     shat);
    }
    return cudaGetLastError();
}

}  // namespace hils
