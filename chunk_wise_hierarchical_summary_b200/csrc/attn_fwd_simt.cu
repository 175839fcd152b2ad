// Stages (c)+(d): per-chunk attention and Eq. 10 fusion, general-shape CUDA-core kernel.
// ("Hierarchical Sparse Attention Done Right", Sec. 3 RQ2 / Eq. 10.)
//
// Used for fp32, for d = 64, for chunk sizes other than 64 and for any shape the tensor-core kernel
// does not cover. One warp per (b, h, query row); lane owns d/32 output dims.
//
// Eq. 10 is evaluated as one online softmax over "adjusted" logits: a window token keeps its logit
// s_j; a token of selected chunk c gets s_j - L_c + s^_c with L_c = LSE_{j in c} s_j, so that the
// chunk's tokens carry total mass exp(s^_c) distributed by the intra-chunk softmax. The per-chunk
// output o_c is therefore never formed; lse = log Z^ falls out of the running (max, sum).
#include "internal.h"

namespace hils {
namespace {

constexpr int kAttnWarps = 4;

template <typename T, int DPL>
__device__ __forceinline__ float dot_lane(const float (&a)[DPL], const T *row, int lane) {
    float s = 0.f;
#pragma unroll
    for (int u = 0; u < DPL; ++u) s = fmaf(a[u], to_f(row[lane + 32 * u]), s);
    return warp_sum(s);
}

template <typename T, int DPL>
__global__ void __launch_bounds__(kAttnWarps * 32)
attn_fwd_simt_kernel(Dims D, const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                     const T *__restrict__ q_hat, const T *__restrict__ k_sum, const float *__restrict__ b_sum,
                     const int *__restrict__ idx, T *__restrict__ out, float *__restrict__ lse) {
    __shared__ float s_logit[kAttnWarps][HILS_MAX_S];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x * kAttnWarps + warp, h = blockIdx.y, b = blockIdx.z;
    if (i >= D.T) return;
    const int g = h / D.G, d = D.d, S = D.S;
    const int pos = D.q_pos0 + i;
    const int l = window_left(pos, D.W, S), n = l / S;
    const size_t qrow = ((size_t)b * D.Hq + h) * D.T + i;
    const T *kb = k + ((size_t)b * D.Hkv + g) * (size_t)D.L * d;
    const T *vb = v + ((size_t)b * D.Hkv + g) * (size_t)D.L * d;

    float qv[DPL], qh[DPL], acc[DPL];
#pragma unroll
    for (int u = 0; u < DPL; ++u) {
        qv[u] = to_f(q[qrow * d + lane + 32 * u]) * D.tau;  // tau folded into q
        qh[u] = to_f(q_hat[qrow * d + lane + 32 * u]) * D.tau;
        acc[u] = 0.f;
    }
    float m = -INFINITY, z = 0.f;

    auto absorb = [&](float s, const T *vrow) {
        if (s > m) {
            const float r = __expf(m - s);
            z *= r;
#pragma unroll
            for (int u = 0; u < DPL; ++u) acc[u] *= r;
            m = s;
        }
        const float w = __expf(s - m);
        z += w;
#pragma unroll
        for (int u = 0; u < DPL; ++u) acc[u] = fmaf(w, to_f(vrow[lane + 32 * u]), acc[u]);
    };

    for (int j = l; j <= pos; ++j) absorb(dot_lane<T, DPL>(qv, kb + (size_t)j * d, lane), vb + (size_t)j * d);

    const int *irow = idx + (((size_t)b * D.Hkv + g) * D.T + i) * D.topk;
    for (int t = 0; t < D.topk; ++t) {
        const int c = irow[t];
        if (c < 0 || c >= n) continue;
        bool dup = false;
        for (int u = 0; u < t; ++u) dup |= (irow[u] == c);
        if (dup) continue;
        const size_t srow = ((size_t)b * D.Hq + h) * D.Nc + c;
        const float shat = dot_lane<T, DPL>(qh, k_sum + srow * d, lane) + b_sum[srow];
        float mx = -INFINITY;
        for (int j = 0; j < S; ++j) {
            const float s = dot_lane<T, DPL>(qv, kb + (size_t)(c * S + j) * d, lane);
            if (lane == 0) s_logit[warp][j] = s;
            mx = fmaxf(mx, s);
        }
        __syncwarp();
        float zc = 0.f;
        for (int j = lane; j < S; j += 32) zc += __expf(s_logit[warp][j] - mx);
        zc = warp_sum(zc);
        const float offset = shat - (mx + logf(zc));
        for (int j = 0; j < S; ++j) absorb(s_logit[warp][j] + offset, vb + (size_t)(c * S + j) * d);
        __syncwarp();
    }

    const float inv = 1.f / z;
#pragma unroll
    for (int u = 0; u < DPL; ++u) out[qrow * d + lane + 32 * u] = from_f<T>(acc[u] * inv);
    if (lane == 0) lse[qrow] = m + logf(z);
}

template <typename T>
cudaError_t launch_t(const Dims &D, const void *q, const void *k, const void *v, const void *q_hat, const void *k_sum,
                     const float *b_sum, const int *idx, void *out, float *lse, cudaStream_t stream) {
    dim3 grid((D.T + kAttnWarps - 1) / kAttnWarps, D.Hq, D.B);
    if (D.d == 128)
        attn_fwd_simt_kernel<T, 4><<<grid, kAttnWarps * 32, 0, stream>>>(
            D, (const T *)q, (const T *)k, (const T *)v, (const T *)q_hat, (const T *)k_sum, b_sum, idx, (T *)out, lse);
    else
        attn_fwd_simt_kernel<T, 2><<<grid, kAttnWarps * 32, 0, stream>>>(
            D, (const T *)q, (const T *)k, (const T *)v, (const T *)q_hat, (const T *)k_sum, b_sum, idx, (T *)out, lse);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_fwd_simt(const Dims &D, int dtype, const void *q, const void *k, const void *v,
                                 const void *q_hat, const void *k_sum, const float *b_sum, const int *idx, void *out,
                                 float *lse, cudaStream_t stream) {
    if (dtype == HILS_BF16) return launch_t<__nv_bfloat16>(D, q, k, v, q_hat, k_sum, b_sum, idx, out, lse, stream);
    return launch_t<float>(D, q, k, v, q_hat, k_sum, b_sum, idx, out, lse, stream);
}

}  // namespace hils
