// Stage (a): landmark chunk summaries, "Hierarchical Sparse Attention Done Right" Eq. 8 (Prop. 3.1).
//
// This file is the general form (fp32 or bf16, any d and S); bf16 with d 128, S 64 and G <= 8 runs the
// streamed tensor-core kernel of summary_mma.cu instead.
// One CTA per (batch b, KV group g, chunk c). The chunk's S keys are read from HBM once into shared
// memory (fp32) and reused by the G query heads of the group, one warp per head:
//   u_j = tau * q'_{h,c} . k_j,  p = softmax(u),  k'_{h,c} = sum_j p_j k_j,  b'_{h,c} = LSE(u) - sum_j p_j u_j
// (the last form is -sum_j p_j log p_j with log p_j = u_j - LSE(u)).
// HBM traffic per chunk: S*d keys + G*d landmark queries in, G*d summary keys + G biases out.
#include "internal.h"

namespace hils {
namespace {

constexpr int kSummaryWarps = 4;

template <typename T>
__global__ void __launch_bounds__(kSummaryWarps * 32)
summary_kernel(Dims D, const T *__restrict__ k, const T *__restrict__ q_land, int shared_q, int c_begin,
               T *__restrict__ k_sum, float *__restrict__ b_sum) {
    extern __shared__ float smem[];
    const int c = c_begin + blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int d = D.d, S = D.S, G = D.G;
    const int ld = d + 1;  // padded row stride: lane j reading row j stays bank-conflict free
    float *ks = smem;                        // [S][d+1]
    float *qs = ks + S * ld;                 // [G][d]
    float *ps = qs + G * d;                  // [warps][S]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const T *kc = k + (((size_t)b * D.Hkv + g) * D.L + (size_t)c * S) * d;
    for (int e = threadIdx.x * 8; e < S * d; e += blockDim.x * 8) {
        float f[8];
        load8(kc + e, f);
        const int j = e / d, t = e % d;
#pragma unroll
        for (int u = 0; u < 8; ++u) ks[j * ld + t + u] = f[u];
    }
    for (int e = threadIdx.x * 8; e < G * d; e += blockDim.x * 8) {
        const int hh = e / d, t = e % d;
        float f[8];
        load8(q_land + landmark_row(D, shared_q, b, g * G + hh, c) * d + t, f);
#pragma unroll
        for (int u = 0; u < 8; ++u) qs[e + u] = f[u];
    }
    __syncthreads();

    float *pw = ps + warp * S;
    for (int hh = warp; hh < G; hh += kSummaryWarps) {
        const float *ql = qs + hh * d;
        // Logits for tokens j = lane, lane+32, ...
        float mx = -INFINITY;
        for (int j = lane; j < S; j += 32) {
            const float *kj = ks + j * ld;
            float s = 0.f;
            for (int t = 0; t < d; ++t) s = fmaf(ql[t], kj[t], s);
            s *= D.tau;
            pw[j] = s;
            mx = fmaxf(mx, s);
        }
        mx = warp_max(mx);
        float z = 0.f;
        for (int j = lane; j < S; j += 32) z += __expf(pw[j] - mx);
        z = warp_sum(z);
        const float lse = mx + logf(z);
        float pu = 0.f;
        __syncwarp();
        for (int j = lane; j < S; j += 32) {
            const float u = pw[j];
            const float pj = __expf(u - lse);
            pu = fmaf(pj, u, pu);
            pw[j] = pj;
        }
        pu = warp_sum(pu);
        __syncwarp();
        const int h = g * G + hh;
        T *out = k_sum + (((size_t)b * D.Hq + h) * D.Nc + c) * d;
        for (int t = lane; t < d; t += 32) {
            float acc = 0.f;
            for (int j = 0; j < S; ++j) acc = fmaf(pw[j], ks[j * ld + t], acc);
            out[t] = from_f<T>(acc);
        }
        if (lane == 0) b_sum[((size_t)b * D.Hq + h) * D.Nc + c] = lse - pu;
        __syncwarp();
    }
}

}  // namespace

bool summary_mma_supported(const Dims &D, int dtype, const void *k, const void *q_land, const void *k_sum);
cudaError_t launch_summary_mma(const Dims &D, const void *k, const void *q_land, bool shared_q, int c_begin,
                               int c_end, void *k_sum, float *b_sum, cudaStream_t stream);

cudaError_t launch_chunk_summary(const Dims &D, int dtype, const void *k, const void *q_land, bool shared_q,
                                 int c_begin, int c_end, void *k_sum, float *b_sum, cudaStream_t stream) {
    if (c_end <= c_begin) return cudaSuccess;
    if (summary_mma_supported(D, dtype, k, q_land, k_sum))
        return launch_summary_mma(D, k, q_land, shared_q, c_begin, c_end, k_sum, b_sum, stream);
    const size_t smem = sizeof(float) * ((size_t)D.S * (D.d + 1) + (size_t)D.G * D.d + (size_t)kSummaryWarps * D.S);
    dim3 grid(c_end - c_begin, D.Hkv, D.B);
    if (dtype == HILS_BF16) {
        auto kern = summary_kernel<__nv_bfloat16>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<grid, kSummaryWarps * 32, smem, stream>>>(D, (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)q_land,
                                                         (int)shared_q, c_begin, (__nv_bfloat16 *)k_sum, b_sum);
    } else {
        auto kern = summary_kernel<float>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<grid, kSummaryWarps * 32, smem, stream>>>(D, (const float *)k, (const float *)q_land,
                                                         (int)shared_q, c_begin, (float *)k_sum, b_sum);
    }
    return cudaGetLastError();
}

}  // namespace hils
