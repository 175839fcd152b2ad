// Stage (a) for bf16 keys, d 128, S 64, up to 8 heads per KV group: landmark chunk summaries
// ("Hierarchical Sparse Attention Done Right", Eq. 8 / Prop. 3.1), streamed at HBM rate.
//
// Persistent kernel. Unit = (batch b, KV group g, chunk c); units are dealt round-robin to the CTAs,
// chunk index fastest, so concurrently running CTAs read neighbouring chunks of one KV head.
//   warp 4     producer: per unit one TMA tile of the chunk's 64 keys (two 64-column boxes, 128-byte
//              swizzle) and the G landmark-query rows (bulk copies), into a kStages-deep ring.
//   warps 0-3  the two small contractions on the warp-level tensor-core instruction (mma.sync
//              m16n8k16, bf16 in, fp32 accumulate), with the group's heads as the 8-wide N side:
//                u^T[j, h] = sum_t k[j, t] q'[h, t]            warp w: tokens 16w .. 16w+15
//                softmax over j per head (max, then sum e and sum e*u, across the 4 warps)
//                k'^T[t, h] = sum_j k[j, t] p[h, j]           warp w: columns 32w .. 32w+31
//              p enters the second product as bf16 hi + lo parts (two MMAs), so k' keeps fp32-level
//              accuracy before its final rounding. b' = LSE(u) - sum_j p_j u_j, the entropy of p.
// HBM traffic per unit: 16 KiB of keys + G*256 B of landmark queries in, G*256 B + 4G B out.
#include <algorithm>

#include "internal.h"
#include "mma_sync.cuh"
#include "tcgen05.cuh"

namespace hils {

bool make_tmap_bf16_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint64_t ld,
                       uint32_t box_rows);

namespace {

// Two stages and five CTAs per SM (more consumer warps per SM) beat three stages at three CTAs: the
// per-tile chain of the consumers, not the copies in flight, bounds the stream.
constexpr int kStages = 2;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kCtasPerSm = 5;
constexpr uint32_t kKBytes = 16384;      // 64 keys x 128 columns bf16
constexpr uint32_t kQRowBytes = 272;     // one landmark row (256 B) padded: conflict-free fragment reads
constexpr uint32_t kQBytes = 8 * kQRowBytes;
constexpr int kPStride = 72;             // bf16 elements per row of p (64 + 8 padding)

__device__ unsigned int g_summary_errors = 0;


__global__ void __launch_bounds__(kThreads, kCtasPerSm)
summary_mma_kernel(const __grid_constant__ CUtensorMap kmap, Dims D, const __nv_bfloat16 *__restrict__ q_land,
                   int shared_q, int c_begin, int nc, __nv_bfloat16 *__restrict__ k_sum, float *__restrict__ b_sum) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
    __shared__ float red_m[kConsumerWarps][8], red_z[kConsumerWarps][8], red_e[kConsumerWarps][8];
    __shared__ __align__(16) __nv_bfloat16 p_hi[8 * kPStride], p_lo[8 * kPStride];
    __shared__ __align__(16) __nv_bfloat16 outs[8][128];
    unsigned char *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = D.G;
    const long long units = (long long)nc * D.Hkv * D.B;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    bool ok = true;

    if (warp == kConsumerWarps) {
        // ---------------------------------------------------------------- producer
        if (lane == 0) {
            int n = 0;
            for (long long u = blockIdx.x; u < units; u += gridDim.x, ++n) {
                const int st = n % kStages;
                if (n >= kStages && !mbar_wait_bounded(&empty[st], ((n / kStages) - 1) & 1)) {
                    ok = false;
                    break;
                }
                const int c = c_begin + (int)(u % nc);
                const long long rest = u / nc;
                const int g = (int)(rest % D.Hkv), b = (int)(rest / D.Hkv);
                unsigned char *Kt = base + st * kKBytes;
                unsigned char *Qt = base + kStages * kKBytes + st * kQBytes;
                mbar_arrive_expect_tx(&full[st], kKBytes + (uint32_t)G * 256u);
                const int y = (b * D.Hkv + g) * D.L + c * D.S;
                tma_load_2d(Kt, &kmap, 0, y, &full[st]);
                tma_load_2d(Kt + 8192, &kmap, 64, y, &full[st]);
                for (int h = 0; h < G; ++h)
                    bulk_g2s(Qt + h * kQRowBytes, q_land + landmark_row(D, shared_q, b, g * G + h, c) * 128, 256,
                             &full[st]);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- consumers
        const int g8 = lane >> 2, t4 = lane & 3;
        const int mi = lane >> 3, r8 = lane & 7;
        const bool hv = g8 < G;
        const float tau = D.tau;
        int n = 0;
        for (long long u = blockIdx.x; u < units; u += gridDim.x, ++n) {
            const int st = n % kStages;
            const bool got = mbar_wait_bounded(&full[st], (n / kStages) & 1);
            const uint32_t Kb = smem_u32(base + st * kKBytes);
            const unsigned char *Qt = base + kStages * kKBytes + st * kQBytes;

            // u^T for tokens 16w..16w+15 (rows), heads 0..7 (columns; rows >= G of q' read as zero)
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int row = 16 * warp + r8 + (mi & 1) * 8;
                const int ch = (ks & 3) * 2 + (mi >> 1);
                uint32_t a[4];
                ldsm_x4(Kb + (ks >> 2) * 8192 + row * 128 + ((ch ^ (row & 7)) << 4), a);
                const unsigned char *qrow = Qt + g8 * kQRowBytes + (ks * 16 + 2 * t4) * 2;
                const uint32_t b0 = hv ? ld_u32(qrow) : 0u, b1 = hv ? ld_u32(qrow + 16) : 0u;
                mma_16816(acc, a, b0, b1);
            }
            const float u00 = acc[0] * tau, u01 = acc[1] * tau, u10 = acc[2] * tau, u11 = acc[3] * tau;
            // per-head max over the warp's 16 tokens (lanes sharing t4), then across warps
            float m0 = fmaxf(u00, u10), m1 = fmaxf(u01, u11);
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
                m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
            }
            if (g8 == 0) {
                red_m[warp][2 * t4] = m0;
                red_m[warp][2 * t4 + 1] = m1;
            }
            if (bar_group_any<kConsumerWarps * 32>(!got)) {  // uniform across the consumer warps
                ok = false;
                break;
            }
            float M0 = red_m[0][2 * t4], M1 = red_m[0][2 * t4 + 1];
#pragma unroll
            for (int w = 1; w < kConsumerWarps; ++w) {
                M0 = fmaxf(M0, red_m[w][2 * t4]);
                M1 = fmaxf(M1, red_m[w][2 * t4 + 1]);
            }
            const float e00 = __expf(u00 - M0), e01 = __expf(u01 - M1), e10 = __expf(u10 - M0),
                        e11 = __expf(u11 - M1);
            float z0 = e00 + e10, z1 = e01 + e11;
            float eu0 = fmaf(e00, u00, e10 * u10), eu1 = fmaf(e01, u01, e11 * u11);
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                z0 += __shfl_xor_sync(0xffffffffu, z0, o);
                z1 += __shfl_xor_sync(0xffffffffu, z1, o);
                eu0 += __shfl_xor_sync(0xffffffffu, eu0, o);
                eu1 += __shfl_xor_sync(0xffffffffu, eu1, o);
            }
            if (g8 == 0) {
                red_z[warp][2 * t4] = z0;
                red_z[warp][2 * t4 + 1] = z1;
                red_e[warp][2 * t4] = eu0;
                red_e[warp][2 * t4 + 1] = eu1;
            }
            bar_group<kConsumerWarps * 32>();
            float Z0 = 0.f, Z1 = 0.f, EU0 = 0.f, EU1 = 0.f;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) {
                Z0 += red_z[w][2 * t4];
                Z1 += red_z[w][2 * t4 + 1];
                EU0 += red_e[w][2 * t4];
                EU1 += red_e[w][2 * t4 + 1];
            }
            const float iz0 = 1.f / Z0, iz1 = 1.f / Z1;
            {
                const int j = 16 * warp + g8;
                const float pv[4] = {e00 * iz0, e01 * iz1, e10 * iz0, e11 * iz1};
                const int hh[4] = {2 * t4, 2 * t4 + 1, 2 * t4, 2 * t4 + 1};
                const int jj[4] = {j, j, j + 8, j + 8};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __nv_bfloat16 hi = __float2bfloat16_rn(pv[e]);
                    p_hi[hh[e] * kPStride + jj[e]] = hi;
                    p_lo[hh[e] * kPStride + jj[e]] = __float2bfloat16_rn(pv[e] - __bfloat162float(hi));
                }
            }
            bar_group<kConsumerWarps * 32>();
            // k'^T for columns 32w..32w+31 (two 16-row tiles), heads 0..7
            float o[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const int j0 = 16 * kk;
                const __nv_bfloat16 *ph = p_hi + g8 * kPStride + j0 + 2 * t4;
                const __nv_bfloat16 *pl = p_lo + g8 * kPStride + j0 + 2 * t4;
                const uint32_t bh0 = ld_u32(ph), bh1 = ld_u32(ph + 8), bl0 = ld_u32(pl), bl1 = ld_u32(pl + 8);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    const int j = j0 + r8 + (mi >> 1) * 8;
                    const int dd = 32 * warp + 16 * mt + (mi & 1) * 8;
                    uint32_t a[4];
                    ldsm_x4_trans(Kb + (dd >> 6) * 8192 + j * 128 + ((((dd & 63) >> 3) ^ (j & 7)) << 4), a);
                    mma_16816(o[mt], a, bh0, bh1);
                    mma_16816(o[mt], a, bl0, bl1);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);  // this warp's last read of the stage is done
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int dd = 32 * warp + 16 * mt + g8;
                outs[2 * t4][dd] = __float2bfloat16_rn(o[mt][0]);
                outs[2 * t4 + 1][dd] = __float2bfloat16_rn(o[mt][1]);
                outs[2 * t4][dd + 8] = __float2bfloat16_rn(o[mt][2]);
                outs[2 * t4 + 1][dd + 8] = __float2bfloat16_rn(o[mt][3]);
            }
            bar_group<kConsumerWarps * 32>();
            const int c = c_begin + (int)(u % nc);
            const long long rest = u / nc;
            const int g = (int)(rest % D.Hkv), b = (int)(rest / D.Hkv);
            if (tid < G * 16) {
                const int h = tid >> 4, ch = tid & 15;
                *reinterpret_cast<uint4 *>(k_sum + (((size_t)b * D.Hq + g * G + h) * D.Nc + c) * 128 + ch * 8) =
                    *reinterpret_cast<const uint4 *>(&outs[h][ch * 8]);
            }
            if (warp == 0 && g8 == 0) {
                const float lse0 = M0 + logf(Z0), lse1 = M1 + logf(Z1);
                if (2 * t4 < G) b_sum[((size_t)b * D.Hq + g * G + 2 * t4) * D.Nc + c] = lse0 - EU0 * iz0;
                if (2 * t4 + 1 < G) b_sum[((size_t)b * D.Hq + g * G + 2 * t4 + 1) * D.Nc + c] = lse1 - EU1 * iz1;
            }
        }
    }
    if (!ok) atomicOr(&g_summary_errors, 1u);
}

}  // namespace

bool summary_mma_supported(const Dims &D, int dtype, const void *k, const void *q_land, const void *k_sum) {
    auto al16 = [](const void *p) { return ((uintptr_t)p & 15u) == 0; };
    return dtype == HILS_BF16 && D.d == 128 && D.S == 64 && D.G >= 1 && D.G <= 8 && al16(k) && al16(q_land) &&
           al16(k_sum) && (long long)D.B * D.Hkv * D.L < (1ll << 31);
}

unsigned int summary_error_flags(bool clear) {
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_summary_errors, sizeof(v));
    if (clear && v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_summary_errors, &zero, sizeof(zero));
    }
    return v;
}

cudaError_t launch_summary_mma(const Dims &D, const void *k, const void *q_land, bool shared_q, int c_begin,
                               int c_end, void *k_sum, float *b_sum, cudaStream_t stream) {
    const int nc = c_end - c_begin;
    if (nc <= 0) return cudaSuccess;
    CUtensorMap kmap;
    if (!make_tmap_bf16_2d(&kmap, k, (uint64_t)D.B * D.Hkv * D.L, 128, 128, 64)) return cudaErrorInvalidValue;
    const size_t smem = 1024 + kStages * (kKBytes + kQBytes);
    cudaFuncSetAttribute(summary_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const long long units = (long long)nc * D.Hkv * D.B;
    const int grid = (int)std::min<long long>(units, (long long)kCtasPerSm * num_sms());
    summary_mma_kernel<<<grid, kThreads, smem, stream>>>(kmap, D, (const __nv_bfloat16 *)q_land, (int)shared_q,
                                                         c_begin, nc,
                                                         (__nv_bfloat16 *)k_sum, b_sum);
    return cudaGetLastError();
}

}  // namespace hils
