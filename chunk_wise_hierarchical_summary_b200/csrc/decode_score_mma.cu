// Decode stage (b) for M > 1 query tokens per sequence (multi-token decode / speculative verification):
// retrieval scores s^_{h,m,c} = tau q^_{h,m} . k'_{h,c} + b'_{h,c} ("Hierarchical Sparse Attention Done
// Right", Eq. 7) of M <= 8 queries against every candidate summary, with each summary row read from
// HBM once for all M queries. bf16, d 128.
//
// Persistent kernel over units (b, head h, slice of 128 candidates), two CTAs per SM:
//   warp 4     producer: the slice's k' rows (TMA, two 64-column boxes, 128-byte swizzle) and the M query
//              rows of the head (bulk copies into padded rows), into a kStages-deep ring.
//   warps 0-3  warp w: rows 32w .. 32w+31 of the slice, as two m16 tiles of mma.sync m16n8k16 (k' rows as
//              A, the M queries as the 8-wide N side). Scores go to [B, Hq, M, n]; each warp also
//              writes, per query, a partial (max, sum exp) over its rows, masked to the query's own
//              candidates c < n_m (the queries sit at consecutive positions, so n_m may differ).
#include <algorithm>

#include "internal.h"
#include "mma_sync.cuh"
#include "tcgen05.cuh"

namespace hils {

bool make_tmap_bf16_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint64_t ld,
                       uint32_t box_rows);

namespace {

constexpr int kStages = 3;
constexpr int kConsumerWarps = 4;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kCtasPerSm = 2;  // shared memory (3 stages of 34 KB) holds two CTAs per SM: the grid stays resident
constexpr int kRows = 128;                      // candidates per slice
constexpr uint32_t kKBytes = kRows * 256;       // 128 rows x 128 columns bf16
constexpr uint32_t kQRowBytes = 272;            // a query row (256 B) padded: conflict-free fragment reads
constexpr uint32_t kQBytes = 8 * kQRowBytes;
constexpr int kMaxM = 8;

__device__ unsigned int g_score_mma_errors = 0;

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
decode_score_mma_kernel(const __grid_constant__ CUtensorMap kmap, Dims D, int n, int nslices,
                        const __nv_bfloat16 *__restrict__ q_hat, const float *__restrict__ b_sum,
                        float *__restrict__ scores, float *__restrict__ part, unsigned int *__restrict__ clear,
                        int nclear) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
    unsigned char *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int M = D.T;
    const long long units = (long long)D.B * D.Hq * nslices;
    grid_dep_launch();  // the selection's CTAs may take SMs as this grid's CTAs finish
    // the later grids' counters start at zero (they read them only after this grid has completed)
    if (blockIdx.x == 0)
        for (int i = tid; i < nclear; i += blockDim.x) clear[i] = 0u;
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
            int k = 0;
            for (long long u = blockIdx.x; u < units; u += gridDim.x, ++k) {
                const int st = k % kStages;
                if (k >= kStages && !mbar_wait_bounded(&empty[st], ((k / kStages) - 1) & 1)) {
                    ok = false;
                    break;
                }
                const int sl = (int)(u % nslices);
                const long long hrow = u / nslices;  // b * Hq + h
                unsigned char *Kt = base + st * kKBytes;
                unsigned char *Qt = base + kStages * kKBytes + st * kQBytes;
                mbar_arrive_expect_tx(&full[st], kKBytes + (uint32_t)M * 256u);
                const int y = (int)(hrow * D.Nc) + sl * kRows;
                tma_load_2d(Kt, &kmap, 0, y, &full[st]);
                tma_load_2d(Kt + kKBytes / 2, &kmap, 64, y, &full[st]);
                for (int m = 0; m < M; ++m)
                    bulk_g2s(Qt + m * kQRowBytes, q_hat + ((size_t)hrow * M + m) * 128, 256, &full[st]);
            }
        }
        __syncwarp();
    } else {
        // ---------------------------------------------------------------- consumers
        const int g8 = lane >> 2, t4 = lane & 3;
        const int mi = lane >> 3, r8 = lane & 7;
        const bool qv = g8 < M;
        // candidates of query m: chunks before its window
        int nq0 = 0, nq1 = 0;
        if (2 * t4 < M) nq0 = window_left(D.q_pos0 + 2 * t4, D.W, D.S) / D.S;
        if (2 * t4 + 1 < M) nq1 = window_left(D.q_pos0 + 2 * t4 + 1, D.W, D.S) / D.S;
        int k = 0;
        for (long long u = blockIdx.x; u < units; u += gridDim.x, ++k) {
            const int st = k % kStages;
            const int sl = (int)(u % nslices);
            const long long hrow = u / nslices;
            const int c0 = sl * kRows;
            // b' of this lane's four rows, fetched before the tile wait
            float bv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int c = c0 + 32 * warp + 8 * q + g8;  // rows 32w + 16mt + g8 (+8): q = 2mt + half
                bv[q] = c < n ? b_sum[(size_t)hrow * D.Nc + c] : 0.f;
            }
            if (!mbar_wait_bounded(&full[st], (k / kStages) & 1)) {
                ok = false;
                break;
            }
            const uint32_t Kb = smem_u32(base + st * kKBytes);
            const unsigned char *Qt = base + kStages * kKBytes + st * kQBytes;
            float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const unsigned char *qrow = Qt + g8 * kQRowBytes + (ks * 16 + 2 * t4) * 2;
                const uint32_t b0 = qv ? ld_u32(qrow) : 0u, b1 = qv ? ld_u32(qrow + 16) : 0u;
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    const int row = 32 * warp + 16 * mt + r8 + (mi & 1) * 8;
                    const int ch = (ks & 3) * 2 + (mi >> 1);
                    uint32_t a[4];
                    ldsm_x4(Kb + (ks >> 2) * (kKBytes / 2) + row * 128 + ((ch ^ (row & 7)) << 4), a);
                    mma_16816(acc[mt], a, b0, b1);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
            // scores and per-query partials of the warp's 32 rows
            float M0 = -INFINITY, Z0 = 0.f, M1 = -INFINITY, Z1 = 0.f;
            float sc[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = c0 + 32 * warp + 16 * mt + g8 + 8 * (e >> 1);
                    const int qq = 2 * t4 + (e & 1);
                    const int nlim = (e & 1) ? nq1 : nq0;
                    const float s = (qq < M && c < nlim) ? fmaf(D.tau, acc[mt][e], bv[2 * mt + (e >> 1)]) : -INFINITY;
                    sc[mt][e] = s;
                    if (e & 1) M1 = fmaxf(M1, s); else M0 = fmaxf(M0, s);
                }
#pragma unroll
            for (int x = 4; x < 32; x <<= 1) {
                M0 = fmaxf(M0, __shfl_xor_sync(0xffffffffu, M0, x));
                M1 = fmaxf(M1, __shfl_xor_sync(0xffffffffu, M1, x));
            }
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float s = sc[mt][e];
                    if (e & 1) Z1 += s > -INFINITY ? __expf(s - M1) : 0.f;
                    else Z0 += s > -INFINITY ? __expf(s - M0) : 0.f;
                }
#pragma unroll
            for (int x = 4; x < 32; x <<= 1) {
                Z0 += __shfl_xor_sync(0xffffffffu, Z0, x);
                Z1 += __shfl_xor_sync(0xffffffffu, Z1, x);
            }
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = c0 + 32 * warp + 16 * mt + g8 + 8 * (e >> 1);
                    const int qq = 2 * t4 + (e & 1);
                    if (qq < M && c < n) scores[((size_t)hrow * M + qq) * n + c] = sc[mt][e];
                }
            if (g8 == 0) {
                if (2 * t4 < M) {
                    float *pp = part + ((((size_t)hrow * M + 2 * t4) * nslices + sl) * kConsumerWarps + warp) * 2;
                    pp[0] = M0;
                    pp[1] = Z0;
                }
                if (2 * t4 + 1 < M) {
                    float *pp = part + ((((size_t)hrow * M + 2 * t4 + 1) * nslices + sl) * kConsumerWarps + warp) * 2;
                    pp[0] = M1;
                    pp[1] = Z1;
                }
            }
        }
    }
    if (!ok) atomicOr(&g_score_mma_errors, 1u);
}

}  // namespace

bool decode_score_mma_supported(const Dims &D, int dtype, const void *q_hat, const void *k_sum) {
    auto al16 = [](const void *p) { return ((uintptr_t)p & 15u) == 0; };
    return dtype == HILS_BF16 && D.d == 128 && D.T >= 1 && D.T <= kMaxM && al16(q_hat) && al16(k_sum) &&
           (long long)D.B * D.Hq * D.Nc < (1ll << 31);
}

unsigned int decode_score_mma_error_flags(bool clear) {
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_score_mma_errors, sizeof(v));
    if (clear && v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_score_mma_errors, &zero, sizeof(zero));
    }
    return v;
}

// scores [B, Hq, M, n] fp32; part [B, Hq, M, nslices, 4 warps, (max, sum)] fp32; slices of 128 candidates.
cudaError_t launch_decode_score_mma(const Dims &D, int n, int nslices, const void *q_hat, const void *k_sum,
                                    const float *b_sum, float *scores, float *part, unsigned int *clear, int nclear,
                                    cudaStream_t stream) {
    CUtensorMap kmap;
    if (!make_tmap_bf16_2d(&kmap, k_sum, (uint64_t)D.B * D.Hq * D.Nc, 128, 128, kRows)) return cudaErrorInvalidValue;
    const size_t smem = 1024 + kStages * (kKBytes + kQBytes);
    cudaFuncSetAttribute(decode_score_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const long long units = (long long)D.B * D.Hq * nslices;
    const int grid = (int)std::min<long long>(units, (long long)kCtasPerSm * num_sms());
    decode_score_mma_kernel<<<grid, kThreads, smem, stream>>>(kmap, D, n, nslices, (const __nv_bfloat16 *)q_hat,
                                                             b_sum, scores, part, clear, nclear);
    return cudaGetLastError();
}

}  // namespace hils
