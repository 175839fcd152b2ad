// Stage (b) on the tensor cores, prefill form: retrieval scores (Eq. 7) and GQA-shared top-k
// ("Hierarchical Sparse Attention Done Right", Sec. 3 RQ1, Sec. 4 "GQA"), bf16, d = 128.
//
// CTA = (128 query rows, KV group g, batch b); 16 warps. For each head h of the group one thread
// TMA-loads the q^ tile [128 x 128] and the summary tile k'_h [128 chunks x 128] (128-byte swizzle,
// three stages, the first loads issued before the setup barrier) and issues 8 tcgen05.mma (M 128, N 128,
// K 16) into TMEM columns [128h, 128h+128): D[i][c] = q^_i . k'_c, committing one barrier per head.
// Then, with rows in TMEM lanes:
//   phase 1  warp (quadrant, head), as soon as its head's product has landed: s^ = tau D + b' (log2
//            units), masked to the row's candidates; LSE_h per row, the next block's TMEM load in flight.
//   phase 2  warp (quadrant, column block of 32): g_c = max_h (s^_{h,c} - LSE_h) as 32-bit keys (score
//            desc cut to 16 mantissa bits, chunk id asc), sorted by a register bitonic network; the
//            exact scores go to shared memory for the gap.
//   phase 3  four lanes of a warp merge a row's four lists (two shuffles a step): top-k ids (ascending,
//            from a 128-bit mask) and the gap, staged in shared memory.
//   phase 4  (optional) each head's s^ of the selected ids, staged in shared memory.
// Ids and scores leave in coalesced copies (the CTA's rows are contiguous).
// Rows whose candidates exceed 128 chunks use the general kernel (select.cu).
//
// Fused Q-Cal (Sec. 4, q^ = q + W_up W_down h with h = q and one rank-32 pair for all heads): the
// loaded tile holds q instead of q^; warps 8-15 (16 rows each) rewrite it in place as q^ before the
// head's MMA: z = W_down q (mma.sync, N = 32), then q + W_up z with z split into bf16 hi + lo, rounded
// once to bf16 into the swizzled tile. The q^ tensor is never formed in HBM.
#include "internal.h"
#include "mma_sync.cuh"
#include "tcgen05.cuh"

namespace hils {

bool make_tmap_bf16_2d(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint64_t ld,
                       uint32_t box_rows);

namespace {

constexpr int kThreads = 512;
constexpr int kRows = 128;
constexpr int kStageBytes = 65536;  // q^ tile (32 KiB) + k' tile (32 KiB)
constexpr int kStages = 3;          // operand stages (heads in flight)
constexpr int kRank = 32;           // Q-Cal rank of the fused path
constexpr int kWdRow = 272;         // W_down row (128 bf16) padded: conflict-free fragment loads
constexpr int kWuRow = 80;          // W_up row (32 bf16) padded
constexpr int kWdBytes = kRank * kWdRow;
constexpr int kWuBytes = 128 * kWuRow;
constexpr int kScoreRow = 129;      // floats per row of exact group scores (odd: conflict-free columns)
template <int K1MAX>
constexpr int kListBytes = (kRows * (4 * K1MAX + 1) * 4 + 15) & ~15;
// Shared memory of the selection: the operand stages, reused after the MMAs for the per-thread sorted
// key lists, the exact group scores and the staged ids (then the staged scores over the lists).
template <int K1MAX>
constexpr size_t select_dyn_smem() {
    const size_t lists = (size_t)kListBytes<K1MAX> + (size_t)kRows * kScoreRow * 4 + (size_t)kRows * 33 * 4;
    return 1024 + (lists > kStages * (size_t)kStageBytes ? lists : kStages * (size_t)kStageBytes);
}

// 32-bit selection key whose ascending order is (score descending, chunk ascending) for chunks < 128:
// the high 25 bits are the order-preserving image of the score cut to 16 mantissa bits, the low 7 the
// chunk. Two scores |v| < 64 apart by more than 2^-10 keep their order; closer ones order by chunk.
__device__ __forceinline__ uint32_t sel_key32(float v, uint32_t c) { return (~float_order_key(v) & ~127u) | c; }

// Ascending bitonic sort of 32 keys held by one thread (compile-time indices: registers only).
__device__ __forceinline__ void sort32_u32(uint32_t (&k)[32]) {
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1)
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int jx = i ^ stride;
                if (jx > i) {
                    const uint32_t a = k[i], b = k[jx];
                    const bool up = (i & size) == 0;
                    k[i] = up ? min(a, b) : max(a, b);
                    k[jx] = up ? max(a, b) : min(a, b);
                }
            }
}

// q -> q^ = q + W_up (W_down q) for rows rb .. rb+15 of a 128 x 128 bf16 tile in the 128-byte-swizzled
// K-major layout (two 64-column halves of 16 KiB), in place. One warp.
__device__ __forceinline__ void qcal_rows(unsigned char *A, const unsigned char *wsm, int rb, int lane) {
    const int g8 = lane >> 2, t4 = lane & 3, mi = lane >> 3, r8 = lane & 7;
    const uint32_t Ab = smem_u32(A);
    const unsigned char *wd = wsm, *wu = wsm + kWdBytes;
    float z[4][4];
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) z[nt][e] = 0.f;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        const int row = rb + r8 + (mi & 1) * 8;
        const int ch = (ks & 3) * 2 + (mi >> 1);
        uint32_t a[4];
        ldsm_x4(Ab + (ks >> 2) * 16384 + row * 128 + ((ch ^ (row & 7)) << 4), a);
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const unsigned char *p = wd + (nt * 8 + g8) * kWdRow + (ks * 16 + 2 * t4) * 2;
            mma_16816(z[nt], a, ld_u32(p), ld_u32(p + 16));
        }
    }
    __syncwarp();  // every lane's fragment loads of these rows are done before any lane rewrites them
    // z (16 x 32, accumulator layout) is the A operand of the second product: k-step kk covers the
    // accumulator tiles 2kk and 2kk+1. Split into bf16 hi + lo so z keeps ~16 significant bits.
    uint32_t ah[2][4], al[2][4];
#pragma unroll
    for (int kk = 0; kk < 2; ++kk)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float x = z[2 * kk + (e >> 1)][2 * (e & 1)], y = z[2 * kk + (e >> 1)][2 * (e & 1) + 1];
            const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
            const float2 hf = __bfloat1622float2(h);
            const __nv_bfloat162 l = __floats2bfloat162_rn(x - hf.x, y - hf.y);
            ah[kk][e] = *reinterpret_cast<const uint32_t *>(&h);
            al[kk][e] = *reinterpret_cast<const uint32_t *>(&l);
        }
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
        float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            const unsigned char *p = wu + (nt * 8 + g8) * kWuRow + (kk * 16 + 2 * t4) * 2;
            const uint32_t b0 = ld_u32(p), b1 = ld_u32(p + 16);
            mma_16816(c, ah[kk], b0, b1);
            mma_16816(c, al[kk], b0, b1);
        }
        const int col = nt * 8 + 2 * t4;
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int row = rb + g8 + 8 * hr;
            unsigned char *qp = A + (col >> 6) * 16384 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2;
            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(qp));
            *reinterpret_cast<__nv_bfloat162 *>(qp) = __floats2bfloat162_rn(f.x + c[2 * hr], f.y + c[2 * hr + 1]);
        }
    }
}

__device__ unsigned int g_select_tc_errors = 0;

// Explicit shared-space accesses (32-bit shared addresses) for the reused operand stages: their
// pointers are derived through the alignment arithmetic, and generic accesses there measured slower.
__device__ __forceinline__ uint32_t lds_u32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ float lds_f32(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void sts_u32(uint32_t a, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void sts_f32(uint32_t a, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(v) : "memory");
}

// Orders every later use of v after the preceding tcgen05.wait::ld: the registers pass through an
// empty volatile asm, which the compiler keeps after the wait and treats as their new definition.
template <int N>
__device__ __forceinline__ void reg_fence(float (&v)[N]) {
#pragma unroll
    for (int i = 0; i < N; ++i) asm volatile("" : "+f"(v[i]));
}

template <int K1MAX, int GATHER, int QCAL>
__global__ void __launch_bounds__(kThreads, 1)
select_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap, Dims D,
                 const float *__restrict__ b_sum, int *__restrict__ idx, float *__restrict__ gap,
                 float *__restrict__ shat, int *__restrict__ ws_idx, float *__restrict__ ws_shat,
                 const __nv_bfloat16 *__restrict__ w_down, const __nv_bfloat16 *__restrict__ w_up) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t tma_bar[kStages], mma_bar[kStages], qcal_bar[kStages], head_bar[4];
    __shared__ __align__(16) unsigned char wsm[QCAL ? kWdBytes + kWuBytes : 16];
    __shared__ uint32_t s_tmem;
    __shared__ __align__(16) float bs[4][kRows];   // b' of the group's heads (natural units)
    __shared__ __align__(16) float bs2[4][kRows];  // b' * log2(e)
    __shared__ float lse[4][kRows];
    __shared__ uint32_t smask[kRows][4];  // selected set of each row (128-bit mask)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int i0 = blockIdx.x * kRows, g = blockIdx.y, b = blockIdx.z;
    const int G = D.G, K = D.topk;
    unsigned char *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);  // 1024-byte aligned
    const uint32_t ncols = G == 1 ? 128 : (G == 2 ? 256 : 512);

    // Operand loads start first: per head h the q^ tile [128 rows x 128] and the summary tile
    // k'_h [128 chunks x 128] (128-byte swizzle) into one of kStages stages.
    auto load = [&](int hh, int st) {
        unsigned char *A = base + st * kStageBytes, *Bt = A + 32768;
        const int hrow = b * D.Hq + g * G + hh;
        mbar_arrive_expect_tx(&tma_bar[st], kStageBytes);
        tma_load_2d(A, &qmap, 0, hrow * D.T + i0, &tma_bar[st]);
        tma_load_2d(A + 16384, &qmap, 64, hrow * D.T + i0, &tma_bar[st]);
        tma_load_2d(Bt, &kmap, 0, hrow * D.Nc, &tma_bar[st]);
        tma_load_2d(Bt + 16384, &kmap, 64, hrow * D.Nc, &tma_bar[st]);
    };
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&tma_bar[i], 1);
            mbar_init(&mma_bar[i], 1);
            mbar_init(&qcal_bar[i], 8);
        }
        for (int i = 0; i < 4; ++i) mbar_init(&head_bar[i], 1);
        fence_mbar_init();
        for (int hh = 0; hh < G && hh < kStages; ++hh) load(hh, hh);
    }
    if (warp == 1) {
        tmem_alloc(&s_tmem, ncols);
        tmem_relinquish();
    }
    if constexpr (QCAL != 0) {
        // W_down [32][128] and W_up [128][32] (bf16, 8 KiB each) into padded rows: one 16-byte piece a thread
        const uint4 wd = reinterpret_cast<const uint4 *>(w_down)[tid];
        const uint4 wu = reinterpret_cast<const uint4 *>(w_up)[tid];
        *reinterpret_cast<uint4 *>(wsm + (tid >> 4) * kWdRow + (tid & 15) * 16) = wd;
        *reinterpret_cast<uint4 *>(wsm + kWdBytes + (tid >> 2) * kWuRow + (tid & 3) * 16) = wu;
    }
    // b' of the group's heads for chunks [0, 128), 0 beyond the summaries.
    for (int e = tid; e < 4 * kRows; e += blockDim.x) {
        const int hh = e / kRows, c = e % kRows;
        const float v = (hh < G && c < D.Nc) ? b_sum[((size_t)b * D.Hq + g * G + hh) * D.Nc + c] : 0.f;
        bs[hh][c] = v;
        bs2[hh][c] = v * kLog2e;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = s_tmem;

    if (warp == 0) {
        // MMA issuer: D_h = q^_h k'_h^T (M 128, N 128, K 128) into TMEM columns [128h, 128h+128); head_bar[h]
        // completes when head h's product has landed (every head's bar is committed, also on error paths).
        if (lane == 0) {
            bool ok = true;
            const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
            int hh = 0;
            for (; hh < G && ok; ++hh) {
                const int st = hh % kStages;
                // the tile is ready once TMA has landed it (and, with Q-Cal, warps 8-15 have rewritten it)
                if (!mbar_wait_bounded(QCAL ? &qcal_bar[st] : &tma_bar[st], (hh / kStages) & 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t A = smem_u32(base + st * kStageBytes), Bt = A + 32768;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    umma_bf16(tmem + hh * 128, sdesc_sw128(A + off, 16, 1024), sdesc_sw128(Bt + off, 16, 1024), idesc,
                              ks > 0);
                }
                umma_commit(&mma_bar[st]);
                umma_commit(&head_bar[hh]);
                if (hh + kStages < G) {
                    if (!mbar_wait_bounded(&mma_bar[st], (hh / kStages) & 1)) { ok = false; ++hh; break; }
                    load(hh + kStages, st);
                }
            }
            for (; hh < G; ++hh) umma_commit(&head_bar[hh]);  // error path: nothing left waits forever
            if (!ok) atomicOr(&g_select_tc_errors, 1u);
        }
        __syncwarp();
    } else if (warp >= 8) {
        if constexpr (QCAL != 0) {
            for (int hh = 0; hh < G; ++hh) {
                const int st = hh % kStages;
                if (!mbar_wait_bounded(&tma_bar[st], (hh / kStages) & 1)) {  // the issuer's wait then expires too
                    if (lane == 0) atomicOr(&g_select_tc_errors, 4u);
                    break;
                }
                qcal_rows(base + st * kStageBytes, wsm, 16 * (warp - 8), lane);
                fence_async_smem();  // generic-proxy writes -> visible to the tensor core's operand reads
                __syncwarp();
                if (lane == 0) mbar_arrive(&qcal_bar[st]);
            }
        }
    }
    const int q = warp & 3, j = warp >> 2;
    const int r = 32 * q + lane;  // tile row = TMEM lane
    const int i = i0 + r;
    const int n_r = (i < D.T) ? window_left(D.q_pos0 + i, D.W, D.S) / D.S : 0;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    bool ok = true;

    if (GATHER) {
        // Gather mode: the caller-given ids of row (query) r are canonicalised once per row (valid ones,
        // distinct, ascending: a 128-bit set in registers, candidates being < 128 here) into shared
        // memory; then each head's warp writes their retrieval scores s^ = tau D + b' to the workspace.
        // The operand stages are dead once every MMA has completed: [0, 66 KiB) holds the per-thread
        // 33-float rows below, the canonical lists follow.
        ok = mbar_wait_bounded(&head_bar[G - 1], 0);  // the last product: every MMA has completed
        tc_fence_after();
        __syncthreads();
        int *clist = reinterpret_cast<int *>(base + (size_t)kThreads * 33 * sizeof(float));
        int *ccount = clist + kRows * D.topk;
        const bool valid = i < D.T;
        if (j == 0) {
            uint32_t m0 = 0u, m1 = 0u, m2 = 0u, m3 = 0u;
            if (valid) {
                const int *src = idx + (((size_t)b * D.Hkv + g) * D.T + i) * K;
                for (int t = 0; t < K; ++t) {
                    const int c = src[t];
                    if (c < 0 || c >= n_r) continue;
                    const uint32_t bit = 1u << (c & 31);
                    const int w = c >> 5;
                    m0 |= (w == 0) ? bit : 0u;
                    m1 |= (w == 1) ? bit : 0u;
                    m2 |= (w == 2) ? bit : 0u;
                    m3 |= (w == 3) ? bit : 0u;
                }
            }
            int ns = 0;
            const uint32_t words[4] = {m0, m1, m2, m3};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint32_t x = words[w];
                while (x) {
                    clist[r * K + ns++] = 32 * w + __ffs(x) - 1;
                    x &= x - 1u;
                }
            }
            ccount[r] = ns;
        }
        __syncthreads();
        if (j < G) {  // warp-uniform: every lane executes the TMEM loads
            const int hh = j;
            const int ns = ccount[r];
            const int *cl = clist + r * K;
            float *dst_s = ws_shat + (((size_t)b * D.Hq + g * G + hh) * D.T + i) * K;
            // each thread copies a 32-column block of its row into a private shared-memory row (stride 33
            // floats, conflict-free) and reads the selected columns back by index
            float *row32 = reinterpret_cast<float *>(base) + (size_t)tid * 33;
            int u = 0;
#pragma unroll 1
            for (int t = 0; t < 4; ++t) {
                float v[32];
                tmem_ld32(lane_base + hh * 128 + 32 * t, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) row32[e] = v[e];
                while (u < ns && cl[u] < 32 * t + 32) {
                    dst_s[u] = fmaf(D.tau, row32[cl[u] - 32 * t], bs[hh][cl[u]]);
                    ++u;
                }
            }
            if (valid) {
                for (int t = ns; t < K; ++t) dst_s[t] = -INFINITY;
                if (hh == 0) {
                    int *dst_i = ws_idx + (((size_t)b * D.Hkv + g) * D.T + i) * K;
                    for (int t = 0; t < K; ++t) dst_i[t] = t < ns ? cl[t] : -1;
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        if (warp == 1) {
            tc_fence_after();
            tmem_dealloc(tmem, ncols);
        }
        if (!ok && tid == 0) atomicOr(&g_select_tc_errors, 2u);
        return;
    }

    // Phase 1: per-head log-partition (log2 units) over the row's candidates, starting as soon as the
    // head's product has landed; one 32-column block at a time (block max, one rescale of the running
    // sum per block), the next block's TMEM load in flight meanwhile.
    if (j < G) {
        const int hh = j;
        ok = mbar_wait_bounded(&head_bar[hh], 0);
        tc_fence_after();
        const float tau2 = D.tau * kLog2e;
        float m = -INFINITY, z = 0.f;
        auto block = [&](float (&v)[32], int t) {
            if (32 * t >= n_r) return;
            const bool full = 32 * t + 32 <= n_r;
            float bm = -INFINITY;
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                float x = fmaf(tau2, v[e], bs2[hh][32 * t + e]);
                if (!full) x = (32 * t + e < n_r) ? x : -INFINITY;
                v[e] = x;
                bm = fmaxf(bm, x);
            }
            if (bm > -INFINITY) {
                const float mn = fmaxf(m, bm);
                float z0 = 0.f, z1 = 0.f;
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    z0 += ex2_approx(v[e] - mn);
                    z1 += ex2_approx(v[e + 1] - mn);
                }
                z = z * ex2_approx(m - mn) + (z0 + z1);  // m = -inf at the first block: 2^-inf = 0
                m = mn;
            }
        };
        const uint32_t col = lane_base + hh * 128;
        float va[32], vb[32];
        tmem_ld32(col, va);
        tmem_wait_ld();
        reg_fence(va);
        tmem_ld32(col + 32, vb);
        block(va, 0);
        tmem_wait_ld();
        reg_fence(vb);
        tmem_ld32(col + 64, va);
        block(vb, 1);
        tmem_wait_ld();
        reg_fence(va);
        tmem_ld32(col + 96, vb);
        block(va, 2);
        tmem_wait_ld();
        reg_fence(vb);
        block(vb, 3);
        lse[hh][r] = (n_r > 0) ? (m + log2f(z)) * kLn2 : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // Phase 2: group scores of column block j (32 candidates a thread) as 32-bit keys, sorted in
    // registers; the exact scores go to shared memory for the gap. The operand stages are dead once every
    // MMA has completed: [0, list bytes) holds the lists, the score rows follow.
    constexpr int kRowKeys = 4 * K1MAX + 1;  // odd: neighbouring rows' lists fall in different banks
    const uint32_t lists = smem_u32(base);                        // uint32 [kRows][kRowKeys]
    const uint32_t gsc = lists + kListBytes<K1MAX>;               // float [kRows][kScoreRow]
    {
        uint32_t key[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int cb = 32 * j + 16 * half;  // first column of this 16-wide piece
            float v[4][16];
#pragma unroll
            for (int hh = 0; hh < 4; ++hh)
                if (hh < G) tmem_ld16(lane_base + hh * 128 + cb, v[hh]);
            tmem_wait_ld();
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) reg_fence(v[hh]);
            float gv[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) gv[e] = -INFINITY;
#pragma unroll
            for (int hh = 0; hh < 4; ++hh) {
                if (hh < G) {
                    const float l = lse[hh][r];
#pragma unroll
                    for (int e = 0; e < 16; ++e) gv[e] = fmaxf(gv[e], fmaf(D.tau, v[hh][e], bs[hh][cb + e]) - l);
                }
            }
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int c = cb + e;
                key[16 * half + e] = (c < n_r) ? sel_key32(gv[e], (uint32_t)c) : 0xffffffffu;
                sts_f32(gsc + 4 * (r * kScoreRow + c), gv[e]);
            }
        }
        sort32_u32(key);
#pragma unroll
        for (int t = 0; t < K1MAX; ++t) sts_u32(lists + 4 * (r * kRowKeys + j * K1MAX + t), t < 32 ? key[t] : 0xffffffffu);
    }
    __syncthreads();

    // Phase 3: the four sorted lists of a row are merged by four lanes of one warp (warp w takes rows
    // 8w .. 8w+7, lane 4u + l holds the head of list l of row 8w + u): per step the row's minimum by two
    // shuffles, the owning lane records it and loads its next key. The first min(K + 1, n) keys give the
    // selected set (a 128-bit mask, one word per lane, read out ascending) and the k-th and (k+1)-th ids
    // for the gap. Ids and scores are staged in shared memory (rows of K + 1 words, conflict-free) and
    // leave in one coalesced copy per tensor: the CTA's rows are contiguous.
    const int KP = K + 1;
    const uint32_t sidx = gsc + kRows * kScoreRow * 4;  // int [kRows][KP]
    const uint32_t sshat = lists;                       // float [G][kRows][KP], once the lists are dead
    {
        const int rr = 8 * warp + (lane >> 2), l = lane & 3;
        const int ii = i0 + rr;
        const int nn = ii < D.T ? window_left(D.q_pos0 + ii, D.W, D.S) / D.S : 0;
        const int need = min(K + 1, nn);
        const uint32_t Lp = lists + 4 * (rr * kRowKeys + l * K1MAX);
        uint32_t a = lds_u32(Lp);
        int p = 1;
        uint32_t word = 0u;  // selected ids c with c >> 5 == l
        uint32_t kk = 0u, kk1 = 0u;
        const int steps = __reduce_max_sync(0xffffffffu, need);
        for (int t = 0; t < steps; ++t) {
            uint32_t m = min(a, __shfl_xor_sync(0xffffffffu, a, 1));
            m = min(m, __shfl_xor_sync(0xffffffffu, m, 2));
            if (t < need) {
                const uint32_t c = m & 127u;
                if (t < K && (int)(c >> 5) == l) word |= 1u << (c & 31);
                if (t == K - 1) kk = c;
                if (t == K) kk1 = c;
                if (a == m) {
                    a = p < K1MAX ? lds_u32(Lp + 4 * p) : 0xffffffffu;
                    ++p;
                }
            }
        }
        // ids of word l go to slots [popc of the lower words, ...); the rest of the row is -1
        const int g4 = lane & ~3;
        const uint32_t w0 = __shfl_sync(0xffffffffu, word, g4), w1 = __shfl_sync(0xffffffffu, word, g4 | 1),
                       w2 = __shfl_sync(0xffffffffu, word, g4 | 2), w3 = __shfl_sync(0xffffffffu, word, g4 | 3);
        if (ii < D.T) {
            const int before = (l > 0 ? __popc(w0) : 0) + (l > 1 ? __popc(w1) : 0) + (l > 2 ? __popc(w2) : 0);
            const int total = __popc(w0) + __popc(w1) + __popc(w2) + __popc(w3);
            const uint32_t row = sidx + 4 * rr * KP;
            int u = before;
            for (uint32_t x = word; x; x &= x - 1u) sts_u32(row + 4 * u++, 32 * l + __ffs(x) - 1);
            if (l == 3)
                for (int t = total; t < K; ++t) sts_u32(row + 4 * t, 0xffffffffu);
            if (gap && l == 0)
                gap[((size_t)b * D.Hkv + g) * D.T + ii] =
                    (nn > K) ? lds_f32(gsc + 4 * (rr * kScoreRow + kk)) - lds_f32(gsc + 4 * (rr * kScoreRow + kk1))
                             : INFINITY;
        } else {
            word = 0u;
        }
        smask[rr][l] = word;
    }

    // Phase 4 (optional): each head's retrieval score s^ = tau D + b' of the selected ids, in id order,
    // -inf in the unused slots. Thread (row, block j) writes the selected columns of its 32-column block
    // for every head (slot = selected ids before it), the next head's TMEM load in flight meanwhile.
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (shat != nullptr) {
        const uint32_t w0 = smask[r][0], w1 = smask[r][1], w2 = smask[r][2], w3 = smask[r][3];
        const uint32_t mj = j == 0 ? w0 : (j == 1 ? w1 : (j == 2 ? w2 : w3));
        const int before = (j > 0 ? __popc(w0) : 0) + (j > 1 ? __popc(w1) : 0) + (j > 2 ? __popc(w2) : 0);
        const int total = __popc(w0) + __popc(w1) + __popc(w2) + __popc(w3);
        const bool valid = i < D.T;
        auto emit = [&](const float (&v)[32], int hh) {
            if (!valid) return;
            const uint32_t dst = sshat + 4 * (hh * kRows + r) * KP;
            int u = before;
#pragma unroll
            for (int e = 0; e < 32; ++e)
                if ((mj >> e) & 1u) sts_f32(dst + 4 * u++, fmaf(D.tau, v[e], bs[hh][32 * j + e]));
            if (j == 3)
                for (int t = total; t < K; ++t) sts_f32(dst + 4 * t, -INFINITY);
        };
        const uint32_t col = lane_base + 32 * j;
        float va[32], vb[32];
        tmem_ld32(col, va);
        tmem_wait_ld();
        reg_fence(va);
        if (G > 1) tmem_ld32(col + 128, vb);
        emit(va, 0);
        if (G > 1) {
            tmem_wait_ld();
            reg_fence(vb);
            if (G > 2) tmem_ld32(col + 256, va);
            emit(vb, 1);
        }
        if (G > 2) {
            tmem_wait_ld();
            reg_fence(va);
            if (G > 3) tmem_ld32(col + 384, vb);
            emit(va, 2);
        }
        if (G > 3) {
            tmem_wait_ld();
            reg_fence(vb);
            emit(vb, 3);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, ncols);
    }
    // coalesced copies out: lane = slot, warps stride over the rows
    const int nr = min(kRows, D.T - i0);
    if (lane < K) {
        int *gidx = idx + (((size_t)b * D.Hkv + g) * D.T + i0) * K;
        for (int rr = warp; rr < nr; rr += kThreads / 32)
            gidx[rr * K + lane] = (int)lds_u32(sidx + 4 * (rr * KP + lane));
        if (shat != nullptr) {
            for (int hh = 0; hh < G; ++hh) {
                float *gs = shat + (((size_t)b * D.Hq + g * G + hh) * D.T + i0) * K;
                const uint32_t ss = sshat + 4 * hh * kRows * KP;
                for (int rr = warp; rr < nr; rr += kThreads / 32) gs[rr * K + lane] = lds_f32(ss + 4 * (rr * KP + lane));
            }
        }
    }
    if (!ok) atomicOr(&g_select_tc_errors, 2u);
}

}  // namespace

bool select_tc_supported(const Dims &D, int dtype) {
    if (dtype != HILS_BF16 || D.d != 128 || D.G > 4 || D.topk > 32 || D.Nc < 1) return false;
    const int n_max = window_left(D.q_pos0 + D.T - 1, D.W, D.S) / D.S;
    return n_max >= 1 && n_max <= kRows;
}

unsigned int select_tc_error_flags(bool clear) {
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_select_tc_errors, sizeof(v));
    if (clear && v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_select_tc_errors, &zero, sizeof(zero));
    }
    return v;
}

namespace {

template <int K1MAX, int QCAL>
void launch_select_variant(const CUtensorMap &qmap, const CUtensorMap &kmap, const Dims &D, const float *b_sum,
                           int *idx, float *gap, float *shat, const __nv_bfloat16 *wd, const __nv_bfloat16 *wu,
                           cudaStream_t stream) {
    const size_t smem = select_dyn_smem<K1MAX>();
    dim3 grid((D.T + kRows - 1) / kRows, D.Hkv, D.B);
    cudaFuncSetAttribute(select_tc_kernel<K1MAX, 0, QCAL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    select_tc_kernel<K1MAX, 0, QCAL><<<grid, kThreads, smem, stream>>>(qmap, kmap, D, b_sum, idx, gap, shat, nullptr,
                                                                        nullptr, wd, wu);
}

}  // namespace

cudaError_t launch_select_tc(const Dims &D, const void *q_hat, const void *k_sum, const float *b_sum, int *idx,
                             float *gap, float *shat, cudaStream_t stream) {
    CUtensorMap qmap, kmap;
    if (!make_tmap_bf16_2d(&qmap, q_hat, (uint64_t)D.B * D.Hq * D.T, 128, 128, 128) ||
        !make_tmap_bf16_2d(&kmap, k_sum, (uint64_t)D.B * D.Hq * D.Nc, 128, 128, 128))
        return cudaErrorInvalidValue;
    if (D.topk <= 16)
        launch_select_variant<17, 0>(qmap, kmap, D, b_sum, idx, gap, shat, nullptr, nullptr, stream);
    else
        launch_select_variant<33, 0>(qmap, kmap, D, b_sum, idx, gap, shat, nullptr, nullptr, stream);
    return cudaGetLastError();
}

// The same selection from q with the Q-Cal projection fused in (rank 32, one W_down [32, 128] and
// W_up [128, 32] pair for every head, bf16, 16-byte aligned).
cudaError_t launch_select_tc_qcal(const Dims &D, const void *q, const void *w_down, const void *w_up,
                                  const void *k_sum, const float *b_sum, int *idx, float *gap, float *shat,
                                  cudaStream_t stream) {
    CUtensorMap qmap, kmap;
    if (!make_tmap_bf16_2d(&qmap, q, (uint64_t)D.B * D.Hq * D.T, 128, 128, 128) ||
        !make_tmap_bf16_2d(&kmap, k_sum, (uint64_t)D.B * D.Hq * D.Nc, 128, 128, 128))
        return cudaErrorInvalidValue;
    const auto *wd = (const __nv_bfloat16 *)w_down;
    const auto *wu = (const __nv_bfloat16 *)w_up;
    if (D.topk <= 16)
        launch_select_variant<17, 1>(qmap, kmap, D, b_sum, idx, gap, shat, wd, wu, stream);
    else
        launch_select_variant<33, 1>(qmap, kmap, D, b_sum, idx, gap, shat, wd, wu, stream);
    return cudaGetLastError();
}

// Canonical selection (valid distinct ids ascending, -1 padded) and the matching retrieval scores of
// every (row, slot), for the tensor-core attention. Same GEMM as the selection; needs topk <= 32.
cudaError_t launch_gather_shat_tc(const Dims &D, const void *q_hat, const void *k_sum, const float *b_sum,
                                  const int *idx, int *ws_idx, float *ws_shat, cudaStream_t stream) {
    CUtensorMap qmap, kmap;
    if (!make_tmap_bf16_2d(&qmap, q_hat, (uint64_t)D.B * D.Hq * D.T, 128, 128, 128) ||
        !make_tmap_bf16_2d(&kmap, k_sum, (uint64_t)D.B * D.Hq * D.Nc, 128, 128, 128))
        return cudaErrorInvalidValue;
    dim3 grid((D.T + kRows - 1) / kRows, D.Hkv, D.B);
    const size_t smem = select_dyn_smem<17>();
    cudaFuncSetAttribute(select_tc_kernel<17, 1, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    select_tc_kernel<17, 1, 0><<<grid, kThreads, smem, stream>>>(qmap, kmap, D, b_sum, const_cast<int *>(idx), nullptr,
                                                                  nullptr, ws_idx, ws_shat, nullptr, nullptr);
    return cudaGetLastError();
}

}  // namespace hils
