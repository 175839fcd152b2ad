// Decode over a long KV cache: stages (b)-(d) for the last M <= 8 query positions, each query with its own
// window and selection (M = 1: the token at L-1) ("Hierarchical Sparse Attention Done Right", Eq. 7,
// Sec. 3 RQ1, Sec. 4 "GQA", Eq. 10).
//
// Three launches (the score grid also clears the two counter arrays the later grids count with; for
// M > 1 the score grid is decode_score_mma.cu's, which reads every summary row once for the M queries):
//  1. score    persistent, one CTA per SM: a producer lane keeps a ring of bulk copies of 128-candidate
//              summary slices (32 KiB at d 128 bf16) in flight; consumer warps compute
//              s^_{h,c} = tau q^_h . k'_{h,c} + b'_{h,c} into a score buffer plus per-warp partials
//              (max, sum exp) of each slice. This launch streams the decode step's dominant bytes.
//  2. select   per (b, KV group): per-head LSE folded from the partials, group score
//              g_c = max_h (s^_{h,c} - LSE_h) as 64-bit keys (score desc, chunk id asc), top-k. For
//              topk <= 32 and G <= 8 one CTA per group: up to 2048 candidates, each of eight warps sorts
//              its 256 keys in registers and warp 0 merges their best 32; longer lists keep an exact
//              lower bound of the top-k and rank the few candidates at or below it (one thread each).
//              With few groups and very long lists several CTAs per group keep their part's top-k and
//              the last CTA to finish (atomic counter, no waiting) merges them.
//  3. attend   bf16 d 128 S 64 G <= 8: decode_attn_mma.cu (split-K CTAs over the group's tiles,
//              warp-level MMAs, online Eq. 10 merge). Otherwise here: one S-token tile (a selected
//              chunk or a window tile) per CTA, K and V staged by bulk copies, all G heads, a partial
//              (max, sum, acc[d]) of the online softmax over adjusted logits (a chunk token carries
//              s_j - L_c + s^_c); the last CTA of each (b, KV group) merges the partials into out, lse.
#include <algorithm>

#include "internal.h"
#include "tma.cuh"

namespace hils {

bool decode_attn_mma_supported(const Dims &D, int dtype, const void *q, const void *k, const void *v, int ntiles);
cudaError_t launch_decode_attn_mma(const Dims &D, int n, int ntiles, const void *q, const void *k_cache,
                                   const void *v_cache, const float *scores, const int *sel, float *partial,
                                   unsigned int *counters, void *out, float *lse, cudaStream_t stream);
unsigned int decode_attn_mma_error_flags(bool clear);
bool decode_score_mma_supported(const Dims &D, int dtype, const void *q_hat, const void *k_sum);
cudaError_t launch_decode_score_mma(const Dims &D, int n, int nslices, const void *q_hat, const void *k_sum,
                                    const float *b_sum, float *scores, float *part, unsigned int *clear, int nclear,
                                    cudaStream_t stream);
unsigned int decode_score_mma_error_flags(bool clear);

namespace {

constexpr int kSelThreads = 256;
constexpr int kSelPart = 1024;    // candidates per select CTA
constexpr int kSelHeadsInFlight = 8;  // heads whose scores each select thread loads up front
constexpr int kSelMerge = 4096;   // shared keys: a part, then the merged lists (nparts * topk <= this)
constexpr int kAttnThreads = 256;

// Device-side error word of this file (bit 0: a bounded wait expired). Read by decode_error_flags().
__device__ unsigned int g_decode_errors = 0;

struct DecodePlan {
    int n;        // candidate chunks of the query at L-1
    int nslices;  // score slices per (b, head)
    int per;      // candidates per slice
    int wtiles;   // window tiles
    int ntiles;   // topk + wtiles
    int nparts;   // select CTAs per (b, KV group)
    size_t off_scores, off_part, off_list, off_sel, off_attn, off_count, off_selcount, total;
};

constexpr int kSliceElems = 16384;  // summary elements per scored slice
constexpr int kScorePartsPerSliceHost = 4;  // partials per slice (one per consumer warp of a slot)

DecodePlan make_plan(const Dims &D) {
    // M = D.T query tokens at positions q_pos0 .. q_pos0 + M - 1 = L - 1 (M = 1: plain decode). The score
    // rows span the last query's candidates (the most); every other query masks to its own.
    DecodePlan P{};
    const int M = D.T;
    const int pos = D.q_pos0 + M - 1;
    const int l = window_left(pos, D.W, D.S);
    P.n = l / D.S;
    const int bg = D.B * D.Hkv;
    P.per = kSliceElems / D.d;  // 128 rows at d 128
    P.nslices = P.n > 0 ? (P.n + P.per - 1) / P.per : 1;
    P.wtiles = 0;
    for (int m = 0; m < M; ++m) {
        const int pm = D.q_pos0 + m, lm = window_left(pm, D.W, D.S);
        P.wtiles = std::max(P.wtiles, (pm - lm + 1 + D.S - 1) / D.S);
    }
    P.ntiles = D.topk + P.wtiles;
    P.nparts = P.n > 0 ? (P.n + kSelPart - 1) / kSelPart : 1;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t at = off;
        off += (bytes + 255) & ~(size_t)255;
        return at;
    };
    P.off_scores = take((size_t)D.B * D.Hq * M * (P.n > 0 ? P.n : 1) * sizeof(float));
    P.off_part = take((size_t)D.B * D.Hq * M * P.nslices * kScorePartsPerSliceHost * 2 * sizeof(float));
    P.off_list = take((size_t)bg * M * P.nparts * D.topk * sizeof(uint64_t));
    P.off_sel = take((size_t)bg * M * D.topk * sizeof(int));
    P.off_attn = take((size_t)D.B * D.Hq * M * P.ntiles * (D.d + 4) * sizeof(float));  // either attention form
    P.off_count = take((size_t)bg * M * sizeof(unsigned int));
    P.off_selcount = take((size_t)bg * M * sizeof(unsigned int));
    P.total = off;
    return P;
}

// ---------------------------------------------------------------------------- 1. score

// Persistent, warp-specialised: one CTA per SM; lane 0 of the last warp keeps a ring of kStages slice
// copies in flight (one TMA bulk copy of P.per summary rows each: 32 KiB in bf16, 64 KiB in fp32).
// kWarpsPerSlot consumer warps share each ring slot, one row per lane. A unit is (b, h, slice); each
// consumer warp writes a partial (max, sum exp) of its rows, so a slice has kWarpsPerSlot partials.
template <typename T>
struct ScoreCfg {
    static constexpr int kStages = sizeof(T) == 2 ? 6 : 3;
    static constexpr int kWarpsPerSlot = 4;
    static constexpr int kConsumers = kStages * kWarpsPerSlot;
    static constexpr int kThreads = (kConsumers + 1) * 32;
    static constexpr int kQFloats = 16 * 12 + 32;  // per-warp q staging (padded chunks)
};

template <typename T>
__global__ void __launch_bounds__(ScoreCfg<T>::kThreads)
decode_score_kernel(Dims D, DecodePlan P, const T *__restrict__ q_hat, const T *__restrict__ k_sum,
                    const float *__restrict__ b_sum, float *__restrict__ scores, float *__restrict__ part,
                    unsigned int *__restrict__ clear, int nclear) {
    using C = ScoreCfg<T>;
    constexpr int NS = C::kStages, WPS = C::kWarpsPerSlot;
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[NS], empty[NS];
    const int d = D.d;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t slot_bytes = (size_t)P.per * d * sizeof(T);
    const int units = D.B * D.Hq * P.nslices;
    grid_dep_launch();  // the selection's CTAs may take SMs as this grid's CTAs finish
    // The later grids' counters start at zero: they read them only after this grid has completed (the
    // selection's griddepcontrol.wait or an ordinary launch; the attention through the selection's).
    if (blockIdx.x == 0)
        for (int i = tid; i < nclear; i += blockDim.x) clear[i] = 0u;
    if (tid == 0) {
        for (int i = 0; i < NS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], WPS);
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (warp == C::kConsumers) {
        if (lane == 0) {
            int k = 0;
            for (int u = blockIdx.x; u < units; u += gridDim.x, ++k) {
                const int slot = k % NS, round = k / NS;
                if (round > 0 && !mbar_wait_bounded(&empty[slot], (round - 1) & 1)) {
                    atomicOr(&g_decode_errors, 1u);
                    break;
                }
                const int sl = u % P.nslices;
                const size_t hrow = (size_t)(u / P.nslices);
                const int c0 = sl * P.per;
                const int R = min(P.n, c0 + P.per) - c0;
                const uint32_t bytes = (uint32_t)(R * d * sizeof(T));
                mbar_arrive_expect_tx(&full[slot], bytes);
                bulk_g2s(smem_raw + slot * slot_bytes, k_sum + (hrow * D.Nc + c0) * d, bytes, &full[slot]);
            }
        }
        return;
    }
    // Consumer warp: ring slot `slot`, quarter `qw` of the slot's rows (rows qw*32 + lane + 128*i).
    // Rows are read in 16-byte chunks in a lane-rotated order (chunk (k + lane) mod NCH at step k), so
    // the 8 lanes of a shared-memory phase hit 8 distinct bank groups; q^ (tau folded) is staged per
    // warp as fp32 chunks with a padded stride.
    constexpr int EC = 16 / sizeof(T);       // elements per 16-byte chunk
    constexpr int QS = (EC == 8) ? 12 : EC;  // padded fp32 stride of one q chunk
    const int NCH = d / EC;
    const int slot = warp / WPS, qw = warp % WPS;
    const T *rows = reinterpret_cast<const T *>(smem_raw + slot * slot_bytes);
    float *qsm = reinterpret_cast<float *>(smem_raw + NS * slot_bytes) + warp * C::kQFloats;
    constexpr int RPL = kSliceElems / 64 / (32 * WPS);  // rows per lane at d 64 (upper bound): 2
    float nq[4], nb[RPL];
    auto rows_of = [&](int u, int &c0, int &R, size_t &hrow, int &sl) {
        sl = u % P.nslices;
        hrow = (size_t)(u / P.nslices);
        c0 = sl * P.per;
        R = min(P.n, c0 + P.per) - c0;
    };
    auto prefetch = [&](int u) {
        if (u >= units) return;
        int c0, R, sl;
        size_t hrow;
        rows_of(u, c0, R, hrow, sl);
#pragma unroll
        for (int i = 0; i < 4; ++i) nq[i] = (lane + 32 * i < d) ? to_f(q_hat[hrow * d + lane + 32 * i]) : 0.f;
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            const int r = qw * 32 + lane + 32 * WPS * i;
            nb[i] = (r < R) ? b_sum[hrow * D.Nc + c0 + r] : 0.f;
        }
    };
    int k = slot;
    prefetch(blockIdx.x + slot * gridDim.x);
    for (int u = blockIdx.x + slot * gridDim.x; u < units; u += NS * gridDim.x, k += NS) {
        const int round = k / NS;
        int c0, R, sl;
        size_t hrow;
        rows_of(u, c0, R, hrow, sl);
        float bcur[RPL];
#pragma unroll
        for (int i = 0; i < RPL; ++i) bcur[i] = nb[i];
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = lane + 32 * i;
            if (e < d) qsm[(e / EC) * QS + (e % EC)] = nq[i] * D.tau;
        }
        __syncwarp();
        prefetch(u + NS * gridDim.x);  // overlaps this unit's wait and compute
        if (!mbar_wait_bounded(&full[slot], round & 1)) {
            if (lane == 0) atomicOr(&g_decode_errors, 1u);
            return;
        }
        float acc[RPL];
#pragma unroll
        for (int i = 0; i < RPL; ++i) acc[i] = 0.f;
#pragma unroll 4
        for (int kk = 0; kk < NCH; ++kk) {
            const int ch = (kk + lane) & (NCH - 1);
            float qv[EC];
#pragma unroll
            for (int e = 0; e < EC; e += 4) {
                const float4 q4 = *reinterpret_cast<const float4 *>(qsm + ch * QS + e);
                qv[e] = q4.x; qv[e + 1] = q4.y; qv[e + 2] = q4.z; qv[e + 3] = q4.w;
            }
#pragma unroll
            for (int i = 0; i < RPL; ++i) {
                const int r = qw * 32 + lane + 32 * WPS * i;
                if (r < R) {
                    float f[EC];
                    if (EC == 8) {
                        load8(reinterpret_cast<const __nv_bfloat16 *>(rows) + (size_t)r * d + ch * EC, f);
                    } else {
                        const float4 v4 = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(rows) +
                                                                            (size_t)r * d + ch * EC);
                        f[0] = v4.x; f[1] = v4.y; f[2] = v4.z; f[3] = v4.w;
                    }
#pragma unroll
                    for (int e = 0; e < EC; ++e) acc[i] = fmaf(f[e], qv[e], acc[i]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);  // this warp is done with the slot
        float m = -INFINITY, z = 0.f;
        float *sch = scores + hrow * P.n + c0;
#pragma unroll
        for (int i = 0; i < RPL; ++i) {
            const int r = qw * 32 + lane + 32 * WPS * i;
            if (r < R) {
                const float sc = acc[i] + bcur[i];
                sch[r] = sc;
                if (sc > m) {
                    z = z * __expf(m - sc) + 1.f;
                    m = sc;
                } else {
                    z += __expf(sc - m);
                }
            }
        }
        const float M = warp_max(m);
        float Z = (m > -INFINITY) ? z * __expf(m - M) : 0.f;
        Z = warp_sum(Z);
        if (lane == 0) {
            float *pp = part + ((hrow * P.nslices + sl) * kScorePartsPerSliceHost + qw) * 2;
            pp[0] = M;
            pp[1] = Z;
        }
    }
}

// ---------------------------------------------------------------------------- 2. select

// Grid (parts, Hkv, B): each CTA owns kSelPart candidates of one group. It folds the per-head score
// partials into LSE_h, forms 64-bit keys (group score desc, chunk id asc; all distinct), keeps its
// local top-k by a shared-memory bitonic sort and writes them to the workspace. The last CTA of the
// group to finish (an atomic counter, no waiting) sorts the parts' lists and writes the group's top-k.
// Exact: every member of the group's top-k is in its own part's top-k.
__global__ void __launch_bounds__(kSelThreads)
decode_select_kernel(Dims D, DecodePlan P, const float *__restrict__ scores, const float *__restrict__ part,
                     uint64_t *__restrict__ lists, unsigned int *__restrict__ counters, int *__restrict__ sel,
                     int *__restrict__ idx_out) {
    __shared__ float lse[64];
    __shared__ __align__(8) uint64_t keys[kSelMerge];
    __shared__ int s_last;
    const int pidx = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int G = D.G, K = D.topk, n = P.n;
    const size_t bg = (size_t)b * D.Hkv + g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    grid_dep_wait();  // the score grid's scores and partials
    int *out = sel + bg * K;
    int *out2 = idx_out ? idx_out + bg * K : nullptr;
    if (n == 0) {
        for (int t = tid; t < K; t += blockDim.x) {
            out[t] = -1;
            if (out2) out2[t] = -1;
        }
        return;
    }
    // Raw scores of this thread's candidates for the first kSelHeadsInFlight heads are loaded before
    // the LSE fold, so both global round trips overlap.
    const int c0 = pidx * kSelPart;
    const float *sc0 = scores + ((size_t)b * D.Hq + g * G) * n;
    constexpr int PER = kSelPart / kSelThreads;
    float raw[kSelHeadsInFlight][PER];
#pragma unroll
    for (int hh = 0; hh < kSelHeadsInFlight; ++hh)
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int c = c0 + i * blockDim.x + tid;
            raw[hh][i] = (hh < G && c < n) ? sc0[(size_t)hh * n + c] : -INFINITY;
        }
    for (int hh = warp; hh < G; hh += nwarps) {
        // online merge of the head's partials: each lane folds its entries, then the warp folds lanes
        const int np = P.nslices * kScorePartsPerSliceHost;
        const float2 *ph = reinterpret_cast<const float2 *>(part + ((size_t)b * D.Hq + g * G + hh) * np * 2);
        float M = -INFINITY, Z = 0.f;
        for (int s0 = 0; s0 < np; s0 += 32 * 8) {
            float2 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int si = s0 + u * 32 + lane;
                v[u] = (si < np) ? ph[si] : make_float2(-INFINITY, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (v[u].x > M) {
                    Z = Z * __expf(M - v[u].x) + v[u].y;
                    M = v[u].x;
                } else if (v[u].x > -INFINITY) {
                    Z += v[u].y * __expf(v[u].x - M);
                }
            }
        }
        const float MM = warp_max(M);
        Z = (M > -INFINITY) ? Z * __expf(M - MM) : 0.f;
        Z = warp_sum(Z);
        if (lane == 0) lse[hh] = MM + logf(Z);
    }
    __syncthreads();
    float gv[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) gv[i] = -INFINITY;
#pragma unroll
    for (int hh = 0; hh < kSelHeadsInFlight; ++hh) {
        if (hh < G) {
            const float l = lse[hh];
#pragma unroll
            for (int i = 0; i < PER; ++i) gv[i] = fmaxf(gv[i], raw[hh][i] - l);
        }
    }
    for (int hh = kSelHeadsInFlight; hh < G; ++hh) {  // groups wider than kSelHeadsInFlight heads
        const float l = lse[hh];
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const int c = c0 + i * blockDim.x + tid;
            if (c < n) gv[i] = fmaxf(gv[i], sc0[(size_t)hh * n + c] - l);
        }
    }
    // Each warp sorts its 32*PER keys in registers and offers its best min(K, 32*PER) to shared memory.
    uint64_t kv[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int c = c0 + i * blockDim.x + tid;
        kv[i] = (c < n) ? desc_value_key(gv[i], (uint32_t)c) : ~0ull;
    }
    warp_bitonic_sort<PER>(kv);
    const int KW = min(K, 32 * PER);  // survivors per warp
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = lane * PER + i;
        if (e < KW) keys[warp * KW + e] = kv[i];
    }
    __syncthreads();
    uint64_t *mine = lists + (bg * P.nparts + pidx) * K;
    {
        // Warp 0 sorts the nwarps*KW survivors (<= 256 = 32 x 8) and writes this part's top-K; more
        // survivors (topk > 32) take the block-wide sort.
        const int E1 = nwarps * KW;
        if (E1 > 256) {
            const int epad = next_pow2(E1);
            for (int e = E1 + tid; e < epad; e += blockDim.x) keys[e] = ~0ull;
            block_bitonic_sort(keys, epad);
            for (int e = tid; e < K; e += blockDim.x) mine[e] = keys[e];
        } else if (warp == 0) {
            uint64_t w8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = lane * 8 + i;
                w8[i] = (e < E1) ? keys[e] : ~0ull;
            }
            warp_bitonic_sort<8>(w8);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = lane * 8 + i;
                if (e < K) mine[e] = w8[i];
            }
        }
    }
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        s_last = (atomicAdd(&counters[bg], 1u) == (unsigned)(P.nparts - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const int E = P.nparts * K;
    if (E <= 256) {
        if (warp == 0) {
            uint64_t w8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = lane * 8 + i;
                w8[i] = (e < E) ? __ldcg(lists + bg * P.nparts * K + e) : ~0ull;
            }
            warp_bitonic_sort<8>(w8);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = lane * 8 + i;
                if (e < K) keys[e] = w8[i];
            }
        }
        __syncthreads();
    } else {
        const int epad = next_pow2(E);
        for (int e = tid; e < epad; e += blockDim.x) keys[e] = (e < E) ? __ldcg(lists + bg * P.nparts * K + e) : ~0ull;
        block_bitonic_sort(keys, epad);
    }
    const int kk = min(K, n);
    for (int t = tid; t < K; t += blockDim.x) {
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

// Lane l receives element l of a warp-sorted sequence of 32*NPL keys (element e at lane e / NPL,
// slot e % NPL): the 32 smallest, one per lane, ascending.
template <int NPL>
__device__ __forceinline__ uint64_t warp_first32(const uint64_t (&v)[NPL]) {
    const int lane = threadIdx.x & 31;
    uint64_t mine = ~0ull;
#pragma unroll
    for (int s = 0; s < NPL; ++s) {
        const uint32_t lo = __shfl_sync(0xffffffffu, (uint32_t)v[s], lane / NPL);
        const uint32_t hi = __shfl_sync(0xffffffffu, (uint32_t)(v[s] >> 32), lane / NPL);
        if (lane % NPL == s) mine = ((uint64_t)hi << 32) | lo;
    }
    return mine;
}

// The 32 smallest of two ascending one-per-lane lists, ascending: min(a_l, b_{31-l}) is bitonic, then a
// bitonic merge.
__device__ __forceinline__ uint64_t warp_merge_lowest32(uint64_t a, uint64_t b) {
    const int lane = threadIdx.x & 31;
    const uint32_t blo = __shfl_sync(0xffffffffu, (uint32_t)b, 31 - lane);
    const uint32_t bhi = __shfl_sync(0xffffffffu, (uint32_t)(b >> 32), 31 - lane);
    const uint64_t br = ((uint64_t)bhi << 32) | blo;
    uint64_t v = a < br ? a : br;
#pragma unroll
    for (int st = 16; st > 0; st >>= 1) {
        const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, st);
        const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), st);
        const uint64_t p = ((uint64_t)hi << 32) | lo;
        v = ((lane & st) == 0) ? (v < p ? v : p) : (v > p ? v : p);
    }
    return v;
}

// Slow path of the single-CTA selection, kept out of line so that its code is fetched only when used
// (massively tied scores overflow the survivor buffer): every warp keeps a running top-32 of its
// candidates, merged in registers batch by batch, and the CTA reduces the warps' lists. Returns the 32
// smallest keys, ascending, to warp 0 (one per lane).
template <int GM>
__device__ __noinline__ uint64_t select_tied_fallback(const float *__restrict__ sc0, size_t hs, int G, int n,
                                                      int rounds, const float (&L)[8], uint64_t *keys) {
    constexpr int kPer = 64 / GM, kRound = 512 * kPer;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    uint64_t best = ~0ull;
    for (int r = 0; r < rounds; ++r) {
        for (int h = 0; h < kPer / 8; ++h) {
            uint64_t kv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int c = r * kRound + warp * (32 * kPer) + (h * 8 + i) * 32 + lane;
                float gv = -INFINITY;
                for (int hh = 0; hh < G; ++hh) gv = fmaxf(gv, (c < n ? sc0[hh * hs + c] : -INFINITY) - L[hh]);
                kv[i] = (c < n) ? desc_value_key(gv, (uint32_t)c) : ~0ull;
            }
            warp_bitonic_sort<8>(kv);
            best = warp_merge_lowest32(best, warp_first32<8>(kv));
        }
    }
    __syncthreads();
    keys[warp * 32 + lane] = best;
    for (int span = 1; span < nwarps; span <<= 1) {
        __syncthreads();
        uint64_t m = ~0ull;
        const bool act = (warp % (2 * span)) == 0 && warp + span < nwarps;
        if (act) m = warp_merge_lowest32(keys[warp * 32 + lane], keys[(warp + span) * 32 + lane]);
        __syncthreads();
        if (act) keys[warp * 32 + lane] = m;
    }
    __syncthreads();
    return warp == 0 ? keys[lane] : ~0ull;
}

// Single-CTA selection of one (b, KV group) for topk <= 32 and G <= 8. Keys as in the multi-CTA form
// (group score desc, chunk id asc; all distinct), so the same ids.
//  1. per-head LSE folded from the score kernel's slice partials; group keys of every candidate, and
//     each thread's best (smallest) key;
//  2. bound: the 32nd smallest of the 512 per-thread best keys. At least 32 candidates (one per
//     thread holding those keys) are at or below it, so the 32 smallest keys overall all are too;
//  3. the candidates at or below the bound (about 32-50 on any non-degenerate scores) are compacted
//     into shared memory and sorted by one warp; their first k are the selection.
// When the survivors overflow the buffer (massively tied scores) select_tied_fallback takes over.
// GM: heads held per candidate (4 or 8); a thread keeps 64 raw scores in flight per round.
constexpr int kSelWThreads = 512;
constexpr int kSelWCap = 128;  // survivor buffer (sorted by one warp, 4 keys per lane)

template <int GM>
__global__ void __launch_bounds__(kSelWThreads)
decode_select_warp_kernel(Dims D, DecodePlan P, const float *__restrict__ scores, const float *__restrict__ part,
                          int *__restrict__ sel, int *__restrict__ idx_out) {
    __shared__ float lse[8];
    __shared__ __align__(8) uint64_t keys[kSelWThreads];
    __shared__ __align__(8) uint64_t surv[kSelWCap];
    __shared__ int sel_ids[32];
    __shared__ uint64_t s_bound;
    __shared__ int s_count;
    // grid (Hkv, B * M): query m of sequence b; its candidates are the chunks before its window
    const int g = blockIdx.x, M = D.T, b = blockIdx.y / M, m = blockIdx.y % M;
    const int G = D.G, K = D.topk;
    const int n = window_left(D.q_pos0 + m, D.W, D.S) / D.S;
    const size_t bgm = ((size_t)b * D.Hkv + g) * M + m;
    // the attention grid may start now: its CTAs load and fold their window tiles while this grid selects
    grid_dep_launch();
    grid_dep_wait();  // the score grid's scores and partials
    const size_t hs = (size_t)M * P.n;  // stride between the group's heads in the score rows
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = kSelWThreads / 32;
    int *out = sel + bgm * K;
    int *out2 = idx_out ? idx_out + bgm * K : nullptr;
    if (n == 0) {
        for (int t = tid; t < K; t += blockDim.x) {
            out[t] = -1;
            if (out2) out2[t] = -1;
        }
        return;
    }
    const float *sc0 = scores + (((size_t)b * D.Hq + g * G) * M + m) * P.n;
    constexpr int kSelWPer = 64 / GM;                     // candidates per thread per round
    constexpr int kSelWRound = kSelWThreads * kSelWPer;
    const int rounds = (n + kSelWRound - 1) / kSelWRound;
    // candidate of (round r, slot i) for this thread, coalesced across the warp. A list shorter than half
    // a round is spread over all threads, so that every thread holds its own best key (held by a few warps
    // it would leave the 32nd-best bound loose and overflow the survivor buffer); longer lists give each
    // warp a contiguous block per round (eight or more warps then hold candidates).
    const bool spread = n < kSelWRound / 2;
    auto cand = [&](int r, int i) {
        return spread ? i * kSelWThreads + tid : r * kSelWRound + warp * (32 * kSelWPer) + i * 32 + lane;
    };
    float raw[GM][kSelWPer];
    auto load_round = [&](int r) {
#pragma unroll
        for (int hh = 0; hh < GM; ++hh)
#pragma unroll
            for (int i = 0; i < kSelWPer; ++i) {
                const int c = cand(r, i);
                raw[hh][i] = (hh < G && c < n) ? sc0[hh * hs + c] : -INFINITY;
            }
    };
    load_round(0);  // in flight during the LSE fold
    if (tid == 0) s_count = 0;
    if (warp < G) {
        const int hh = warp;
        const int np = P.nslices * kScorePartsPerSliceHost;
        const float2 *ph = reinterpret_cast<const float2 *>(part + (((size_t)b * D.Hq + g * G + hh) * M + m) * np * 2);
        float M = -INFINITY, Z = 0.f;
        for (int s0 = 0; s0 < np; s0 += 32 * 8) {
            float2 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int si = s0 + u * 32 + lane;
                v[u] = (si < np) ? ph[si] : make_float2(-INFINITY, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (v[u].x > M) {
                    Z = Z * __expf(M - v[u].x) + v[u].y;
                    M = v[u].x;
                } else if (v[u].x > -INFINITY) {
                    Z += v[u].y * __expf(v[u].x - M);
                }
            }
        }
        const float MM = warp_max(M);
        Z = (M > -INFINITY) ? Z * __expf(M - MM) : 0.f;
        Z = warp_sum(Z);
        if (lane == 0) lse[hh] = MM + logf(Z);
    }
    __syncthreads();
    float L[8];
#pragma unroll
    for (int hh = 0; hh < 8; ++hh) L[hh] = hh < G ? lse[hh] : 0.f;
    auto key_of = [&](int r, int i) -> uint64_t {
        const int c = cand(r, i);
        float gv = -INFINITY;
#pragma unroll
        for (int hh = 0; hh < GM; ++hh)
            if (hh < G) gv = fmaxf(gv, raw[hh][i] - L[hh]);
        return (c < n) ? desc_value_key(gv, (uint32_t)c) : ~0ull;
    };

    // 1. each thread's best key
    uint64_t mine = ~0ull;
    for (int r = 0; r < rounds; ++r) {
        if (r > 0) load_round(r);
#pragma unroll
        for (int i = 0; i < kSelWPer; ++i) {
            const uint64_t k = key_of(r, i);
            mine = k < mine ? k : mine;
        }
    }
    // 2. the 32nd smallest of the per-thread best keys: sort within each warp, then merge the warps'
    //    ascending lists pairwise
    {
        uint64_t one[1] = {mine};
        warp_bitonic_sort<1>(one);
        keys[warp * 32 + lane] = one[0];
    }
    for (int span = 1; span < nwarps; span <<= 1) {
        __syncthreads();
        uint64_t m = ~0ull;
        const bool act = (warp % (2 * span)) == 0 && warp + span < nwarps;
        if (act) m = warp_merge_lowest32(keys[warp * 32 + lane], keys[(warp + span) * 32 + lane]);
        __syncthreads();
        if (act) keys[warp * 32 + lane] = m;
    }
    __syncthreads();
    if (tid == 0) s_bound = keys[31];
    __syncthreads();
    const uint64_t bound = s_bound;
    // 3. compact the candidates at or below the bound (scores reloaded when they did not fit one round)
    for (int r = 0; r < rounds; ++r) {
        if (rounds > 1) load_round(r);
#pragma unroll
        for (int i = 0; i < kSelWPer; ++i) {
            const uint64_t k = key_of(r, i);
            const bool take = k <= bound && k != ~0ull;  // (padding slots never qualify)
            const unsigned m = __ballot_sync(0xffffffffu, take);
            if (m) {
                int base = 0;
                if (lane == 0) base = atomicAdd(&s_count, __popc(m));
                base = __shfl_sync(0xffffffffu, base, 0);
                const int at = base + __popc(m & ((1u << lane) - 1));
                if (take && at < kSelWCap) surv[at] = k;
            }
        }
    }
    __syncthreads();
    const int count = s_count;
    const int kk = min(K, n);
    if (count <= kSelWCap) {
        // The keys are distinct: a survivor's rank is the number of smaller survivors (one thread each,
        // every read a shared-memory broadcast). The kk best go to sel_ids in score order; then each of
        // those ids is ranked among them and written in ascending order.
        if (tid < count) {
            const uint64_t k = surv[tid];
            int rank = 0;
            for (int j = 0; j < count; ++j) rank += surv[j] < k ? 1 : 0;
            if (rank < kk) sel_ids[rank] = (int)desc_key_index(k);
        }
        __syncthreads();
        if (tid < K) {
            int v = -1;
            if (tid < kk) {
                const int id = sel_ids[tid];
                int r2 = 0;
                for (int j = 0; j < kk; ++j) r2 += sel_ids[j] < id ? 1 : 0;
                out[r2] = id;
                if (out2) out2[r2] = id;
            } else {
                out[tid] = v;
                if (out2) out2[tid] = v;
            }
        }
        return;
    }
    uint64_t top = select_tied_fallback<GM>(sc0, hs, G, n, rounds, L, keys);  // warp 0: keys ascending
    if (warp == 0) {
        // the selected ids (first kk keys), written ascending, -1 padded
        uint64_t ids[1] = {(lane < kk && top != ~0ull) ? (uint64_t)desc_key_index(top) : ~0ull};
        warp_bitonic_sort<1>(ids);
        if (lane < K) {
            const int v = ids[0] == ~0ull ? -1 : (int)ids[0];
            out[lane] = v;
            if (out2) out2[lane] = v;
        }
    }
}

// Short candidate lists (n <= 2048, topk <= 32, G <= GM): one CTA of eight warps per (b, KV group, query)
// with every memory read issued up front. Warp w holds candidates [256w, 256w + 256), eight a lane; the
// per-head LSE is folded from the score kernel's slice partials as in the kernel above; each warp sorts
// its 256 keys in registers and keeps the best 32, and warp 0 merges the warps' lists. Same keys as the
// kernel above (group score desc, chunk id asc), so the same ids; about a third of its latency on short
// lists, whose cost was its phases' barriers and round trips rather than the candidates.
constexpr int kSelSThreads = 256;
constexpr int kSelSNpl = 8;
constexpr int kSelSMax = kSelSThreads * kSelSNpl;

template <int GM>
__global__ void __launch_bounds__(kSelSThreads, 1)
decode_select_short_kernel(Dims D, DecodePlan P, const float *__restrict__ scores, const float *__restrict__ part,
                           int *__restrict__ sel, int *__restrict__ idx_out) {
    __shared__ float lse[8];
    __shared__ __align__(8) uint64_t lists[kSelSThreads / 32][32];
    const int g = blockIdx.x, M = D.T, b = blockIdx.y / M, m = blockIdx.y % M;
    const int G = D.G, K = D.topk;
    const int n = window_left(D.q_pos0 + m, D.W, D.S) / D.S;
    const size_t bgm = ((size_t)b * D.Hkv + g) * M + m;
    // the attention grid may start now: its CTAs load and fold their window tiles while this grid selects
    grid_dep_launch();
    grid_dep_wait();  // the score grid's scores and partials
    const size_t hs = (size_t)M * P.n;  // stride between the group's heads in the score rows
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int *out = sel + bgm * K;
    int *out2 = idx_out ? idx_out + bgm * K : nullptr;
    if (n == 0) {
        for (int t = tid; t < K; t += blockDim.x) {
            out[t] = -1;
            if (out2) out2[t] = -1;
        }
        return;
    }
    const float *sc0 = scores + (((size_t)b * D.Hq + g * G) * M + m) * P.n;
    float raw[GM][kSelSNpl];
#pragma unroll
    for (int hh = 0; hh < GM; ++hh)
#pragma unroll
        for (int i = 0; i < kSelSNpl; ++i) {
            const int c = warp * 32 * kSelSNpl + i * 32 + lane;
            raw[hh][i] = (hh < G && c < n) ? sc0[hh * hs + c] : -INFINITY;
        }
    if (warp < G) {
        const int hh = warp;
        const int np = P.nslices * kScorePartsPerSliceHost;
        const float2 *ph = reinterpret_cast<const float2 *>(part + (((size_t)b * D.Hq + g * G + hh) * M + m) * np * 2);
        float Mx = -INFINITY, Z = 0.f;
        for (int s0 = 0; s0 < np; s0 += 32 * 8) {
            float2 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int si = s0 + u * 32 + lane;
                v[u] = (si < np) ? ph[si] : make_float2(-INFINITY, 0.f);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (v[u].x > Mx) {
                    Z = Z * __expf(Mx - v[u].x) + v[u].y;
                    Mx = v[u].x;
                } else if (v[u].x > -INFINITY) {
                    Z += v[u].y * __expf(v[u].x - Mx);
                }
            }
        }
        const float MM = warp_max(Mx);
        Z = (Mx > -INFINITY) ? Z * __expf(Mx - MM) : 0.f;
        Z = warp_sum(Z);
        if (lane == 0) lse[hh] = MM + logf(Z);
    }
    __syncthreads();
    float L[GM];
#pragma unroll
    for (int hh = 0; hh < GM; ++hh) L[hh] = hh < G ? lse[hh] : 0.f;
    uint64_t kv[kSelSNpl];
#pragma unroll
    for (int i = 0; i < kSelSNpl; ++i) {
        const int c = warp * 32 * kSelSNpl + i * 32 + lane;
        float gv = -INFINITY;
#pragma unroll
        for (int hh = 0; hh < GM; ++hh)
            if (hh < G) gv = fmaxf(gv, raw[hh][i] - L[hh]);
        kv[i] = (c < n) ? desc_value_key(gv, (uint32_t)c) : ~0ull;
    }
    const int nwarps = (n + 32 * kSelSNpl - 1) / (32 * kSelSNpl);  // warps holding candidates
    if (warp < nwarps) {
        warp_bitonic_sort<kSelSNpl>(kv);
        lists[warp][lane] = warp_first32<kSelSNpl>(kv);
    }
    __syncthreads();
    if (warp == 0) {
        uint64_t top = lists[0][lane];
        for (int w = 1; w < nwarps; ++w) top = warp_merge_lowest32(top, lists[w][lane]);
        // the selected ids (first min(K, n) keys), written ascending, -1 padded
        const int kk = min(K, n);
        uint64_t ids[1] = {(lane < kk && top != ~0ull) ? (uint64_t)desc_key_index(top) : ~0ull};
        warp_bitonic_sort<1>(ids);
        if (lane < K) {
            const int v = ids[0] == ~0ull ? -1 : (int)ids[0];
            out[lane] = v;
            if (out2) out2[lane] = v;
        }
    }
}

// ---------------------------------------------------------------------------- 3. attend (+ combine)

template <typename T, int DPL>
__global__ void __launch_bounds__(kAttnThreads)
decode_attn_kernel(Dims D, DecodePlan P, const T *__restrict__ q, const T *__restrict__ kc,
                   const T *__restrict__ vc, const float *__restrict__ scores, const int *__restrict__ sel,
                   float *__restrict__ partial, unsigned int *__restrict__ counters, T *__restrict__ out,
                   float *__restrict__ lse) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t bar;
    __shared__ int s_last;
    const int t = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int d = D.d, S = D.S, G = D.G;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
    const size_t bg = (size_t)b * D.Hkv + g;
    const int pos = D.L - 1;
    const int l = window_left(pos, D.W, S);
    T *ks = reinterpret_cast<T *>(smem_raw);                    // [S][d]
    T *vs = ks + (size_t)S * d;                                 // [S][d]
    float *ws = reinterpret_cast<float *>(vs + (size_t)S * d);  // [G][S] logits, then weights
    constexpr int EC = 16 / sizeof(T);        // elements per 16-byte chunk
    constexpr int QS = (EC == 8) ? 12 : EC;   // padded fp32 stride of one q chunk
    const int NCH = d / EC;
    float *qs = ws + ((G * S + 3) & ~3);      // [G][NCH][QS] q chunks, tau folded (16-byte aligned)
    float *shat = qs + G * NCH * QS;          // [G] retrieval scores of the tile's chunk
    float *half = shat + ((G + 3) & ~3);      // [2G][32][DPL] value-product halves

    int c = -1, j0 = 0, jn = 0;
    if (t < D.topk) {
        c = sel[bg * D.topk + t];
        if (c >= 0) { j0 = c * S; jn = S; }
    } else {
        j0 = l + (t - D.topk) * S;
        jn = min(S, pos + 1 - j0);
    }
    bool ok = true;
    if (jn > 0) {
        const uint32_t bytes = (uint32_t)(jn * d * sizeof(T));
        if (tid == 0) {
            mbar_init(&bar, 1);
            fence_mbar_init();
        }
        __syncthreads();
        if (tid == 0) {
            mbar_arrive_expect_tx(&bar, 2 * bytes);
            bulk_g2s(ks, kc + (bg * D.L + j0) * d, bytes, &bar);
            bulk_g2s(vs, vc + (bg * D.L + j0) * d, bytes, &bar);
        }
        for (int e = tid; e < G * d; e += blockDim.x) {
            const int hh = e / d, x = e % d;
            qs[(hh * NCH + x / EC) * QS + x % EC] = to_f(q[((size_t)b * D.Hq + g * G) * d + e]) * D.tau;
        }
        if (c >= 0)  // the chunk's retrieval score per head, fetched while the tile is in flight
            for (int hh = tid; hh < G; hh += blockDim.x) shat[hh] = scores[((size_t)b * D.Hq + g * G + hh) * P.n + c];
        ok = mbar_wait_bounded(&bar, 0);
        if (!ok && tid == 0) atomicOr(&g_decode_errors, 1u);
        __syncthreads();
    }
    if (jn > 0 && ok) {
        // Logits: one (token j, head) item per thread; K chunks read in a token-rotated order so the 8
        // lanes of a shared-memory phase hit distinct bank groups.
        for (int e = tid; e < G * S; e += blockDim.x) {
            const int j = e % S, hh = e / S;
            float acc = -INFINITY;
            if (j < jn) {
                float acc2 = 0.f;  // second chain halves the dependent-FMA latency
                acc = 0.f;
                const float *qh = qs + hh * NCH * QS;
#pragma unroll 4
                for (int kk = 0; kk < NCH; ++kk) {
                    const int ch = (kk + j) & (NCH - 1);
                    float f[EC];
                    if (EC == 8) {
                        load8(reinterpret_cast<const __nv_bfloat16 *>(ks) + (size_t)j * d + ch * EC, f);
                    } else {
                        const float4 v4 = *reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(ks) +
                                                                            (size_t)j * d + ch * EC);
                        f[0] = v4.x; f[1] = v4.y; f[2] = v4.z; f[3] = v4.w;
                    }
#pragma unroll
                    for (int x = 0; x < EC; x += 4) {
                        const float4 q4 = *reinterpret_cast<const float4 *>(qh + ch * QS + x);
                        acc = fmaf(f[x], q4.x, acc);
                        acc2 = fmaf(f[x + 1], q4.y, acc2);
                        acc = fmaf(f[x + 2], q4.z, acc);
                        acc2 = fmaf(f[x + 3], q4.w, acc2);
                    }
                }
                acc += acc2;
            }
            ws[hh * S + j] = acc;
        }
        __syncthreads();
        for (int hh = warp; hh < G; hh += nwarps) {
            float mx = -INFINITY;
            for (int j = lane; j < S; j += 32) mx = fmaxf(mx, ws[hh * S + j]);
            mx = warp_max(mx);
            float z = 0.f;
            for (int j = lane; j < S; j += 32) {
                const float e = __expf(ws[hh * S + j] - mx);  // padding: exp(-inf) = 0
                ws[hh * S + j] = e;
                z += e;
            }
            z = warp_sum(z);
            // Chunk tile: tokens carry exp(s_j - L_c + s^_c); relative to m = s^_c - log z their weights
            // are exp(s_j - mx) and sum to z. Window tile: m = mx.
            if (lane == 0) {
                float *pp = partial + (((size_t)b * D.Hq + g * G + hh) * P.ntiles + t) * (d + 2);
                pp[0] = (c >= 0) ? shat[hh] - logf(z) : mx;
                pp[1] = z;
            }
        }
        __syncthreads();
        // Value product: (head, half of the tokens) per warp, lane owns DPL dims; halves meet in smem.
        for (int wk = warp; wk < 2 * G; wk += nwarps) {
            const int hh = wk >> 1, hf = wk & 1;
            const int jb = hf * ((jn + 1) / 2), je = hf ? jn : (jn + 1) / 2;
            float acc[DPL], acc2[DPL];
#pragma unroll
            for (int u = 0; u < DPL; ++u) { acc[u] = 0.f; acc2[u] = 0.f; }
            int j = jb;
            for (; j + 1 < je; j += 2) {
                const float w0 = ws[hh * S + j], w1 = ws[hh * S + j + 1];
#pragma unroll
                for (int u = 0; u < DPL; ++u) {
                    acc[u] = fmaf(w0, to_f(vs[(size_t)j * d + lane * DPL + u]), acc[u]);
                    acc2[u] = fmaf(w1, to_f(vs[(size_t)(j + 1) * d + lane * DPL + u]), acc2[u]);
                }
            }
            if (j < je) {
                const float w0 = ws[hh * S + j];
#pragma unroll
                for (int u = 0; u < DPL; ++u) acc[u] = fmaf(w0, to_f(vs[(size_t)j * d + lane * DPL + u]), acc[u]);
            }
#pragma unroll
            for (int u = 0; u < DPL; ++u) half[(wk * 32 + lane) * DPL + u] = acc[u] + acc2[u];
        }
        __syncthreads();
        for (int e = tid; e < G * d; e += blockDim.x) {
            const int hh = e / d, x = e % d;
            const int ln = x / DPL, u = x % DPL;
            partial[(((size_t)b * D.Hq + g * G + hh) * P.ntiles + t) * (d + 2) + 2 + x] =
                half[((2 * hh) * 32 + ln) * DPL + u] + half[((2 * hh + 1) * 32 + ln) * DPL + u];
        }
    } else {
        for (int hh = tid; hh < G; hh += blockDim.x) {
            float *pp = partial + (((size_t)b * D.Hq + g * G + hh) * P.ntiles + t) * (d + 2);
            pp[0] = -INFINITY;
            pp[1] = 0.f;
        }
    }
    // The last tile of this (b, group) to finish merges all tiles' partials (no CTA waits on another).
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        s_last = (atomicAdd(&counters[bg], 1u) == (unsigned)(P.ntiles - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int hh = warp; hh < G; hh += nwarps) {
        const size_t bh = (size_t)b * D.Hq + g * G + hh;
        const float *ph = partial + bh * P.ntiles * (d + 2);
        float M = -INFINITY;
        for (int u = lane; u < P.ntiles; u += 32) M = fmaxf(M, __ldcg(ph + (size_t)u * (d + 2)));
        M = warp_max(M);
        float Z = 0.f;
        for (int u = lane; u < P.ntiles; u += 32) {
            const float mu = __ldcg(ph + (size_t)u * (d + 2));
            if (mu > -INFINITY) Z += __ldcg(ph + (size_t)u * (d + 2) + 1) * __expf(mu - M);
        }
        Z = warp_sum(Z);
        // tile weights exp(m_t - M), held by lane t % 32 (two registers for up to 64 tiles)
        float r0 = 0.f, r1 = 0.f;
        if (lane < P.ntiles) {
            const float mu = __ldcg(ph + (size_t)lane * (d + 2));
            r0 = (mu > -INFINITY) ? __expf(mu - M) : 0.f;
        }
        if (lane + 32 < P.ntiles) {
            const float mu = __ldcg(ph + (size_t)(lane + 32) * (d + 2));
            r1 = (mu > -INFINITY) ? __expf(mu - M) : 0.f;
        }
        float acc[DPL];
#pragma unroll
        for (int u = 0; u < DPL; ++u) acc[u] = 0.f;
#pragma unroll 8
        for (int tt = 0; tt < P.ntiles; ++tt) {
            const float r = __shfl_sync(0xffffffffu, tt < 32 ? r0 : r1, tt & 31);
#pragma unroll
            for (int u = 0; u < DPL; ++u) acc[u] = fmaf(__ldcg(ph + (size_t)tt * (d + 2) + 2 + lane * DPL + u), r, acc[u]);
        }
        const float inv = 1.f / Z;
#pragma unroll
        for (int u = 0; u < DPL; ++u) out[bh * d + lane * DPL + u] = from_f<T>(acc[u] * inv);
        if (lane == 0) lse[bh] = M + logf(Z);
    }
}

template <typename T, int DPL>
cudaError_t launch_t(const Dims &D, const void *q, const void *q_hat, const void *k_cache, const void *v_cache,
                     const void *k_sum, const float *b_sum, void *out, float *lse, int *idx_out, void *ws,
                     cudaStream_t stream) {
    const DecodePlan P = make_plan(D);
    unsigned char *w = (unsigned char *)ws;
    float *scores = (float *)(w + P.off_scores);
    float *part = (float *)(w + P.off_part);
    uint64_t *lists = (uint64_t *)(w + P.off_list);
    int *sel = (int *)(w + P.off_sel);
    float *partial = (float *)(w + P.off_attn);
    unsigned int *counters = (unsigned int *)(w + P.off_count);
    // Both counter arrays (attention, selection) are adjacent; the score grid clears them, and without
    // candidates (no score grid) one memset does.
    const int nclear = (int)((P.total - P.off_count) / sizeof(unsigned int));
    if (P.n == 0) {
        cudaError_t e = cudaMemsetAsync(counters, 0, P.total - P.off_count, stream);
        if (e != cudaSuccess) return e;
    }
    if (P.n > 0 && D.T > 1) {
        cudaError_t es = launch_decode_score_mma(D, P.n, P.nslices, q_hat, k_sum, b_sum, scores, part, counters,
                                                 nclear, stream);
        if (es != cudaSuccess) return es;
    } else if (P.n > 0) {
        using C = ScoreCfg<T>;
        static_assert(C::kWarpsPerSlot == kScorePartsPerSliceHost, "one partial per consumer warp of a slot");
        const size_t smem1 = (size_t)C::kStages * P.per * D.d * sizeof(T) +
                             (size_t)C::kConsumers * C::kQFloats * sizeof(float);
        auto k1 = decode_score_kernel<T>;
        cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
        const int units = D.B * D.Hq * P.nslices;
        const int sms = num_sms();
        const int grid = units < sms ? units : sms;
        k1<<<grid, ScoreCfg<T>::kThreads, smem1, stream>>>(D, P, (const T *)q_hat, (const T *)k_sum, b_sum, scores,
                                                           part, counters, nclear);
    }
    unsigned int *selcount = (unsigned int *)(w + P.off_selcount);
    // One CTA per (b, KV group, query) selects the top-k of a whole candidate list. With few groups and a
    // long list (a few sequences over a cache of a million tokens or more) that leaves most SMs idle: the
    // list is then split over ceil(n / 1024) CTAs per group whose top-k lists the last CTA merges.
    // (Measured at B1: 8184 candidates faster on one CTA, 16376 and more faster split.)
    const bool wide = D.T == 1 && D.B * D.Hkv < 32 && P.n >= 12288 && next_pow2(P.nparts * D.topk) <= kSelMerge;
    cudaError_t es;
    if (!wide && D.topk <= 32 && P.n <= kSelSMax && D.G <= 4)
        es = launch_pdl(decode_select_short_kernel<4>, dim3(D.Hkv, D.B * D.T), dim3(kSelSThreads), 0, stream, D, P,
                        (const float *)scores, (const float *)part, sel, idx_out);
    else if (!wide && D.topk <= 32 && P.n <= kSelSMax && D.G <= 8)
        es = launch_pdl(decode_select_short_kernel<8>, dim3(D.Hkv, D.B * D.T), dim3(kSelSThreads), 0, stream, D, P,
                        (const float *)scores, (const float *)part, sel, idx_out);
    else if (!wide && D.topk <= 32 && D.G <= 4)
        es = launch_pdl(decode_select_warp_kernel<4>, dim3(D.Hkv, D.B * D.T), dim3(kSelWThreads), 0, stream, D, P,
                        (const float *)scores, (const float *)part, sel, idx_out);
    else if (!wide && D.topk <= 32 && D.G <= 8)
        es = launch_pdl(decode_select_warp_kernel<8>, dim3(D.Hkv, D.B * D.T), dim3(kSelWThreads), 0, stream, D, P,
                        (const float *)scores, (const float *)part, sel, idx_out);
    else {
        // an ordinary launch: started early behind the score grid this split form measured slower
        decode_select_kernel<<<dim3(P.nparts, D.Hkv, D.B), kSelThreads, 0, stream>>>(D, P, scores, part, lists,
                                                                                     selcount, sel, idx_out);
        es = cudaGetLastError();
    }
    if (es != cudaSuccess) return es;
    if (decode_attn_mma_supported(D, sizeof(T) == 2 ? HILS_BF16 : HILS_FP32, q, k_cache, v_cache, P.ntiles))
        return launch_decode_attn_mma(D, P.n, P.ntiles, q, k_cache, v_cache, scores, sel, partial, counters, out, lse,
                                      stream);
    const size_t smem3 = 2 * (size_t)D.S * D.d * sizeof(T) +
                         sizeof(float) * ((size_t)D.G * D.S + 4 + (size_t)D.G * D.d * 3 / 2 + D.G + 4 +
                                          2 * (size_t)D.G * D.d);
    auto k3 = decode_attn_kernel<T, DPL>;
    if (smem3 > 48 * 1024) cudaFuncSetAttribute(k3, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem3);
    k3<<<dim3(P.ntiles, D.Hkv, D.B), kAttnThreads, smem3, stream>>>(D, P, (const T *)q, (const T *)k_cache,
                                                                     (const T *)v_cache, scores, sel, partial,
                                                                     counters, (T *)out, lse);
    return cudaGetLastError();
}

}  // namespace

size_t decode_workspace_bytes(const Dims &D) { return make_plan(D).total; }

bool decode_supported(const Dims &D) {
    // The attention tile (K and V of one chunk plus the per-head rows) must fit in shared memory.
    const size_t el = 4;  // worst case fp32
    const size_t smem3 = 2 * (size_t)D.S * D.d * el + 4 * ((size_t)D.G * D.S + 4 + (size_t)D.G * D.d * 3 / 2 + D.G + 4 + 2 * (size_t)D.G * D.d);
    const DecodePlan P = make_plan(D);
    return D.G <= 64 && D.topk + (D.W + 2 * D.S) / D.S <= 64 && next_pow2(P.nparts * D.topk) <= kSelMerge &&
           smem3 <= 200 * 1024;
}

// M > 1 query tokens run on the bf16 d 128 S 64 kernels only (streamed scores, single-CTA selection,
// split-K attention); the general kernels are single-token.
bool decode_multi_supported(const Dims &D, int dtype, const void *q, const void *q_hat, const void *k,
                            const void *v, const void *k_sum) {
    if (D.T == 1) return true;
    const DecodePlan P = make_plan(D);
    return D.T <= 8 && D.topk <= 32 && D.G <= 8 && decode_score_mma_supported(D, dtype, q_hat, k_sum) &&
           decode_attn_mma_supported(D, dtype, q, k, v, P.ntiles);
}

unsigned int decode_error_flags(bool clear) {
    unsigned int v = decode_attn_mma_error_flags(clear) | decode_score_mma_error_flags(clear);
    unsigned int mine = 0;
    cudaMemcpyFromSymbol(&mine, g_decode_errors, sizeof(mine));
    v |= mine;
    if (clear && mine) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_decode_errors, &zero, sizeof(zero));
    }
    return v;
}

cudaError_t launch_decode(const Dims &D, int dtype, const void *q, const void *q_hat, const void *k_cache,
                          const void *v_cache, const void *k_sum, const float *b_sum, void *out, float *lse,
                          int *idx_out, void *ws, cudaStream_t stream) {
    if (dtype == HILS_BF16) {
        if (D.d == 128)
            return launch_t<__nv_bfloat16, 4>(D, q, q_hat, k_cache, v_cache, k_sum, b_sum, out, lse, idx_out, ws, stream);
        return launch_t<__nv_bfloat16, 2>(D, q, q_hat, k_cache, v_cache, k_sum, b_sum, out, lse, idx_out, ws, stream);
    }
    if (D.d == 128) return launch_t<float, 4>(D, q, q_hat, k_cache, v_cache, k_sum, b_sum, out, lse, idx_out, ws, stream);
    return launch_t<float, 2>(D, q, q_hat, k_cache, v_cache, k_sum, b_sum, out, lse, idx_out, ws, stream);
}

}  // namespace hils
