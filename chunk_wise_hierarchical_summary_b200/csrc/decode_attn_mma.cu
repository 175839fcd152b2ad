// Decode stages (c)+(d) for bf16, d 128, S 64, up to 8 heads per KV group: attention of the new token
// over its selected chunks and its window, fused by Eq. 10 ("Hierarchical Sparse Attention Done Right",
// Sec. 3 RQ2, Eq. 10; Sec. 4 "GQA": the group's heads share every gathered tile).
//
// grid (nsplit, Hkv, B * M) for M = T query tokens per sequence (M > 1: multi-token decode): the tiles of
// one (b, KV group, query) - its window tiles, then its selected chunks - are dealt round-robin to
// nsplit CTAs. A CTA's window tiles depend on no earlier grid, so they are loaded and folded into its
// running softmax before griddepcontrol.wait, while the selection grid still runs. Per CTA:
//   warp 4     producer: K and V tiles (TMA, 128-byte swizzle) into a kStages-deep ring.
//   warps 0-3  per tile, on the warp-level tensor-core instruction (mma.sync m16n8k16, bf16 in, fp32
//              accumulate) with the group's heads as the 8-wide N side:
//                s^T[j, h] = k_j . q_h              warp w: tokens 16w .. 16w+15
//                tile max m and e_j = exp(s_j - m), z = sum e_j (per head, across the 4 warps)
//                the tile's mass anchor: a selected chunk carries exp(s^_c) split by its intra-chunk
//                softmax e_j / z, so its anchor is s^_c - log z; a window tile's anchor is m
//                online merge into the running (M, l, o): o and l scaled by exp(M - M'), the tile's
//                e_j by exp(anchor - M'), then o^T[t, h] += sum_j v[j, t] p[h, j]   warp w: cols 32w..
//              p enters the value product as bf16 hi + lo parts (two MMAs).
// Each CTA writes its (M, l, o) per head; the last CTA of the (b, KV group) to finish (atomic counter,
// no waiting) merges the nsplit partials into out and lse = log Z^.
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
constexpr int kCtasPerSm = 2;
constexpr int kMaxTiles = 64;
constexpr uint32_t kTileBytes = 16384;  // 64 tokens x 128 columns bf16
constexpr uint32_t kQRowBytes = 272;
constexpr int kPStride = 72;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kPartStride = 132;  // floats per (head, split) partial: M, l, 2 pad, o[128] (16-byte aligned)
constexpr int kMaxSplits = 32;    // CTAs per (b, KV group, query)

__device__ unsigned int g_decode_attn_errors = 0;


struct Tile {
    int j0, jn, c;  // first token, valid tokens, chunk id (-1: window tile)
};

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
decode_attn_mma_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap, Dims D,
                       int n, int ntiles, const __nv_bfloat16 *__restrict__ q, const float *__restrict__ scores,
                       const int *__restrict__ sel, float *__restrict__ partial, unsigned int *__restrict__ counters,
                       __nv_bfloat16 *__restrict__ out, float *__restrict__ lse) {
    extern __shared__ unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
    __shared__ float red_m[kConsumerWarps][8], red_z[kConsumerWarps][8];
    __shared__ __align__(16) __nv_bfloat16 p_hi[8 * kPStride], p_lo[8 * kPStride];
    __shared__ __align__(16) unsigned char qs[8 * kQRowBytes];
    __shared__ Tile tiles[kMaxTiles];
    __shared__ int s_nt, s_last;
    unsigned char *base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
    // grid z = b * M + m: query m (of M = D.T, at position q_pos0 + m) of sequence b
    const int split = blockIdx.x, nsplit = gridDim.x, g = blockIdx.y, M = D.T;
    const int b = blockIdx.z / M, m = blockIdx.z % M;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = D.G, S = D.S, K = D.topk;
    const size_t bg = (size_t)b * D.Hkv + g;  // K/V rows
    const size_t bgm = bg * M + m;            // this query's ids and counter
    const int pos = D.q_pos0 + m;
    const int l = window_left(pos, D.W, S);
    const int wt = ntiles - K;  // window tiles of the sequence; the selected chunks follow them
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_mbar_init();
        int nt = 0;
        for (int t = split; t < wt && nt < kMaxTiles; t += nsplit) {
            Tile tl;
            tl.j0 = l + t * S;
            tl.jn = min(S, pos + 1 - tl.j0);
            tl.c = -1;
            if (tl.jn <= 0) continue;
            tiles[nt++] = tl;
        }
        s_nt = nt;
    }
    for (int e = tid; e < G * 16; e += blockDim.x) {  // the group's query rows, 16 bytes per thread
        const int h = e >> 4, ch = e & 15;
        *reinterpret_cast<uint4 *>(qs + h * kQRowBytes + ch * 16) =
            *reinterpret_cast<const uint4 *>(q + (((size_t)b * D.Hq + g * G + h) * M + m) * 128 + ch * 8);
    }
    __syncthreads();
    const int nw = s_nt;  // this CTA's window tiles: the head of its list
    int nt = nw;
    bool ok = true;

    // running state of the consumer threads for heads 2*t4 and 2*t4+1 (log2 units)
    float M0 = -INFINITY, M1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    const int g8 = lane >> 2, t4 = lane & 3;

    // The selected chunks of this CTA, appended once the selection grid has completed.
    auto append_selected = [&]() {
        grid_dep_wait();  // the selection grid's ids (and, through it, the scores)
        __syncthreads();  // every thread is past its pre-wait tiles before the list grows
        if (warp == 0) {
            // this CTA's selected slots t0, t0 + nsplit, ... read 32 at a time, one per lane, in order
            int n2 = nw;
            for (int t = split + ((wt - split + nsplit - 1) / nsplit) * nsplit + lane * nsplit;
                 __any_sync(0xffffffffu, t < ntiles); t += 32 * nsplit) {
                const int c = (t < ntiles && t >= wt) ? sel[bgm * K + (t - wt)] : -1;
                const unsigned take = __ballot_sync(0xffffffffu, c >= 0);
                const int at = n2 + __popc(take & ((1u << lane) - 1u));
                if (c >= 0 && at < kMaxTiles) {
                    Tile tl;
                    tl.j0 = c * S;
                    tl.jn = S;
                    tl.c = c;
                    tiles[at] = tl;
                }
                n2 += __popc(take);
            }
            if (lane == 0) s_nt = min(n2, kMaxTiles);
        }
        __syncthreads();
        nt = s_nt;
    };

    if (warp == kConsumerWarps) {
        // ---------------------------------------------------------------- producer
        auto produce = [&](int i0, int i1) {
            if (lane == 0) {
                for (int i = i0; i < i1 && ok; ++i) {
                    const int st = i % kStages;
                    if (i >= kStages && !mbar_wait_bounded(&empty[st], ((i / kStages) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    unsigned char *Kt = base + st * 2 * kTileBytes;
                    const int y = (int)(bg * D.L) + tiles[i].j0;
                    mbar_arrive_expect_tx(&full[st], 2 * kTileBytes);
                    tma_load_2d(Kt, &kmap, 0, y, &full[st]);
                    tma_load_2d(Kt + 8192, &kmap, 64, y, &full[st]);
                    tma_load_2d(Kt + kTileBytes, &vmap, 0, y, &full[st]);
                    tma_load_2d(Kt + kTileBytes + 8192, &vmap, 64, y, &full[st]);
                }
            }
            __syncwarp();
        };
        produce(0, nw);
        append_selected();
        produce(nw, nt);
    } else {
        // ---------------------------------------------------------------- consumers
        const int mi = lane >> 3, r8 = lane & 7;
        const bool hv = g8 < G;
        const float sc2 = D.tau * kLog2e;
        // query rows (b, head, m) of [B, Hq, M, ...]: head h of the group at hrow0 + h * M
        const size_t hrow0 = ((size_t)b * D.Hq + g * G) * M + m;
        auto consume = [&](int i0, int i1) {
          for (int i = i0; i < i1; ++i) {
            const int st = i % kStages;
            const Tile tl = tiles[i];
            // the chunk's retrieval score for this thread's two heads, fetched before the tile wait
            float sh0 = 0.f, sh1 = 0.f;
            if (tl.c >= 0) {
                if (2 * t4 < G) sh0 = scores[(hrow0 + (size_t)(2 * t4) * M) * n + tl.c] * kLog2e;
                if (2 * t4 + 1 < G) sh1 = scores[(hrow0 + (size_t)(2 * t4 + 1) * M) * n + tl.c] * kLog2e;
            }
            const bool got = mbar_wait_bounded(&full[st], (i / kStages) & 1);
            const uint32_t Kb = smem_u32(base + st * 2 * kTileBytes), Vb = Kb + kTileBytes;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const int row = 16 * warp + r8 + (mi & 1) * 8;
                const int ch = (ks & 3) * 2 + (mi >> 1);
                uint32_t a[4];
                ldsm_x4(Kb + (ks >> 2) * 8192 + row * 128 + ((ch ^ (row & 7)) << 4), a);
                const unsigned char *qrow = qs + g8 * kQRowBytes + (ks * 16 + 2 * t4) * 2;
                const uint32_t b0 = hv ? ld_u32(qrow) : 0u, b1 = hv ? ld_u32(qrow + 16) : 0u;
                mma_16816(acc, a, b0, b1);
            }
            const int ja = 16 * warp + g8, jb = ja + 8;
            const float s00 = ja < tl.jn ? acc[0] * sc2 : -INFINITY, s01 = ja < tl.jn ? acc[1] * sc2 : -INFINITY;
            const float s10 = jb < tl.jn ? acc[2] * sc2 : -INFINITY, s11 = jb < tl.jn ? acc[3] * sc2 : -INFINITY;
            float m0 = fmaxf(s00, s10), m1 = fmaxf(s01, s11);
#pragma unroll
            for (int x = 4; x < 32; x <<= 1) {
                m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, x));
                m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, x));
            }
            if (g8 == 0) {
                red_m[warp][2 * t4] = m0;
                red_m[warp][2 * t4 + 1] = m1;
            }
            if (bar_group_any<kConsumerWarps * 32>(!got)) {
                ok = false;
                break;
            }
            float mt0 = red_m[0][2 * t4], mt1 = red_m[0][2 * t4 + 1];
#pragma unroll
            for (int w = 1; w < kConsumerWarps; ++w) {
                mt0 = fmaxf(mt0, red_m[w][2 * t4]);
                mt1 = fmaxf(mt1, red_m[w][2 * t4 + 1]);
            }
            const float e00 = ex2_approx(s00 - mt0), e01 = ex2_approx(s01 - mt1), e10 = ex2_approx(s10 - mt0), e11 = ex2_approx(s11 - mt1);
            float z0 = e00 + e10, z1 = e01 + e11;
#pragma unroll
            for (int x = 4; x < 32; x <<= 1) {
                z0 += __shfl_xor_sync(0xffffffffu, z0, x);
                z1 += __shfl_xor_sync(0xffffffffu, z1, x);
            }
            if (g8 == 0) {
                red_z[warp][2 * t4] = z0;
                red_z[warp][2 * t4 + 1] = z1;
            }
            bar_group<kConsumerWarps * 32>();
            float Z0 = 0.f, Z1 = 0.f;
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) {
                Z0 += red_z[w][2 * t4];
                Z1 += red_z[w][2 * t4 + 1];
            }
            const float A0 = tl.c >= 0 ? sh0 - __log2f(Z0) : mt0;
            const float A1 = tl.c >= 0 ? sh1 - __log2f(Z1) : mt1;
            const float N0 = fmaxf(M0, A0), N1 = fmaxf(M1, A1);
            const float fo0 = ex2_approx(M0 - N0), fo1 = ex2_approx(M1 - N1);  // 0 while M is still -inf
            const float fn0 = ex2_approx(A0 - N0), fn1 = ex2_approx(A1 - N1);
            M0 = N0;
            M1 = N1;
            l0 = l0 * fo0 + Z0 * fn0;
            l1 = l1 * fo1 + Z1 * fn1;
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                o[mt][0] *= fo0;
                o[mt][1] *= fo1;
                o[mt][2] *= fo0;
                o[mt][3] *= fo1;
            }
            {
                const float pv[4] = {e00 * fn0, e01 * fn1, e10 * fn0, e11 * fn1};
                const int hh[4] = {2 * t4, 2 * t4 + 1, 2 * t4, 2 * t4 + 1};
                const int jj[4] = {ja, ja, jb, jb};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const __nv_bfloat16 hi = __float2bfloat16_rn(pv[e]);
                    p_hi[hh[e] * kPStride + jj[e]] = hi;
                    p_lo[hh[e] * kPStride + jj[e]] = __float2bfloat16_rn(pv[e] - __bfloat162float(hi));
                }
            }
            bar_group<kConsumerWarps * 32>();
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
                    ldsm_x4_trans(Vb + (dd >> 6) * 8192 + j * 128 + ((((dd & 63) >> 3) ^ (j & 7)) << 4), a);
                    mma_16816(o[mt], a, bh0, bh1);
                    mma_16816(o[mt], a, bl0, bl1);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);
          }
        };
        consume(0, nw);
        append_selected();
        if (ok) consume(nw, nt);
        // this CTA's partial per head: (M, l, -, -) then o[128], laid out [B*Hq][nsplit][kPartStride]
        if (ok) {
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                const int dd = 32 * warp + 16 * mt + g8;
                if (2 * t4 < G) {
                    float *pp = partial + ((hrow0 + (size_t)(2 * t4) * M) * nsplit + split) * kPartStride + 4;
                    pp[dd] = o[mt][0];
                    pp[dd + 8] = o[mt][2];
                }
                if (2 * t4 + 1 < G) {
                    float *pp = partial + ((hrow0 + (size_t)(2 * t4 + 1) * M) * nsplit + split) * kPartStride + 4;
                    pp[dd] = o[mt][1];
                    pp[dd + 8] = o[mt][3];
                }
            }
            if (warp == 0 && g8 == 0) {
                if (2 * t4 < G) {
                    float *pp = partial + ((hrow0 + (size_t)(2 * t4) * M) * nsplit + split) * kPartStride;
                    pp[0] = M0;
                    pp[1] = l0;
                }
                if (2 * t4 + 1 < G) {
                    float *pp = partial + ((hrow0 + (size_t)(2 * t4 + 1) * M) * nsplit + split) * kPartStride;
                    pp[0] = M1;
                    pp[1] = l1;
                }
            }
        }
    }
    if (!ok) atomicOr(&g_decode_attn_errors, 1u);
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        s_last = (atomicAdd(&counters[bgm], 1u) == (unsigned)(nsplit - 1));
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // merge the nsplit (<= 32) partials of each head: one warp per head. Lane s fetches split s's (M, l),
    // the warp reduces them, then each lane accumulates its 4 columns over the splits, four loads in
    // flight at a time.
    for (int hh = warp; hh < G; hh += blockDim.x >> 5) {
        const size_t hr = ((size_t)b * D.Hq + g * G + hh) * M + m;
        const float *ph = partial + hr * nsplit * kPartStride;
        // every load of the head's partials in flight at once (nsplit <= kMaxSplits)
        const float ms = lane < nsplit ? __ldcg(ph + (size_t)lane * kPartStride) : -INFINITY;
        const float ls = lane < nsplit ? __ldcg(ph + (size_t)lane * kPartStride + 1) : 0.f;
        float4 v4[kMaxSplits];
#pragma unroll
        for (int s2 = 0; s2 < kMaxSplits; ++s2)
            v4[s2] = s2 < nsplit ? __ldcg(reinterpret_cast<const float4 *>(ph + (size_t)s2 * kPartStride + 4) + lane)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
        const float Mx = warp_max(ms);
        const float rs = ms == -INFINITY ? 0.f : ex2_approx(ms - Mx);  // a CTA with no tiles has weight 0
        const float Z = warp_sum(ls * rs);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s2 = 0; s2 < kMaxSplits; ++s2) {
            const float r = __shfl_sync(0xffffffffu, rs, s2);  // 0 for s2 >= nsplit (ms = -inf there)
            acc[0] = fmaf(v4[s2].x, r, acc[0]);
            acc[1] = fmaf(v4[s2].y, r, acc[1]);
            acc[2] = fmaf(v4[s2].z, r, acc[2]);
            acc[3] = fmaf(v4[s2].w, r, acc[3]);
        }
        const float inv = Z > 0.f ? 1.f / Z : 0.f;
        const __nv_bfloat162 h01 = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
        const __nv_bfloat162 h23 = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
        uint2 w2;
        w2.x = *reinterpret_cast<const uint32_t *>(&h01);
        w2.y = *reinterpret_cast<const uint32_t *>(&h23);
        *reinterpret_cast<uint2 *>(out + hr * 128 + lane * 4) = w2;
        if (lane == 0) lse[hr] = (Mx + log2f(Z)) * (1.f / kLog2e);
    }
}

}  // namespace

bool decode_attn_mma_supported(const Dims &D, int dtype, const void *q, const void *k, const void *v, int ntiles) {
    auto al16 = [](const void *p) { return ((uintptr_t)p & 15u) == 0; };
    return dtype == HILS_BF16 && D.d == 128 && D.S == 64 && D.G >= 1 && D.G <= 8 && ntiles <= kMaxTiles &&
           al16(q) && al16(k) && al16(v) && (long long)D.B * D.Hkv * D.L < (1ll << 31);
}

// The number of CTAs per (b, KV group, query): as many as two per SM allow, at most one per tile and at
// most 16 (so the last CTA merges few partials: at small batches a split is then 2-3 tiles).
int decode_attn_mma_splits(const Dims &D, int ntiles) {
    const int per_bg = std::max(1, (kCtasPerSm * num_sms()) / std::max(1, D.B * D.Hkv * D.T));
    return std::max(1, std::min(std::min(per_bg, ntiles), kMaxSplits));
}

unsigned int decode_attn_mma_error_flags(bool clear) {
    unsigned int v = 0;
    cudaMemcpyFromSymbol(&v, g_decode_attn_errors, sizeof(v));
    if (clear && v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbol(g_decode_attn_errors, &zero, sizeof(zero));
    }
    return v;
}

// `partial` holds B * Hq * T * nsplit * 132 floats (16-byte aligned); `counters` B * Hkv * T zeros.
cudaError_t launch_decode_attn_mma(const Dims &D, int n, int ntiles, const void *q, const void *k_cache,
                                   const void *v_cache, const float *scores, const int *sel, float *partial,
                                   unsigned int *counters, void *out, float *lse, cudaStream_t stream) {
    CUtensorMap kmap, vmap;
    if (!make_tmap_bf16_2d(&kmap, k_cache, (uint64_t)D.B * D.Hkv * D.L, 128, 128, 64) ||
        !make_tmap_bf16_2d(&vmap, v_cache, (uint64_t)D.B * D.Hkv * D.L, 128, 128, 64))
        return cudaErrorInvalidValue;
    const size_t smem = 1024 + kStages * 2 * kTileBytes;
    cudaFuncSetAttribute(decode_attn_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int nsplit = decode_attn_mma_splits(D, ntiles);
    return launch_pdl(decode_attn_mma_kernel, dim3(nsplit, D.Hkv, D.B * D.T), dim3(kThreads), smem, stream, kmap, vmap,
                      D, n, ntiles, (const __nv_bfloat16 *)q, scores, sel, partial, counters, (__nv_bfloat16 *)out,
                      lse);
}

}  // namespace hils
