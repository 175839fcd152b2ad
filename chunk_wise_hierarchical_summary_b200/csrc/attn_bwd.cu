// Backward of the HiLS forward (summaries + Eq. 10 attention) with the selection held fixed
// ("Hierarchical Sparse Attention Done Right", Sec. 3 RQ2: the LM-loss gradient reaches the landmark
// summaries through s^ in Z^). Notation per (b, h, query i): lse = log Z^, D = dout . out,
// a_j = exp(s_j - lse) (window), beta_c = exp(s^_c - lse), pi_cj = exp(s_j - L_c), dv.. = dout . v_j:
//   window: ds_j = a_j (dout.v_j - D)                  dv_j += a_j dout
//   chunk : ds^_c = beta_c (dout.o_c - D), ds_j = beta_c pi_cj (dout.v_j - dout.o_c), dv_j += beta_c pi_cj dout
//   dq = tau sum_j ds_j k_j, dk_j += tau ds_j q, dq^ = tau sum_c ds^_c k'_c, dk'_c += tau ds^_c q^, db'_c += ds^_c
//   Eq. 8 backward: du_j = p_j (dk'.(k_j - k') - db' (log p_j + b')), dq'_c = tau sum_j du_j k_j,
//                   dk_j += p_j dk' + tau du_j q'_c
//
// This file is the general form (CUDA cores, any dtype, d and S); bf16 with d 128, S 64, G <= 4 and
// at most 128 chunks runs the tensor-core backward of attn_bwd_tc.cu instead.
// Two deterministic kernels (no atomics):
//   bwd_dq    query-major, one warp per (b, h, i): D, dq, dq^.
//   bwd_dkdv  chunk-major, one CTA per (b, KV group, chunk c): every (query, head) touching the chunk
//             (window queries: a contiguous range; selecting queries: found by scanning idx in query
//             order), accumulating dk/dv for the chunk's tokens and dk'_c/db'_c, then the chunk's
//             Eq. 8 backward (dq'_c and its dk share). Requires T == L and q_pos0 == 0.
#include "internal.h"

namespace hils {

bool attn_bwd_tc_supported(const Dims &D, int dtype);
size_t attn_bwd_tc_workspace(const Dims &D);
cudaError_t launch_attn_bwd_tc(const Dims &D, const void *q, const void *k, const void *v, const void *q_hat,
                               const void *q_land, const void *k_sum, const float *b_sum, const int *idx,
                               const void *out, const float *lse, const void *dout, void *dq, void *dk, void *dv,
                               void *dq_hat, void *dq_land, void *ws, cudaStream_t stream);

namespace {

constexpr int kDqWarps = 4;
constexpr int kDkvThreads = 256;

template <typename T, int DPL>
__device__ __forceinline__ float wdot(const float (&a)[DPL], const T *row, int lane) {
    float s = 0.f;
#pragma unroll
    for (int u = 0; u < DPL; ++u) s = fmaf(a[u], to_f(row[lane + 32 * u]), s);
    return warp_sum(s);
}

template <typename T, int DPL>
__global__ void __launch_bounds__(kDqWarps * 32)
bwd_dq_kernel(Dims D, const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
              const T *__restrict__ q_hat, const T *__restrict__ k_sum, const float *__restrict__ b_sum,
              const int *__restrict__ idx, const T *__restrict__ out, const float *__restrict__ lse,
              const T *__restrict__ dout, T *__restrict__ dq, T *__restrict__ dq_hat, float *__restrict__ Dbuf) {
    __shared__ float s_log[kDqWarps][HILS_MAX_S];
    __shared__ float s_dov[kDqWarps][HILS_MAX_S];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x * kDqWarps + warp, h = blockIdx.y, b = blockIdx.z;
    if (i >= D.T) return;
    const int g = h / D.G, d = D.d, S = D.S;
    const int pos = D.q_pos0 + i;
    const int l = window_left(pos, D.W, S), n = l / S;
    const size_t row = ((size_t)b * D.Hq + h) * D.T + i;
    const T *kb = k + ((size_t)b * D.Hkv + g) * (size_t)D.L * d;
    const T *vb = v + ((size_t)b * D.Hkv + g) * (size_t)D.L * d;
    float qv[DPL], qh[DPL], dov[DPL], gq[DPL], gqh[DPL];
    float Dp = 0.f;
#pragma unroll
    for (int u = 0; u < DPL; ++u) {
        qv[u] = to_f(q[row * d + lane + 32 * u]) * D.tau;
        qh[u] = to_f(q_hat[row * d + lane + 32 * u]) * D.tau;
        dov[u] = to_f(dout[row * d + lane + 32 * u]);
        Dp = fmaf(dov[u], to_f(out[row * d + lane + 32 * u]), Dp);
        gq[u] = 0.f;
        gqh[u] = 0.f;
    }
    const float Dv = warp_sum(Dp);
    const float lz = lse[row];
    if (lane == 0) Dbuf[row] = Dv;

    for (int j = l; j <= pos; ++j) {
        const float s = wdot<T, DPL>(qv, kb + (size_t)j * d, lane);
        const float a = __expf(s - lz);
        const float ds = a * (wdot<T, DPL>(dov, vb + (size_t)j * d, lane) - Dv);
#pragma unroll
        for (int u = 0; u < DPL; ++u) gq[u] = fmaf(ds, to_f(kb[(size_t)j * d + lane + 32 * u]), gq[u]);
    }
    const int *irow = idx + (((size_t)b * D.Hkv + g) * D.T + i) * D.topk;
    for (int t = 0; t < D.topk; ++t) {
        const int c = irow[t];
        if (c < 0 || c >= n) continue;
        bool dup = false;
        for (int u = 0; u < t; ++u) dup |= (irow[u] == c);
        if (dup) continue;
        const size_t srow = ((size_t)b * D.Hq + h) * D.Nc + c;
        const float shat = wdot<T, DPL>(qh, k_sum + srow * d, lane) + b_sum[srow];
        const float beta = __expf(shat - lz);
        float mx = -INFINITY;
        for (int j = 0; j < S; ++j) {
            const float s = wdot<T, DPL>(qv, kb + (size_t)(c * S + j) * d, lane);
            const float dv = wdot<T, DPL>(dov, vb + (size_t)(c * S + j) * d, lane);
            if (lane == 0) { s_log[warp][j] = s; s_dov[warp][j] = dv; }
            mx = fmaxf(mx, s);
        }
        __syncwarp();
        float z = 0.f, zo = 0.f;
        for (int j = lane; j < S; j += 32) {
            const float e = __expf(s_log[warp][j] - mx);
            z += e;
            zo = fmaf(e, s_dov[warp][j], zo);
        }
        z = warp_sum(z);
        zo = warp_sum(zo);
        const float doo = zo / z;  // dout . o_c
        const float Lc = mx + logf(z);
        const float dshat = beta * (doo - Dv);
        for (int j = 0; j < S; ++j) {
            const float ds = beta * __expf(s_log[warp][j] - Lc) * (s_dov[warp][j] - doo);
#pragma unroll
            for (int u = 0; u < DPL; ++u) gq[u] = fmaf(ds, to_f(kb[(size_t)(c * S + j) * d + lane + 32 * u]), gq[u]);
        }
#pragma unroll
        for (int u = 0; u < DPL; ++u) gqh[u] = fmaf(dshat, to_f(k_sum[srow * d + lane + 32 * u]), gqh[u]);
        __syncwarp();
    }
#pragma unroll
    for (int u = 0; u < DPL; ++u) {
        dq[row * d + lane + 32 * u] = from_f<T>(gq[u] * D.tau);
        dq_hat[row * d + lane + 32 * u] = from_f<T>(gqh[u] * D.tau);
    }
}

struct DkvSmem {
    int ld;
    size_t k_off, v_off, dk_off, dv_off, q_off, do_off, qh_off, s_off, dov_off, w_off, ds_off, dks_off, sc_off, list_off,
        total;
};

__host__ __device__ inline DkvSmem dkv_layout(int S, int d, int G) {
    DkvSmem L{};
    L.ld = d + 1;
    size_t off = 0;
    auto take = [&](size_t floats) {
        size_t at = off;
        off += (floats + 3) & ~(size_t)3;
        return at;
    };
    L.k_off = take((size_t)S * L.ld);
    L.v_off = take((size_t)S * L.ld);
    L.dk_off = take((size_t)S * d);
    L.dv_off = take((size_t)S * d);
    L.q_off = take((size_t)G * d);
    L.do_off = take((size_t)G * d);
    L.qh_off = take((size_t)G * d);
    L.s_off = take((size_t)G * S);
    L.dov_off = take((size_t)G * S);
    L.w_off = take((size_t)G * S);
    L.ds_off = take((size_t)G * S);
    L.dks_off = take((size_t)G * (d + 1));  // dk'_c (d) and db'_c per head
    L.sc_off = take((size_t)G * 4);          // per-head scalars
    L.list_off = take(kDkvThreads + 32);     // query list (ints) + warp counts
    L.total = off * sizeof(float);
    return L;
}

template <typename T>
__global__ void __launch_bounds__(kDkvThreads)
bwd_dkdv_kernel(Dims D, const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                const T *__restrict__ q_hat, const T *__restrict__ q_land, const T *__restrict__ k_sum,
                const float *__restrict__ b_sum, const int *__restrict__ idx, const float *__restrict__ lse,
                const T *__restrict__ dout, const float *__restrict__ Dbuf, T *__restrict__ dk, T *__restrict__ dv,
                T *__restrict__ dq_land) {
    extern __shared__ __align__(16) float sm[];
    const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int d = D.d, S = D.S, G = D.G;
    const DkvSmem Ly = dkv_layout(S, d, G);
    const int ld = Ly.ld;
    float *Ks = sm + Ly.k_off, *Vs = sm + Ly.v_off, *dK = sm + Ly.dk_off, *dV = sm + Ly.dv_off;
    float *Qs = sm + Ly.q_off, *DOs = sm + Ly.do_off, *QHs = sm + Ly.qh_off;
    float *Sl = sm + Ly.s_off, *DOV = sm + Ly.dov_off, *Wt = sm + Ly.w_off, *DS = sm + Ly.ds_off;
    float *DKS = sm + Ly.dks_off;
    int *list = reinterpret_cast<int *>(sm + Ly.list_off);
    int *wcount = list + kDkvThreads;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nwarps = blockDim.x >> 5;
    const int j0 = c * S;
    const int jn = min(S, D.L - j0);
    const size_t bg = (size_t)b * D.Hkv + g;
    const T *kb = k + (bg * D.L + j0) * d;
    const T *vb = v + (bg * D.L + j0) * d;

    for (int e = tid; e < S * ld; e += blockDim.x) { Ks[e] = 0.f; Vs[e] = 0.f; }
    __syncthreads();
    for (int e = tid; e < jn * d; e += blockDim.x) {
        const int j = e / d, t = e % d;
        Ks[j * ld + t] = to_f(kb[e]);
        Vs[j * ld + t] = to_f(vb[e]);
    }
    for (int e = tid; e < S * d; e += blockDim.x) { dK[e] = 0.f; dV[e] = 0.f; }
    for (int e = tid; e < G * (d + 1); e += blockDim.x) DKS[e] = 0.f;
    __syncthreads();

    // One (query i, all G heads) contribution; `sel` = chunk-selection type, else window type.
    auto contribute = [&](int i, bool sel) {
        const int pos = D.q_pos0 + i;
        const int l = window_left(pos, D.W, S);
        for (int e = tid; e < G * d; e += blockDim.x) {
            const int hh = e / d, t = e % d;
            const size_t row = ((size_t)b * D.Hq + g * G + hh) * D.T + i;
            Qs[e] = to_f(q[row * d + t]);
            DOs[e] = to_f(dout[row * d + t]);
            QHs[e] = sel ? to_f(q_hat[row * d + t]) : 0.f;
        }
        __syncthreads();
        // Logits and dout.v_j for every (head, token) of the chunk.
        for (int e = tid; e < G * S; e += blockDim.x) {
            const int hh = e / S, j = e % S;
            const float *kj = Ks + j * ld, *vj = Vs + j * ld, *qq = Qs + hh * d, *dd = DOs + hh * d;
            float s = 0.f, o = 0.f;
            for (int t = 0; t < d; ++t) {
                s = fmaf(qq[t], kj[t], s);
                o = fmaf(dd[t], vj[t], o);
            }
            const int jabs = j0 + j;
            const bool valid = sel ? (j < jn) : (j < jn && jabs >= l && jabs <= pos);
            Sl[e] = valid ? s * D.tau : -INFINITY;
            DOV[e] = o;
        }
        __syncthreads();
        for (int hh = warp; hh < G; hh += nwarps) {
            const size_t row = ((size_t)b * D.Hq + g * G + hh) * D.T + i;
            const float lz = lse[row], Dv = Dbuf[row];
            float *sl = Sl + hh * S, *dov = DOV + hh * S, *wt = Wt + hh * S, *ds = DS + hh * S;
            if (sel) {
                float mx = -INFINITY;
                for (int j = lane; j < S; j += 32) mx = fmaxf(mx, sl[j]);
                mx = warp_max(mx);
                float z = 0.f, zo = 0.f;
                for (int j = lane; j < S; j += 32) {
                    const float e = __expf(sl[j] - mx);
                    z += e;
                    zo = fmaf(e, dov[j], zo);
                }
                z = warp_sum(z);
                zo = warp_sum(zo);
                const float doo = zo / z, Lc = mx + logf(z);
                const size_t srow = ((size_t)b * D.Hq + g * G + hh) * D.Nc + c;
                float sh = 0.f;
                for (int t = lane; t < d; t += 32) sh = fmaf(QHs[hh * d + t], to_f(k_sum[srow * d + t]), sh);
                sh = warp_sum(sh) * D.tau + b_sum[srow];
                const float beta = __expf(sh - lz);
                const float dshat = beta * (doo - Dv);
                for (int j = lane; j < S; j += 32) {
                    const float w = beta * __expf(sl[j] - Lc);
                    wt[j] = w;
                    ds[j] = w * (dov[j] - doo);
                }
                for (int t = lane; t < d; t += 32) DKS[hh * (d + 1) + t] += D.tau * dshat * QHs[hh * d + t];
                if (lane == 0) DKS[hh * (d + 1) + d] += dshat;
            } else {
                for (int j = lane; j < S; j += 32) {
                    const float a = __expf(sl[j] - lz);  // -inf logits give 0
                    wt[j] = a;
                    ds[j] = a * (dov[j] - Dv);
                }
            }
        }
        __syncthreads();
        for (int e = tid; e < S * d; e += blockDim.x) {
            const int j = e / d, t = e % d;
            float gk = 0.f, gv = 0.f;
            for (int hh = 0; hh < G; ++hh) {
                gk = fmaf(DS[hh * S + j], Qs[hh * d + t], gk);
                gv = fmaf(Wt[hh * S + j], DOs[hh * d + t], gv);
            }
            dK[e] = fmaf(D.tau, gk, dK[e]);
            dV[e] += gv;
        }
        __syncthreads();
    };

    // Window queries: positions whose aligned window reaches into this chunk.
    const int wi_end = min(D.T - 1, j0 + S + D.W - 2);
    for (int i = j0; i <= wi_end; ++i) contribute(i, false);

    // Selecting queries (only complete chunks can be candidates), in query order.
    if (c < D.Nc) {
        const int i_first = (c + 1) * S + D.W - 1;  // first position with chunk c as a candidate
        for (int base = i_first; base < D.T; base += blockDim.x) {
            const int i = base + tid;
            bool hit = false;
            if (i < D.T) {
                const int *irow = idx + (bg * D.T + i) * D.topk;
                const int n = window_left(D.q_pos0 + i, D.W, S) / S;
                for (int t = 0; t < D.topk; ++t) hit |= (irow[t] == c && c < n);
            }
            const unsigned m = __ballot_sync(0xffffffffu, hit);
            if (lane == 0) wcount[warp] = __popc(m);
            __syncthreads();
            int before = 0, total = 0;
            for (int w = 0; w < nwarps; ++w) {
                before += (w < warp) ? wcount[w] : 0;
                total += wcount[w];
            }
            if (hit) list[before + __popc(m & ((1u << lane) - 1))] = i;
            __syncthreads();
            for (int u = 0; u < total; ++u) contribute(list[u], true);
        }

        // Eq. 8 backward for this chunk, per head.
        for (int hh = warp; hh < G; hh += nwarps) {
            const size_t crow = ((size_t)b * D.Hq + g * G + hh) * D.Nc + c;
            float *u_ = Sl + hh * S, *p_ = Wt + hh * S, *du = DS + hh * S;
            const T *ql = q_land + crow * d;
            float mx = -INFINITY;
            for (int j = lane; j < S; j += 32) {
                float s = 0.f;
                for (int t = 0; t < d; ++t) s = fmaf(to_f(ql[t]), Ks[j * ld + t], s);
                s *= D.tau;
                u_[j] = s;
                mx = fmaxf(mx, s);
            }
            mx = warp_max(mx);
            float z = 0.f;
            for (int j = lane; j < S; j += 32) z += __expf(u_[j] - mx);
            z = warp_sum(z);
            const float lu = mx + logf(z);
            float ent = 0.f;
            for (int j = lane; j < S; j += 32) {
                const float lp = u_[j] - lu;
                const float pj = __expf(lp);
                p_[j] = pj;
                ent -= pj * lp;
            }
            ent = warp_sum(ent);
            __syncwarp();
            // k' recomputed in fp32; Qs[hh] reused as scratch for it.
            float *kp = Qs + hh * d;
            for (int t = lane; t < d; t += 32) {
                float acc = 0.f;
                for (int j = 0; j < S; ++j) acc = fmaf(p_[j], Ks[j * ld + t], acc);
                kp[t] = acc;
            }
            __syncwarp();
            const float *dks = DKS + hh * (d + 1);
            const float dbs = dks[d];
            float kk = 0.f;
            for (int t = lane; t < d; t += 32) kk = fmaf(dks[t], kp[t], kk);
            kk = warp_sum(kk);
            for (int j = lane; j < S; j += 32) {
                float a = 0.f;
                for (int t = 0; t < d; ++t) a = fmaf(dks[t], Ks[j * ld + t], a);
                du[j] = p_[j] * (a - kk - dbs * ((u_[j] - lu) + ent));
            }
            __syncwarp();
            T *dql = dq_land + crow * d;
            for (int t = lane; t < d; t += 32) {
                float acc = 0.f;
                for (int j = 0; j < S; ++j) acc = fmaf(du[j], Ks[j * ld + t], acc);
                dql[t] = from_f<T>(D.tau * acc);
            }
            __syncwarp();
        }
        __syncthreads();
        // dk_j += p_j dk' + tau du_j q' (all heads of the group), reusing the per-head p and du rows.
        for (int e = tid; e < S * d; e += blockDim.x) {
            const int j = e / d, t = e % d;
            float a = 0.f;
            for (int hh = 0; hh < G; ++hh) {
                const size_t crow = ((size_t)b * D.Hq + g * G + hh) * D.Nc + c;
                a = fmaf(Wt[hh * S + j], DKS[hh * (d + 1) + t], a);
                a = fmaf(D.tau * DS[hh * S + j], to_f(q_land[crow * d + t]), a);
            }
            dK[e] += a;
        }
        __syncthreads();
    }

    for (int e = tid; e < jn * d; e += blockDim.x) {
        dk[(bg * D.L + j0) * d + e] = from_f<T>(dK[e]);
        dv[(bg * D.L + j0) * d + e] = from_f<T>(dV[e]);
    }
}

template <typename T>
cudaError_t launch_t(const Dims &D, const void *q, const void *k, const void *v, const void *q_hat, const void *q_land,
                     const void *k_sum, const float *b_sum, const int *idx, const void *out, const float *lse,
                     const void *dout, void *dq, void *dk, void *dv, void *dq_hat, void *dq_land, void *ws,
                     cudaStream_t stream) {
    float *Dbuf = (float *)ws;
    dim3 g1((D.T + kDqWarps - 1) / kDqWarps, D.Hq, D.B);
    if (D.d == 128)
        bwd_dq_kernel<T, 4><<<g1, kDqWarps * 32, 0, stream>>>(D, (const T *)q, (const T *)k, (const T *)v,
                                                             (const T *)q_hat, (const T *)k_sum, b_sum, idx,
                                                             (const T *)out, lse, (const T *)dout, (T *)dq,
                                                             (T *)dq_hat, Dbuf);
    else
        bwd_dq_kernel<T, 2><<<g1, kDqWarps * 32, 0, stream>>>(D, (const T *)q, (const T *)k, (const T *)v,
                                                             (const T *)q_hat, (const T *)k_sum, b_sum, idx,
                                                             (const T *)out, lse, (const T *)dout, (T *)dq,
                                                             (T *)dq_hat, Dbuf);
    const DkvSmem Ly = dkv_layout(D.S, D.d, D.G);
    auto kern = bwd_dkdv_kernel<T>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Ly.total);
    dim3 g2((D.L + D.S - 1) / D.S, D.Hkv, D.B);
    kern<<<g2, kDkvThreads, Ly.total, stream>>>(D, (const T *)q, (const T *)k, (const T *)v, (const T *)q_hat,
                                               (const T *)q_land, (const T *)k_sum, b_sum, idx, lse, (const T *)dout,
                                               Dbuf, (T *)dk, (T *)dv, (T *)dq_land);
    return cudaGetLastError();
}

}  // namespace

size_t bwd_workspace_bytes(const Dims &D, int dtype) {
    if (attn_bwd_tc_supported(D, dtype)) return attn_bwd_tc_workspace(D);
    return ((size_t)D.B * D.Hq * D.T * sizeof(float) + 255) & ~(size_t)255;
}

size_t bwd_smem_bytes(const Dims &D) { return dkv_layout(D.S, D.d, D.G).total; }

cudaError_t launch_attn_bwd(const Dims &D, int dtype, const void *q, const void *k, const void *v, const void *q_hat,
                            const void *q_land, const void *k_sum, const float *b_sum, const int *idx,
                            const void *out, const float *lse, const void *dout, void *dq, void *dk, void *dv,
                            void *dq_hat, void *dq_land, void *ws, cudaStream_t stream) {
    if (attn_bwd_tc_supported(D, dtype))
        return launch_attn_bwd_tc(D, q, k, v, q_hat, q_land, k_sum, b_sum, idx, out, lse, dout, dq, dk, dv, dq_hat,
                                  dq_land, ws, stream);
    if (dtype == HILS_BF16)
        return launch_t<__nv_bfloat16>(D, q, k, v, q_hat, q_land, k_sum, b_sum, idx, out, lse, dout, dq, dk, dv,
                                       dq_hat, dq_land, ws, stream);
    return launch_t<float>(D, q, k, v, q_hat, q_land, k_sum, b_sum, idx, out, lse, dout, dq, dk, dv, dq_hat, dq_land,
                           ws, stream);
}

}  // namespace hils
