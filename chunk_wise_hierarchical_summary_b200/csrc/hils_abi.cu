// C ABI of the HiLS hot path: argument validation, workspace sizing and kernel dispatch.
// Every check runs on the host before any launch; no C++ exception crosses the boundary.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <string>

#include "internal.h"

namespace hils {

size_t bwd_smem_bytes(const Dims &D);
bool decode_supported(const Dims &D);
bool decode_multi_supported(const Dims &D, int dtype, const void *q, const void *q_hat, const void *k, const void *v,
                            const void *k_sum);
cudaError_t launch_attn_fwd_simt(const Dims &D, int dtype, const void *q, const void *k, const void *v,
                                 const void *q_hat, const void *k_sum, const float *b_sum, const int *idx, void *out,
                                 float *lse, cudaStream_t stream);
bool attn_fwd_tc_supported(const Dims &D, int dtype);
cudaError_t launch_attn_fwd_tc(const Dims &D, const void *q, const void *k, const void *v, const void *q_hat,
                               const void *k_sum, const float *b_sum, const int *idx, void *out, float *lse,
                               void *ws, cudaStream_t stream);
unsigned int attn_tc_error_flags(bool clear);
size_t attn_fwd_tc_workspace(const Dims &D);
hils_status check_device_errors();
bool select_tc_supported(const Dims &D, int dtype);
cudaError_t launch_select_tc(const Dims &D, const void *q_hat, const void *k_sum, const float *b_sum, int *idx,
                             float *gap, float *shat, cudaStream_t stream);
unsigned int select_tc_error_flags(bool clear);
unsigned int summary_error_flags(bool clear);
unsigned int attn_bwd_tc_error_flags(bool clear);
unsigned int bsa_error_flags(bool clear);
cudaError_t launch_select_tc_qcal(const Dims &D, const void *q, const void *w_down, const void *w_up,
                                  const void *k_sum, const float *b_sum, int *idx, float *gap, float *shat,
                                  cudaStream_t stream);
bool attn_fwd_shat_supported(const Dims &D, int dtype);
cudaError_t launch_attn_fwd_tc_shat(const Dims &D, const void *q, const void *k, const void *v, const int *idx,
                                    const float *shat, void *out, float *lse, cudaStream_t stream);
int bsa_max_candidates(const Dims &D);
cudaError_t launch_bsa_select_topk(const Dims &D, int dtype, const void *q, const void *k, int *idx, float *gap,
                                   float *mass, cudaStream_t stream);
unsigned int wait_expiry_error_flags(bool clear);
cudaError_t launch_wait_expiry(uint32_t max_polls, int arrive_first, cudaStream_t stream);

namespace {

constexpr size_t kMaxSmem = 227 * 1024;
thread_local std::string g_last_error;

hils_status fail(hils_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

hils_status cuda_status(cudaError_t e, const char *where) {
    if (e == cudaSuccess) return HILS_OK;
    return fail(HILS_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

#define HILS_REQUIRE_PTR(ptr)                                                                        \
    do {                                                                                            \
        if ((ptr) == nullptr) return fail(HILS_ERR_INVALID_ARG, "%s: %s is NULL", fn, #ptr);       \
        if (!aligned16(ptr)) return fail(HILS_ERR_INVALID_ARG, "%s: %s is not 16-byte aligned", fn, #ptr); \
    } while (0)

// Validates the sizes shared by every call and resolves them into Dims.
hils_status resolve(const hils_params *p, const char *fn, Dims *D) {
    if (p == nullptr) return fail(HILS_ERR_INVALID_ARG, "%s: params is NULL", fn);
    if (p->B < 1 || p->T < 1 || p->L < 1 || p->Hq < 1 || p->Hkv < 1 || p->d < 1 || p->S < 1 || p->topk < 1 ||
        p->window < 1)
        return fail(HILS_ERR_INVALID_ARG, "%s: every size must be >= 1 (B=%d T=%d L=%d Hq=%d Hkv=%d d=%d S=%d topk=%d "
                    "window=%d)", fn, p->B, p->T, p->L, p->Hq, p->Hkv, p->d, p->S, p->topk, p->window);
    if (p->Hq % p->Hkv != 0) return fail(HILS_ERR_INVALID_ARG, "%s: Hq=%d is not a multiple of Hkv=%d", fn, p->Hq, p->Hkv);
    if (p->q_pos0 < 0 || (int64_t)p->q_pos0 + p->T > p->L)
        return fail(HILS_ERR_INVALID_ARG, "%s: query rows [%d, %d) exceed the KV length L=%d", fn, p->q_pos0,
                    p->q_pos0 + p->T, p->L);
    if (p->dtype != HILS_BF16 && p->dtype != HILS_FP32)
        return fail(HILS_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, p->dtype);
    if (!(p->scale >= 0.f) || isinf(p->scale)) return fail(HILS_ERR_INVALID_ARG, "%s: scale must be finite and >= 0", fn);
    if (p->d != 64 && p->d != 128) return fail(HILS_ERR_UNSUPPORTED, "%s: d=%d (supported: 64, 128)", fn, p->d);
    if (p->S > HILS_MAX_S) return fail(HILS_ERR_UNSUPPORTED, "%s: S=%d > %d", fn, p->S, HILS_MAX_S);
    if (p->topk > HILS_MAX_TOPK) return fail(HILS_ERR_UNSUPPORTED, "%s: topk=%d > %d", fn, p->topk, HILS_MAX_TOPK);
    if (p->Hq > 65535 || p->B > 65535) return fail(HILS_ERR_UNSUPPORTED, "%s: Hq and B must be <= 65535", fn);
    D->B = p->B; D->T = p->T; D->L = p->L; D->Hq = p->Hq; D->Hkv = p->Hkv; D->d = p->d; D->S = p->S;
    D->topk = p->topk; D->W = p->window; D->q_pos0 = p->q_pos0;
    D->G = p->Hq / p->Hkv;
    D->Nc = p->L / p->S;
    D->tau = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->d);
    return HILS_OK;
}

hils_status check_ws(const char *fn, void *ws, size_t have, size_t need) {
    if (need == 0) return HILS_OK;
    if (ws == nullptr || have < need)
        return fail(HILS_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need, ws ? have : 0);
    if (((uintptr_t)ws & 255u) != 0) return fail(HILS_ERR_INVALID_ARG, "%s: workspace is not 256-byte aligned", fn);
    return HILS_OK;
}

}  // namespace

// Lets other translation units of the library set the thread-local message of hils_last_error().
void record_error(const char *msg) { g_last_error = msg; }

hils_status check_device_errors() {
    if (summary_error_flags(true) != 0)
        return fail(HILS_ERR_TIMEOUT, "hils_check: a summary tile's copy did not complete within its wait budget; "
                    "that call's summaries are invalid");
    if (select_tc_error_flags(true) != 0)
        return fail(HILS_ERR_TIMEOUT, "hils_check: a tensor-core selection tile's wait expired; that call's ids are "
                    "invalid");
    const unsigned int af = attn_tc_error_flags(true);
    if (af & 1u)
        return fail(HILS_ERR_TIMEOUT, "hils_check: a tensor-core attention tile's wait expired; that call's output "
                    "is invalid");
    if (af & 2u)
        return fail(HILS_ERR_INVALID_ARG, "hils_check: hils_attn_fwd_shat was given a row of ids not in canonical "
                    "form (candidate ids strictly ascending, then -1); that call's output is invalid");
    if (attn_bwd_tc_error_flags(true) != 0)
        return fail(HILS_ERR_TIMEOUT, "hils_check: a tensor-core backward tile's wait expired; that call's "
                    "gradients are invalid");
    if (bsa_error_flags(true) != 0)
        return fail(HILS_ERR_TIMEOUT, "hils_check: a naive-BSA mass tile's wait expired; that call's masses and ids "
                    "are invalid");
    if (decode_error_flags(true) != 0)
        return fail(HILS_ERR_TIMEOUT, "hils_check: a decode tile's bulk copy did not complete within its wait "
                    "budget; that call's output is invalid");
    if (wait_expiry_error_flags(true) != 0)
        return fail(HILS_ERR_TIMEOUT, "hils_check: the test hook's bounded wait expired (nothing arrived at its "
                    "barrier)");
    return HILS_OK;
}

}  // namespace hils

using namespace hils;

extern "C" {

const char *hils_version(void) { return "hils-b200 0.1 (sm_100a)"; }

const char *hils_status_string(hils_status s) {
    switch (s) {
        case HILS_OK: return "HILS_OK";
        case HILS_ERR_INVALID_ARG: return "HILS_ERR_INVALID_ARG";
        case HILS_ERR_UNSUPPORTED: return "HILS_ERR_UNSUPPORTED";
        case HILS_ERR_WORKSPACE: return "HILS_ERR_WORKSPACE";
        case HILS_ERR_CUDA: return "HILS_ERR_CUDA";
        case HILS_ERR_TIMEOUT: return "HILS_ERR_TIMEOUT";
    }
    return "HILS_ERR_UNKNOWN";
}

const char *hils_last_error(void) { return g_last_error.c_str(); }

size_t hils_workspace_size(const hils_params *p, int op) {
    Dims D;
    if (resolve(p, "hils_workspace_size", &D) != HILS_OK) return (size_t)-1;
    switch (op) {
        case HILS_OP_SUMMARY: return 0;
        case HILS_OP_SELECT: return 0;
        case HILS_OP_ATTN_FWD: return attn_fwd_tc_supported(D, p->dtype) ? attn_fwd_tc_workspace(D) : 0;
        case HILS_OP_DECODE: return decode_workspace_bytes(D);
        case HILS_OP_ATTN_BWD: return bwd_workspace_bytes(D, p->dtype);
        default: return (size_t)-1;
    }
}

namespace {

hils_status chunk_summary_common(const char *fn, const hils_params *p, const void *k, const void *q_land,
                                 bool shared_q, int32_t c_begin, int32_t c_end, void *k_sum, float *b_sum,
                                 hils_stream_t stream) {
    Dims D;
    hils_status st = resolve(p, fn, &D);
    if (st != HILS_OK) return st;
    if (c_begin < 0 || c_end < c_begin || c_end > D.Nc)
        return fail(HILS_ERR_INVALID_ARG, "%s: chunk range [%d, %d) outside [0, %d]", fn, c_begin, c_end, D.Nc);
    if (c_end == c_begin) return HILS_OK;  // empty range: nothing is read or written
    HILS_REQUIRE_PTR(k);
    {
        const char *qn = shared_q ? "q_shared" : "q_land";
        if (q_land == nullptr) return fail(HILS_ERR_INVALID_ARG, "%s: %s is NULL", fn, qn);
        if (!aligned16(q_land)) return fail(HILS_ERR_INVALID_ARG, "%s: %s is not 16-byte aligned", fn, qn);
    }
    HILS_REQUIRE_PTR(k_sum);
    HILS_REQUIRE_PTR(b_sum);
    if (D.Hkv > 65535) return fail(HILS_ERR_UNSUPPORTED, "%s: Hkv must be <= 65535", fn);
    return cuda_status(
        launch_chunk_summary(D, p->dtype, k, q_land, shared_q, c_begin, c_end, k_sum, b_sum, (cudaStream_t)stream), fn);
}

}  // namespace

hils_status hils_chunk_summary(const hils_params *p, const void *k, const void *q_land, int32_t c_begin,
                               int32_t c_end, void *k_sum, float *b_sum, hils_stream_t stream) {
    return chunk_summary_common("hils_chunk_summary", p, k, q_land, false, c_begin, c_end, k_sum, b_sum, stream);
}

hils_status hils_chunk_summary_shared_query(const hils_params *p, const void *k, const void *q_shared,
                                            int32_t c_begin, int32_t c_end, void *k_sum, float *b_sum,
                                            hils_stream_t stream) {
    return chunk_summary_common("hils_chunk_summary_shared_query", p, k, q_shared, true, c_begin, c_end, k_sum, b_sum,
                                stream);
}

hils_status hils_select_topk(const hils_params *p, const void *q_hat, const void *k_sum, const float *b_sum,
                             int32_t *idx, float *gap, float *shat, void *workspace, size_t workspace_bytes,
                             hils_stream_t stream) {
    const char *fn = "hils_select_topk";
    Dims D;
    hils_status st = resolve(p, fn, &D);
    if (st != HILS_OK) return st;
    HILS_REQUIRE_PTR(q_hat);
    HILS_REQUIRE_PTR(idx);
    if (D.Nc > 0) {
        HILS_REQUIRE_PTR(k_sum);
        HILS_REQUIRE_PTR(b_sum);
    }
    if (gap != nullptr && !aligned16(gap)) return fail(HILS_ERR_INVALID_ARG, "%s: gap is not 16-byte aligned", fn);
    if (shat != nullptr && !aligned16(shat)) return fail(HILS_ERR_INVALID_ARG, "%s: shat is not 16-byte aligned", fn);
    if (select_smem_bytes(D) > kMaxSmem)
        return fail(HILS_ERR_UNSUPPORTED, "%s: %d chunks x %d heads exceed one CTA's shared memory; use hils_decode",
                    fn, D.Nc, D.G);
    st = check_ws(fn, workspace, workspace_bytes, 0);
    if (st != HILS_OK) return st;
    if (select_tc_supported(D, p->dtype))
        return cuda_status(launch_select_tc(D, q_hat, k_sum, b_sum, idx, gap, shat, (cudaStream_t)stream), fn);
    return cuda_status(launch_select_topk(D, p->dtype, q_hat, k_sum, b_sum, idx, gap, shat, (cudaStream_t)stream), fn);
}

hils_status hils_select_topk_qcal(const hils_params *p, const void *q, const void *w_down, const void *w_up,
                                  int32_t rank, const void *k_sum, const float *b_sum, int32_t *idx, float *gap,
                                  float *shat, hils_stream_t stream) {
    const char *fn = "hils_select_topk_qcal";
    Dims D;
    hils_status st = resolve(p, fn, &D);
    if (st != HILS_OK) return st;
    if (rank != 32) return fail(HILS_ERR_UNSUPPORTED, "%s: rank %d (the fused path takes 32)", fn, rank);
    if (!select_tc_supported(D, p->dtype))
        return fail(HILS_ERR_UNSUPPORTED, "%s: needs bf16, d 128, G <= 4, topk <= 32 and 1..128 candidates per row "
                    "(otherwise form q^ and call hils_select_topk)", fn);
    HILS_REQUIRE_PTR(q);
    HILS_REQUIRE_PTR(w_down);
    HILS_REQUIRE_PTR(w_up);
    HILS_REQUIRE_PTR(k_sum);
    HILS_REQUIRE_PTR(b_sum);
    HILS_REQUIRE_PTR(idx);
    if (gap != nullptr && !aligned16(gap)) return fail(HILS_ERR_INVALID_ARG, "%s: gap is not 16-byte aligned", fn);
    if (shat != nullptr && !aligned16(shat)) return fail(HILS_ERR_INVALID_ARG, "%s: shat is not 16-byte aligned", fn);
    return cuda_status(launch_select_tc_qcal(D, q, w_down, w_up, k_sum, b_sum, idx, gap, shat, (cudaStream_t)stream),
                       fn);
}

hils_status hils_bsa_select_topk(const hils_params *p, const void *q, const void *k, int32_t *idx, float *gap,
                                 float *mass, hils_stream_t stream) {
    const char *fn = "hils_bsa_select_topk";
    Dims D;
    hils_status st = resolve(p, fn, &D);
    if (st != HILS_OK) return st;
    if (D.topk > 32) return fail(HILS_ERR_UNSUPPORTED, "%s: topk %d > 32", fn, D.topk);
    if (bsa_max_candidates(D) > 1024)
        return fail(HILS_ERR_UNSUPPORTED, "%s: %d candidate chunks per row > 1024", fn, bsa_max_candidates(D));
    HILS_REQUIRE_PTR(q);
    HILS_REQUIRE_PTR(k);
    HILS_REQUIRE_PTR(idx);
    if (D.Nc > 0) HILS_REQUIRE_PTR(mass);
    if (gap != nullptr && !aligned16(gap)) return fail(HILS_ERR_INVALID_ARG, "%s: gap is not 16-byte aligned", fn);
    return cuda_status(launch_bsa_select_topk(D, p->dtype, q, k, idx, gap, mass, (cudaStream_t)stream), fn);
}

hils_status hils_attn_fwd(const hils_params *p, const void *q, const void *k, const void *v, const void *q_hat,
                          const void *k_sum, const float *b_sum, const int32_t *idx, void *out, float *lse,
                          void *workspace, size_t workspace_bytes, hils_stream_t stream) {
    const char *fn = "hils_attn_fwd";
    Dims D;
    hils_status st = resolve(p, fn, &D);
    if (st != HILS_OK) return st;
    HILS_REQUIRE_PTR(q);
    HILS_REQUIRE_PTR(k);
    HILS_REQUIRE_PTR(v);
    HILS_REQUIRE_PTR(q_hat);
    HILS_REQUIRE_PTR(idx);
    HILS_REQUIRE_PTR(out);
    HILS_REQUIRE_PTR(lse);
    if (D.Nc > 0) {
        HILS_REQUIRE_PTR(k_sum);
        HILS_REQUIRE_PTR(b_sum);
    }
    const bool tc = attn_fwd_tc_supported(D, p->dtype);
    st = check_ws(fn, workspace, workspace_bytes, tc ? attn_fwd_tc_workspace(D) : 0);
    if (st != HILS_OK) return st;
    if (tc)
        return cuda_status(
            launch_attn_fwd_tc(D, q, k, v, q_hat, k_sum, b_sum, idx, out, lse, workspace, (cudaStream_t)stream), fn);
    return cuda_status(
        launch_attn_fwd_simt(D, p->dtype, q, k, v, q_hat, k_sum, b_sum, idx, out, lse, (cudaStream_t)stream), fn);
}

hils_status hils_attn_fwd_shat(const hils_params *p, const void *q, const void *k, const void *v, const int32_t *idx,
                               const float *shat, void *out, float *lse, hils_stream_t stream) {
    const char *fn = "hils_attn_fwd_shat";
    Dims D;
    hils_status st = resolve(p, fn, &D);
    if (st != HILS_OK) return st;
    if (!attn_fwd_shat_supported(D, p->dtype))
        return fail(HILS_ERR_UNSUPPORTED, "%s: needs bf16, d 128, S 64, 128 %% G == 0, topk <= 32 and at most 8192 "
                    "chunks (otherwise call hils_attn_fwd)", fn);
    HILS_REQUIRE_PTR(q);
    HILS_REQUIRE_PTR(k);
    HILS_REQUIRE_PTR(v);
    HILS_REQUIRE_PTR(idx);
    HILS_REQUIRE_PTR(shat);
    HILS_REQUIRE_PTR(out);
    HILS_REQUIRE_PTR(lse);
    return cuda_status(launch_attn_fwd_tc_shat(D, q, k, v, idx, shat, out, lse, (cudaStream_t)stream), fn);
}

hils_status hils_decode(const hils_params *p, const void *q, const void *q_hat, const void *k_cache,
                        const void *v_cache, const void *k_sum, const float *b_sum, void *out, float *lse,
                        int32_t *idx_out, void *workspace, size_t workspace_bytes, hils_stream_t stream) {
    const char *fn = "hils_decode";
    Dims D;
    hils_status st = resolve(p, fn, &D);
    if (st != HILS_OK) return st;
    if (D.T < 1 || D.T > 8 || D.q_pos0 != D.L - D.T)
        return fail(HILS_ERR_INVALID_ARG, "%s: needs 1 <= T <= 8 and q_pos0 == L-T (got T=%d q_pos0=%d L=%d)", fn, D.T,
                    D.q_pos0, D.L);
    HILS_REQUIRE_PTR(q);
    HILS_REQUIRE_PTR(q_hat);
    HILS_REQUIRE_PTR(k_cache);
    HILS_REQUIRE_PTR(v_cache);
    HILS_REQUIRE_PTR(out);
    HILS_REQUIRE_PTR(lse);
    if (D.Nc > 0) {
        HILS_REQUIRE_PTR(k_sum);
        HILS_REQUIRE_PTR(b_sum);
    }
    if (idx_out != nullptr && !aligned16(idx_out))
        return fail(HILS_ERR_INVALID_ARG, "%s: idx_out is not 16-byte aligned", fn);
    if (D.Hkv > 65535) return fail(HILS_ERR_UNSUPPORTED, "%s: Hkv must be <= 65535", fn);
    if (!decode_supported(D))
        return fail(HILS_ERR_UNSUPPORTED, "%s: %d candidate chunks with G=%d, topk=%d exceed the selection buffers", fn,
                    D.Nc, D.G, D.topk);
    if (!decode_multi_supported(D, p->dtype, q, q_hat, k_cache, v_cache, k_sum))
        return fail(HILS_ERR_UNSUPPORTED, "%s: T=%d > 1 needs bf16, d 128, S 64, G <= 8, topk <= 32 and 16-byte "
                    "aligned q, q_hat, caches and k_sum", fn, D.T);
    st = check_ws(fn, workspace, workspace_bytes, decode_workspace_bytes(D));
    if (st != HILS_OK) return st;
    return cuda_status(launch_decode(D, p->dtype, q, q_hat, k_cache, v_cache, k_sum, b_sum, out, lse, idx_out, workspace,
                                     (cudaStream_t)stream),
                       fn);
}

hils_status hils_attn_bwd(const hils_params *p, const void *q, const void *k, const void *v, const void *q_hat,
                          const void *q_land, const void *k_sum, const float *b_sum, const int32_t *idx,
                          const void *out, const float *lse, const void *dout, void *dq, void *dk, void *dv,
                          void *dq_hat, void *dq_land, void *workspace, size_t workspace_bytes,
                          hils_stream_t stream) {
    const char *fn = "hils_attn_bwd";
    Dims D;
    hils_status st = resolve(p, fn, &D);
    if (st != HILS_OK) return st;
    if (D.q_pos0 != 0 || D.T != D.L)
        return fail(HILS_ERR_INVALID_ARG, "%s: needs a self-attention prefill (q_pos0 == 0, T == L)", fn);
    HILS_REQUIRE_PTR(q);
    HILS_REQUIRE_PTR(k);
    HILS_REQUIRE_PTR(v);
    HILS_REQUIRE_PTR(q_hat);
    HILS_REQUIRE_PTR(idx);
    HILS_REQUIRE_PTR(out);
    HILS_REQUIRE_PTR(lse);
    HILS_REQUIRE_PTR(dout);
    HILS_REQUIRE_PTR(dq);
    HILS_REQUIRE_PTR(dk);
    HILS_REQUIRE_PTR(dv);
    HILS_REQUIRE_PTR(dq_hat);
    if (D.Nc > 0) {
        HILS_REQUIRE_PTR(q_land);
        HILS_REQUIRE_PTR(k_sum);
        HILS_REQUIRE_PTR(b_sum);
        HILS_REQUIRE_PTR(dq_land);
    }
    if (D.Hkv > 65535) return fail(HILS_ERR_UNSUPPORTED, "%s: Hkv must be <= 65535", fn);
    if (bwd_smem_bytes(D) > kMaxSmem)
        return fail(HILS_ERR_UNSUPPORTED, "%s: S=%d, d=%d, G=%d exceed one CTA's shared memory", fn, D.S, D.d, D.G);
    st = check_ws(fn, workspace, workspace_bytes, bwd_workspace_bytes(D, p->dtype));
    if (st != HILS_OK) return st;
    return cuda_status(launch_attn_bwd(D, p->dtype, q, k, v, q_hat, q_land, k_sum, b_sum, idx, out, lse, dout, dq, dk,
                                       dv, dq_hat, dq_land, workspace, (cudaStream_t)stream),
                       fn);
}

hils_status hils_test_wait_expiry(uint32_t max_polls, int32_t arrive_first, hils_stream_t stream) {
    const char *fn = "hils_test_wait_expiry";
    if (max_polls < 1 || max_polls > HILS_TEST_WAIT_MAX_POLLS)
        return fail(HILS_ERR_INVALID_ARG, "%s: max_polls=%u outside [1, %u]", fn, max_polls,
                    (unsigned)HILS_TEST_WAIT_MAX_POLLS);
    return cuda_status(launch_wait_expiry(max_polls, arrive_first != 0, (cudaStream_t)stream), fn);
}

hils_status hils_check(hils_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_status(e, "hils_check");
    return check_device_errors();
}

}  // extern "C"
