// hils_decode_noalloc: the decode step with its scratch memory in a static device array.
//
// hils_decode needs a caller-provided workspace. Some callers cannot provide one: a serving engine
// whose memory planner owns the whole device and forbids allocations by libraries, a binding from a
// language runtime that hands over tensor pointers but exposes no device allocator, or a latency-
// critical decode loop that cannot afford the device-wide synchronisation cudaMalloc may imply. For
// them this entry point takes the same inputs and outputs and keeps the scratch in a file-scope
// __device__ array of HILS_DECODE_NOALLOC_MAX_BYTES, which every GPU that loads the library holds
// until the process exits. It allocates nothing (no cudaMalloc/cudaFree, no allocating library call).
#include <stdio.h>

#include <mutex>

#include "internal.h"

namespace hils {
void record_error(const char *msg);
}

using namespace hils;

namespace {

// The scratch of every hils_decode_noalloc call on this device. In host code this name is only a
// host-side stand-in for the symbol: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_decode_scratch[HILS_DECODE_NOALLOC_MAX_BYTES];

constexpr int kMaxDevices = 256;
std::mutex g_setup_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Once per device, with that device current: resolve the array's device address.
hils_status scratch_for_current_device(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        record_error("hils_decode_noalloc: cudaGetDevice failed");
        return HILS_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) {
        record_error("hils_decode_noalloc: device ordinal out of range");
        return HILS_ERR_UNSUPPORTED;
    }
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (g_scratch_addr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || p == nullptr) {
            record_error("hils_decode_noalloc: cudaGetSymbolAddress of the static scratch failed");
            return HILS_ERR_CUDA;
        }
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return HILS_OK;
}

}  // namespace

extern "C" hils_status hils_decode_noalloc(const hils_params *p, const void *q, const void *q_hat,
                                           const void *k_cache, const void *v_cache, const void *k_sum,
                                           const float *b_sum, void *out, float *lse, int32_t *idx_out,
                                           hils_stream_t stream) {
    const size_t need = hils_workspace_size(p, HILS_OP_DECODE);
    if (need == (size_t)-1) return HILS_ERR_INVALID_ARG;  // message already recorded by the size query
    if (need > (size_t)HILS_DECODE_NOALLOC_MAX_BYTES) {
        char buf[256];
        snprintf(buf, sizeof(buf),
                 "hils_decode_noalloc: these sizes need %zu bytes of scratch but the static buffer holds %zu; "
                 "use hils_decode with a caller workspace",
                 need, (size_t)HILS_DECODE_NOALLOC_MAX_BYTES);
        record_error(buf);
        return HILS_ERR_UNSUPPORTED;
    }
    void *scratch = nullptr;
    hils_status st = scratch_for_current_device(&scratch);
    if (st != HILS_OK) return st;
    return hils_decode(p, q, q_hat, k_cache, v_cache, k_sum, b_sum, out, lse, idx_out, scratch,
                       (size_t)HILS_DECODE_NOALLOC_MAX_BYTES, stream);
}
