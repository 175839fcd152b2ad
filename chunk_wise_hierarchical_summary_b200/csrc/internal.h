// Internal launch interface between the C ABI (hils_abi.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "common.cuh"

namespace hils {

// Each launcher enqueues its kernels on `stream` and returns the launch status.
cudaError_t launch_chunk_summary(const Dims &D, int dtype, const void *k, const void *q_land, bool shared_q,
                                 int c_begin, int c_end, void *k_sum, float *b_sum, cudaStream_t stream);

size_t select_smem_bytes(const Dims &D);
cudaError_t launch_select_topk(const Dims &D, int dtype, const void *q_hat, const void *k_sum, const float *b_sum,
                               int *idx, float *gap, float *shat, cudaStream_t stream);

cudaError_t launch_attn_fwd(const Dims &D, int dtype, const void *q, const void *k, const void *v, const void *q_hat,
                            const void *k_sum, const float *b_sum, const int *idx, void *out, float *lse,
                            cudaStream_t stream);

size_t decode_workspace_bytes(const Dims &D);
cudaError_t launch_decode(const Dims &D, int dtype, const void *q, const void *q_hat, const void *k_cache,
                          const void *v_cache, const void *k_sum, const float *b_sum, void *out, float *lse,
                          int *idx_out, void *ws, cudaStream_t stream);

// Device-side error words (bit set when a bounded wait expired); reading with clear resets them.
unsigned int decode_error_flags(bool clear);

size_t bwd_workspace_bytes(const Dims &D, int dtype);
cudaError_t launch_attn_bwd(const Dims &D, int dtype, const void *q, const void *k, const void *v, const void *q_hat,
                            const void *q_land, const void *k_sum, const float *b_sum, const int *idx,
                            const void *out, const float *lse, const void *dout, void *dq, void *dk, void *dv,
                            void *dq_hat, void *dq_land, void *ws, cudaStream_t stream);

}  // namespace hils
