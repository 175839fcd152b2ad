// Warp-level tensor-core helpers (ldmatrix, mma.sync m16n8k16 bf16 -> fp32) and consumer-group
// barriers, as inline PTX, for the kernels whose contractions are too narrow for tcgen05 tiles
// (one query row per head in decode, G heads per chunk in the summaries, small reductions).
//
// Fragment layout of mma.sync.m16n8k16.row.col (lane = 4 * g8 + t4):
//   A (16 x 16, row-major): a0 = A[g8][2t4..2t4+1], a1 = A[g8+8][..], a2 = A[g8][2t4+8..], a3 = A[g8+8][2t4+8..]
//   B (16 x 8, col-major):  b0 = B[2t4..2t4+1][g8], b1 = B[2t4+8..2t4+9][g8]
//   C (16 x 8, fp32):       c0, c1 = C[g8][2t4, 2t4+1], c2, c3 = C[g8+8][2t4, 2t4+1]
// ldmatrix .x4 takes matrix m's eight row addresses from lanes 8m .. 8m+7; without .trans lane t
// receives row t/4, elements 2(t%4), 2(t%4)+1 of each matrix, with .trans the transpose.
#pragma once

#include <stdint.h>

namespace hils {

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// c += a (16x16, row) * b (16x8, col), bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Named barrier 1, completed by NT arriving threads (the whole warps that execute it).
template <int NT>
__device__ __forceinline__ void bar_group() {
    asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory");
}
// The same barrier, also returning to each arriving thread whether any of them passed pred.
template <int NT>
__device__ __forceinline__ bool bar_group_any(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "bar.red.or.pred p, 1, %2, q;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "n"(NT)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ uint32_t ld_u32(const void *p) { return *reinterpret_cast<const uint32_t *>(p); }

}  // namespace hils
