// Device-side helpers shared by the HiLS kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hils.h"

namespace hils {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Sizes of one problem, resolved on the host (tau filled in, derived counts computed).
struct Dims {
    int B, T, L, Hq, Hkv, d, S, topk, W, q_pos0;
    int G, Nc;
    float tau;
};

// Row of the landmark query used for (b, query head h, chunk c): q_land [B, Hq, Nc, d], or with a
// shared query (one learned vector per head, Sec. 4 "landmark tokens" alternative) q_land [Hq, d].
__host__ __device__ __forceinline__ size_t landmark_row(const Dims &D, int shared_q, int b, int h, int c) {
    return shared_q ? (size_t)h : ((size_t)b * D.Hq + h) * D.Nc + c;
}

__host__ __device__ __forceinline__ int window_left(int pos, int W, int S) {
    int e = pos - W + 1;
    if (e < 0) e = 0;
    return (e / S) * S;
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

// Float -> uint32 whose unsigned order equals the float order (for radix / sort keys).
__device__ __forceinline__ uint32_t float_order_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float float_from_order_key(uint32_t k) {
    uint32_t u = (k & 0x80000000u) ? (k & 0x7fffffffu) : ~k;
    return __uint_as_float(u);
}

// Sort key that orders by (value descending, index ascending) under an ascending 64-bit sort.
__device__ __forceinline__ uint64_t desc_value_key(float v, uint32_t index) {
    return ((uint64_t)(~float_order_key(v)) << 32) | (uint64_t)index;
}
__device__ __forceinline__ float desc_key_value(uint64_t key) { return float_from_order_key(~(uint32_t)(key >> 32)); }
__device__ __forceinline__ uint32_t desc_key_index(uint64_t key) { return (uint32_t)key; }

// Ascending bitonic sort of n (a power of two) 64-bit keys in shared memory by the whole block.
__device__ __forceinline__ void block_bitonic_sort(uint64_t *keys, int n) {
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncthreads();
            for (int t = threadIdx.x; t < (n >> 1); t += blockDim.x) {
                int lo = 2 * t - (t & (stride - 1));
                int hi = lo + stride;
                bool up = ((lo & size) == 0);
                uint64_t a = keys[lo], b = keys[hi];
                if ((a > b) == up) { keys[lo] = b; keys[hi] = a; }
            }
        }
    }
    __syncthreads();
}

// Ascending bitonic sort of 32*NPL 64-bit keys held in registers by one warp; element e of the
// sequence is v[e % NPL] of lane e / NPL. No shared memory, no barriers.
template <int NPL>
__device__ __forceinline__ void warp_bitonic_sort(uint64_t (&v)[NPL]) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int size = 2; size <= 32 * NPL; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            if (stride >= NPL) {
                const int ls = stride / NPL;
                const bool lower = (lane & ls) == 0;
#pragma unroll
                for (int i = 0; i < NPL; ++i) {
                    const int e = lane * NPL + i;
                    const bool up = (e & size) == 0;
                    const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v[i], ls);
                    const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v[i] >> 32), ls);
                    const uint64_t p = ((uint64_t)hi << 32) | lo;
                    const bool keep_min = (lower == up);
                    v[i] = keep_min ? (v[i] < p ? v[i] : p) : (v[i] > p ? v[i] : p);
                }
            } else {
#pragma unroll
                for (int i = 0; i < NPL; ++i) {
                    const int j = i ^ stride;
                    if (j > i) {
                        const int e = lane * NPL + i;
                        const bool up = (e & size) == 0;
                        if ((v[i] > v[j]) == up) {
                            const uint64_t t = v[i];
                            v[i] = v[j];
                            v[j] = t;
                        }
                    }
                }
            }
        }
    }
}

// Block (x, y, z) of a grid, renumbered so that x varies slowest in launch order (blocks are launched
// with x fastest): returns the x, y and z this block works on. With work that shrinks as x grows, every
// (y, z) slice's heaviest blocks then start first and the grid's tail is made of light ones.
struct XSlowest {
    int x, y, z;
};
__device__ __forceinline__ XSlowest x_slowest_block() {
    const unsigned lin = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
    const unsigned nyz = gridDim.y * gridDim.z;
    const unsigned rem = lin % nyz;
    return XSlowest{(int)(lin / nyz), (int)(rem % gridDim.y), (int)(rem / gridDim.y)};
}

// Programmatic dependent launch: a kernel launched with launch_pdl may start while the grid before it
// on the stream is still running; grid_dep_wait() blocks until that grid has completed and its memory
// is visible (a no-op for an ordinary launch). Every CTA of such a kernel calls it before reading what
// the previous grid wrote and before it exits, so completion stays transitive along the chain.
// grid_dep_launch() lets the next PDL-launched grid start early.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" :::); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Number of SMs of the current device (cached per device ordinal).
inline int num_sms() {
    static int cache[256] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

__host__ __device__ __forceinline__ int next_pow2(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

// Load `n` consecutive elements (n a multiple of 8 for bf16, 4 for fp32; 16-byte aligned) as floats.
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float *out) {
    uint4 raw = *reinterpret_cast<const uint4 *>(p);
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&raw);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        float2 f = __bfloat1622float2(h[t]);
        out[2 * t] = f.x;
        out[2 * t + 1] = f.y;
    }
}
__device__ __forceinline__ void load8(const float *p, float *out) {
    float4 a = *reinterpret_cast<const float4 *>(p);
    float4 b = *reinterpret_cast<const float4 *>(p + 4);
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
    out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}

}  // namespace hils
