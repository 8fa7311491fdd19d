// common.cuh -- shared device helpers of the vnsa CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/vnsa.h"

namespace vnsa {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Device status word: the first error a kernel detects wins.
__device__ __forceinline__ void report(uint32_t *status, uint32_t code) {
    if (status) atomicCAS(status, 0u, code);
}

// Workspace counters written by the partition kernel.
struct Counts {
    int n_vision;    // N_v
    int n_text;      // N_t
    int contiguous;  // 1 if the vision tokens are one run of positions
    int vis_base;    // position of the first vision token (if contiguous)
    int nb;          // complete blocks N_v / block
    int pad[3];      // (decode step state)
    int txt_contiguous;  // 1 if the text tokens are one run of positions
    int txt_base;        // position of the first text token (if contiguous)
    int nc;              // compression blocks (N_v - block) / stride + 1 (= nb at stride block)
};

// Compression blocks visible to vision query i: those whose last token
// c*S + B - 1 is at or before i, at most nc.  With S = B this is (i + 1) / B.
__host__ __device__ __forceinline__ int cmp_visible(int i, int B, int S, int nc) {
    if (i < B - 1) return 0;
    const int c = (i - B + 1) / S + 1;
    return c < nc ? c : nc;
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Load 8 consecutive elements as floats (16-byte aligned for bf16, 32 for fp32).
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&x)[8]) {
    uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void load8(const float *p, float (&x)[8]) {
    float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }

// Programmatic dependent launch: a kernel launched with the programmatic
// stream-serialisation attribute may start while the previous kernel on its
// stream drains; this waits until that kernel has completed and its writes are
// visible.  Without the attribute it returns at once.
__device__ __forceinline__ void wait_prior_grid() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

}  // namespace vnsa
