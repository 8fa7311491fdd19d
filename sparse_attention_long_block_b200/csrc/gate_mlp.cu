// gate_mlp.cu -- the gate perceptron of the hybrid layer: the branch logits of
// every token from the layer input.
//
// "VideoNSA: Native Sparse Attention Scales Video Understanding" (paper notes),
// section "Method": a two-layer MLP with a sigmoid gives each head its own
// weights for the compression, selection and window branches.  Read here as
//   logits_t = SiLU(x_t . G1 + c1) . G2 + c2,
// x_t the layer input (h_q * d wide), G1 [D][H], G2 [H][3 h_q]; column 3h + c is
// the logit of branch c (cmp, slc, swa) of head h, i.e. the gate-logit layout
// the attention kernels read.  In bf16 the hidden activations are rounded to
// bf16: they are the operand of the second product.
//
// Tensor-core kernel (bf16, D a multiple of 64, H in {64, 128, 192, 256}, 3 h_q
// <= 256): persistent CTAs over 128-token tiles.  Warp 0 streams x tiles
// (128 x 64) and G1 tiles (64 x H) by TMA through a 3-stage ring; one thread of
// warp 1 issues the tcgen05 MMAs of the first layer into TMEM (H fp32
// columns); warps 2-5 add c1, apply SiLU, round to bf16 and write the hidden
// row back into the first H/2 TMEM columns as packed pairs, which is the A
// operand of the second layer's MMA against G2 (staged once per CTA in shared
// memory); the same warps add c2 and store the logits.  The first layer reads
// x once: the kernel is bound by HBM (D * 2 bytes per token) or by the tensor
// pipe (2 D H flops per token), whichever is slower.
//
// Other settings run the SIMT kernel: 8 tokens per CTA, fp32 accumulation.
#include <cuda.h>
#include <cuda_bf16.h>
#include <math.h>

#include "kernels.h"
#include "tc_attn.h"
#include "tc_ptx.cuh"

namespace vnsa {
namespace {

constexpr int kGmThreads = 192;
constexpr int kGmRows = 128;         // tokens per tile (MMA M)
constexpr int kGmStages = 3;
constexpr uint32_t kGmA = 16384;     // x tile: 128 tokens x 64 inputs, bf16
constexpr int kGmMaxSmem = 227 * 1024;

__device__ __forceinline__ float silu_g(float z) { return z / (1.f + expf(-z)); }

struct GmLayout {
    uint32_t stage_bytes, g2, c1, c2, bar, total;
};

// Shared memory of the tensor-core kernel (offsets from a 1024-byte aligned
// base): the stage ring (x tile, then H/64 G1 slabs of 64 x 64), G2 as a
// K-major 128-byte swizzled [n_out_pad][H] operand (H/64 chunks of n_out_pad
// rows x 128 bytes), c1, c2, then the barriers.
__host__ __device__ inline GmLayout gm_layout(int hidden, int n_out_pad) {
    GmLayout l;
    l.stage_bytes = kGmA + (uint32_t)hidden * 128u;
    l.g2 = kGmStages * l.stage_bytes;
    l.c1 = l.g2 + (uint32_t)n_out_pad * (uint32_t)hidden * 2u;
    l.c2 = l.c1 + (uint32_t)hidden * 4u;
    l.bar = (l.c2 + (uint32_t)n_out_pad * 4u + 7u) & ~7u;
    l.total = l.bar + 128u;
    return l;
}

// barrier slots
constexpr int GB_FULL = 0, GB_EMPTY = 3, GB_ACC1 = 6, GB_HID = 7, GB_ACC2 = 8, GB_FINAL = 9;

struct GateTc {
    CUtensorMap tm_x;    // x [n][dm], boxes 64 x 128
    CUtensorMap tm_g1;   // G1 [dm][hidden], boxes 64 x 64
    const __nv_bfloat16 *g2;
    const float *c1, *c2;
    float *out;
    uint32_t *status;
    int n, dm, hidden, n_out, n_out_pad, tiles, acc2_col;
    uint32_t tmem_cols;
};

__global__ void __launch_bounds__(kGmThreads, 1) gate_mlp_tc_kernel(const __grid_constant__ GateTc P) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = ptx::smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t *base = smem_raw + pad;
    const uint32_t base_u32 = raw + pad;
    const GmLayout Lo = gm_layout(P.hidden, P.n_out_pad);
    auto bar = [&](int i) { return base_u32 + Lo.bar + 8u * (uint32_t)i; };
    uint32_t *tmem_slot = (uint32_t *)(base + Lo.bar + 80);
    volatile int *abort = (volatile int *)(base + Lo.bar + 88);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kc_n = P.dm / 64;
    const int H = P.hidden;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kGmStages; ++s) {
            ptx::mbar_init(bar(GB_FULL + s), 1);
            ptx::mbar_init(bar(GB_EMPTY + s), 1);
        }
        ptx::mbar_init(bar(GB_ACC1), 1);
        ptx::mbar_init(bar(GB_HID), 4);  // one arrival per epilogue warp
        ptx::mbar_init(bar(GB_ACC2), 1);
        ptx::mbar_init(bar(GB_FINAL), 1);
        *abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(tmem_slot), P.tmem_cols);
        ptx::tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&P.tm_x);
        ptx::prefetch_tmap(&P.tm_g1);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---- producer: x and G1 tiles of every (tile, 64-input chunk)
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x) {
                for (int kc = 0; kc < kc_n; ++kc, ++it) {
                    const uint32_t s = it % kGmStages;
                    if (it >= (uint32_t)kGmStages &&
                        !ptx::mbar_wait(bar(GB_EMPTY + s), ((it / kGmStages) - 1) & 1, abort,
                                        P.status)) {
                        ok = false;
                        break;
                    }
                    const uint32_t st = base_u32 + s * Lo.stage_bytes;
                    ptx::mbar_expect_tx(bar(GB_FULL + s), Lo.stage_bytes);
                    ptx::tma_load_2d(st, &P.tm_x, bar(GB_FULL + s), kc * 64, tile * kGmRows);
                    for (int hb = 0; hb < H / 64; ++hb)
                        ptx::tma_load_2d(st + kGmA + (uint32_t)hb * 8192u, &P.tm_g1,
                                         bar(GB_FULL + s), hb * 64, kc * 64);
                }
            }
            // no load may still be landing in shared memory when the CTA ends
            for (uint32_t back = 1; back <= (uint32_t)kGmStages && back <= it; ++back) {
                const uint32_t u = it - back;
                if (!ptx::mbar_drain(bar(GB_FULL + u % kGmStages), (u / kGmStages) & 1)) break;
            }
        }
    } else if (warp == 1) {
        // ---- MMA issuer
        if (lane == 0) {
            const uint32_t idesc1 = ptx::idesc_f16kind(kGmRows, H, 0, 1, 1u);
            const uint32_t idesc2 = ptx::idesc_f16kind(kGmRows, P.n_out_pad, 0, 0, 1u);
            const uint32_t chunk2 = (uint32_t)P.n_out_pad * 128u;
            uint32_t it = 0, nt = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < P.tiles; tile += gridDim.x, ++nt) {
                for (int kc = 0; kc < kc_n; ++kc, ++it) {
                    const uint32_t s = it % kGmStages;
                    if (!ptx::mbar_wait(bar(GB_FULL + s), (it / kGmStages) & 1, abort, P.status)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t st = base_u32 + s * Lo.stage_bytes;
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        ptx::mma_ss(tmem, ptx::sdesc_sw128(st + (uint32_t)k * 32u, 16, 1024),
                                    ptx::sdesc_sw128(st + kGmA + (uint32_t)k * 2048u, 8192, 1024),
                                    idesc1, (kc > 0 || k > 0) ? 1u : 0u);
                    ptx::mma_commit(bar(GB_EMPTY + s));
                }
                if (!ok) break;
                ptx::mma_commit(bar(GB_ACC1));
                // second layer, once the hidden row is back in TMEM as bf16 pairs
                if (!ptx::mbar_wait(bar(GB_HID), nt & 1, abort, P.status)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                for (int k = 0; k < H / 16; ++k)
                    ptx::mma_ts(tmem + (uint32_t)P.acc2_col, tmem + (uint32_t)k * 8u,
                                ptx::sdesc_sw128(base_u32 + Lo.g2 + (uint32_t)(k >> 2) * chunk2 +
                                                     (uint32_t)(k & 3) * 32u,
                                                 16, 1024),
                                idesc2, k > 0 ? 1u : 0u);
                ptx::mma_commit(bar(GB_ACC2));
            }
            // every MMA this thread issued has completed once this barrier flips
            ptx::mma_commit(bar(GB_FINAL));
            ptx::mbar_drain(bar(GB_FINAL), 0);
        }
        __syncwarp();
    } else {
        // ---- epilogue warps 2-5: thread owns MMA row / TMEM lane `row`
        const int wq = warp & 3;
        const int row = wq * 32 + lane;
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        const int et = threadIdx.x - 64;  // 0..127
        float *c1s = (float *)(base + Lo.c1);
        float *c2s = (float *)(base + Lo.c2);
        for (int x = et; x < H; x += 128) c1s[x] = P.c1[x];
        for (int x = et; x < P.n_out_pad; x += 128) c2s[x] = x < P.n_out ? P.c2[x] : 0.f;
        // G2 -> K-major operand: row o (output), 8 hidden elements per 16 bytes
        const int units = P.n_out_pad * (H / 8);
        for (int u = et; u < units; u += 128) {
            const int o = u / (H / 8), hc0 = (u % (H / 8)) * 8;
            uint4 val = make_uint4(0u, 0u, 0u, 0u);
            if (o < P.n_out) {
                __nv_bfloat16 e8[8];
#pragma unroll
                for (int z = 0; z < 8; ++z) e8[z] = P.g2[(size_t)(hc0 + z) * P.n_out + o];
                val = *reinterpret_cast<const uint4 *>(e8);
            }
            const int c = (hc0 & 63) >> 3;
            *reinterpret_cast<uint4 *>(base + Lo.g2 + (size_t)(hc0 >> 6) * P.n_out_pad * 128 +
                                       o * 128 + ((c ^ (o & 7)) << 4)) = val;
        }
        ptx::fence_proxy_async();
        ptx::named_bar_sync(1, 128);
        uint32_t nt = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < P.tiles; tile += gridDim.x, ++nt) {
            bool r = ptx::mbar_wait(bar(GB_ACC1), nt & 1, abort, P.status);
            ok = __all_sync(0xffffffffu, r && ok);
            if (!ok) break;
            ptx::tc_fence_after();
            for (int c64 = 0; c64 < H / 64; ++c64) {
                float a[32], b[32];
                ptx::tmem_ld32(tmem + lane_base + (uint32_t)c64 * 64u, a);
                ptx::tmem_ld32(tmem + lane_base + (uint32_t)c64 * 64u + 32u, b);
                ptx::tmem_wait_ld();
                uint32_t pk[32];
#pragma unroll
                for (int z = 0; z < 16; ++z) {
                    const float *cb = c1s + c64 * 64;
                    __nv_bfloat162 h0 = __floats2bfloat162_rn(silu_g(a[2 * z] + cb[2 * z]),
                                                              silu_g(a[2 * z + 1] + cb[2 * z + 1]));
                    __nv_bfloat162 h1 = __floats2bfloat162_rn(
                        silu_g(b[2 * z] + cb[32 + 2 * z]), silu_g(b[2 * z + 1] + cb[32 + 2 * z + 1]));
                    pk[z] = *reinterpret_cast<uint32_t *>(&h0);
                    pk[16 + z] = *reinterpret_cast<uint32_t *>(&h1);
                }
                // hidden elements 64 c64 .. 64 c64 + 63 -> columns 32 c64 .. 32 c64 + 31
                // (columns of this thread's row already read)
                ptx::tmem_st32u(tmem + lane_base + (uint32_t)c64 * 32u, pk);
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar(GB_HID));
            r = ptx::mbar_wait(bar(GB_ACC2), nt & 1, abort, P.status);
            ok = __all_sync(0xffffffffu, r && ok);
            if (!ok) break;
            ptx::tc_fence_after();
            const long long token = (long long)tile * kGmRows + row;
            for (int c = 0; c * 32 < P.n_out_pad; ++c) {
                float o[32];
                ptx::tmem_ld32(tmem + lane_base + (uint32_t)(P.acc2_col + c * 32), o);
                ptx::tmem_wait_ld();
                if (token < P.n) {
                    float *orow = P.out + (size_t)token * P.n_out;
#pragma unroll
                    for (int z = 0; z < 32; ++z) {
                        const int col = c * 32 + z;
                        if (col < P.n_out) orow[col] = o[z] + c2s[col];
                    }
                }
            }
            ptx::tc_fence_before();
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, P.tmem_cols);
}

// SIMT kernel: 8 tokens per CTA of 256 threads; the hidden rows in shared
// memory, x in chunks of 256 inputs.
constexpr int kGsTok = 8;
constexpr int kGsChunk = 256;

template <typename T>
__global__ void __launch_bounds__(256) gate_mlp_simt_kernel(int n, int dm, int H, int n_out,
                                                            const T *__restrict__ x,
                                                            const T *__restrict__ g1,
                                                            const float *__restrict__ c1,
                                                            const T *__restrict__ g2,
                                                            const float *__restrict__ c2,
                                                            float *__restrict__ out) {
    __shared__ float xs[kGsTok][kGsChunk];
    __shared__ float hid[kGsTok][kCmpMlpMaxHidden];
    const int t0 = blockIdx.x * kGsTok;
    const int nt = min(kGsTok, n - t0);
    for (int a0 = 0; a0 < H; a0 += 256) {
        const int a = a0 + threadIdx.x;
        float acc[kGsTok];
#pragma unroll
        for (int t = 0; t < kGsTok; ++t) acc[t] = 0.f;
        for (int e0 = 0; e0 < dm; e0 += kGsChunk) {
            __syncthreads();
            for (int u = threadIdx.x; u < kGsTok * kGsChunk; u += 256) {
                const int t = u / kGsChunk, e = e0 + u % kGsChunk;
                xs[t][u % kGsChunk] = (t < nt && e < dm) ? to_f(x[(size_t)(t0 + t) * dm + e]) : 0.f;
            }
            __syncthreads();
            if (a < H) {
                const int ee = min(kGsChunk, dm - e0);
                for (int e = 0; e < ee; ++e) {
                    const float w = to_f(g1[(size_t)(e0 + e) * H + a]);
#pragma unroll
                    for (int t = 0; t < kGsTok; ++t) acc[t] = fmaf(xs[t][e], w, acc[t]);
                }
            }
        }
        if (a < H) {
#pragma unroll
            for (int t = 0; t < kGsTok; ++t) {
                float h = silu_g(acc[t] + c1[a]);
                if (sizeof(T) == 2) h = __bfloat162float(__float2bfloat16_rn(h));
                hid[t][a] = h;
            }
        }
    }
    __syncthreads();
    for (int o = threadIdx.x; o < n_out; o += 256) {
        float acc[kGsTok];
#pragma unroll
        for (int t = 0; t < kGsTok; ++t) acc[t] = c2[o];
        for (int a = 0; a < H; ++a) {
            const float w = to_f(g2[(size_t)a * n_out + o]);
#pragma unroll
            for (int t = 0; t < kGsTok; ++t) acc[t] = fmaf(hid[t][a], w, acc[t]);
        }
        for (int t = 0; t < nt; ++t) out[(size_t)(t0 + t) * n_out + o] = acc[t];
    }
}

uint32_t pow2_cols(int c) {
    uint32_t p = 32;
    while (p < (uint32_t)c) p <<= 1;
    return p;
}

}  // namespace

cudaError_t launch_gate_mlp(int dtype, int n, int dm, int hidden, int n_out, const void *x,
                            const void *g1, const float *c1, const void *g2, const float *c2,
                            float *out, uint32_t *status, cudaStream_t s, int *launches) {
    if (n < 1) return cudaSuccess;
    if (hidden < 1 || hidden > kCmpMlpMaxHidden || dm < 1 || n_out < 1)
        return cudaErrorInvalidValue;
    const int n_out_pad = (n_out + 15) / 16 * 16;
    const int out_cols = (n_out_pad + 31) / 32 * 32;
    const GmLayout lo = gm_layout(hidden, n_out_pad);
    const bool tc = dtype == VNSA_BF16 && dm % 64 == 0 && hidden % 64 == 0 && hidden <= 256 &&
                    n_out_pad <= 256 && lo.total + 1024 <= (uint32_t)kGmMaxSmem &&
                    pow2_cols(hidden + out_cols) <= 512;
    if (tc) {
        GateTc P;
        memset(&P, 0, sizeof(P));
        if (tma_map_2d_bf16(&P.tm_x, x, dm, n, 64, kGmRows) &&
            tma_map_2d_bf16(&P.tm_g1, g1, hidden, dm, 64, 64)) {
            P.g2 = (const __nv_bfloat16 *)g2;
            P.c1 = c1;
            P.c2 = c2;
            P.out = out;
            P.status = status;
            P.n = n;
            P.dm = dm;
            P.hidden = hidden;
            P.n_out = n_out;
            P.n_out_pad = n_out_pad;
            P.tiles = (n + kGmRows - 1) / kGmRows;
            P.acc2_col = hidden;
            P.tmem_cols = pow2_cols(hidden + out_cols);
            int dev = 0, sms = 148;
            cudaGetDevice(&dev);
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            const int smem = (int)lo.total + 1024;
            cudaError_t e = cudaFuncSetAttribute(gate_mlp_tc_kernel,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (e != cudaSuccess) return e;
            gate_mlp_tc_kernel<<<min(P.tiles, sms), kGmThreads, smem, s>>>(P);
            if (launches) ++*launches;
            return cudaGetLastError();
        }
        // no tensor maps (driver entry point missing): the SIMT kernel
    }
    const int grid = (n + kGsTok - 1) / kGsTok;
    if (dtype == VNSA_BF16)
        gate_mlp_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
            n, dm, hidden, n_out, (const __nv_bfloat16 *)x, (const __nv_bfloat16 *)g1, c1,
            (const __nv_bfloat16 *)g2, c2, out);
    else if (dtype == VNSA_FP32)
        gate_mlp_simt_kernel<float><<<grid, 256, 0, s>>>(n, dm, hidden, n_out, (const float *)x,
                                                         (const float *)g1, c1, (const float *)g2,
                                                         c2, out);
    else
        return cudaErrorInvalidValue;
    if (launches) ++*launches;
    return cudaGetLastError();
}

}  // namespace vnsa
