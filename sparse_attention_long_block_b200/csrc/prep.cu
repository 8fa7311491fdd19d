// prep.cu -- vision/text partition, block mean-pool + projection, top-k block
// selection.
//
// Method: "VideoNSA: Native Sparse Attention Scales Video Understanding" (paper
// notes), section "Method": tokens are split into vision and text sets by their
// position IDs; the compression branch averages each 64-token vision block into
// one block key and value through a learned projection (a d x d linear map
// here); the selection branch keeps the top-k blocks ranked by importance.
#include "kernels.h"
#include "topk.cuh"

namespace vnsa {

// ---------------------------------------------------------------------------
// Partition: one CTA of 1024 threads walks the flags in stripes of 4096
// positions, four consecutive flags per thread; a stripe is compacted with a
// warp scan of the threads' vision counts and a scan of the 32 warp totals.
// vis[i] = position of the i-th vision token, txt[x] = position of the x-th
// text token.
__global__ void __launch_bounds__(1024) partition_kernel(const uint8_t *__restrict__ isv,
                                                         int n, int block, int stride,
                                                         int32_t *__restrict__ vis,
                                                         int32_t *__restrict__ txt,
                                                         Counts *counts) {
    constexpr int kPer = 4;
    constexpr int kStripe = 1024 * kPer;
    __shared__ int s_warp[32];  // exclusive prefix of the warps' vision counts
    __shared__ int s_stripe;    // vision tokens of the current stripe
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int nv = 0, nt = 0;  // totals before the current stripe (same in every thread)
    for (int base = 0; base < n; base += kStripe) {
        const int t0 = base + tid * kPer;
        bool f[kPer];
        int c = 0;
#pragma unroll
        for (int e = 0; e < kPer; ++e) {
            f[e] = t0 + e < n && isv[t0 + e] != 0;
            c += f[e];
        }
        // inclusive scan of c over the warp
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) s_warp[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int x = s_warp[lane];
            int wi = x;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o) wi += y;
            }
            s_warp[lane] = wi - x;
            if (lane == 31) s_stripe = wi;
        }
        __syncthreads();
        int vb = s_warp[warp] + incl - c;  // vision tokens before t0 in the stripe
#pragma unroll
        for (int e = 0; e < kPer; ++e) {
            const int t = t0 + e;
            if (t >= n) break;
            if (f[e]) vis[nv + vb++] = t;
            else txt[nt + (t - base) - vb] = t;
        }
        const int sv = s_stripe;
        nv += sv;
        nt += min(kStripe, n - base) - sv;
        __syncthreads();  // s_warp / s_stripe are rewritten by the next stripe
    }
    if (tid == 0) {
        Counts cn;
        cn.n_vision = nv;
        cn.n_text = nt;
        cn.nb = nv / block;
        cn.nc = nv >= block ? (nv - block) / stride + 1 : 0;
        cn.vis_base = nv > 0 ? vis[0] : 0;
        cn.contiguous = (nv == 0) || (vis[nv - 1] - vis[0] == nv - 1);
        cn.pad[0] = cn.pad[1] = cn.pad[2] = 0;
        cn.txt_base = nt > 0 ? txt[0] : 0;
        cn.txt_contiguous = (nt == 0) || (txt[nt - 1] - txt[0] == nt - 1);
        *counts = cn;
    }
}

cudaError_t launch_partition(const uint8_t *is_vision, int n, int block, int stride,
                             int32_t *vis, int32_t *txt, Counts *counts, cudaStream_t s) {
    partition_kernel<<<1, 1024, 0, s>>>(is_vision, n, block, stride, vis, txt, counts);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Pool + projection.  CTA (tile of JB compression blocks, KV head g, K or V):
// mean of each block's `block` vision rows in fp32 (block j starts at vision
// rank j * stride: the blocks overlap when stride < block), then mean . W
// (d x d) and one rounding to the storage type.  Rows are read with vector
// loads, one row per warp step.
template <typename T, int PER>
__device__ __forceinline__ void load_row_part(const T *p, float (&x)[PER]) {
    if constexpr (sizeof(T) == 2 && PER == 4) {
        uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
        float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    } else if constexpr (sizeof(T) == 2 && PER == 2) {
        float2 a = __bfloat1622float2(__ldg(reinterpret_cast<const __nv_bfloat162 *>(p)));
        x[0] = a.x; x[1] = a.y;
    } else if constexpr (sizeof(T) == 4 && PER == 4) {
        float4 a = __ldg(reinterpret_cast<const float4 *>(p));
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    } else {
        float2 a = __ldg(reinterpret_cast<const float2 *>(p));
        x[0] = a.x; x[1] = a.y;
    }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) pool_proj_kernel(
    const T *__restrict__ k, const T *__restrict__ v, const int32_t *__restrict__ vis,
    const Counts *__restrict__ counts, const T *__restrict__ w_k, const T *__restrict__ w_v,
    T *__restrict__ k_cmp, T *__restrict__ v_cmp, int h_kv, int block, int stride,
    int from_pad) {
    constexpr int JB = 16;             // blocks per CTA
    constexpr int PER = D / 32;        // elements per lane in a row
    constexpr int NPART = 256 / D;     // threads per output column
    constexpr int JBP = JB / NPART;    // blocks per thread in the projection
    __shared__ float mean[JB][D];
    wait_prior_grid();
    const int nb = counts->nc;
    // from_pad: only the blocks from counts->pad[0] on (the block a decode
    // step completed, or none)
    const int j0 = (from_pad ? counts->pad[0] : 0) + blockIdx.x * JB;
    if (j0 >= nb) return;
    const int g = blockIdx.y;
    const bool is_v = blockIdx.z != 0;
    const T *src = is_v ? v : k;
    const T *W = is_v ? w_v : w_k;
    T *dst = is_v ? v_cmp : k_cmp;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float inv = 1.0f / (float)block;
    for (int jb = warp; jb < JB; jb += 8) {
        const int j = j0 + jb;
        float acc[PER];
#pragma unroll
        for (int c = 0; c < PER; ++c) acc[c] = 0.f;
        if (j < nb) {
            const int32_t *rows = vis + (size_t)j * stride;
#pragma unroll 8
            for (int u = 0; u < block; ++u) {
                const T *p = src + ((size_t)rows[u] * h_kv + g) * D + lane * PER;
                float x[PER];
                load_row_part<T, PER>(p, x);
#pragma unroll
                for (int c = 0; c < PER; ++c) acc[c] += x[c];
            }
        }
#pragma unroll
        for (int c = 0; c < PER; ++c) mean[jb][lane * PER + c] = acc[c] * inv;
    }
    __syncthreads();
    const int col = threadIdx.x % D, part = threadIdx.x / D;
    float o[JBP];
#pragma unroll
    for (int x = 0; x < JBP; ++x) o[x] = 0.f;
    for (int e = 0; e < D; ++e) {
        const float w = to_f(W[(size_t)e * D + col]);
#pragma unroll
        for (int x = 0; x < JBP; ++x) o[x] = fmaf(mean[part * JBP + x][e], w, o[x]);
    }
#pragma unroll
    for (int x = 0; x < JBP; ++x) {
        const int j = j0 + part * JBP + x;
        if (j < nb) dst[((size_t)j * h_kv + g) * D + col] = from_f<T>(o[x]);
    }
}

// The compression branch's "learnable MLP" ("VideoNSA: Native Sparse Attention
// Scales Video Understanding", section "Method"), read as a two-layer
// perceptron with SiLU on the block mean: the same CTA tiling and mean as
// pool_proj_kernel, then hidden = SiLU(mean . w1 + b1) in fp32 shared memory and
// K_cmp = hidden . w2 + b2, rounded once to the storage type.
__device__ __forceinline__ float silu_f(float z) { return z / (1.f + expf(-z)); }

template <typename T, int D>
__global__ void __launch_bounds__(256) pool_mlp_kernel(
    const T *__restrict__ k, const T *__restrict__ v, const int32_t *__restrict__ vis,
    const Counts *__restrict__ counts, CmpMlp mlp, T *__restrict__ k_cmp,
    T *__restrict__ v_cmp, int h_kv, int block, int stride, int from_pad) {
    constexpr int JB = 16;
    constexpr int PER = D / 32;
    constexpr int NPART = 256 / D;
    constexpr int JBP = JB / NPART;
    __shared__ float mean[JB][D];
    __shared__ float hid[JB][kCmpMlpMaxHidden];
    wait_prior_grid();
    const int nb = counts->nc;
    const int j0 = (from_pad ? counts->pad[0] : 0) + blockIdx.x * JB;
    if (j0 >= nb) return;
    const int g = blockIdx.y;
    const int z = blockIdx.z;
    const T *src = z ? v : k;
    const T *W1 = (const T *)mlp.w1[z];
    const T *W2 = (const T *)mlp.w2[z];
    const float *B1 = mlp.b1[z];
    const float *B2 = mlp.b2[z];
    const int H = mlp.hidden;
    T *dst = z ? v_cmp : k_cmp;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float inv = 1.0f / (float)block;
    for (int jb = warp; jb < JB; jb += 8) {
        const int j = j0 + jb;
        float acc[PER];
#pragma unroll
        for (int c = 0; c < PER; ++c) acc[c] = 0.f;
        if (j < nb) {
            const int32_t *rows = vis + (size_t)j * stride;
#pragma unroll 8
            for (int u = 0; u < block; ++u) {
                const T *p = src + ((size_t)rows[u] * h_kv + g) * D + lane * PER;
                float x[PER];
                load_row_part<T, PER>(p, x);
#pragma unroll
                for (int c = 0; c < PER; ++c) acc[c] += x[c];
            }
        }
#pragma unroll
        for (int c = 0; c < PER; ++c) mean[jb][lane * PER + c] = acc[c] * inv;
    }
    __syncthreads();
    for (int x = threadIdx.x; x < H; x += 256) {
        float a[JB];
        const float b = B1[x];
#pragma unroll
        for (int jb = 0; jb < JB; ++jb) a[jb] = b;
        for (int e = 0; e < D; ++e) {
            const float w = to_f(W1[(size_t)e * H + x]);
#pragma unroll
            for (int jb = 0; jb < JB; ++jb) a[jb] = fmaf(mean[jb][e], w, a[jb]);
        }
#pragma unroll
        for (int jb = 0; jb < JB; ++jb) hid[jb][x] = silu_f(a[jb]);
    }
    __syncthreads();
    const int col = threadIdx.x % D, part = threadIdx.x / D;
    float o[JBP];
    const float b2 = B2[col];
#pragma unroll
    for (int x = 0; x < JBP; ++x) o[x] = b2;
    for (int e = 0; e < H; ++e) {
        const float w = to_f(W2[(size_t)e * D + col]);
#pragma unroll
        for (int x = 0; x < JBP; ++x) o[x] = fmaf(hid[part * JBP + x][e], w, o[x]);
    }
#pragma unroll
    for (int x = 0; x < JBP; ++x) {
        const int j = j0 + part * JBP + x;
        if (j < nb) dst[((size_t)j * h_kv + g) * D + col] = from_f<T>(o[x]);
    }
}

cudaError_t launch_pool_proj(int dtype, int d, const void *k, const void *v,
                             const int32_t *vis, const Counts *counts, const void *w_k,
                             const void *w_v, void *k_cmp, void *v_cmp, int h_kv, int block,
                             int stride, int nb_max, cudaStream_t s, int from_pad,
                             const CmpMlp *mlp) {
    if (nb_max <= 0) return cudaSuccess;
    dim3 grid(from_pad ? 1 : (nb_max + 15) / 16, h_kv, 2);
    if (mlp && mlp->hidden > 0) {
        if (mlp->hidden > kCmpMlpMaxHidden) return cudaErrorInvalidValue;
#define VNSA_POOL_MLP(T, D)                                                              \
    pool_mlp_kernel<T, D><<<grid, 256, 0, s>>>((const T *)k, (const T *)v, vis, counts,  \
                                               *mlp, (T *)k_cmp, (T *)v_cmp, h_kv, block, \
                                               stride, from_pad)
        if (dtype == VNSA_BF16 && d == 128) VNSA_POOL_MLP(__nv_bfloat16, 128);
        else if (dtype == VNSA_BF16 && d == 64) VNSA_POOL_MLP(__nv_bfloat16, 64);
        else if (dtype == VNSA_FP32 && d == 128) VNSA_POOL_MLP(float, 128);
        else if (dtype == VNSA_FP32 && d == 64) VNSA_POOL_MLP(float, 64);
        else return cudaErrorInvalidValue;
#undef VNSA_POOL_MLP
        return cudaGetLastError();
    }
#define VNSA_POOL(T, D)                                                                  \
    pool_proj_kernel<T, D><<<grid, 256, 0, s>>>(                                         \
        (const T *)k, (const T *)v, vis, counts, (const T *)w_k, (const T *)w_v,         \
        (T *)k_cmp, (T *)v_cmp, h_kv, block, stride, from_pad)
    if (dtype == VNSA_BF16 && d == 128) VNSA_POOL(__nv_bfloat16, 128);
    else if (dtype == VNSA_BF16 && d == 64) VNSA_POOL(__nv_bfloat16, 64);
    else if (dtype == VNSA_FP32 && d == 128) VNSA_POOL(float, 128);
    else if (dtype == VNSA_FP32 && d == 64) VNSA_POOL(float, 64);
    else return cudaErrorInvalidValue;
#undef VNSA_POOL
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Top-k block selection (topk.cuh): one warp per (group g, vision query i).
__global__ void __launch_bounds__(256) topk_kernel(LayerParams p) {
    __shared__ uint64_t sh_buf[8][kTopkBuf];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x * 8 + warp;
    const int g = blockIdx.y;
    const Counts cn = *p.counts;
    if (i >= cn.n_vision) return;
    int c = (i + 1) / p.block;
    if (c > cn.nb) c = cn.nb;
    topk_select_row<true>(p.imp_sel + ((size_t)g * p.n_max + i) * p.imp_sel_stride, c,
                          i / p.block,
                          p.top_k, p.force_first, p.force_local, sh_buf[warp], lane,
                          p.idx + ((size_t)g * p.n_max + i) * p.top_k, p.status);
}

cudaError_t launch_topk(const LayerParams &p, cudaStream_t s) {
    dim3 grid((p.n_max + 7) / 8, p.h_kv);
    topk_kernel<<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

// Overlapping compression blocks (stride S < block B; "VideoNSA: Native Sparse
// Attention Scales Video Understanding", paper notes, section "Method", and the
// native sparse attention design it builds on): the importance of selection
// block j is the group's compression probability mass spread over the
// selection blocks by the tokens each compression block puts in them,
//   imp_sel[j] = sum_c |[c S, c S + B) ^ [j B, j B + B)| / B * imp[c],
// over the compression blocks c visible to the query (last token <= i); only
// the selection blocks j < (i + 1) / B (the top-k candidates) are written.
// One warp per (group, vision query), lanes over j.
__global__ void __launch_bounds__(256) imp_remap_kernel(LayerParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int i = blockIdx.x * 8 + warp;
    const int g = blockIdx.y;
    const Counts cn = *p.counts;
    if (i >= cn.n_vision) return;
    const int B = p.block, S = p.stride;
    const int ncv = cmp_visible(i, B, S, cn.nc);
    const int nsel = min((i + 1) / B, cn.nb);
    const float *src = p.imp + ((size_t)g * p.n_max + i) * p.imp_stride;
    float *dst = p.imp_sel + ((size_t)g * p.n_max + i) * p.imp_sel_stride;
    const float inv_b = 1.f / (float)B;
    for (int j = lane; j < nsel; j += 32) {
        const int a = j * B, b = a + B;             // tokens of selection block j
        int c0 = a - B + 1 > 0 ? (a - B + 1 + S - 1) / S : 0;  // first c with c S + B > a
        int c1 = (b - 1) / S;                       // last c with c S < b
        if (c1 > ncv - 1) c1 = ncv - 1;
        float acc = 0.f;
        for (int c = c0; c <= c1; ++c) {
            const int lo = max(c * S, a), hi = min(c * S + B, b);
            acc = fmaf((float)(hi - lo) * inv_b, src[c], acc);
        }
        dst[j] = acc;
    }
}

cudaError_t launch_imp_remap(const LayerParams &p, cudaStream_t s) {
    dim3 grid((p.n_max + 7) / 8, p.h_kv);
    imp_remap_kernel<<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace vnsa

namespace vnsa {

// ---------------------------------------------------------------------------
// Debug exports: copies of workspace tensors into caller buffers, sized by the
// device-side vision count (so the host never has to synchronise for it).
__global__ void export_kernel(LayerParams p, int esize, float *lse_out, int32_t *idx_out,
                              float *imp_out, size_t imp_stride_out, uint32_t *kc_out,
                              uint32_t *vc_out) {
    const Counts cn = *p.counts;
    const size_t nv = (size_t)cn.n_vision, nb = (size_t)cn.nb;
    const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t step = (size_t)gridDim.x * blockDim.x;
    if (lse_out)
        for (size_t x = tid; x < nv * p.h_q; x += step) lse_out[x] = p.lse[x];
    if (idx_out) {
        const size_t k = (size_t)p.top_k;
        for (size_t x = tid; x < (size_t)p.h_kv * nv * k; x += step) {
            const size_t g = x / (nv * k), rem = x % (nv * k);
            const size_t i = rem / k, c = rem % k;
            idx_out[(g * p.n + i) * k + c] = p.idx_src[(g * p.idx_rows + i) * k + c];
        }
    }
    if (imp_out && nb > 0) {
        for (size_t x = tid; x < (size_t)p.h_kv * nv * nb; x += step) {
            const size_t j = x % nb, gi = x / nb;
            const size_t g = gi / nv, i = gi % nv;
            if ((int)j < (int)((i + 1) / p.block))
                imp_out[(g * p.n + i) * imp_stride_out + j] =
                    p.imp_sel[(g * p.n_max + i) * p.imp_sel_stride + j];
        }
    }
    const size_t words = (size_t)cn.nc * p.h_kv * p.d * esize / 4;
    if (kc_out)
        for (size_t x = tid; x < words; x += step) kc_out[x] = ((const uint32_t *)p.k_cmp)[x];
    if (vc_out)
        for (size_t x = tid; x < words; x += step) vc_out[x] = ((const uint32_t *)p.v_cmp)[x];
}

cudaError_t launch_export(const LayerParams &p, int esize, float *lse_out, int32_t *idx_out,
                          float *imp_out, size_t imp_stride_out, void *kc_out, void *vc_out,
                          cudaStream_t s) {
    export_kernel<<<592, 256, 0, s>>>(p, esize, lse_out, idx_out, imp_out, imp_stride_out,
                                      (uint32_t *)kc_out, (uint32_t *)vc_out);
    return cudaGetLastError();
}

}  // namespace vnsa
