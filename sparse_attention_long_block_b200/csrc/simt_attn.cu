// simt_attn.cu -- CUDA-core (SIMT) attention kernels: compression attention +
// block importance, the vision branches (selection, sliding window) with the
// sigmoid gate combine, and dense text GQA.
//
// These carry the fp32 path, whose 1e-4 tolerance rules out tf32/bf16 tensor
// cores.  Method: "VideoNSA: Native Sparse Attention Scales Video
// Understanding" (paper notes), section "Method".
//
// Work split: one CTA per (query, GQA group), one warp per query head of the
// group, so the heads of a group read the same key/value rows through L1.
// A warp walks its key list 32 keys at a time: lane u scores key u against the
// query held in shared memory, the warp updates an online softmax, then each
// lane accumulates D/32 output dims over the 32 keys.
#include "kernels.h"

namespace vnsa {

template <typename T, int D>
struct RowState {
    static constexpr int PER = D / 32;
    float m, l;
    float o[PER];
    __device__ __forceinline__ void init() {
        m = -INFINITY;
        l = 0.f;
#pragma unroll
        for (int c = 0; c < PER; ++c) o[c] = 0.f;
    }
};

// Score of this lane's key (row `key` of a [rows][h_kv][D] tensor at head
// offset applied by `base`), in log2 units: qs is the query pre-multiplied by
// scale * log2(e).
template <typename T, int D>
__device__ __forceinline__ float score(const float *__restrict__ qs, const T *__restrict__ kr) {
    float acc = 0.f;
#pragma unroll
    for (int e = 0; e < D; e += 8) {
        float x[8];
        load8(kr + e, x);
#pragma unroll
        for (int z = 0; z < 8; ++z) acc = fmaf(qs[e + z], x[z], acc);
    }
    return acc;
}

// Online-softmax update with the 32 keys held one per lane (key_row < 0 =
// masked).  All lanes take the same branches.
template <typename T, int D>
__device__ __forceinline__ void online_chunk(RowState<T, D> &st, const float *qs,
                                             const T *__restrict__ kbase,
                                             const T *__restrict__ vbase, size_t stride,
                                             int key_row, int lane) {
    float s = -INFINITY;
    if (key_row >= 0) s = score<T, D>(qs, kbase + (size_t)key_row * stride);
    const float cm = warp_max(s);
    if (cm == -INFINITY) return;
    const float mn = fmaxf(st.m, cm);
    const float corr = exp2f(st.m - mn);
    const float pr = key_row >= 0 ? exp2f(s - mn) : 0.f;
    st.l = st.l * corr + warp_sum(pr);
#pragma unroll
    for (int c = 0; c < RowState<T, D>::PER; ++c) st.o[c] *= corr;
    st.m = mn;
#pragma unroll 4
    for (int u = 0; u < 32; ++u) {
        const float pu = __shfl_sync(0xffffffffu, pr, u);
        const int ru = __shfl_sync(0xffffffffu, key_row, u);
        if (ru < 0) continue;
        const T *vr = vbase + (size_t)ru * stride;
#pragma unroll
        for (int c = 0; c < RowState<T, D>::PER; ++c)
            st.o[c] = fmaf(pu, to_f(vr[lane + 32 * c]), st.o[c]);
    }
}

template <typename T, int D>
__device__ __forceinline__ void load_query(float *qs, const T *qrow, float mul, int lane) {
    for (int e = lane; e < D; e += 32) qs[e] = to_f(qrow[e]) * mul;
    __syncwarp();
}

// ---------------------------------------------------------------------------
// Compression attention over the block keys/values, with exact probabilities
// (two passes: log-sum-exp, then p = exp(s - lse)) so that the importance of
// block j for group g, sum over the group's heads of p_h[j], can be summed.
// Block j is visible to vision query i iff its last token j*S + B - 1 <= i
// (S = B unless the compression blocks overlap).
template <typename T, int D>
__global__ void cmp_simt_kernel(LayerParams p) {
    extern __shared__ float smem[];
    const int i = blockIdx.x, g = blockIdx.y;
    const Counts cn = *p.counts;
    if (i >= cn.n_vision) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = g * p.r + warp;
    const int t = p.vis[i];
    float *imp_s = smem;                              // [nb_max]
    float *qs = smem + p.nb_max + warp * D;           // [r][D]
    const int c = cmp_visible(i, p.block, p.stride, cn.nc);
    load_query<T, D>(qs, (const T *)p.q + ((size_t)t * p.h_q + h) * D, p.scale_log2, lane);
    __syncthreads();
    const size_t stride = (size_t)p.h_kv * D;
    const T *kb = (const T *)p.k_cmp + (size_t)g * D;
    const T *vb = (const T *)p.v_cmp + (size_t)g * D;
    // pass 1: log2-sum-exp
    float m = -INFINITY, l = 0.f;
    for (int base = 0; base < c; base += 32) {
        const int j = base + lane;
        const float s = j < c ? score<T, D>(qs, kb + (size_t)j * stride) : -INFINITY;
        const float cm = warp_max(s);
        const float mn = fmaxf(m, cm);
        l = l * exp2f(m - mn) + warp_sum(j < c ? exp2f(s - mn) : 0.f);
        m = mn;
    }
    const float lse2 = c > 0 ? m + log2f(l) : -INFINITY;
    // pass 2: exact probabilities, importance and output
    float o[D / 32];
#pragma unroll
    for (int x = 0; x < D / 32; ++x) o[x] = 0.f;
    float *ps = smem + p.nb_max + p.r * D;            // [r][32] probabilities
    for (int base = 0; base < c; base += 32) {
        const int j = base + lane;
        float pr = 0.f;
        if (j < c) pr = exp2f(score<T, D>(qs, kb + (size_t)j * stride) - lse2);
        ps[warp * 32 + lane] = pr;
        __syncthreads();
        if (warp == 0 && j < c) {  // fixed summation order over the group's heads
            float acc = 0.f;
            for (int w = 0; w < p.r; ++w) acc += ps[w * 32 + lane];
            imp_s[j] = acc;
        }
        __syncthreads();
        const int nk = min(32, c - base);
        for (int u = 0; u < nk; ++u) {
            const float pu = __shfl_sync(0xffffffffu, pr, u);
            const T *vr = vb + (size_t)(base + u) * stride;
#pragma unroll
            for (int x = 0; x < D / 32; ++x) o[x] = fmaf(pu, to_f(vr[lane + 32 * x]), o[x]);
        }
    }
    float *orow = p.o_cmp_ws + ((size_t)i * p.h_q + h) * D;
#pragma unroll
    for (int x = 0; x < D / 32; ++x) orow[lane + 32 * x] = o[x];
    if (lane == 0) p.lse[(size_t)i * p.h_q + h] = c > 0 ? lse2 * kLn2 : -INFINITY;
    __syncthreads();
    float *irow = p.imp + ((size_t)g * p.n_max + i) * p.imp_stride;
    for (int j = threadIdx.x; j < c; j += blockDim.x) irow[j] = imp_s[j];
}

// ---------------------------------------------------------------------------
// Vision rows: selection branch over the tokens of the selected blocks (causal
// inside the query's own block), sliding window over [i-w+1, i], then
// out = sig(g_cmp) o_cmp + sig(g_slc) o_slc + sig(g_swa) o_swa at position vis[i].
template <typename T, int D>
__global__ void vision_simt_kernel(LayerParams p) {
    extern __shared__ float smem[];
    const int i = blockIdx.x, g = blockIdx.y;
    const Counts cn = *p.counts;
    if (i >= cn.n_vision) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = g * p.r + warp;
    const int t = p.vis[i];
    float *qs = smem + warp * D;
    load_query<T, D>(qs, (const T *)p.q + ((size_t)t * p.h_q + h) * D, p.scale_log2, lane);
    const size_t stride = (size_t)p.h_kv * D;
    const T *kb = (const T *)p.k + (size_t)g * D;
    const T *vb = (const T *)p.v + (size_t)g * D;
    const int B = p.block, nv = cn.n_vision;
    RowState<T, D> st;
    // selection
    st.init();
    const int32_t *sel = p.idx_src + ((size_t)g * p.idx_rows + i) * p.top_k;
    for (int x = 0; x < p.top_k; ++x) {
        const int j = sel[x];
        if (j < 0) continue;
        if (j > i / B) { report(p.status, VNSA_ERR_BOUNDS); continue; }
        for (int half = 0; half < B; half += 32) {
            const int u = j * B + half + lane;
            const int kr = (half + lane < B && u <= i && u < nv) ? p.vis[u] : -1;
            online_chunk<T, D>(st, qs, kb, vb, stride, kr, lane);
        }
    }
    float o_s[D / 32];
    const float inv_s = st.l > 0.f ? 1.f / st.l : 0.f;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) o_s[c] = st.o[c] * inv_s;
    // sliding window
    st.init();
    const int lo = max(0, i - p.window + 1);
    for (int base = lo; base <= i; base += 32) {
        const int u = base + lane;
        online_chunk<T, D>(st, qs, kb, vb, stride, u <= i ? p.vis[u] : -1, lane);
    }
    const float inv_w = st.l > 0.f ? 1.f / st.l : 0.f;
    const float *gl = p.gate + ((size_t)t * p.h_q + h) * 3;
    const float gc = sigmoidf_(gl[0]), gs = sigmoidf_(gl[1]), gw = sigmoidf_(gl[2]);
    const float *oc = p.o_cmp_ws + ((size_t)i * p.h_q + h) * D;
    T *orow = (T *)p.out + ((size_t)t * p.h_q + h) * D;
    const size_t drow = ((size_t)t * p.h_q + h) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
        const int e = lane + 32 * c;
        const float ow = st.o[c] * inv_w;
        const float occ = oc[e];
        orow[e] = from_f<T>(gc * occ + gs * o_s[c] + gw * ow);
        if (p.dbg_o_cmp) p.dbg_o_cmp[drow + e] = occ;
        if (p.dbg_o_slc) p.dbg_o_slc[drow + e] = o_s[c];
        if (p.dbg_o_swa) p.dbg_o_swa[drow + e] = ow;
    }
}

// ---------------------------------------------------------------------------
// Text rows: dense causal GQA over every token u <= t.
template <typename T, int D>
__global__ void text_simt_kernel(LayerParams p) {
    extern __shared__ float smem[];
    const int x = blockIdx.x, g = blockIdx.y;
    const Counts cn = *p.counts;
    if (x >= cn.n_text) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = g * p.r + warp;
    const int t = p.txt[x];
    float *qs = smem + warp * D;
    load_query<T, D>(qs, (const T *)p.q + ((size_t)t * p.h_q + h) * D, p.scale_log2, lane);
    const size_t stride = (size_t)p.h_kv * D;
    const T *kb = (const T *)p.k + (size_t)g * D;
    const T *vb = (const T *)p.v + (size_t)g * D;
    RowState<T, D> st;
    st.init();
    for (int base = 0; base <= t; base += 32) {
        const int u = base + lane;
        online_chunk<T, D>(st, qs, kb, vb, stride, u <= t ? u : -1, lane);
    }
    const float inv = 1.f / st.l;
    T *orow = (T *)p.out + ((size_t)t * p.h_q + h) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) orow[lane + 32 * c] = from_f<T>(st.o[c] * inv);
}

// ---------------------------------------------------------------------------
#define VNSA_DISPATCH(KERNEL)                                                              \
    static cudaError_t launch_##KERNEL(int dtype, const LayerParams &p, dim3 grid,         \
                                       size_t smem, cudaStream_t s) {                      \
        const int threads = 32 * p.r;                                                      \
        void (*fn)(LayerParams) = nullptr;                                                 \
        if (dtype == VNSA_BF16 && p.d == 128) fn = KERNEL<__nv_bfloat16, 128>;             \
        else if (dtype == VNSA_BF16 && p.d == 64) fn = KERNEL<__nv_bfloat16, 64>;          \
        else if (dtype == VNSA_FP32 && p.d == 128) fn = KERNEL<float, 128>;                \
        else if (dtype == VNSA_FP32 && p.d == 64) fn = KERNEL<float, 64>;                  \
        else return cudaErrorInvalidValue;                                                 \
        if (smem > 48 * 1024) {                                                            \
            cudaError_t e = cudaFuncSetAttribute(                                          \
                fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);               \
            if (e != cudaSuccess) return e;                                                \
        }                                                                                  \
        fn<<<grid, threads, smem, s>>>(p);                                                 \
        return cudaGetLastError();                                                         \
    }
VNSA_DISPATCH(cmp_simt_kernel)
VNSA_DISPATCH(vision_simt_kernel)
VNSA_DISPATCH(text_simt_kernel)
#undef VNSA_DISPATCH

cudaError_t launch_cmp_simt(int dtype, const LayerParams &p, cudaStream_t s) {
    const size_t smem = sizeof(float) * ((size_t)p.nb_max + (size_t)p.r * p.d + 32 * p.r);
    return launch_cmp_simt_kernel(dtype, p, dim3(p.n_max, p.h_kv), smem, s);
}
cudaError_t launch_vision_simt(int dtype, const LayerParams &p, cudaStream_t s) {
    const size_t smem = sizeof(float) * (size_t)p.r * p.d;
    return launch_vision_simt_kernel(dtype, p, dim3(p.n_max, p.h_kv), smem, s);
}
cudaError_t launch_text_simt(int dtype, const LayerParams &p, cudaStream_t s) {
    const size_t smem = sizeof(float) * (size_t)p.r * p.d;
    return launch_text_simt_kernel(dtype, p, dim3(p.n_max, p.h_kv), smem, s);
}

}  // namespace vnsa
