// decode.cu -- one decode step of the hybrid layer: the attention output of a
// single new token appended to the token stream of the previous prefill or
// decode step on the same handle.
//
// Method: "VideoNSA: Native Sparse Attention Scales Video Understanding" (paper
// notes), section "Method", applied to one query: a vision token attends through
// compression (the complete blocks of the vision stream so far), selection (the
// top-k blocks of its group's importance, block 0 and its own block forced) and
// the sliding window, mixed by its sigmoid gates; a text token attends densely
// to every earlier token.  The result is, by definition, the last row of the
// prefill of the whole stream.
//
// State kept in the handle's workspace between steps: the vision / text
// position lists, the counts, and K_cmp / V_cmp of the complete blocks.  A step:
//   1. decode_prep:   appends the token to its list (one thread);
//   2. pool:          K_cmp / V_cmp of the block the token completes, if any;
//   3. decode_cmp:    compression scores and split partial softmax states;
//   4. decode_select: the group importance and top-k;
//   5. decode_attn:   selection + window (vision) or dense (text) partials;
//   6. decode_combine: the three branches' partials, the gates and the output row.
// Every kernel spreads its keys over kSplit CTAs per KV group (split-K); the
// query's group heads are processed together so every K/V row is read once.
#include <math.h>

#include "decode.h"
#include "topk.cuh"

namespace vnsa {

namespace {

constexpr int kWarps = 8;  // warps per CTA of the split kernels
constexpr int kBatch = 4;  // keys a warp loads before it computes (loads in flight)

// Row pieces: lane owns elements [lane * PER, lane * PER + PER) of a d-row.
template <typename T, int PER>
__device__ __forceinline__ void load_piece(const T *p, float (&x)[PER]) {
    if constexpr (sizeof(T) == 2 && PER == 4) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
        const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    } else if constexpr (sizeof(T) == 2 && PER == 2) {
        const float2 a = __bfloat1622float2(__ldg(reinterpret_cast<const __nv_bfloat162 *>(p)));
        x[0] = a.x; x[1] = a.y;
    } else if constexpr (sizeof(T) == 4 && PER == 4) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
        x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    } else {
#pragma unroll
        for (int e = 0; e < PER; ++e) x[e] = to_f(p[e]);
    }
}

// Split softmax states of one (branch, group): per head the largest split
// maximum M, the weights f_b = 2^(m_b - M) / L of every split, L = sum l_b f'_b,
// into shared memory fw [R_max][kSplit] (threads of the CTA cooperate).  The
// head's output element e is then sum_b o_b[e] fw[hh][b].
__device__ void split_weights(const float *part, int r, int d, float *fw, float *lse) {
    for (int hh = threadIdx.x >> 5; hh < r; hh += blockDim.x >> 5) {
        const int lane = threadIdx.x & 31;
        float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
#pragma unroll
        for (int z = 0; z < 2; ++z) {
            const int b = lane + 32 * z;
            if (b < kSplit) {
                const float *w = part + ((size_t)b * r + hh) * (d + 2);
                m[z] = w[d];
                l[z] = w[d + 1];
            }
        }
        const float M = warp_max(fmaxf(m[0], m[1]));
        float L = 0.f;
#pragma unroll
        for (int z = 0; z < 2; ++z)
            if (M != -INFINITY && l[z] > 0.f) L += l[z] * exp2f(m[z] - M);
        L = warp_sum(L);
#pragma unroll
        for (int z = 0; z < 2; ++z) {
            const int b = lane + 32 * z;
            if (b < kSplit)
                fw[hh * kSplit + b] = (L > 0.f && l[z] > 0.f) ? exp2f(m[z] - M) / L : 0.f;
        }
        if (lane == 0 && lse) lse[hh] = L > 0.f ? M + log2f(L) : -INFINITY;
    }
}

// Online softmax state of one head over this lane's part of d.
template <int PER>
struct Acc {
    float m, l, o[PER];
    __device__ void init() {
        m = -INFINITY;
        l = 0.f;
#pragma unroll
        for (int e = 0; e < PER; ++e) o[e] = 0.f;
    }
    // U keys at once (scores s, log2 units; -inf for a key to skip): one
    // rescale of the state per batch
    template <int U>
    __device__ void add_batch(const float (&s)[U], const float (&v)[U][PER]) {
        float mx = m;
#pragma unroll
        for (int u = 0; u < U; ++u) mx = fmaxf(mx, s[u]);
        if (mx == -INFINITY) return;  // no key so far and none in this batch
        const float corr = exp2f(m - mx);  // 0 when m = -inf
        l *= corr;
#pragma unroll
        for (int e = 0; e < PER; ++e) o[e] *= corr;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const float pu = exp2f(s[u] - mx);  // 0 for a skipped key
            l += pu;
#pragma unroll
            for (int e = 0; e < PER; ++e) o[e] = fmaf(pu, v[u][e], o[e]);
        }
        m = mx;
    }
};

// Scores (log2 units) of R heads against U keys: the U x R warp reductions are
// independent, so their shuffles overlap.
template <int PER, int R, int U>
__device__ __forceinline__ void batch_scores(const float (&q)[R][PER], const float (&kx)[U][PER],
                                             int r, float scale_log2, float (&s)[U][R]) {
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
        for (int hh = 0; hh < R; ++hh) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < PER; ++e) a = fmaf(q[hh][e], kx[u][e], a);
            s[u][hh] = a;
        }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int hh = 0; hh < R; ++hh)
                if (hh < r) s[u][hh] += __shfl_xor_sync(0xffffffffu, s[u][hh], o);
#pragma unroll
    for (int u = 0; u < U; ++u)
#pragma unroll
        for (int hh = 0; hh < R; ++hh) s[u][hh] *= scale_log2;
}

// Combine the kWarps per-warp states of R heads through shared memory and
// write one partial [R][D + 2] (O, m, l) per CTA.
template <int PER, int R>
__device__ void combine_warps(Acc<PER> (&acc)[R], int r, float *sm, float *dst) {
    constexpr int D = PER * 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // sm: [kWarps][R][D + 2]
#pragma unroll
    for (int hh = 0; hh < R; ++hh) {
        if (hh >= r) break;
        float *w = sm + ((size_t)warp * R + hh) * (D + 2);
#pragma unroll
        for (int e = 0; e < PER; ++e) w[lane * PER + e] = acc[hh].o[e];
        if (lane == 0) {
            w[D] = acc[hh].m;
            w[D + 1] = acc[hh].l;
        }
    }
    __syncthreads();
    for (int x = threadIdx.x; x < r * D; x += blockDim.x) {
        const int hh = x / D, e = x % D;
        float M = -INFINITY;
        for (int ww = 0; ww < kWarps; ++ww) M = fmaxf(M, sm[((size_t)ww * R + hh) * (D + 2) + D]);
        float L = 0.f, O = 0.f;
        if (M != -INFINITY) {
            for (int ww = 0; ww < kWarps; ++ww) {
                const float *w = sm + ((size_t)ww * R + hh) * (D + 2);
                const float f = exp2f(w[D] - M);
                L += w[D + 1] * f;
                O += w[e] * f;
            }
        }
        float *o = dst + (size_t)hh * (D + 2);
        o[e] = O;
        if (e == 0) {
            o[D] = M;
            o[D + 1] = L;
        }
    }
}

// Partial states of split b, branch br, group g: [R][D + 2]
__device__ __forceinline__ float *part_of(const DecodeParams &p, int br, int g, int b) {
    return p.part + (((size_t)br * p.h_kv + g) * kSplit + b) * (size_t)p.r * (p.d + 2);
}

// ---------------------------------------------------------------------------
__global__ void decode_prep_kernel(DecodeParams p) {
    wait_prior_grid();
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    Counts cn = *p.counts;
    const int t = p.n - 1;
    if (p.is_vision[t]) {
        const int i = cn.n_vision;
        p.vis[i] = t;
        if (i == 0) {
            cn.vis_base = t;
            cn.contiguous = 1;
        } else {
            cn.contiguous = cn.contiguous && (t == cn.vis_base + i);
        }
        cn.n_vision = i + 1;
        cn.nb = cn.n_vision / p.block;
        cn.nc = cn.nb;  // decode runs with the compression stride equal to the block
        cn.pad[0] = (cn.n_vision % p.block == 0) ? cn.nb - 1 : cn.nb;  // block to pool
        cn.pad[1] = 1;
        cn.pad[2] = i;
    } else {
        const int x = cn.n_text;
        p.txt[x] = t;
        if (x == 0) {
            cn.txt_base = t;
            cn.txt_contiguous = 1;
        } else {
            cn.txt_contiguous = cn.txt_contiguous && (t == cn.txt_base + x);
        }
        cn.n_text = x + 1;
        cn.pad[0] = cn.nb;
        cn.pad[1] = 0;
        cn.pad[2] = x;
    }
    *p.counts = cn;
}

// ---------------------------------------------------------------------------
// Compression: split b of the c visible blocks of group g.  Scores (log2 units)
// go to s_cmp for the importance; the split's softmax state to the partials.
template <typename T, int D, int R>
__global__ void __launch_bounds__(kWarps * 32) decode_cmp_kernel(DecodeParams p) {
    wait_prior_grid();
    constexpr int PER = D / 32;
    extern __shared__ float sm[];
    const Counts cn = *p.counts;
    if (!cn.pad[1]) return;  // a text token has no compression branch
    const int i = cn.pad[2];
    const int c = min((i + 1) / p.block, cn.nb);
    const int g = blockIdx.y, b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = p.r;
    const T *Q = (const T *)p.q;
    const T *KC = (const T *)p.k_cmp;
    const T *VC = (const T *)p.v_cmp;
    float q[R][PER];
    Acc<PER> acc[R];
#pragma unroll
    for (int hh = 0; hh < R; ++hh) {
        acc[hh].init();
        if (hh < r) load_piece<T, PER>(Q + (size_t)(g * r + hh) * D + lane * PER, q[hh]);
    }
    const int lo = (int)((long long)c * b / kSplit), hi = (int)((long long)c * (b + 1) / kSplit);
    for (int j0 = lo + warp * kBatch; j0 < hi; j0 += kWarps * kBatch) {
        float kx[kBatch][PER], vx[kBatch][PER];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int j = min(j0 + u, hi - 1);  // in range; keys past hi are skipped
            load_piece<T, PER>(KC + ((size_t)j * p.h_kv + g) * D + lane * PER, kx[u]);
            load_piece<T, PER>(VC + ((size_t)j * p.h_kv + g) * D + lane * PER, vx[u]);
        }
        float sc[kBatch][R];
        batch_scores<PER, R, kBatch>(q, kx, r, p.scale_log2, sc);
#pragma unroll
        for (int hh = 0; hh < R; ++hh) {
            if (hh >= r) break;
            float su[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const bool in = j0 + u < hi;
                su[u] = in ? sc[u][hh] : -INFINITY;
                if (in && lane == u) p.s_cmp[((size_t)g * r + hh) * p.nb_max + j0 + u] = sc[u][hh];
            }
            acc[hh].add_batch<kBatch>(su, vx);
        }
    }
    combine_warps<PER, R>(acc, r, sm, part_of(p, 0, g, b));
}

// ---------------------------------------------------------------------------
// Per group: the group importance of every visible block and the top-k
// selection.
template <int D>
__global__ void __launch_bounds__(1024) decode_select_kernel(DecodeParams p) {
    wait_prior_grid();
    extern __shared__ float sm[];  // lse [16], split weights [16][kSplit], importance
    __shared__ uint64_t buf[128];
    const Counts cn = *p.counts;
    if (!cn.pad[1]) return;
    const int i = cn.pad[2];
    const int c = min((i + 1) / p.block, cn.nb);
    const int g = blockIdx.x, r = p.r;
    float *lse = sm;
    float *fw = sm + 16;                    // [16][kSplit]
    float *imp = fw + 16 * kSplit + 4;      // 16-byte aligned: 16 + 16 * 37 + 4 floats
    // the log2-sum-exp of every head from the compression partials
    const float *part0 = part_of(p, 0, g, 0);
    split_weights(part0, r, D, fw, lse);
    __syncthreads();
    // importance: the exact compression probabilities summed over the heads
    // (the head loads of a block are issued together)
    for (int j = threadIdx.x; j < c; j += blockDim.x) {
        float s = 0.f;
#pragma unroll 8
        for (int hh = 0; hh < r; ++hh)
            s += exp2f(p.s_cmp[((size_t)g * r + hh) * p.nb_max + j] - lse[hh]);
        imp[j] = s;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        int32_t *out = p.sel + (size_t)g * p.top_k;
        topk_select_row<false>(imp, c, i / p.block, p.top_k, p.force_first, p.force_local, buf,
                               threadIdx.x, out, p.status);
        __syncwarp();
        if (p.sel_out)
            for (int x = threadIdx.x; x < p.top_k; x += 32) p.sel_out[(size_t)g * p.top_k + x] = out[x];
    }
}

// ---------------------------------------------------------------------------
// Selection + window (vision token) or dense (text token) partials.  A
// selection key is (x-th selected block, offset); a window key a vision rank;
// a dense key a position.  Each split takes an even share of each key range.
template <typename T, int D, int R>
__global__ void __launch_bounds__(kWarps * 32) decode_attn_kernel(DecodeParams p) {
    wait_prior_grid();
    constexpr int PER = D / 32;
    extern __shared__ float sm[];
    const Counts cn = *p.counts;
    const bool vision = cn.pad[1] != 0;
    const int g = blockIdx.y, b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = p.r;
    const T *Q = (const T *)p.q;
    const T *K = (const T *)p.k;
    const T *V = (const T *)p.v;
    float q[R][PER];
#pragma unroll
    for (int hh = 0; hh < R; ++hh)
        if (hh < r) load_piece<T, PER>(Q + (size_t)(g * r + hh) * D + lane * PER, q[hh]);
    auto vis_pos = [&](int u) { return cn.contiguous ? cn.vis_base + u : p.vis[u]; };
    // kBatch keys at positions t[u] (-1: skip) into the R accumulators; all
    // loads are issued before any score is computed
    auto attend = [&](Acc<PER>(&acc)[R], const int (&t)[kBatch]) {
        float kx[kBatch][PER], vx[kBatch][PER];
        int any = 0;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            any |= t[u] >= 0;
            const size_t row = ((size_t)max(t[u], 0) * p.h_kv + g) * D + lane * PER;
            load_piece<T, PER>(K + row, kx[u]);
            load_piece<T, PER>(V + row, vx[u]);
        }
        if (!any) return;
        float sc[kBatch][R];
        batch_scores<PER, R, kBatch>(q, kx, r, p.scale_log2, sc);
#pragma unroll
        for (int hh = 0; hh < R; ++hh) {
            if (hh >= r) break;
            float su[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) su[u] = t[u] >= 0 ? sc[u][hh] : -INFINITY;
            acc[hh].add_batch<kBatch>(su, vx);
        }
    };
    Acc<PER> acc[R];
    if (vision) {
        const int i = cn.pad[2];
        const int32_t *sel = p.sel + (size_t)g * p.top_k;
        // selection: flat keys over the selected blocks
        {
#pragma unroll
            for (int hh = 0; hh < R; ++hh) acc[hh].init();
            const int nk = p.top_k * p.block;
            const int lo = (int)((long long)nk * b / kSplit), hi = (int)((long long)nk * (b + 1) / kSplit);
            for (int x0 = lo + warp * kBatch; x0 < hi; x0 += kWarps * kBatch) {
                int t[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int x = x0 + u;
                    t[u] = -1;
                    if (x < hi) {
                        const int blk = sel[x / p.block];
                        const int rank = blk * p.block + x % p.block;
                        if (blk >= 0 && rank <= i) t[u] = vis_pos(rank);
                    }
                }
                attend(acc, t);
            }
            __syncthreads();
            combine_warps<PER, R>(acc, r, sm, part_of(p, 1, g, b));
            __syncthreads();
        }
        // window: vision ranks [i - w + 1, i]
        {
#pragma unroll
            for (int hh = 0; hh < R; ++hh) acc[hh].init();
            const int u0 = max(0, i - p.window + 1), nk = i - u0 + 1;
            const int lo = (int)((long long)nk * b / kSplit), hi = (int)((long long)nk * (b + 1) / kSplit);
            for (int x0 = lo + warp * kBatch; x0 < hi; x0 += kWarps * kBatch) {
                int t[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) t[u] = x0 + u < hi ? vis_pos(u0 + x0 + u) : -1;
                attend(acc, t);
            }
            combine_warps<PER, R>(acc, r, sm, part_of(p, 2, g, b));
        }
    } else {
        // dense: every position up to the token's own
#pragma unroll
        for (int hh = 0; hh < R; ++hh) acc[hh].init();
        const int nk = p.n;
        const int lo = (int)((long long)nk * b / kSplit), hi = (int)((long long)nk * (b + 1) / kSplit);
        for (int x0 = lo + warp * kBatch; x0 < hi; x0 += kWarps * kBatch) {
            int t[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) t[u] = x0 + u < hi ? x0 + u : -1;
            attend(acc, t);
        }
        combine_warps<PER, R>(acc, r, sm, part_of(p, 2, g, b));
    }
}

// ---------------------------------------------------------------------------
// One CTA per query head: the branch partials (compression, selection,
// window or text), the gates, the output row.
template <typename T, int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(DecodeParams p) {
    wait_prior_grid();
    __shared__ float fw[3][kSplit];
    const Counts cn = *p.counts;
    const bool vision = cn.pad[1] != 0;
    const int h = blockIdx.x, g = h / p.r, hh = h % p.r, e = threadIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // split weights of this head for branch br (0 compression, 1 selection,
    // 2 window / text), one warp per branch (D = 64: two warps take three)
    for (int br = warp; br < 3; br += D / 32) {
        if (!vision && br != 2) continue;
        const float *part = part_of(p, br, g, 0);
        float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
#pragma unroll
        for (int z = 0; z < 2; ++z) {
            const int b = lane + 32 * z;
            if (b < kSplit) {
                const float *w = part + ((size_t)b * p.r + hh) * (D + 2);
                m[z] = w[D];
                l[z] = w[D + 1];
            }
        }
        const float M = warp_max(fmaxf(m[0], m[1]));
        float L = 0.f;
#pragma unroll
        for (int z = 0; z < 2; ++z)
            if (M != -INFINITY && l[z] > 0.f) L += l[z] * exp2f(m[z] - M);
        L = warp_sum(L);
#pragma unroll
        for (int z = 0; z < 2; ++z) {
            const int b = lane + 32 * z;
            if (b < kSplit) fw[br][b] = (L > 0.f && l[z] > 0.f) ? exp2f(m[z] - M) / L : 0.f;
        }
    }
    __syncthreads();
    // every split's element is loaded before the sum (kSplit loads in flight)
    auto branch = [&](int br) {
        const float *part = part_of(p, br, g, 0);
        float x[kSplit];
#pragma unroll
        for (int b = 0; b < kSplit; ++b) x[b] = part[((size_t)b * p.r + hh) * (D + 2) + e];
        float O = 0.f;
#pragma unroll
        for (int b = 0; b < kSplit; ++b) O = fmaf(x[b], fw[br][b], O);
        return O;
    };
    float o;
    if (vision) {
        const float *gl = p.gate + (size_t)h * 3;
        o = sigmoidf_(gl[0]) * branch(0) + sigmoidf_(gl[1]) * branch(1) +
            sigmoidf_(gl[2]) * branch(2);
    } else {
        o = branch(2);
        if (p.sel_out && hh == 0 && e < p.top_k) p.sel_out[(size_t)g * p.top_k + e] = -1;
    }
    ((T *)p.out)[(size_t)h * D + e] = from_f<T>(o);
}

// A decode step is a chain of small dependent kernels; each is launched with
// programmatic stream serialisation, so it is scheduled while the previous one
// drains and waits for it in wait_prior_grid().
template <typename Kern>
cudaError_t launch_pdl(Kern kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       const DecodeParams &p) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

template <typename T, int D, int R>
cudaError_t launch_typed(const DecodeParams &p, cudaStream_t s, int *launches) {
    const size_t part_smem = (size_t)kWarps * R * (D + 2) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(decode_cmp_kernel<T, D, R>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)part_smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(decode_attn_kernel<T, D, R>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)part_smem);
    const size_t sel_smem = (16 + 16 * kSplit + 4 + (size_t)p.nb_max + 4) * sizeof(float);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(decode_select_kernel<D>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_smem);
    if (e != cudaSuccess) return e;
    const dim3 split(kSplit, p.h_kv);
    if (e == cudaSuccess)
        e = launch_pdl(decode_cmp_kernel<T, D, R>, split, dim3(kWarps * 32), part_smem, s, p);
    if (e == cudaSuccess)
        e = launch_pdl(decode_select_kernel<D>, dim3(p.h_kv), dim3(1024), sel_smem, s, p);
    if (e == cudaSuccess)
        e = launch_pdl(decode_attn_kernel<T, D, R>, split, dim3(kWarps * 32), part_smem, s, p);
    if (e == cudaSuccess)
        e = launch_pdl(decode_combine_kernel<T, D>, dim3(p.h_q), dim3(D), 0, s, p);
    *launches += 4;
    return e;
}

template <typename T, int D>
cudaError_t launch_r(const DecodeParams &p, cudaStream_t s, int *launches) {
    // the group's heads are held in registers: R is a compile-time bound on r
    if (p.r <= 1) return launch_typed<T, D, 1>(p, s, launches);
    if (p.r <= 4) return launch_typed<T, D, 4>(p, s, launches);
    if (p.r <= 8) return launch_typed<T, D, 8>(p, s, launches);
    return launch_typed<T, D, 16>(p, s, launches);
}

}  // namespace

size_t decode_workspace_bytes(int h_kv, int r, int d, int nb_max) {
    const size_t s_cmp = (size_t)h_kv * r * (nb_max > 0 ? nb_max : 1) * 4;
    const size_t part = (size_t)3 * h_kv * kSplit * r * (d + 2) * 4;
    return s_cmp + part + 256;
}

cudaError_t launch_decode(int dtype, const DecodeParams &p, cudaStream_t s, int *launches) {
    decode_prep_kernel<<<1, 32, 0, s>>>(p);
    ++*launches;
    cudaError_t e = launch_pool_proj(dtype, p.d, p.k, p.v, p.vis, p.counts, p.w_k, p.w_v,
                                     p.k_cmp, p.v_cmp, p.h_kv, p.block, p.block, p.nb_max, s,
                                     1, &p.mlp);
    ++*launches;
    if (e != cudaSuccess) return e;
    if (dtype == VNSA_BF16 && p.d == 128) return launch_r<__nv_bfloat16, 128>(p, s, launches);
    if (dtype == VNSA_BF16 && p.d == 64) return launch_r<__nv_bfloat16, 64>(p, s, launches);
    if (dtype == VNSA_FP32 && p.d == 128) return launch_r<float, 128>(p, s, launches);
    if (dtype == VNSA_FP32 && p.d == 64) return launch_r<float, 64>(p, s, launches);
    return cudaErrorInvalidValue;
}

}  // namespace vnsa
