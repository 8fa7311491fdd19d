// sgl_attn.cu -- tile-major pass of the selection branch (block 64).
//
// Method: "VideoNSA: Native Sparse Attention Scales Video Understanding" (paper
// notes), section "Method": each vision query attends to the tokens of the
// blocks it selected.  The union pass of tc_attn.cu attends, for 128 MMA rows
// (consecutive queries x the heads of one GQA group), the 64-key tiles that
// three or more of those queries selected.  A tile that only one or two of
// them selected would cost a whole 128-row tile of tensor work for 7 or 14
// useful rows, so the union kernel hands such (query, tile) pairs to this
// pass instead.  Here the pairs are grouped by tile (bucket = group x tile):
// a chunk is up to 128 / r pairs of one tile, and a thread block takes a
// contiguous range of chunks, so a tile's K/V is loaded once and serves every
// chunk of it in the range.
//
// Per chunk: S = Q K^T (M 128, N 64, K 128, bf16), the softmax of each row over
// the tile's keys at or before its query, P (fp16) back into TMEM, O = P V
// against the scaled fp16 copy of V (the scale is multiplied back here).
// Each pair row's output is written normalised in fp16, in the units of the
// scaled V copy (a convex combination of values below 2^15, so it cannot
// overflow), with its log-sum-exp and the power of two that restores its
// units; the union pass merges them.
//
//   warp 0     lane 0: TMA loads of each new tile's K and V (one stage)
//   warp 1     lane 0: the MMAs
//   warps 2-5  one thread per MMA row: softmax and epilogue; each warp gathers
//              its 32 rows' Q by cp.async two chunks ahead into a double
//              buffer (half a warp per 256-byte row, so every 32-byte sector
//              is read whole) and stores its rows' outputs through shared
//              memory (eight 64-byte row pieces per instruction)
#include <math.h>

#include "sgl_attn.h"
#include "tc_ptx.cuh"

namespace vnsa {
namespace {

constexpr int kThreads = 192;
constexpr int kRows = 128;
constexpr int kKeys = 64;
constexpr int kD = 128;

constexpr uint32_t SM_Q = 0;         // 2 x [128 rows][128] bf16, 32 KB each
constexpr uint32_t Q_BYTES = 32768;
constexpr uint32_t SM_K = 65536;     // one K tile: 2 boxes of 64 keys x 64 d (16 KB)
constexpr uint32_t SM_V = 81920;     // one V tile (16 KB)
constexpr uint32_t SM_STG = 98304;   // per softmax warp: 32 rows x 64 B of output (+16 B pad)
constexpr uint32_t STG_ROW = 80, STG_WARP = 32 * STG_ROW;
constexpr uint32_t SM_BAR = SM_STG + 4 * STG_WARP;
constexpr uint32_t SMEM_BYTES = SM_BAR + 256 + 1024;  // + alignment slack
// two CTAs per SM: 2 x (SMEM_BYTES + 1 KB reserved) within the SM's 228 KB
static_assert(2 * (SMEM_BYTES + 1024) <= 228 * 1024, "two CTAs per SM");

enum { B_Q_FULL = 0, B_KV_FULL = 2, B_KV_EMPTY = 3, B_S_FULL = 4, B_P_FULL = 6, B_PV_DONE = 8,
       B_FINAL = 9, B_COUNT = 10 };

// TMEM: two S buffers (chunk j uses j & 1; its P overwrites the first 32
// columns) and O.
constexpr uint32_t TM_S = 0, TM_O = 128, TM_COLS = 256;

struct Sm {
    uint8_t *base;
    uint32_t u32;
    __device__ uint32_t bar(int i) const { return u32 + SM_BAR + 8u * (uint32_t)i; }
    __device__ uint32_t *tmem_slot() const { return (uint32_t *)(base + SM_BAR + 8 * B_COUNT); }
    __device__ volatile int *abort_flag() const {
        return (volatile int *)(base + SM_BAR + 8 * B_COUNT + 8);
    }
    __device__ uint32_t *failed_flag() const {
        return (uint32_t *)(base + SM_BAR + 8 * B_COUNT + 16);
    }
};

__device__ __forceinline__ uint64_t desc_kmajor(uint32_t addr) {
    return ptx::sdesc_sw128(addr, 16, 1024);
}
__device__ __forceinline__ uint64_t desc_vmajor(uint32_t addr) {
    return ptx::sdesc_sw128(addr, 8192, 1024);
}

// ---------------------------------------------------------------------------
__device__ void producer(const SglParams &P, const Sm &sm, int lo, int hi) {
    volatile int *abort = sm.abort_flag();
    const Counts cn = *P.counts;
    // vision rank u is row vbase + u of the chosen maps
    const CUtensorMap *mk = cn.contiguous ? &P.tm_k : &P.tm_kc;
    const CUtensorMap *mv = cn.contiguous ? &P.tm_v : &P.tm_vc;
    const int vbase = cn.contiguous ? cn.vis_base : 0;
    int kvi = 0;  // tile loads issued
    for (int x = lo; x < hi; ++x) {
        const int b = P.items[x].x;
        if (x > lo && b == P.items[x - 1].x) continue;  // same tile: already in place
        if (kvi > 0 &&
            !ptx::mbar_wait(sm.bar(B_KV_EMPTY), (kvi - 1) & 1, abort, P.status, P.wait_ns))
            break;
        const int g = b / P.nbt, tile = b % P.nbt;
        const int y = vbase + tile * kKeys, xc = g * kD;
        const uint32_t fb = sm.bar(B_KV_FULL);
        ptx::mbar_expect_tx(fb, 4u * 8192u);
        ptx::tma_load_2d(sm.u32 + SM_K, mk, fb, xc, y);
        ptx::tma_load_2d(sm.u32 + SM_K + 8192, mk, fb, xc + 64, y);
        ptx::tma_load_2d(sm.u32 + SM_V, mv, fb, xc, y);
        ptx::tma_load_2d(sm.u32 + SM_V + 8192, mv, fb, xc + 64, y);
        ++kvi;
    }
    // the last load must have landed before the CTA ends (also after an abort)
    if (kvi > 0) ptx::mbar_drain(sm.bar(B_KV_FULL), (kvi - 1) & 1);
}

// ---------------------------------------------------------------------------
__device__ void mma_issuer(const SglParams &P, const Sm &sm, uint32_t tmem, int lo, int hi) {
    volatile int *abort = sm.abort_flag();
    constexpr uint32_t idesc_s = ptx::idesc_f16kind(kRows, kKeys, 0, 0, 1u);
    constexpr uint32_t idesc_pv = ptx::idesc_f16kind(kRows, kD, 0, 1, 0u);
    // P V of local chunk jj, once its P is in TMEM; the last chunk of a tile
    // then frees the K/V stage for the next tile's load
    auto finish = [&](int jj, bool last_of_tile) -> bool {
        if (!ptx::mbar_wait(sm.bar(B_P_FULL + (jj & 1)), (jj >> 1) & 1, abort, P.status,
                            P.wait_ns))
            return false;
        ptx::tc_fence_after();
        const uint32_t pa = tmem + TM_S + (uint32_t)(jj & 1) * 64u;
#pragma unroll
        for (int k = 0; k < kKeys / 16; ++k)
            ptx::mma_ts(tmem + TM_O, pa + (uint32_t)k * 8u,
                        desc_vmajor(sm.u32 + SM_V + (uint32_t)k * 2048u), idesc_pv,
                        k > 0 ? 1u : 0u);
        ptx::mma_commit(sm.bar(B_PV_DONE));
        if (last_of_tile) ptx::mma_commit(sm.bar(B_KV_EMPTY));
        return true;
    };
    int kvi = 0;  // tile loads consumed
    bool ok = true;
    for (int x = lo; ok && x < hi; ++x) {
        const int j = x - lo;
        const bool first = x == lo || P.items[x].x != P.items[x - 1].x;
        if (first) {
            // the previous tile's last P V comes before this tile's load
            if (j > 0 && !finish(j - 1, true)) { ok = false; break; }
            if (!ptx::mbar_wait(sm.bar(B_KV_FULL), kvi & 1, abort, P.status, P.wait_ns)) {
                ok = false;
                break;
            }
            ++kvi;
        }
        if (!ptx::mbar_wait(sm.bar(B_Q_FULL + (j & 1)), (j >> 1) & 1, abort, P.status,
                            P.wait_ns)) {
            ok = false;
            break;
        }
        ptx::tc_fence_after();
        const uint32_t qa = sm.u32 + SM_Q + (uint32_t)(j & 1) * Q_BYTES;
        const uint32_t sd = tmem + TM_S + (uint32_t)(j & 1) * 64u;
#pragma unroll
        for (int k = 0; k < kD / 16; ++k) {
            const uint32_t off = (uint32_t)(k >> 2) * 16384u + (uint32_t)(k & 3) * 32u;
            const uint32_t koff = (uint32_t)(k >> 2) * 8192u + (uint32_t)(k & 3) * 32u;
            ptx::mma_ss(sd, desc_kmajor(qa + off), desc_kmajor(sm.u32 + SM_K + koff), idesc_s,
                        k > 0 ? 1u : 0u);
        }
        ptx::mma_commit(sm.bar(B_S_FULL + (j & 1)));
        // the previous chunk of the same tile: its P V follows this Q K^T
        if (!first && !finish(j - 1, false)) { ok = false; break; }
    }
    if (ok && hi > lo) finish(hi - lo - 1, true);
    // every MMA issued has completed before the CTA frees its TMEM
    ptx::mma_commit(sm.bar(B_FINAL));
    ptx::mbar_drain(sm.bar(B_FINAL), 0);
}

// ---------------------------------------------------------------------------
// Softmax / epilogue warps: thread rho owns MMA row rho = pair slot rho / r,
// head rho % r of the chunk.
__device__ void rows(const SglParams &P, const Sm &sm, uint32_t tmem, int lo, int hi) {
    volatile int *abort = sm.abort_flag();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wq = warp & 3;
    const int rho = wq * 32 + lane;
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const int r = P.r;
    const int slot = rho / r, hl = rho % r;
    const float sc = P.scale_log2;

    const int qt = kRows / r;  // pairs per chunk
    // This row's entry in chunk x (global index): (pair id, vision rank,
    // position, bucket), pair id -1 for no pair; one independent load, made
    // two chunks before its use (the entries rotate through e_a, e_b, e_c).
    auto entry = [&](int x) -> int4 {
        return (x < hi && slot < qt) ? P.sorted[(size_t)x * qt + slot] : make_int4(-1, 0, 0, 0);
    };
    // the row's Q row index (token x h_q + head) in q, -1 for no pair
    auto q_off = [&](const int4 &e) -> int {
        if (e.x < 0) return -1;
        const int h = (e.w / P.nbt) * r + hl;
        return e.z * P.h_q + h;
    };
    // The warp's 32 rows into Q buffer `buf`, 16-byte pieces in the 128-byte
    // swizzled K-major layout of the MMA's A operand; a row without a pair is
    // zero-filled.  Each instruction copies two whole rows (lanes 0-15 one,
    // 16-31 the next), so the sectors of a row are read in full and together.
    // One cp.async group per call.
    auto gather = [&](int off, int buf) {
        const uint32_t qb = sm.u32 + SM_Q + (uint32_t)buf * Q_BYTES;
        const int c16 = lane & 15;
        const uint32_t hf = (uint32_t)(c16 >> 3), c = (uint32_t)(c16 & 7);
#pragma unroll
        for (int z = 0; z < 16; ++z) {
            const int t = 2 * z + (lane >> 4);  // row wq * 32 + t is lane t's
            const int o = __shfl_sync(0xffffffffu, off, t);
            const uint32_t row = (uint32_t)(wq * 32 + t);
            const uint32_t dst = qb + hf * 16384u + row * 128u + ((c ^ (row & 7u)) << 4);
            const bool valid = o >= 0;
            ptx::cp_async16(dst, valid ? (const void *)(P.q + (size_t)o * kD + c16 * 8) : (const void *)P.q,
                            valid ? 16u : 0u);
        }
        ptx::cp_async_commit();
    };
    int4 e_a = entry(lo), e_b = entry(lo + 1), e_c = entry(lo + 2);
    gather(q_off(e_a), 0);
    gather(q_off(e_b), 1);
    ptx::cp_async_wait<1>();
    ptx::fence_proxy_async();
    if (hi > lo) ptx::mbar_arrive(sm.bar(B_Q_FULL));

    bool ok = true;
    for (int x = lo; ok && x < hi; ++x) {
        const int j = x - lo;
        const int4 e = e_a;  // this chunk's entry
        e_a = e_b;           // chunk x + 1
        e_b = e_c;           // chunk x + 2: gathered below
        e_c = entry(x + 3);
        const bool valid = e.x >= 0;
        const int sid = e.x, i = e.y, tile = e.w % P.nbt;
        const int hi_key = valid ? min(i - tile * kKeys, kKeys - 1) : -1;
        const bool none = __all_sync(0xffffffffu, hi_key < 0);
        const uint32_t s_col = tmem + lane_base + TM_S + (uint32_t)(j & 1) * 64u;
        {
            bool rr = ptx::mbar_wait(sm.bar(B_S_FULL + (j & 1)), (j >> 1) & 1, abort, P.status,
                                     P.wait_ns);
            ok = __all_sync(0xffffffffu, rr);
            if (!ok) break;
        }
        ptx::tc_fence_after();
        // Q K^T of this chunk is done, so its buffer takes chunk x + 2
        gather(q_off(e_b), j & 1);

        float m_run = -INFINITY, l_run = 0.f;
        uint32_t pk[32];
        if (none) {
#pragma unroll
            for (int k = 0; k < 32; ++k) pk[k] = 0u;
        } else {
            float sv[64];
            {
                float a[32], c[32];
                ptx::tmem_ld32(s_col, a);
                ptx::tmem_ld32(s_col + 32, c);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 32; ++k) { sv[k] = a[k]; sv[32 + k] = c[k]; }
            }
            const bool live = hi_key >= 0;
            // keys after the query masked on the raw scores (scale > 0 keeps
            // the order); a row without a pair keeps its finite scores (Q row
            // 0) and gets P = 0 through 2^(s * 0 - inf)
            if (live && hi_key < kKeys - 1) {
#pragma unroll
                for (int k = 0; k < 64; ++k) sv[k] = k <= hi_key ? sv[k] : -INFINITY;
            }
            float mx = -INFINITY;
#pragma unroll
            for (int k = 0; k < 64; k += 2) mx = ptx::fmax3(mx, sv[k], sv[k + 1]);
            mx *= sc;
            const float s_r = live ? sc : 0.f;
            const float b_r = live ? -mx : -INFINITY;
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int k = 0; k < 64; k += 2) {
                ptx::ffma2(sv[k], sv[k + 1], sv[k], sv[k + 1], s_r, s_r, b_r, b_r);
                sv[k] = ptx::ex2(sv[k]);
                sv[k + 1] = ptx::ex2(sv[k + 1]);
                ptx::fadd2(a0, a1, a0, a1, sv[k], sv[k + 1]);
            }
            if (live) {
                m_run = mx;
                l_run = a0 + a1;
            }
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                __half2 h2 = __floats2half2_rn(sv[2 * k], sv[2 * k + 1]);
                pk[k] = *reinterpret_cast<uint32_t *>(&h2);
            }
        }
        ptx::tmem_st32u(s_col, pk);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(sm.bar(B_P_FULL + (j & 1)));
        // the next chunk's rows (gathered one chunk ago) go to the MMA now, after
        // this chunk's softmax: the copies had that long to land, and the next
        // Q K^T still runs while this chunk's P V and epilogue do
        ptx::cp_async_wait<1>();
        ptx::fence_proxy_async();
        if (x + 1 < hi) ptx::mbar_arrive(sm.bar(B_Q_FULL + ((j + 1) & 1)));
        if (none) continue;  // no row of this warp writes anything
        {
            bool rr = ptx::mbar_wait(sm.bar(B_PV_DONE), j & 1, abort, P.status, P.wait_ns);
            ok = __all_sync(0xffffffffu, rr);
            if (!ok) break;
        }
        ptx::tc_fence_after();
        // epilogue: the normalised row in the scaled V's units (fp16), 32
        // columns at a time through the warp's staging rows, then stored by
        // eight lanes' 64-byte pieces per instruction (whole sectors)
        const float mul = l_run > 0.f ? 1.f / l_run : 0.f;
        const int orow = hi_key >= 0 ? sid * r + hl : -1;  // output row, -1: none
        uint8_t *stg = sm.base + SM_STG + (uint32_t)wq * STG_WARP;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
            float o[32];
            ptx::tmem_ld32(tmem + lane_base + TM_O + ch * 32, o);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; k += 8) {
                uint4 v;
                __half2 *h2 = reinterpret_cast<__half2 *>(&v);
#pragma unroll
                for (int z = 0; z < 4; ++z)
                    h2[z] = __floats2half2_rn(o[k + 2 * z] * mul, o[k + 2 * z + 1] * mul);
                *reinterpret_cast<uint4 *>(stg + lane * STG_ROW + k * 2) = v;
            }
            __syncwarp();
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                const int t = 8 * z + (lane >> 2), pc = lane & 3;
                const int dst = __shfl_sync(0xffffffffu, orow, t);
                const uint4 v = *reinterpret_cast<const uint4 *>(stg + t * STG_ROW + pc * 16);
                if (dst >= 0)
                    *reinterpret_cast<uint4 *>(P.o + (size_t)dst * kD + ch * 32 + pc * 8) = v;
            }
            __syncwarp();  // the staging rows are rewritten by the next columns
        }
        if (hi_key >= 0)
            P.lse[(size_t)sid * r + hl] = l_run > 0.f ? m_run + log2f(l_run) : -INFINITY;
    }
    // no copy may still be landing in shared memory when the CTA ends
    ptx::cp_async_wait<0>();
}

__global__ void __launch_bounds__(kThreads, 2) sgl_attn_kernel(const __grid_constant__ SglParams P) {
    extern __shared__ uint8_t smem_raw[];
    Sm sm;
    {
        const uint32_t raw = ptx::smem_u32(smem_raw);
        const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
        sm.base = smem_raw + pad;
        sm.u32 = raw + pad;
    }
    if (threadIdx.x == 0) *sm.failed_flag() = *(volatile uint32_t *)P.status;
    __syncthreads();
    if (*sm.failed_flag() != 0) return;
    const int items = *P.n_items;
    const int lo = (int)((long long)items * blockIdx.x / gridDim.x);
    const int hi = (int)((long long)items * (blockIdx.x + 1) / gridDim.x);
    if (hi <= lo) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(sm.bar(B_Q_FULL + b), 128);
            ptx::mbar_init(sm.bar(B_S_FULL + b), 1);
            ptx::mbar_init(sm.bar(B_P_FULL + b), 4);
        }
        ptx::mbar_init(sm.bar(B_KV_FULL), 1);
        ptx::mbar_init(sm.bar(B_KV_EMPTY), 1);
        ptx::mbar_init(sm.bar(B_PV_DONE), 1);
        ptx::mbar_init(sm.bar(B_FINAL), 1);
        *sm.abort_flag() = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(ptx::smem_u32(sm.tmem_slot()), TM_COLS);
        ptx::tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        ptx::prefetch_tmap(&P.tm_k);
        ptx::prefetch_tmap(&P.tm_v);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *sm.tmem_slot();
    if (warp == 0) {
        if (lane == 0) producer(P, sm, lo, hi);
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) mma_issuer(P, sm, tmem, lo, hi);
        __syncwarp();
    } else {
        rows(P, sm, tmem, lo, hi);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, TM_COLS);
}

}  // namespace

cudaError_t sgl_prepare() {
    return cudaFuncSetAttribute(sgl_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)SMEM_BYTES);
}

cudaError_t launch_sgl_attn(const SglParams &p, int num_sms, cudaStream_t s) {
    sgl_attn_kernel<<<2 * num_sms, kThreads, SMEM_BYTES, s>>>(p);
    return cudaGetLastError();
}

}  // namespace vnsa
