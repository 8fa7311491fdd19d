// tc_attn.cu -- tensor-core path of the bf16 layer prefill (head dim 128):
// compression attention + importance, selection + sliding window + gate, and
// dense text GQA, on tcgen05 MMAs with TMEM accumulators fed by TMA.
//
// Method: "VideoNSA: Native Sparse Attention Scales Video Understanding" (paper
// notes), section "Method": vision tokens attend through compression,
// selection and a sliding window mixed by per-head sigmoid gates; text tokens
// attend densely (GQA).
//
// One persistent kernel template serves three modes.  A CTA (8 warps, one per
// SM) walks work items; an item is an M tile of 128 MMA rows, row = (query,
// head of one GQA group): 128 / (h_q/h_kv) consecutive queries times the
// group's heads, so the heads of a group share every K/V tile (18 queries x 7
// heads = 126 rows for 28/4 heads).  Per item the CTA streams 64-key tiles:
//   warp 0   TMA loads of K (and V) tiles into a 3-stage ring;
//   warp 1   one thread issues S = Q K^T (M 128, N 64, K 128) into one of two
//            TMEM S buffers, then O += P V (M 128, N 128, K 64) into TMEM;
//   warps 4-7  one thread per row: S row from TMEM, mask, softmax, P (bf16)
//            into shared memory in the 128-byte swizzled K-major layout,
//            lazy O rescaling, epilogue.
// Modes:
//   CMP   items over vision queries; keys = compressed blocks (K_cmp, V_cmp).
//         Segment 1 computes each row's log-sum-exp; segment 2 recomputes S,
//         forms exact probabilities, sums them over the group's heads into
//         the block importance, and accumulates O = P V (already normalised).
//   VIS   items over vision queries; segment 1 = the union of the blocks the
//         item's queries selected (a query's row masks blocks it did not
//         select), segment 2 = the window keys; the epilogue adds the three
//         gated branch outputs and writes the final vision rows.
//   TEXT  items = (text query tile, key split); partial O, max and sum go to a
//         buffer that a small combine kernel reduces.
#include <cuda.h>
#include <math.h>
#include <string.h>

#include "tc_attn.h"
#include "tc_ptx.cuh"

namespace vnsa {

namespace {

constexpr int kThreads = 256;
constexpr int kRows = 128;        // MMA M
constexpr int kKeys = 64;         // keys per tile
constexpr int kD = 128;           // head dim of this path
constexpr int kStages = 3;
constexpr float kRescale = 8.0f;  // lazy rescale threshold (log2 units)
constexpr int kTextSplitKeys = 8192;
constexpr size_t kTextPartBytes = 256ull << 20;
constexpr int kPartStride = kD + 2;  // floats per partial row: O, m, l

constexpr uint32_t SM_Q = 0;                                  // 2 x [128][64] bf16
constexpr uint32_t SM_KV = 32768;                             // stages x (K, V)
constexpr uint32_t KV_BYTES = 32768;
constexpr uint32_t SM_P = SM_KV + kStages * KV_BYTES;         // 2 x [128][64] fp16
constexpr uint32_t P_BYTES = 16384;
constexpr uint32_t SM_P32 = SM_P + 2 * P_BYTES;               // [128][65] fp32
constexpr uint32_t P32_STRIDE = 65;
constexpr int kPlanSmem = 1152;                               // selection tiles per item
constexpr uint32_t SM_PLAN = SM_P32 + kRows * P32_STRIDE * 4; // [2][kPlanSmem] int32
constexpr uint32_t SM_BAR = SM_PLAN + 2 * kPlanSmem * 4;      // barriers
constexpr uint32_t SM_TOTAL = SM_BAR + 256;
constexpr uint32_t SMEM_BYTES = SM_TOTAL + 1024;              // + alignment slack

// barrier slots (8 bytes each) after SM_BAR
constexpr int B_KV_FULL = 0, B_KV_EMPTY = 3, B_S_FULL = 6, B_P_FULL = 8, B_PV_DONE = 10,
              B_Q_FULL = 12, B_GRP = 13, B_FINAL = 14, B_COUNT = 15;

constexpr uint32_t TM_S0 = 0, TM_O0 = 128, TM_O1 = 256, TM_COLS = 512;

enum Mode { MODE_CMP = 0, MODE_VIS = 1, MODE_TEXT = 2 };
enum Kind { K_STATS = 0, K_EXACT = 1, K_SLC = 2, K_SWA = 3, K_TEXT = 4 };

struct TcParams {
    CUtensorMap tm_k, tm_v;    // K (bf16, the caller's) and V (fp16 copy): [n rows][h_kv*d]
    CUtensorMap tm_kc, tm_vc;  // compacted vision K (bf16), V (fp16), if not contiguous
    CUtensorMap tm_kb, tm_vb;  // K_cmp (bf16), V_cmp (fp16): [nb_max rows][h_kv*d]
    LayerParams L;
    const int32_t *plan;       // VIS: [item][1 + 2*plan_max]
    int plan_max;
    float *part;               // TEXT partials: [item][128][kPartStride]
    int part_items;
    int mode;
};

// ---------------------------------------------------------------------------
// Work decomposition shared by every role (all compute the same values).
struct Work {
    int qt;        // queries per item
    int rows;      // used MMA rows = qt * r
    int n_q;       // queries of the item kind (N_v or N_t)
    int n_tiles_q; // query tiles per group
    int nsplit;    // text key splits
    int split_len; // keys per split
    int items;
    int nb;
    int contiguous, vis_base;
};

__device__ __forceinline__ Work make_work(const TcParams &P, const Counts &cn) {
    Work w;
    const LayerParams &L = P.L;
    w.qt = kRows / L.r;
    w.rows = w.qt * L.r;
    w.nb = cn.nb;
    w.contiguous = cn.contiguous;
    w.vis_base = cn.vis_base;
    w.nsplit = 1;
    w.split_len = 0;
    if (P.mode == MODE_TEXT) {
        w.n_q = cn.n_text;
        w.n_tiles_q = (w.n_q + w.qt - 1) / w.qt;
        const int span = w.n_q > 0 ? L.txt[w.n_q - 1] + 1 : 0;
        int ns = (span + kTextSplitKeys - 1) / kTextSplitKeys;
        const int tiles = L.h_kv * w.n_tiles_q;
        if (tiles > 0) ns = min(ns, max(1, P.part_items / tiles));
        w.nsplit = max(1, ns);
        const int per = (span + w.nsplit - 1) / w.nsplit;
        w.split_len = (per + kKeys - 1) / kKeys * kKeys;
        w.items = tiles * w.nsplit;
    } else {
        w.n_q = cn.n_vision;
        w.n_tiles_q = (w.n_q + w.qt - 1) / w.qt;
        w.items = L.h_kv * w.n_tiles_q;
    }
    return w;
}

struct Item {
    int g, q0, nq, split;
    int last_pos;   // TEXT: position of the item's last query; else its vision rank
    int nseg;
    int seg_kind[2];
    int seg_tiles[2];
    int key_lo;     // VIS window start (vision rank) / TEXT split start (position)
    int key_hi;     // VIS: last query rank; TEXT: last key (inclusive)
};

__device__ __forceinline__ Item make_item(const TcParams &P, const Work &w, int item) {
    const LayerParams &L = P.L;
    Item it;
    int tile;
    if (P.mode == MODE_TEXT) {
        const int per_split = L.h_kv * w.n_tiles_q;
        it.split = item / per_split;
        const int rem = item % per_split;
        it.g = rem / w.n_tiles_q;
        tile = rem % w.n_tiles_q;
    } else {
        it.split = 0;
        it.g = item / w.n_tiles_q;
        tile = item % w.n_tiles_q;
    }
    it.q0 = tile * w.qt;
    it.nq = min(w.qt, w.n_q - it.q0);
    const int ql = it.q0 + it.nq - 1;
    it.key_lo = 0;
    it.key_hi = 0;
    if (P.mode == MODE_CMP) {
        it.last_pos = ql;
        const int c_last = min((ql + 1) / L.block, w.nb);
        const int t = (c_last + kKeys - 1) / kKeys;
        it.nseg = 2;
        it.seg_kind[0] = K_STATS;
        it.seg_kind[1] = K_EXACT;
        it.seg_tiles[0] = t;
        it.seg_tiles[1] = t;
    } else if (P.mode == MODE_VIS) {
        it.last_pos = ql;
        it.nseg = 2;
        it.seg_kind[0] = K_SLC;
        it.seg_kind[1] = K_SWA;
        it.seg_tiles[0] = P.plan[(size_t)item * (1 + 2 * P.plan_max)];
        it.key_lo = max(0, it.q0 - L.window + 1);
        it.key_hi = ql;
        it.seg_tiles[1] = (ql - it.key_lo + kKeys) / kKeys;
    } else {
        it.last_pos = L.txt[ql];
        it.nseg = 1;
        it.seg_kind[0] = K_TEXT;
        it.seg_kind[1] = K_TEXT;
        it.key_lo = it.split * w.split_len;
        it.key_hi = min(it.key_lo + w.split_len, it.last_pos + 1) - 1;
        it.seg_tiles[0] = it.key_hi >= it.key_lo ? (it.key_hi - it.key_lo + kKeys) / kKeys : 0;
        it.seg_tiles[1] = 0;
    }
    return it;
}

__device__ __forceinline__ int item_tiles(const Item &it) {
    return it.seg_tiles[0] + (it.nseg > 1 ? it.seg_tiles[1] : 0);
}

__device__ __forceinline__ bool kind_has_pv(int kind) { return kind != K_STATS; }

// First key of tile x of a segment: a vision rank (SLC, SWA), a compressed
// block (STATS, EXACT) or a position (TEXT).
__device__ __forceinline__ int tile_key0(const TcParams &P, const Item &it, int item, int kind,
                                         int x) {
    switch (kind) {
        case K_SLC: return P.plan[(size_t)item * (1 + 2 * P.plan_max) + 1 + x] * kKeys;
        case K_SWA: return it.key_lo + x * kKeys;
        case K_TEXT: return it.key_lo + x * kKeys;
        default: return x * kKeys;
    }
}

// ---------------------------------------------------------------------------
struct Smem {
    uint8_t *base;
    uint32_t base_u32;
    __device__ uint32_t bar(int i) const { return base_u32 + SM_BAR + 8u * (uint32_t)i; }
    __device__ uint32_t *tmem_slot() const { return (uint32_t *)(base + SM_BAR + 8 * B_COUNT); }
    __device__ volatile int *abort_flag() const {
        return (volatile int *)(base + SM_BAR + 8 * B_COUNT + 8);
    }
};

__device__ __forceinline__ uint64_t desc_kmajor(uint32_t addr) {
    return ptx::sdesc_sw128(addr, 16, 1024);
}
__device__ __forceinline__ uint64_t desc_vmajor(uint32_t addr) {
    return ptx::sdesc_sw128(addr, 8192, 1024);
}

// ---------------------------------------------------------------------------
// Producer: TMA loads of the K (and V) tiles of every item, in order.
__device__ void run_producer(const TcParams &P, const Work &w, const Smem &sm) {
    const LayerParams &L = P.L;
    volatile int *abort = sm.abort_flag();
    uint32_t gt = 0;
    const CUtensorMap *mk, *mv;
    for (int item = blockIdx.x; item < w.items; item += gridDim.x) {
        const Item it = make_item(P, w, item);
        int vbase = 0;
        if (P.mode == MODE_CMP) {
            mk = &P.tm_kb;
            mv = &P.tm_vb;
        } else if (P.mode == MODE_VIS) {
            mk = w.contiguous ? &P.tm_k : &P.tm_kc;
            mv = w.contiguous ? &P.tm_v : &P.tm_vc;
            vbase = w.contiguous ? w.vis_base : 0;
        } else {
            mk = &P.tm_k;
            mv = &P.tm_v;
        }
        for (int s = 0; s < it.nseg; ++s) {
            const int kind = it.seg_kind[s];
            for (int x = 0; x < it.seg_tiles[s]; ++x, ++gt) {
                const uint32_t st = gt % kStages;
                if (gt >= (uint32_t)kStages &&
                    !ptx::mbar_wait(sm.bar(B_KV_EMPTY + st), ((gt / kStages) - 1) & 1, abort,
                                    L.status))
                    return;
                const int key0 = tile_key0(P, it, item, kind, x);
                const int y = (kind == K_SLC || kind == K_SWA) ? vbase + key0 : key0;
                const bool pv = kind_has_pv(kind);
                const uint32_t kv = sm.base_u32 + SM_KV + st * KV_BYTES;
                ptx::mbar_expect_tx(sm.bar(B_KV_FULL + st), pv ? 32768u : 16384u);
                const int xc = it.g * kD;
                ptx::tma_load_2d(kv, mk, sm.bar(B_KV_FULL + st), xc, y);
                ptx::tma_load_2d(kv + 8192, mk, sm.bar(B_KV_FULL + st), xc + 64, y);
                if (pv) {
                    ptx::tma_load_2d(kv + 16384, mv, sm.bar(B_KV_FULL + st), xc, y);
                    ptx::tma_load_2d(kv + 16384 + 8192, mv, sm.bar(B_KV_FULL + st), xc + 64, y);
                }
            }
        }
    }
    // make sure no load is still landing in shared memory when the CTA ends
    for (uint32_t back = 1; back <= (uint32_t)kStages && back <= gt; ++back) {
        const uint32_t t = gt - back;
        if (!ptx::mbar_wait(sm.bar(B_KV_FULL + t % kStages), (t / kStages) & 1, abort, L.status))
            return;
    }
}

// ---------------------------------------------------------------------------
// MMA issuer (one thread).
__device__ void run_mma(const TcParams &P, const Work &w, const Smem &sm, uint32_t tmem) {
    const LayerParams &L = P.L;
    volatile int *abort = sm.abort_flag();
    // S = Q K^T with bf16 operands; O += P V with fp16 operands (P and V in
    // fp16: 11-bit significands keep the probability rounding small)
    constexpr uint32_t idesc_s = ptx::idesc_f16kind(kRows, kKeys, 0, 0, 1u);
    constexpr uint32_t idesc_pv = ptx::idesc_f16kind(kRows, kD, 0, 1, 0u);
    const uint32_t q_addr = sm.base_u32 + SM_Q;
    uint32_t gt = 0, nitems = 0;
    uint32_t npv = 0;  // P V products issued; P buffer and PV-done barrier = npv & 1
    bool ok = true;
    for (int item = blockIdx.x; ok && item < w.items; item += gridDim.x) {
        const Item it = make_item(P, w, item);
        if (item_tiles(it) == 0) continue;
        if (!ptx::mbar_wait(sm.bar(B_Q_FULL), nitems & 1, abort, L.status)) { ok = false; break; }
        ++nitems;
        ptx::tc_fence_after();
        bool pending = false;
        uint32_t pend_st = 0, pend_col = 0, pend_acc = 0, pend_gt = 0;
        for (int s = 0; ok && s < it.nseg; ++s) {
            const int kind = it.seg_kind[s];
            const uint32_t ocol = (kind == K_SWA) ? TM_O1 : TM_O0;
            for (int x = 0; x < it.seg_tiles[s]; ++x, ++gt) {
                const uint32_t st = gt % kStages, b = gt & 1;
                if (gt >= 2 && !ptx::mbar_wait(sm.bar(B_P_FULL + b), ((gt - 2) >> 1) & 1, abort,
                                               L.status)) { ok = false; break; }
                if (!ptx::mbar_wait(sm.bar(B_KV_FULL + st), (gt / kStages) & 1, abort, L.status)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t kv = sm.base_u32 + SM_KV + st * KV_BYTES;
#pragma unroll
                for (int k = 0; k < kD / 16; ++k) {
                    const uint32_t off = (uint32_t)(k >> 2) * 16384u + (uint32_t)(k & 3) * 32u;
                    const uint32_t koff = (uint32_t)(k >> 2) * 8192u + (uint32_t)(k & 3) * 32u;
                    ptx::mma_ss(tmem + TM_S0 + b * kKeys, desc_kmajor(q_addr + off),
                                desc_kmajor(kv + koff), idesc_s, k > 0 ? 1u : 0u);
                }
                ptx::mma_commit(sm.bar(B_S_FULL + b));
                if (!kind_has_pv(kind)) ptx::mma_commit(sm.bar(B_KV_EMPTY + st));
                if (pending) {
                    if (!ptx::mbar_wait(sm.bar(B_P_FULL + (pend_gt & 1)), (pend_gt >> 1) & 1, abort,
                                        L.status)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t vb = sm.base_u32 + SM_KV + pend_st * KV_BYTES + 16384;
                    const uint32_t pa = sm.base_u32 + SM_P + (npv & 1) * P_BYTES;
#pragma unroll
                    for (int k = 0; k < kKeys / 16; ++k)
                        ptx::mma_ss(tmem + pend_col, desc_kmajor(pa + (uint32_t)k * 32u),
                                    desc_vmajor(vb + (uint32_t)k * 2048u), idesc_pv,
                                    (k > 0 || pend_acc) ? 1u : 0u);
                    ptx::mma_commit(sm.bar(B_PV_DONE + (npv & 1)));
                    ptx::mma_commit(sm.bar(B_KV_EMPTY + pend_st));
                    ++npv;
                    pending = false;
                }
                if (kind_has_pv(kind)) {
                    pending = true;
                    pend_st = st;
                    pend_col = ocol;
                    pend_acc = x > 0 ? 1u : 0u;
                    pend_gt = gt;
                }
            }
        }
        if (ok && pending) {
            if (!ptx::mbar_wait(sm.bar(B_P_FULL + (pend_gt & 1)), (pend_gt >> 1) & 1, abort,
                                L.status)) { ok = false; break; }
            ptx::tc_fence_after();
            const uint32_t vb = sm.base_u32 + SM_KV + pend_st * KV_BYTES + 16384;
            const uint32_t pa = sm.base_u32 + SM_P + (npv & 1) * P_BYTES;
#pragma unroll
            for (int k = 0; k < kKeys / 16; ++k)
                ptx::mma_ss(tmem + pend_col, desc_kmajor(pa + (uint32_t)k * 32u),
                            desc_vmajor(vb + (uint32_t)k * 2048u), idesc_pv,
                            (k > 0 || pend_acc) ? 1u : 0u);
            ptx::mma_commit(sm.bar(B_PV_DONE + (npv & 1)));
            ptx::mma_commit(sm.bar(B_KV_EMPTY + pend_st));
            ++npv;
        }
    }
    // every MMA this thread issued has completed once this barrier flips
    ptx::mma_commit(sm.bar(B_FINAL));
    ptx::mbar_wait(sm.bar(B_FINAL), 0, abort, L.status, 200000000ull);
}

// ---------------------------------------------------------------------------
// Softmax / epilogue warpgroup (warps 4-7): thread rho owns MMA row rho.
struct RowCtx {
    bool valid;
    int qi, hl, h;
    int i;      // vision rank (CMP/VIS) or text rank (TEXT)
    int t;      // position of the query token
    int c_vis;  // CMP: visible compressed blocks
};

__device__ __forceinline__ void group_sync(const Smem &sm, uint32_t &phase, bool &ok,
                                           const LayerParams &L) {
    ptx::mbar_arrive(sm.bar(B_GRP));
    bool r = ptx::mbar_wait(sm.bar(B_GRP), phase & 1, sm.abort_flag(), L.status);
    ++phase;
    ok = __all_sync(0xffffffffu, r && ok);
}

// P row (fp16) into the 128-byte swizzled K-major layout: 16-byte chunk c8 of
// row rho goes to chunk c8 ^ (rho % 8).
__device__ __forceinline__ void store_p_f16(const Smem &sm, uint32_t buf, int rho,
                                            const float (&p)[64]) {
    uint8_t *row = sm.base + SM_P + buf * P_BYTES + rho * 128;
#pragma unroll
    for (int c8 = 0; c8 < 8; ++c8) {
        uint4 v;
        __half2 a = __floats2half2_rn(p[8 * c8 + 0], p[8 * c8 + 1]);
        __half2 b = __floats2half2_rn(p[8 * c8 + 2], p[8 * c8 + 3]);
        __half2 c = __floats2half2_rn(p[8 * c8 + 4], p[8 * c8 + 5]);
        __half2 d = __floats2half2_rn(p[8 * c8 + 6], p[8 * c8 + 7]);
        v.x = *reinterpret_cast<uint32_t *>(&a);
        v.y = *reinterpret_cast<uint32_t *>(&b);
        v.z = *reinterpret_cast<uint32_t *>(&c);
        v.w = *reinterpret_cast<uint32_t *>(&d);
        *reinterpret_cast<uint4 *>(row + ((c8 ^ (rho & 7)) << 4)) = v;
    }
}

__device__ void run_softmax(const TcParams &P, const Work &w, const Smem &sm, uint32_t tmem) {
    const LayerParams &L = P.L;
    volatile int *abort = sm.abort_flag();
    const int rho = threadIdx.x - 128;          // 0..127
    const int wq = (threadIdx.x >> 5) & 3;      // TMEM lane quadrant of this warp
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const float sc = L.scale_log2;
    const __nv_bfloat16 *Q = (const __nv_bfloat16 *)L.q;
    uint32_t gt = 0, npv = 0, gphase = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < w.items; item += gridDim.x) {
        const Item it = make_item(P, w, item);
        // per-row context
        RowCtx rc;
        rc.qi = rho / L.r;
        rc.hl = rho % L.r;
        rc.h = it.g * L.r + rc.hl;
        rc.valid = rho < w.rows && rc.qi < it.nq;
        rc.i = it.q0 + min(rc.qi, max(it.nq - 1, 0));
        if (P.mode == MODE_TEXT) rc.t = it.nq > 0 ? L.txt[rc.i] : 0;
        else rc.t = it.nq > 0 ? L.vis[rc.i] : 0;
        rc.c_vis = min((rc.i + 1) / L.block, w.nb);
        const int ntiles = item_tiles(it);
        if (ntiles == 0) {
            // nothing attended: empty branch outputs
            if (rc.valid) {
                if (P.mode == MODE_CMP) {
                    float *orow = L.o_cmp_ws + ((size_t)rc.i * L.h_q + rc.h) * kD;
                    for (int e = 0; e < kD; e += 4)
                        *reinterpret_cast<float4 *>(orow + e) = make_float4(0.f, 0.f, 0.f, 0.f);
                    L.lse[(size_t)rc.i * L.h_q + rc.h] = -INFINITY;
                } else if (P.mode == MODE_TEXT) {
                    float *pr = P.part + ((size_t)item * kRows + rho) * kPartStride;
                    pr[kD] = -INFINITY;
                    pr[kD + 1] = 0.f;
                }
            }
            continue;
        }
        // ---- Q tile: rows gathered from their positions, 16-byte pieces
        for (int e = rho; e < kRows * 16; e += 128) {
            const int row = e >> 4, c16 = e & 15;
            const int qi = row / L.r, hl = row % L.r;
            uint4 val = make_uint4(0u, 0u, 0u, 0u);
            if (row < w.rows && qi < it.nq) {
                const int q = it.q0 + qi;
                const int t = (P.mode == MODE_TEXT) ? L.txt[q] : L.vis[q];
                const __nv_bfloat16 *src =
                    Q + ((size_t)t * L.h_q + it.g * L.r + hl) * kD + c16 * 8;
                val = __ldg(reinterpret_cast<const uint4 *>(src));
            }
            const int hf = c16 >> 3, c = c16 & 7;
            *reinterpret_cast<uint4 *>(sm.base + SM_Q + hf * 16384 + row * 128 +
                                       ((c ^ (row & 7)) << 4)) = val;
        }
        ptx::fence_proxy_async();
        ptx::mbar_arrive(sm.bar(B_Q_FULL));

        // VIS: the item's selection tiles (first key, query mask) into shared
        // memory, once every thread is done with the previous item's copy
        const int32_t *plan_s = (const int32_t *)(sm.base + SM_PLAN);
        if (P.mode == MODE_VIS) {
            group_sync(sm, gphase, ok, L);
            if (!ok) break;
            int32_t *dst = (int32_t *)(sm.base + SM_PLAN);
            const int32_t *src = P.plan + (size_t)item * (1 + 2 * P.plan_max);
            for (int x = rho; x < it.seg_tiles[0]; x += 128) {
                dst[x] = src[1 + x] * kKeys;
                dst[kPlanSmem + x] = src[1 + P.plan_max + x];
            }
            group_sync(sm, gphase, ok, L);
            if (!ok) break;
        }

        float lse2 = -INFINITY;                 // CMP: from the stats segment
        float m_s = -INFINITY, l_s = 0.f;       // segment 0 running max / sum
        float l_w = 0.f;                        // segment 1 (VIS window) sum
        for (int s = 0; ok && s < it.nseg; ++s) {
            const int kind = it.seg_kind[s];
            float m_run = -INFINITY, l_run = 0.f;
            const uint32_t ocol = (kind == K_SWA) ? TM_O1 : TM_O0;
            for (int x = 0; x < it.seg_tiles[s]; ++x, ++gt) {
                const uint32_t b = gt & 1;
                const int key0 = kind == K_SLC ? plan_s[x] : tile_key0(P, it, item, kind, x);
                // column range [lo, hi] of valid keys for this row
                int lo = 1, hi = 0;
                if (rc.valid) {
                    switch (kind) {
                        case K_STATS:
                        case K_EXACT: lo = 0; hi = rc.c_vis - 1 - key0; break;
                        case K_SLC:
                            if (((uint32_t)plan_s[kPlanSmem + x] >> rc.qi) & 1u) {
                                lo = 0;
                                hi = rc.i - key0;
                            }
                            break;
                        case K_SWA: lo = rc.i - L.window + 1 - key0; hi = rc.i - key0; break;
                        default: lo = 0; hi = rc.t - key0; break;
                    }
                    lo = max(lo, 0);
                    hi = min(hi, kKeys - 1);
                }
                const bool full = __all_sync(0xffffffffu, lo == 0 && hi == kKeys - 1);
                bool r = ptx::mbar_wait(sm.bar(B_S_FULL + b), (gt >> 1) & 1, abort, L.status);
                ok = __all_sync(0xffffffffu, r && ok);
                if (!ok) break;
                ptx::tc_fence_after();
                float sv[64];
                {
                    float a[32], c[32];
                    ptx::tmem_ld32(tmem + lane_base + TM_S0 + b * kKeys, a);
                    ptx::tmem_ld32(tmem + lane_base + TM_S0 + b * kKeys + 32, c);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 32; ++k) { sv[k] = a[k]; sv[32 + k] = c[k]; }
                }
                if (full) {
#pragma unroll
                    for (int k = 0; k < 64; ++k) sv[k] *= sc;
                } else {
#pragma unroll
                    for (int k = 0; k < 64; ++k) sv[k] = (k >= lo && k <= hi) ? sv[k] * sc : -INFINITY;
                }
                float mx;
                {
                    float m8[8];
#pragma unroll
                    for (int z = 0; z < 8; ++z) m8[z] = sv[z];
#pragma unroll
                    for (int k = 8; k < 64; ++k) m8[k & 7] = fmaxf(m8[k & 7], sv[k]);
                    mx = fmaxf(fmaxf(fmaxf(m8[0], m8[1]), fmaxf(m8[2], m8[3])),
                               fmaxf(fmaxf(m8[4], m8[5]), fmaxf(m8[6], m8[7])));
                }
                if (kind == K_STATS) {
                    const float mn = fmaxf(m_run, mx);
                    const float mu = mn == -INFINITY ? 0.f : mn;
                    float a8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int k = 0; k < 64; ++k) a8[k & 7] += ptx::ex2(sv[k] - mu);
                    const float acc = ((a8[0] + a8[1]) + (a8[2] + a8[3])) +
                                      ((a8[4] + a8[5]) + (a8[6] + a8[7]));
                    l_run = l_run * ptx::ex2(m_run - mu) + acc;
                    m_run = mn;
                    ptx::tc_fence_before();
                    ptx::mbar_arrive(sm.bar(B_P_FULL + b));
                    continue;
                }
                float pv[64];
                if (kind == K_EXACT) {
                    const bool live = lse2 != -INFINITY;
#pragma unroll
                    for (int k = 0; k < 64; ++k) pv[k] = live ? ptx::ex2(sv[k] - lse2) : 0.f;
                    // importance: sum of the group's heads for each (query, block)
                    float *p32 = (float *)(sm.base + SM_P32);
#pragma unroll
                    for (int k = 0; k < 64; ++k) p32[rho * P32_STRIDE + k] = pv[k];
                    group_sync(sm, gphase, ok, L);
                    if (!ok) break;
                    for (int pair = rho; pair < it.nq * 64; pair += 128) {
                        const int qi = pair >> 6, col = pair & 63;
                        const int iq = it.q0 + qi;
                        const int cq = min((iq + 1) / L.block, w.nb);
                        if (key0 + col < cq) {
                            float acc = 0.f;
                            for (int hh = 0; hh < L.r; ++hh)
                                acc += p32[(qi * L.r + hh) * P32_STRIDE + col];
                            L.imp[((size_t)it.g * L.n_max + iq) * L.imp_stride + key0 + col] = acc;
                        }
                    }
                    group_sync(sm, gphase, ok, L);
                    if (!ok) break;
                } else {
                    // online softmax with lazy rescaling of O
                    const float mn = fmaxf(m_run, mx);
                    const bool need = mn > m_run + kRescale;
                    float factor = 1.f;
                    if (need) {
                        factor = ptx::ex2(m_run - mn);  // 0 if m_run = -inf
                        l_run *= factor;
                        m_run = mn;
                    }
                    const float mu = m_run == -INFINITY ? 0.f : m_run;
                    float a8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int k = 0; k < 64; ++k) {
                        pv[k] = ptx::ex2(sv[k] - mu);
                        a8[k & 7] += pv[k];
                    }
                    l_run += ((a8[0] + a8[1]) + (a8[2] + a8[3])) + ((a8[4] + a8[5]) + (a8[6] + a8[7]));
                    const bool resc = __any_sync(0xffffffffu, need && x > 0);
                    if (resc) {
                        // O may only be rescaled once every earlier P V has landed
                        if (npv > 0) {
                            bool r2 = ptx::mbar_wait(sm.bar(B_PV_DONE + ((npv - 1) & 1)),
                                                     ((npv - 1) >> 1) & 1, abort, L.status);
                            ok = __all_sync(0xffffffffu, r2 && ok);
                            if (!ok) break;
                        }
                        ptx::tc_fence_after();
                        const float f = (need && x > 0) ? factor : 1.f;
#pragma unroll
                        for (int ch = 0; ch < 4; ++ch) {
                            float o[32];
                            ptx::tmem_ld32(tmem + lane_base + ocol + ch * 32, o);
                            ptx::tmem_wait_ld();
#pragma unroll
                            for (int k = 0; k < 32; ++k) o[k] *= f;
                            ptx::tmem_st32(tmem + lane_base + ocol + ch * 32, o);
                        }
                        ptx::tmem_wait_st();
                    }
                }
                // P into buffer npv & 1 once the P V that last read it (#npv-2) is done
                if (npv > 1) {
                    bool r3 = ptx::mbar_wait(sm.bar(B_PV_DONE + (npv & 1)), ((npv - 2) >> 1) & 1,
                                             abort, L.status);
                    ok = __all_sync(0xffffffffu, r3 && ok);
                    if (!ok) break;
                }
                store_p_f16(sm, npv & 1, rho, pv);
                ptx::fence_proxy_async();
                ptx::tc_fence_before();
                ptx::mbar_arrive(sm.bar(B_P_FULL + b));
                ++npv;
            }
            if (!ok) break;
            if (kind == K_STATS) {
                lse2 = (m_run == -INFINITY || l_run <= 0.f) ? -INFINITY : m_run + log2f(l_run);
            } else if (s == 0) {
                m_s = m_run;
                l_s = l_run;
            } else {
                l_w = l_run;
            }
        }
        if (!ok) break;
        // ---- epilogue: wait for the item's last P V (#npv-1)
        {
            bool r = ptx::mbar_wait(sm.bar(B_PV_DONE + ((npv - 1) & 1)), ((npv - 1) >> 1) & 1,
                                    abort, L.status);
            ok = __all_sync(0xffffffffu, r && ok);
            if (!ok) break;
            ptx::tc_fence_after();
        }
        if (P.mode == MODE_CMP) {
            float *orow = L.o_cmp_ws + ((size_t)rc.i * L.h_q + rc.h) * kD;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float o[32];
                ptx::tmem_ld32(tmem + lane_base + TM_O0 + ch * 32, o);
                ptx::tmem_wait_ld();
                if (rc.valid) {
#pragma unroll
                    for (int k = 0; k < 32; k += 4)
                        *reinterpret_cast<float4 *>(orow + ch * 32 + k) =
                            make_float4(o[k], o[k + 1], o[k + 2], o[k + 3]);
                }
            }
            if (rc.valid) L.lse[(size_t)rc.i * L.h_q + rc.h] = lse2 * kLn2;
        } else if (P.mode == MODE_VIS) {
            const float *gl = L.gate + ((size_t)rc.t * L.h_q + rc.h) * 3;
            float gc = 0.f, gs = 0.f, gw = 0.f;
            if (rc.valid) {
                gc = sigmoidf_(gl[0]);
                gs = sigmoidf_(gl[1]);
                gw = sigmoidf_(gl[2]);
            }
            const float inv_s = l_s > 0.f ? 1.f / l_s : 0.f;
            const float inv_w = l_w > 0.f ? 1.f / l_w : 0.f;
            const float *oc = L.o_cmp_ws + ((size_t)rc.i * L.h_q + rc.h) * kD;
            __nv_bfloat16 *orow = (__nv_bfloat16 *)L.out + ((size_t)rc.t * L.h_q + rc.h) * kD;
            const size_t drow = ((size_t)rc.t * L.h_q + rc.h) * kD;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float a[32], c[32];
                ptx::tmem_ld32(tmem + lane_base + TM_O0 + ch * 32, a);
                ptx::tmem_ld32(tmem + lane_base + TM_O1 + ch * 32, c);
                ptx::tmem_wait_ld();
                if (!rc.valid) continue;
#pragma unroll
                for (int k = 0; k < 32; k += 8) {
                    float o8[8];
#pragma unroll
                    for (int z = 0; z < 8; ++z) {
                        const int e = ch * 32 + k + z;
                        const float os = l_s > 0.f ? a[k + z] * inv_s : 0.f;
                        const float ow = l_w > 0.f ? c[k + z] * inv_w : 0.f;
                        const float occ = oc[e];
                        o8[z] = gc * occ + gs * os + gw * ow;
                        if (L.dbg_o_cmp) L.dbg_o_cmp[drow + e] = occ;
                        if (L.dbg_o_slc) L.dbg_o_slc[drow + e] = os;
                        if (L.dbg_o_swa) L.dbg_o_swa[drow + e] = ow;
                    }
                    uint4 v;
                    __nv_bfloat162 b0 = __floats2bfloat162_rn(o8[0], o8[1]);
                    __nv_bfloat162 b1 = __floats2bfloat162_rn(o8[2], o8[3]);
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(o8[4], o8[5]);
                    __nv_bfloat162 b3 = __floats2bfloat162_rn(o8[6], o8[7]);
                    v.x = *reinterpret_cast<uint32_t *>(&b0);
                    v.y = *reinterpret_cast<uint32_t *>(&b1);
                    v.z = *reinterpret_cast<uint32_t *>(&b2);
                    v.w = *reinterpret_cast<uint32_t *>(&b3);
                    *reinterpret_cast<uint4 *>(orow + ch * 32 + k) = v;
                }
            }
        } else if (w.nsplit == 1) {
            // one key split: the item holds the whole softmax, write the row
            const float inv = l_s > 0.f ? 1.f / l_s : 0.f;
            __nv_bfloat16 *orow = (__nv_bfloat16 *)L.out + ((size_t)rc.t * L.h_q + rc.h) * kD;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float o[32];
                ptx::tmem_ld32(tmem + lane_base + TM_O0 + ch * 32, o);
                ptx::tmem_wait_ld();
                if (!rc.valid) continue;
#pragma unroll
                for (int k = 0; k < 32; k += 2) {
                    const float a = l_s > 0.f ? o[k] * inv : 0.f;
                    const float c = l_s > 0.f ? o[k + 1] * inv : 0.f;
                    *reinterpret_cast<__nv_bfloat162 *>(orow + ch * 32 + k) =
                        __floats2bfloat162_rn(a, c);
                }
            }
        } else {
            float *pr = P.part + ((size_t)item * kRows + rho) * kPartStride;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float o[32];
                ptx::tmem_ld32(tmem + lane_base + TM_O0 + ch * 32, o);
                ptx::tmem_wait_ld();
                if (rc.valid) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) pr[ch * 32 + k] = o[k];
                }
            }
            if (rc.valid) {
                pr[kD] = m_s;
                pr[kD + 1] = l_s;
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1) tc_attn_kernel(const __grid_constant__ TcParams P) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint32_t s_failed;
    const LayerParams &L = P.L;
    // skip the work if an earlier kernel already failed (one read, shared by
    // the whole CTA so that every thread takes the same path)
    if (threadIdx.x == 0) s_failed = *(volatile uint32_t *)L.status;
    __syncthreads();
    if (s_failed != 0) return;
    Smem sm;
    {
        const uint32_t raw = ptx::smem_u32(smem_raw);
        const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
        sm.base = smem_raw + pad;
        sm.base_u32 = raw + pad;
    }
    const Counts cn = *L.counts;
    const Work w = make_work(P, cn);
    if ((int)blockIdx.x >= w.items) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(sm.bar(B_KV_FULL + s), 1);
            ptx::mbar_init(sm.bar(B_KV_EMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(sm.bar(B_S_FULL + b), 1);
            ptx::mbar_init(sm.bar(B_P_FULL + b), 128);
        }
        ptx::mbar_init(sm.bar(B_PV_DONE), 1);
        ptx::mbar_init(sm.bar(B_PV_DONE + 1), 1);
        ptx::mbar_init(sm.bar(B_Q_FULL), 128);
        ptx::mbar_init(sm.bar(B_GRP), 128);
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
        if (lane == 0) run_producer(P, w, sm);
    } else if (warp == 1) {
        if (lane == 0) run_mma(P, w, sm, tmem);
        __syncwarp();
    } else if (warp >= 4) {
        run_softmax(P, w, sm, tmem);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, TM_COLS);
}

// ---------------------------------------------------------------------------
// Operand preparation for the tensor-core kernels:
//  * fp16 copies of V (all positions) and of V_cmp for the P V products.  A
//    bf16 value converts to fp16 exactly when its magnitude lies in the fp16
//    normal range; a value beyond the fp16 range is reported as a bounds error.
//  * vision K (bf16) and V (fp16) in vision order when the vision tokens are
//    not one contiguous run of positions (the TMA tiles need consecutive rows).
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 u, bool &overflow) {
    const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&u);
    uint4 r;
    __half2 *h = reinterpret_cast<__half2 *>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(b[i]);
        h[i] = __floats2half2_rn(f.x, f.y);
        if (fabsf(f.x) > 65504.f || fabsf(f.y) > 65504.f) overflow = true;
    }
    return r;
}

__global__ void prepare_kernel(LayerParams p, __nv_bfloat16 *kc, __half *vhc, __half *vh,
                               __half *vh_cmp) {
    const Counts cn = *p.counts;
    const size_t row_vec = (size_t)p.h_kv * kD / 8;  // 16-byte pieces per row
    const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t step = (size_t)gridDim.x * blockDim.x;
    bool overflow = false;
    const uint4 *v = reinterpret_cast<const uint4 *>(p.v);
    for (size_t e = tid; e < (size_t)p.n * row_vec; e += step)
        reinterpret_cast<uint4 *>(vh)[e] = bf16x8_to_f16x8(__ldg(v + e), overflow);
    const uint4 *vb = reinterpret_cast<const uint4 *>(p.v_cmp);
    for (size_t e = tid; e < (size_t)cn.nb * row_vec; e += step)
        reinterpret_cast<uint4 *>(vh_cmp)[e] = bf16x8_to_f16x8(vb[e], overflow);
    if (!cn.contiguous) {
        for (size_t e = tid; e < (size_t)cn.n_vision * row_vec; e += step) {
            const size_t u = e / row_vec, c = e % row_vec;
            const size_t src = (size_t)p.vis[u] * row_vec + c;
            reinterpret_cast<uint4 *>(kc)[e] = __ldg(reinterpret_cast<const uint4 *>(p.k) + src);
            reinterpret_cast<uint4 *>(vhc)[e] = bf16x8_to_f16x8(__ldg(v + src), overflow);
        }
    }
    if (overflow) report(p.status, VNSA_ERR_BOUNDS);
}

// ---------------------------------------------------------------------------
// Union of the blocks selected by the queries of each VIS item, with a mask of
// the queries that chose each block.  One warp per item.
__global__ void union_kernel(LayerParams p, int32_t *plan, int plan_max, int words) {
    extern __shared__ uint32_t sh[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wpb = blockDim.x >> 5;
    uint32_t *bm = sh + (size_t)warp * (2 * words + plan_max);
    uint32_t *pre = bm + words;
    uint32_t *qm = pre + words;
    const Counts cn = *p.counts;
    const int qt = kRows / p.r;
    const int n_tiles = (cn.n_vision + qt - 1) / qt;
    const int items = p.h_kv * n_tiles;
    for (int item = blockIdx.x * wpb + warp; item < items; item += gridDim.x * wpb) {
        const int g = item / n_tiles, q0 = (item % n_tiles) * qt;
        const int nq = min(qt, cn.n_vision - q0);
        for (int x = lane; x < words; x += 32) bm[x] = 0u;
        __syncwarp();
        const int ne = nq * p.top_k;
        for (int e = lane; e < ne; e += 32) {
            const int qi = e / p.top_k, x = e % p.top_k;
            const int j = p.idx_src[((size_t)g * p.idx_rows + q0 + qi) * p.top_k + x];
            if (j >= 0 && (j >> 5) < words) atomicOr(&bm[j >> 5], 1u << (j & 31));
        }
        __syncwarp();
        // exclusive prefix of popcounts over the words (lane-strided chunks)
        const int per = (words + 31) / 32;
        int local = 0;
        for (int x = lane * per; x < min(words, (lane + 1) * per); ++x) local += __popc(bm[x]);
        int incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - local;
        for (int x = lane * per; x < min(words, (lane + 1) * per); ++x) {
            pre[x] = run;
            run += __popc(bm[x]);
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        __syncwarp();
        int32_t *out = plan + (size_t)item * (1 + 2 * plan_max);
        for (int x = lane; x < total && x < plan_max; x += 32) qm[x] = 0u;
        for (int x = lane; x < words; x += 32) {
            uint32_t wbits = bm[x];
            int r = pre[x];
            while (wbits) {
                const int bit = __ffs(wbits) - 1;
                wbits &= wbits - 1;
                if (r < plan_max) out[1 + r] = x * 32 + bit;
                ++r;
            }
        }
        __syncwarp();
        for (int e = lane; e < ne; e += 32) {
            const int qi = e / p.top_k, x = e % p.top_k;
            const int j = p.idx_src[((size_t)g * p.idx_rows + q0 + qi) * p.top_k + x];
            if (j < 0 || (j >> 5) >= words) continue;
            const int r = pre[j >> 5] + __popc(bm[j >> 5] & ((1u << (j & 31)) - 1u));
            if (r < plan_max) atomicOr(&qm[r], 1u << qi);
        }
        __syncwarp();
        for (int x = lane; x < total && x < plan_max; x += 32) out[1 + plan_max + x] = (int)qm[x];
        if (lane == 0) {
            out[0] = min(total, plan_max);
            if (total > plan_max) report(p.status, VNSA_ERR_BOUNDS);
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// Text split-KV combine: one warp per (text query, head).
__device__ void text_combine_row(const LayerParams &p, const float *part, int part_items,
                                 int n_tt, int qt, int x, int h, int lane) {
    const Counts &cn = *p.counts;
    // same split rule as make_work
    const int span = p.txt[cn.n_text - 1] + 1;
    int ns = (span + kTextSplitKeys - 1) / kTextSplitKeys;
    const int tiles = p.h_kv * n_tt;
    ns = min(ns, max(1, part_items / tiles));
    ns = max(1, ns);
    const int g = h / p.r, hl = h % p.r;
    const int tt = x / qt, qi = x % qt;
    const int rho = qi * p.r + hl;
    float mmax = -INFINITY;
    for (int s = 0; s < ns; ++s) {
        const size_t item = (size_t)s * tiles + (size_t)g * n_tt + tt;
        const float *pr = part + (item * kRows + rho) * kPartStride;
        if (pr[kD + 1] > 0.f) mmax = fmaxf(mmax, pr[kD]);
    }
    float o[kD / 32];
#pragma unroll
    for (int c = 0; c < kD / 32; ++c) o[c] = 0.f;
    float l = 0.f;
    for (int s = 0; s < ns; ++s) {
        const size_t item = (size_t)s * tiles + (size_t)g * n_tt + tt;
        const float *pr = part + (item * kRows + rho) * kPartStride;
        const float ls = pr[kD + 1];
        if (!(ls > 0.f)) continue;
        const float wgt = exp2f(pr[kD] - mmax);
        l += wgt * ls;
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) o[c] += wgt * pr[lane + 32 * c];
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int t = p.txt[x];
    __nv_bfloat16 *orow = (__nv_bfloat16 *)p.out + ((size_t)t * p.h_q + h) * kD;
#pragma unroll
    for (int c = 0; c < kD / 32; ++c) orow[lane + 32 * c] = __float2bfloat16_rn(o[c] * inv);
}

__global__ void text_combine_kernel(LayerParams p, const float *part, int part_items) {
    const Counts cn = *p.counts;
    const int lane = threadIdx.x & 31;
    const int qt = kRows / p.r;
    const int n_tt = (cn.n_text + qt - 1) / qt;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    if (cn.n_text == 0) return;
    {
        // with a single key split the attention kernel wrote the rows itself
        const int span = p.txt[cn.n_text - 1] + 1;
        const int tiles = p.h_kv * n_tt;
        const int ns = max(1, min((span + kTextSplitKeys - 1) / kTextSplitKeys,
                                  max(1, part_items / tiles)));
        if (ns == 1) return;
    }
    for (int wi = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; wi < cn.n_text * p.h_q;
         wi += nwarps)
        text_combine_row(p, part, part_items, n_tt, qt, wi / p.h_q, wi % p.h_q, lane);
}

// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)ptr;
        cudaGetLastError();
    }
    return fn;
}

// 2-D map over [rows][h_kv*128] 16-bit elements with 64 x 64 boxes, 128-byte
// swizzle.
bool make_map(CUtensorMap *m, const void *base, int h_kv, long long rows, bool f16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || rows < 1) return false;
    cuuint64_t dims[2] = {(cuuint64_t)h_kv * kD, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)h_kv * kD * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
              const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

struct TcState {
    vnsa_config cfg;
    int num_sms;
    int plan_max;
    int part_items;
    __nv_bfloat16 *kc;  // vision K in vision order (non-contiguous vision only)
    __half *vhc;        // vision V (fp16) in vision order (non-contiguous vision only)
    __half *vh;         // V in fp16, all positions
    __half *vh_cmp;     // V_cmp in fp16
    int32_t *plan;
    float *part;
};

bool tc_supported(const vnsa_config &c) {
    const int qt = kRows / (c.h_q / c.h_kv);
    return c.dtype == VNSA_BF16 && c.d == kD && c.block == kKeys && c.h_q / c.h_kv <= 16 &&
           qt * c.top_k <= kPlanSmem && encode_fn() != nullptr;
}

static size_t plan_bytes(const vnsa_config &c) {
    const int qt = kRows / (c.h_q / c.h_kv);
    const size_t items = (size_t)c.h_kv * ((c.n_max + qt - 1) / qt);
    return items * (1 + 2 * (size_t)qt * c.top_k) * 4;
}

size_t tc_workspace_bytes(const vnsa_config &c) {
    if (c.dtype != VNSA_BF16 || c.d != kD || c.block != kKeys) return 0;
    const size_t kv = (size_t)c.n_max * c.h_kv * kD * 2;
    const size_t kvb = (size_t)(c.n_max / c.block + 1) * c.h_kv * kD * 2;
    return up256(kv) * 3 + up256(kvb) + up256(plan_bytes(c)) + kTextPartBytes;
}

cudaError_t tc_create(const vnsa_config &c, void *ws, TcState **out) {
    *out = nullptr;
    if (!tc_supported(c)) return cudaSuccess;
    TcState *st = new TcState();
    st->cfg = c;
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&st->num_sms, cudaDevAttrMultiProcessorCount, dev);
    const int qt = kRows / (c.h_q / c.h_kv);
    st->plan_max = qt * c.top_k;
    st->part_items = (int)(kTextPartBytes / ((size_t)kRows * kPartStride * 4));
    char *p = (char *)ws;
    const size_t kv = up256((size_t)c.n_max * c.h_kv * kD * 2);
    const size_t kvb = up256((size_t)(c.n_max / c.block + 1) * c.h_kv * kD * 2);
    st->kc = (__nv_bfloat16 *)p;
    st->vhc = (__half *)(p + kv);
    st->vh = (__half *)(p + 2 * kv);
    st->vh_cmp = (__half *)(p + 3 * kv);
    st->plan = (int32_t *)(p + 3 * kv + kvb);
    st->part = (float *)(p + 3 * kv + kvb + up256(plan_bytes(c)));
    cudaError_t e = cudaFuncSetAttribute(tc_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) {
        delete st;
        return e;
    }
    *out = st;
    return cudaSuccess;
}

cudaError_t tc_forward(TcState *st, const LayerParams &L, cudaStream_t s, cudaEvent_t *ev,
                       int *ran, int *launches, bool forced) {
    if (!st) return cudaErrorNotSupported;
    const vnsa_config &c = st->cfg;
    TcParams P;
    memset(&P, 0, sizeof(P));
    P.L = L;
    P.plan = st->plan;
    P.plan_max = st->plan_max;
    P.part = st->part;
    P.part_items = st->part_items;
    const int nb_rows = c.n_max / c.block > 0 ? c.n_max / c.block : 1;
    if (!make_map(&P.tm_k, L.k, c.h_kv, L.n, false) ||
        !make_map(&P.tm_v, st->vh, c.h_kv, L.n, true) ||
        !make_map(&P.tm_kc, st->kc, c.h_kv, c.n_max, false) ||
        !make_map(&P.tm_vc, st->vhc, c.h_kv, c.n_max, true) ||
        !make_map(&P.tm_kb, L.k_cmp, c.h_kv, nb_rows, false) ||
        !make_map(&P.tm_vb, st->vh_cmp, c.h_kv, nb_rows, true))
        return cudaErrorInvalidValue;
    auto begin = [&](int stg) {
        if (ev) cudaEventRecord(ev[2 * stg], s);
        ran[stg] = 1;
    };
    auto end = [&](int stg) {
        if (ev) cudaEventRecord(ev[2 * stg + 1], s);
    };
    const int grid = st->num_sms;
    cudaError_t e;
    // compression (vision K/V compaction first, for the later window/selection)
    prepare_kernel<<<st->num_sms * 4, 256, 0, s>>>(L, st->kc, st->vhc, st->vh, st->vh_cmp);
    ++*launches;
    begin(VNSA_STAGE_CMP);
    P.mode = MODE_CMP;
    tc_attn_kernel<<<grid, kThreads, SMEM_BYTES, s>>>(P);
    ++*launches;
    end(VNSA_STAGE_CMP);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // selection
    begin(VNSA_STAGE_TOPK);
    if (!forced) {
        if ((e = launch_topk(L, s)) != cudaSuccess) return e;
        ++*launches;
    }
    {
        const int words = (L.nb_max + 1 + 31) / 32 + 1;
        const int wpb = 4;
        const size_t smem = (size_t)wpb * (2 * words + st->plan_max) * 4;
        if (smem > 48 * 1024) {
            e = cudaFuncSetAttribute(union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem);
            if (e != cudaSuccess) return e;
        }
        union_kernel<<<st->num_sms * 8, wpb * 32, smem, s>>>(L, st->plan, st->plan_max, words);
        ++*launches;
    }
    end(VNSA_STAGE_TOPK);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    begin(VNSA_STAGE_SWA);
    P.mode = MODE_VIS;
    tc_attn_kernel<<<grid, kThreads, SMEM_BYTES, s>>>(P);
    ++*launches;
    end(VNSA_STAGE_SWA);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    begin(VNSA_STAGE_TEXT);
    P.mode = MODE_TEXT;
    tc_attn_kernel<<<grid, kThreads, SMEM_BYTES, s>>>(P);
    ++*launches;
    // grid-stride over (text query, head); the kernel reads N_t on the device
    text_combine_kernel<<<st->num_sms * 4, 256, 0, s>>>(L, st->part, st->part_items);
    ++*launches;
    end(VNSA_STAGE_TEXT);
    return cudaGetLastError();
}

void tc_destroy(TcState *st) { delete st; }

}  // namespace vnsa
