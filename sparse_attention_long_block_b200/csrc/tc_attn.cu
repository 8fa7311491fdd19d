// tc_attn.cu -- tensor-core path of the bf16 layer prefill (head dim 128):
// compression attention + importance, selection, sliding window + gate, and
// dense text GQA, on tcgen05 MMAs with TMEM accumulators fed by TMA.
//
// Method: "VideoNSA: Native Sparse Attention Scales Video Understanding" (paper
// notes), section "Method": vision tokens attend through compression,
// selection and a sliding window mixed by per-head sigmoid gates; text tokens
// attend densely (GQA).
//
// One persistent kernel serves the modes below; two CTAs share each SM so that one
// CTA's softmax overlaps the other's tensor-core work.  A CTA (6 warps) walks
// work items; an item is an M tile of 128 MMA rows, row = (query, head of one
// GQA group): consecutive queries times the group's heads, so every K/V tile
// serves the whole group.  Per item the CTA streams 64-key tiles:
//   warp 0     TMA loads of K (and V) tiles into a 2-stage ring;
//   warp 1     one thread issues S = Q K^T (M 128, N 64, K 128, bf16) into one
//              of two TMEM S buffers, a tile ahead of the softmax, and
//              O += P V (M 128, N 128, K 64, fp16, P read from TMEM);
//   warps 2-5  one thread per row: S row from TMEM, mask, softmax, P (fp16)
//              into the same TMEM buffer, lazy O rescaling, epilogue.
// P V takes fp16 operands: P keeps 11 significant bits (bf16 would keep 8,
// which costs up to ~6e-3 of output error).  V and V_cmp enter as fp16 copies
// divided by a power of two chosen per call from their largest magnitude, so
// no bf16 value overflows fp16; the epilogues multiply that power back.
// Modes:
//   CMP   keys = compressed blocks.  Segment 1: each row's log-sum-exp.
//         Segment 2: exact probabilities, their sum over the group's heads
//         (the block importance, a warp reduce-scatter: rows are 16 queries x
//         8 head slots) and O = P V, already normalised.
//   SLC   the union of the blocks the item's queries selected; a row masks the
//         blocks its query did not select.  Epilogue: the fp32 gated partial
//         (sig(g_cmp) o_cmp so far) gains sig(g_slc) o_slc.  With block 64 the
//         tiles only one of the item's queries reaches are attended by the
//         tile-major pass (sgl_attn.cu) beforehand; the epilogue merges their
//         normalised outputs with the union's softmax by log-sum-exp weights.
//   SWA   the window keys; epilogue: out = partial + sig(g_swa) o_swa, the one
//         rounding of the vision row (to bf16).
//   TEXT  items = (text query tile, key split); partial O, max and sum to a
//         buffer that a small combine kernel reduces (or the row directly).
#include <cuda.h>
#include <math.h>

#include <algorithm>
#include <string.h>

#include "config.h"
#include "sgl_attn.h"
#include "tc_attn.h"
#include "tc_ptx.cuh"

namespace vnsa {

namespace {

constexpr int kThreads = 192;
constexpr int kRows = 128;        // MMA M
constexpr int kKeys = 64;         // keys per tile
constexpr int kD = 128;           // head dim of this path
constexpr int kStages = 2;
constexpr float kRescale = 8.0f;  // lazy rescale threshold (log2 units)
constexpr int kTextSplitKeys = 8192;
constexpr size_t kTextPartBytes = 256ull << 20;
constexpr int kPartStride = kD + 2;  // floats per partial row: O, m, l
constexpr int kSglSlots = 16;        // tile-major pairs per (group, query) at most
constexpr int kSglShare = 3;         // tiles of at most this many queries leave the union

constexpr uint32_t SM_Q = 0;                                  // 2 x [128][64] bf16
constexpr uint32_t SM_KV = 32768;                             // K ring, then V ring
constexpr uint32_t K_BYTES = 16384;                           // one 64-key K or V tile
constexpr uint32_t KV_BYTES = 2 * K_BYTES;
constexpr int kPlanSmem = 1152;                               // selection tiles per item
constexpr int kPrefetch = 4;                                  // tiles prefetched into L2 ahead
constexpr uint32_t SM_PLAN = SM_KV + kStages * KV_BYTES;      // [2][kPlanSmem] int32 (softmax)
constexpr uint32_t SM_BAR = SM_PLAN + 2 * kPlanSmem * 4;      // barriers
constexpr uint32_t SM_TOTAL = SM_BAR + 256;
constexpr uint32_t SMEM_BYTES = SM_TOTAL + 1024;              // + alignment slack

// barrier slots (8 bytes each) after SM_BAR; S_FULL and P_FULL per S buffer
constexpr int B_K_FULL = 0, B_V_FULL = 2, B_K_EMPTY = 4, B_V_EMPTY = 6, B_S_FULL = 8,
              B_P_FULL = 10, B_PV_DONE = 12, B_Q_FULL = 14, B_GRP = 15, B_FINAL = 16,
              B_Q_EMPTY = 17, B_COUNT = 18;

// TMEM columns: two S buffers (fp32, 64 each) and O (fp32, 128).  Tile x uses
// S buffer x & 1; its P (fp16 pairs) overwrites the first 32 columns of that
// buffer once the row is in registers, and Q K^T of tile x + 2 reuses the
// buffer after P V of tile x (MMAs of one thread run in issue order).
constexpr uint32_t TM_S = 0, TM_O = 128, TM_COLS = 256;

// Selection runs over 64-key tiles of vision ranks.  When the block size is a
// multiple of 64 every tile lies inside one block and a query either takes a
// whole tile or none of it (MODE_SLC); otherwise a tile holds parts of several
// blocks and each row's keys are the parts of its own selected blocks
// (MODE_SLC_UNALIGNED).
enum Mode { MODE_CMP = 0, MODE_SLC = 1, MODE_SWA = 2, MODE_TEXT = 3, MODE_SLC_UNALIGNED = 4 };
__host__ __device__ constexpr bool is_slc(int m) {
    return m == MODE_SLC || m == MODE_SLC_UNALIGNED;
}
enum Kind { K_STATS = 0, K_EXACT = 1, K_SLC = 2, K_SWA = 3, K_TEXT = 4 };

struct TcParams {
    CUtensorMap tm_k, tm_v;    // K (bf16, the caller's) and V (scaled fp16 copy): [n rows][h_kv*d]
    CUtensorMap tm_kc, tm_vc;  // compacted vision K (bf16), V (scaled fp16), if not contiguous
    CUtensorMap tm_kb, tm_vb;  // K_cmp (bf16), V_cmp (scaled fp16): [nb_max rows][h_kv*d]
    const float *v_scale;      // [0]: the power of two V was divided by, [1]: V_cmp's
    CUtensorMap tm_q;          // Q (bf16) as [n][h_q][d], box {64, rows per query, queries}
    LayerParams L;
    const int32_t *plan;       // SLC: [item][1 + 2*plan_max]
    int plan_max;
    float *part;               // TEXT partials: [item][128][kPartStride]
    int part_items;
    int mode;
    // Selection tiles that one or two queries of an item reach (block 64
    // only): the union kernel takes them out of the item's plan and records
    // each (query, tile) pair; the tile-major pass (sgl_attn.cu) attends them,
    // and the merge kernel combines each query's pairs with its union part.
    int sgl_on;                // 1: the selection branch runs split this way
    __half *slc_u;             // [n_max][h_q][d] the union tiles' normalised output
    float *slc_lse;            // [n_max][h_q] their log-sum-exp (log2 units)
    // With the split selection the merge kernel writes the output rows; the
    // window epilogue then stores sig(g_swa) o_swa here ([n_max][h_q][d] fp16,
    // in units of V / v_scale like the selection parts) instead of reading the
    // partial (null: the window epilogue writes the rows).
    __half *swa_part;
    int exact_kind;            // K_EXACT (a run-time value, for the exact pass's segment)
};

__host__ __device__ __forceinline__ int pow2_at_least(int r) {
    int p = 1;
    while (p < r) p <<= 1;
    return p;
}

// ---------------------------------------------------------------------------
// Work decomposition shared by every role (all compute the same values).
struct Work {
    int rpad;      // MMA rows per query (>= heads per group)
    int qt;        // queries per item
    int n_q;       // queries of the item kind (N_v or N_t)
    int n_tiles_q; // query tiles per group
    int nsplit;    // text key splits
    int split_len; // keys per split
    int items;
    int nb;
    int contiguous, vis_base;
    int q_tma;     // Q tiles arrive by one TMA box (the item kind's tokens are one run)
    int q_base;    // position of the first token of that run
};

template <int MODE>
__device__ __forceinline__ Work make_work(const TcParams &P, const Counts &cn) {
    Work w;
    const LayerParams &L = P.L;
    w.rpad = MODE == MODE_CMP ? pow2_at_least(L.r) : L.r;
    w.qt = kRows / w.rpad;
    w.nb = MODE == MODE_CMP ? cn.nc : cn.nb;  // compression blocks for CMP
    w.contiguous = cn.contiguous;
    w.vis_base = cn.vis_base;
    w.q_tma = MODE == MODE_TEXT ? cn.txt_contiguous : cn.contiguous;
    w.q_base = MODE == MODE_TEXT ? cn.txt_base : cn.vis_base;
    w.nsplit = 1;
    w.split_len = 0;
    if (MODE == MODE_TEXT) {
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
    int nseg;
    int seg_kind[2];
    int seg_tiles[2];
    int key_lo;     // SWA window start (vision rank) / TEXT split start (position)
};

template <int MODE, int PASS = 0>
__device__ __forceinline__ Item make_item(const TcParams &P, const Work &w, int item) {
    const LayerParams &L = P.L;
    Item it;
    int tile;
    if (MODE == MODE_TEXT) {
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
    it.seg_tiles[1] = 0;
    it.seg_kind[1] = K_EXACT;
    if (MODE == MODE_CMP) {
        // PASS 0: both segments; 1: the statistics pass alone; 2: the exact
        // pass alone (its log-sum-exp from pass 1)
        const int c_last = cmp_visible(ql, L.block, L.stride, w.nb);
        const int t = (c_last + kKeys - 1) / kKeys;
        it.nseg = PASS == 0 ? 2 : 1;
        it.seg_kind[0] = PASS == 2 ? P.exact_kind : K_STATS;
        it.seg_tiles[0] = t;
        it.seg_tiles[1] = PASS == 0 ? t : 0;
    } else if (is_slc(MODE)) {
        it.nseg = 1;
        it.seg_kind[0] = K_SLC;
        it.seg_tiles[0] = P.plan[(size_t)item * (1 + 2 * P.plan_max)];
    } else if (MODE == MODE_SWA) {
        it.nseg = 1;
        it.seg_kind[0] = K_SWA;
        it.key_lo = max(0, it.q0 - L.window + 1);
        it.seg_tiles[0] = (ql - it.key_lo + kKeys) / kKeys;
    } else {
        const int last_pos = L.txt[ql];
        it.nseg = 1;
        it.seg_kind[0] = K_TEXT;
        it.key_lo = it.split * w.split_len;
        const int key_hi = min(it.key_lo + w.split_len, last_pos + 1) - 1;
        it.seg_tiles[0] = key_hi >= it.key_lo ? (key_hi - it.key_lo + kKeys) / kKeys : 0;
    }
    return it;
}

__device__ __forceinline__ int item_tiles(const Item &it) {
    return it.seg_tiles[0] + (it.nseg > 1 ? it.seg_tiles[1] : 0);
}

__device__ __forceinline__ bool kind_has_pv(int kind) { return kind != K_STATS; }


// ---------------------------------------------------------------------------
struct Smem {
    uint8_t *base;
    uint32_t base_u32;
    __device__ uint32_t bar(int i) const { return base_u32 + SM_BAR + 8u * (uint32_t)i; }
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

// First key of tile x: a vision rank (SLC, SWA), a compressed block (STATS,
// EXACT) or a position (TEXT).  SLC reads the item's plan.
__device__ __forceinline__ int tile_key0(const TcParams &P, const Item &it, int item, int kind,
                                         int x) {
    switch (kind) {
        case K_SLC: return P.plan[(size_t)item * (1 + 2 * P.plan_max) + 1 + x] * kKeys;
        case K_SWA:
        case K_TEXT: return it.key_lo + x * kKeys;
        default: return x * kKeys;
    }
}

// ---------------------------------------------------------------------------
// Producer (warp 0): TMA loads of the K tiles (lane 0) and V tiles (lane 1) of
// every item, in order, each lane with its own ring and waits: a K stage is
// free once its Q K^T is done, a V stage only after its P V, so the K loads
// run ahead.  Lane 0 also prefetches the tiles kPrefetch ahead into L2.
template <int MODE, int PASS = 0>
__device__ void run_producer(const TcParams &P, const Work &w, const Smem &sm, int lane) {
    if (lane > 1) return;
    const LayerParams &L = P.L;
    volatile int *abort = sm.abort_flag();
    const bool is_k = lane == 0;
    const int ring_full = is_k ? B_K_FULL : B_V_FULL;
    const int ring_empty = is_k ? B_K_EMPTY : B_V_EMPTY;
    const uint32_t ring_base = sm.base_u32 + SM_KV + (is_k ? 0u : kStages * K_BYTES);
    uint32_t t = 0;  // tiles issued on this lane's ring
    const CUtensorMap *mk = &P.tm_k, *mv = &P.tm_v;
    int vbase = 0;
    if (MODE == MODE_CMP) {
        mk = &P.tm_kb;
        mv = &P.tm_vb;
    } else if (is_slc(MODE) || MODE == MODE_SWA) {
        mk = w.contiguous ? &P.tm_k : &P.tm_kc;
        mv = w.contiguous ? &P.tm_v : &P.tm_vc;
        vbase = w.contiguous ? w.vis_base : 0;
    }
    const CUtensorMap *mine = is_k ? mk : mv;
    uint32_t nq = 0;  // Q tiles loaded (lane 0, TMA path)
    const int qrows = MODE == MODE_CMP ? w.rpad : L.r;  // MMA rows per query
    for (int item = blockIdx.x; item < w.items; item += gridDim.x) {
        const Item it = make_item<MODE, PASS>(P, w, item);
        const int xc = it.g * kD;
        if (is_k && w.q_tma && item_tiles(it) > 0) {
            // the item's Q rows (query, head) are one box of the [n][h_q][d]
            // tensor: queries vis_base + q0 .., heads g r .., in MMA row order;
            // the buffer is free once the previous item's Q K^T are done
            if (nq > 0 && !ptx::mbar_wait(sm.bar(B_Q_EMPTY), (nq - 1) & 1, abort, L.status, L.wait_ns))
                goto drain;
            const uint32_t qb = sm.bar(B_Q_FULL);
            ptx::mbar_expect_tx(qb, (uint32_t)(w.qt * qrows) * 2u * kD);
            ptx::tma_load_3d(sm.base_u32 + SM_Q, &P.tm_q, qb, 0, it.g * L.r, w.q_base + it.q0);
            ptx::tma_load_3d(sm.base_u32 + SM_Q + 16384, &P.tm_q, qb, 64, it.g * L.r,
                             w.q_base + it.q0);
            ++nq;
        }
        // row coordinate of tile x of a segment (both CMP segments share keys)
        auto row_of = [&](int kind, int x) {
            const int key0 = tile_key0(P, it, item, kind, x);
            return (kind == K_SLC || kind == K_SWA) ? vbase + key0 : key0;
        };
        if (is_k) {
            const int pf0 = min(kPrefetch, it.seg_tiles[0]);
            for (int x = 0; x < pf0; ++x) {
                const int y = row_of(it.seg_kind[0], x);
                ptx::tma_prefetch_2d(mk, xc, y);
                ptx::tma_prefetch_2d(mk, xc + 64, y);
                ptx::tma_prefetch_2d(mv, xc, y);
                ptx::tma_prefetch_2d(mv, xc + 64, y);
            }
        }
        for (int s = 0; s < it.nseg; ++s) {
            const int kind = it.seg_kind[s];
            if (!is_k && !kind_has_pv(kind)) continue;
            int y_next = it.seg_tiles[s] > 0 ? row_of(kind, 0) : 0;
            for (int x = 0; x < it.seg_tiles[s]; ++x, ++t) {
                const int y = y_next;
                if (x + 1 < it.seg_tiles[s]) y_next = row_of(kind, x + 1);
                const uint32_t st = t % kStages;
                if (t >= (uint32_t)kStages &&
                    !ptx::mbar_wait(sm.bar(ring_empty + st), ((t / kStages) - 1) & 1, abort,
                                    L.status, L.wait_ns))
                    goto drain;
                const uint32_t dst = ring_base + st * K_BYTES;
                ptx::mbar_expect_tx(sm.bar(ring_full + st), K_BYTES);
                ptx::tma_load_2d(dst, mine, sm.bar(ring_full + st), xc, y);
                ptx::tma_load_2d(dst + 8192, mine, sm.bar(ring_full + st), xc + 64, y);
                if (is_k && s == 0 && x + kPrefetch < it.seg_tiles[0]) {
                    const int yp = row_of(kind, x + kPrefetch);
                    ptx::tma_prefetch_2d(mk, xc, yp);
                    ptx::tma_prefetch_2d(mk, xc + 64, yp);
                    ptx::tma_prefetch_2d(mv, xc, yp);
                    ptx::tma_prefetch_2d(mv, xc + 64, yp);
                }
            }
        }
    }
    // no load may still be landing in shared memory when the CTA ends (also
    // after an abort: these waits do not give up on the abort flag)
drain:
    for (uint32_t back = 1; back <= (uint32_t)kStages && back <= t; ++back) {
        const uint32_t u = t - back;
        if (!ptx::mbar_drain(sm.bar(ring_full + u % kStages), (u / kStages) & 1)) return;
    }
    if (is_k && nq > 0) ptx::mbar_drain(sm.bar(B_Q_FULL), (nq - 1) & 1);
}

// ---------------------------------------------------------------------------
// MMA issuer (one thread).
template <int MODE, int PASS = 0>
__device__ void run_mma(const TcParams &P, const Work &w, const Smem &sm, uint32_t tmem) {
    const LayerParams &L = P.L;
    volatile int *abort = sm.abort_flag();
    // S = Q K^T: bf16 operands, both K-major.  O += P V: fp16 operands, P from
    // TMEM, V as an MN-major shared-memory operand.
    constexpr uint32_t idesc_s = ptx::idesc_f16kind(kRows, kKeys, 0, 0, 1u);
    constexpr uint32_t idesc_pv = ptx::idesc_f16kind(kRows, kD, 0, 1, 0u);
    const uint32_t q_addr = sm.base_u32 + SM_Q;
    uint32_t gt = 0, nitems = 0, npv = 0;  // npv: P V products = V tiles consumed
    bool ok = true;
    // Tile `pg` (global count) is finished once its softmax is done with the S
    // buffer: wait for that, then issue its P V if the tile has one.
    auto finish = [&](uint32_t pg, bool has_pv, uint32_t acc) -> bool {
        if (!ptx::mbar_wait(sm.bar(B_P_FULL + (pg & 1)), (pg >> 1) & 1, abort, L.status, L.wait_ns))
            return false;
        if (!has_pv) return true;
        const uint32_t sv = npv % kStages;
        if (!ptx::mbar_wait(sm.bar(B_V_FULL + sv), (npv / kStages) & 1, abort, L.status, L.wait_ns))
            return false;
        ptx::tc_fence_after();
        const uint32_t vb = sm.base_u32 + SM_KV + kStages * K_BYTES + sv * K_BYTES;
        const uint32_t pa = tmem + TM_S + (pg & 1) * 64;
#pragma unroll
        for (int k = 0; k < kKeys / 16; ++k)
            ptx::mma_ts(tmem + TM_O, pa + (uint32_t)k * 8u, desc_vmajor(vb + (uint32_t)k * 2048u),
                        idesc_pv, (k > 0 || acc) ? 1u : 0u);
        ptx::mma_commit(sm.bar(B_PV_DONE + (npv & 1)));
        ptx::mma_commit(sm.bar(B_V_EMPTY + sv));
        ++npv;
        return true;
    };
    for (int item = blockIdx.x; ok && item < w.items; item += gridDim.x) {
        const Item it = make_item<MODE, PASS>(P, w, item);
        if (item_tiles(it) == 0) continue;
        if (!ptx::mbar_wait(sm.bar(B_Q_FULL), nitems & 1, abort, L.status, L.wait_ns)) { ok = false; break; }
        ++nitems;
        ptx::tc_fence_after();
        bool pending = false, pend_pv = false;
        uint32_t pend_acc = 0;
        int uq = 0;  // Q K^T issued for this item
        for (int s = 0; ok && s < it.nseg; ++s) {
            const int kind = it.seg_kind[s];
            for (int x = 0; x < it.seg_tiles[s]; ++x, ++gt) {
                const uint32_t st = gt % kStages;
                if (!ptx::mbar_wait(sm.bar(B_K_FULL + st), (gt / kStages) & 1, abort, L.status, L.wait_ns)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t kb = sm.base_u32 + SM_KV + st * K_BYTES;
                const uint32_t sd = tmem + TM_S + (gt & 1) * 64;
#pragma unroll
                for (int k = 0; k < kD / 16; ++k) {
                    const uint32_t off = (uint32_t)(k >> 2) * 16384u + (uint32_t)(k & 3) * 32u;
                    const uint32_t koff = (uint32_t)(k >> 2) * 8192u + (uint32_t)(k & 3) * 32u;
                    ptx::mma_ss(sd, desc_kmajor(q_addr + off), desc_kmajor(kb + koff), idesc_s,
                                k > 0 ? 1u : 0u);
                }
                ptx::mma_commit(sm.bar(B_S_FULL + (gt & 1)));
                ptx::mma_commit(sm.bar(B_K_EMPTY + st));  // K is dead once Q K^T is done
                // after the item's last Q K^T the Q buffer is free for the next item
                if (w.q_tma && ++uq == item_tiles(it)) ptx::mma_commit(sm.bar(B_Q_EMPTY));
                // the previous tile: its P V follows this Q K^T in the pipe, and
                // its S buffer is free for the next Q K^T after that
                if (pending && !finish(gt - 1, pend_pv, pend_acc)) { ok = false; break; }
                pending = true;
                pend_pv = kind_has_pv(kind);
                pend_acc = x > 0 ? 1u : 0u;
            }
        }
        if (ok && pending && !finish(gt - 1, pend_pv, pend_acc)) ok = false;
    }
    // every MMA this thread issued has completed once this barrier flips (also
    // after an abort, before the CTA frees its TMEM)
    ptx::mma_commit(sm.bar(B_FINAL));
    ptx::mbar_drain(sm.bar(B_FINAL), 0);
}

// ---------------------------------------------------------------------------
// Softmax / epilogue warps 2-5: thread rho owns MMA row rho = TMEM lane rho.
struct RowCtx {
    bool valid;
    int qi, hl, h;
    int i;      // vision rank (CMP/SLC/SWA) or text rank (TEXT)
    int t;      // position of the query token
    int c_vis;  // visible compressed blocks
};

__device__ __forceinline__ void group_sync(const Smem &sm, uint32_t &phase, bool &ok,
                                           const LayerParams &L) {
    ptx::mbar_arrive(sm.bar(B_GRP));
    bool r = ptx::mbar_wait(sm.bar(B_GRP), phase & 1, sm.abort_flag(), L.status, L.wait_ns);
    ++phase;
    ok = __all_sync(0xffffffffu, r && ok);
}

// Block importance of one S tile: the sum over the RPAD rows (head slots) of a
// query of its 64 probabilities, as a reduce-scatter across the RPAD lanes
// that hold the query's rows: each lane ends with 64/RPAD consecutive column
// sums starting at column `first`.
template <int RPAD>
__device__ __forceinline__ void imp_reduce_store(float (&p)[64], int lane, float *irow, int lim) {
    int first = 0;
#pragma unroll
    for (int sh = RPAD / 2, width = 32; sh >= 1; sh >>= 1, width >>= 1) {
        const bool upper = (lane & sh) != 0;
#pragma unroll
        for (int c = 0; c < width; ++c) {
            const float mine = upper ? p[width + c] : p[c];
            const float other = upper ? p[c] : p[width + c];
            p[c] = mine + __shfl_xor_sync(0xffffffffu, other, sh);
        }
        if (upper) first += width;
    }
    // columns [first, first + 64/RPAD) of the tile, valid below lim
    constexpr int kCnt = 64 / RPAD;
    if (irow == nullptr) return;
    if (first + kCnt <= lim && (kCnt & 3) == 0) {
#pragma unroll
        for (int z = 0; z < kCnt; z += 4)
            *reinterpret_cast<float4 *>(irow + first + z) =
                make_float4(p[z], p[z + 1], p[z + 2], p[z + 3]);
    } else {
#pragma unroll
        for (int z = 0; z < kCnt; ++z)
            if (first + z < lim) irow[first + z] = p[z];
    }
}

// Valid columns of the 64-key tile at vision rank key0 for a query of vision
// rank i whose selected blocks (block size B) are sel[0..k), ascending with -1
// after the last: the parts of those blocks inside the tile, at or before i.
// Tiles come in ascending order, so blocks that end before this tile are
// skipped for good (cur).
__device__ __forceinline__ uint64_t sel_coverage(const int32_t *sel, int &cur, int k, int B,
                                                 int key0, int i) {
    while (cur < k) {
        const int j = sel[cur];
        if (j < 0 || (j + 1) * B > key0) break;
        ++cur;
    }
    uint64_t cov = 0ull;
    for (int e = cur; e < k; ++e) {
        const int j = sel[e];
        if (j < 0 || j * B >= key0 + kKeys) break;
        const int a = max(j * B - key0, 0), b = min((j + 1) * B - key0, kKeys);
        cov |= (b >= 64 ? ~0ull : ((1ull << b) - 1ull)) & (~0ull << a);
    }
    const int hi = i - key0;  // causal: keys at or before the query
    if (hi < 63) cov &= hi < 0 ? 0ull : ((2ull << hi) - 1ull);
    return cov;
}

// RPAD: the compression mode's head slots per query (4, 8 or 16), fixed per
// instantiation so that each compression kernel carries one importance reduce
template <int MODE, int RPAD, int PASS = 0>
__device__ void run_softmax(const TcParams &P, const Work &w, const Smem &sm, uint32_t tmem) {
    const LayerParams &L = P.L;
    volatile int *abort = sm.abort_flag();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wq = warp & 3;                     // TMEM lane quadrant of this warp
    const int rho = wq * 32 + lane;              // MMA row / TMEM lane
    const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
    const float sc = L.scale_log2;
    const __nv_bfloat16 *Q = (const __nv_bfloat16 *)L.q;
    const int32_t *plan_s = (const int32_t *)(sm.base + SM_PLAN);
    uint32_t gt = 0, npv = 0, gphase = 0;
    bool ok = true;
    for (int item = blockIdx.x; ok && item < w.items; item += gridDim.x) {
        const Item it = make_item<MODE, PASS>(P, w, item);
        RowCtx rc;
        rc.qi = rho / w.rpad;
        rc.hl = rho % w.rpad;
        rc.h = it.g * L.r + min(rc.hl, L.r - 1);
        rc.valid = rc.qi < it.nq && rc.hl < L.r;
        rc.i = it.q0 + min(rc.qi, max(it.nq - 1, 0));
        if (MODE == MODE_TEXT) {
            rc.t = it.nq > 0 ? L.txt[rc.i] : 0;
        } else {
            rc.t = it.nq > 0 ? L.vis[rc.i] : 0;
        }
        rc.c_vis = cmp_visible(rc.i, L.block, L.stride, w.nb);
        if (item_tiles(it) == 0) {
            // nothing attended: empty branch outputs (the exact pass writes
            // those of the compression branch)
            if (rc.valid && !(MODE == MODE_CMP && PASS == 1)) {
                float *part = L.o_cmp_ws + ((size_t)rc.i * L.h_q + rc.h) * kD;
                const size_t prow = ((size_t)rc.t * L.h_q + rc.h) * kD;
                if (MODE == MODE_CMP) {
                    for (int e = 0; e < kD; e += 4)
                        *reinterpret_cast<float4 *>(part + e) = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (L.dbg_o_cmp)
                        for (int e = 0; e < kD; ++e) L.dbg_o_cmp[prow + e] = 0.f;
                    L.lse[(size_t)rc.i * L.h_q + rc.h] = -INFINITY;
                } else if (MODE == MODE_TEXT) {
                    float *pr = P.part + ((size_t)item * kRows + rho) * kPartStride;
                    pr[kD] = -INFINITY;
                    pr[kD + 1] = 0.f;
                } else if (MODE == MODE_SLC && P.sgl_on) {
                    // no union tile (nor pair: the union keeps at least one
                    // tile of an item that has any)
                    for (int e = 0; e < kD; e += 8)
                        *reinterpret_cast<uint4 *>(P.slc_u + ((size_t)rc.i * L.h_q + rc.h) * kD +
                                                   e) = make_uint4(0u, 0u, 0u, 0u);
                    P.slc_lse[(size_t)rc.i * L.h_q + rc.h] = -INFINITY;
                } else {
                    // no selected / window key: this branch adds nothing
                    float *dbg = is_slc(MODE) ? L.dbg_o_slc : L.dbg_o_swa;
                    for (int e = 0; e < kD; ++e) {
                        if (dbg) dbg[prow + e] = 0.f;
                        if (MODE == MODE_SWA && P.swa_part)
                            P.swa_part[((size_t)rc.i * L.h_q + rc.h) * kD + e] = __float2half_rn(0.f);
                        else if (MODE == MODE_SWA)
                            ((__nv_bfloat16 *)L.out)[prow + e] = __float2bfloat16_rn(part[e]);
                    }
                }
            }
            continue;
        }
        // ---- Q tile (without the TMA box): rows gathered from their
        // positions, 16-byte pieces
        for (int e = rho; !w.q_tma && e < kRows * 16; e += 128) {
            const int row = e >> 4, c16 = e & 15;
            const int qi = row / w.rpad, hl = row % w.rpad;
            uint4 val = make_uint4(0u, 0u, 0u, 0u);
            if (qi < it.nq && hl < L.r) {
                const int q = it.q0 + qi;
                const int t = (MODE == MODE_TEXT) ? L.txt[q] : L.vis[q];
                const __nv_bfloat16 *src =
                    Q + ((size_t)t * L.h_q + it.g * L.r + hl) * kD + c16 * 8;
                val = __ldg(reinterpret_cast<const uint4 *>(src));
            }
            const int hf = c16 >> 3, c = c16 & 7;
            *reinterpret_cast<uint4 *>(sm.base + SM_Q + hf * 16384 + row * 128 +
                                       ((c ^ (row & 7)) << 4)) = val;
        }
        if (!w.q_tma) {
            ptx::fence_proxy_async();
            ptx::mbar_arrive(sm.bar(B_Q_FULL));
        }
        // L2 prefetch of this row's epilogue inputs and of its Q row in the
        // next item, so that neither waits on DRAM when it is needed
        if (rc.valid) {
            ptx::prefetch_l2(L.gate + ((size_t)rc.t * L.h_q + rc.h) * 3);
            // the partial, where the epilogue reads it (not with the split
            // selection, whose merge kernel adds the parts)
            if ((is_slc(MODE) && !P.sgl_on) || (MODE == MODE_SWA && !P.swa_part)) {
                const float *part = L.o_cmp_ws + ((size_t)rc.i * L.h_q + rc.h) * kD;
#pragma unroll
                for (int z = 0; z < kD; z += 32) ptx::prefetch_l2(part + z);
            }
        }
        if (item + (int)gridDim.x < w.items) {
            const Item nx = make_item<MODE, PASS>(P, w, item + gridDim.x);
            const int qn = rho / w.rpad, hn = rho % w.rpad;
            if (qn < nx.nq && hn < L.r) {
                const int tn = (MODE == MODE_TEXT) ? L.txt[nx.q0 + qn] : L.vis[nx.q0 + qn];
                const __nv_bfloat16 *qr = Q + ((size_t)tn * L.h_q + nx.g * L.r + hn) * kD;
                ptx::prefetch_l2(qr);
                ptx::prefetch_l2(qr + 64);
            }
        }
        // SLC: the item's selection tiles (first key, and the query mask or,
        // for blocks not aligned to tiles, every query's selected blocks) into
        // shared memory, once every thread is done with the previous item's copy
        if (is_slc(MODE)) {
            group_sync(sm, gphase, ok, L);
            if (!ok) break;
            int32_t *dst = (int32_t *)(sm.base + SM_PLAN);
            const int32_t *src = P.plan + (size_t)item * (1 + 2 * P.plan_max);
            for (int x = rho; x < it.seg_tiles[0]; x += 128) {
                dst[x] = src[1 + x] * kKeys;
                if (MODE == MODE_SLC) dst[kPlanSmem + x] = src[1 + P.plan_max + x];
            }
            if (MODE == MODE_SLC_UNALIGNED) {
                for (int x = rho; x < w.qt * L.top_k; x += 128) {
                    const int qi = x / L.top_k;
                    dst[kPlanSmem + x] =
                        qi < it.nq ? L.idx_src[((size_t)it.g * L.idx_rows + it.q0 + qi) * L.top_k +
                                               x % L.top_k]
                                   : -1;
                }
            }
            group_sync(sm, gphase, ok, L);
            if (!ok) break;
        }
        // MODE_SLC_UNALIGNED: this row's selected blocks (ascending, -1 after
        // the last) and the first of them that can still reach a later tile
        const int32_t *my_sel = plan_s + kPlanSmem + min(rc.qi, w.qt - 1) * L.top_k;
        int sel_cur = 0;

        // CMP: from the statistics segment (pass 2: from pass 1, log2 units)
        float lse2 = (MODE == MODE_CMP && PASS == 2 && rc.valid)
                         ? L.lse[(size_t)rc.i * L.h_q + rc.h]
                         : -INFINITY;
        float m_run = -INFINITY, l_run = 0.f;   // running max / sum (log2 units)
        for (int s = 0; ok && s < it.nseg; ++s) {
            const int kind = it.seg_kind[s];
            m_run = -INFINITY;
            l_run = 0.f;
            // selection tiles: the plan entry of the next tile is read from
            // shared memory one tile ahead, off the tile's critical path
            int nkey0 = 0;
            uint32_t nmask = 0u;
            if (kind == K_SLC && it.seg_tiles[s] > 0) {
                nkey0 = plan_s[0];
                if (MODE == MODE_SLC) nmask = (uint32_t)plan_s[kPlanSmem];
            }
            for (int x = 0; x < it.seg_tiles[s]; ++x, ++gt) {
                const int key0 = kind == K_SLC ? nkey0 : tile_key0(P, it, item, kind, x);
                const uint32_t qmask = nmask;
                // column range [lo, hi] of valid keys for this row, or (blocks
                // not aligned to tiles) the bit set `cov` of its valid columns
                int lo = 1, hi = 0;
                uint64_t cov = 0ull;
                if (MODE == MODE_SLC_UNALIGNED) {
                    if (rc.valid) cov = sel_coverage(my_sel, sel_cur, L.top_k, L.block, key0, rc.i);
                } else if (rc.valid) {
                    switch (kind) {
                        case K_STATS:
                        case K_EXACT: lo = 0; hi = rc.c_vis - 1 - key0; break;
                        case K_SLC:
                            if ((qmask >> rc.qi) & 1u) {
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
                const bool row_in = MODE == MODE_SLC_UNALIGNED ? cov != 0ull : lo <= hi;
                const bool row_full =
                    MODE == MODE_SLC_UNALIGNED ? cov == ~0ull : (lo == 0 && hi == kKeys - 1);
                // every row of the warp either takes the whole tile or none of
                // it (selection tiles off the diagonal, interior window and
                // text tiles): rows are masked by their exponent bias alone
                const bool rowwise = __all_sync(0xffffffffu, row_full || !row_in);
                // every row of this warp masked (common in selection tiles:
                // most queries did not pick a given block): P = 0, no S read
                const bool none = __all_sync(0xffffffffu, !row_in);
                // a masked row in a row-wise tile: 2^(s * 0 - inf) = 0 for its
                // whole row (scores of finite inputs are finite)
                const bool kill = rowwise && !row_in;
                const uint32_t sbuf = gt & 1;
                const uint32_t s_col = tmem + lane_base + TM_S + sbuf * 64;
                bool r = ptx::mbar_wait(sm.bar(B_S_FULL + sbuf), (gt >> 1) & 1, abort, L.status, L.wait_ns);
                ok = __all_sync(0xffffffffu, r && ok);
                if (!ok) break;
                ptx::tc_fence_after();
                if (kind == K_SLC && x + 1 < it.seg_tiles[s]) {
                    nkey0 = plan_s[x + 1];
                    if (MODE == MODE_SLC) nmask = (uint32_t)plan_s[kPlanSmem + x + 1];
                }
                float sv[64];
                bool need = false;
                float factor = 1.f;
                if (none) {
                    if (kind == K_STATS) {
                        ptx::tc_fence_before();
                        __syncwarp();
                        if (lane == 0) ptx::mbar_arrive(sm.bar(B_P_FULL + sbuf));
                        continue;
                    }
#pragma unroll
                    for (int k = 0; k < 64; ++k) sv[k] = 0.f;
                } else {
                {
                    float a[32], c[32];
                    ptx::tmem_ld32(s_col, a);
                    ptx::tmem_ld32(s_col + 32, c);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 32; ++k) { sv[k] = a[k]; sv[32 + k] = c[k]; }
                }
                if (kind == K_STATS) {
                    // no P: the S buffer is free as soon as the row is read
                    ptx::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(sm.bar(B_P_FULL + sbuf));
                }
                // mask on the raw scores (scale > 0 keeps the order)
                if (!rowwise) {
                    if (MODE == MODE_SLC_UNALIGNED) {
                        const uint32_t c0 = (uint32_t)cov, c1 = (uint32_t)(cov >> 32);
#pragma unroll
                        for (int k = 0; k < 32; ++k) {
                            sv[k] = ((c0 >> k) & 1u) ? sv[k] : -INFINITY;
                            sv[32 + k] = ((c1 >> k) & 1u) ? sv[32 + k] : -INFINITY;
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < 64; ++k) sv[k] = (k >= lo && k <= hi) ? sv[k] : -INFINITY;
                    }
                }
                float mx;  // row max of this tile, in log2 units
                {
                    float m8[8];
#pragma unroll
                    for (int z = 0; z < 8; ++z) {
                        m8[z] = ptx::fmax3(sv[z], sv[8 + z], sv[16 + z]);        // 0..23
                        m8[z] = ptx::fmax3(m8[z], sv[24 + z], sv[32 + z]);       // 24..39
                        m8[z] = ptx::fmax3(m8[z], sv[40 + z], sv[48 + z]);       // 40..55
                        m8[z] = fmaxf(m8[z], sv[56 + z]);                        // 56..63
                    }
                    mx = ptx::fmax3(ptx::fmax3(m8[0], m8[1], m8[2]), ptx::fmax3(m8[3], m8[4], m8[5]),
                                    fmaxf(m8[6], m8[7])) * sc;
                    if (kill) mx = -INFINITY;
                }
                // sv[k] <- 2^(sv[k] * sc - sub) in place, returning the sum
                auto exp_sum = [&](float sub) {
                    const float s_r = kill ? 0.f : sc;
                    const float b_r = kill ? -INFINITY : -sub;
                    float a0 = 0.f, a1 = 0.f, b0 = 0.f, b1 = 0.f;
#pragma unroll
                    for (int k = 0; k < 64; k += 4) {
                        ptx::ffma2(sv[k], sv[k + 1], sv[k], sv[k + 1], s_r, s_r, b_r, b_r);
                        ptx::ffma2(sv[k + 2], sv[k + 3], sv[k + 2], sv[k + 3], s_r, s_r, b_r, b_r);
                        sv[k] = ptx::ex2(sv[k]);
                        sv[k + 1] = ptx::ex2(sv[k + 1]);
                        sv[k + 2] = ptx::ex2(sv[k + 2]);
                        sv[k + 3] = ptx::ex2(sv[k + 3]);
                        ptx::fadd2(a0, a1, a0, a1, sv[k], sv[k + 1]);
                        ptx::fadd2(b0, b1, b0, b1, sv[k + 2], sv[k + 3]);
                    }
                    return (a0 + a1) + (b0 + b1);
                };
                if (kind == K_STATS) {
                    const float mn = fmaxf(m_run, mx);
                    const float mu = mn == -INFINITY ? 0.f : mn;
                    const float acc = exp_sum(mu);
                    l_run = l_run * ptx::ex2(m_run - mu) + acc;
                    m_run = mn;
                    continue;
                }
                if (kind == K_EXACT) {
                    if (lse2 != -INFINITY) {
                        exp_sum(lse2);
                    } else {
#pragma unroll
                        for (int k = 0; k < 64; ++k) sv[k] = 0.f;
                    }
                } else {
                    // online softmax with lazy rescaling of O
                    const float mn = fmaxf(m_run, mx);
                    if (mn > m_run + kRescale) {
                        // a row with no key so far has O = 0 and l = 0 (all its
                        // earlier P were 0): only a finite running max rescales
                        if (m_run != -INFINITY) {
                            need = true;
                            factor = ptx::ex2(m_run - mn);
                            l_run *= factor;
                        }
                        m_run = mn;
                    }
                    l_run += exp_sum(m_run == -INFINITY ? 0.f : m_run);
                }
                }  // !none
                if (__any_sync(0xffffffffu, need && x > 0)) {
                    // O may only be rescaled once every earlier P V has landed
                    if (npv > 0) {
                        bool r2 = ptx::mbar_wait(sm.bar(B_PV_DONE + ((npv - 1) & 1)),
                                                 ((npv - 1) >> 1) & 1, abort, L.status, L.wait_ns);
                        ok = __all_sync(0xffffffffu, r2 && ok);
                        if (!ok) break;
                    }
                    ptx::tc_fence_after();
                    const float f = (need && x > 0) ? factor : 1.f;
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        float o[32];
                        ptx::tmem_ld32(tmem + lane_base + TM_O + ch * 32, o);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 32; ++k) o[k] *= f;
                        ptx::tmem_st32(tmem + lane_base + TM_O + ch * 32, o);
                    }
                }
                {
                    uint32_t pk[32];
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        __half2 h2 = __floats2half2_rn(sv[2 * k], sv[2 * k + 1]);
                        pk[k] = *reinterpret_cast<uint32_t *>(&h2);
                    }
                    ptx::tmem_st32u(s_col, pk);
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(sm.bar(B_P_FULL + sbuf));  // one per warp
                ++npv;
                if (kind == K_EXACT && !none) {
                    // block importance: the sum of the probabilities over the
                    // query's head slots (P is already handed to the MMA)
                    const int iq = it.q0 + rc.qi;
                    const int cq = cmp_visible(iq, L.block, L.stride, w.nb);
                    float *irow = rc.qi < it.nq
                                      ? L.imp + ((size_t)it.g * L.n_max + iq) * L.imp_stride + key0
                                      : nullptr;
                    const int lim = cq - key0;  // valid columns of this tile for the query
                    imp_reduce_store<RPAD>(sv, lane, irow, lim);
                }
            }
            if (!ok) break;
            if (kind == K_STATS)
                lse2 = (m_run == -INFINITY || l_run <= 0.f) ? -INFINITY : m_run + log2f(l_run);
        }
        if (!ok) break;
        if (MODE == MODE_CMP && PASS == 1) {
            // the statistics pass hands the exact pass its log-sum-exp (log2
            // units; the exact pass's epilogue stores it in natural units)
            if (rc.valid) L.lse[(size_t)rc.i * L.h_q + rc.h] = lse2;
            continue;
        }
        // ---- epilogue: wait for the item's last P V (#npv-1)
        {
            bool r = ptx::mbar_wait(sm.bar(B_PV_DONE + ((npv - 1) & 1)), ((npv - 1) >> 1) & 1,
                                    abort, L.status, L.wait_ns);
            ok = __all_sync(0xffffffffu, r && ok);
            if (!ok) break;
            ptx::tc_fence_after();
        }
        const size_t qrow = ((size_t)rc.i * L.h_q + rc.h) * kD;   // by vision rank
        const size_t prow = ((size_t)rc.t * L.h_q + rc.h) * kD;   // by position
        // The gated vision partial lives in the workspace as fp32 [N_v][h_q][d]:
        // CMP writes sig(g_cmp) o_cmp, SLC adds sig(g_slc) o_slc in place, SWA
        // adds sig(g_swa) o_swa and rounds the sum once, to the bf16 output row.
        float *part = L.o_cmp_ws + qrow;
        // O was accumulated against V (or V_cmp) divided by this power of two
        const float vsc = P.v_scale[MODE == MODE_CMP ? 1 : 0];
        if (MODE == MODE_CMP) {
            const float gc = rc.valid ? sigmoidf_(L.gate[((size_t)rc.t * L.h_q + rc.h) * 3]) : 0.f;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float o[32];
                ptx::tmem_ld32(tmem + lane_base + TM_O + ch * 32, o);
                ptx::tmem_wait_ld();
                if (rc.valid) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) o[k] *= vsc;
#pragma unroll
                    for (int k = 0; k < 32; k += 4)
                        __stcg(reinterpret_cast<float4 *>(part + ch * 32 + k),
                               make_float4(gc * o[k], gc * o[k + 1], gc * o[k + 2], gc * o[k + 3]));
                    if (L.dbg_o_cmp)
                        for (int k = 0; k < 32; ++k) L.dbg_o_cmp[prow + ch * 32 + k] = o[k];
                }
            }
            if (rc.valid) L.lse[(size_t)rc.i * L.h_q + rc.h] = lse2 * kLn2;
        } else if (MODE == MODE_SLC && P.sgl_on) {
            // The selection softmax of this row is split into the union's tiles
            // and the query's (query, tile) pairs (the tile-major pass); the
            // merge kernel combines them.  Here: the union part, normalised, in
            // the units of the scaled V copy (fp16: a convex combination of
            // values below 2^15), and its log-sum-exp (log2 units).
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            __half *orow = P.slc_u + qrow;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float o[32];
                ptx::tmem_ld32(tmem + lane_base + TM_O + ch * 32, o);
                ptx::tmem_wait_ld();
                if (!rc.valid) continue;
#pragma unroll
                for (int k = 0; k < 32; k += 8) {
                    uint4 v;
                    __half2 *h2 = reinterpret_cast<__half2 *>(&v);
#pragma unroll
                    for (int z = 0; z < 4; ++z)
                        h2[z] = __floats2half2_rn(o[k + 2 * z] * inv, o[k + 2 * z + 1] * inv);
                    __stcg(reinterpret_cast<uint4 *>(orow + ch * 32 + k), v);
                }
            }
            if (rc.valid)
                P.slc_lse[(size_t)rc.i * L.h_q + rc.h] = l_run > 0.f ? m_run + log2f(l_run) : -INFINITY;
        } else if (is_slc(MODE) || MODE == MODE_SWA) {
            const float g =
                rc.valid ? sigmoidf_(L.gate[((size_t)rc.t * L.h_q + rc.h) * 3 + (is_slc(MODE) ? 1 : 2)])
                         : 0.f;
            const float inv = l_run > 0.f ? vsc / l_run : 0.f;
            float *dbg = is_slc(MODE) ? L.dbg_o_slc : L.dbg_o_swa;
            __nv_bfloat16 *orow = (__nv_bfloat16 *)L.out + prow;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float o[32];
                ptx::tmem_ld32(tmem + lane_base + TM_O + ch * 32, o);
                ptx::tmem_wait_ld();
                if (!rc.valid) continue;
                if (MODE == MODE_SWA && P.swa_part) {
                    // the merge kernel adds this to the partial and the
                    // selection and writes the row: store sig(g_swa) o_swa in
                    // units of V / v_scale (|value| < 2^15, inside fp16)
                    const float inv_u = l_run > 0.f ? 1.f / l_run : 0.f;
                    __half *dst = P.swa_part + qrow + ch * 32;
#pragma unroll
                    for (int k = 0; k < 32; k += 8) {
                        uint4 v;
                        __half2 *h2 = reinterpret_cast<__half2 *>(&v);
#pragma unroll
                        for (int z = 0; z < 4; ++z)
                            h2[z] = __floats2half2_rn(g * (o[k + 2 * z] * inv_u),
                                                      g * (o[k + 2 * z + 1] * inv_u));
                        __stcg(reinterpret_cast<uint4 *>(dst + k), v);
                        if (dbg)
                            for (int z = 0; z < 8; ++z)
                                dbg[prow + ch * 32 + k + z] = l_run > 0.f ? o[k + z] * inv : 0.f;
                    }
                    continue;
                }
#pragma unroll
                for (int k = 0; k < 32; k += 8) {
                    const float4 p0 = __ldcg(reinterpret_cast<const float4 *>(part + ch * 32 + k));
                    const float4 p1 = __ldcg(reinterpret_cast<const float4 *>(part + ch * 32 + k + 4));
                    float b8[8];
#pragma unroll
                    for (int z = 0; z < 8; ++z) b8[z] = l_run > 0.f ? o[k + z] * inv : 0.f;
                    if (dbg)
                        for (int z = 0; z < 8; ++z) dbg[prow + ch * 32 + k + z] = b8[z];
                    const float f8[8] = {p0.x + g * b8[0], p0.y + g * b8[1], p0.z + g * b8[2],
                                         p0.w + g * b8[3], p1.x + g * b8[4], p1.y + g * b8[5],
                                         p1.z + g * b8[6], p1.w + g * b8[7]};
                    if (is_slc(MODE)) {
                        __stcg(reinterpret_cast<float4 *>(part + ch * 32 + k),
                               make_float4(f8[0], f8[1], f8[2], f8[3]));
                        __stcg(reinterpret_cast<float4 *>(part + ch * 32 + k + 4),
                               make_float4(f8[4], f8[5], f8[6], f8[7]));
                    } else {
                        uint4 v;
                        __nv_bfloat162 *b2 = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
                        for (int z = 0; z < 4; ++z) b2[z] = __floats2bfloat162_rn(f8[2 * z], f8[2 * z + 1]);
                        __stcs(reinterpret_cast<uint4 *>(orow + ch * 32 + k), v);
                    }
                }
            }
        } else if (w.nsplit == 1) {
            // one key split: the item holds the whole softmax, write the row
            const float inv = l_run > 0.f ? vsc / l_run : 0.f;
            __nv_bfloat16 *orow = (__nv_bfloat16 *)L.out + prow;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float o[32];
                ptx::tmem_ld32(tmem + lane_base + TM_O + ch * 32, o);
                ptx::tmem_wait_ld();
                if (!rc.valid) continue;
#pragma unroll
                for (int k = 0; k < 32; k += 2) {
                    const float a = l_run > 0.f ? o[k] * inv : 0.f;
                    const float c = l_run > 0.f ? o[k + 1] * inv : 0.f;
                    *reinterpret_cast<__nv_bfloat162 *>(orow + ch * 32 + k) =
                        __floats2bfloat162_rn(a, c);
                }
            }
        } else {
            float *pr = P.part + ((size_t)item * kRows + rho) * kPartStride;
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                float o[32];
                ptx::tmem_ld32(tmem + lane_base + TM_O + ch * 32, o);
                ptx::tmem_wait_ld();
                if (rc.valid) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) pr[ch * 32 + k] = o[k] * vsc;
                }
            }
            if (rc.valid) {
                pr[kD] = m_run;
                pr[kD + 1] = l_run;
            }
        }
    }
}

template <int MODE, int RPAD = 8, int PASS = 0>
__global__ void __launch_bounds__(kThreads, 2) tc_attn_kernel(const __grid_constant__ TcParams P) {
    extern __shared__ uint8_t smem_raw[];
    const LayerParams &L = P.L;
    Smem sm;
    {
        const uint32_t raw = ptx::smem_u32(smem_raw);
        const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
        sm.base = smem_raw + pad;
        sm.base_u32 = raw + pad;
    }
    // skip the work if an earlier kernel already failed (one read, shared by
    // the whole CTA so that every thread takes the same path)
    if (threadIdx.x == 0) *sm.failed_flag() = *(volatile uint32_t *)L.status;
    __syncthreads();
    if (*sm.failed_flag() != 0) return;
    const Counts cn = *L.counts;
    const Work w = make_work<MODE>(P, cn);
    if ((int)blockIdx.x >= w.items) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (w.q_tma) {
        // MMA rows the Q box never writes (128 is not a multiple of the rows per
        // query): zero once, so masked rows read finite values
        const int q_rows = w.qt * (MODE == MODE_CMP ? w.rpad : L.r);
        for (int e = q_rows * 8 + (int)threadIdx.x; e < kRows * 8; e += blockDim.x)
            for (int hf = 0; hf < 2; ++hf)
                *reinterpret_cast<uint4 *>(sm.base + SM_Q + hf * 16384 + e * 16) =
                    make_uint4(0u, 0u, 0u, 0u);
        ptx::fence_proxy_async();
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(sm.bar(B_K_FULL + s), 1);
            ptx::mbar_init(sm.bar(B_V_FULL + s), 1);
            ptx::mbar_init(sm.bar(B_K_EMPTY + s), 1);
            ptx::mbar_init(sm.bar(B_V_EMPTY + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            ptx::mbar_init(sm.bar(B_S_FULL + b), 1);
            ptx::mbar_init(sm.bar(B_P_FULL + b), 4);
            ptx::mbar_init(sm.bar(B_PV_DONE + b), 1);
        }
        ptx::mbar_init(sm.bar(B_Q_FULL), w.q_tma ? 1 : 128);
        ptx::mbar_init(sm.bar(B_Q_EMPTY), 1);
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
        run_producer<MODE, PASS>(P, w, sm, lane);
    } else if (warp == 1) {
        if (lane == 0) run_mma<MODE, PASS>(P, w, sm, tmem);
        __syncwarp();
    } else {
        run_softmax<MODE, RPAD, PASS>(P, w, sm, tmem);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc(tmem, TM_COLS);
}

// ---------------------------------------------------------------------------
// Operands of the P V products.  P is fp16 (11 significant bits), so V and
// V_cmp enter as fp16 copies; to keep every bf16 value inside the fp16 range,
// each is divided by a power of two 2^e chosen per call so that its largest
// magnitude lands in [2^14, 2^15) (e may be negative: small values then keep
// fp16's full precision too).  Division by a power of two is exact; the
// epilogues multiply O by 2^e.  Inf / NaN inputs keep e = 0.
//
// vmax_kernel: the largest |V| over the n tokens and |V_cmp| over the blocks
// (atomicMax on the bit patterns of non-negative floats, which order like the
// values); *vmax must start at zero.
__global__ void vmax_kernel(LayerParams p, unsigned *vmax) {
    const Counts cn = *p.counts;
    const size_t row_vec = (size_t)p.h_kv * kD / 8;  // 16-byte pieces per row
    const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t step = (size_t)gridDim.x * blockDim.x;
    float m[2] = {0.f, 0.f};
    const uint4 *src[2] = {reinterpret_cast<const uint4 *>(p.v),
                           reinterpret_cast<const uint4 *>(p.v_cmp)};
    const size_t cnt[2] = {(size_t)p.n * row_vec, (size_t)cn.nc * row_vec};
#pragma unroll
    for (int w = 0; w < 2; ++w)
        for (size_t e = tid; e < cnt[w]; e += step) {
            const uint4 u = __ldg(src[w] + e);
            const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(b[i]);
                m[w] = fmaxf(m[w], fmaxf(fabsf(f.x), fabsf(f.y)));
            }
        }
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        const float r = warp_max(m[w]);
        if ((threadIdx.x & 31) == 0 && r > 0.f) atomicMax(vmax + w, __float_as_uint(r));
    }
}

// 2^-e for the largest magnitude m (see above), and 2^e into *scale_out.
__device__ __forceinline__ float v_prescale(unsigned mbits, float *scale_out) {
    const float m = __uint_as_float(mbits);
    int e = 0;
    if (m > 0.f && m <= 3.0e38f) e = (int)((mbits >> 23) & 255u) - 127 - 14;
    if (e < -100) e = -100;
    if (scale_out) *scale_out = ldexpf(1.f, e);
    return ldexpf(1.f, -e);
}

__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 u, float mul) {
    const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&u);
    uint4 r;
    __half2 *h = reinterpret_cast<__half2 *>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(b[i]);
        h[i] = __floats2half2_rn(f.x * mul, f.y * mul);
    }
    return r;
}

// The scaled fp16 copies of V (all positions) and V_cmp, and the vision K
// (bf16) and V (scaled fp16) in vision order when the vision tokens are not
// one contiguous run of positions (the TMA tiles need consecutive rows).
__global__ void prepare_kernel(LayerParams p, const unsigned *vmax, float *v_scale,
                               __nv_bfloat16 *kc, __half *vhc, __half *vh, __half *vh_cmp) {
    const Counts cn = *p.counts;
    const bool first = blockIdx.x == 0 && threadIdx.x == 0;
    const float mv = v_prescale(vmax[0], first ? v_scale : nullptr);
    const float mc = v_prescale(vmax[1], first ? v_scale + 1 : nullptr);
    const size_t row_vec = (size_t)p.h_kv * kD / 8;  // 16-byte pieces per row
    const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t step = (size_t)gridDim.x * blockDim.x;
    const uint4 *v = reinterpret_cast<const uint4 *>(p.v);
    for (size_t e = tid; e < (size_t)p.n * row_vec; e += step)
        reinterpret_cast<uint4 *>(vh)[e] = bf16x8_to_f16x8(__ldg(v + e), mv);
    const uint4 *vb = reinterpret_cast<const uint4 *>(p.v_cmp);
    for (size_t e = tid; e < (size_t)cn.nc * row_vec; e += step)
        reinterpret_cast<uint4 *>(vh_cmp)[e] = bf16x8_to_f16x8(vb[e], mc);
    if (!cn.contiguous) {
        for (size_t e = tid; e < (size_t)cn.n_vision * row_vec; e += step) {
            const size_t u = e / row_vec, c = e % row_vec;
            const size_t src = (size_t)p.vis[u] * row_vec + c;
            reinterpret_cast<uint4 *>(kc)[e] = __ldg(reinterpret_cast<const uint4 *>(p.k) + src);
            reinterpret_cast<uint4 *>(vhc)[e] = bf16x8_to_f16x8(__ldg(v + src), mv);
        }
    }
}

// ---------------------------------------------------------------------------
// Union over the queries of each SLC item of the 64-key tiles their selected
// blocks reach (a block of B keys covers the tiles from key j*B to key
// min(j*B + B - 1, i) of query i), with a mask of the queries that reach each
// tile.  One warp per item.
__device__ __forceinline__ void sel_tiles(int j, int B, int i, int &t0, int &t1) {
    if (B == kKeys) {  // one tile per block
        t0 = t1 = j;
        return;
    }
    const long long a = (long long)j * B;
    t0 = (int)(a / kKeys);
    t1 = (int)(min(a + B - 1, (long long)i) / kKeys);
}

// Where the tiles that leave the union go (SglArgs.on): pair records, the
// per-bucket counts, and each query's pair count.
struct SglArgs {
    int on, nbt, cap;
    int32_t *meta;  // [0] pairs, [1] items, [2, 2 + h_kv*nbt) pairs per bucket
    int4 *rec;      // [cap] (bucket, pair id, rank in bucket, position)
    int32_t *n;     // [h_kv][n_max] pairs (slots used) of each query
};

__global__ void union_kernel(LayerParams p, int32_t *plan, int plan_max, int words, SglArgs sg) {
    extern __shared__ uint32_t sh[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wpb = blockDim.x >> 5;
    const unsigned lt = (1u << lane) - 1u;
    uint32_t *bm = sh + (size_t)warp * (2 * words + 2 * plan_max + 32);
    uint32_t *pre = bm + words;
    uint32_t *qm = pre + words;
    uint32_t *qcnt = qm + plan_max;  // per query of the item: its pair slots taken
    int *sslot = (int *)(qcnt + 32); // per tile: its pair slot, -1 if it stays
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
            if (j < 0) continue;
            if (j > (q0 + qi) / p.block) {
                // a block after the query's own (a caller selection out of
                // range): reported and left out
                report(p.status, VNSA_ERR_BOUNDS);
                continue;
            }
            int t0, t1;
            sel_tiles(j, p.block, q0 + qi, t0, t1);
            for (int t = t0; t <= t1 && (t >> 5) < words; ++t)
                atomicOr(&bm[t >> 5], 1u << (t & 31));
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
            if (j < 0 || j > (q0 + qi) / p.block) continue;
            int t0, t1;
            sel_tiles(j, p.block, q0 + qi, t0, t1);
            for (int t = t0; t <= t1 && (t >> 5) < words; ++t) {
                const int r = pre[t >> 5] + __popc(bm[t >> 5] & ((1u << (t & 31)) - 1u));
                if (r < plan_max) atomicOr(&qm[r], 1u << qi);
            }
        }
        __syncwarp();
        int tot = min(total, plan_max);
        if (sg.on) {
            // Tiles that at most kSglShare queries of the item reach leave the
            // plan for the tile-major pass (sgl_attn.cu) as (query, tile) pairs:
            // a 128-row union tile costs the same whatever number of its rows
            // attend, and a pair costs a gathered Q row block, an output row
            // block and its merge, which is about a union tile's cost for three
            // queries.  Up to kSglSlots pairs per query: first its single-query
            // tiles in tile order, then the two-query and then the three-query
            // tiles in tile order while each of the tile's queries has a slot
            // left (the rest stay), and only while at least one tile stays.
            // The pair (vision query i of group g, slot s) has the id
            // (g n_max + i) kSglSlots + s, so the merge finds a query's pairs
            // without a lookup.  sslot[x]: -1 (stays), the slot of a
            // single-query tile, or 32 + the slots of the tile's queries in
            // 5-bit fields, lowest query first.
            qcnt[lane] = 0u;
            __syncwarp();
            int npair = 0;   // pairs
            int nleave = 0;  // tiles that leave
            for (int xb = 0; xb < tot; xb += 32) {
                const int x = xb + lane;
                const uint32_t m = x < tot ? qm[x] : 0u;
                const bool single = x < tot && __popc(m) == 1;
                const int key = single ? __ffs(m) - 1 : 32 + lane;  // others: unique keys
                const unsigned grp = __match_any_sync(0xffffffffu, key);
                const int slot = single ? (int)qcnt[key] + __popc(grp & lt) : -1;
                __syncwarp();
                if (single && (grp & lt) == 0) qcnt[key] += (uint32_t)__popc(grp);
                __syncwarp();
                const bool pair = single && slot < kSglSlots;
                if (x < tot) sslot[x] = pair ? slot : -1;
                npair += __popc(__ballot_sync(0xffffffffu, pair));
            }
            nleave = npair;
            __syncwarp();
            // then the tiles of two, then of three queries, each kind one tile
            // after the other in tile order (a few dozen per item), so a tile
            // takes all its slots or none and no slot is left unused below a
            // query's count; lane q holds query q's count
            uint32_t myc = qcnt[lane];
            for (int want = 2; want <= kSglShare; ++want) {
                for (int xb = 0; xb < tot; xb += 32) {
                    const int x = xb + lane;
                    const uint32_t m = x < tot ? qm[x] : 0u;
                    unsigned sel = __ballot_sync(0xffffffffu, x < tot && __popc(m) == want);
                    int mine = -1;
                    while (sel) {  // the same tiles on every lane
                        const int b = __ffs(sel) - 1;
                        sel &= sel - 1;
                        const uint32_t mb = __shfl_sync(0xffffffffu, m, b);
                        bool room = true;
                        int v = 0, sh = 0;
                        for (uint32_t mm = mb; mm; mm &= mm - 1, sh += 5) {
                            const uint32_t cq = __shfl_sync(0xffffffffu, myc, __ffs(mm) - 1);
                            room = room && cq < (uint32_t)kSglSlots;
                            v |= (int)cq << sh;
                        }
                        if (room) {
                            if ((mb >> lane) & 1u) ++myc;
                            if (lane == b) mine = 32 + v;
                            npair += want;
                            ++nleave;
                        }
                    }
                    if (mine >= 0) sslot[x] = mine;
                }
            }
            qcnt[lane] = myc;
            __syncwarp();
            if (nleave >= tot) {  // every tile would leave: the item keeps them all
                for (int x = lane; x < tot; x += 32) sslot[x] = -1;
                npair = 0;
            }
            int base = 0;
            if (npair > 0) {
                if (lane == 0) base = atomicAdd(&sg.meta[0], npair);
                base = __shfl_sync(0xffffffffu, base, 0);
                if (base + npair > sg.cap) {  // cannot happen: cap holds every slot
                    if (lane == 0) report(p.status, VNSA_ERR_BOUNDS);
                    for (int x = lane; x < tot; x += 32) sslot[x] = -1;
                    npair = 0;
                }
            }
            __syncwarp();
            if (npair > 0) {
                int kept = 0, si = 0;
                for (int xb = 0; xb < tot; xb += 32) {
                    const int x = xb + lane;
                    const uint32_t m = x < tot ? qm[x] : 0u;
                    const int tl = x < tot ? out[1 + x] : 0;
                    const int sl = x < tot ? sslot[x] : -1;
                    const bool pair = sl >= 0;
                    const bool keep = x < tot && !pair;
                    // pairs of this tile (one per query) and their offset in the batch
                    const int cnt = pair ? (sl >= 32 ? __popc(m) : 1) : 0;
                    int incl = cnt;
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        const int v = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += v;
                    }
                    const int all = __shfl_sync(0xffffffffu, incl, 31);
                    // every lane holds its entry before any entry is moved down
                    const unsigned bk = __ballot_sync(0xffffffffu, keep);
                    if (keep) {
                        const int pos = kept + __popc(bk & lt);
                        out[1 + pos] = tl;
                        qm[pos] = m;
                    }
                    if (pair) {
                        const int bucket = g * sg.nbt + tl;
                        const int at = base + si + incl - cnt;
                        const int lp = atomicAdd(&sg.meta[2 + bucket], cnt);
                        const int v = sl >= 32 ? sl - 32 : sl;  // 5-bit slot fields
                        uint32_t mm = m;
                        for (int e = 0; e < cnt; ++e, mm &= mm - 1) {
                            const int i = q0 + __ffs(mm) - 1;
                            const int se = (v >> (5 * e)) & 31;
                            sg.rec[at + e] = make_int4(bucket, (g * p.n_max + i) * kSglSlots + se,
                                                       lp + e, p.vis[i]);
                        }
                    }
                    kept += __popc(bk);
                    si += all;
                    __syncwarp();
                }
                tot = kept;
            }
            __syncwarp();
            for (int qi = lane; qi < nq; qi += 32)
                sg.n[(size_t)g * p.n_max + q0 + qi] =
                    npair > 0 ? min((int)qcnt[qi], kSglSlots) : 0;
        }
        for (int x = lane; x < tot; x += 32) out[1 + plan_max + x] = (int)qm[x];
        if (lane == 0) {
            out[0] = tot;
            if (total > plan_max) report(p.status, VNSA_ERR_BOUNDS);
        }
        __syncwarp();
    }
}

// Offsets of the (query, tile) pairs grouped by bucket (group, tile) and of the
// tile-major pass's chunks (qt pairs of one bucket): exclusive prefix sums
// over the bucket counts, one block.
__global__ void __launch_bounds__(1024) sgl_scan_kernel(int32_t *meta, int nbk, int qt) {
    __shared__ int wsum[2][32];
    const int32_t *hist = meta + 2;
    int32_t *off = meta + 2 + nbk, *choff = meta + 2 + 2 * nbk;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (nbk + blockDim.x - 1) / blockDim.x;
    const int b0 = min(nbk, tid * per), b1 = min(nbk, b0 + per);
    int a = 0, c = 0;
    for (int b = b0; b < b1; ++b) {
        a += hist[b];
        c += (hist[b] + qt - 1) / qt;
    }
    int ia = a, ic = c;  // inclusive scans within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int va = __shfl_up_sync(0xffffffffu, ia, o), vc = __shfl_up_sync(0xffffffffu, ic, o);
        if (lane >= o) {
            ia += va;
            ic += vc;
        }
    }
    if (lane == 31) {
        wsum[0][warp] = ia;
        wsum[1][warp] = ic;
    }
    __syncthreads();
    if (warp == 0) {
        int xa = lane < (int)(blockDim.x >> 5) ? wsum[0][lane] : 0;
        int xc = lane < (int)(blockDim.x >> 5) ? wsum[1][lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int va = __shfl_up_sync(0xffffffffu, xa, o), vc = __shfl_up_sync(0xffffffffu, xc, o);
            if (lane >= o) {
                xa += va;
                xc += vc;
            }
        }
        wsum[0][lane] = xa;  // inclusive over warps
        wsum[1][lane] = xc;
    }
    __syncthreads();
    int ra = ia - a + (warp > 0 ? wsum[0][warp - 1] : 0);
    int rc = ic - c + (warp > 0 ? wsum[1][warp - 1] : 0);
    for (int b = b0; b < b1; ++b) {
        off[b] = ra;
        choff[b] = rc;
        ra += hist[b];
        rc += (hist[b] + qt - 1) / qt;
    }
    if (tid == (int)blockDim.x - 1) {
        choff[nbk] = rc;
        meta[1] = rc;
    }
}

// The tile-major pass's chunk table and entries.  Chunk c of bucket b is item
// choff[b] + c = (b, first entry, pairs, 0); entries are laid out qt per chunk,
// entry (chunk x, slot s) at x qt + s = (pair id, vision rank, position,
// bucket), and the slots of a bucket's last chunk past its pairs hold
// (-1, 0, 0, bucket).  So a row of the tile-major pass finds its entry in one
// independent load.
__global__ void sgl_scatter_kernel(const int32_t *meta, const int4 *rec, int4 *sorted,
                                   int4 *items, int nbk, int cap, int qt, int n_max) {
    const int n = min(meta[0], cap);
    const int32_t *hist = meta + 2, *choff = meta + 2 + 2 * nbk;
    const int tid = blockIdx.x * blockDim.x + threadIdx.x, step = gridDim.x * blockDim.x;
    for (int k = tid; k < n; k += step) {
        const int4 e = rec[k];  // (bucket, id, rank in bucket, position)
        const int i = (e.y / kSglSlots) % n_max;
        sorted[(size_t)choff[e.x] * qt + e.z] = make_int4(e.y, i, e.w, e.x);
    }
    for (int b = tid; b < nbk; b += step) {
        const int cnt = hist[b];
        const int nch = (cnt + qt - 1) / qt;
        for (int c = 0; c < nch; ++c)
            items[choff[b] + c] =
                make_int4(b, (choff[b] + c) * qt, min(qt, cnt - c * qt), 0);
        for (int x = cnt; x < nch * qt; ++x)
            sorted[(size_t)choff[b] * qt + x] = make_int4(-1, 0, 0, b);
    }
}

// The selection output of each (vision query, head): the union tiles' part
// (slc_u, slc_lse) and the query's (query, tile) pairs (slot ids qg kSglSlots +
// z, z < n[qg]: sgl_o, sgl_lse), each the exact softmax over its keys,
// combined with the weights 2^(lse_part - M) / sum over the parts; then the
// vision output row out = partial (compression) + sigmoid(g_slc) * o_slc +
// swa_part (window), rounded once to bf16, and the optional export.  Every
// address follows from (group, query, slot), so a row's loads are independent.
// One warp per (group, query); its r heads x 128 dims are cut into 16-dim
// chunks, chunk c = lane + 32 k (head c / 8), so a warp's load instruction
// covers four heads contiguously and each lane computes the weights of its
// own (at most two) heads.
struct SlcMergeArgs {
    const int32_t *n;
    const __half *sgl_o, *slc_u;
    const float *sgl_lse, *slc_lse, *v_scale;
    const __half *swa_part;  // sig(g_swa) o_swa / v_scale of the window pass
};

__device__ __forceinline__ void acc_half8(float (&acc)[8], uint4 u, float w) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float2 f = __half22float2(h[q]);
        acc[2 * q] = fmaf(w, f.x, acc[2 * q]);
        acc[2 * q + 1] = fmaf(w, f.y, acc[2 * q + 1]);
    }
}

__global__ void __launch_bounds__(256) slc_merge_kernel(LayerParams p, SlcMergeArgs a) {
    const Counts cn = *p.counts;
    const int lane = threadIdx.x & 31;
    const int r = p.r, nv = cn.n_vision;
    const int nchunk = r * (kD / 16);  // 16-dim chunks of a row (56 for 7 heads)
    const float vsc = *a.v_scale;
    const int rows = p.h_kv * nv;
    for (int wid = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; wid < rows;
         wid += (gridDim.x * blockDim.x) >> 5) {
        const int g = wid / nv, i = wid - g * nv;
        const int h0 = g * r;
        const int t = p.vis[i];
        const size_t qg = (size_t)g * p.n_max + i;
        const size_t id0 = qg * kSglSlots;
        const int ns = a.n[qg];
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int c = lane + 32 * k;
            if (c >= nchunk) continue;
            const int hl = c >> 3, d0 = (c & 7) * 16;
            // weights of this chunk's head (slots past the count are not read)
            const float lu = a.slc_lse[(size_t)i * p.h_q + h0 + hl];
            float lz[kSglSlots];
#pragma unroll
            for (int z = 0; z < kSglSlots; ++z)
                lz[z] = z < ns ? a.sgl_lse[(id0 + z) * r + hl] : -INFINITY;
            const size_t urow = ((size_t)i * p.h_q + h0 + hl) * kD + d0;
            const uint4 *us = reinterpret_cast<const uint4 *>(a.slc_u + urow);
            const uint4 u0 = __ldcs(us), u1 = __ldcs(us + 1);
            // the first half of the slots' outputs in flight with the weights
            constexpr int kHalf = kSglSlots / 2;
            uint4 pz[kHalf][2];
            auto load_half = [&](int zb) {
#pragma unroll
                for (int z = 0; z < kHalf; ++z) {
                    if (zb + z < ns) {
                        const uint4 *ps = reinterpret_cast<const uint4 *>(
                            a.sgl_o + ((id0 + zb + z) * r + hl) * kD + d0);
                        pz[z][0] = __ldcs(ps);
                        pz[z][1] = __ldcs(ps + 1);
                    }
                }
            };
            load_half(0);
            const float gl = sigmoidf_(p.gate[((size_t)t * p.h_q + h0 + hl) * 3 + 1]);
            float mx = lu;
#pragma unroll
            for (int z = 0; z < kSglSlots; ++z) mx = fmaxf(mx, lz[z]);
            const float wu = lu == -INFINITY ? 0.f : exp2f(lu - mx);
            float wsum = wu;
#pragma unroll
            for (int z = 0; z < kSglSlots; ++z) {
                lz[z] = lz[z] == -INFINITY ? 0.f : exp2f(lz[z] - mx);
                wsum += lz[z];
            }
            const float norm = wsum > 0.f ? vsc / wsum : 0.f;  // back to V's units
            float acc0[8], acc1[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc0[e] = acc1[e] = 0.f;
            acc_half8(acc0, u0, wu * norm);
            acc_half8(acc1, u1, wu * norm);
#pragma unroll
            for (int z = 0; z < kHalf; ++z) {
                if (z < ns) {
                    acc_half8(acc0, pz[z][0], lz[z] * norm);
                    acc_half8(acc1, pz[z][1], lz[z] * norm);
                }
            }
            if (ns > kHalf) {
                load_half(kHalf);
#pragma unroll
                for (int z = 0; z < kHalf; ++z) {
                    if (kHalf + z < ns) {
                        acc_half8(acc0, pz[z][0], lz[kHalf + z] * norm);
                        acc_half8(acc1, pz[z][1], lz[kHalf + z] * norm);
                    }
                }
            }
            const float4 *pr = reinterpret_cast<const float4 *>(p.o_cmp_ws + urow);
            const uint4 *sw = reinterpret_cast<const uint4 *>(a.swa_part + urow);
            float4 pv[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) pv[q] = __ldcs(pr + q);
            const uint4 sw0 = __ldcs(sw), sw1 = __ldcs(sw + 1);
            float wf[16];
            {
                const __half2 *h0 = reinterpret_cast<const __half2 *>(&sw0);
                const __half2 *h1 = reinterpret_cast<const __half2 *>(&sw1);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float2 f0 = __half22float2(h0[q]), f1 = __half22float2(h1[q]);
                    wf[2 * q] = f0.x * vsc;
                    wf[2 * q + 1] = f0.y * vsc;
                    wf[8 + 2 * q] = f1.x * vsc;
                    wf[8 + 2 * q + 1] = f1.y * vsc;
                }
            }
            const float4 *wv = reinterpret_cast<const float4 *>(wf);
            const float *ac[2] = {acc0, acc1};
            uint4 ob[2];
            __nv_bfloat162 *b2 = reinterpret_cast<__nv_bfloat162 *>(ob);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float *o4 = ac[q >> 1] + 4 * (q & 1);
                const float x0 = fmaf(gl, o4[0], pv[q].x) + wv[q].x;
                const float x1 = fmaf(gl, o4[1], pv[q].y) + wv[q].y;
                const float x2 = fmaf(gl, o4[2], pv[q].z) + wv[q].z;
                const float x3 = fmaf(gl, o4[3], pv[q].w) + wv[q].w;
                b2[2 * q] = __floats2bfloat162_rn(x0, x1);
                b2[2 * q + 1] = __floats2bfloat162_rn(x2, x3);
            }
            uint4 *orow = reinterpret_cast<uint4 *>((__nv_bfloat16 *)p.out +
                                                    ((size_t)t * p.h_q + h0 + hl) * kD + d0);
            __stcs(orow, ob[0]);
            __stcs(orow + 1, ob[1]);
            if (p.dbg_o_slc) {
                float *dbg = p.dbg_o_slc + ((size_t)t * p.h_q + h0 + hl) * kD + d0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    dbg[e] = acc0[e];
                    dbg[8 + e] = acc1[e];
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Text split-KV combine: one warp per (text query, head).
__device__ void text_combine_row(const LayerParams &p, const float *part, int ns, int n_tt,
                                 int qt, int x, int h, int lane) {
    const int tiles = p.h_kv * n_tt;
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
    if (cn.n_text == 0) return;
    const int lane = threadIdx.x & 31;
    const int qt = kRows / p.r;
    const int n_tt = (cn.n_text + qt - 1) / qt;
    // the same split rule as make_work
    const int span = p.txt[cn.n_text - 1] + 1;
    const int tiles = p.h_kv * n_tt;
    const int ns = max(1, min((span + kTextSplitKeys - 1) / kTextSplitKeys,
                              max(1, part_items / tiles)));
    if (ns == 1) return;  // with a single key split the attention kernel wrote the rows
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int wi = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; wi < cn.n_text * p.h_q;
         wi += nwarps)
        text_combine_row(p, part, ns, n_tt, qt, wi / p.h_q, wi % p.h_q, lane);
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
              const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map over Q [n][h_q][128] bf16 with boxes {64 of d, rq heads, qt tokens}
// and the 128-byte swizzle: one box is a Q tile of qt queries x rq head rows in
// MMA row order (row = query * rq + head).
bool make_map_q(CUtensorMap *m, const void *q, int h_q, long long n, int rq, int qt) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || n < 1) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)h_q, (cuuint64_t)n};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)h_q * kD * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)rq, (cuuint32_t)qt};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

}  // namespace

bool tma_map_2d_bf16(CUtensorMap *m, const void *base, long long inner, long long rows,
                     int box_inner, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || inner < 1 || rows < 1) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)inner * 2};
    cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct TcState {
    vnsa_config cfg;
    int num_sms;
    int plan_max;
    int part_items;
    __nv_bfloat16 *kc;  // vision K in vision order (non-contiguous vision only)
    __half *vhc;        // vision V (scaled fp16) in vision order (non-contiguous vision only)
    __half *vh;         // V as scaled fp16, all positions
    __half *vh_cmp;     // V_cmp as scaled fp16
    unsigned *vmax;     // [2] largest |V|, |V_cmp| of the call (float bits)
    float *v_scale;     // [2] their powers of two
    int32_t *plan;
    float *part;
    // selection tiles of one or two queries (block 64): see TcParams and sgl_attn.h
    int sgl_on, sgl_nbt, sgl_cap;
    int32_t *sgl_meta, *sgl_n;
    int4 *sgl_rec, *sgl_sorted, *sgl_items;
    __half *sgl_o, *slc_u;
    float *sgl_lse, *slc_lse;
    __half *swa_part;
};


struct SglSizes {
    int on, nbt, nbk, cap;
    size_t meta, rec, sorted, items, n, o, lse, u, ulse, swa, total;
};

static SglSizes sgl_sizes(const vnsa_config &c) {
    SglSizes z;
    memset(&z, 0, sizeof(z));
    z.on = c.block == kKeys;
    if (!z.on) return z;
    const int r = c.h_q / c.h_kv;
    z.nbt = (c.n_max + kKeys - 1) / kKeys;
    z.nbk = c.h_kv * z.nbt;
    const int qt = kRows / r;
    z.cap = c.h_kv * c.n_max * kSglSlots;  // every (group, query, slot) id
    const size_t chunks = (size_t)z.cap / qt + z.nbk + 1;
    z.meta = up256((size_t)(2 + 3 * z.nbk + 1) * 4);
    z.rec = up256((size_t)z.cap * 16);
    z.sorted = up256(chunks * qt * 16);
    z.items = up256(chunks * 16);
    z.n = up256((size_t)c.h_kv * c.n_max * 4);
    z.o = up256((size_t)z.cap * r * kD * 2);
    z.lse = up256((size_t)z.cap * r * 4);
    z.u = up256((size_t)c.n_max * c.h_q * kD * 2);
    z.ulse = up256((size_t)c.n_max * c.h_q * 4);
    z.swa = up256((size_t)c.n_max * c.h_q * kD * 2);
    z.total = z.meta + z.rec + z.sorted + z.items + z.n + z.o + z.lse + z.u + z.ulse + z.swa;
    return z;
}

// Most 64-key selection tiles of one item: every query reaches at most top_k
// blocks, each over at most `per_block` tiles, and there are only so many tiles.
static int plan_tiles_max(const vnsa_config &c) {
    const int qt = kRows / (c.h_q / c.h_kv);
    const int B = c.block;
    int per_block;
    if (B % kKeys == 0) per_block = B / kKeys;
    else if (kKeys % B == 0) per_block = 1;
    else per_block = (B + kKeys - 2) / kKeys + 1;
    const long long bound = (long long)qt * c.top_k * per_block;
    const long long tiles = (c.n_max + kKeys - 1) / kKeys;
    return (int)std::min(bound, tiles);
}

// The tensor-core path: bf16, d = 128, 4 to 16 query heads per KV head (the
// selection query masks are 32-bit: at most 32 queries per item), and an item's
// selection plan and per-query block lists must fit the shared-memory copy.
bool tc_supported(const vnsa_config &c) {
    const int r = c.h_q / c.h_kv;
    if (c.dtype != VNSA_BF16 || c.d != kD || r < 4 || r > 16) return false;
    const int qt = kRows / r;
    return qt * c.top_k <= kPlanSmem && plan_tiles_max(c) <= kPlanSmem && encode_fn() != nullptr;
}

static size_t plan_bytes(const vnsa_config &c) {
    const int qt = kRows / (c.h_q / c.h_kv);
    const size_t items = (size_t)c.h_kv * ((c.n_max + qt - 1) / qt);
    return items * (1 + 2 * (size_t)plan_tiles_max(c)) * 4;
}

size_t tc_workspace_bytes(const vnsa_config &c) {
    if (!tc_supported(c)) return 0;
    const size_t kv = (size_t)c.n_max * c.h_kv * kD * 2;
    const size_t kvb = (size_t)(cmp_blocks(c.n_max, c.block, cmp_stride_of(c)) + 1) * c.h_kv * kD * 2;
    return up256(kv) * 3 + up256(kvb) + 256 + up256(plan_bytes(c)) + kTextPartBytes +
           sgl_sizes(c).total;
}

cudaError_t tc_create(const vnsa_config &c, void *ws, TcState **out) {
    *out = nullptr;
    if (!tc_supported(c)) return cudaSuccess;
    TcState *st = new TcState();
    st->cfg = c;
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&st->num_sms, cudaDevAttrMultiProcessorCount, dev);
    st->plan_max = plan_tiles_max(c);
    st->part_items = (int)(kTextPartBytes / ((size_t)kRows * kPartStride * 4));
    char *p = (char *)ws;
    const size_t kv = up256((size_t)c.n_max * c.h_kv * kD * 2);
    const size_t kvb =
        up256((size_t)(cmp_blocks(c.n_max, c.block, cmp_stride_of(c)) + 1) * c.h_kv * kD * 2);
    st->kc = (__nv_bfloat16 *)p;
    st->vhc = (__half *)(p + kv);
    st->vh = (__half *)(p + 2 * kv);
    st->vh_cmp = (__half *)(p + 3 * kv);
    st->vmax = (unsigned *)(p + 3 * kv + kvb);
    st->v_scale = (float *)(p + 3 * kv + kvb + 16);
    p += 256;  // vmax and v_scale
    st->plan = (int32_t *)(p + 3 * kv + kvb);
    st->part = (float *)(p + 3 * kv + kvb + up256(plan_bytes(c)));
    {
        const SglSizes z = sgl_sizes(c);
        st->sgl_on = z.on;
        st->sgl_nbt = z.nbt;
        st->sgl_cap = z.cap;
        char *q = p + 3 * kv + kvb + up256(plan_bytes(c)) + kTextPartBytes;
        st->sgl_meta = (int32_t *)q;
        st->sgl_rec = (int4 *)(q += z.meta);
        st->sgl_sorted = (int4 *)(q += z.rec);
        st->sgl_items = (int4 *)(q += z.sorted);
        st->sgl_n = (int32_t *)(q += z.items);
        st->sgl_o = (__half *)(q += z.n);
        st->sgl_lse = (float *)(q += z.o);
        st->slc_u = (__half *)(q += z.lse);
        st->slc_lse = (float *)(q += z.u);
        st->swa_part = (__half *)(q += z.ulse);
    }
    cudaError_t e = cudaSuccess;
    for (auto fn : {tc_attn_kernel<MODE_CMP, 4, 1>, tc_attn_kernel<MODE_CMP, 4, 2>,
                    tc_attn_kernel<MODE_CMP, 8, 1>, tc_attn_kernel<MODE_CMP, 8, 2>,
                    tc_attn_kernel<MODE_CMP, 16, 1>, tc_attn_kernel<MODE_CMP, 16, 2>,
                    tc_attn_kernel<MODE_SLC>, tc_attn_kernel<MODE_SWA>, tc_attn_kernel<MODE_TEXT>,
                    tc_attn_kernel<MODE_SLC_UNALIGNED>})
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e == cudaSuccess) e = sgl_prepare();
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
    // a kernel argument rather than a constant: with the kind fixed at compile
    // time the exact pass's register allocation spills
    P.exact_kind = K_EXACT;
    P.L = L;
    P.plan = st->plan;
    P.plan_max = st->plan_max;
    P.part = st->part;
    P.part_items = st->part_items;
    const bool sgl = st->sgl_on && c.block == kKeys;
    P.sgl_on = 0;  // set for the selection launch below
    P.slc_u = st->slc_u;
    P.slc_lse = st->slc_lse;
    const int nb_rows = L.nb_max > 0 ? L.nb_max : 1;  // compression blocks
    if (!make_map(&P.tm_k, L.k, c.h_kv, L.n, false) ||
        !make_map(&P.tm_v, st->vh, c.h_kv, L.n, true) ||
        !make_map(&P.tm_kc, st->kc, c.h_kv, c.n_max, false) ||
        !make_map(&P.tm_vc, st->vhc, c.h_kv, c.n_max, true) ||
        !make_map(&P.tm_kb, L.k_cmp, c.h_kv, nb_rows, false) ||
        !make_map(&P.tm_vb, st->vh_cmp, c.h_kv, nb_rows, true))
        return cudaErrorInvalidValue;
    P.v_scale = st->v_scale;
    auto begin = [&](int stg) {
        if (ev) cudaEventRecord(ev[2 * stg], s);
        ran[stg] = 1;
    };
    auto end = [&](int stg) {
        if (ev) cudaEventRecord(ev[2 * stg + 1], s);
    };
    const int grid = 2 * st->num_sms;  // two CTAs per SM
    cudaError_t e;
    auto attn = [&](int mode) -> cudaError_t {
        P.mode = mode;
        {
            const int rq = mode == MODE_CMP ? pow2_at_least(L.r) : L.r;
            if (!make_map_q(&P.tm_q, L.q, c.h_q, L.n, rq, kRows / rq)) return cudaErrorInvalidValue;
        }
        switch (mode) {
            case MODE_CMP:
                // head slots per query 4, 8 or 16 (4 to 16 heads per KV head);
                // the statistics pass, then the exact pass, as two launches so
                // that each kernel carries only its pass's code
                if (pow2_at_least(L.r) == 4) {
                    tc_attn_kernel<MODE_CMP, 4, 1><<<grid, kThreads, SMEM_BYTES, s>>>(P);
                    tc_attn_kernel<MODE_CMP, 4, 2><<<grid, kThreads, SMEM_BYTES, s>>>(P);
                } else if (pow2_at_least(L.r) == 8) {
                    tc_attn_kernel<MODE_CMP, 8, 1><<<grid, kThreads, SMEM_BYTES, s>>>(P);
                    tc_attn_kernel<MODE_CMP, 8, 2><<<grid, kThreads, SMEM_BYTES, s>>>(P);
                } else {
                    tc_attn_kernel<MODE_CMP, 16, 1><<<grid, kThreads, SMEM_BYTES, s>>>(P);
                    tc_attn_kernel<MODE_CMP, 16, 2><<<grid, kThreads, SMEM_BYTES, s>>>(P);
                }
                ++*launches;
                break;
            case MODE_SLC: tc_attn_kernel<MODE_SLC><<<grid, kThreads, SMEM_BYTES, s>>>(P); break;
            case MODE_SLC_UNALIGNED:
                tc_attn_kernel<MODE_SLC_UNALIGNED><<<grid, kThreads, SMEM_BYTES, s>>>(P);
                break;
            case MODE_SWA: tc_attn_kernel<MODE_SWA><<<grid, kThreads, SMEM_BYTES, s>>>(P); break;
            default: tc_attn_kernel<MODE_TEXT><<<grid, kThreads, SMEM_BYTES, s>>>(P); break;
        }
        ++*launches;
        return cudaSuccess;
    };
    cudaError_t e0 = cudaMemsetAsync(st->vmax, 0, 2 * sizeof(unsigned), s);
    if (e0 != cudaSuccess) return e0;
    vmax_kernel<<<st->num_sms * 4, 256, 0, s>>>(L, st->vmax);
    prepare_kernel<<<st->num_sms * 4, 256, 0, s>>>(L, st->vmax, st->v_scale, st->kc, st->vhc,
                                                   st->vh, st->vh_cmp);
    *launches += 2;
    begin(VNSA_STAGE_CMP);
    if ((e = attn(MODE_CMP)) != cudaSuccess) return e;
    end(VNSA_STAGE_CMP);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (sgl) {
        // the window pass writes only its own gated part here (the selection
        // merge writes the rows), so it needs neither the top-k nor the
        // selection
        begin(VNSA_STAGE_SWA);
        P.swa_part = st->swa_part;
        if ((e = attn(MODE_SWA)) != cudaSuccess) return e;
        P.swa_part = nullptr;
        end(VNSA_STAGE_SWA);
    }
    begin(VNSA_STAGE_TOPK);
    if (L.stride != L.block) {
        // overlapping compression blocks: their importance onto the selection blocks
        if ((e = launch_imp_remap(L, s)) != cudaSuccess) return e;
        ++*launches;
    }
    if (!forced) {
        if ((e = launch_topk(L, s)) != cudaSuccess) return e;
        ++*launches;
    }
    {
        const int words = ((c.n_max + kKeys - 1) / kKeys + 31) / 32 + 1;
        const int wpb = 4;
        const size_t smem = (size_t)wpb * (2 * words + 2 * st->plan_max + 32) * 4;
        if (smem > 48 * 1024) {
            e = cudaFuncSetAttribute(union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem);
            if (e != cudaSuccess) return e;
        }
        SglArgs sa;
        memset(&sa, 0, sizeof(sa));
        if (sgl) {
            // pair count and per-bucket counts start at zero
            e = cudaMemsetAsync(st->sgl_meta, 0, (size_t)(2 + c.h_kv * st->sgl_nbt) * 4, s);
            if (e != cudaSuccess) return e;
            sa.on = 1;
            sa.nbt = st->sgl_nbt;
            sa.cap = st->sgl_cap;
            sa.meta = st->sgl_meta;
            sa.rec = st->sgl_rec;
            sa.n = st->sgl_n;
        }
        union_kernel<<<st->num_sms * 8, wpb * 32, smem, s>>>(L, st->plan, st->plan_max, words, sa);
        ++*launches;
        if (sgl) {
            const int nbk = c.h_kv * st->sgl_nbt;
            sgl_scan_kernel<<<1, 1024, 0, s>>>(st->sgl_meta, nbk, kRows / L.r);
            sgl_scatter_kernel<<<st->num_sms * 4, 256, 0, s>>>(st->sgl_meta, st->sgl_rec,
                                                               st->sgl_sorted, st->sgl_items, nbk,
                                                               st->sgl_cap, kRows / L.r,
                                                               c.n_max);
            *launches += 2;
        }
    }
    end(VNSA_STAGE_TOPK);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    begin(VNSA_STAGE_SLC);
    if (sgl) {
        // the (query, tile) pairs tile-major, the union tiles, then the merge
        // of both into the selection output, which with the compression
        // partial and the window part gives the vision output rows
        SglParams sp;
        memset(&sp, 0, sizeof(sp));
        sp.tm_k = P.tm_k;
        sp.tm_v = P.tm_v;
        sp.tm_kc = P.tm_kc;
        sp.tm_vc = P.tm_vc;
        sp.counts = L.counts;
        sp.q = (const __nv_bfloat16 *)L.q;
        sp.h_q = c.h_q;
        sp.r = L.r;
        sp.nbt = st->sgl_nbt;
        sp.scale_log2 = L.scale_log2;
        sp.n_items = st->sgl_meta + 1;
        sp.sorted = st->sgl_sorted;
        sp.items = st->sgl_items;
        sp.o = st->sgl_o;
        sp.lse = st->sgl_lse;
        sp.status = L.status;
        sp.wait_ns = L.wait_ns;
        if ((e = launch_sgl_attn(sp, st->num_sms, s)) != cudaSuccess) return e;
        ++*launches;
        P.sgl_on = 1;
        if ((e = attn(MODE_SLC)) != cudaSuccess) return e;
        P.sgl_on = 0;
        SlcMergeArgs ma;
        ma.n = st->sgl_n;
        ma.sgl_o = st->sgl_o;
        ma.slc_u = st->slc_u;
        ma.sgl_lse = st->sgl_lse;
        ma.slc_lse = st->slc_lse;
        ma.v_scale = st->v_scale;
        ma.swa_part = st->swa_part;
        slc_merge_kernel<<<st->num_sms * 16, 256, 0, s>>>(L, ma);
        ++*launches;
    } else if ((e = attn(c.block % kKeys == 0 ? MODE_SLC : MODE_SLC_UNALIGNED)) != cudaSuccess) {
        return e;
    }
    end(VNSA_STAGE_SLC);
    if (!sgl) {
        // the window epilogue adds its part to the partial and writes the rows
        begin(VNSA_STAGE_SWA);
        if ((e = attn(MODE_SWA)) != cudaSuccess) return e;
        end(VNSA_STAGE_SWA);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    begin(VNSA_STAGE_TEXT);
    if ((e = attn(MODE_TEXT)) != cudaSuccess) return e;
    // grid-stride over (text query, head); the kernel reads N_t on the device
    text_combine_kernel<<<st->num_sms * 4, 256, 0, s>>>(L, st->part, st->part_items);
    ++*launches;
    end(VNSA_STAGE_TEXT);
    return cudaGetLastError();
}

void tc_destroy(TcState *st) { delete st; }

}  // namespace vnsa
