// topk.cuh -- block selection of one (group, query) row by one warp; used by
// the prefill top-k kernel and by the decode step.
#pragma once

#include "common.cuh"

namespace vnsa {

// ---------------------------------------------------------------------------
// Top-k block selection: one warp per (group g, vision query i).
// Forced blocks: 0 and the query's own block i/B (when enabled) count within
// top_k.  The remaining m slots take the visible, non-forced blocks with the
// largest importance, ties to the lower block index.  Output ascending, -1
// padded.
//
// Importance values are non-negative floats, so their bit patterns order like
// the values; a block's sort key is (bits << 32) | ~index, so that the larger
// key is the block the rule prefers (keys are unique).
//   1. Each lane keeps the T largest candidate bit patterns of blocks lane,
//      lane + 32, ... (neighbouring blocks, whose importances tend to be alike,
//      fall to different lanes); T = 2 for m <= 32, else 4.  t0 = the m-th
//      largest of those 32 T values (m rounds of a warp max, each round taking
//      one copy of the maximum out of its lane's list) cannot exceed the m-th
//      largest candidate, so only candidates at or above it can be selected;
//      with T = 4 it stays close to it even for m near 64.
//   2. A second pass over the row (now in cache) collects those survivors in
//      block order into shared memory (ballot compaction).
//   3. Each survivor's rank is the number of survivors with a larger key; the
//      m of rank < m are the selection.  Survivors are in block order, so a
//      ballot prefix over "selected" gives each selected block its output
//      position (plus the forced blocks below it).  (More than 128 survivors:
//      m rounds of a warp argmax over the keys below the previous pick, then
//      4.)
//   4. The output position of a selected block is the number of selected
//      blocks with a lower index plus the forced blocks below it.
// No sorting network: shared memory is touched once per survivor and once per
// rank comparison (broadcast reads).  Shared memory is 1 KB per warp.
constexpr int kTopkBuf = 128;  // survivors per warp in shared memory

// The selection of one (group, query) row by one warp.  row: the query's
// importance over its c visible blocks (global memory when kGlobal, else
// shared memory); own: the query's own block; buf: 128 keys of warp scratch in
// shared memory; out: top_k entries, ascending, -1 padded.
template <bool kGlobal>
__device__ __forceinline__ void topk_select_row(const float *row, int c, int own, int top_k,
                                                int force_first, int force_local, uint64_t *buf,
                                                int lane, int32_t *out, uint32_t *status) {
    const bool f0 = force_first && c > 0;
    const bool fo = force_local && own < c && !(f0 && own == 0);
    const int nforced =
        (force_first ? 1 : 0) + ((force_local && !(force_first && own == 0)) ? 1 : 0);
    const int m = top_k - nforced;
    const int ncand = c - (f0 ? 1 : 0) - (fo ? 1 : 0);
    const unsigned lt = (1u << lane) - 1u;  // lanes below this one
    auto load = [&](int j) { return kGlobal ? __ldg(row + j) : row[j]; };
    auto is_cand = [&](int j) { return j < c && !(f0 && j == 0) && !(fo && j == own); };
    auto bits_of = [&](float v) { return __float_as_uint(fmaxf(v, 0.f)); };
    auto key_of = [&](float v, int j) {
        return ((uint64_t)bits_of(v) << 32) | (uint32_t)(~(uint32_t)j);
    };
    int nsel = 0;  // selected non-forced blocks, their keys in buf[0, nsel)
    bool direct = false;   // positions already written by the survivor ranks
    int below_direct = 0;  // and the count of selected blocks below `own`
    if (m > 0 && ncand > m) {
        // 1. the lane's T largest candidate bit patterns, descending
        uint32_t t[4] = {0u, 0u, 0u, 0u};
        // (every load of the lane's stripe is issued before the candidate test,
        // so a batch of 16 is in flight at once; masked values count as 0)
        if (m <= 32) {
#pragma unroll 16
            for (int j = lane; j < c; j += 32) {
                const float v = load(j);
                const uint32_t kj = is_cand(j) ? bits_of(v) : 0u;
                if (kj > t[0]) { t[1] = t[0]; t[0] = kj; }
                else if (kj > t[1]) { t[1] = kj; }
            }
        } else {
#pragma unroll 16
            for (int j = lane; j < c; j += 32) {
                const float v = load(j);
                const uint32_t kj = is_cand(j) ? bits_of(v) : 0u;
                if (kj <= t[3]) continue;
                if (kj > t[0]) { t[3] = t[2]; t[2] = t[1]; t[1] = t[0]; t[0] = kj; }
                else if (kj > t[1]) { t[3] = t[2]; t[2] = t[1]; t[1] = kj; }
                else if (kj > t[2]) { t[3] = t[2]; t[2] = kj; }
                else { t[3] = kj; }
            }
        }
        // t0: the m-th largest of the 32 T values, counted with multiplicity
        // (zeros of unused slots and of lanes with fewer candidates only lower
        // it): round r takes the warp maximum and removes one copy of it, the
        // head of the lowest lane that holds it
        uint32_t t0 = 0;
        if (m <= 32) {
            for (int r = 0; r < m; ++r) {
                t0 = __reduce_max_sync(0xffffffffu, t[0]);
                const unsigned who = __ballot_sync(0xffffffffu, t[0] == t0);
                if (lane == __ffs(who) - 1) { t[0] = t[1]; t[1] = 0u; }
            }
        } else {
            for (int r = 0; r < m; ++r) {
                t0 = __reduce_max_sync(0xffffffffu, t[0]);
                const unsigned who = __ballot_sync(0xffffffffu, t[0] == t0);
                if (lane == __ffs(who) - 1) { t[0] = t[1]; t[1] = t[2]; t[2] = t[3]; t[3] = 0u; }
            }
        }
        // 2. survivors in block order
        int cnt = 0;
#pragma unroll 8
        for (int base = 0; base < c; base += 32) {
            const int j = base + lane;
            const float v = j < c ? load(j) : 0.f;
            const bool sv = is_cand(j) && bits_of(v) >= t0;
            const unsigned bal = __ballot_sync(0xffffffffu, sv);
            const int pos = cnt + __popc(bal & lt);
            if (sv && pos < kTopkBuf) buf[pos] = key_of(v, j);
            cnt += __popc(bal);
        }
        __syncwarp();
        if (cnt <= kTopkBuf) {
            // 3. rank of each survivor among the survivors (only the words that
            // hold survivors are compared); rank < m is selected
            uint64_t k4[kTopkBuf / 32];
            int r4[kTopkBuf / 32];
#pragma unroll
            for (int s = 0; s < kTopkBuf / 32; ++s) {
                k4[s] = lane + 32 * s < cnt ? buf[lane + 32 * s] : 0ull;
                r4[s] = 0;
            }
            if (cnt <= 32) {
                for (int y = 0; y < cnt; ++y) r4[0] += buf[y] > k4[0] ? 1 : 0;
            } else if (cnt <= 64) {
                for (int y = 0; y < cnt; ++y) {
                    const uint64_t ky = buf[y];
                    r4[0] += ky > k4[0] ? 1 : 0;
                    r4[1] += ky > k4[1] ? 1 : 0;
                }
            } else {
                for (int y = 0; y < cnt; ++y) {
                    const uint64_t ky = buf[y];
#pragma unroll
                    for (int s = 0; s < kTopkBuf / 32; ++s) r4[s] += ky > k4[s] ? 1 : 0;
                }
            }
            // output positions: survivors are in block order, so the selected
            // ones below a block are counted by a ballot prefix
            int base = 0;
#pragma unroll
            for (int s = 0; s < kTopkBuf / 32; ++s) {
                if (32 * s >= cnt) break;
                const bool sel = lane + 32 * s < cnt && r4[s] < m;
                const unsigned bal = __ballot_sync(0xffffffffu, sel);
                const int jx = (int)(~(uint32_t)k4[s]);
                if (sel) {
                    const int pos = (f0 ? 1 : 0) + base + __popc(bal & lt) + ((fo && jx > own) ? 1 : 0);
                    if (pos < top_k) out[pos] = jx;
                }
                below_direct += __popc(__ballot_sync(0xffffffffu, sel && fo && jx < own));
                base += __popc(bal);
            }
            direct = true;
        } else {
            // exact fallback: m rounds of a warp argmax over the keys below the
            // previous pick
            uint64_t last = ~0ull;
            for (int round = 0; round < m; ++round) {
                uint64_t best = 0;
                for (int j = lane; j < c; j += 32) {
                    if (!is_cand(j)) continue;
                    const uint64_t kk = key_of(load(j), j);
                    if (kk < last && kk > best) best = kk;
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const uint64_t other = __shfl_xor_sync(0xffffffffu, best, o);
                    if (other > best) best = other;
                }
                __syncwarp();
                if (lane == 0) buf[round] = best;
                last = best;
                __syncwarp();
            }
        }
        nsel = m;
    } else if (m > 0) {
        // every non-forced visible block is selected
        int cnt = 0;
        for (int base = 0; base < c; base += 32) {
            const int j = base + lane;
            const bool t = is_cand(j);
            const unsigned bal = __ballot_sync(0xffffffffu, t);
            const int pos = cnt + __popc(bal & lt);
            if (t && pos < kTopkBuf) buf[pos] = (uint32_t)(~(uint32_t)j);
            cnt += __popc(bal);
        }
        nsel = min(cnt, kTopkBuf);
    }
    __syncwarp();
    // 4. ascending output: block 0 (forced, visible) first; a selected block j
    // goes after the selected blocks below it and after the forced own block if
    // that is below j; the forced own block after the selected blocks below it
    int below_own = direct ? below_direct : 0;
    for (int base = 0; !direct && base < nsel; base += 32) {
        const int x = base + lane;
        int jx = 0, before = 0;
        if (x < nsel) {
            jx = (int)(~(uint32_t)buf[x]);
            for (int y = 0; y < nsel; ++y) before += (int)(~(uint32_t)buf[y]) < jx ? 1 : 0;
        }
        below_own += __popc(__ballot_sync(0xffffffffu, x < nsel && fo && jx < own));
        const int pos = (f0 ? 1 : 0) + before + ((fo && jx > own) ? 1 : 0);
        if (x < nsel && pos < top_k) out[pos] = jx;
    }
    if (lane == 0) {
        if (f0) out[0] = 0;
        if (fo) {
            const int pos = (f0 ? 1 : 0) + below_own;
            if (pos < top_k) out[pos] = own;
        }
    }
    int total = nsel + (f0 ? 1 : 0) + (fo ? 1 : 0);
    const bool extra = (force_local && own >= c) || (force_first && c == 0);
    if (extra) {
        if (lane == 0 && total < top_k) out[total] = own;
        ++total;
    }
    for (int x = total + lane; x < top_k; x += 32) out[x] = -1;
    if (total > top_k && lane == 0) report(status, VNSA_ERR_BOUNDS);
    __syncwarp();
}

}  // namespace vnsa
