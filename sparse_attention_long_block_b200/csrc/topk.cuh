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
// key is the block the rule prefers (keys are unique).  Pass 1 (float4 loads
// of the importance row) keeps each lane's two largest candidate bit
// patterns; the m-th largest of those 64 values cannot exceed the m-th
// largest candidate, so only candidates at or above it can be selected.
// Pass 2 re-reads the row (now in cache) and collects those survivors; if at
// most 128 survive they are sorted (bitonic, in shared memory) and the first
// m taken, otherwise m rounds of a warp argmax over keys below the previous
// pick select them exactly.  Shared memory is 1 KB per warp.
__device__ __forceinline__ void warp_sort_desc(uint64_t *v, int n, int lane) {
    // bitonic sort of n (power of two, <= 256) keys in shared memory, descending
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            for (int t = lane; t < n / 2; t += 32) {
                const int lo = 2 * t - (t & (stride - 1));
                const int hi = lo + stride;
                const bool desc = ((lo & size) == 0);
                const uint64_t a = v[lo], b = v[hi];
                if ((a < b) == desc) {
                    v[lo] = b;
                    v[hi] = a;
                }
            }
            __syncwarp();
        }
    }
}

constexpr int kTopkBuf = 128;  // survivors sorted in shared memory, per warp

// The selection of one (group, query) row by one warp.  row: the query's
// importance over its c visible blocks (16-byte aligned; global memory when
// kGlobal, else shared memory); own: the query's own block; buf: 128 keys of
// warp scratch in shared memory; out: top_k entries, ascending, -1 padded.
template <bool kGlobal>
__device__ __forceinline__ void topk_select_row(const float *row, int c, int own, int top_k, int force_first,
                                int force_local, uint64_t *buf, int lane, int32_t *out,
                                uint32_t *status) {
    const bool f0 = force_first && c > 0;
    const bool fo = force_local && own < c && !(f0 && own == 0);
    const int nforced =
        (force_first ? 1 : 0) + ((force_local && !(force_first && own == 0)) ? 1 : 0);
    const int m = top_k - nforced;
    const int ncand = c - (f0 ? 1 : 0) - (fo ? 1 : 0);
    const float4 *row4 = reinterpret_cast<const float4 *>(row);
    const int c4 = (c + 3) / 4;
    auto load4 = [&](int q) { return kGlobal ? __ldg(row4 + q) : row4[q]; };
    auto is_cand = [&](int j) { return j < c && !(f0 && j == 0) && !(fo && j == own); };
    auto key_of = [&](float v, int j) {
        return ((uint64_t)__float_as_uint(fmaxf(v, 0.f)) << 32) | (uint32_t)(~(uint32_t)j);
    };
    int sel = 0;  // selected non-forced blocks, their keys in buf[0, sel)
    if (m > 0 && ncand > m) {
        uint32_t t1 = 0, t2 = 0;  // the lane's two largest candidate bit patterns
#pragma unroll 4
        for (int q = lane; q < c4; q += 32) {
            const float4 v4 = load4(q);
            const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (!is_cand(4 * q + e)) continue;
                const uint32_t kj = __float_as_uint(fmaxf(vv[e], 0.f));
                if (kj > t1) { t2 = t1; t1 = kj; }
                else if (kj > t2) { t2 = kj; }
            }
        }
        // lower bound t0 of the m-th largest candidate value
        buf[lane] = t1;
        buf[lane + 32] = t2;
        __syncwarp();
        warp_sort_desc(buf, 64, lane);
        const uint32_t t0 = (uint32_t)buf[min(m, 64) - 1];
        __syncwarp();
        // survivors: candidates with bits >= t0
        int cnt = 0;
#pragma unroll 2
        for (int base = 0; base < c4; base += 32) {
            const int q = base + lane;
            float vv[4] = {0.f, 0.f, 0.f, 0.f};
            if (q < c4) {
                const float4 v4 = load4(q);
                vv[0] = v4.x; vv[1] = v4.y; vv[2] = v4.z; vv[3] = v4.w;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = 4 * q + e;
                const bool sv = q < c4 && is_cand(j) && __float_as_uint(fmaxf(vv[e], 0.f)) >= t0;
                const unsigned bal = __ballot_sync(0xffffffffu, sv);
                const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
                if (sv && pos < kTopkBuf) buf[pos] = key_of(vv[e], j);
                cnt += __popc(bal);
            }
        }
        __syncwarp();
        if (cnt <= kTopkBuf) {
            int n2 = 32;
            while (n2 < cnt) n2 <<= 1;
            for (int x = cnt + lane; x < n2; x += 32) buf[x] = 0ull;  // smallest keys
            __syncwarp();
            warp_sort_desc(buf, n2, lane);
        } else {
            // exact fallback: m rounds of a warp argmax over the keys below the
            // previous pick
            uint64_t last = ~0ull;
            for (int round = 0; round < m; ++round) {
                uint64_t best = 0;
                for (int q = lane; q < c4; q += 32) {
                    const float4 v4 = load4(q);
                    const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 4 * q + e;
                        if (!is_cand(j)) continue;
                        const uint64_t kk = key_of(vv[e], j);
                        if (kk < last && kk > best) best = kk;
                    }
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
        sel = m;
    } else if (m > 0) {
        // every non-forced visible block is selected
        int cnt = 0;
        for (int base = 0; base < c; base += 32) {
            const int j = base + lane;
            const bool t = is_cand(j);
            const unsigned bal = __ballot_sync(0xffffffffu, t);
            const int pos = cnt + __popc(bal & ((1u << lane) - 1u));
            if (t && pos < kTopkBuf) buf[pos] = (uint32_t)(~(uint32_t)j);
            cnt += __popc(bal);
        }
        sel = min(cnt, kTopkBuf);
    }
    __syncwarp();
    // ascending output: the picks and the visible forced blocks sorted by
    // index (keys ~j, descending), then the own block when it is forced but
    // not yet complete (it is above every visible one)
    for (int x = lane; x < sel; x += 32) buf[x] = (uint32_t)buf[x];
    __syncwarp();
    int total = sel;
    if (lane == 0) {
        if (f0) buf[total] = (uint32_t)(~0u);
        if (fo) buf[total + (f0 ? 1 : 0)] = (uint32_t)(~(uint32_t)own);
    }
    total += (f0 ? 1 : 0) + (fo ? 1 : 0);
    int n2 = 32;
    while (n2 < total) n2 <<= 1;
    __syncwarp();
    for (int x = total + lane; x < n2; x += 32) buf[x] = 0ull;
    __syncwarp();
    warp_sort_desc(buf, n2, lane);
    for (int x = lane; x < total && x < top_k; x += 32) out[x] = (int)(~(uint32_t)buf[x]);
    int cnt = total;
    const bool extra = (force_local && own >= c) || (force_first && c == 0);
    if (extra) {
        if (lane == 0 && cnt < top_k) out[cnt] = own;
        ++cnt;
    }
    for (int x = cnt + lane; x < top_k; x += 32) out[x] = -1;
    if (cnt > top_k && lane == 0) report(status, VNSA_ERR_BOUNDS);
}


}  // namespace vnsa
