// sgl_attn.h -- the tile-major pass of the selection branch: (query, tile)
// pairs of the 64-key tiles that only one or two queries of a 128-row item
// reach, grouped by tile, attended with the tile's K/V held in shared memory
// while the pairs' query rows stream through.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

#include "kernels.h"

namespace vnsa {

struct SglParams {
    CUtensorMap tm_k, tm_v;    // K (bf16) and V (fp16 copy divided by a power of two)
                               // as [n][h_kv * 128], 64 x 64 boxes
    CUtensorMap tm_kc, tm_vc;  // the same in vision order (used when the vision tokens
                               // are not one contiguous run)
    const Counts *counts;      // vision count, contiguity and first vision position
    const __nv_bfloat16 *q;  // [n][h_q][128]
    int h_q, r;              // query heads; heads per KV group (rows per pair)
    int nbt;                 // 64-key tiles per group: bucket b = group * nbt + tile
    float scale_log2;        // softmax scale * log2(e)
    const int32_t *n_items;  // number of chunks (device)
    const int4 *sorted;      // entry (chunk x, slot s) at x * (128 / r) + s: (pair id,
                             // vision rank, position, bucket); pair id -1: no pair
    const int4 *items;       // chunk c: (bucket, first entry, pairs, 0)
    __half *o;               // [pair id][r][128] normalised output in the units of the
                             // scaled V copy (fp16)
    float *lse;              // [pair id][r] log-sum-exp of the pair's keys (log2 units)
    uint32_t *status;        // device status word
    unsigned long long wait_ns;
};

// Bytes of dynamic shared memory the kernel takes (set once per device by
// sgl_prepare).
cudaError_t sgl_prepare();

// One launch over every chunk; grid = 2 CTAs per SM.
cudaError_t launch_sgl_attn(const SglParams &p, int num_sms, cudaStream_t s);

}  // namespace vnsa
