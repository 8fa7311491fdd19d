// decode.h -- the decode step's parameters and launcher (internal to libvnsa.so).
#pragma once

#include "kernels.h"

namespace vnsa {

constexpr int kSplit = 37;  // CTAs per KV group in the split-K decode kernels

struct DecodeParams {
    int n;                        // tokens in the stream, the new one at n - 1
    int h_q, h_kv, d, r, block, top_k, window, force_first, force_local, nb_max;
    float scale_log2;             // softmax scale * log2(e)
    const void *q;                // [h_q][d] the new token's query
    const void *k, *v;            // [n][h_kv][d] the whole stream (the cache)
    const uint8_t *is_vision;     // [n]
    const float *gate;            // [h_q][3] the new token's gate logits
    void *out;                    // [h_q][d] the new token's output row
    int32_t *vis, *txt;           // position lists (workspace, extended by one)
    Counts *counts;               // workspace counts (updated)
    uint32_t *status;
    void *k_cmp, *v_cmp;          // [nb_max][h_kv][d] block keys/values (extended)
    const void *w_k, *w_v;        // [d][d] projections
    CmpMlp mlp;                   // compression perceptron (hidden 0: the projections)
    float *s_cmp;                 // [h_kv][r][nb_max] compression scores (log2 units)
    float *part;                  // [3][h_kv][kSplit][r][d + 2] split softmax states
    int32_t *sel;                 // [h_kv][top_k] the selection
    int32_t *sel_out;             // optional export [h_kv][top_k]
};

size_t decode_workspace_bytes(int h_kv, int r, int d, int nb_max);

cudaError_t launch_decode(int dtype, const DecodeParams &p, cudaStream_t s, int *launches);

}  // namespace vnsa
