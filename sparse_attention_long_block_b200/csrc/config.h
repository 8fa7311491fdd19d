// config.h -- validation of a vnsa_config, shared by every entry point of the
// library (vnsa_create / vnsa_workspace_bytes and vnsa_select_noalloc), so that
// they accept the same layers and reject the rest with the same codes.
#pragma once

#include <math.h>

#include "../../include/vnsa.h"

namespace vnsa {

constexpr int kMaxTokens = 262144;  // tokens per call (n_max, or n without a handle)

// The compression stride of a config (0 stands for the block size).
inline int cmp_stride_of(const vnsa_config &c) { return c.cmp_stride > 0 ? c.cmp_stride : c.block; }

// Compression blocks over n vision tokens: [c*s, c*s + block) for c < this.
inline int cmp_blocks(int n, int block, int stride) {
    return n >= block ? (n - block) / stride + 1 : 0;
}

// Argument errors (VNSA_ERR_INVALID_ARG) first, then layers that are valid
// but not implemented (VNSA_ERR_UNSUPPORTED).  `n` is the token count the
// workspace is sized for: cfg->n_max for a handle, the call's n otherwise.
inline vnsa_status check_config(const vnsa_config *c, int n) {
    if (!c) return VNSA_ERR_INVALID_ARG;
    if (n < 1 || c->h_q < 1 || c->h_kv < 1 || c->d < 1) return VNSA_ERR_INVALID_ARG;
    if (c->h_q % c->h_kv != 0) return VNSA_ERR_INVALID_ARG;
    if (c->top_k < 1 || c->window < 1 || c->block < 1) return VNSA_ERR_INVALID_ARG;
    if ((c->force_first != 0 && c->force_first != 1) ||
        (c->force_local != 0 && c->force_local != 1))
        return VNSA_ERR_INVALID_ARG;
    if (c->top_k < c->force_first + c->force_local) return VNSA_ERR_INVALID_ARG;
    if (c->cmp_stride < 0 || c->cmp_stride > c->block) return VNSA_ERR_INVALID_ARG;
    if (!(c->scale >= 0.f) || isinf(c->scale)) return VNSA_ERR_INVALID_ARG;
    if (c->dtype != VNSA_BF16 && c->dtype != VNSA_FP32) return VNSA_ERR_INVALID_ARG;
    if (n > kMaxTokens) return VNSA_ERR_UNSUPPORTED;
    if (c->d != 64 && c->d != 128) return VNSA_ERR_UNSUPPORTED;
    if (c->h_q / c->h_kv > 16) return VNSA_ERR_UNSUPPORTED;
    if (c->top_k > 64) return VNSA_ERR_UNSUPPORTED;
    return VNSA_OK;
}

}  // namespace vnsa
