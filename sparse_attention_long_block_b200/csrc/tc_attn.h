// tc_attn.h -- tensor-core (tcgen05 / TMEM / TMA) attention path of the bf16
// layer prefill, behind the C ABI of vnsa_api.cu.
#pragma once

#include <cuda.h>

#include "kernels.h"

namespace vnsa {

struct TcState;

// True if the bf16 tensor-core path handles this configuration.
bool tc_supported(const vnsa_config &c);

// Extra workspace bytes the tensor-core path needs for n_max tokens.
size_t tc_workspace_bytes(const vnsa_config &c);

// Set up the path (tensor maps are rebuilt per forward); ws is its workspace.
cudaError_t tc_create(const vnsa_config &c, void *ws, TcState **out);

// Compression, top-k, selection, window + gate, text: enqueued on s.  `ev`
// (nullable) holds the per-stage timing events (begin, end) of vnsa_api.cu;
// `ran` marks the stages that ran; `launches` counts kernel launches.
cudaError_t tc_forward(TcState *st, const LayerParams &p, cudaStream_t s, cudaEvent_t *ev,
                       int *ran, int *launches, bool forced);

void tc_destroy(TcState *st);

// 2-D TMA map over a row-major bf16 matrix [rows][inner] (row stride inner * 2
// bytes, a multiple of 16) with boxes of box_inner x box_rows elements and the
// 128-byte swizzle (box_inner * 2 must be 128).  False if the driver entry
// point is missing or the encoding fails.
bool tma_map_2d_bf16(CUtensorMap *m, const void *base, long long inner, long long rows,
                     int box_inner, int box_rows);

}  // namespace vnsa
