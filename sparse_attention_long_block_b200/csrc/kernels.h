// kernels.h -- host-side launchers of the vnsa kernels (internal to libvnsa.so).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace vnsa {

// Everything one forward needs, passed by value to the kernels.
struct LayerParams {
    int n, n_max, h_q, h_kv, d, r, block, top_k, window, force_first, force_local;
    int stride;                       // compression stride (block: no overlap)
    int nb_max;                       // capacity in compression blocks (K_cmp, imp rows)
    float scale_log2;                 // softmax scale * log2(e)
    const void *q, *k, *v;            // [n][h][d] dtype
    const uint8_t *is_vision;         // [n]
    const float *gate;                // [n][h_q][3]
    void *out;                        // [n][h_q][d] dtype
    const int32_t *vis, *txt;         // vision / text positions by rank
    const Counts *counts;
    uint32_t *status;
    const void *k_cmp, *v_cmp;        // [nb][h_kv][d] dtype
    float *lse;                       // [n_max][h_q] natural-log LSE of compression
    float *imp;                       // [h_kv][n_max][imp_stride] compression-block importance
    size_t imp_stride;
    float *imp_sel;                   // [h_kv][n_max][imp_sel_stride] selection-block
    size_t imp_sel_stride;            // importance (top-k input); = imp at stride block
    int32_t *idx;                     // [h_kv][n_max][top_k] (workspace)
    const int32_t *idx_src;           // selection read by the selection branch
    size_t idx_rows;                  // rows per group of idx_src
    float *o_cmp_ws;                  // [n_max][h_q][d] fp32 ungated compression output
    float *dbg_o_cmp, *dbg_o_slc, *dbg_o_swa;  // optional [n][h_q][d] exports
    unsigned long long wait_ns;       // limit of the kernels' bounded waits (0: default)
};

cudaError_t launch_partition(const uint8_t *is_vision, int n, int block, int stride,
                             int32_t *vis, int32_t *txt, Counts *counts, cudaStream_t s);

// The compression branch's perceptron (when hidden > 0): K_cmp = SiLU(mean .
// w1 + b1) . w2 + b2, w1 [d][hidden], w2 [hidden][d] in the layer dtype, b1, b2
// fp32; index 0 for K, 1 for V.  hidden == 0: the linear projection W_K, W_V.
constexpr int kCmpMlpMaxHidden = 512;
struct CmpMlp {
    int hidden;
    const void *w1[2], *w2[2];
    const float *b1[2], *b2[2];
};

// K_cmp / V_cmp: dtype 0 = bf16, 1 = fp32.
cudaError_t launch_pool_proj(int dtype, int d, const void *k, const void *v,
                             const int32_t *vis, const Counts *counts, const void *w_k,
                             const void *w_v, void *k_cmp, void *v_cmp, int h_kv, int block,
                             int stride, int nb_max, cudaStream_t s, int from_pad = 0,
                             const CmpMlp *mlp = nullptr);

// Gate logits [n][n_out] fp32 of the layer input x [n][dm] through the gate
// perceptron SiLU(x . g1 + c1) . g2 + c2 (g1 [dm][hidden], g2 [hidden][n_out]
// in the layer dtype, c1, c2 fp32); in bf16 the hidden activations are rounded
// to bf16.  `status` receives device-detected errors.
cudaError_t launch_gate_mlp(int dtype, int n, int dm, int hidden, int n_out, const void *x,
                            const void *g1, const float *c1, const void *g2, const float *c2,
                            float *out, uint32_t *status, cudaStream_t s, int *launches);

cudaError_t launch_topk(const LayerParams &p, cudaStream_t s);

// Selection-block importance (imp_sel) from the compression-block importance
// (imp) when the compression blocks overlap (stride < block).
cudaError_t launch_imp_remap(const LayerParams &p, cudaStream_t s);

// Copies of workspace tensors into the optional debug buffers of vnsa_debug.
cudaError_t launch_export(const LayerParams &p, int esize, float *lse_out, int32_t *idx_out,
                          float *imp_out, size_t imp_stride_out, void *kc_out, void *vc_out,
                          cudaStream_t s);

// SIMT attention (fp32 path; also the bf16 path where no tensor-core kernel
// is wired in).
cudaError_t launch_cmp_simt(int dtype, const LayerParams &p, cudaStream_t s);
cudaError_t launch_vision_simt(int dtype, const LayerParams &p, cudaStream_t s);
cudaError_t launch_text_simt(int dtype, const LayerParams &p, cudaStream_t s);

}  // namespace vnsa
