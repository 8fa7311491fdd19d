// vnsa_api.cu -- the C ABI declared in include/vnsa.h: argument validation,
// workspace ownership, and the launch sequence of one layer prefill.
//
// One forward enqueues, on the caller's stream and without host syncs:
//   partition -> pool+projection -> compression attention (+ importance)
//   -> top-k -> vision branches + gate -> text GQA.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <new>

#include "config.h"
#include "decode.h"
#include "kernels.h"
#include "tc_attn.h"

using namespace vnsa;

namespace {

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Layout {
    size_t vis, txt, counts, status, w_k, w_v, k_cmp, v_cmp, lse, imp, imp_sel, idx, o_cmp, tc,
        dec, dec_sel;
    size_t total;
    size_t imp_stride, imp_sel_stride;
};

Layout make_layout(const vnsa_config &c) {
    const size_t es = c.dtype == VNSA_BF16 ? 2 : 4;
    const size_t n = (size_t)c.n_max;
    const size_t nb = (size_t)(c.n_max / c.block);  // selection blocks
    const int stride = cmp_stride_of(c);
    const size_t nc = (size_t)cmp_blocks(c.n_max, c.block, stride);  // compression blocks
    Layout L;
    L.imp_stride = nc > 0 ? (nc + 3) / 4 * 4 : 4;
    L.imp_sel_stride = nb > 0 ? (nb + 3) / 4 * 4 : 4;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off += align_up(bytes > 0 ? bytes : 1); return o; };
    L.vis = take(n * 4);
    L.txt = take(n * 4);
    L.counts = take(sizeof(Counts));
    L.status = take(16);
    L.w_k = take((size_t)c.d * c.d * es);
    L.w_v = take((size_t)c.d * c.d * es);
    L.k_cmp = take(nc * c.h_kv * c.d * es);
    L.v_cmp = take(nc * c.h_kv * c.d * es);
    L.lse = take(n * c.h_q * 4);
    L.imp = take((size_t)c.h_kv * n * L.imp_stride * 4);
    // the selection-block importance has a buffer of its own only when the
    // compression blocks overlap
    L.imp_sel = stride != c.block ? take((size_t)c.h_kv * n * L.imp_sel_stride * 4) : L.imp;
    L.idx = take((size_t)c.h_kv * n * c.top_k * 4);
    L.o_cmp = take(n * c.h_q * c.d * 4);
    L.tc = take(tc_workspace_bytes(c));
    L.dec = take(decode_workspace_bytes(c.h_kv, c.h_q / c.h_kv, c.d, (int)nb));
    L.dec_sel = take((size_t)c.h_kv * c.top_k * 4);
    L.total = off;
    return L;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Streamed host calls (vnsa_forward_host_async): two device staging slots,
// one copy stream per direction, and per slot the events that order them.
// Call t uses slot t & 1.  Its input copies wait until the attention of call
// t - 2 (the slot's previous user) has run; its attention waits for its input
// copies and for the output copy of call t - 2; its output copy waits for its
// attention.  So while call t computes, the inputs of call t + 1 and the output
// of call t - 1 cross the bus.
struct HostPipe {
    char *mem;
    size_t slot_bytes;
    cudaStream_t h2d, d2h;
    cudaEvent_t in_done[2], comp_done[2], out_done[2];
    unsigned long long next;  // tickets issued so far
};

void host_pipe_free(HostPipe *p) {
    if (!p) return;
    if (p->h2d) cudaStreamSynchronize(p->h2d);
    if (p->d2h) cudaStreamSynchronize(p->d2h);
    for (int s = 0; s < 2; ++s) {
        if (p->in_done[s]) cudaEventDestroy(p->in_done[s]);
        if (p->comp_done[s]) cudaEventDestroy(p->comp_done[s]);
        if (p->out_done[s]) cudaEventDestroy(p->out_done[s]);
    }
    if (p->h2d) cudaStreamDestroy(p->h2d);
    if (p->d2h) cudaStreamDestroy(p->d2h);
    if (p->mem) cudaFree(p->mem);
    delete p;
}

}  // namespace

struct vnsa_handle {
    vnsa_config cfg;
    int device;
    int r, nb_max;
    size_t esize;
    Layout L;
    char *ws;
    Counts *counts;
    uint32_t *status;
    char *stage;  // staging buffers of vnsa_forward_host (allocated on first use)
    size_t stage_bytes;
    TcState *tc;
    int timing;
    long long stream_n;  // tokens the last forward / decode step processed (-1: none)
    cudaEvent_t ev[2 * VNSA_NUM_STAGES];
    int ran[VNSA_NUM_STAGES];
    int launches;
    CmpMlp mlp;     // compression perceptron (hidden 0: the linear W_K, W_V)
    char *mlp_mem;  // its weights (owned)
    HostPipe *pipe; // streamed host calls (created on first use)
    unsigned long long wait_ns;  // limit of the kernels' bounded waits (0: default)
};

extern "C" {

const char *vnsa_status_string(vnsa_status s) {
    switch (s) {
        case VNSA_OK: return "ok";
        case VNSA_ERR_INVALID_ARG: return "invalid argument";
        case VNSA_ERR_UNSUPPORTED: return "unsupported configuration";
        case VNSA_ERR_CUDA: return "CUDA error";
        case VNSA_ERR_TIMEOUT: return "device wait timed out";
        case VNSA_ERR_BOUNDS: return "device index out of bounds";
        case VNSA_ERR_NO_DEVICE: return "no CUDA device";
    }
    return "unknown status";
}

const char *vnsa_stage_name(int stage) {
    static const char *names[VNSA_NUM_STAGES] = {"partition", "pool", "cmp", "topk",
                                                 "slc", "swa", "text"};
    if (stage < 0 || stage >= VNSA_NUM_STAGES) return nullptr;
    return names[stage];
}

vnsa_status vnsa_workspace_bytes(const vnsa_config *cfg, size_t *bytes) {
    if (!bytes) return VNSA_ERR_INVALID_ARG;
    vnsa_status st = check_config(cfg, cfg ? cfg->n_max : 0);
    if (st != VNSA_OK) return st;
    *bytes = make_layout(*cfg).total;
    return VNSA_OK;
}

vnsa_status vnsa_create(const vnsa_config *cfg, const void *w_k, const void *w_v,
                        vnsa_handle **out) {
    if (!out) return VNSA_ERR_INVALID_ARG;
    *out = nullptr;
    vnsa_status st = check_config(cfg, cfg ? cfg->n_max : 0);
    if (st != VNSA_OK) return st;
    if (!w_k || !w_v || !aligned16(w_k) || !aligned16(w_v)) return VNSA_ERR_INVALID_ARG;
    int ndev = 0;
    if (cudaGetDeviceCount(&ndev) != cudaSuccess || ndev == 0) {
        cudaGetLastError();
        return VNSA_ERR_NO_DEVICE;
    }
    vnsa_handle *h = new (std::nothrow) vnsa_handle();
    if (!h) return VNSA_ERR_CUDA;
    h->cfg = *cfg;
    if (h->cfg.scale == 0.f) h->cfg.scale = 1.0f / sqrtf((float)cfg->d);
    cudaGetDevice(&h->device);
    h->r = cfg->h_q / cfg->h_kv;
    h->stream_n = -1;
    h->nb_max = cmp_blocks(cfg->n_max, cfg->block, cmp_stride_of(*cfg));
    h->esize = cfg->dtype == VNSA_BF16 ? 2 : 4;
    h->L = make_layout(h->cfg);
    if (cudaMalloc(&h->ws, h->L.total) != cudaSuccess) {
        cudaGetLastError();
        delete h;
        return VNSA_ERR_CUDA;
    }
    h->counts = (Counts *)(h->ws + h->L.counts);
    h->status = (uint32_t *)(h->ws + h->L.status);
    const size_t wbytes = (size_t)cfg->d * cfg->d * h->esize;
    bool ok = cudaMemset(h->ws + h->L.status, 0, 16) == cudaSuccess &&
              cudaMemset(h->ws + h->L.counts, 0, sizeof(Counts)) == cudaSuccess &&
              cudaMemcpy(h->ws + h->L.w_k, w_k, wbytes, cudaMemcpyDefault) == cudaSuccess &&
              cudaMemcpy(h->ws + h->L.w_v, w_v, wbytes, cudaMemcpyDefault) == cudaSuccess;
    if (ok) ok = tc_create(h->cfg, h->ws + h->L.tc, &h->tc) == cudaSuccess;
    for (int e = 0; ok && e < 2 * VNSA_NUM_STAGES; ++e)
        ok = cudaEventCreate(&h->ev[e]) == cudaSuccess;
    if (!ok) {
        cudaGetLastError();
        vnsa_destroy(h);
        return VNSA_ERR_CUDA;
    }
    *out = h;
    return VNSA_OK;
}

vnsa_status vnsa_forward(vnsa_handle *h, int n, const void *q, const void *k, const void *v,
                         const uint8_t *is_vision, const float *gate_logits, void *out,
                         const vnsa_debug *dbg, void *stream) {
    if (!h || !q || !k || !v || !is_vision || !gate_logits || !out) return VNSA_ERR_INVALID_ARG;
    if (n < 1 || n > h->cfg.n_max) return VNSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        !aligned16(gate_logits))
        return VNSA_ERR_INVALID_ARG;
    if (dbg && dbg->imp && dbg->imp_stride < n / h->cfg.block) return VNSA_ERR_INVALID_ARG;
    const vnsa_config &c = h->cfg;
    cudaStream_t s = (cudaStream_t)stream;
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess) return VNSA_ERR_CUDA;

    LayerParams p;
    memset(&p, 0, sizeof(p));
    p.n = n;
    p.n_max = c.n_max;
    p.h_q = c.h_q;
    p.h_kv = c.h_kv;
    p.d = c.d;
    p.r = h->r;
    p.block = c.block;
    p.stride = cmp_stride_of(c);
    p.top_k = c.top_k;
    p.window = c.window;
    p.force_first = c.force_first;
    p.force_local = c.force_local;
    p.nb_max = h->nb_max;
    p.scale_log2 = c.scale * kLog2e;
    p.q = q;
    p.k = k;
    p.v = v;
    p.is_vision = is_vision;
    p.gate = gate_logits;
    p.out = out;
    p.vis = (const int32_t *)(h->ws + h->L.vis);
    p.txt = (const int32_t *)(h->ws + h->L.txt);
    p.counts = h->counts;
    p.status = h->status;
    p.k_cmp = h->ws + h->L.k_cmp;
    p.v_cmp = h->ws + h->L.v_cmp;
    p.lse = (float *)(h->ws + h->L.lse);
    p.imp = (float *)(h->ws + h->L.imp);
    p.imp_stride = h->L.imp_stride;
    p.imp_sel = (float *)(h->ws + h->L.imp_sel);
    p.imp_sel_stride = h->L.imp_sel == h->L.imp ? h->L.imp_stride : h->L.imp_sel_stride;
    p.idx = (int32_t *)(h->ws + h->L.idx);
    p.idx_src = p.idx;
    p.idx_rows = (size_t)c.n_max;
    p.o_cmp_ws = (float *)(h->ws + h->L.o_cmp);
    p.wait_ns = h->wait_ns;
    const bool forced = dbg && dbg->forced_idx;
    if (forced) {
        p.idx_src = dbg->forced_idx;
        p.idx_rows = (size_t)n;  // caller layout [h_kv][n][top_k]
    }
    if (dbg) {
        p.dbg_o_cmp = dbg->o_cmp;
        p.dbg_o_slc = dbg->o_slc;
        p.dbg_o_swa = dbg->o_swa;
    }

    const int dt = (int)c.dtype;
    const bool use_tc = tc_supported(c);
    h->launches = 0;
    for (int x = 0; x < VNSA_NUM_STAGES; ++x) h->ran[x] = 0;
    cudaError_t e = cudaSuccess;
    auto begin = [&](int stg) {
        if (h->timing) cudaEventRecord(h->ev[2 * stg], s);
        h->ran[stg] = 1;
    };
    auto end = [&](int stg) {
        if (h->timing) cudaEventRecord(h->ev[2 * stg + 1], s);
    };
#define VNSA_RUN(call)                                \
    do {                                              \
        if (e == cudaSuccess) {                       \
            e = (call);                               \
            ++h->launches;                            \
        }                                             \
    } while (0)

    begin(VNSA_STAGE_PARTITION);
    VNSA_RUN(launch_partition(is_vision, n, c.block, p.stride, (int32_t *)p.vis,
                              (int32_t *)p.txt, h->counts, s));
    end(VNSA_STAGE_PARTITION);
    begin(VNSA_STAGE_POOL);
    VNSA_RUN(launch_pool_proj(dt, c.d, k, v, p.vis, h->counts, h->ws + h->L.w_k,
                              h->ws + h->L.w_v, (void *)p.k_cmp, (void *)p.v_cmp, c.h_kv,
                              c.block, p.stride, h->nb_max, s, 0, &h->mlp));
    end(VNSA_STAGE_POOL);
    if (use_tc) {
        // counts its own launches
        if (e == cudaSuccess)
            e = tc_forward(h->tc, p, s, h->timing ? h->ev : nullptr, h->ran, &h->launches, forced);
    } else {
        begin(VNSA_STAGE_CMP);
        VNSA_RUN(launch_cmp_simt(dt, p, s));
        end(VNSA_STAGE_CMP);
        begin(VNSA_STAGE_TOPK);
        if (p.stride != p.block) VNSA_RUN(launch_imp_remap(p, s));
        if (!forced) VNSA_RUN(launch_topk(p, s));
        end(VNSA_STAGE_TOPK);
        begin(VNSA_STAGE_SWA);
        VNSA_RUN(launch_vision_simt(dt, p, s));
        end(VNSA_STAGE_SWA);
        begin(VNSA_STAGE_TEXT);
        VNSA_RUN(launch_text_simt(dt, p, s));
        end(VNSA_STAGE_TEXT);
    }
    if (dbg && (dbg->lse_cmp || dbg->idx || dbg->imp || dbg->k_cmp || dbg->v_cmp))
        VNSA_RUN(launch_export(p, (int)h->esize, dbg->lse_cmp, dbg->idx, dbg->imp,
                               (size_t)dbg->imp_stride, dbg->k_cmp, dbg->v_cmp, s));
#undef VNSA_RUN
    if (cur != h->device && cur >= 0) cudaSetDevice(cur);
    if (e != cudaSuccess) {
        fprintf(stderr, "vnsa_forward: %s\n", cudaGetErrorString(e));
        h->stream_n = -1;
        return VNSA_ERR_CUDA;
    }
    h->stream_n = n;
    return VNSA_OK;
}

vnsa_status vnsa_decode(vnsa_handle *h, int n, const void *q_new, const void *k, const void *v,
                        const uint8_t *is_vision, const float *gate_new, void *out_new,
                        int32_t *sel_out, void *stream) {
    if (!h || !q_new || !k || !v || !is_vision || !gate_new || !out_new)
        return VNSA_ERR_INVALID_ARG;
    if (n < 2 || n > h->cfg.n_max || h->stream_n != (long long)n - 1) return VNSA_ERR_INVALID_ARG;
    if (cmp_stride_of(h->cfg) != h->cfg.block) return VNSA_ERR_UNSUPPORTED;
    if (!aligned16(q_new) || !aligned16(k) || !aligned16(v) || !aligned16(out_new) ||
        !aligned16(gate_new) || (sel_out && !aligned16(sel_out)))
        return VNSA_ERR_INVALID_ARG;
    const vnsa_config &c = h->cfg;
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess) return VNSA_ERR_CUDA;
    DecodeParams p;
    memset(&p, 0, sizeof(p));
    p.n = n;
    p.h_q = c.h_q;
    p.h_kv = c.h_kv;
    p.d = c.d;
    p.r = h->r;
    p.block = c.block;
    p.top_k = c.top_k;
    p.window = c.window;
    p.force_first = c.force_first;
    p.force_local = c.force_local;
    p.nb_max = h->nb_max;
    p.scale_log2 = c.scale * kLog2e;
    p.q = q_new;
    p.k = k;
    p.v = v;
    p.is_vision = is_vision;
    p.gate = gate_new;
    p.out = out_new;
    p.vis = (int32_t *)(h->ws + h->L.vis);
    p.txt = (int32_t *)(h->ws + h->L.txt);
    p.counts = h->counts;
    p.status = h->status;
    p.k_cmp = h->ws + h->L.k_cmp;
    p.v_cmp = h->ws + h->L.v_cmp;
    p.w_k = h->ws + h->L.w_k;
    p.w_v = h->ws + h->L.w_v;
    p.mlp = h->mlp;
    char *dec = h->ws + h->L.dec;
    p.s_cmp = (float *)dec;
    p.part = (float *)(dec + (size_t)c.h_kv * h->r * (h->nb_max > 0 ? h->nb_max : 1) * 4);
    p.sel = (int32_t *)(h->ws + h->L.dec_sel);
    p.sel_out = sel_out;
    h->launches = 0;
    for (int x = 0; x < VNSA_NUM_STAGES; ++x) h->ran[x] = 0;
    const cudaError_t e = launch_decode((int)c.dtype, p, (cudaStream_t)stream, &h->launches);
    if (cur != h->device && cur >= 0) cudaSetDevice(cur);
    if (e != cudaSuccess) {
        fprintf(stderr, "vnsa_decode: %s\n", cudaGetErrorString(e));
        h->stream_n = -1;
        return VNSA_ERR_CUDA;
    }
    h->stream_n = n;
    return VNSA_OK;
}

vnsa_status vnsa_forward_host(vnsa_handle *h, int n, const void *q, const void *k,
                              const void *v, const uint8_t *is_vision,
                              const float *gate_logits, void *out, void *stream) {
    if (!h || !q || !k || !v || !is_vision || !gate_logits || !out) return VNSA_ERR_INVALID_ARG;
    if (n < 1 || n > h->cfg.n_max) return VNSA_ERR_INVALID_ARG;
    const vnsa_config &c = h->cfg;
    const size_t nm = (size_t)c.n_max;
    const size_t bq = align_up(nm * c.h_q * c.d * h->esize);
    const size_t bk = align_up(nm * c.h_kv * c.d * h->esize);
    const size_t bg = align_up(nm * c.h_q * 3 * 4);
    const size_t bi = align_up(nm);
    const size_t need = 2 * bq + 2 * bk + bg + bi;
    if (!h->stage) {
        if (cudaMalloc(&h->stage, need) != cudaSuccess) {
            cudaGetLastError();
            h->stage = nullptr;
            return VNSA_ERR_CUDA;
        }
        h->stage_bytes = need;
    }
    char *dq = h->stage, *dk = dq + bq, *dv = dk + bk, *dg = dv + bk, *di = dg + bg,
         *dout = di + bi;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t nq = (size_t)n * c.h_q * c.d * h->esize;
    const size_t nk = (size_t)n * c.h_kv * c.d * h->esize;
    bool ok = cudaMemcpyAsync(dq, q, nq, cudaMemcpyHostToDevice, s) == cudaSuccess &&
              cudaMemcpyAsync(dk, k, nk, cudaMemcpyHostToDevice, s) == cudaSuccess &&
              cudaMemcpyAsync(dv, v, nk, cudaMemcpyHostToDevice, s) == cudaSuccess &&
              cudaMemcpyAsync(dg, gate_logits, (size_t)n * c.h_q * 3 * 4,
                              cudaMemcpyHostToDevice, s) == cudaSuccess &&
              cudaMemcpyAsync(di, is_vision, (size_t)n, cudaMemcpyHostToDevice, s) ==
                  cudaSuccess;
    if (!ok) {
        cudaGetLastError();
        return VNSA_ERR_CUDA;
    }
    vnsa_status st = vnsa_forward(h, n, dq, dk, dv, (const uint8_t *)di, (const float *)dg,
                                  dout, nullptr, stream);
    if (st != VNSA_OK) return st;
    if (cudaMemcpyAsync(out, dout, nq, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return VNSA_ERR_CUDA;
    }
    return VNSA_OK;
}

vnsa_status vnsa_forward_host_async(vnsa_handle *h, int n, const void *q, const void *k,
                                    const void *v, const uint8_t *is_vision,
                                    const float *gate_logits, void *out, void *stream,
                                    unsigned long long *ticket) {
    if (!h || !q || !k || !v || !is_vision || !gate_logits || !out || !ticket)
        return VNSA_ERR_INVALID_ARG;
    if (n < 1 || n > h->cfg.n_max) return VNSA_ERR_INVALID_ARG;
    const vnsa_config &c = h->cfg;
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess) return VNSA_ERR_CUDA;
    const size_t nm = (size_t)c.n_max;
    const size_t bq = align_up(nm * c.h_q * c.d * h->esize);
    const size_t bk = align_up(nm * c.h_kv * c.d * h->esize);
    const size_t bg = align_up(nm * c.h_q * 3 * 4);
    const size_t bi = align_up(nm);
    if (!h->pipe) {
        HostPipe *p = new (std::nothrow) HostPipe();
        if (!p) return VNSA_ERR_CUDA;
        p->slot_bytes = 2 * bq + 2 * bk + bg + bi;
        bool ok = cudaMalloc(&p->mem, 2 * p->slot_bytes) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&p->h2d, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaStreamCreateWithFlags(&p->d2h, cudaStreamNonBlocking) == cudaSuccess;
        for (int s = 0; ok && s < 2; ++s)
            ok = cudaEventCreateWithFlags(&p->in_done[s], cudaEventDisableTiming) == cudaSuccess &&
                 cudaEventCreateWithFlags(&p->comp_done[s], cudaEventDisableTiming) ==
                     cudaSuccess &&
                 cudaEventCreateWithFlags(&p->out_done[s], cudaEventDisableTiming) == cudaSuccess;
        if (!ok) {
            cudaGetLastError();
            host_pipe_free(p);
            return VNSA_ERR_CUDA;
        }
        h->pipe = p;
    }
    HostPipe *p = h->pipe;
    const unsigned long long t = p->next;
    const int slot = (int)(t & 1ull);
    char *dq = p->mem + slot * p->slot_bytes, *dk = dq + bq, *dv = dk + bk, *dg = dv + bk,
         *di = dg + bg, *dout = di + bi;
    cudaStream_t s = (cudaStream_t)stream;
    const size_t nq = (size_t)n * c.h_q * c.d * h->esize;
    const size_t nk = (size_t)n * c.h_kv * c.d * h->esize;
    // inputs of this slot: free once the attention of call t - 2 has run
    bool ok = (t < 2 || cudaStreamWaitEvent(p->h2d, p->comp_done[slot], 0) == cudaSuccess) &&
              cudaMemcpyAsync(dq, q, nq, cudaMemcpyHostToDevice, p->h2d) == cudaSuccess &&
              cudaMemcpyAsync(dk, k, nk, cudaMemcpyHostToDevice, p->h2d) == cudaSuccess &&
              cudaMemcpyAsync(dv, v, nk, cudaMemcpyHostToDevice, p->h2d) == cudaSuccess &&
              cudaMemcpyAsync(dg, gate_logits, (size_t)n * c.h_q * 3 * 4,
                              cudaMemcpyHostToDevice, p->h2d) == cudaSuccess &&
              cudaMemcpyAsync(di, is_vision, (size_t)n, cudaMemcpyHostToDevice, p->h2d) ==
                  cudaSuccess &&
              cudaEventRecord(p->in_done[slot], p->h2d) == cudaSuccess &&
              cudaStreamWaitEvent(s, p->in_done[slot], 0) == cudaSuccess &&
              // output of this slot: free once call t - 2's copy to the host ran
              (t < 2 || cudaStreamWaitEvent(s, p->out_done[slot], 0) == cudaSuccess);
    if (!ok) {
        cudaGetLastError();
        return VNSA_ERR_CUDA;
    }
    vnsa_status st = vnsa_forward(h, n, dq, dk, dv, (const uint8_t *)di, (const float *)dg,
                                  dout, nullptr, stream);
    if (st != VNSA_OK) return st;
    ok = cudaEventRecord(p->comp_done[slot], s) == cudaSuccess &&
         cudaStreamWaitEvent(p->d2h, p->comp_done[slot], 0) == cudaSuccess &&
         cudaMemcpyAsync(out, dout, nq, cudaMemcpyDeviceToHost, p->d2h) == cudaSuccess &&
         cudaEventRecord(p->out_done[slot], p->d2h) == cudaSuccess;
    if (!ok) {
        cudaGetLastError();
        return VNSA_ERR_CUDA;
    }
    p->next = t + 1;
    *ticket = t;
    return VNSA_OK;
}

vnsa_status vnsa_host_wait(vnsa_handle *h, unsigned long long ticket) {
    if (!h || !h->pipe || ticket >= h->pipe->next) return VNSA_ERR_INVALID_ARG;
    // the slot's event was last recorded for `ticket` or a later call on the
    // same slot; copies to the host run in submission order on one stream
    if (cudaEventSynchronize(h->pipe->out_done[ticket & 1ull]) != cudaSuccess) {
        cudaGetLastError();
        return VNSA_ERR_CUDA;
    }
    return VNSA_OK;
}

vnsa_status vnsa_host_join(vnsa_handle *h, void *stream) {
    if (!h) return VNSA_ERR_INVALID_ARG;
    HostPipe *p = h->pipe;
    if (!p || p->next == 0) return VNSA_OK;
    cudaStream_t s = (cudaStream_t)stream;
    // the last call's copy to the host follows every earlier one on its stream
    if (cudaStreamWaitEvent(s, p->out_done[(p->next - 1) & 1ull], 0) != cudaSuccess) {
        cudaGetLastError();
        return VNSA_ERR_CUDA;
    }
    return VNSA_OK;
}

vnsa_status vnsa_get_device_status(vnsa_handle *h, void *stream, uint32_t *code) {
    if (!h || !code) return VNSA_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t v = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess ||
        cudaMemcpy(&v, h->status, 4, cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemset(h->status, 0, 4) != cudaSuccess) {
        cudaGetLastError();
        return VNSA_ERR_CUDA;
    }
    *code = v;
    return VNSA_OK;
}

vnsa_status vnsa_get_counts(vnsa_handle *h, void *stream, int *n_vision, int *n_text) {
    if (!h || !n_vision || !n_text) return VNSA_ERR_INVALID_ARG;
    Counts cn;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess ||
        cudaMemcpy(&cn, h->counts, sizeof(cn), cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return VNSA_ERR_CUDA;
    }
    *n_vision = cn.n_vision;
    *n_text = cn.n_text;
    return VNSA_OK;
}

vnsa_status vnsa_set_timing(vnsa_handle *h, int enable) {
    if (!h) return VNSA_ERR_INVALID_ARG;
    h->timing = enable ? 1 : 0;
    return VNSA_OK;
}

vnsa_status vnsa_get_timing(vnsa_handle *h, float *ms) {
    if (!h || !ms) return VNSA_ERR_INVALID_ARG;
    for (int x = 0; x < VNSA_NUM_STAGES; ++x) {
        ms[x] = 0.f;
        if (!h->timing || !h->ran[x]) continue;
        if (cudaEventSynchronize(h->ev[2 * x + 1]) != cudaSuccess ||
            cudaEventElapsedTime(&ms[x], h->ev[2 * x], h->ev[2 * x + 1]) != cudaSuccess) {
            cudaGetLastError();
            return VNSA_ERR_CUDA;
        }
    }
    return VNSA_OK;
}

vnsa_status vnsa_set_wait_limit(vnsa_handle *h, unsigned long long ns) {
    if (!h) return VNSA_ERR_INVALID_ARG;
    h->wait_ns = ns;
    return VNSA_OK;
}

vnsa_status vnsa_get_path(const vnsa_handle *h, int *path) {
    if (!h || !path) return VNSA_ERR_INVALID_ARG;
    *path = tc_supported(h->cfg) ? VNSA_PATH_TCGEN05 : VNSA_PATH_SIMT;
    return VNSA_OK;
}

vnsa_status vnsa_get_launch_count(vnsa_handle *h, int *launches) {
    if (!h || !launches) return VNSA_ERR_INVALID_ARG;
    *launches = h->launches;
    return VNSA_OK;
}

vnsa_status vnsa_set_cmp_mlp(vnsa_handle *h, int hidden, const void *w1_k, const float *b1_k,
                             const void *w2_k, const float *b2_k, const void *w1_v,
                             const float *b1_v, const void *w2_v, const float *b2_v) {
    if (!h || hidden < 0 || hidden > kCmpMlpMaxHidden) return VNSA_ERR_INVALID_ARG;
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess) return VNSA_ERR_CUDA;
    vnsa_status rc = VNSA_OK;
    if (hidden == 0) {
        // back to the linear projections given at create
        cudaDeviceSynchronize();
        if (h->mlp_mem) cudaFree(h->mlp_mem);
        h->mlp_mem = nullptr;
        memset(&h->mlp, 0, sizeof(h->mlp));
    } else if (!w1_k || !b1_k || !w2_k || !b2_k || !w1_v || !b1_v || !w2_v || !b2_v) {
        rc = VNSA_ERR_INVALID_ARG;
    } else {
        const size_t d = (size_t)h->cfg.d, H = (size_t)hidden;
        const size_t wb = d * H * h->esize;  // each of w1, w2
        const size_t sizes[4] = {wb, H * 4, wb, d * 4};
        size_t total = 0;
        for (int t = 0; t < 2; ++t)
            for (int x = 0; x < 4; ++x) total += (sizes[x] + 255) / 256 * 256;
        char *mem = nullptr;
        if (cudaMalloc(&mem, total) != cudaSuccess) {
            cudaGetLastError();
            rc = VNSA_ERR_CUDA;
        } else {
            const void *src[2][4] = {{w1_k, b1_k, w2_k, b2_k}, {w1_v, b1_v, w2_v, b2_v}};
            void *dst[2][4];
            size_t off = 0;
            bool ok = true;
            for (int t = 0; t < 2; ++t)
                for (int x = 0; x < 4; ++x) {
                    dst[t][x] = mem + off;
                    off += (sizes[x] + 255) / 256 * 256;
                    ok = ok && cudaMemcpy(dst[t][x], src[t][x], sizes[x], cudaMemcpyDefault) ==
                                   cudaSuccess;
                }
            if (!ok) {
                cudaGetLastError();
                cudaFree(mem);
                rc = VNSA_ERR_INVALID_ARG;
            } else {
                cudaDeviceSynchronize();
                if (h->mlp_mem) cudaFree(h->mlp_mem);
                h->mlp_mem = mem;
                h->mlp.hidden = hidden;
                for (int t = 0; t < 2; ++t) {
                    h->mlp.w1[t] = dst[t][0];
                    h->mlp.b1[t] = (const float *)dst[t][1];
                    h->mlp.w2[t] = dst[t][2];
                    h->mlp.b2[t] = (const float *)dst[t][3];
                }
            }
        }
    }
    if (cur != h->device && cur >= 0) cudaSetDevice(cur);
    return rc;
}

vnsa_status vnsa_gate_mlp(vnsa_handle *h, int n, int d_model, int hidden, const void *x,
                          const void *g1, const float *c1, const void *g2, const float *c2,
                          float *gate_logits, void *stream) {
    if (!h || !x || !g1 || !c1 || !g2 || !c2 || !gate_logits) return VNSA_ERR_INVALID_ARG;
    if (n < 1 || d_model < 1 || hidden < 1 || hidden > kCmpMlpMaxHidden)
        return VNSA_ERR_INVALID_ARG;
    if (h->cfg.dtype == VNSA_BF16 && d_model % 8 != 0) return VNSA_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(g1) || !aligned16(g2) || !aligned16(gate_logits))
        return VNSA_ERR_INVALID_ARG;
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != h->device && cudaSetDevice(h->device) != cudaSuccess) return VNSA_ERR_CUDA;
    h->launches = 0;
    cudaError_t e = launch_gate_mlp((int)h->cfg.dtype, n, d_model, hidden, 3 * h->cfg.h_q, x, g1,
                                    c1, g2, c2, gate_logits, h->status, (cudaStream_t)stream,
                                    &h->launches);
    if (cur != h->device && cur >= 0) cudaSetDevice(cur);
    if (e != cudaSuccess) {
        fprintf(stderr, "vnsa_gate_mlp: %s\n", cudaGetErrorString(e));
        return VNSA_ERR_CUDA;
    }
    return VNSA_OK;
}

vnsa_status vnsa_destroy(vnsa_handle *h) {
    if (!h) return VNSA_ERR_INVALID_ARG;
    cudaDeviceSynchronize();
    tc_destroy(h->tc);
    for (int e = 0; e < 2 * VNSA_NUM_STAGES; ++e)
        if (h->ev[e]) cudaEventDestroy(h->ev[e]);
    if (h->stage) cudaFree(h->stage);
    host_pipe_free(h->pipe);
    if (h->mlp_mem) cudaFree(h->mlp_mem);
    if (h->ws) cudaFree(h->ws);
    cudaGetLastError();
    delete h;
    return VNSA_OK;
}

}  // extern "C"
