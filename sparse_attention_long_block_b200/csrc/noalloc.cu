// noalloc.cu -- vnsa_select_noalloc: the block-selection chain (vision/text
// partition, block mean-pool + projection, compression attention with group
// importance, top-k) for callers that cannot allocate device memory.
//
// Who needs this: code that runs where cudaMalloc is not allowed or not wanted
// -- inside CUDA stream capture (allocation is not a capturable operation),
// inside a host framework that hands out all device memory from its own pool
// (inference-server or engine plugins), or on a latency-critical path that must
// not take the allocator's implicit device synchronisation.  vnsa_create
// allocates a workspace; this entry point instead keeps every intermediate of
// the selection chain in one fixed array in device global memory, declared
// below, so a call performs no allocation at all.
//
// The array is a file-scope __device__ object: every GPU that loads this
// library holds kScratchBytes of it until the process exits.  Host code cannot
// use the symbol as a device address (the host-side name is only a stand-in),
// so the first call on each device looks the address up with
// cudaGetSymbolAddress while that device is current and caches it (one atomic
// slot per device ordinal; the address belongs to the device's primary
// context, which is the context the CUDA runtime uses).
//
// The first 256 bytes of the array hold the device status word of the last
// call (read and cleared by vnsa_select_noalloc_status); the intermediates of
// a call follow it.
#include <math.h>
#include <string.h>

#include <atomic>

#include "config.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = 8u << 20;  // 8 MiB
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_select_scratch[kScratchBytes];

// per-device address of g_select_scratch, looked up on first use; racing
// first calls store the same value
std::atomic<void *> g_scratch_addr[kMaxDevices];

constexpr size_t kStatusOffset = 0;     // the status word of the last call
constexpr size_t kScratchHeader = 256;  // intermediates start after it

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

struct ScratchPlan {
    size_t vis, txt, counts, k_cmp, v_cmp, lse, imp, imp_sel, total;
    size_t imp_stride, imp_sel_stride;
};

ScratchPlan plan_for(const vnsa_config &c, int n) {
    const size_t es = c.dtype == VNSA_BF16 ? 2 : 4;
    const size_t nb = (size_t)(n / c.block);  // selection blocks
    const int stride = vnsa::cmp_stride_of(c);
    const size_t nc = (size_t)vnsa::cmp_blocks(n, c.block, stride);  // compression blocks
    ScratchPlan s;
    s.imp_stride = nc > 0 ? (nc + 3) / 4 * 4 : 4;
    s.imp_sel_stride = nb > 0 ? (nb + 3) / 4 * 4 : 4;
    size_t off = kScratchHeader;
    auto take = [&](size_t b) { size_t o = off; off += up256(b > 0 ? b : 1); return o; };
    s.vis = take((size_t)n * 4);
    s.txt = take((size_t)n * 4);
    s.counts = take(sizeof(vnsa::Counts));
    s.k_cmp = take(nc * c.h_kv * c.d * es);
    s.v_cmp = take(nc * c.h_kv * c.d * es);
    s.lse = take((size_t)n * c.h_q * 4);
    s.imp = take((size_t)c.h_kv * n * s.imp_stride * 4);
    s.imp_sel = stride != c.block ? take((size_t)c.h_kv * n * s.imp_sel_stride * 4) : s.imp;
    s.total = off;
    return s;
}

// The device address of the scratch array on the current device (looked up
// once per device), or nullptr with *st set on failure.
char *scratch_base(vnsa_status *st) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        *st = VNSA_ERR_NO_DEVICE;
        return nullptr;
    }
    void *ptr = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!ptr) {
        if (cudaGetSymbolAddress(&ptr, g_select_scratch) != cudaSuccess || !ptr) {
            cudaGetLastError();
            *st = VNSA_ERR_CUDA;
            return nullptr;
        }
        g_scratch_addr[dev].store(ptr, std::memory_order_release);
    }
    *st = VNSA_OK;
    return (char *)ptr;
}

}  // namespace

extern "C" vnsa_status vnsa_select_noalloc(const vnsa_config *cfg, int n, const void *q,
                                           const void *k, const void *v,
                                           const uint8_t *is_vision, const void *w_k,
                                           const void *w_v, float *o_cmp, int32_t *idx,
                                           void *stream) {
    using namespace vnsa;
    const vnsa_status cst = check_config(cfg, n);
    if (cst != VNSA_OK) return cst;
    if (!q || !k || !v || !is_vision || !w_k || !w_v || !o_cmp || !idx) return VNSA_ERR_INVALID_ARG;
    const uintptr_t al = (uintptr_t)q | (uintptr_t)k | (uintptr_t)v | (uintptr_t)w_k |
                         (uintptr_t)w_v | (uintptr_t)o_cmp | (uintptr_t)idx;
    if (al & 15u) return VNSA_ERR_INVALID_ARG;
    const ScratchPlan s = plan_for(*cfg, n);
    if (s.total > kScratchBytes) return VNSA_ERR_UNSUPPORTED;  // too large for the scratch
    vnsa_status bst;
    char *base = scratch_base(&bst);
    if (!base) return bst;
    cudaStream_t st = (cudaStream_t)stream;
    const vnsa_config &c = *cfg;
    const int dt = (int)c.dtype;
    const float scale = c.scale > 0.f ? c.scale : 1.0f / sqrtf((float)c.d);

    LayerParams p;
    memset(&p, 0, sizeof(p));
    p.n = n;
    p.n_max = n;
    p.h_q = c.h_q;
    p.h_kv = c.h_kv;
    p.d = c.d;
    p.r = c.h_q / c.h_kv;
    p.block = c.block;
    p.stride = cmp_stride_of(c);
    p.top_k = c.top_k;
    p.window = c.window;
    p.force_first = c.force_first;
    p.force_local = c.force_local;
    p.nb_max = cmp_blocks(n, c.block, p.stride);
    p.scale_log2 = scale * kLog2e;
    p.q = q;
    p.k = k;
    p.v = v;
    p.is_vision = is_vision;
    p.vis = (const int32_t *)(base + s.vis);
    p.txt = (const int32_t *)(base + s.txt);
    p.counts = (const Counts *)(base + s.counts);
    p.status = (uint32_t *)(base + kStatusOffset);
    p.k_cmp = base + s.k_cmp;
    p.v_cmp = base + s.v_cmp;
    p.lse = (float *)(base + s.lse);
    p.imp = (float *)(base + s.imp);
    p.imp_stride = s.imp_stride;
    p.imp_sel = (float *)(base + s.imp_sel);
    p.imp_sel_stride = s.imp_sel == s.imp ? s.imp_stride : s.imp_sel_stride;
    p.idx = idx;  // caller's output [h_kv][n][top_k]
    p.idx_src = idx;
    p.idx_rows = (size_t)n;
    p.o_cmp_ws = o_cmp;  // caller's output [n][h_q][d], by vision rank

    // The array keeps the previous call's contents; only the status word must
    // start at zero (the kernels overwrite everything else they later read).
    cudaError_t e = cudaMemsetAsync(base + kStatusOffset, 0, 16, st);
    if (e == cudaSuccess)
        e = launch_partition(is_vision, n, c.block, p.stride, (int32_t *)p.vis, (int32_t *)p.txt,
                             (Counts *)p.counts, st);
    if (e == cudaSuccess)
        e = launch_pool_proj(dt, c.d, k, v, p.vis, p.counts, w_k, w_v, (void *)p.k_cmp,
                             (void *)p.v_cmp, c.h_kv, c.block, p.stride, p.nb_max, st);
    if (e == cudaSuccess) e = launch_cmp_simt(dt, p, st);
    if (e == cudaSuccess && p.stride != p.block) e = launch_imp_remap(p, st);
    if (e == cudaSuccess) e = launch_topk(p, st);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return VNSA_ERR_CUDA;
    }
    return VNSA_OK;
}

extern "C" vnsa_status vnsa_select_noalloc_status(void *stream, uint32_t *code) {
    if (!code) return VNSA_ERR_INVALID_ARG;
    *code = 0;
    vnsa_status bst;
    char *base = scratch_base(&bst);
    if (!base) return bst;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t word = 0;
    if (cudaStreamSynchronize(st) != cudaSuccess ||
        cudaMemcpy(&word, base + kStatusOffset, sizeof(word), cudaMemcpyDeviceToHost) !=
            cudaSuccess ||
        cudaMemset(base + kStatusOffset, 0, sizeof(word)) != cudaSuccess) {
        cudaGetLastError();
        return VNSA_ERR_CUDA;
    }
    *code = word;
    return VNSA_OK;
}
