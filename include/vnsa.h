/*
 * vnsa.h -- C ABI of the VideoNSA hybrid sparse-attention layer prefill on one
 * NVIDIA B200 (sm_100a).
 *
 * What it computes ("VideoNSA: Native Sparse Attention Scales Video
 * Understanding", paper notes, section "Method"; "VideoNSA: Native Sparse
 * Attention for Video Understanding", model card, section "Model
 * Architecture"): the attention of one decoder layer over a prompt of n tokens.
 * A per-token flag splits the tokens into a vision set and a text set.  Vision
 * tokens attend through three branches over the vision subsequence, each
 * weighted by a per-head sigmoid gate:
 *   compression  mean of each block of `block` vision keys/values, projected
 *                by W_K / W_V, attended causally at block granularity;
 *   selection    the top_k blocks ranked by the compression probabilities
 *                summed over each GQA group (block 0 and the query's own block
 *                always kept), attended token by token;
 *   window       the `window` most recent vision tokens.
 * Text tokens attend densely and causally to every earlier token (GQA).  The
 * outputs are written at the tokens' original positions.
 *
 * Layouts (row-major, contiguous, all device pointers unless stated):
 *   q, out        [n][h_q][d]        dtype (bf16 or fp32)
 *   k, v          [n][h_kv][d]       dtype
 *   is_vision     [n]                uint8, nonzero = vision token
 *   gate_logits   [n][h_q][3]        fp32, branch order (cmp, slc, swa);
 *                                    ignored for text rows
 *   w_k, w_v      [d][d]             dtype; block key = mean(K_block) . W_K
 * Query head h uses KV head h / (h_q / h_kv).
 *
 * Ownership: the caller owns every tensor it passes and the stream.  The handle
 * owns its workspace (sized for n_max tokens at create time) and a copy of
 * W_K, W_V.  One handle must not run two forwards concurrently.
 *
 * Errors: every call returns a vnsa_status.  Argument errors are found on the
 * host before anything is launched.  vnsa_forward is asynchronous on `stream`
 * and never synchronises; a failed launch returns VNSA_ERR_CUDA.  Conditions
 * the kernels detect (a bounded wait that gave up, an index out of range) set a
 * device status word, read and cleared by vnsa_get_device_status.
 */
#ifndef VNSA_H
#define VNSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum vnsa_status {
    VNSA_OK = 0,
    VNSA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned pointer    */
    VNSA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. d not 64/128) */
    VNSA_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed             */
    VNSA_ERR_TIMEOUT = 4,      /* device: a bounded wait gave up                */
    VNSA_ERR_BOUNDS = 5,       /* device: an index fell outside its tensor      */
    VNSA_ERR_NO_DEVICE = 6     /* no CUDA device is visible                     */
} vnsa_status;

typedef enum vnsa_dtype { VNSA_BF16 = 0, VNSA_FP32 = 1 } vnsa_dtype;

typedef struct vnsa_config {
    int n_max;        /* largest n a forward will see (sizes the workspace)     */
    int h_q, h_kv;    /* query heads, KV heads; h_q % h_kv == 0, h_q/h_kv <= 16  */
    int d;            /* head dim: 64 or 128                                    */
    int block;        /* compression block = selection block, >= 1: the vision */
                      /* tokens per frame (64 in the pages' setting; the pages  */
                      /* treat tokens per frame as a task knob).                */
                      /* Every block size runs on the GPU; the tensor-core      */
                      /* path takes bf16, d 128, 4..16 query heads per KV head  */
                      /* and a selection of at most 1152 64-key tiles per 128-  */
                      /* row item, other settings the SIMT kernels.             */
    int top_k;        /* blocks kept per (group, query), 1..64, >= #forced      */
    int window;       /* sliding window in vision tokens, >= 1                  */
    int force_first;  /* 1: block 0 is always selected (default 1)              */
    int force_local;  /* 1: the query's own block is always selected (def. 1)   */
    float scale;      /* softmax scale; 0 -> 1/sqrt(d)                          */
    vnsa_dtype dtype; /* storage type of q, k, v, w, out                        */
    int cmp_stride;   /* compression stride, 1..block; 0 -> block.  Below the   */
                      /* block size the compression blocks overlap (the native  */
                      /* sparse attention design the pages build on): block c   */
                      /* averages vision tokens [c*s, c*s + block) and is       */
                      /* visible to query i once its last token is <= i; the    */
                      /* importance of selection block j is the compression     */
                      /* mass spread over the selection blocks by the tokens    */
                      /* each compression block puts in them.  vnsa_decode      */
                      /* takes cmp_stride = block only.                         */
} vnsa_config;

typedef struct vnsa_handle vnsa_handle;

/*
 * Optional per-step exports and an optional selection override, all device
 * pointers, each may be NULL.  N_v = number of vision tokens, nb = N_v / block.
 * Per-vision-token arrays are indexed by vision rank (0..N_v-1) and sized for
 * n rows (the forward's token count); rows N_v..n-1 are left untouched.
 */
typedef struct vnsa_debug {
    float *o_cmp;            /* [n][h_q][d] ungated compression output, by position  */
    float *o_slc;            /* [n][h_q][d] ungated selection output, by position    */
    float *o_swa;            /* [n][h_q][d] ungated window output, by position       */
    float *lse_cmp;          /* [n][h_q] compression log-sum-exp (natural log), rank */
    int32_t *idx;            /* [h_kv][n][top_k] selected blocks, ascending, -1 pad  */
    float *imp;              /* [h_kv][n][imp_stride] selection-block importance;
                                only the visible blocks j < (i+1)/block of row i
                                are written                                          */
    int imp_stride;          /* row stride of imp in floats (>= n / block)           */
    void *k_cmp;             /* [nc][h_kv][d] dtype block keys (nc compression
                                blocks: nb when cmp_stride = block)                  */
    void *v_cmp;             /* [nc][h_kv][d] dtype block values                     */
    const int32_t *forced_idx; /* input [h_kv][n][top_k]: used instead of the top-k  */
} vnsa_debug;

/* Stages timed by vnsa_get_timing, in launch order. */
typedef enum vnsa_stage {
    VNSA_STAGE_PARTITION = 0, /* vision/text split                                  */
    VNSA_STAGE_POOL = 1,      /* block mean-pool + projection -> K_cmp, V_cmp       */
    VNSA_STAGE_CMP = 2,       /* compression attention + importance                 */
    VNSA_STAGE_TOPK = 3,      /* block selection                                    */
    VNSA_STAGE_SLC = 4,       /* selection attention (block 64, tensor cores: with  */
                              /* the merge that writes the vision output rows)      */
    VNSA_STAGE_SWA = 5,       /* sliding window (other configurations: + gate       */
                              /* combine + vision output)                           */
    VNSA_STAGE_TEXT = 6,      /* dense text GQA                                     */
    VNSA_NUM_STAGES = 7
} vnsa_stage;

/* Human-readable text of a status code (static storage). */
const char *vnsa_status_string(vnsa_status s);

/* Name of a stage ("partition", "pool", ...), or NULL if out of range. */
const char *vnsa_stage_name(int stage);

/* Bytes of device workspace vnsa_create would allocate for cfg. */
vnsa_status vnsa_workspace_bytes(const vnsa_config *cfg, size_t *bytes);

/*
 * Validate cfg, allocate the workspace on the current device and copy the
 * projections w_k, w_v ([d][d], dtype, device pointers) into it.  Synchronous.
 * On success *out holds the handle; on failure *out is NULL and nothing leaks.
 */
vnsa_status vnsa_create(const vnsa_config *cfg, const void *w_k, const void *w_v,
                        vnsa_handle **out);

/*
 * One layer prefill of n (1..n_max) tokens, enqueued on `stream` (a
 * cudaStream_t; NULL = the legacy default stream).  Pointers must be device
 * pointers, 16-byte aligned, in the layouts above.  `dbg` may be NULL.
 * Returns after enqueueing; errors found by the kernels are reported by
 * vnsa_get_device_status.  The call neither allocates nor synchronises, so it
 * may be captured into a CUDA graph on `stream`; a replay recomputes the layer
 * from the captured buffers' current contents (same n and pointers; the
 * handle's workspace is reused, so replays on one handle must not overlap).
 */
vnsa_status vnsa_forward(vnsa_handle *h, int n, const void *q, const void *k,
                         const void *v, const uint8_t *is_vision,
                         const float *gate_logits, void *out, const vnsa_debug *dbg,
                         void *stream);

/*
 * The same layer prefill from HOST buffers (same layouts): copies the inputs
 * to handle-owned device staging buffers, runs vnsa_forward on `stream`, copies
 * `out` back and synchronises the stream before returning.  Page-locked host
 * buffers give the fastest copies.  Allocates nothing per call.
 */
vnsa_status vnsa_forward_host(vnsa_handle *h, int n, const void *q, const void *k,
                              const void *v, const uint8_t *is_vision,
                              const float *gate_logits, void *out, void *stream);

/*
 * Streamed layer prefills from HOST buffers, for a caller that feeds one layer
 * call after another from host memory: the copies of neighbouring calls
 * overlap the attention of the call between them.  (Not a step of the method:
 * the pages run the layer on data already on the device.)
 *
 * vnsa_forward_host_async enqueues one call and returns without waiting.  Its
 * inputs are copied on a copy stream the handle owns into one of two device
 * staging slots (call t uses slot t % 2; allocated on the first call, held
 * until vnsa_destroy), the layer runs on `stream` as vnsa_forward, and `out`
 * is copied back on a second handle-owned copy stream.  Events order the
 * three: call t's input copies wait for the attention of call t - 2, its
 * attention for its input copies and for call t - 2's output copy, its output
 * copy for its attention.  While call t computes, the inputs of call t + 1 and
 * the output of call t - 1 cross the bus.  *ticket receives the call's number
 * (0, 1, 2, ... per handle).  The host buffers (same layouts as vnsa_forward)
 * must stay valid and unchanged until vnsa_host_wait(ticket) returns; only
 * page-locked buffers let the copies run asynchronously.  Calls on one handle
 * must come from one host thread and use one `stream`.  Argument errors return
 * before anything is enqueued; device-detected errors go to the status word.
 *
 * vnsa_host_wait blocks the host until call `ticket`'s output is in host
 * memory (VNSA_ERR_INVALID_ARG for a ticket not issued yet).  vnsa_host_join
 * makes `stream` wait, without blocking the host, until every call submitted
 * so far has its output on the host (e.g. before recording a timing event).
 */
vnsa_status vnsa_forward_host_async(vnsa_handle *h, int n, const void *q, const void *k,
                                    const void *v, const uint8_t *is_vision,
                                    const float *gate_logits, void *out, void *stream,
                                    unsigned long long *ticket);
vnsa_status vnsa_host_wait(vnsa_handle *h, unsigned long long ticket);
vnsa_status vnsa_host_join(vnsa_handle *h, void *stream);

/*
 * One decode step ("VideoNSA: Native Sparse Attention Scales Video
 * Understanding", paper notes, section "Method", applied to a single new
 * token): the attention output of token n-1, appended to the token stream that
 * the previous vnsa_forward or vnsa_decode on this handle processed (that call
 * must have covered exactly tokens 0..n-2 of the same stream; otherwise
 * VNSA_ERR_INVALID_ARG).  The result equals row n-1 of vnsa_forward over all n
 * tokens: a vision token attends through compression (the complete vision
 * blocks so far), selection and the window with its gates, a text token
 * densely to every token 0..n-1.
 *
 * Inputs (device, 16-byte aligned): k, v [n][h_kv][d] and is_vision [n] hold the
 * whole stream, the new token last (the caller appends it to its cache);
 * q_new [h_q][d] and gate_new [h_q][3] (fp32, ignored for a text token) belong
 * to the new token.  Output: out_new [h_q][d].  sel_out, if not NULL, receives
 * the selected blocks [h_kv][top_k] (ascending, -1 padded; all -1 for a text
 * token).  The handle's workspace keeps the stream's vision/text lists and the
 * block keys/values; the step extends them (pooling the block the token
 * completes, if any).  n <= n_max.  Asynchronous on `stream`; device-detected
 * errors go to the status word.  A handle whose cmp_stride is below its block
 * returns VNSA_ERR_UNSUPPORTED.
 */
vnsa_status vnsa_decode(vnsa_handle *h, int n, const void *q_new, const void *k, const void *v,
                        const uint8_t *is_vision, const float *gate_new, void *out_new,
                        int32_t *sel_out, void *stream);

/*
 * The compression branch's "learnable MLP" ("VideoNSA: Native Sparse Attention
 * Scales Video Understanding", paper notes, section "Method": blocks are
 * averaged into block keys/values through a learnable MLP), read as a
 * two-layer perceptron on the block mean that replaces the linear W_K / W_V of
 * vnsa_create:  K_cmp = SiLU(Kbar . w1_k + b1_k) . w2_k + b2_k, the same for V
 * with its own weights, shared by the KV heads; SiLU(z) = z / (1 + e^-z).
 *
 * hidden: width of the hidden layer, 1..512; 0 returns to the linear maps (the
 * weight pointers may then be NULL).  w1_* [d][hidden] and w2_* [hidden][d] in
 * the layer dtype, b1_* [hidden] and b2_* [d] fp32; host or device pointers,
 * copied into memory the handle owns before the call returns (it
 * synchronises the device).  The hidden layer is computed in fp32; K_cmp,
 * V_cmp are rounded once to the layer dtype.  Applies to later vnsa_forward and
 * vnsa_decode calls (vnsa_select_noalloc keeps the linear maps it is given).
 * Errors: VNSA_ERR_INVALID_ARG (hidden out of range, a NULL weight, a copy that
 * failed), VNSA_ERR_CUDA (allocation).
 */
vnsa_status vnsa_set_cmp_mlp(vnsa_handle *h, int hidden, const void *w1_k, const float *b1_k,
                             const void *w2_k, const float *b2_k, const void *w1_v,
                             const float *b1_v, const void *w2_v, const float *b2_v);

/*
 * Gate logits from the layer input (same page and section: a two-layer MLP and
 * a sigmoid give each head its weights for the three branches), read as
 *   gate_logits[t] = SiLU(x_t . g1 + c1) . g2 + c2,
 * x [n][d_model] the layer input (h_q * d wide in the pages' model), g1
 * [d_model][hidden], g2 [hidden][3 h_q] in the layer dtype, c1 [hidden] and c2
 * [3 h_q] fp32.  Output gate_logits [n][h_q][3] fp32: column 3h + c of token t
 * is the logit of branch c (cmp, slc, swa) of head h, ready for vnsa_forward
 * (which applies the sigmoid).  In bf16 the hidden activations are rounded to
 * bf16 before the second product.  1 <= hidden <= 512; bf16 needs d_model a
 * multiple of 8.  The tensor-core kernel runs for bf16 with d_model a multiple
 * of 64, hidden in {64, 128, 192, 256} and 3 h_q <= 256; other settings run a
 * SIMT kernel.  Device pointers; x, g1, g2 and gate_logits 16-byte aligned.
 * Asynchronous on `stream`; counts toward vnsa_get_launch_count.
 */
vnsa_status vnsa_gate_mlp(vnsa_handle *h, int n, int d_model, int hidden, const void *x,
                          const void *g1, const float *c1, const void *g2, const float *c2,
                          float *gate_logits, void *stream);

/*
 * Synchronise `stream`, then read and clear the handle's device status word.
 * *code receives VNSA_OK or the first device-detected error (TIMEOUT, BOUNDS).
 */
vnsa_status vnsa_get_device_status(vnsa_handle *h, void *stream, uint32_t *code);

/*
 * Vision / text counts of the last forward (synchronises `stream`).
 */
vnsa_status vnsa_get_counts(vnsa_handle *h, void *stream, int *n_vision, int *n_text);

/*
 * Per-stage timing.  With timing on, each forward records CUDA events between
 * its stages on its stream; vnsa_get_timing synchronises on the last event and
 * writes VNSA_NUM_STAGES milliseconds (0 for a stage that did not run).
 */
vnsa_status vnsa_set_timing(vnsa_handle *h, int enable);
vnsa_status vnsa_get_timing(vnsa_handle *h, float *ms);

/*
 * Limit of the kernels' bounded waits, in nanoseconds of device time, for the
 * later calls on this handle; 0 restores the default (400 ms).  A wait that
 * runs out makes its thread block stop its work, wait (within its own bound)
 * for the copies and tensor-core operations it has in flight, free its tensor
 * memory and exit; the status word then reads VNSA_ERR_TIMEOUT and the layer's
 * output of that call is undefined.  Later kernels of the call skip their work
 * once the status word is set.  A very small limit makes a forward time out on
 * purpose, which is how failure detection is tested.  (A library knob, not a
 * step of the method.)
 */
vnsa_status vnsa_set_wait_limit(vnsa_handle *h, unsigned long long ns);

/* Which kernels a handle's layer runs on. */
typedef enum vnsa_path {
    VNSA_PATH_SIMT = 0,     /* CUDA-core kernels (fp32, d 64, 1..3 query heads per
                               KV head, or a selection plan beyond the shared-
                               memory copy); far slower at scale                */
    VNSA_PATH_TCGEN05 = 1   /* tensor-core (tcgen05 + TMA) attention kernels    */
} vnsa_path;

/* *path receives the kernel family vnsa_forward uses for this handle. */
vnsa_status vnsa_get_path(const vnsa_handle *h, int *path);

/* Kernel launches the last forward enqueued (for launch accounting). */
vnsa_status vnsa_get_launch_count(vnsa_handle *h, int *launches);

/* Free the workspace and the handle (synchronises the device first). */
vnsa_status vnsa_destroy(vnsa_handle *h);

/*
 * Block selection without any device allocation (the paper has no counterpart:
 * this is a library-only entry point).  For callers that cannot call
 * cudaMalloc -- code under CUDA stream capture, plugins that must draw all
 * device memory from a host framework's own pool, latency-critical paths that
 * cannot take the allocator's synchronisation -- it runs the selection chain
 * of one layer: vision/text split, block mean-pool + projection, compression
 * attention with group importance, top-k.  No handle is needed.
 *
 * Inputs (device, 16-byte aligned, layouts as above): q, k, v, is_vision for
 * n tokens, w_k, w_v [d][d]; cfg as for vnsa_create (n_max is ignored).
 * Outputs (device, caller-owned): o_cmp [n][h_q][d] fp32, the ungated
 * compression output of each vision token by vision rank; idx
 * [h_kv][n][top_k], the selected blocks by vision rank, ascending, -1 padded.
 * Rows N_v..n-1 of both are left untouched.
 *
 * Scratch: every intermediate lives in one 8 MiB array in device global
 * memory that the library declares statically; each GPU that loads the library
 * holds it until the process exits.  A call whose intermediates do not fit
 * returns VNSA_ERR_UNSUPPORTED before launching anything (for 28/4 heads, d 128
 * this allows about 5,000 tokens).  cfg is checked exactly as vnsa_create
 * checks it, with n in place of n_max (same limits, same codes).  The first
 * call on a device looks up the array's device address (cudaGetSymbolAddress)
 * with that device current and keeps it for the process; the address belongs
 * to the device's primary context, the one the CUDA runtime uses, so callers
 * that run under a context of their own (a driver-API cuCtxCreate) cannot use
 * this entry point.  Make that first call before any stream capture.  All calls
 * on a device share the one array and it keeps the previous call's contents, so
 * calls that overlap on the GPU (different streams, or concurrent host threads)
 * race and must be serialised by the caller.  Asynchronous on `stream` (a
 * cudaStream_t).  Errors the kernels detect (an index out of range) go to a
 * status word inside the array, cleared when a call starts: read it with
 * vnsa_select_noalloc_status after the call and before the next one.
 */
vnsa_status vnsa_select_noalloc(const vnsa_config *cfg, int n, const void *q, const void *k,
                                const void *v, const uint8_t *is_vision, const void *w_k,
                                const void *w_v, float *o_cmp, int32_t *idx, void *stream);

/*
 * Device status of the last vnsa_select_noalloc call on the current device:
 * synchronises `stream` (the call's stream), then reads and clears the status
 * word the call's kernels write.  *code receives VNSA_OK or the first
 * device-detected error (e.g. VNSA_ERR_BOUNDS).  Allocates nothing.  Errors:
 * VNSA_ERR_INVALID_ARG (code NULL), VNSA_ERR_NO_DEVICE, VNSA_ERR_CUDA.  (No
 * counterpart in the paper: a library-only entry point, like the call it
 * reports on.)
 */
vnsa_status vnsa_select_noalloc_status(void *stream, uint32_t *code);

#ifdef __cplusplus
}
#endif
#endif /* VNSA_H */
