/*
 * vnsa_oracle.c -- plain fp64 CPU oracle of the VideoNSA hybrid sparse-attention
 * layer prefill.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load
 * this file: it exists so that the tests, the smoke check and the CPU-baseline leg
 * of the benchmark have an independent, obviously correct answer to compare with.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * Sources (page title, then the section it falls in):
 *   [M]  "VideoNSA: Native Sparse Attention Scales Video Understanding" (paper
 *        notes), section "Method": 28 query heads / 4 KV heads (GQA); tokens split
 *        into vision and text sets by position IDs; vision tokens go through
 *        compression (blocks of 64 averaged into block keys/values, then a
 *        learnable projection), selection (top-k blocks by importance) and a
 *        sliding window; a per-head sigmoid gate combines the three branch
 *        outputs; text tokens use standard GQA; outputs are written back at the
 *        original positions.
 *   [A]  "VideoNSA: Native Sparse Attention for Video Understanding" (model card),
 *        section "Model Architecture": three branches (mean of each frame's
 *        key/value block; a subset of blocks ranked as most useful; a local
 *        window), mixed with weights that are learned separately per head.
 *   [K]  same paper notes, section "Key claims": the vision/text split by
 *        position ID is taken at every layer; dense attention is kept for text.
 *
 * Readings of points the pages leave open (each is repeated in the design notes):
 *   R1  Vision queries see only the vision subsequence; blocks are formed over
 *       vision order (index i = rank of the token among vision tokens).
 *   R2  A compressed block j is visible to vision query i iff its last token is
 *       at or before i, i.e. j < floor((i+1)/B).  No visible block -> the branch
 *       output is 0 and the block importances are 0.
 *   R3  The projection is a d x d linear map per tensor (W_K, W_V), applied to
 *       the block mean as a row vector: K_cmp = mean(K_block) . W_K.  In bf16
 *       runs K_cmp / V_cmp are rounded to bf16 (round-to-nearest-even) after the
 *       exact computation, because the kernel stores them in bf16.
 *   R4  Block importance = the normalised compression softmax probability,
 *       summed over the query heads of one GQA group.
 *   R5  Block 0 and the query's own block floor(i/B) are always selected and
 *       count within top_k; the other top_k - #forced blocks are the best by
 *       importance among visible, non-forced blocks, ties going to the lower
 *       block index.  Fewer candidates than slots -> all are taken, the rest
 *       of the index row is -1.  Indices are stored ascending.
 *   R6  Selection attends to every token of the selected blocks that is at or
 *       before the query (causal mask inside the query's own block).
 *   R7  The window holds the w most recent vision tokens including the query:
 *       [i-w+1, i].
 *   R8  out = sig(g_cmp) o_cmp + sig(g_slc) o_slc + sig(g_swa) o_swa with the
 *       logistic sigmoid and no normalisation; text rows ignore gate logits.
 *   R9  Every branch uses the same softmax scale (default 1/sqrt(d)).
 *   R10 A text token at global position t attends to every token u <= t,
 *       vision or text, with KV head floor(h / (H_q/H_kv)).
 *   R11 The "learnable MLP" of the compression branch [M], when a hidden width
 *       H_c is given instead of R3's linear map: a two-layer perceptron on the
 *       block mean, K_cmp = SiLU(Kbar . W1 + b1) . W2 + b2 with W1 [d][H_c],
 *       W2 [H_c][d], SiLU(z) = z / (1 + e^-z); its own weights for K and for V,
 *       shared by the KV heads.  The hidden layer is exact; the output is
 *       rounded as in R3.
 *   R12 The gate [M] ("a two-layer MLP + sigmoid gate per head"): the branch
 *       logits of token t come from the layer input x_t (h_q * d wide) through
 *       logits = SiLU(x_t . G1 + c1) . G2 + c2, G1 [D][H], G2 [H][3 h_q]; output
 *       column 3h + c is the logit of branch c (cmp, slc, swa) of head h, and
 *       the sigmoid of R8 turns it into the gate.  In bf16 runs the hidden
 *       activations are rounded to bf16 (round-to-nearest-even): they are the
 *       operand of the second product.
 *   R13 Compression blocks may overlap (a compression stride s below the
 *       block size B, the native sparse attention design the pages build on):
 *       compression block c averages the B vision tokens [c s, c s + B), for
 *       c = 0 .. nc-1 with nc = floor((N_v - B) / s) + 1, and is visible to
 *       query i iff its last token c s + B - 1 is at or before i (R2 is the
 *       case s = B).  Selection blocks stay the non-overlapping blocks of B
 *       tokens.  The importance of selection block j is the group's
 *       compression probability mass distributed over the selection blocks in
 *       proportion to the tokens of each compression block that lie in them:
 *       imp[j] = sum_c |[c s, c s + B) ^ [j B, j B + B)| / B * p_c.  With s = B
 *       this is p_j, R4 unchanged.  Candidates and forced blocks follow R5.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int n;              /* tokens in the sequence                        */
    int h_q, h_kv, d;   /* query heads, KV heads (= groups), head dim     */
    int block;          /* compression block = stride = selection block  */
    int top_k;          /* selected blocks per (group, query)            */
    int window;         /* sliding-window length in vision tokens        */
    int force_first;    /* always keep block 0                           */
    int force_local;    /* always keep the query's own block             */
    double scale;       /* softmax scale                                 */
    int round_cmp_bf16; /* round K_cmp / V_cmp to bf16 (R3)              */
    int stride;         /* compression stride, 1..block (0: = block, R13) */
} vnsa_oracle_cfg;

enum { ORACLE_OK = 0, ORACLE_EINVAL = 1, ORACLE_ENOMEM = 2 };

/* Round to the nearest bfloat16 value (8 significant bits), ties to even.  */
double vnsa_oracle_round_bf16(double x)
{
    if (x == 0.0 || !isfinite(x)) return x;
    int e = ilogb(x);                 /* x = m * 2^e, 1 <= |m| < 2 */
    if (e < -126) e = -126;           /* bf16 subnormal spacing 2^-133 */
    double quantum = ldexp(1.0, e - 7);
    return rint(x / quantum) * quantum; /* rint: round half to even */
}

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* SiLU (R11, R12): z * sigmoid(z). */
static double silu(double z) { return z / (1.0 + exp(-z)); }

/* The compression map of one tensor (K or V), fp64: R3's linear map w [d][d]
 * when hidden == 0, else R11's perceptron w1 [d][hidden], b1 [hidden],
 * w2 [hidden][d], b2 [d]. */
typedef struct {
    int hidden;
    const double *w, *w1, *b1, *w2, *b2;
} cmp_map;

/* Public form of R11's weights (fp32 values, as handed to the GPU). */
typedef struct {
    int hidden;                               /* H_c >= 1                       */
    const float *w1_k, *b1_k, *w2_k, *b2_k;   /* [d][H_c], [H_c], [H_c][d], [d] */
    const float *w1_v, *b1_v, *w2_v, *b2_v;
} vnsa_oracle_cmp_mlp;

/* out[d] = the compression map applied to the block mean m[d]; h: scratch of
 * `hidden` values. */
static void apply_cmp_map(const cmp_map *mp, int d, const double *m, double *h, double *out)
{
    if (mp->hidden == 0) {
        for (int col = 0; col < d; ++col) {
            double a = 0.0;
            for (int e = 0; e < d; ++e) a += m[e] * mp->w[(size_t)e * d + col];
            out[col] = a;
        }
        return;
    }
    const int H = mp->hidden;
    for (int x = 0; x < H; ++x) {
        double a = mp->b1[x];
        for (int e = 0; e < d; ++e) a += m[e] * mp->w1[(size_t)e * H + x];
        h[x] = silu(a);
    }
    for (int col = 0; col < d; ++col) {
        double a = mp->b2[col];
        for (int x = 0; x < H; ++x) a += h[x] * mp->w2[(size_t)x * d + col];
        out[col] = a;
    }
}

/*
 * One softmax attention of query q (d values, already fp64) over a key list.
 * Key u of the list has its key at kb + keys[u]*stride and its value at
 * vb + keys[u]*stride.  Computes s_u = scale * q.k_u, p = softmax(s),
 * o = sum_u p_u v_u; returns log(sum exp(s)) (or -inf for an empty list, with
 * o = 0).  If p_out is given, p_u is written there in list order.
 */
static double attend(const double *q, const double *kb, const double *vb,
                     size_t stride, const int *keys, int nk, int d, double scale,
                     double *o, double *p_out, double *s)
{
    for (int e = 0; e < d; ++e) o[e] = 0.0;
    if (nk == 0) return -INFINITY;
    double m = -INFINITY;
    for (int u = 0; u < nk; ++u) {
        const double *k = kb + (size_t)keys[u] * stride;
        double acc = 0.0;
        for (int e = 0; e < d; ++e) acc += q[e] * k[e];
        s[u] = scale * acc;
        if (s[u] > m) m = s[u];
    }
    double z = 0.0;
    for (int u = 0; u < nk; ++u) z += exp(s[u] - m);
    for (int u = 0; u < nk; ++u) {
        double p = exp(s[u] - m) / z;
        if (p_out) p_out[u] = p;
        const double *v = vb + (size_t)keys[u] * stride;
        for (int e = 0; e < d; ++e) o[e] += p * v[e];
    }
    return m + log(z);
}

/* Vision / text partition [M], [K]: vis[i] = global position of the i-th
 * vision token; returns the vision count. */
static int partition(const uint8_t *is_vision, int n, int *vis)
{
    int nv = 0;
    for (int t = 0; t < n; ++t)
        if (is_vision[t]) vis[nv++] = t;
    return nv;
}

/* Compression stride (R13): 0 means the block size. */
static int cmp_stride(const vnsa_oracle_cfg *c) { return c->stride > 0 ? c->stride : c->block; }

/* Number of compression blocks over nv vision tokens (R13). */
static int cmp_blocks(const vnsa_oracle_cfg *c, int nv)
{
    return nv >= c->block ? (nv - c->block) / cmp_stride(c) + 1 : 0;
}

static int check_cfg(const vnsa_oracle_cfg *c)
{
    if (!c || c->n < 0 || c->h_q <= 0 || c->h_kv <= 0 || c->d <= 0) return 0;
    if (c->h_q % c->h_kv != 0) return 0;
    if (c->block <= 0 || c->window <= 0 || c->top_k <= 0) return 0;
    if (c->stride < 0 || c->stride > c->block) return 0;
    int forced = (c->force_first ? 1 : 0) + (c->force_local ? 1 : 0);
    if (c->top_k < forced) return 0;
    return 1;
}

/*
 * Compression keys/values [M], [A]: each block of B consecutive vision tokens
 * is averaged, and the mean is mapped to one block key / block value:
 *   Kbar_j = (1/B) sum_{u<B} K[vis[j s + u]],   K_cmp_j = Kbar_j . W_K   (R3),
 * per KV head, for the nb compression blocks (stride s = B unless R13).  Same
 * for V.  k_cmp, v_cmp: [nb][h_kv][d].  Kd, Vd: fp64 copies of K, V
 * [n][h_kv][d].
 */
static void pool_proj(const vnsa_oracle_cfg *c, const double *Kd, const double *Vd,
                      const int *vis, int nb, const cmp_map *mk, const cmp_map *mv,
                      double *k_cmp, double *v_cmp)
{
    const int d = c->d, hk = c->h_kv, B = c->block, S = cmp_stride(c);
    const int H = mk->hidden > mv->hidden ? mk->hidden : mv->hidden;
    #pragma omp parallel for schedule(static)
    for (int j = 0; j < nb; ++j) {
        double *kbar = malloc(sizeof(double) * (2 * d + (H > 0 ? H : 1)));
        double *vbar = kbar + d;
        double *hid = vbar + d;
        for (int g = 0; g < hk; ++g) {
            for (int e = 0; e < d; ++e) { kbar[e] = 0.0; vbar[e] = 0.0; }
            for (int u = 0; u < B; ++u) {
                size_t row = ((size_t)vis[j * S + u] * hk + g) * d;
                for (int e = 0; e < d; ++e) { kbar[e] += Kd[row + e]; vbar[e] += Vd[row + e]; }
            }
            for (int e = 0; e < d; ++e) { kbar[e] /= B; vbar[e] /= B; }
            double *ko = k_cmp + ((size_t)j * hk + g) * d;
            double *vo = v_cmp + ((size_t)j * hk + g) * d;
            apply_cmp_map(mk, d, kbar, hid, ko);
            apply_cmp_map(mv, d, vbar, hid, vo);
            if (c->round_cmp_bf16)
                for (int col = 0; col < d; ++col) {
                    ko[col] = vnsa_oracle_round_bf16(ko[col]);
                    vo[col] = vnsa_oracle_round_bf16(vo[col]);
                }
        }
        free(kbar);
    }
}

/* fp64 copies of a compression map's weights (R3 from w, or R11 from the
 * perceptron); returns 0 on allocation failure.  free_cmp_map releases them. */
static int load_cmp_map(cmp_map *mp, int d, const float *w, int hidden, const float *w1,
                        const float *b1, const float *w2, const float *b2)
{
    memset(mp, 0, sizeof(*mp));
    mp->hidden = hidden;
    if (hidden == 0) {
        double *x = malloc(sizeof(double) * (size_t)d * d);
        if (!x) return 0;
        for (size_t e = 0; e < (size_t)d * d; ++e) x[e] = w[e];
        mp->w = x;
        return 1;
    }
    const size_t n1 = (size_t)d * hidden;
    double *x = malloc(sizeof(double) * (2 * n1 + hidden + d));
    if (!x) return 0;
    for (size_t e = 0; e < n1; ++e) { x[e] = w1[e]; x[n1 + e] = w2[e]; }
    for (int e = 0; e < hidden; ++e) x[2 * n1 + e] = b1[e];
    for (int e = 0; e < d; ++e) x[2 * n1 + hidden + e] = b2[e];
    mp->w1 = x;
    mp->w2 = x + n1;
    mp->b1 = x + 2 * n1;
    mp->b2 = x + 2 * n1 + hidden;
    return 1;
}

static void free_cmp_map(cmp_map *mp)
{
    free((void *)(mp->hidden == 0 ? mp->w : mp->w1));
}

static int load_cmp_maps(cmp_map *mk, cmp_map *mv, int d, const float *w_k, const float *w_v,
                         const vnsa_oracle_cmp_mlp *mlp)
{
    int okk, okv;
    if (mlp) {
        okk = load_cmp_map(mk, d, NULL, mlp->hidden, mlp->w1_k, mlp->b1_k, mlp->w2_k, mlp->b2_k);
        okv = load_cmp_map(mv, d, NULL, mlp->hidden, mlp->w1_v, mlp->b1_v, mlp->w2_v, mlp->b2_v);
    } else {
        okk = load_cmp_map(mk, d, w_k, 0, NULL, NULL, NULL, NULL);
        okv = load_cmp_map(mv, d, w_v, 0, NULL, NULL, NULL, NULL);
    }
    if (okk && okv) return 1;
    if (okk) free_cmp_map(mk);
    if (okv) free_cmp_map(mv);
    return 0;
}

static int mlp_ok(const vnsa_oracle_cmp_mlp *m)
{
    return m && m->hidden >= 1 && m->w1_k && m->b1_k && m->w2_k && m->b2_k && m->w1_v &&
           m->b1_v && m->w2_v && m->b2_v;
}

/*
 * Top-k block selection [M]: the blocks with the highest importance are kept
 * (32 in the paper's setting), with the forced blocks and tie rule of R5.
 * imp: importance of the nvis visible blocks 0..nvis-1 of query i.
 * Writes k entries to out (ascending, -1 padded); returns the count selected.
 */
static int select_blocks(const double *imp, int nvis, int i, int B, int k,
                         int force_first, int force_local, int *out, char *taken)
{
    int cnt = 0;
    int own = i / B;
    if (force_first) out[cnt++] = 0;
    if (force_local && !(force_first && own == 0)) out[cnt++] = own;
    for (int j = 0; j < nvis; ++j) taken[j] = 0;
    for (int f = 0; f < cnt; ++f)
        if (out[f] < nvis) taken[out[f]] = 1;
    while (cnt < k) {
        int best = -1;
        for (int j = 0; j < nvis; ++j) {
            if (taken[j]) continue;
            /* strict total order: larger importance first, lower j on ties */
            if (best < 0 || imp[j] > imp[best]) best = j;
        }
        if (best < 0) break;
        taken[best] = 1;
        out[cnt++] = best;
    }
    int nsel = cnt;
    /* ascending order (insertion sort), then -1 padding */
    for (int a = 1; a < nsel; ++a) {
        int x = out[a], b = a - 1;
        while (b >= 0 && out[b] > x) { out[b + 1] = out[b]; --b; }
        out[b + 1] = x;
    }
    for (int a = nsel; a < k; ++a) out[a] = -1;
    return nsel;
}

static int pool_impl(const vnsa_oracle_cfg *c, const float *k, const float *v,
                     const uint8_t *is_vision, const float *w_k, const float *w_v,
                     const vnsa_oracle_cmp_mlp *mlp, double *k_cmp, double *v_cmp)
{
    const int n = c->n, d = c->d, hk = c->h_kv;
    int *vis = malloc(sizeof(int) * (n > 0 ? n : 1));
    double *Kd = malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * hk * d);
    double *Vd = malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * hk * d);
    cmp_map mk, mv;
    if (!vis || !Kd || !Vd || !load_cmp_maps(&mk, &mv, d, w_k, w_v, mlp)) {
        free(vis); free(Kd); free(Vd);
        return ORACLE_ENOMEM;
    }
    for (size_t x = 0; x < (size_t)n * hk * d; ++x) { Kd[x] = k[x]; Vd[x] = v[x]; }
    int nv = partition(is_vision, n, vis);
    pool_proj(c, Kd, Vd, vis, cmp_blocks(c, nv), &mk, &mv, k_cmp, v_cmp);
    free(vis); free(Kd); free(Vd); free_cmp_map(&mk); free_cmp_map(&mv);
    return ORACLE_OK;
}

/* K_cmp / V_cmp only (for the pooling parity checks). Outputs [nc][h_kv][d],
 * nc compression blocks (R13). */
int vnsa_oracle_pool_proj(const vnsa_oracle_cfg *c, const float *k, const float *v,
                          const uint8_t *is_vision, const float *w_k, const float *w_v,
                          double *k_cmp, double *v_cmp)
{
    if (!check_cfg(c) || !w_k || !w_v) return ORACLE_EINVAL;
    return pool_impl(c, k, v, is_vision, w_k, w_v, NULL, k_cmp, v_cmp);
}

/* The same with R11's compression perceptron. */
int vnsa_oracle_pool_mlp(const vnsa_oracle_cfg *c, const float *k, const float *v,
                         const uint8_t *is_vision, const vnsa_oracle_cmp_mlp *mlp,
                         double *k_cmp, double *v_cmp)
{
    if (!check_cfg(c) || !mlp_ok(mlp)) return ORACLE_EINVAL;
    return pool_impl(c, k, v, is_vision, NULL, NULL, mlp, k_cmp, v_cmp);
}

/*
 * Gate logits (R12) of n tokens: x [n][dm] (the layer input), g1 [dm][hidden],
 * c1 [hidden], g2 [hidden][n_out], c2 [n_out] -> out [n][n_out] (n_out =
 * 3 h_q, column 3h + c = branch c of head h).
 */
int vnsa_oracle_gate_mlp(int n, int dm, int hidden, int n_out, const float *x, const float *g1,
                         const float *c1, const float *g2, const float *c2,
                         int round_hidden_bf16, double *out)
{
    if (n < 0 || dm < 1 || hidden < 1 || n_out < 1 || !x || !g1 || !c1 || !g2 || !c2 || !out)
        return ORACLE_EINVAL;
    int fail = 0;
    #pragma omp parallel
    {
        double *h = malloc(sizeof(double) * (size_t)hidden);
        if (!h) {
            #pragma omp atomic write
            fail = 1;
        }
        #pragma omp for schedule(static)
        for (int t = 0; t < n; ++t) {
            if (!h) continue;
            const float *xt = x + (size_t)t * dm;
            for (int a = 0; a < hidden; ++a) {
                double z = c1[a];
                for (int e = 0; e < dm; ++e) z += (double)xt[e] * g1[(size_t)e * hidden + a];
                h[a] = silu(z);
                if (round_hidden_bf16) h[a] = vnsa_oracle_round_bf16(h[a]);
            }
            for (int o = 0; o < n_out; ++o) {
                double z = c2[o];
                for (int a = 0; a < hidden; ++a) z += h[a] * g2[(size_t)a * n_out + o];
                out[(size_t)t * n_out + o] = z;
            }
        }
        free(h);
    }
    return fail ? ORACLE_ENOMEM : ORACLE_OK;
}

/*
 * Full layer prefill for a list of query rows (global positions).
 *
 * Inputs (row-major, values already exact in fp32: bf16 inputs are widened):
 *   q [n][h_q][d], k, v [n][h_kv][d], is_vision [n], gate [n][h_q][3]
 *   (cmp, slc, swa), w_k, w_v [d][d].
 *   rows[n_rows]: global positions to compute (NULL with n_rows = n: all).
 *   forced_idx: optional [n_rows][h_kv][top_k]; when given, vision rows use these
 *   selected blocks instead of computing the top-k (used to compare a branch
 *   when the kernel legitimately swapped near-tied blocks).
 * Outputs (each optional except out), row r of the list:
 *   out [n_rows][h_q][d]                gated vision output / dense text output
 *   o_cmp, o_slc, o_swa [n_rows][h_q][d] ungated branch outputs (vision rows)
 *   lse_cmp [n_rows][h_q]               compression log-sum-exp (-inf if empty)
 *   idx [n_rows][h_kv][top_k]           selected blocks (-1 for text rows)
 *   imp [n_rows][h_kv][nb]              selection-block importance (R4, R13; 0
 *                                       beyond visibility)
 *   nb_out                              number of complete selection blocks
 */
static int forward_impl(const vnsa_oracle_cfg *c, const float *q, const float *k,
                        const float *v, const uint8_t *is_vision, const float *gate,
                        const float *w_k, const float *w_v, const vnsa_oracle_cmp_mlp *mlp,
                        int n_rows, const int *rows,
                        const int *forced_idx, double *out, double *o_cmp, double *o_slc,
                        double *o_swa, double *lse_cmp, int *idx, double *imp, int *nb_out)
{
    if (!check_cfg(c) || !q || !k || !v || !is_vision || !gate || !out) return ORACLE_EINVAL;
    if (n_rows < 0 || (!rows && n_rows != c->n)) return ORACLE_EINVAL;
    const int n = c->n, d = c->d, hq = c->h_q, hk = c->h_kv, B = c->block, K = c->top_k;
    const int r = hq / hk;
    const size_t nn = (size_t)(n > 0 ? n : 1);

    int *vis = malloc(sizeof(int) * nn);
    int *vpos = malloc(sizeof(int) * nn);
    double *Kd = malloc(sizeof(double) * nn * hk * d);
    double *Vd = malloc(sizeof(double) * nn * hk * d);
    cmp_map mk, mv;
    if (!vis || !vpos || !Kd || !Vd || !load_cmp_maps(&mk, &mv, d, w_k, w_v, mlp)) {
        free(vis); free(vpos); free(Kd); free(Vd);
        return ORACLE_ENOMEM;
    }
    for (size_t x = 0; x < (size_t)n * hk * d; ++x) { Kd[x] = k[x]; Vd[x] = v[x]; }
    const int nv = partition(is_vision, n, vis);
    for (int t = 0; t < n; ++t) vpos[t] = -1;
    for (int i = 0; i < nv; ++i) vpos[vis[i]] = i;
    const int nb = nv / B;            /* selection blocks */
    const int S = cmp_stride(c);
    const int nc = cmp_blocks(c, nv); /* compression blocks (nc = nb when S = B) */
    if (nb_out) *nb_out = nb;
    double *k_cmp = malloc(sizeof(double) * (size_t)(nc > 0 ? nc : 1) * hk * d);
    double *v_cmp = malloc(sizeof(double) * (size_t)(nc > 0 ? nc : 1) * hk * d);
    pool_proj(c, Kd, Vd, vis, nc, &mk, &mv, k_cmp, v_cmp);

    #pragma omp parallel
    {
        /* per-thread scratch: key lists, scores, probabilities, row buffers */
        int *keys = malloc(sizeof(int) * 2 * nn); /* selection list + window list */
        double *s = malloc(sizeof(double) * nn);
        double *p = malloc(sizeof(double) * nn);
        double *impg = malloc(sizeof(double) * (size_t)(nb > 0 ? nb : 1));
        double *impc = malloc(sizeof(double) * (size_t)(nc > 0 ? nc : 1));
        char *taken = malloc((size_t)(nb > 0 ? nb : 1));
        int *sel = malloc(sizeof(int) * (size_t)K);
        double *qd = malloc(sizeof(double) * d);
        double *oc = malloc(sizeof(double) * d);
        double *os = malloc(sizeof(double) * d);
        double *ow = malloc(sizeof(double) * d);

        #pragma omp for schedule(dynamic, 1)
        for (int rr = 0; rr < n_rows; ++rr) {
            const int t = rows ? rows[rr] : rr;
            const int i = vpos[t];
            double *orow = out + (size_t)rr * hq * d;
            if (i < 0) {
                /* R10: dense causal GQA over every token u <= t [M], [K]. */
                for (int u = 0; u <= t; ++u) keys[u] = u;
                for (int h = 0; h < hq; ++h) {
                    const int g = h / r;
                    for (int e = 0; e < d; ++e) qd[e] = q[((size_t)t * hq + h) * d + e];
                    attend(qd, Kd + (size_t)g * d, Vd + (size_t)g * d, (size_t)hk * d,
                           keys, t + 1, d, c->scale, orow + (size_t)h * d, NULL, s);
                    if (o_cmp) memset(o_cmp + ((size_t)rr * hq + h) * d, 0, sizeof(double) * d);
                    if (o_slc) memset(o_slc + ((size_t)rr * hq + h) * d, 0, sizeof(double) * d);
                    if (o_swa) memset(o_swa + ((size_t)rr * hq + h) * d, 0, sizeof(double) * d);
                    if (lse_cmp) lse_cmp[(size_t)rr * hq + h] = -INFINITY;
                }
                if (idx) for (int x = 0; x < hk * K; ++x) idx[(size_t)rr * hk * K + x] = -1;
                if (imp) for (int x = 0; x < hk * nb; ++x) imp[(size_t)rr * hk * nb + x] = 0.0;
                continue;
            }
            /* R2 / R13: visible compression blocks of vision query i (last
             * token at or before i), and the complete selection blocks at or
             * before i (the top-k candidates). */
            int ncv = i >= B - 1 ? (i - B + 1) / S + 1 : 0;
            if (ncv > nc) ncv = nc;
            int nvis = (i + 1) / B;
            if (nvis > nb) nvis = nb;
            for (int g = 0; g < hk; ++g) {
                /* Compression branch and importance (R4). */
                for (int j = 0; j < nb; ++j) impg[j] = 0.0;
                for (int x = 0; x < ncv; ++x) { impc[x] = 0.0; keys[x] = x; }
                for (int hl = 0; hl < r; ++hl) {
                    const int h = g * r + hl;
                    for (int e = 0; e < d; ++e) qd[e] = q[((size_t)t * hq + h) * d + e];
                    double lse = attend(qd, k_cmp + (size_t)g * d, v_cmp + (size_t)g * d,
                                        (size_t)hk * d, keys, ncv, d, c->scale, oc, p, s);
                    for (int x = 0; x < ncv; ++x) impc[x] += p[x];
                    if (lse_cmp) lse_cmp[(size_t)rr * hq + h] = lse;
                    memcpy(orow + (size_t)h * d, oc, sizeof(double) * d); /* park o_cmp */
                    if (o_cmp) memcpy(o_cmp + ((size_t)rr * hq + h) * d, oc, sizeof(double) * d);
                }
                /* R13: each compression block's mass to the selection blocks
                 * its tokens lie in, in proportion (the identity when S = B). */
                for (int x = 0; x < ncv; ++x) {
                    const int a0 = x * S, a1 = x * S + B; /* tokens [a0, a1) */
                    for (int j = a0 / B; j <= (a1 - 1) / B && j < nb; ++j) {
                        const int lo2 = a0 > j * B ? a0 : j * B;
                        const int hi2 = a1 < (j + 1) * B ? a1 : (j + 1) * B;
                        impg[j] += (double)(hi2 - lo2) / B * impc[x];
                    }
                }
                if (imp) memcpy(imp + ((size_t)rr * hk + g) * nb, impg, sizeof(double) * nb);
                /* Selection of blocks (R5), or the caller's forced indices. */
                if (forced_idx) {
                    for (int x = 0; x < K; ++x) sel[x] = forced_idx[((size_t)rr * hk + g) * K + x];
                } else {
                    select_blocks(impg, nvis, i, B, K, c->force_first, c->force_local, sel, taken);
                }
                if (idx) memcpy(idx + ((size_t)rr * hk + g) * K, sel, sizeof(int) * K);
                /* Selection key list (R6): tokens of the chosen blocks, u <= i. */
                int nk = 0;
                for (int x = 0; x < K; ++x) {
                    const int j = sel[x];
                    if (j < 0) continue;
                    for (int u = j * B; u < (j + 1) * B && u < nv && u <= i; ++u) keys[nk++] = vis[u];
                }
                /* Sliding-window key list (R7): vision tokens [i-w+1, i]. */
                int *wkeys = keys + nk;
                int nkw = 0;
                int lo = i - c->window + 1;
                if (lo < 0) lo = 0;
                for (int u = lo; u <= i; ++u) wkeys[nkw++] = vis[u];
                for (int hl = 0; hl < r; ++hl) {
                    const int h = g * r + hl;
                    for (int e = 0; e < d; ++e) qd[e] = q[((size_t)t * hq + h) * d + e];
                    attend(qd, Kd + (size_t)g * d, Vd + (size_t)g * d, (size_t)hk * d,
                           keys, nk, d, c->scale, os, NULL, s);
                    attend(qd, Kd + (size_t)g * d, Vd + (size_t)g * d, (size_t)hk * d,
                           wkeys, nkw, d, c->scale, ow, NULL, s);
                    /* Gate (R8) [M], [A]: per-head sigmoid weights of the branches. */
                    const float *gl = gate + ((size_t)t * hq + h) * 3;
                    const double gc = sigmoid(gl[0]), gs = sigmoid(gl[1]), gw = sigmoid(gl[2]);
                    double *o = orow + (size_t)h * d;
                    for (int e = 0; e < d; ++e) o[e] = gc * o[e] + gs * os[e] + gw * ow[e];
                    if (o_slc) memcpy(o_slc + ((size_t)rr * hq + h) * d, os, sizeof(double) * d);
                    if (o_swa) memcpy(o_swa + ((size_t)rr * hq + h) * d, ow, sizeof(double) * d);
                }
            }
        }
        free(keys); free(s); free(p); free(impg); free(impc); free(taken); free(sel);
        free(qd); free(oc); free(os); free(ow);
    }
    free(vis); free(vpos); free(Kd); free(Vd); free(k_cmp); free(v_cmp);
    free_cmp_map(&mk); free_cmp_map(&mv);
    return ORACLE_OK;
}

int vnsa_oracle_forward(const vnsa_oracle_cfg *c, const float *q, const float *k,
                        const float *v, const uint8_t *is_vision, const float *gate,
                        const float *w_k, const float *w_v, int n_rows, const int *rows,
                        const int *forced_idx, double *out, double *o_cmp, double *o_slc,
                        double *o_swa, double *lse_cmp, int *idx, double *imp, int *nb_out)
{
    if (!w_k || !w_v) return ORACLE_EINVAL;
    return forward_impl(c, q, k, v, is_vision, gate, w_k, w_v, NULL, n_rows, rows, forced_idx,
                        out, o_cmp, o_slc, o_swa, lse_cmp, idx, imp, nb_out);
}

/* The layer prefill with R11's compression perceptron instead of R3's map. */
int vnsa_oracle_forward_mlp(const vnsa_oracle_cfg *c, const float *q, const float *k,
                            const float *v, const uint8_t *is_vision, const float *gate,
                            const vnsa_oracle_cmp_mlp *mlp, int n_rows, const int *rows,
                            const int *forced_idx, double *out, double *o_cmp, double *o_slc,
                            double *o_swa, double *lse_cmp, int *idx, double *imp, int *nb_out)
{
    if (!mlp_ok(mlp)) return ORACLE_EINVAL;
    return forward_impl(c, q, k, v, is_vision, gate, NULL, NULL, mlp, n_rows, rows, forced_idx,
                        out, o_cmp, o_slc, o_swa, lse_cmp, idx, imp, nb_out);
}

/* Threads the OpenMP runtime will use (for the CPU-baseline report). */
int vnsa_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
