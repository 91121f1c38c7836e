/*
 * ssa_oracle.c -- plain fp64 CPU oracle for the decode step of Simplified
 * Sparse Attention (gist tokens), single level and two level (gist-of-gist).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * includes this file; only the tests, the package smoke check and the bench's
 * CPU-baseline leg use it.  It shares no code, header or table with the CUDA
 * path.
 *
 * Source: "Simplified Sparse Attention via Gist Tokens" (Mao, Li, Fox),
 *   sec. 3.2  gist-based relevance scoring (query . gist key dot products),
 *   sec. 3.3  top-k chunk selection and hybrid attention over the unfolded
 *             context,
 *   sec. 3.5 / App. B.2  coarse-to-fine (gist-of-gist) selection,
 *   sec. 3.6  split-K partial attention + combination compute the same
 *             softmax as the single pass written here.
 * Readings taken where the pages leave a step open (each is also listed in
 * the design notes):
 *   - chunk score = max over the GQA group's query heads and the chunk's g
 *     gist tokens of q.k / sqrt(d); the selection is shared by the group;
 *   - ties go to the lower chunk index; NaN scores rank as -inf;
 *   - context = gist K/V of the unselected complete chunks + raw K/V of every
 *     token of the selected chunks + raw K/V of the incomplete tail chunk
 *     (the selected chunks' own gists are not in it);
 *   - two level: meta-gist K/V of unselected complete superchunks + gist K/V
 *     of unselected candidate chunks (children of selected superchunks plus
 *     the remainder chunks that belong to no complete superchunk) + raw K/V
 *     of the selected chunks + tail;
 *   - seq_lens counts every cached raw token; all of them are visible.
 * Variants (oracle_decode_v):
 *   - context "selected only" (sec. 3.3 read literally: a selected chunk
 *     brings both its gists and its raw tokens, and the other chunks are
 *     left out): gist K/V and raw K/V of the selected chunks + raw K/V of
 *     the tail; unselected chunks contribute nothing;
 *   - selection "per head + union" (App. A: the heads choose their chunks
 *     separately and the group unfolds their union): every query head scores the
 *     chunks with its own query only (max over the chunk's g gist tokens of
 *     q_h.k / sqrt(d)) and keeps its own top-k (ties to the lower index); the
 *     KV head's selection is the union of its group's selections, ascending,
 *     and every head of the group attends over the context it defines.
 *
 * Inputs are fp32 arrays (bf16 values convert to fp32 exactly); every sum,
 * product and exponential is fp64.  Layouts (row-major):
 *   q [B,Hq,d]; k_raw, v_raw [B,Hkv,n_max,d]; k_gist, v_gist [B,Hkv,M_max,g,d]
 *   (M_max = n_max / C); k_meta, v_meta [B,Hkv,S_max,gm,d] (S_max = M_max / J).
 *
 * Mutants: building with -DORACLE_MUTANT=<n> plants one deliberate mistake
 * (see the MUT() sites) so the tests can show that the pins catch it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif
#define MUT(n) (ORACLE_MUTANT == (n))

typedef struct {
    int B, Hq, Hkv, d, n_max, C, g;
} oshape;

static int ok_shape(const oshape* s) {
    if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->d < 1 || s->C < 1 || s->g < 1) return 0;
    if (s->Hq % s->Hkv) return 0;
    if (s->n_max < 1 || s->n_max % s->C) return 0;
    return 1;
}

/* Number of cached raw tokens of sequence b, or -1 if outside [1, n_max]. */
static int seq_len(const oshape* s, const int32_t* seq_lens, int b) {
    int n = seq_lens[b];
    if (n < 1 || n > s->n_max) return -1;
    return n;
}

static double dot(const float* a, const float* b, int d) {
    double acc = 0.0;
    for (int i = 0; i < d; ++i) acc += (double)a[i] * (double)b[i];
    return acc;
}

static double scale_of(int d) {
    if (MUT(1)) return 1.0;           /* mutant 1: scale dropped from scoring */
    return 1.0 / sqrt((double)d);
}

/* Score of one summary slot: max over the group's query heads and the slot's
 * `ntok` summary tokens (rows[0..ntok)) of q.k * scale (sec. 3.2; aggregation
 * reading above). */
static double slot_score(const oshape* s, const float* q, int b, int j, const float* const* rows,
                         int ntok) {
    const int G = s->Hq / s->Hkv;
    const double sc = scale_of(s->d);
    double best = -INFINITY;
    for (int gh = 0; gh < G; ++gh) {
        if (MUT(6) && gh > 0) break;  /* mutant 6: only the group's first head */
        const int h = MUT(8) ? (j + gh * s->Hkv) : (j * G + gh); /* mutant 8: wrong head map */
        const float* qh = q + ((size_t)b * s->Hq + h) * s->d;
        for (int t = 0; t < ntok; ++t) {
            double v = dot(qh, rows[t], s->d) * sc;
            if (v > best) best = v;
        }
    }
    return best;
}

static const float* gist_row(const oshape* s, const float* base, int b, int j, int m, int t) {
    const int M_max = s->n_max / s->C;
    if (MUT(10)) /* mutant 10: gist index transposed (t-major instead of chunk-major) */
        return base + ((((size_t)b * s->Hkv + j) * M_max * s->g) + (size_t)t * M_max + m) * s->d;
    return base + ((((size_t)b * s->Hkv + j) * M_max + m) * s->g + t) * s->d;
}

static const float* raw_row(const oshape* s, const float* base, int b, int j, int i) {
    return base + (((size_t)b * s->Hkv + j) * s->n_max + i) * s->d;
}


static double chunk_score(const oshape* s, const float* q, const float* k_gist, int b, int j,
                          int m) {
    const float** r = (const float**)malloc(sizeof(float*) * (size_t)s->g);
    for (int t = 0; t < s->g; ++t) r[t] = gist_row(s, k_gist, b, j, m, t);
    double v = slot_score(s, q, b, j, r, s->g);
    free((void*)r);
    return v;
}

/* Per-head score of chunk m of KV head j (selection variant "per head +
 * union", App. A): max over the chunk's g gist tokens of q_h.k * scale for
 * the single query head h of the group. */
static double head_score(const oshape* s, const float* q, const float* k_gist, int b, int j,
                         int h, int m) {
    const double sc = scale_of(s->d);
    const float* qh = q + ((size_t)b * s->Hq + h) * s->d;
    double best = -INFINITY;
    for (int t = 0; t < s->g; ++t) {
        double v = dot(qh, gist_row(s, k_gist, b, j, m, t), s->d) * sc;
        if (v > best) best = v;
    }
    return best;
}

static double super_score(const oshape* s, const float* q, const float* k_meta, int S_max,
                          int gm, int b, int j, int x) {
    const float** r = (const float**)malloc(sizeof(float*) * (size_t)gm);
    for (int t = 0; t < gm; ++t)
        r[t] = k_meta + ((((size_t)b * s->Hkv + j) * S_max + x) * gm + t) * s->d;
    double v = slot_score(s, q, b, j, r, gm);
    free((void*)r);
    return v;
}

/* ---------------------------------------------------------------- top-k --- */

typedef struct {
    double v;
    int i;
} keyed;

/* Order: larger score first; equal scores -> lower index first (tie reading).
 * NaN ranks as -inf. */
static int cmp_desc(const void* pa, const void* pb) {
    const keyed* a = (const keyed*)pa;
    const keyed* b = (const keyed*)pb;
    double va = isnan(a->v) ? -INFINITY : a->v;
    double vb = isnan(b->v) ? -INFINITY : b->v;
    if (va > vb) return -1;
    if (va < vb) return 1;
    if (MUT(3)) return (a->i > b->i) ? -1 : (a->i < b->i); /* mutant 3: ties to higher index */
    return (a->i < b->i) ? -1 : (a->i > b->i);
}

static int cmp_int(const void* pa, const void* pb) {
    int a = *(const int*)pa, b = *(const int*)pb;
    return (a > b) - (a < b);
}

/* The k largest of vals[cand[0..n)] (sec. 3.3 top-k), written ascending by
 * index into out[0..k), padded with -1 up to `cap`.  Returns k. */
static int topk_of(const double* vals, const int* cand, int n, int topk, int* out, int cap) {
    int k = topk < n ? topk : n;
    if (k < 0) k = 0;
    keyed* tmp = (keyed*)malloc(sizeof(keyed) * (size_t)(n > 0 ? n : 1));
    for (int c = 0; c < n; ++c) {
        tmp[c].v = vals[cand[c]];
        tmp[c].i = cand[c];
    }
    qsort(tmp, (size_t)n, sizeof(keyed), cmp_desc);
    for (int c = 0; c < k; ++c) out[c] = tmp[c].i;
    if (!MUT(11)) qsort(out, (size_t)k, sizeof(int), cmp_int); /* mutant 11: not re-sorted */
    for (int c = k; c < cap; ++c) out[c] = -1;
    free(tmp);
    return k;
}

/* ------------------------------------------------------------- attention --- */

/* Softmax attention of one query head over an explicit list of (key, value)
 * row pointers: out = sum_x softmax_x(q.k_x * scale) v_x, with the maximum
 * subtracted before exponentiation.  Writes out[d] and the log-sum-exp. */
static void attend_list(const float* qh, int d, const float** ks, const float** vs, int n,
                        double* out, double* lse) {
    const double sc = MUT(2) ? 1.0 : 1.0 / sqrt((double)d); /* mutant 2: no attention scale */
    for (int i = 0; i < d; ++i) out[i] = 0.0;
    if (n == 0) {
        *lse = -INFINITY;
        return;
    }
    double* logit = (double*)malloc(sizeof(double) * (size_t)n);
    double mx = -INFINITY;
    for (int x = 0; x < n; ++x) {
        logit[x] = dot(qh, ks[x], d) * sc;
        if (logit[x] > mx) mx = logit[x];
    }
    double den = 0.0;
    for (int x = 0; x < n; ++x) {
        double p = exp(logit[x] - mx);
        den += p;
        for (int i = 0; i < d; ++i) out[i] += p * (double)vs[x][i];
    }
    for (int i = 0; i < d; ++i) out[i] /= den;
    *lse = mx + log(den);
    free(logit);
}

/* Append the raw rows [lo, hi) of (b, j) to the context list. */
static int push_raw(const oshape* s, const float* k_raw, const float* v_raw, int b, int j, int lo,
                    int hi, const float** ks, const float** vs, int n) {
    for (int i = lo; i < hi; ++i) {
        ks[n] = raw_row(s, k_raw, b, j, i);
        vs[n] = raw_row(s, v_raw, b, j, i);
        ++n;
    }
    return n;
}

static int is_in(const int* sorted, int k, int m) {
    for (int c = 0; c < k; ++c)
        if (sorted[c] == m) return 1;
    return 0;
}

/* ----------------------------------------------------- single level path --- */

/*
 * oracle_decode_v: the whole single-level decode step, with the context and
 * selection readings chosen by context_mode (0: unselected gists + selected
 * raw + tail; 1: selected gists + selected raw + tail) and select_mode (0:
 * one selection per KV head from the max over its group's heads; 1: per-head
 * top-k, union over the group).
 *   scores  [B,Hkv,M_max] (select_mode 0) or [B,Hq,M_max] (select_mode 1):
 *           chunk scores, -inf for m >= M_b                          (out)
 *   sel     [B,Hkv,cap]    selected chunks ascending, -1 padded; cap = topk
 *                          (select_mode 0) or G * topk (select_mode 1) (in/out)
 *   out     [B,Hq,d]       attention output                         (out)
 *   lse     [B,Hq]         natural log-sum-exp of the logits         (out)
 *   ctx     [B,Hkv]        context size |X| of each (b, j)           (out)
 * force_sel != 0: `sel` is an input (a given selection, e.g. the GPU's at a
 * near tie) and only the attention step runs on it.
 * Returns 0, or -1 for a bad shape or mode, or 1 + b for a bad seq_lens[b]
 * (that sequence's outputs are zero, its selections -1).
 */
int oracle_decode_v(int B, int Hq, int Hkv, int d, int n_max, int C, int g, int topk,
                    int context_mode, int select_mode, const float* q, const float* k_raw,
                    const float* v_raw, const float* k_gist, const float* v_gist,
                    const int32_t* seq_lens, int force_sel, double* scores, int32_t* sel,
                    double* out, double* lse, int32_t* ctx) {
    oshape s = {B, Hq, Hkv, d, n_max, C, g};
    if (!ok_shape(&s) || topk < 0) return -1;
    if (context_mode < 0 || context_mode > 1 || select_mode < 0 || select_mode > 1) return -1;
    const int G = Hq / Hkv;
    const int M_max = n_max / C;
    const int cap = select_mode ? G * topk : topk;
    int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int j = 0; j < Hkv; ++j) {
            const int n = seq_len(&s, seq_lens, b);
            const size_t pj = (size_t)b * Hkv + j;
            /* score rows of this pair: one (select_mode 0) or G (one per head) */
            const int nrows = select_mode ? G : 1;
            double* sc = scores ? scores + pj * (size_t)nrows * M_max : NULL;
            int32_t* sl = sel + pj * (size_t)cap;
            if (n < 0) {
#pragma omp critical
                if (!bad || b + 1 < bad) bad = b + 1;
                for (int m = 0; m < nrows * M_max && sc; ++m) sc[m] = -INFINITY;
                if (!force_sel)
                    for (int c = 0; c < cap; ++c) sl[c] = -1;
                for (int gh = 0; gh < G; ++gh) {
                    const size_t h = (size_t)b * Hq + (size_t)j * G + gh;
                    for (int i = 0; i < d; ++i) out[h * d + i] = 0.0;
                    if (lse) lse[h] = -INFINITY;
                }
                if (ctx) ctx[pj] = 0;
                continue;
            }
            const int M = n / C;       /* complete chunks */
            const int tail0 = M * C;   /* first tail token */
            double* own = (double*)malloc(sizeof(double) * (size_t)(M_max > 0 ? M_max : 1));
            int* chosen = (int*)malloc(sizeof(int) * (size_t)(cap > 0 ? cap : 1));
            int* all = (int*)malloc(sizeof(int) * (size_t)(M > 0 ? M : 1));
            for (int m = 0; m < M; ++m) all[m] = m;
            if (!force_sel)
                for (int c = 0; c < cap; ++c) sl[c] = -1;
            int nch = 0; /* select_mode 1: size of the union so far, in chosen[] */
            for (int r = 0; r < nrows; ++r) {
                /* select_mode 0: the group's score; 1: query head j*G + r's own */
                for (int m = 0; m < M_max; ++m) own[m] = -INFINITY;
                for (int m = 0; m < M; ++m)
                    own[m] = select_mode ? head_score(&s, q, k_gist, b, j, j * G + r, m)
                                         : chunk_score(&s, q, k_gist, b, j, m);
                if (sc)
                    for (int m = 0; m < M_max; ++m) sc[(size_t)r * M_max + m] = own[m];
                if (force_sel) continue;
                if (!select_mode) {
                    topk_of(own, all, M, topk, sl, topk);
                } else if (r == 0 || !MUT(12)) { /* mutant 12: union of head 0 only */
                    int* mine = (int*)malloc(sizeof(int) * (size_t)(topk > 0 ? topk : 1));
                    const int kh = topk_of(own, all, M, topk, mine, topk);
                    for (int c = 0; c < kh; ++c)
                        if (!is_in(chosen, nch, mine[c])) chosen[nch++] = mine[c];
                    free(mine);
                }
            }
            if (select_mode && !force_sel) {
                qsort(chosen, (size_t)nch, sizeof(int), cmp_int);
                for (int c = 0; c < cap; ++c) sl[c] = c < nch ? chosen[c] : -1;
            }
            int k = 0;
            for (int c = 0; c < cap; ++c)
                if (sl[c] >= 0) chosen[k++] = sl[c];
            free(all);
            /* context list (sec. 3.3, reading above, or the variant) */
            const int xcap = (M * g) + M * C + C + 8;
            const float** ks = (const float**)malloc(sizeof(float*) * (size_t)xcap);
            const float** vs = (const float**)malloc(sizeof(float*) * (size_t)xcap);
            int nx = 0;
            for (int m = 0; m < M; ++m) {
                const int selected = is_in(chosen, k, m);
                int gists;
                if (!context_mode)
                    gists = !selected || MUT(4); /* mutant 4: selected chunks keep their gists */
                else
                    gists = selected && !MUT(13); /* mutant 13: variant drops selected gists */
                if (gists) {
                    for (int t = 0; t < g; ++t) {
                        ks[nx] = gist_row(&s, k_gist, b, j, m, t);
                        vs[nx] = gist_row(&s, v_gist, b, j, m, t);
                        ++nx;
                    }
                }
                if (selected) nx = push_raw(&s, k_raw, v_raw, b, j, m * C, m * C + C, ks, vs, nx);
            }
            if (!MUT(5)) /* mutant 5: tail dropped; mutant 7: tail starts one late */
                nx = push_raw(&s, k_raw, v_raw, b, j, tail0 + (MUT(7) ? 1 : 0), n, ks, vs, nx);
            if (ctx) ctx[pj] = nx;
            for (int gh = 0; gh < G; ++gh) {
                const size_t h = (size_t)b * Hq + (size_t)j * G + gh;
                double l;
                attend_list(q + h * d, d, ks, vs, nx, out + h * d, &l);
                if (lse) lse[h] = l;
            }
            free(ks);
            free(vs);
            free(chosen);
            free(own);
        }
    }
    return bad;
}

/* oracle_decode: the step under the default readings (context_mode 0,
 * select_mode 0), sel [B,Hkv,topk]. */
int oracle_decode(int B, int Hq, int Hkv, int d, int n_max, int C, int g, int topk,
                  const float* q, const float* k_raw, const float* v_raw, const float* k_gist,
                  const float* v_gist, const int32_t* seq_lens, int force_sel, double* scores,
                  int32_t* sel, double* out, double* lse, int32_t* ctx) {
    return oracle_decode_v(B, Hq, Hkv, d, n_max, C, g, topk, 0, 0, q, k_raw, v_raw, k_gist,
                           v_gist, seq_lens, force_sel, scores, sel, out, lse, ctx);
}

/* ------------------------------------------------------- two level path --- */

/*
 * oracle_decode_h2: two-level (gist-of-gist) decode step (sec. 3.5, App. B.2).
 * Level 2 scores the S_b = floor(M_b / J) complete superchunks with their gm
 * meta-gist keys and keeps the top topk_super; the candidates are the J
 * children of each kept superchunk plus the remainder chunks S_b*J .. M_b-1;
 * level 1 scores the candidates with their gist keys and keeps the top
 * topk_chunk.  Outputs:
 *   super_scores [B,Hkv,S_max] (-inf past S_b), chunk_scores [B,Hkv,M_max]
 *   (-inf for non-candidates), sel_super [B,Hkv,topk_super],
 *   sel [B,Hkv,topk_chunk], out, lse, ctx as in oracle_decode.
 * force_sel bit 0: sel_super is given; bit 1: sel is given.
 */
int oracle_decode_h2(int B, int Hq, int Hkv, int d, int n_max, int C, int g, int J, int gm,
                     int topk_super, int topk_chunk, const float* q, const float* k_raw,
                     const float* v_raw, const float* k_gist, const float* v_gist,
                     const float* k_meta, const float* v_meta, const int32_t* seq_lens,
                     int force_sel, double* super_scores, double* chunk_scores,
                     int32_t* sel_super, int32_t* sel, double* out, double* lse, int32_t* ctx) {
    oshape s = {B, Hq, Hkv, d, n_max, C, g};
    if (!ok_shape(&s) || J < 1 || gm < 1 || topk_super < 0 || topk_chunk < 0) return -1;
    const int G = Hq / Hkv;
    const int M_max = n_max / C;
    const int S_max = M_max / J;
    int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int j = 0; j < Hkv; ++j) {
            const int n = seq_len(&s, seq_lens, b);
            const size_t pj = (size_t)b * Hkv + j;
            int32_t* ss = sel_super + pj * (size_t)topk_super;
            int32_t* sl = sel + pj * (size_t)topk_chunk;
            double* s2 = super_scores ? super_scores + pj * (size_t)S_max : NULL;
            double* s1 = chunk_scores ? chunk_scores + pj * (size_t)M_max : NULL;
            if (n < 0) {
#pragma omp critical
                if (!bad || b + 1 < bad) bad = b + 1;
                if (!(force_sel & 1))
                    for (int c = 0; c < topk_super; ++c) ss[c] = -1;
                if (!(force_sel & 2))
                    for (int c = 0; c < topk_chunk; ++c) sl[c] = -1;
                for (int x = 0; x < S_max && s2; ++x) s2[x] = -INFINITY;
                for (int x = 0; x < M_max && s1; ++x) s1[x] = -INFINITY;
                for (int gh = 0; gh < G; ++gh) {
                    const size_t h = (size_t)b * Hq + (size_t)j * G + gh;
                    for (int i = 0; i < d; ++i) out[h * d + i] = 0.0;
                    if (lse) lse[h] = -INFINITY;
                }
                if (ctx) ctx[pj] = 0;
                continue;
            }
            const int M = n / C;
            const int S = M / J;   /* complete superchunks */
            const int tail0 = M * C;
            /* level 2 */
            double* sup = (double*)malloc(sizeof(double) * (size_t)(S_max > 0 ? S_max : 1));
            for (int x = 0; x < S_max; ++x) sup[x] = -INFINITY;
            for (int x = 0; x < S; ++x)
                sup[x] = super_score(&s, q, k_meta, S_max, gm, b, j, x);
            if (s2)
                for (int x = 0; x < S_max; ++x) s2[x] = sup[x];
            int* ksel = (int*)malloc(sizeof(int) * (size_t)(topk_super > 0 ? topk_super : 1));
            int ks_n;
            if (force_sel & 1) {
                ks_n = 0;
                for (int c = 0; c < topk_super; ++c)
                    if (ss[c] >= 0) ksel[ks_n++] = ss[c];
            } else {
                int* all = (int*)malloc(sizeof(int) * (size_t)(S > 0 ? S : 1));
                for (int x = 0; x < S; ++x) all[x] = x;
                ks_n = topk_of(sup, all, S, topk_super, ksel, topk_super);
                for (int c = 0; c < topk_super; ++c) ss[c] = ksel[c];
                free(all);
            }
            /* candidates, ascending */
            int* cand = (int*)malloc(sizeof(int) * (size_t)(M > 0 ? M : 1));
            int nc = 0;
            for (int c = 0; c < ks_n; ++c)
                for (int i = 0; i < J; ++i) cand[nc++] = ksel[c] * J + i;
            for (int m = S * J; m < M; ++m) cand[nc++] = m;
            /* level 1 */
            double* own = (double*)malloc(sizeof(double) * (size_t)(M_max > 0 ? M_max : 1));
            for (int m = 0; m < M_max; ++m) own[m] = -INFINITY;
            for (int c = 0; c < nc; ++c)
                own[cand[c]] = chunk_score(&s, q, k_gist, b, j, cand[c]);
            if (s1)
                for (int m = 0; m < M_max; ++m) s1[m] = own[m];
            int* csel = (int*)malloc(sizeof(int) * (size_t)(topk_chunk > 0 ? topk_chunk : 1));
            int kc_n;
            if (force_sel & 2) {
                kc_n = 0;
                for (int c = 0; c < topk_chunk; ++c)
                    if (sl[c] >= 0) csel[kc_n++] = sl[c];
            } else {
                kc_n = topk_of(own, cand, nc, topk_chunk, csel, topk_chunk);
                for (int c = 0; c < topk_chunk; ++c) sl[c] = csel[c];
            }
            /* context */
            const int cap = S * gm + nc * g + kc_n * C + C + 8;
            const float** kx = (const float**)malloc(sizeof(float*) * (size_t)cap);
            const float** vx = (const float**)malloc(sizeof(float*) * (size_t)cap);
            int nx = 0;
            for (int x = 0; x < S; ++x) {
                if (is_in(ksel, ks_n, x)) continue;
                for (int t = 0; t < gm; ++t) {
                    const size_t r = ((((size_t)b * Hkv + j) * S_max + x) * gm + t) * d;
                    kx[nx] = k_meta + r;
                    vx[nx] = v_meta + r;
                    ++nx;
                }
            }
            for (int c = 0; c < nc; ++c) {
                const int m = cand[c];
                if (is_in(csel, kc_n, m)) {
                    nx = push_raw(&s, k_raw, v_raw, b, j, m * C, m * C + C, kx, vx, nx);
                } else {
                    for (int t = 0; t < g; ++t) {
                        kx[nx] = gist_row(&s, k_gist, b, j, m, t);
                        vx[nx] = gist_row(&s, v_gist, b, j, m, t);
                        ++nx;
                    }
                }
            }
            nx = push_raw(&s, k_raw, v_raw, b, j, tail0, n, kx, vx, nx);
            if (ctx) ctx[pj] = nx;
            for (int gh = 0; gh < G; ++gh) {
                const size_t h = (size_t)b * Hq + (size_t)j * G + gh;
                double l;
                attend_list(q + h * d, d, kx, vx, nx, out + h * d, &l);
                if (lse) lse[h] = l;
            }
            free(kx);
            free(vx);
            free(csel);
            free(own);
            free(cand);
            free(ksel);
            free(sup);
        }
    }
    return bad;
}

/* ------------------------------------------------------ t level path --- */

/*
 * oracle_decode_hier: coarse-to-fine selection over `levels` = t levels
 * (sec. 3.5: more levels of summaries as the context grows; App. B.2,
 * t = ceil(log_J M) levels), the two-level reading applied level by
 * level.  Level-1 units are the chunks (g gist tokens each).  A level-l unit
 * (l >= 2) groups J level-(l-1) units and has gs[l-2] summary tokens in
 * k_sum[l-2], v_sum[l-2] laid out [B,Hkv,Umax(l),gs[l-2],d] with Umax(l) =
 * M_max / J^(l-1).  Complete units: U_1 = M_b, U_l = floor(U_{l-1} / J).
 * From the top: the candidates of level t are its U_t units; those of level
 * l < t are the J children of every unit kept at level l+1 (ascending), then
 * the remainder units U_{l+1} J .. U_l - 1, which lie in no complete parent.
 * Each level keeps the topks[l-1] best candidates (score = max over the
 * group's query heads and the unit's summary tokens of q.k/sqrt(d); ties to
 * the lower index).  Context: the summary tokens of every unkept candidate
 * at levels >= 2, the gists of the unkept candidate chunks, the raw tokens of
 * the kept chunks and the raw tail.
 *   scores[l-1] [B,Hkv,Umax(l)]  candidate scores, -inf elsewhere      (out)
 *   sels[l-1]   [B,Hkv,topks[l-1]] kept units ascending, -1 padded  (in/out)
 *   out, lse, ctx as in oracle_decode.  force_sel != 0: every level's
 *   selection is given in sels.
 * Returns 0, -1 for bad arguments, or 1 + b for a bad seq_lens[b].
 */
#define ORACLE_MAX_LEVELS 8
int oracle_decode_hier(int B, int Hq, int Hkv, int d, int n_max, int C, int g, int J, int levels,
                       const int32_t* gs, const int32_t* topks, const float* q,
                       const float* k_raw, const float* v_raw, const float* k_gist,
                       const float* v_gist, const float* const* k_sum,
                       const float* const* v_sum, const int32_t* seq_lens, int force_sel,
                       double* const* scores, int32_t* const* sels, double* out, double* lse,
                       int32_t* ctx) {
    oshape s = {B, Hq, Hkv, d, n_max, C, g};
    if (!ok_shape(&s) || J < 1 || levels < 1 || levels > ORACLE_MAX_LEVELS) return -1;
    for (int l = 0; l < levels; ++l)
        if (topks[l] < 0 || (l > 0 && gs[l - 1] < 1)) return -1;
    const int G = Hq / Hkv;
    const int M_max = n_max / C;
    int umax[ORACLE_MAX_LEVELS];
    umax[0] = M_max;
    for (int l = 1; l < levels; ++l) umax[l] = umax[l - 1] / J;
    int bad = 0;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int j = 0; j < Hkv; ++j) {
            const int n = seq_len(&s, seq_lens, b);
            const size_t pj = (size_t)b * Hkv + j;
            if (n < 0) {
#pragma omp critical
                if (!bad || b + 1 < bad) bad = b + 1;
                for (int l = 0; l < levels; ++l) {
                    for (int x = 0; x < umax[l] && scores && scores[l]; ++x)
                        scores[l][pj * (size_t)umax[l] + x] = -INFINITY;
                    if (!force_sel)
                        for (int c = 0; c < topks[l]; ++c) sels[l][pj * (size_t)topks[l] + c] = -1;
                }
                for (int gh = 0; gh < G; ++gh) {
                    const size_t h = (size_t)b * Hq + (size_t)j * G + gh;
                    for (int i = 0; i < d; ++i) out[h * d + i] = 0.0;
                    if (lse) lse[h] = -INFINITY;
                }
                if (ctx) ctx[pj] = 0;
                continue;
            }
            const int M = n / C;
            int U[ORACLE_MAX_LEVELS];
            U[0] = M;
            for (int l = 1; l < levels; ++l) U[l] = U[l - 1] / J;
            /* context capacity: every candidate's summaries or raw tokens */
            size_t xcap = (size_t)M * (g + C) + C + 8;
            for (int l = 1; l < levels; ++l) xcap += (size_t)(U[l - 1] + 1) * gs[l - 1];
            const float** kx = (const float**)malloc(sizeof(float*) * xcap);
            const float** vx = (const float**)malloc(sizeof(float*) * xcap);
            int nx = 0;
            int* kept = NULL;   /* units kept at the level above, ascending */
            int nkept = 0;
            for (int l = levels - 1; l >= 0; --l) {
                /* candidates of level l + 1 (1-based) */
                const int ncap = (l == levels - 1) ? U[l] : nkept * J + U[l];
                int* cand = (int*)malloc(sizeof(int) * (size_t)(ncap > 0 ? ncap : 1));
                int nc = 0;
                if (l == levels - 1) {
                    for (int x = 0; x < U[l]; ++x) cand[nc++] = x;
                } else {
                    for (int c = 0; c < nkept; ++c)
                        for (int i = 0; i < J; ++i) cand[nc++] = kept[c] * J + i;
                    if (!MUT(14)) /* mutant 14: remainder units never candidates */
                        for (int x = U[l + 1] * J; x < U[l]; ++x) cand[nc++] = x;
                }
                double* sc = (double*)malloc(sizeof(double) * (size_t)(umax[l] > 0 ? umax[l] : 1));
                for (int x = 0; x < umax[l]; ++x) sc[x] = -INFINITY;
                for (int c = 0; c < nc; ++c) {
                    const int x = cand[c];
                    sc[x] = l == 0 ? chunk_score(&s, q, k_gist, b, j, x)
                                   : super_score(&s, q, k_sum[l - 1], umax[l], gs[l - 1], b, j, x);
                }
                if (scores && scores[l])
                    for (int x = 0; x < umax[l]; ++x) scores[l][pj * (size_t)umax[l] + x] = sc[x];
                int32_t* sl = sels[l] + pj * (size_t)topks[l];
                int* keep = (int*)malloc(sizeof(int) * (size_t)(topks[l] > 0 ? topks[l] : 1));
                int nk;
                if (force_sel) {
                    nk = 0;
                    for (int c = 0; c < topks[l]; ++c)
                        if (sl[c] >= 0) keep[nk++] = sl[c];
                } else {
                    nk = topk_of(sc, cand, nc, topks[l], keep, topks[l]);
                    for (int c = 0; c < topks[l]; ++c) sl[c] = keep[c];
                }
                /* context of this level */
                for (int c = 0; c < nc; ++c) {
                    const int x = cand[c];
                    const int picked = is_in(keep, nk, x);
                    if (l == 0) {
                        if (picked) {
                            nx = push_raw(&s, k_raw, v_raw, b, j, x * C, x * C + C, kx, vx, nx);
                        } else {
                            for (int t = 0; t < g; ++t) {
                                kx[nx] = gist_row(&s, k_gist, b, j, x, t);
                                vx[nx] = gist_row(&s, v_gist, b, j, x, t);
                                ++nx;
                            }
                        }
                    } else if (!picked) {
                        for (int t = 0; t < gs[l - 1]; ++t) {
                            const size_t r =
                                ((((size_t)b * Hkv + j) * umax[l] + x) * gs[l - 1] + t) * d;
                            kx[nx] = k_sum[l - 1] + r;
                            vx[nx] = v_sum[l - 1] + r;
                            ++nx;
                        }
                    }
                }
                free(sc);
                free(cand);
                free(kept);
                kept = keep;
                nkept = nk;
            }
            free(kept);
            nx = push_raw(&s, k_raw, v_raw, b, j, M * C, n, kx, vx, nx);
            if (ctx) ctx[pj] = nx;
            for (int gh = 0; gh < G; ++gh) {
                const size_t h = (size_t)b * Hq + (size_t)j * G + gh;
                double l2;
                attend_list(q + h * d, d, kx, vx, nx, out + h * d, &l2);
                if (lse) lse[h] = l2;
            }
            free(kx);
            free(vx);
        }
    }
    return bad;
}

int oracle_mutant_id(void) { return ORACLE_MUTANT; }
