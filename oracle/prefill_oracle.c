/*
 * prefill_oracle.c -- plain fp64 CPU oracle for the prefill attention of
 * Simplified Sparse Attention (gist tokens), its block mask, and the
 * adaptive top-k budget.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * includes this file; only the tests and the bench's CPU-baseline leg use
 * it.  It shares no code, header or table with the CUDA path.
 *
 * Source: "Simplified Sparse Attention via Gist Tokens" (Mao, Li, Fox),
 *   sec. 3.1  the gist attention mask: the training/prefill sequence
 *             interleaves every chunk of C raw tokens with its g gist tokens;
 *             a token sees, causally, the tokens of its own chunk (the gists
 *             belong to the chunk they follow) and the gist tokens of every
 *             earlier chunk, and never an earlier chunk's raw tokens;
 *   sec. 3.6  prefill: the key columns are permuted so that the summary
 *             (gist) columns, visible to many rows, come before the local
 *             (raw) columns; attention then runs block-sparse over
 *             (query tile, key block) pairs, skipping the empty ones, and
 *             computes the same masked softmax;
 *   App. A    adaptive top-k: the per-level budget from n_kv, the effective
 *             compression L_eff (L for SSA, L*J for H-SSA), the group size G
 *             and the chunk size L, plus one so that a chunk is always
 *             chosen, the same k at both H-SSA levels.
 * Readings taken where the pages leave a step open (each is also listed in
 * the design notes):
 *   - the trailing raw tokens after the last complete chunk form chunk M
 *     (M = floor(n / C) complete chunks); that chunk has no gists yet;
 *   - positions: chunk m occupies [m (C+g), m (C+g) + C) with its raw tokens
 *     and the next g positions with its gists; the tail follows M (C+g);
 *   - the permuted column order is every gist (chunk-major, then gist index)
 *     followed by every raw token; the rows use the same two-part order,
 *     which is the cache layout (q, k, v each held as a raw and a gist
 *     array);
 *   - adaptive top-k: k = floor(n_kv / (L_eff * G * L)) + 1, n_kv = raw
 *     tokens in the cache.  The pages print no formula: this value is
 *     parity unpinned; only the properties they state are checked.
 *
 * Inputs are fp32 arrays (bf16 values convert to fp32 exactly); sums,
 * products and exponentials are fp64.  Layouts (row-major):
 *   q_raw [B,Hq,n_max,d], q_gist [B,Hq,M_max,g,d];
 *   k_raw, v_raw [B,Hkv,n_max,d]; k_gist, v_gist [B,Hkv,M_max,g,d];
 *   M_max = n_max / C; query head h reads KV head h / (Hq / Hkv).
 *
 * Mutants: -DORACLE_MUTANT=<n> plants one deliberate mistake (the MUT()
 * sites) so the tests can show that the pins catch it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif
#define MUT(n) (ORACLE_MUTANT == (n))

/* ------------------------------------------------------ adaptive top-k --- */

/* App. A: budget per level.  J = 1 is single-level SSA (L_eff = L); J > 1
 * is H-SSA (L_eff = L * J), whose meta-gist and gist levels use the same k.
 * Returns -1 for n_kv < 0 or L, G, J < 1. */
int64_t oracle_adaptive_topk(int64_t n_kv, int L, int G, int J) {
    if (n_kv < 0 || L < 1 || G < 1 || J < 1) return -1;
    int64_t l_eff = MUT(16) ? (int64_t)L : (int64_t)L * J;
    int64_t per = l_eff * (int64_t)G * (int64_t)L;
    int64_t k = n_kv / per;
    return MUT(15) ? k : k + 1;
}

/* ------------------------------------------------------- the gist mask --- */

/* Where a token of the split layout sits in the interleaved sequence.
 * kind 0: raw token i; kind 1: gist (m, t) given as r = m g + t. */
static int64_t position_of(int kind, int64_t idx, int C, int g, int64_t M) {
    if (kind == 0) {
        int64_t m = idx / C, s = idx % C;
        if (m >= M) return M * (C + g) + (idx - M * (int64_t)C); /* tail */
        return m * (C + g) + s + (MUT(19) ? g : 0);
    }
    int64_t m = idx / g, t = idx % g;
    return m * (C + g) + (MUT(19) ? 0 : C) + t;
}

static int64_t chunk_of(int kind, int64_t idx, int C, int g) {
    return kind == 0 ? idx / C : idx / g;
}

/* sec. 3.1: query (kq, iq) sees key (kk, ik) iff the key is not later in the
 * interleaved sequence and it is either in the query's own chunk or a gist of
 * an earlier chunk. */
static int visible(int kq, int64_t iq, int kk, int64_t ik, int C, int g, int64_t M) {
    int64_t pq = position_of(kq, iq, C, g, M), pk = position_of(kk, ik, C, g, M);
    if (pk > pq) return 0;
    int64_t mq = chunk_of(kq, iq, C, g), mk = chunk_of(kk, ik, C, g);
    if (MUT(17) && kk == 0) return 1;                  /* earlier raw leaks */
    if (MUT(18) && kq == 1 && kk == 1) return mk < mq; /* own gists hidden */
    if (mk == mq) return 1;
    return kk == 1 && mk < mq;
}

/* ---------------------------------------------------- prefill attention --- */

static const float* row_of(const float* base, int64_t heads, int64_t h, int64_t b, int64_t rows,
                           int64_t r, int d) {
    return base + (((b * heads + h) * rows + r) * (int64_t)d);
}

/* One output row: query (kq, iq) of head h, sequence b (n raw tokens), over
 * every visible key, into o[0..d). */
static void prefill_row(int Hq, int Hkv, int d, int64_t n_max, int C, int g, int b, int h,
                        int64_t n, int kq, int64_t iq, const float* q_raw, const float* q_gist,
                        const float* k_raw, const float* k_gist, const float* v_raw,
                        const float* v_gist, double scale, double* o) {
    const int G = Hq / Hkv, j = h / G;
    const int64_t M = n / C, ng = M * g, T = n + ng, gr_max = (n_max / C) * g;
    const float* q = kq ? row_of(q_gist, Hq, h, b, gr_max, iq, d)
                        : row_of(q_raw, Hq, h, b, n_max, iq, d);
    double* lg = (double*)malloc((size_t)T * sizeof(double));
    double mx = -INFINITY;
    for (int64_t ki = 0; ki < T; ++ki) {
        const int kk = ki < n ? 0 : 1;
        const int64_t ik = kk ? ki - n : ki;
        lg[ki] = -INFINITY;
        if (!visible(kq, iq, kk, ik, C, g, M)) continue;
        const float* k = kk ? row_of(k_gist, Hkv, j, b, gr_max, ik, d)
                            : row_of(k_raw, Hkv, j, b, n_max, ik, d);
        double s = 0.0;
        for (int c = 0; c < d; ++c) s += (double)q[c] * (double)k[c];
        lg[ki] = s * scale;
        if (lg[ki] > mx) mx = lg[ki];
    }
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    double den = 0.0;
    for (int64_t ki = 0; ki < T; ++ki) {
        if (lg[ki] == -INFINITY) continue;
        const int kk = ki < n ? 0 : 1;
        const int64_t ik = kk ? ki - n : ki;
        const float* v = kk ? row_of(v_gist, Hkv, j, b, gr_max, ik, d)
                            : row_of(v_raw, Hkv, j, b, n_max, ik, d);
        const double p = exp(lg[ki] - mx);
        den += p;
        for (int c = 0; c < d; ++c) o[c] += p * (double)v[c];
    }
    for (int c = 0; c < d; ++c) o[c] /= den;
    free(lg);
}

/* Dense masked softmax attention of every row of every sequence: o_raw
 * [B,Hq,n_max,d] and o_gist [B,Hq,M_max,g,d] (fp64) for rows < n_b and
 * < M_b g; other rows are left untouched.  Returns -1 on bad shapes, else the
 * number of sequences whose n_b was outside [0, n_max] (skipped). */
int oracle_prefill(int B, int Hq, int Hkv, int d, int n_max, int C, int g,
                   const int32_t* seq_lens, const float* q_raw, const float* q_gist,
                   const float* k_raw, const float* k_gist, const float* v_raw,
                   const float* v_gist, double* o_raw, double* o_gist) {
    if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || d < 1 || C < 1 || g < 1 || n_max < 0 ||
        n_max % C)
        return -1;
    const int64_t M_max = n_max / C, gr_max = M_max * g;
    const double scale = MUT(20) ? 1.0 : 1.0 / sqrt((double)d);
    int bad = 0;
    for (int b = 0; b < B; ++b) {
        const int64_t n = seq_lens[b];
        if (n < 0 || n > n_max) {
            ++bad;
            continue;
        }
        const int64_t M = n / C, ng = M * g, T = n + ng;
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
        for (int h = 0; h < Hq; ++h) {
            for (int64_t qi = 0; qi < T; ++qi) {
                const int kq = qi < n ? 0 : 1;
                const int64_t iq = kq ? qi - n : qi;
                double* o = kq ? o_gist + (((int64_t)b * Hq + h) * gr_max + iq) * d
                               : o_raw + (((int64_t)b * Hq + h) * n_max + iq) * d;
                prefill_row(Hq, Hkv, d, n_max, C, g, b, h, n, kq, iq, q_raw, q_gist, k_raw,
                            k_gist, v_raw, v_gist, scale, o);
            }
        }
    }
    return bad;
}

/* The same rows for a list of queries only: query i is sequence rows[4 i],
 * head rows[4 i + 1], part rows[4 i + 2] (0 raw, 1 gist), row rows[4 i + 3];
 * its output goes to out[i * d ..].  Returns -1 on bad shapes or a query
 * outside the sequence, else 0. */
int oracle_prefill_rows(int B, int Hq, int Hkv, int d, int n_max, int C, int g,
                        const int32_t* seq_lens, const float* q_raw, const float* q_gist,
                        const float* k_raw, const float* k_gist, const float* v_raw,
                        const float* v_gist, int64_t n_rows, const int32_t* rows, double* out) {
    if (B < 0 || Hq < 1 || Hkv < 1 || Hq % Hkv || d < 1 || C < 1 || g < 1 || n_max < 0 ||
        n_max % C)
        return -1;
    for (int64_t i = 0; i < n_rows; ++i) {
        const int b = rows[4 * i], h = rows[4 * i + 1], kq = rows[4 * i + 2];
        const int64_t r = rows[4 * i + 3];
        if (b < 0 || b >= B || h < 0 || h >= Hq || (kq != 0 && kq != 1) || r < 0) return -1;
        const int64_t n = seq_lens[b];
        if (n < 0 || n > n_max || r >= (kq ? (n / C) * g : n)) return -1;
    }
    const double scale = MUT(20) ? 1.0 : 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < n_rows; ++i)
        prefill_row(Hq, Hkv, d, n_max, C, g, rows[4 * i], rows[4 * i + 1], seq_lens[rows[4 * i]],
                    rows[4 * i + 2], rows[4 * i + 3], q_raw, q_gist, k_raw, k_gist, v_raw,
                    v_gist, scale, out + i * d);
    return 0;
}

/* ----------------------------------------------------------- block mask --- */

/* Block mask of one sequence of n raw tokens over the permuted layout (sec.
 * 3.6), found by testing every (row, column) pair of the mask above.  Query
 * tiles: BM consecutive rows of one part (raw rows first, then gist rows),
 * tile r0 = BM * tile index; key blocks: BN consecutive columns of one part.
 * A block is listed for a tile when one of its pairs is visible; it is full
 * when the tile's valid rows see all BN of its columns (every column then
 * exists), else partial.  Per tile (in order: raw tiles, gist tiles) writes 4
 * ints to tiles: kind, r0, rows (valid rows), entry count; its entries follow
 * the previous tile's in entries as (block << 2) | (part << 1) | full, part 0
 * = gist columns, listed first (ascending), then part 1 = raw columns.
 * There are ceil(n / BM) + ceil(M g / BM) tiles.  Returns the number of
 * entries written, or -1 if a capacity is exceeded. */
int64_t oracle_prefill_blocks(int64_t n, int C, int g, int BM, int BN, int32_t* tiles,
                              int64_t tiles_cap, int32_t* entries, int64_t entries_cap) {
    if (n < 0 || C < 1 || g < 1 || BM < 1 || BN < 1) return -1;
    const int64_t M = n / C, ng = M * g;
    const int64_t count[2] = {n, ng};
    int64_t nt = 0, ne = 0;
    for (int kq = 0; kq < 2; ++kq) {
        for (int64_t r0 = 0; r0 < count[kq]; r0 += BM) {
            const int64_t rows = count[kq] - r0 < BM ? count[kq] - r0 : BM;
            if (nt >= tiles_cap) return -1;
            int64_t listed = 0;
            for (int part = 0; part < 2; ++part) {
                const int kk = part == 0 ? 1 : 0; /* gist columns first */
                const int64_t cols = count[kk];
                for (int64_t c0 = 0; c0 < cols; c0 += BN) {
                    int64_t seen = 0;
                    for (int64_t r = r0; r < r0 + rows; ++r)
                        for (int64_t c = c0; c < c0 + BN && c < cols; ++c)
                            seen += visible(kq, r, kk, c, C, g, M);
                    if (!seen) continue;
                    int full = seen == rows * (int64_t)BN;
                    if (MUT(21)) full = seen == rows * ((c0 + BN < cols ? c0 + BN : cols) - c0);
                    if (ne >= entries_cap) return -1;
                    entries[ne++] = (int32_t)(((c0 / BN) << 2) | (part << 1) | full);
                    ++listed;
                }
            }
            tiles[4 * nt + 0] = kq;
            tiles[4 * nt + 1] = (int32_t)r0;
            tiles[4 * nt + 2] = (int32_t)rows;
            tiles[4 * nt + 3] = (int32_t)listed;
            ++nt;
        }
    }
    return ne;
}
