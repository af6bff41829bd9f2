/*
 * bsa_oracle.c -- plain CPU oracle for block-sparse compressed-key decode attention.
 *
 * TEST INFRASTRUCTURE. Only the tests, the package's smoke check and the benchmark's CPU-baseline
 * leg may load this library; the CUDA library shares no code with it. Each function follows one
 * step of the method in double precision; the sources and the readings of the pages are listed in
 * bsa_oracle.h. Build: gcc -O2 -std=c11 -fopenmp -ffp-contract=off -shared -fPIC.
 */
#include "bsa_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

double bsa_oracle_load(const void* base, int dtype, int64_t i) {
    if (dtype == ORC_F32) return (double)((const float*)base)[i];
    /* bf16 is the upper half of an IEEE binary32 pattern */
    uint32_t bits = (uint32_t)((const uint16_t*)base)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

double bsa_oracle_round(double x, int dtype) {
    if (dtype == ORC_F32) return (double)(float)x; /* C conversion: nearest, ties to even */
    if (x == 0.0 || isnan(x) || isinf(x)) return x;
    /* bf16: 8 significant bits, binary32 exponent range (normal from 2^-126, subnormal step 2^-133) */
    int e;
    frexp(x, &e); /* |x| in [2^(e-1), 2^e) */
    int lead = e - 1;
    if (lead < -126) lead = -126;
    double quantum = ldexp(1.0, lead - 7);
    double r = rint(x / quantum) * quantum; /* rint: nearest, ties to even (default mode) */
    if (fabs(r) >= ldexp(1.0, 128)) r = copysign(INFINITY, x);
    return r;
}

void bsa_oracle_round_array(const double* x, int64_t n, int dtype, double* y) {
    for (int64_t i = 0; i < n; ++i) y[i] = bsa_oracle_round(x[i], dtype);
}

int64_t bsa_oracle_num_windows(int64_t T, int l, int s) {
    if (T < l) return 0;
    return (T - l) / s + 1;
}

int64_t bsa_oracle_num_blocks(int64_t T, int block_size) {
    return (T + block_size - 1) / block_size;
}

/* Theoretical Foundation, Eq. (2): K~_j = Mean(K[j*s : j*s + l]). */
int64_t bsa_oracle_compress(const void* k, int dtype, int64_t T, int d, int l, int s,
                            int round_dtype, double* ck) {
    int64_t nc = bsa_oracle_num_windows(T, l, s);
    for (int64_t j = 0; j < nc; ++j) {
        for (int c = 0; c < d; ++c) {
            double sum = 0.0;
            for (int r = 0; r < l; ++r) sum += bsa_oracle_load(k, dtype, (j * s + r) * (int64_t)d + c);
            double mean = sum / (double)l;
            ck[j * d + c] = (round_dtype == ORC_NO_ROUND) ? mean : bsa_oracle_round(mean, round_dtype);
        }
    }
    return nc;
}

/* Indexer Training, Eq. (6), target side: S = sum over the group's heads of softmax(q_h K~^T / tau). */
void bsa_oracle_group_scores(const double* q, const double* ck, int64_t nc, int G, int d,
                             double tau, double* S) {
    for (int64_t j = 0; j < nc; ++j) S[j] = 0.0;
    if (nc <= 0) return;
    double* x = (double*)malloc((size_t)nc * sizeof(double));
    for (int h = 0; h < G; ++h) {
        double m = -INFINITY;
        for (int64_t j = 0; j < nc; ++j) {
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += q[h * d + c] * ck[j * d + c];
            x[j] = dot / tau;
            if (x[j] > m) m = x[j];
        }
        double z = 0.0;
        for (int64_t j = 0; j < nc; ++j) z += exp(x[j] - m);
        for (int64_t j = 0; j < nc; ++j) S[j] += exp(x[j] - m) / z;
    }
    free(x);
}

/* SparDA Architecture, Eq. (4), with the Compact Forecast Indexer: one Forecast vector f per GQA
 * group scores every compressed key as f . K~_j, with no softmax. */
void bsa_oracle_forecast_scores(const double* f, const double* ck, int64_t nc, int d, double* S) {
    for (int64_t j = 0; j < nc; ++j) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += f[c] * ck[j * d + c];
        S[j] = dot;
    }
}

/* Fine-grained supervision: scores max-pooled down to the standard block grid. A window overlaps
 * block b when it shares at least one token with [BS*b, BS*(b+1)). */
void bsa_oracle_block_scores(const double* S, int64_t nc, int64_t nb, int l, int s,
                             int block_size, double* sb) {
    for (int64_t b = 0; b < nb; ++b) {
        double best = -INFINITY;
        for (int64_t j = 0; j < nc; ++j) {
            int64_t first = j * s, end = j * s + l; /* tokens [first, end) */
            if (first < (int64_t)block_size * (b + 1) && end > (int64_t)block_size * b) {
                if (S[j] > best) best = S[j];
            }
        }
        sb[b] = best;
    }
}

typedef struct {
    double score;
    int64_t block;
} orc_cand_t;

/* Higher score first; equal scores: lower block index first. */
static int orc_cand_cmp(const void* pa, const void* pb) {
    const orc_cand_t* a = (const orc_cand_t*)pa;
    const orc_cand_t* b = (const orc_cand_t*)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->block < b->block) ? -1 : (a->block > b->block);
}

/* Theoretical Foundation, Eq. (1), with SparDA Architecture, Eq. (4)'s f_top(., k). */
int bsa_oracle_select(const double* sb, int64_t nb, int n_init, int n_local, int top_k,
                      int32_t* idx, double* boundary) {
    boundary[0] = NAN;
    boundary[1] = NAN;
    if (nb <= 0) return 0;
    char* chosen = (char*)calloc((size_t)nb, 1);
    int64_t init_end = n_init < nb ? n_init : nb;
    int64_t local_begin = nb - n_local > 0 ? nb - n_local : 0;
    for (int64_t b = 0; b < init_end; ++b) chosen[b] = 1;
    for (int64_t b = local_begin; b < nb; ++b) chosen[b] = 1;

    orc_cand_t* cand = (orc_cand_t*)malloc((size_t)nb * sizeof(orc_cand_t));
    int64_t nc = 0;
    for (int64_t b = 0; b < nb; ++b) {
        if (!chosen[b]) {
            cand[nc].score = sb[b];
            cand[nc].block = b;
            ++nc;
        }
    }
    qsort(cand, (size_t)nc, sizeof(orc_cand_t), orc_cand_cmp);
    int64_t take = top_k < nc ? top_k : nc;
    for (int64_t i = 0; i < take; ++i) chosen[cand[i].block] = 1;
    if (take > 0) boundary[0] = cand[take - 1].score;
    if (take < nc) boundary[1] = cand[take].score;

    int n = 0;
    for (int64_t b = 0; b < nb; ++b)
        if (chosen[b]) idx[n++] = (int32_t)b;
    free(cand);
    free(chosen);
    return n;
}

/* SparDA Architecture, Eq. (5): O = Attn(Q, K[B], V[B]) over the tokens of the selected blocks. */
void bsa_oracle_attend(const double* q, const void* k, const void* v, int dtype, int64_t T, int d,
                       int G, const int32_t* idx, int n_sel, int block_size, double scale,
                       double* out, double* lse) {
    /* list the attended tokens */
    int64_t n_tok = 0;
    for (int i = 0; i < n_sel; ++i) {
        if (idx[i] < 0) continue; /* -1 marks an unused slot */
        int64_t lo = (int64_t)idx[i] * block_size, hi = lo + block_size;
        if (hi > T) hi = T;
        if (hi > lo) n_tok += hi - lo;
    }
    int64_t* tok = (int64_t*)malloc((size_t)(n_tok > 0 ? n_tok : 1) * sizeof(int64_t));
    double* x = (double*)malloc((size_t)(n_tok > 0 ? n_tok : 1) * sizeof(double));
    int64_t n = 0;
    for (int i = 0; i < n_sel; ++i) {
        if (idx[i] < 0) continue;
        int64_t lo = (int64_t)idx[i] * block_size, hi = lo + block_size;
        if (hi > T) hi = T;
        for (int64_t t = lo; t < hi; ++t) tok[n++] = t;
    }
    for (int h = 0; h < G; ++h) {
        double* o = out + (int64_t)h * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        if (n_tok == 0) {
            lse[h] = -INFINITY;
            continue;
        }
        double m = -INFINITY;
        for (int64_t i = 0; i < n_tok; ++i) {
            double dot = 0.0;
            for (int c = 0; c < d; ++c) dot += q[h * d + c] * bsa_oracle_load(k, dtype, tok[i] * d + c);
            x[i] = dot * scale;
            if (x[i] > m) m = x[i];
        }
        double z = 0.0;
        for (int64_t i = 0; i < n_tok; ++i) z += exp(x[i] - m);
        for (int64_t i = 0; i < n_tok; ++i) {
            double w = exp(x[i] - m) / z;
            for (int c = 0; c < d; ++c) o[c] += w * bsa_oracle_load(v, dtype, tok[i] * d + c);
        }
        lse[h] = m + log(z);
    }
    free(tok);
    free(x);
}

static int orc_problem_ok(const orc_problem_t* P) {
    if (!P) return 0;
    if (P->batch < 1 || P->num_kv_heads < 1 || P->num_q_heads < 1) return 0;
    if (P->num_q_heads % P->num_kv_heads) return 0;
    if (P->head_dim < 1 || P->cmp_kernel < 1 || P->cmp_stride < 1 || P->block_size < 1) return 0;
    if (P->n_init < 0 || P->n_local < 0 || P->top_k < 0 || P->max_seq_len < 1) return 0;
    if (P->dtype != ORC_F32 && P->dtype != ORC_BF16) return 0;
    return 1;
}

static size_t orc_elem_size(int dtype) { return dtype == ORC_F32 ? 4 : 2; }

/* q rows of one group as doubles: heads kvh*G .. kvh*G + G - 1 of batch b. */
static void orc_group_q(const orc_problem_t* P, const void* q, int b, int kvh, double* qg) {
    int G = P->num_q_heads / P->num_kv_heads, d = P->head_dim;
    for (int h = 0; h < G; ++h)
        for (int c = 0; c < d; ++c)
            qg[h * d + c] = bsa_oracle_load(
                q, P->dtype, ((int64_t)b * P->num_q_heads + (int64_t)kvh * G + h) * d + c);
}

static const void* orc_pair_rows(const orc_problem_t* P, const void* cache, int pair) {
    size_t off = (size_t)pair * (size_t)P->max_seq_len * (size_t)P->head_dim * orc_elem_size(P->dtype);
    return (const char*)cache + off;
}

/* Select (from q, or from the Forecast vectors f when given) and attend, per listed pair. The
 * compressed keys are formed from the cache (Eq. 2), or taken from ck_given [n_pairs][nc_cap][d]
 * (already rounded, as bsa_oracle_compress_cache writes them) when that is not NULL. With out ==
 * NULL (and f and ck_given given) only the selection runs: q, k_cache and v_cache are not read. */
static int orc_decode(const orc_problem_t* P, const void* f, const void* q, const void* k_cache,
                      const void* v_cache, const double* ck_given, const int32_t* seq_lens,
                      const int32_t* pairs, int n_pairs, const int32_t* given_idx,
                      const int32_t* given_n_sel, int32_t* idx, int32_t* n_sel,
                      double* block_scores, double* boundary, double* out, double* lse) {
    if (!orc_problem_ok(P) || n_pairs < 0) return -1;
    const int G = P->num_q_heads / P->num_kv_heads, d = P->head_dim;
    const int sel_cap = P->n_init + P->n_local + P->top_k;
    const int64_t nb_cap = bsa_oracle_num_blocks(P->max_seq_len, P->block_size);
    for (int i = 0; i < n_pairs; ++i) {
        if (pairs[i] < 0 || pairs[i] >= P->batch * P->num_kv_heads) return -1;
        int64_t T = seq_lens[pairs[i] / P->num_kv_heads];
        if (T < 0 || T > P->max_seq_len) return -1;
    }
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int i = 0; i < n_pairs; ++i) {
        const int pair = pairs[i], b = pair / P->num_kv_heads, kvh = pair % P->num_kv_heads;
        const int64_t T = seq_lens[b];
        const int64_t nb = bsa_oracle_num_blocks(T, P->block_size);
        const int attend = out != NULL;
        const void* kp = attend || !ck_given ? orc_pair_rows(P, k_cache, pair) : NULL;
        const void* vp = attend ? orc_pair_rows(P, v_cache, pair) : NULL;
        double* qg = (double*)malloc((size_t)G * d * sizeof(double));
        if (attend || !f) orc_group_q(P, q, b, kvh, qg);
        int32_t* my_idx = idx + (int64_t)i * sel_cap;
        for (int r = 0; r < sel_cap; ++r) my_idx[r] = -1;
        int ns;
        double* bs = block_scores ? block_scores + (int64_t)i * nb_cap : NULL;
        if (bs)
            for (int64_t r = 0; r < nb_cap; ++r) bs[r] = -INFINITY;
        if (boundary) {
            boundary[2 * i] = NAN;
            boundary[2 * i + 1] = NAN;
        }
        if (given_idx) {
            ns = given_n_sel[i];
            if (ns < 0 || ns > sel_cap) {
                bad |= 1;
                ns = 0;
            }
            for (int r = 0; r < ns; ++r) my_idx[r] = given_idx[(int64_t)i * sel_cap + r];
        } else {
            int64_t nc = bsa_oracle_num_windows(T, P->cmp_kernel, P->cmp_stride);
            const int64_t nc_cap = bsa_oracle_num_windows(P->max_seq_len, P->cmp_kernel, P->cmp_stride);
            double* ck_own = ck_given ? NULL : (double*)malloc((size_t)(nc > 0 ? nc : 1) * d * sizeof(double));
            const double* ck = ck_given ? ck_given + (int64_t)i * nc_cap * d : ck_own;
            double* S = (double*)malloc((size_t)(nc > 0 ? nc : 1) * sizeof(double));
            double* sb = (double*)malloc((size_t)(nb > 0 ? nb : 1) * sizeof(double));
            double bnd[2];
            if (!ck_given) bsa_oracle_compress(kp, P->dtype, T, d, P->cmp_kernel, P->cmp_stride, P->dtype, ck_own);
            if (f) {
                double* fv = (double*)malloc((size_t)d * sizeof(double));
                for (int c = 0; c < d; ++c) fv[c] = bsa_oracle_load(f, P->dtype, (int64_t)pair * d + c);
                bsa_oracle_forecast_scores(fv, ck, nc, d, S);
                free(fv);
            } else {
                bsa_oracle_group_scores(qg, ck, nc, G, d, P->tau, S);
            }
            bsa_oracle_block_scores(S, nc, nb, P->cmp_kernel, P->cmp_stride, P->block_size, sb);
            ns = bsa_oracle_select(sb, nb, P->n_init, P->n_local, P->top_k, my_idx, bnd);
            if (bs)
                for (int64_t r = 0; r < nb; ++r) bs[r] = sb[r];
            if (boundary) {
                boundary[2 * i] = bnd[0];
                boundary[2 * i + 1] = bnd[1];
            }
            free(ck_own);
            free(S);
            free(sb);
        }
        n_sel[i] = ns;
        if (attend)
            bsa_oracle_attend(qg, kp, vp, P->dtype, T, d, G, my_idx, ns, P->block_size, P->scale,
                              out + (int64_t)i * G * d, lse + (int64_t)i * G);
        free(qg);
    }
    return bad ? -1 : 0;
}

int bsa_oracle_decode(const orc_problem_t* P, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* seq_lens, const int32_t* pairs,
                      int n_pairs, const int32_t* given_idx, const int32_t* given_n_sel,
                      int32_t* idx, int32_t* n_sel, double* block_scores, double* boundary,
                      double* out, double* lse) {
    return orc_decode(P, NULL, q, k_cache, v_cache, NULL, seq_lens, pairs, n_pairs, given_idx,
                      given_n_sel, idx, n_sel, block_scores, boundary, out, lse);
}

/* bsa_oracle_decode with the compressed keys of the listed pairs given (ck [n_pairs][nc_cap][d],
 * e.g. from bsa_oracle_compress_cache): a decode step on a cache whose keys were compressed
 * beforehand, as at decode time. */
int bsa_oracle_decode_ck(const orc_problem_t* P, const void* q, const double* ck,
                         const void* k_cache, const void* v_cache, const int32_t* seq_lens,
                         const int32_t* pairs, int n_pairs, int32_t* idx, int32_t* n_sel,
                         double* block_scores, double* boundary, double* out, double* lse) {
    if (!ck) return -1;
    return orc_decode(P, NULL, q, k_cache, v_cache, ck, seq_lens, pairs, n_pairs, NULL, NULL, idx,
                      n_sel, block_scores, boundary, out, lse);
}

/* SparDA Architecture: the blocks of Eq. (4), selected with the Forecast vectors f [B][Hkv][d]
 * (one per GQA group), attended by the queries q as in Eq. (5). */
int bsa_oracle_decode_forecast(const orc_problem_t* P, const void* f, const void* q,
                               const void* k_cache, const void* v_cache, const int32_t* seq_lens,
                               const int32_t* pairs, int n_pairs, int32_t* idx, int32_t* n_sel,
                               double* block_scores, double* boundary, double* out, double* lse) {
    if (!f) return -1;
    return orc_decode(P, f, q, k_cache, v_cache, NULL, seq_lens, pairs, n_pairs, NULL, NULL, idx,
                      n_sel, block_scores, boundary, out, lse);
}

/* bsa_oracle_decode_forecast with the listed pairs' compressed keys given, as bsa_oracle_decode_ck. */
int bsa_oracle_decode_forecast_ck(const orc_problem_t* P, const void* f, const void* q, const double* ck,
                                  const void* k_cache, const void* v_cache, const int32_t* seq_lens,
                                  const int32_t* pairs, int n_pairs, int32_t* idx, int32_t* n_sel,
                                  double* block_scores, double* boundary, double* out, double* lse) {
    if (!f || !ck) return -1;
    return orc_decode(P, f, q, k_cache, v_cache, ck, seq_lens, pairs, n_pairs, NULL, NULL, idx, n_sel,
                      block_scores, boundary, out, lse);
}

/* The selection of bsa_oracle_decode_forecast_ck alone (SparDA Architecture, Eq. 4): the blocks
 * that the Forecast vectors f choose among the given compressed keys ck; with one-layer lookahead
 * (the abstract's lookahead selection) f is layer l's and ck layer l + 1's. */
int bsa_oracle_select_forecast_ck(const orc_problem_t* P, const void* f, const double* ck,
                                  const int32_t* seq_lens, const int32_t* pairs, int n_pairs,
                                  int32_t* idx, int32_t* n_sel, double* block_scores, double* boundary) {
    if (!f || !ck) return -1;
    return orc_decode(P, f, NULL, NULL, NULL, ck, seq_lens, pairs, n_pairs, NULL, NULL, idx, n_sel,
                      block_scores, boundary, NULL, NULL);
}

/* Block-sparse prefill of a chunk (page "SparDA: Sparse Decoupled Attention for Efficient
 * Long-Context LLM Inference", Theoretical Foundation, Eq. 1, with the selection made per query
 * tile as in the tile-level operations of the page "CoSA: Accelerating Long-Context Inference via
 * Proxy-Kernel Co-Designed Sparse Attention", Kascade abstract). The chunk's C queries of sequence b
 * sit at positions T - C .. T - 1 (T = seq_lens[b], the chunk's keys and values already in the
 * cache). Query tile r holds the chunk's positions inside block r; for each (tile, kv head):
 *   scores: S[j] = sum over the tile's positions and the group's heads of softmax_j(q . K~_j / tau),
 *           over the windows complete before the tile's block begins (s j + l <= BS r), Eq. 6;
 *   blocks: the maximum of S over the windows overlapping each block, blocks 0 .. r ("Fine-grained
 *           supervision"), and the selection of Eq. 1 among those r + 1 blocks (init, local = the
 *           last n_local of them, top-k by score with ties to the lower block);
 *   attention: the query at position p attends the selected blocks' tokens u <= p (Eq. 5).
 * q is [B][C][Hq][d]; idx [n][tiles_cap][sel_cap], n_sel [n][tiles_cap] (tile i of pair i0 is
 * block (T - C) / BS + i; tiles past the chunk are -1 / 0), boundary [n][tiles_cap][2] (as in the
 * decode driver: the k-th taken and the best rejected block score; may be NULL); out [n][C][G][d],
 * lse [n][C][G] for the listed pairs. Returns 0, or -1 on an invalid argument. */
int bsa_oracle_prefill(const orc_problem_t* P, const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* seq_lens, int chunk, const int32_t* pairs, int n_pairs, int tiles_cap,
                       int32_t* idx, int32_t* n_sel, double* boundary, double* out, double* lse) {
    if (!orc_problem_ok(P) || n_pairs < 0 || chunk < 1 || tiles_cap < 1) return -1;
    const int G = P->num_q_heads / P->num_kv_heads, d = P->head_dim, BS = P->block_size;
    const int sel_cap = P->n_init + P->n_local + P->top_k;
    for (int i = 0; i < n_pairs; ++i) {
        if (pairs[i] < 0 || pairs[i] >= P->batch * P->num_kv_heads) return -1;
        const int64_t T = seq_lens[pairs[i] / P->num_kv_heads];
        if (T < chunk || T > P->max_seq_len) return -1;
        if ((T - 1) / BS - (T - chunk) / BS + 1 > tiles_cap) return -1;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n_pairs; ++i) {
        const int pair = pairs[i], b = pair / P->num_kv_heads, kvh = pair % P->num_kv_heads;
        const int64_t T = seq_lens[b], t0 = T - chunk;
        const void* kp = orc_pair_rows(P, k_cache, pair);
        const void* vp = orc_pair_rows(P, v_cache, pair);
        const int64_t nc_all = bsa_oracle_num_windows(T, P->cmp_kernel, P->cmp_stride);
        double* ck = (double*)malloc((size_t)(nc_all > 0 ? nc_all : 1) * d * sizeof(double));
        bsa_oracle_compress(kp, P->dtype, T, d, P->cmp_kernel, P->cmp_stride, P->dtype, ck);
        double* qg = (double*)malloc((size_t)G * d * sizeof(double));
        double* S = (double*)malloc((size_t)(nc_all > 0 ? nc_all : 1) * sizeof(double));
        double* St = (double*)malloc((size_t)(nc_all > 0 ? nc_all : 1) * sizeof(double));
        const int64_t r_lo = t0 / BS, r_hi = (T - 1) / BS;
        double* sb = (double*)malloc((size_t)(r_hi + 1) * sizeof(double));
        for (int ti = 0; ti < tiles_cap; ++ti) {
            int32_t* my_idx = idx + ((int64_t)i * tiles_cap + ti) * sel_cap;
            for (int r = 0; r < sel_cap; ++r) my_idx[r] = -1;
            n_sel[(int64_t)i * tiles_cap + ti] = 0;
            if (boundary) boundary[2 * ((int64_t)i * tiles_cap + ti)] = boundary[2 * ((int64_t)i * tiles_cap + ti) + 1] = NAN;
        }
        for (int64_t r = r_lo; r <= r_hi; ++r) {
            /* windows complete before block r begins: s j + l <= BS r */
            int64_t nc = bsa_oracle_num_windows(BS * r, P->cmp_kernel, P->cmp_stride);
            if (nc > nc_all) nc = nc_all;
            const int64_t p_lo = t0 > BS * r ? t0 : BS * r, p_hi = T < BS * (r + 1) ? T : BS * (r + 1);
            for (int64_t j = 0; j < nc; ++j) S[j] = 0.0;
            for (int64_t p = p_lo; p < p_hi; ++p) {
                for (int h = 0; h < G; ++h)
                    for (int c = 0; c < d; ++c)
                        qg[h * d + c] = bsa_oracle_load(q, P->dtype,
                                                        (((int64_t)b * chunk + (p - t0)) * P->num_q_heads + (int64_t)kvh * G + h) * d + c);
                bsa_oracle_group_scores(qg, ck, nc, G, d, P->tau, St);
                for (int64_t j = 0; j < nc; ++j) S[j] += St[j];
            }
            const int64_t nb = r + 1;
            bsa_oracle_block_scores(S, nc, nb, P->cmp_kernel, P->cmp_stride, BS, sb);
            int32_t* my_idx = idx + ((int64_t)i * tiles_cap + (r - r_lo)) * sel_cap;
            double bnd[2];
            const int ns = bsa_oracle_select(sb, nb, P->n_init, P->n_local, P->top_k, my_idx, bnd);
            n_sel[(int64_t)i * tiles_cap + (r - r_lo)] = ns;
            if (boundary) {
                boundary[2 * ((int64_t)i * tiles_cap + (r - r_lo))] = bnd[0];
                boundary[2 * ((int64_t)i * tiles_cap + (r - r_lo)) + 1] = bnd[1];
            }
            for (int64_t p = p_lo; p < p_hi; ++p) {
                for (int h = 0; h < G; ++h)
                    for (int c = 0; c < d; ++c)
                        qg[h * d + c] = bsa_oracle_load(q, P->dtype,
                                                        (((int64_t)b * chunk + (p - t0)) * P->num_q_heads + (int64_t)kvh * G + h) * d + c);
                /* causal: the tokens of the selected blocks before and at p */
                bsa_oracle_attend(qg, kp, vp, P->dtype, p + 1, d, G, my_idx, ns, BS, P->scale,
                                  out + (((int64_t)i * chunk + (p - t0)) * G) * d,
                                  lse + ((int64_t)i * chunk + (p - t0)) * G);
            }
        }
        free(ck);
        free(qg);
        free(S);
        free(St);
        free(sb);
    }
    return 0;
}

/* The token-level index of the CLSA abstract (page "HySparse2: Hybrid Sparse Attention with
 * Two-Level KV Sharing"): one indexer selects tokens once and every layer sharing it attends them.
 * The indexer is the base selector (Eq. 6 of the SparDA page's Indexer Training) at token
 * granularity: S[t] = sum over the group's heads of softmax_t(q_h . K_t / tau) over the tokens
 * t < T of the index layer's keys. The first n_init * BS and the last n_local * BS tokens are always
 * taken, and top_k * BS more by score (ties to the lower token), ascending: Eq. 1 with blocks of one
 * token and the block configuration's token budget. idx [n][tok_cap] (-1 padded, tok_cap =
 * (n_init + n_local + top_k) * BS), n_sel [n], boundary [n][2] and the token scores
 * scores [n][max_seq_len] (-inf past T) (both may be NULL). */
int bsa_oracle_token_select(const orc_problem_t* P, const void* q, const void* k_cache, const int32_t* seq_lens,
                            const int32_t* pairs, int n_pairs, int32_t* idx, int32_t* n_sel, double* boundary,
                            double* scores) {
    if (!orc_problem_ok(P) || n_pairs < 0) return -1;
    const int G = P->num_q_heads / P->num_kv_heads, d = P->head_dim, BS = P->block_size;
    const int tok_cap = (P->n_init + P->n_local + P->top_k) * BS;
    for (int i = 0; i < n_pairs; ++i) {
        if (pairs[i] < 0 || pairs[i] >= P->batch * P->num_kv_heads) return -1;
        const int64_t T = seq_lens[pairs[i] / P->num_kv_heads];
        if (T < 0 || T > P->max_seq_len) return -1;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n_pairs; ++i) {
        const int pair = pairs[i], b = pair / P->num_kv_heads, kvh = pair % P->num_kv_heads;
        const int64_t T = seq_lens[b];
        const void* kp = orc_pair_rows(P, k_cache, pair);
        double* keys = (double*)malloc((size_t)(T > 0 ? T : 1) * d * sizeof(double));
        for (int64_t t = 0; t < T * d; ++t) keys[t] = bsa_oracle_load(kp, P->dtype, t);
        double* qg = (double*)malloc((size_t)G * d * sizeof(double));
        orc_group_q(P, q, b, kvh, qg);
        double* S = (double*)malloc((size_t)(T > 0 ? T : 1) * sizeof(double));
        bsa_oracle_group_scores(qg, keys, T, G, d, P->tau, S);
        int32_t* my_idx = idx + (int64_t)i * tok_cap;
        for (int r = 0; r < tok_cap; ++r) my_idx[r] = -1;
        double bnd[2];
        n_sel[i] = bsa_oracle_select(S, T, P->n_init * BS, P->n_local * BS, P->top_k * BS, my_idx, bnd);
        if (boundary) {
            boundary[2 * i] = bnd[0];
            boundary[2 * i + 1] = bnd[1];
        }
        if (scores)
            for (int64_t t = 0; t < P->max_seq_len; ++t) scores[(int64_t)i * P->max_seq_len + t] = t < T ? S[t] : -INFINITY;
        free(keys);
        free(qg);
        free(S);
    }
    return 0;
}

int bsa_oracle_attend_pairs(const orc_problem_t* P, const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* seq_lens, const int32_t* pairs,
                            int n_pairs, const int32_t* idx, const int32_t* n_sel, double* out,
                            double* lse) {
    if (!orc_problem_ok(P) || n_pairs < 0) return -1;
    const int sel_cap = P->n_init + P->n_local + P->top_k;
    /* the decode driver copies the given indices into its idx output; give it scratch for that */
    int32_t* idx_copy = (int32_t*)malloc((size_t)(n_pairs > 0 ? n_pairs : 1) * sel_cap * sizeof(int32_t) + 4);
    int32_t* nsel_copy = (int32_t*)malloc((size_t)(n_pairs > 0 ? n_pairs : 1) * sizeof(int32_t));
    int rc = bsa_oracle_decode(P, q, k_cache, v_cache, seq_lens, pairs, n_pairs, idx, n_sel,
                               idx_copy, nsel_copy, NULL, NULL, out, lse);
    free(idx_copy);
    free(nsel_copy);
    return rc;
}

int bsa_oracle_compress_cache(const orc_problem_t* P, const void* k_cache,
                              const int32_t* seq_lens, const int32_t* pairs, int n_pairs,
                              double* ck) {
    if (!orc_problem_ok(P) || n_pairs < 0) return -1;
    const int d = P->head_dim;
    const int64_t nc_cap = bsa_oracle_num_windows(P->max_seq_len, P->cmp_kernel, P->cmp_stride);
    for (int i = 0; i < n_pairs; ++i) {
        if (pairs[i] < 0 || pairs[i] >= P->batch * P->num_kv_heads) return -1;
        int64_t T = seq_lens[pairs[i] / P->num_kv_heads];
        if (T < 0 || T > P->max_seq_len) return -1;
    }
#pragma omp parallel for schedule(dynamic, 1)
    for (int i = 0; i < n_pairs; ++i) {
        const int pair = pairs[i];
        const int64_t T = seq_lens[pair / P->num_kv_heads];
        double* dst = ck + (int64_t)i * nc_cap * d;
        for (int64_t r = 0; r < nc_cap * d; ++r) dst[r] = 0.0;
        bsa_oracle_compress(orc_pair_rows(P, k_cache, pair), P->dtype, T, d, P->cmp_kernel,
                            P->cmp_stride, P->dtype, dst);
    }
    return 0;
}

/* Threads of the OpenMP loops over pairs (n >= 1); timing only, no effect on the results. */
void bsa_oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n >= 1) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int bsa_oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
