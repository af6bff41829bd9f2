/*
 * bsa_oracle.h -- plain CPU oracle for block-sparse compressed-key decode attention.
 *
 * TEST INFRASTRUCTURE. Only the tests, the package's smoke check and the benchmark's CPU-baseline
 * leg may load this library. The CUDA library never includes this header, never links this code
 * and shares no helper, table or constant with it.
 *
 * Everything is computed in IEEE double precision, in the order the method states it, with no
 * blocking, fusion or reordering. Element tensors that the GPU sees in bf16 or fp32 are read in
 * their storage format and widened to double on load.
 *
 * Method sources (page title, then section / equation):
 *   [SparDA] "SparDA: Sparse Decoupled Attention for Efficient Long-Context LLM Inference"
 *            (picx.dev summary of arXiv 2606.04511)
 *       - Theoretical Foundation, Eq. (1): block set = init blocks U local blocks U top-k blocks.
 *       - Theoretical Foundation, Eq. (2): compressed key = mean of K over a window of
 *         l = 32 rows starting at stride s = 16.
 *       - SparDA Architecture, Eq. (4): f_top, the top-k of the block scores; the Forecast F_l of
 *         layer l scores the compressed keys of layer l + 1 (F_l K~^T).
 *       - SparDA Architecture, "Compact Forecast Indexer": one Forecast head per GQA group, and no
 *         softmax normalisation of its scores.
 *       - SparDA Architecture, Eq. (5): exact attention over the selected blocks only.
 *       - Indexer Training, Eq. (6): the original selector's score of a GQA group is the sum over the
 *         group's heads of softmax(q_h K~^T / tau).
 *       - Indexer Training, "Fine-grained supervision": compressed scores are max-pooled down to the
 *         standard block grid.
 *   [CLSA]   page "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing", first abstract:
 *            one routing index computed once and reused across layers.
 *   [Kascade] page "CoSA: Accelerating Long-Context Inference via Proxy-Kernel Co-Designed Sparse
 *            Attention", second abstract: exact top-k in an anchor layer, reused in later layers.
 *
 * Readings where the pages leave a step open (each one is fixed here and listed in the design notes):
 *   - tau in Eq. (6) is sqrt(head_dim), the attention temperature.
 *   - A window j overlaps block b when s*j < BS*(b+1) and s*j + l > BS*b; the block score is the
 *     maximum of the group score over the overlapping complete windows, -inf when there is none.
 *   - Only complete windows (s*j + l <= T) exist.
 *   - Init blocks are [0, n_init), local blocks are the last n_local blocks of ceil(T/BS); both are
 *     removed from the top-k candidates, so the union has exactly k + n_init + n_local blocks when
 *     there are enough blocks.
 *   - Ties between equal block scores go to the lower block index.
 *   - Compressed keys are rounded (round-to-nearest-even) to the cache's element type, because they
 *     are stored in it; the rounded values feed the scoring.
 */
#ifndef BSA_ORACLE_H
#define BSA_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Storage element types of the tensors the oracle reads. */
#define ORC_F32 0
#define ORC_BF16 1
/* "No rounding" marker for bsa_oracle_compress. */
#define ORC_NO_ROUND (-1)

/* Round a double to the nearest value of the given storage type (ties to even). */
double bsa_oracle_round(double x, int dtype);

/* y[i] = bsa_oracle_round(x[i], dtype) for i < n. */
void bsa_oracle_round_array(const double* x, int64_t n, int dtype, double* y);

/* Widen element i of a bf16 / fp32 array to double. */
double bsa_oracle_load(const void* base, int dtype, int64_t i);

/* Number of complete windows of length l at stride s in T rows. */
int64_t bsa_oracle_num_windows(int64_t T, int l, int s);

/* Number of selection blocks covering T tokens. */
int64_t bsa_oracle_num_blocks(int64_t T, int block_size);

/* Eq. (2): ck[j][c] = mean_{r<l} K[s*j + r][c] for every complete window j, optionally rounded to
 * the storage type round_dtype (ORC_NO_ROUND keeps full double). K is [T][d] of type dtype.
 * ck must hold num_windows(T, l, s) * d doubles. Returns the number of windows. */
int64_t bsa_oracle_compress(const void* k, int dtype, int64_t T, int d, int l, int s,
                            int round_dtype, double* ck);

/* Eq. (6) target form: S[j] = sum_h softmax_j(q_h . ck_j / tau) for the G heads of one group.
 * q is [G][d], ck is [nc][d]. */
void bsa_oracle_group_scores(const double* q, const double* ck, int64_t nc, int G, int d,
                             double tau, double* S);

/* Eq. (4) with the Compact Forecast Indexer: S[j] = f . ck_j for one group's Forecast vector
 * f [d] (no softmax). ck is [nc][d]. */
void bsa_oracle_forecast_scores(const double* f, const double* ck, int64_t nc, int d, double* S);

/* Max of S over the complete windows overlapping each block, -inf where there is none. */
void bsa_oracle_block_scores(const double* S, int64_t nc, int64_t nb, int l, int s,
                             int block_size, double* sb);

/* Eq. (1) with Eq. (4)'s f_top: selected blocks in ascending order. idx must hold
 * n_init + n_local + top_k entries. boundary[0] receives the score of the last block taken by the
 * top-k, boundary[1] the score of the best candidate left out (NaN when such a block does not
 * exist). Returns the number of selected blocks. */
int bsa_oracle_select(const double* sb, int64_t nb, int n_init, int n_local, int top_k,
                      int32_t* idx, double* boundary);

/* Eq. (5): softmax attention of the G query heads over the tokens of the selected blocks
 * (token t < T). K and V are [T_rows][d] of type dtype. out is [G][d]; lse[h] is the natural log
 * of the softmax denominator (-inf when no token is attended). */
void bsa_oracle_attend(const double* q, const void* k, const void* v, int dtype, int64_t T, int d,
                       int G, const int32_t* idx, int n_sel, int block_size, double scale,
                       double* out, double* lse);

/* One decode problem: the shapes of a batch of sequences sharing one set of parameters. */
typedef struct {
    int batch, num_q_heads, num_kv_heads, head_dim;
    int cmp_kernel, cmp_stride, block_size;
    int n_init, n_local, top_k;
    int64_t max_seq_len; /* rows allocated per (batch, kv head) in the caches */
    int dtype;           /* ORC_F32 or ORC_BF16, for q, caches and compressed keys */
    double scale;        /* attention scale in Eq. (5) */
    double tau;          /* temperature in Eq. (6) */
} orc_problem_t;

/* Select + attend for the (batch, kv-head) pairs listed in `pairs` (pair = b * Hkv + kvh), in
 * parallel over pairs with OpenMP. q is [B][Hq][d], caches are [B][Hkv][max_seq_len][d], all of
 * type dtype; seq_lens is [B]. Per listed pair i the outputs are written at position i:
 * idx [n][sel_cap] (-1 padded), n_sel [n], block_scores [n][nb_cap] (-inf past nb),
 * boundary [n][2], out [n][G][d], lse [n][G].
 * When given_idx is not NULL the selection step is skipped and given_idx/given_n_sel (laid out
 * like idx/n_sel) are attended instead. Returns 0, or -1 on an invalid argument. */
int bsa_oracle_decode(const orc_problem_t* P, const void* q, const void* k_cache,
                      const void* v_cache, const int32_t* seq_lens, const int32_t* pairs,
                      int n_pairs, const int32_t* given_idx, const int32_t* given_n_sel,
                      int32_t* idx, int32_t* n_sel, double* block_scores, double* boundary,
                      double* out, double* lse);

/* As bsa_oracle_decode, but the blocks are selected from the Forecast vectors f [B][Hkv][d]
 * (type dtype, one per GQA group) with bsa_oracle_forecast_scores in place of the group scores;
 * q still attends them. block_scores hold the max-pooled raw forecast scores. */
int bsa_oracle_decode_forecast(const orc_problem_t* P, const void* f, const void* q,
                               const void* k_cache, const void* v_cache, const int32_t* seq_lens,
                               const int32_t* pairs, int n_pairs, int32_t* idx, int32_t* n_sel,
                               double* block_scores, double* boundary, double* out, double* lse);

/* [CLSA]/[Kascade] shared index: attend one layer's q/K/V with block indices computed elsewhere
 * (by bsa_oracle_decode on the anchor layer). Same layouts as bsa_oracle_decode. */
int bsa_oracle_attend_pairs(const orc_problem_t* P, const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* seq_lens, const int32_t* pairs,
                            int n_pairs, const int32_t* idx, const int32_t* n_sel, double* out,
                            double* lse);

/* Compressed keys of whole caches: ck[B][Hkv][nc_cap][d] as doubles rounded to dtype, rows past a
 * sequence's window count set to 0. Parallel over pairs. */
int bsa_oracle_compress_cache(const orc_problem_t* P, const void* k_cache,
                              const int32_t* seq_lens, const int32_t* pairs, int n_pairs,
                              double* ck);

/* Number of OpenMP threads the parallel drivers use. */
int bsa_oracle_num_threads(void);
void bsa_oracle_set_num_threads(int n);
/* bsa_oracle_decode with the listed pairs' compressed keys given ([n_pairs][nc_cap][d], rounded to
 * the cache type, as bsa_oracle_compress_cache writes them) instead of formed from the cache. */
int bsa_oracle_decode_forecast_ck(const orc_problem_t* P, const void* f, const void* q, const double* ck,
                                  const void* k_cache, const void* v_cache, const int32_t* seq_lens,
                                  const int32_t* pairs, int n_pairs, int32_t* idx, int32_t* n_sel,
                                  double* block_scores, double* boundary, double* out, double* lse);
int bsa_oracle_decode_ck(const orc_problem_t* P, const void* q, const double* ck,
                         const void* k_cache, const void* v_cache, const int32_t* seq_lens,
                         const int32_t* pairs, int n_pairs, int32_t* idx, int32_t* n_sel,
                         double* block_scores, double* boundary, double* out, double* lse);
/* The Forecast selection of bsa_oracle_decode_forecast_ck alone (no attention): f [B][Hkv][d]
 * against the given compressed keys ck [n_pairs][nc_cap][d] (for one-layer lookahead, f of layer
 * l and ck of layer l + 1). */
/* Block-sparse prefill of a chunk of C queries per sequence ([B][C][Hq][d], at positions
 * seq_lens[b] - C .. seq_lens[b] - 1), one selection per query tile (the chunk's positions inside
 * one block) and kv head from the windows complete before that block, causal attention per query;
 * see bsa_oracle.c for the definition. Outputs per listed pair i: idx [n][tiles_cap][sel_cap],
 * n_sel [n][tiles_cap], boundary [n][tiles_cap][2] (may be NULL), out [n][C][G][d], lse [n][C][G]. */
int bsa_oracle_prefill(const orc_problem_t* P, const void* q, const void* k_cache, const void* v_cache,
                       const int32_t* seq_lens, int chunk, const int32_t* pairs, int n_pairs, int tiles_cap,
                       int32_t* idx, int32_t* n_sel, double* boundary, double* out, double* lse);
/* CLSA token-level index (see bsa_oracle.c): the tokens of each listed pair that the base selector,
 * at token granularity, picks with the block configuration's token budget. idx [n][tok_cap]
 * (tok_cap = (n_init + n_local + top_k) * block_size), n_sel [n], boundary [n][2] and the token
 * scores [n][max_seq_len] (both may be NULL).
 * Every layer sharing the index attends them: bsa_oracle_attend_pairs with block_size 1. */
int bsa_oracle_token_select(const orc_problem_t* P, const void* q, const void* k_cache, const int32_t* seq_lens,
                            const int32_t* pairs, int n_pairs, int32_t* idx, int32_t* n_sel, double* boundary,
                            double* scores);
int bsa_oracle_select_forecast_ck(const orc_problem_t* P, const void* f, const double* ck,
                                  const int32_t* seq_lens, const int32_t* pairs, int n_pairs,
                                  int32_t* idx, int32_t* n_sel, double* block_scores, double* boundary);

#ifdef __cplusplus
}
#endif
#endif
