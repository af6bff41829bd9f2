/*
 * bsa.h -- C ABI of the B200 block-sparse compressed-key decode attention library (libbsa.so).
 *
 * The method (InfLLM-V2 style block-sparse decode, as summarised on the page
 * "SparDA: Sparse Decoupled Attention for Efficient Long-Context LLM Inference"):
 *   1. compressed keys: K~_j = mean of K over rows [s*j, s*j + l), l = 32, s = 16
 *      (Theoretical Foundation, Eq. 2);
 *   2. group scoring: per GQA group, S[j] = sum over the group's query heads of
 *      softmax_j(q_h . K~_j / tau) (Indexer Training, Eq. 6, the original selector's distribution);
 *   3. block reduction: the score of a 64-token block is the maximum of S over the complete windows
 *      that overlap it (Indexer Training, "Fine-grained supervision": max-pooled to the block grid);
 *   4. selection: top-k blocks by that score, ties to the lower block index, united with the first
 *      n_init and last n_local blocks (Theoretical Foundation, Eq. 1; SparDA Architecture, Eq. 4);
 *   5. attention: exact softmax attention of every query head over the tokens of its group's
 *      selected blocks (SparDA Architecture, Eq. 5).
 * A shared-index mode reuses one layer's selection for several layers (page "HySparse2: Hybrid
 * Sparse Attention with Two-Level KV Sharing", first abstract; page "CoSA: Accelerating
 * Long-Context Inference via Proxy-Kernel Co-Designed Sparse Attention", second abstract), also
 * with several anchor layers (bsa_decode_step_anchored). A Forecast-indexer selection scores with
 * one given vector per GQA group instead of the query heads (SparDA Architecture, Eq. 4 and
 * "Compact Forecast Indexer"; bsa_select_blocks_forecast).
 *
 * Conventions for every entry point:
 *   - All tensors are dense, row-major, on the current CUDA device, owned by the caller. The
 *     library allocates no memory and keeps no state between calls except inside the caller's
 *     workspace (bsa_sparse_decode_noalloc, at the end, uses a fixed scratch array instead).
 *     Pointers must be 16-byte aligned.
 *   - Every call is asynchronous on `stream` (cudaStream_t; 0 = legacy default stream) and does
 *     not synchronize, except bsa_read_device_error.
 *   - Arguments are validated on the host before anything is launched; a rejected call returns a
 *     status other than BSA_OK, launches nothing and leaves all buffers untouched.
 *   - Conditions that only the device can see (a sequence length above the capacity, a block
 *     index out of range) set a bit in the workspace's error word (bsa_device_error_t), skip the
 *     affected (batch, kv-head) pair and never trap; read it with bsa_read_device_error.
 *   - Kernels that use the workspace need it zero-filled once before first use
 *     (bsa_workspace_init); they leave it ready for the next call. Calls that share a workspace
 *     must not overlap on the GPU (same stream, or ordered by events).
 *
 * Tensor layouts (B = batch, Hq / Hkv = query / kv heads, G = Hq / Hkv, d = head_dim,
 * T_cap = max_seq_len, NC_cap = number of windows in T_cap rows, NB_cap = ceil(T_cap / BS),
 * SEL_cap = n_init + n_local + top_k; "elem" is fp32 or bf16 per bsa_params_t.dtype):
 *   q            [B][Hq][d]          elem   query head h belongs to kv head h / G
 *   k_cache      [B][Hkv][T_cap][d]  elem   rows >= seq_lens[b] are never read for attention
 *   v_cache      [B][Hkv][T_cap][d]  elem
 *   ck           [B][Hkv][NC_cap][d] elem   compressed keys (rounded to nearest even from fp64)
 *   seq_lens     [B]                 int32  tokens in each sequence (incl. the current one)
 *   block_idx    [B][Hkv][SEL_cap]   int32  selected blocks, ascending, then -1 padding
 *   n_sel        [B][Hkv]            int32  number of valid entries in block_idx
 *   block_scores [B][Hkv][NB_cap]    fp32   max-pooled group score per block, -inf where no
 *                                           complete window overlaps the block and past the end
 *   out          [B][Hq][d]          elem   attention output
 *   lse          [B][Hq]             fp32   natural log of each head's softmax denominator
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define BSA_ABI_VERSION 1
#define BSA_MAX_LAYERS 16

typedef enum {
    BSA_OK = 0,
    BSA_ERR_INVALID_ARG = 1, /* a null/misaligned pointer, bad shape or inconsistent parameter */
    BSA_ERR_UNSUPPORTED = 2, /* valid but not implemented (head_dim, group size, dtype, sizes) */
    BSA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than bsa_workspace_size() */
    BSA_ERR_CUDA = 4,        /* a CUDA runtime call failed (launch or memset) */
    BSA_ERR_DEVICE_CHECK = 5 /* bsa_read_device_error found a device-side error bit set */
} bsa_status_t;

typedef enum { BSA_F32 = 0, BSA_BF16 = 1 } bsa_dtype_t;

/* Bits of the device error word (bsa_read_device_error). */
typedef enum {
    BSA_DEVERR_SEQ_LEN = 1u << 0,   /* seq_lens[b] < 0 or > max_seq_len: pair skipped */
    BSA_DEVERR_CAPACITY = 1u << 1,  /* bsa_compress_append with seq_lens[b] == max_seq_len */
    BSA_DEVERR_BLOCK_IDX = 1u << 2, /* block index outside [0, ceil(T/BS)): entry skipped */
    BSA_DEVERR_N_SEL = 1u << 3,     /* n_sel outside [0, SEL_cap]: clamped */
    BSA_DEVERR_TIMEOUT = 1u << 4    /* a pipeline wait gave up (never expected): output invalid */
} bsa_device_error_t;

/* Problem shape and method parameters. Supported: dtype fp32 or bf16; head_dim 64 or 128;
 * G = Hq / Hkv in 1..8; block_size a multiple of 16 in 16..256; cmp_kernel, cmp_stride >= 1;
 * 1 <= n_init + n_local + top_k <= 4096; NB_cap <= 32768; num_layers in 1..BSA_MAX_LAYERS;
 * bf16: B * Hkv * max_seq_len below 2^31 (cache rows are addressed with 32-bit TMA coordinates).
 * Parameters outside these limits are reported as BSA_ERR_UNSUPPORTED. */
typedef struct {
    int32_t batch;        /* B */
    int32_t num_q_heads;  /* Hq */
    int32_t num_kv_heads; /* Hkv */
    int32_t head_dim;     /* d */
    int32_t cmp_kernel;   /* l, compression window length (32 in Eq. 2) */
    int32_t cmp_stride;   /* s, compression window stride (16 in Eq. 2) */
    int32_t block_size;   /* BS, tokens per selection block (64) */
    int32_t n_init;       /* first blocks always selected */
    int32_t n_local;      /* last blocks always selected (sliding window) */
    int32_t top_k;        /* blocks chosen by score among the others */
    int64_t max_seq_len;  /* T_cap, rows allocated per (batch, kv head) in the caches */
    int32_t num_layers;   /* layers attended with one selection (shared-index mode); sizes ws */
    int32_t dtype;        /* bsa_dtype_t of q, caches, ck and out */
    float scale;          /* attention scale of Eq. 5; 0 selects 1/sqrt(head_dim) */
    float score_tau;      /* tau of Eq. 6; 0 selects sqrt(head_dim) */
} bsa_params_t;

/* Derived sizes of a parameter set. */
typedef struct {
    int64_t nc_cap;          /* NC_cap: windows in max_seq_len rows */
    int64_t nb_cap;          /* NB_cap: blocks in max_seq_len rows */
    int32_t sel_cap;         /* SEL_cap: n_init + n_local + top_k */
    int32_t group;           /* G */
    size_t workspace_bytes;  /* what bsa_workspace_size returns */
} bsa_sizes_t;

/* Human-readable name of a status. Never NULL. */
const char* bsa_status_string(bsa_status_t status);

/* Library ABI version (BSA_ABI_VERSION at build time). */
int32_t bsa_abi_version(void);

/* Validate a parameter set (host only; no CUDA call). */
bsa_status_t bsa_check_params(const bsa_params_t* params);

/* Fill *sizes for a valid parameter set (host only). */
bsa_status_t bsa_get_sizes(const bsa_params_t* params, bsa_sizes_t* sizes);

/* Bytes of device workspace that bsa_select_blocks, bsa_sparse_decode(_layers) and
 * bsa_decode_step need for these parameters; 0 for invalid parameters. Holds the error word,
 * per-pair completion counters, fp32 window terms [B*Hkv][NC_cap][G] with per-chunk statistics,
 * block scores and attention partials. */
size_t bsa_workspace_size(const bsa_params_t* params);

/* Zero the workspace's error word and counters (cudaMemsetAsync on `stream`). Call once after
 * allocating a workspace, or after a call was aborted. */
bsa_status_t bsa_workspace_init(const bsa_params_t* params, void* workspace, size_t workspace_bytes,
                                cudaStream_t stream);

/* Eq. 2 over whole caches (prefill): ck[b][h][j] = mean(k_cache[b][h][s*j : s*j + l]) for every
 * complete window j of sequence b (s*j + l <= seq_lens[b]); other rows of ck are not written.
 * Sums are formed in fp64 and rounded once to the element type. No workspace. */
bsa_status_t bsa_compress_keys(const bsa_params_t* params, const void* k_cache,
                               const int32_t* seq_lens, void* ck, cudaStream_t stream);

/* Decode-time append of one token per sequence: writes k_new[b][h] / v_new[b][h] ([B][Hkv][d])
 * into row seq_lens[b] of the caches, increments seq_lens[b], and when that completes a window
 * (new length T >= l and (T - l) % s == 0) writes ck row (T - l) / s as in bsa_compress_keys.
 * A sequence already at max_seq_len is left unchanged and sets BSA_DEVERR_CAPACITY in the
 * workspace error word when a workspace is given (workspace may be NULL). */
bsa_status_t bsa_compress_append(const bsa_params_t* params, void* k_cache, void* v_cache,
                                 const void* k_new, const void* v_new, int32_t* seq_lens, void* ck,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Steps 2-4: score q against ck per GQA group (Eq. 6), reduce the window scores onto blocks
 * (max over overlapping complete windows), pick top_k blocks among those that are neither init
 * nor local (ties to the lower index) and write the union with the init and local blocks in
 * ascending order to block_idx (-1 padded) with its count in n_sel. block_scores (optional, may be
 * NULL) receives the per-block scores. Uses the workspace. */
bsa_status_t bsa_select_blocks(const bsa_params_t* params, const void* q, const void* ck,
                               const int32_t* seq_lens, int32_t* block_idx, int32_t* n_sel,
                               float* block_scores, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/* SparDA Architecture, Eq. (4), with the "Compact Forecast Indexer": the same selection as
 * bsa_select_blocks, but each (batch, kv head) pair is scored by ONE Forecast vector
 * f[b][kvh] (params->head_dim elements of params->dtype, [batch][num_kv_heads][head_dim],
 * 16-byte aligned, caller-owned) instead of its group's query heads, with no softmax: the window
 * score is the raw dot product f . ck_j (fp32 accumulation of exact products), the block score
 * its maximum over the block's complete windows (-inf when there is none; written to
 * block_scores when that is not NULL). top_k, init and local blocks, tie rule, outputs and
 * workspace (bsa_workspace_size(params)) are those of bsa_select_blocks; q then attends the
 * blocks through bsa_sparse_decode. Errors as bsa_select_blocks. */
bsa_status_t bsa_select_blocks_forecast(const bsa_params_t* params, const void* f, const void* ck,
                                        const int32_t* seq_lens, int32_t* block_idx, int32_t* n_sel,
                                        float* block_scores, void* workspace,
                                        size_t workspace_bytes, cudaStream_t stream);

/* Step 5 (Eq. 5): for every query head, softmax attention (scale params->scale) over the tokens
 * t < seq_lens[b] of the first n_sel[b][kvh] blocks listed in block_idx[b][kvh] (any order; -1
 * entries are skipped). Writes out and, if not NULL, lse. A pair with no attended token gets a
 * zero output and lse = -inf. Uses the workspace for split partials. */
bsa_status_t bsa_sparse_decode(const bsa_params_t* params, const void* q, const void* k_cache,
                               const void* v_cache, const int32_t* seq_lens,
                               const int32_t* block_idx, const int32_t* n_sel, void* out,
                               float* lse, void* workspace, size_t workspace_bytes,
                               cudaStream_t stream);

/* Shared-index mode: bsa_sparse_decode for num_layers layers at once, all with the same
 * block_idx / n_sel / seq_lens. q, k_caches, v_caches, outs and lses are HOST arrays of
 * num_layers device pointers (lses may be NULL, or contain NULLs). num_layers must not exceed
 * params->num_layers. One launch covers all layers. */
bsa_status_t bsa_sparse_decode_layers(const bsa_params_t* params, int32_t num_layers,
                                      const void* const* q, const void* const* k_caches,
                                      const void* const* v_caches, const int32_t* seq_lens,
                                      const int32_t* block_idx, const int32_t* n_sel,
                                      void* const* outs, float* const* lses, void* workspace,
                                      size_t workspace_bytes, cudaStream_t stream);

/* Anchored index reuse ([CoSA] Kascade abstract: exact top-k indices computed in a few anchor
 * layers and reused, head by head, by the layers that follow; [HySparse2] CLSA abstract: one
 * routing index shared across layers). anchors is a HOST array of num_anchors layer numbers,
 * ascending, anchors[0] == 0, each < num_layers <= params->num_layers. For anchor i this runs
 * bsa_select_blocks on q[anchors[i]] and cks[anchors[i]], writing its selection to
 * block_idx + i * (batch * num_kv_heads * (n_init + n_local + top_k)) and
 * n_sel + i * (batch * num_kv_heads) (per kv head, so the reuse is head-aware), then
 * bsa_sparse_decode_layers on layers [anchors[i], anchors[i+1]) (the last group runs to
 * num_layers) with that selection. q, k_caches, v_caches, cks, outs and lses are HOST arrays of
 * num_layers device pointers (cks is read at the anchors only; lses may be NULL or contain NULLs).
 * Everything is queued on `stream` with no host synchronisation. Errors as the two calls it
 * chains; an invalid schedule is BSA_ERR_INVALID_ARG. */
bsa_status_t bsa_decode_step_anchored(const bsa_params_t* params, int32_t num_layers,
                                      const int32_t* anchors, int32_t num_anchors,
                                      const void* const* q, const void* const* k_caches,
                                      const void* const* v_caches, const void* const* cks,
                                      const int32_t* seq_lens, int32_t* block_idx, int32_t* n_sel,
                                      void* const* outs, float* const* lses, void* workspace,
                                      size_t workspace_bytes, cudaStream_t stream);

/* One decode step of one layer (steps 2-5, after an optional append when k_new and v_new are both
 * non-NULL), queued on `stream` with no host synchronisation. block_idx / n_sel receive the
 * selection; block_scores and lse may be NULL. It runs the fused step (as bsa_decode_step_fused)
 * when that is possible and there are enough (batch, kv head) pairs to keep most SMs streaming
 * (at least two thirds of the SM count), else the chained launches of bsa_select_blocks and
 * bsa_sparse_decode with programmatic dependent launch; bsa_decode_step_info tells which. The
 * selection is the same bit for bit either way. */
bsa_status_t bsa_decode_step(const bsa_params_t* params, const void* q, void* k_cache,
                             void* v_cache, void* ck, const void* k_new, const void* v_new,
                             int32_t* seq_lens, int32_t* block_idx, int32_t* n_sel,
                             float* block_scores, void* out, float* lse, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream);

/* bsa_decode_step as one kernel (after the optional append's): a CTA per (batch, kv head) pair,
 * one per SM (a persistent grid walks the pairs when there are more pairs than SMs), scores the
 * pair's compressed keys with the group's query heads, keeps the window terms in the SM's tensor
 * memory, takes the block maxima and the top-k there and in shared memory, and attends the
 * selected blocks, writing out and lse directly (no split partials, no combine pass). Same
 * arguments, results and selection as bsa_decode_step; the workspace holds only the error word.
 * Supported: bf16, blocks of four compression strides (BS = 4s, l = s or 2s, BS a multiple of 64),
 * max_seq_len of at least one window (l) and window terms within 512 tensor-memory columns (about
 * 260K tokens at G = 4); other parameter sets return BSA_ERR_UNSUPPORTED. Each SM streams at most ~50 GB/s, so with few pairs the chained
 * kernels of bsa_decode_step are faster. */
bsa_status_t bsa_decode_step_fused(const bsa_params_t* params, const void* q, void* k_cache,
                                   void* v_cache, void* ck, const void* k_new, const void* v_new,
                                   int32_t* seq_lens, int32_t* block_idx, int32_t* n_sel,
                                   float* block_scores, void* out, float* lse, void* workspace,
                                   size_t workspace_bytes, cudaStream_t stream);

/* One layer l of one-layer-lookahead decoding (page "SparDA: Sparse Decoupled Attention for
 * Efficient Long-Context LLM Inference", SparDA Architecture, Eqs. 4 and 5, and the lookahead
 * selection of its abstract): layer l attends the blocks chosen for it beforehand while layer
 * l + 1's blocks are chosen from layer l's Forecast vectors, in the same kernel.
 *   attention (Eq. 5): q (this layer's queries, [batch][num_q_heads][head_dim]) over the tokens of
 *     the blocks in block_idx / n_sel ([batch][num_kv_heads][n_init + n_local + top_k] and
 *     [batch][num_kv_heads], as bsa_select_blocks writes them; entries outside the sequence's
 *     blocks, such as the -1 padding, are skipped) of k_cache / v_cache -> out, lse (may be NULL);
 *   selection (Eq. 4): f ([batch][num_kv_heads][head_dim], one Forecast vector per GQA group)
 *     against ck_next (the NEXT layer's compressed keys, [batch][num_kv_heads][nc_cap][head_dim])
 *     exactly as bsa_select_blocks_forecast -> block_idx_next, n_sel_next, block_scores_next (may
 *     be NULL).
 * The blocks of this layer stream while the next layer's are being chosen (the kernel has no
 * selection-to-attention dependency). block_idx_next / n_sel_next must not overlap block_idx /
 * n_sel. The first layer's blocks come from bsa_select_blocks (its own queries) or
 * bsa_select_blocks_forecast; the last layer attends with bsa_sparse_decode. All device pointers
 * are caller-owned, 16-byte aligned (4-byte for the int32 / fp32 arrays); seq_lens as
 * bsa_decode_step (not modified); the workspace holds the error word. Runs the fused step kernel,
 * so the parameter sets of bsa_decode_step_fused only; others return BSA_ERR_UNSUPPORTED. */
bsa_status_t bsa_decode_step_lookahead(const bsa_params_t* params, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* block_idx,
                                       const int32_t* n_sel, const void* f, const void* ck_next,
                                       const int32_t* seq_lens, int32_t* block_idx_next,
                                       int32_t* n_sel_next, float* block_scores_next, void* out,
                                       float* lse, void* workspace, size_t workspace_bytes,
                                       cudaStream_t stream);

/* Token-level shared index (page "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing",
 * CLSA abstract: one indexer computes a token-level top-k once and the layers reuse it). The index
 * is the base selector at token granularity on layer 0: per (batch, kv head),
 * S[t] = sum over the group's query heads of softmax_t(q_h . K_t / tau) over the tokens t < T of
 * k_caches[0] (no compression). The first n_init * block_size and the last n_local * block_size
 * tokens are always taken, and top_k * block_size more by score (ties to the lower token); the
 * ascending token list goes to tok_idx [batch][num_kv_heads][(n_init + n_local + top_k) *
 * block_size] (-1 padded) with its length in n_tok [batch][num_kv_heads]. Every layer
 * i < num_layers (<= params->num_layers, <= BSA_MAX_LAYERS) then attends exactly those tokens with
 * its own q[i] [batch][num_q_heads][head_dim], k_caches[i] and v_caches[i] (as bsa_sparse_decode's)
 * into outs[i] and lses[i] (lses, or an entry of it, may be NULL). q, k_caches, v_caches, outs and
 * lses are HOST arrays of device pointers. The workspace must hold bsa_clsa_workspace_size(params)
 * bytes (the token scorer's terms: about 4 * num_kv_heads * max_seq_len * 4 B per sequence).
 * Supported: bf16, max_seq_len up to about 50K tokens (the token keys of a sequence, 4 bytes each,
 * sit in one CTA's shared memory); others return BSA_ERR_UNSUPPORTED. Queued on `stream`, no host
 * sync. */
bsa_status_t bsa_decode_step_clsa(const bsa_params_t* params, int32_t num_layers, const void* const* q,
                                  const void* const* k_caches, const void* const* v_caches,
                                  const int32_t* seq_lens, int32_t* tok_idx, int32_t* n_tok, void* const* outs,
                                  float* const* lses, void* workspace, size_t workspace_bytes,
                                  cudaStream_t stream);

/* Workspace bytes of bsa_decode_step_clsa for these parameters (host only); 0 when unsupported. */
size_t bsa_clsa_workspace_size(const bsa_params_t* params);

/* Block-sparse prefill of a chunk (page "SparDA: Sparse Decoupled Attention for Efficient
 * Long-Context LLM Inference", Theoretical Foundation, Eq. 1, and the prefill workload of its
 * Efficiency Results; one selection per query tile, as the tile-level operations of the page "CoSA:
 * Accelerating Long-Context Inference via Proxy-Kernel Co-Designed Sparse Attention", Kascade
 * abstract). The last `chunk` positions of every sequence are queried: q is
 * [batch][chunk][num_q_heads][head_dim] (query c of sequence b at position seq_lens[b] - chunk + c),
 * the chunk's keys and values are already in k_cache / v_cache and ck holds the compressed keys of
 * the whole sequences (bsa_compress_keys after the chunk was written). Query tile i of a
 * (batch, kv head) pair holds the chunk's positions inside block (seq_lens[b] - chunk) / block_size
 * + i; per tile and kv head the group's heads score, over every position of the tile, the windows
 * complete before the tile's block begins (softmax per position and head, summed), the block
 * scores are the maxima over overlapping windows, and the blocks of Eq. 1 among blocks 0 .. the
 * tile's own are written to block_idx [batch][num_kv_heads][tiles][n_init + n_local + top_k]
 * (ascending, -1 padded; tiles = bsa_prefill_tiles(chunk, block_size); tiles past a chunk's last are
 * empty) and n_sel [batch][num_kv_heads][tiles]. Each query then attends the tokens of its tile's
 * blocks at or before its own position: out [batch][chunk][num_q_heads][head_dim], lse
 * [batch][chunk][num_q_heads] (natural log; may be NULL). seq_lens[b] must be in
 * [chunk, max_seq_len]. Supported: bf16, head_dim 128, 2 or 4 query heads per kv head, blocks of
 * 64 tokens, windows of 32 with stride 16 and compressed keys whose window scores fit the selection
 * kernel's shared memory (max_seq_len up to about 128K tokens); others return BSA_ERR_UNSUPPORTED.
 * The scoring runs on the tensor cores (tcgen05) with accumulators in tensor memory. */
bsa_status_t bsa_prefill(const bsa_params_t* params, int32_t chunk, const void* q, const void* k_cache,
                         const void* v_cache, const void* ck, const int32_t* seq_lens, int32_t* block_idx,
                         int32_t* n_sel, void* out, float* lse, void* workspace, size_t workspace_bytes,
                         cudaStream_t stream);

/* The attention of bsa_prefill alone, with the tiles' blocks given (block_idx / n_sel laid out as
 * bsa_prefill writes them; entries outside blocks 0 .. the tile's own are skipped). */
bsa_status_t bsa_prefill_attend(const bsa_params_t* params, int32_t chunk, const void* q, const void* k_cache,
                                const void* v_cache, const int32_t* seq_lens, const int32_t* block_idx,
                                const int32_t* n_sel, void* out, float* lse, void* workspace,
                                size_t workspace_bytes, cudaStream_t stream);

/* Query tiles per (batch, kv head) pair of a prefill chunk: ceil(chunk / block_size) + 1 (a chunk
 * that starts inside a block spans one more); 0 for non-positive arguments. Host only. */
int32_t bsa_prefill_tiles(int32_t chunk, int32_t block_size);

/* How bsa_decode_step runs for these parameters (host only, no CUDA call): *fused is 1 when it
 * runs the one-kernel step of bsa_decode_step_fused, 0 when it chains the scoring, selection,
 * attention and combine kernels; *launches is the number of kernel launches of one call, counting
 * the append when `append` is non-zero. Either output pointer may be NULL. */
bsa_status_t bsa_decode_step_info(const bsa_params_t* params, int32_t append, int32_t* fused,
                                  int32_t* launches);

/* Copy the workspace error word to *flags (bits of bsa_device_error_t), clear it, and
 * synchronize `stream`. Returns BSA_ERR_DEVICE_CHECK when a bit was set, BSA_OK otherwise. */
bsa_status_t bsa_read_device_error(void* workspace, size_t workspace_bytes, uint32_t* flags,
                                   cudaStream_t stream);

/* Size of the fixed device scratch of bsa_sparse_decode_noalloc, per device: 4 MiB. */
#define BSA_NOALLOC_SCRATCH_BYTES (4u << 20)

/* bsa_sparse_decode for callers that cannot allocate device memory, and so cannot provide a
 * workspace. Examples are a host runtime whose allocator must not be entered from the calling
 * thread, and a process with a fixed memory budget that has no room for a second buffer. The
 * paper has no counterpart: it is a deployment variant of the step 5 entry point. It computes
 * the same results with the same kernels and allocates nothing: no cudaMalloc, no allocating
 * library routine.
 *
 * Scratch: the split partials and per-pair completion counters live in a fixed array inside
 * libbsa, BSA_NOALLOC_SCRATCH_BYTES per device.
 *   - Size limit. A parameter set whose partials do not fit returns BSA_ERR_WORKSPACE before any
 *     CUDA call and launches nothing. The call attends one layer, so params->num_layers plays no
 *     part in the size: the partials need about B*Hkv*Gp*(d + 2)*4 bytes per partial slot, where
 *     Gp is G rounded up to a power of two. For example, B=16, Hkv=8, G=4, d=128 with 69 selected
 *     blocks needs 1.3 MiB.
 *   - Device. The scratch used is the current device's, so `stream` must belong to the current
 *     device (or be a default stream); a stream of another device is BSA_ERR_INVALID_ARG.
 *   - First call on a device. It looks up the array's device address (cudaGetSymbolAddress), with
 *     that device current. The lookup may load the library's device code. Make the first call on
 *     each device outside any stream capture.
 *   - Zeroing. The counters and the scratch's error word must start at zero. Every call clears
 *     them with a cudaMemsetAsync on `stream` ahead of its kernel.
 *   - Concurrency. All calls on one device share the one array. Calls that overlap on the GPU
 *     (different streams without an event between them, or several host threads) race on it and
 *     give wrong results. Calls on one stream are ordered and safe.
 *
 * device_error: optional device pointer to a caller-owned, 4-byte aligned word.
 *   - If it is given, device-side error bits (bsa_device_error_t) are OR-ed into it. The caller
 *     zeroes the word and reads it back.
 *   - If it is NULL, they go to the scratch's error word and are not reported.
 * Other arguments, layouts and results are those of bsa_sparse_decode for one layer. */
bsa_status_t bsa_sparse_decode_noalloc(const bsa_params_t* params, const void* q,
                                       const void* k_cache, const void* v_cache,
                                       const int32_t* seq_lens, const int32_t* block_idx,
                                       const int32_t* n_sel, void* out, float* lse,
                                       uint32_t* device_error, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* BSA_H */
