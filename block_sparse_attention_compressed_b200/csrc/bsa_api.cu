// Host side of libbsa: parameter validation, launch planning, workspace layout and the C ABI
// declared in include/bsa.h. Nothing here allocates device memory or synchronizes (except
// bsa_read_device_error, which is documented to).
#include <math.h>
#include <string.h>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr size_t kAlign = 256;
constexpr int kNumSMs = 148;  // B200; only used to size work splits, never for correctness

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int64_t num_windows(int64_t T, int l, int s) { return T < l ? 0 : (T - l) / s + 1; }

bool is_aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

bsa_status_t make_plan(const bsa_params_t* prm, Plan* p) {
    if (!prm || !p) return BSA_ERR_INVALID_ARG;
    const bsa_params_t& q = *prm;
    if (q.batch < 1 || q.num_q_heads < 1 || q.num_kv_heads < 1) return BSA_ERR_INVALID_ARG;
    if (q.num_q_heads % q.num_kv_heads != 0) return BSA_ERR_INVALID_ARG;
    if (q.cmp_kernel < 1 || q.cmp_stride < 1 || q.block_size < 1) return BSA_ERR_INVALID_ARG;
    if (q.n_init < 0 || q.n_local < 0 || q.top_k < 0) return BSA_ERR_INVALID_ARG;
    if (q.max_seq_len < 1 || q.max_seq_len > ((int64_t)1 << 31) - 1) return BSA_ERR_INVALID_ARG;
    if (q.num_layers < 1) return BSA_ERR_INVALID_ARG;
    if (!(q.scale >= 0.f) || isinf(q.scale) || !(q.score_tau >= 0.f) || isinf(q.score_tau))
        return BSA_ERR_INVALID_ARG;
    if (q.dtype != BSA_F32 && q.dtype != BSA_BF16) return BSA_ERR_UNSUPPORTED;
    if (q.head_dim != 64 && q.head_dim != 128) return BSA_ERR_UNSUPPORTED;
    const int G = q.num_q_heads / q.num_kv_heads;
    if (G > kMaxG) return BSA_ERR_UNSUPPORTED;
    if (q.block_size % 16 != 0 || q.block_size > 256) return BSA_ERR_UNSUPPORTED;
    if (q.num_layers > BSA_MAX_LAYERS) return BSA_ERR_UNSUPPORTED;
    const int64_t sel = (int64_t)q.n_init + q.n_local + q.top_k;
    if (sel < 1) return BSA_ERR_INVALID_ARG;
    if (sel > 4096) return BSA_ERR_UNSUPPORTED;
    const int64_t pairs = (int64_t)q.batch * q.num_kv_heads;
    if (pairs > (1 << 24)) return BSA_ERR_UNSUPPORTED;

    Plan& P = *p;
    memset(&P, 0, sizeof P);
    P.B = q.batch;
    P.Hq = q.num_q_heads;
    P.Hkv = q.num_kv_heads;
    P.G = G;
    P.Gp = 1;
    while (P.Gp < G) P.Gp <<= 1;
    P.D = q.head_dim;
    P.l = q.cmp_kernel;
    P.s = q.cmp_stride;
    P.BS = q.block_size;
    P.n_init = q.n_init;
    P.n_local = q.n_local;
    P.top_k = q.top_k;
    P.sel_cap = (int)sel;
    P.layers = q.num_layers;
    P.dtype = q.dtype;
    P.T_cap = q.max_seq_len;
    P.nc_cap = num_windows(P.T_cap, P.l, P.s);
    P.nb_cap = (P.T_cap + P.BS - 1) / P.BS;
    P.lg_stride = (P.nc_cap + 3) / 4 * 4;
    if (P.nb_cap > kMaxNbCap) return BSA_ERR_UNSUPPORTED;
    P.pairs = (int)pairs;
    const double log2e = 1.4426950408889634;
    const double scale = q.scale > 0.f ? (double)q.scale : 1.0 / sqrt((double)P.D);
    const double tau = q.score_tau > 0.f ? (double)q.score_tau : sqrt((double)P.D);
    P.scale_log2 = (float)(scale * log2e);
    P.score_log2 = (float)(log2e / tau);

    // Scoring: 64-row chunks, spread evenly over a persistent grid at launch time.
    P.nchunk = (P.nc_cap + 63) / 64;
    P.total_chunks = (int64_t)P.pairs * P.nchunk;
    P.nstat = P.nchunk;  // softmax statistics per 64-row chunk
    // three CTAs per SM: 3 x 64 KB of compressed-key stages in flight per SM
    P.score_ctas = (int)(P.total_chunks < 3 * kNumSMs ? (P.total_chunks > 0 ? P.total_chunks : 1)
                                                       : 3 * kNumSMs);
    if (P.dtype == BSA_BF16 && (int64_t)P.pairs * P.nc_cap > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
    // Selection: one CTA per pair when there are enough pairs to fill the GPU in one wave,
    // otherwise the pairs' windows are split into parts of at least 256 windows. A part's window
    // scores sit in shared memory next to the key array, so very long contexts get more parts.
    {
        const int64_t nc = P.nc_cap > 0 ? P.nc_cap : 1;
        const int64_t wmax = (P.BS + P.l - 2) / P.s + 2;  // windows overlapping one block, bound
        // the key array also stages the chunk statistics (2 words per float2)
        P.select_keys = (size_t)P.nb_cap > (size_t)(2 * P.nstat * P.Gp)
                            ? (size_t)P.nb_cap : (size_t)(2 * P.nstat * P.Gp);
        const int64_t smem_words = (int64_t)(200 * 1024) / (int64_t)sizeof(uint32_t);
        const int64_t max_pw = smem_words - (int64_t)P.select_keys - wmax;
        if (max_pw < 256) return BSA_ERR_UNSUPPORTED;
        int64_t parts = kNumSMs / P.pairs;
        const int64_t most = (nc + 255) / 256;
        if (parts > most) parts = most;
        if (parts < 1) parts = 1;
        if ((nc + parts - 1) / parts > max_pw) parts = (nc + max_pw - 1) / max_pw;
        const int64_t pw = (nc + parts - 1) / parts;
        P.select_part_windows = (int)pw;
        P.select_parts = (int)((nc + pw - 1) / pw);
        if ((int64_t)P.pairs * P.select_parts > 0x7fffffff) return BSA_ERR_UNSUPPORTED;
        P.select_smem = (P.select_keys + (size_t)pw + (size_t)wmax) * sizeof(uint32_t);
        if (P.select_smem > 200 * 1024) return BSA_ERR_UNSUPPORTED;
        // one part per pair: the pair's window terms stream through a ring of 16 KB shared-memory stages,
        // next to the keys, the window scores and one weight per (chunk, head)
        P.select_ring = 0;
        if (P.select_parts == 1) {
            // 200 KB of dynamic shared memory at most: the top-k's histogram is static (16 KB)
            const size_t rest = 1024 + P.select_smem + (size_t)P.nstat * P.Gp * sizeof(float);
            int64_t ring = ((size_t)200 * 1024 > rest) ? ((size_t)200 * 1024 - rest) / (16 * 1024) : 0;
            if (ring > 8) ring = 8;
            if (ring >= 2) P.select_ring = (int)ring;
        }
    }
    // Decode split: about eight blocks per SM slot in flight, whole blocks per CTA.
    {
        const int64_t total = (int64_t)P.layers * P.pairs * P.sel_cap;
        int64_t bpc = total / (kNumSMs * 8);
        if (bpc < 1) bpc = 1;
        if (bpc > 16) bpc = 16;
        if (bpc > P.sel_cap) bpc = P.sel_cap;
        int64_t splits = (P.sel_cap + bpc - 1) / bpc;
        if (splits * P.Gp > kMaxCombineSlots) splits = kMaxCombineSlots / P.Gp;
        P.dec_splits = (int)splits;
        P.dec_bpc = (int)((P.sel_cap + splits - 1) / splits);
        // bf16: C persistent CTAs, each an equal contiguous share of the layers * pairs * SEL_cap
        // block slots; a (layer, pair) then spans at most ceil(SEL_cap / per_cta) + 1 CTAs
        const int64_t slots_total = (int64_t)P.layers * P.pairs * P.sel_cap;
        int64_t ctas = 2 * kNumSMs;
        if (ctas > (slots_total + 1) / 2) ctas = (slots_total + 1) / 2;
        if (ctas < 1) ctas = 1;
        P.dec_ctas = (int)ctas;
        const int64_t per_cta = slots_total / ctas > 0 ? slots_total / ctas : 1;
        P.dec_slots = P.dtype == BSA_BF16 ? (int)((P.sel_cap + per_cta - 1) / per_cta + 2) : P.dec_splits;
        if ((int64_t)P.dec_slots * P.Gp > kMaxCombineSlots) return BSA_ERR_UNSUPPORTED;
        P.stage_tokens = P.BS % 64 == 0 ? 64 : (P.BS % 32 == 0 ? 32 : 16);
        // TMA row coordinates are 32-bit: every cache row must be addressable
        if (P.dtype == BSA_BF16 && (int64_t)P.pairs * P.T_cap > 0x7fffffffLL)
            return BSA_ERR_UNSUPPORTED;
    }
    // Fused step (bf16): blocks of four windows (BS = 4s, l = s or 2s; the paper's 64 / 16 / 32),
    // BS a multiple of the 64-token attention unit, the pair's window terms in tensor memory (512
    // columns: tiles of 32 blocks, four per 4 * Gp columns, plus the slack of one block-maximum load
    // of up to two tiles) and the rest in one CTA.
    {
        P.step_fused = 0;
        const bool geo = P.BS == 4 * P.s && (P.l == P.s || P.l == 2 * P.s) && P.BS % 64 == 0;
        if (P.dtype == BSA_BF16 && geo && P.nc_cap > 0 && P.nb_cap <= 16384) {
            P.step_sgp = P.Gp;
            P.step_nch_cap = (int)((P.nc_cap + 63) / 64);
            const int64_t tiles = (P.step_nch_cap + 1) / 2;
            const int64_t block_tiles = (P.nb_cap + 31) / 32;
            const int64_t t_max = tiles > block_tiles ? tiles : block_tiles;
            const int64_t cols = ((t_max + 3) / 4 + 2) * 4 * P.Gp;
            uint32_t tc = 32;
            while ((int64_t)tc < cols) tc <<= 1;
            P.step_key_words = (int)((P.nb_cap + 3) / 4 * 4);
            P.step_smem = step_smem_bytes(P.D, P.Gp, P.G, P.step_nch_cap, P.step_key_words, P.sel_cap);
            if (tc <= 512 && P.step_smem > 0) {
                P.step_tmem_cols = tc;
                P.step_ctas = P.pairs < kNumSMs ? P.pairs : kNumSMs;
                P.step_fused = 1;
                // one CTA per pair streams at most ~50 GB/s: with fewer pairs than about two thirds
                // of the SMs, the chained kernels (spread over every SM) are faster
                P.step_preferred = 3 * P.pairs >= 2 * kNumSMs;
            }
        }
    }
    // Workspace
    size_t off = 0;
    P.off_err = off;
    off = align_up(off + sizeof(uint32_t));
    P.off_sel_cnt = off;
    off = align_up(off + (size_t)P.pairs * sizeof(int));
    P.off_dec_cnt = off;
    off = align_up(off + (size_t)P.layers * P.pairs * sizeof(int));
    P.off_logits = off;
    off = align_up(off + (size_t)P.pairs * P.lg_stride * P.Gp * sizeof(float));
    P.off_stats = off;
    off = align_up(off + (size_t)P.pairs * P.nstat * P.Gp * sizeof(float2));
    P.off_bscores = off;
    off = align_up(off + (size_t)P.pairs * P.nb_cap * sizeof(float));
    P.off_part_ml = off;
    off = align_up(off + (size_t)P.layers * P.pairs * P.dec_slots * P.Gp * sizeof(float2));
    P.off_part_acc = off;
    off = align_up(off + (size_t)P.layers * P.pairs * P.dec_slots * P.Gp * P.D * sizeof(float));
    P.ws_bytes = off;
    return BSA_OK;
}

template <typename T>
T* ws_at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

bsa_status_t check_ws(const Plan& P, void* ws, size_t bytes) {
    if (!ws || bytes < P.ws_bytes || !is_aligned(ws, kAlign)) return BSA_ERR_WORKSPACE;
    return BSA_OK;
}

bsa_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? BSA_OK : BSA_ERR_CUDA; }

bool ok16(const void* p) { return p && is_aligned(p, 16); }
bool ok4(const void* p) { return p && is_aligned(p, 4); }

ScoreArgs score_args(const Plan& P, const void* q, const void* ck, const int32_t* seq_lens,
                     void* ws) {
    ScoreArgs a;
    memset(&a, 0, sizeof a);
    a.q = q;
    a.ck = ck;
    a.seq_lens = seq_lens;
    a.err = ws_at<uint32_t>(ws, P.off_err);
    a.logits = ws_at<float>(ws, P.off_logits);
    a.stats = ws_at<float2>(ws, P.off_stats);
    a.B = P.B;
    a.Hq = P.Hq;
    a.Hkv = P.Hkv;
    a.G = P.G;
    a.Gp = P.Gp;
    a.l = P.l;
    a.s = P.s;
    a.T_cap = P.T_cap;
    a.nc_cap = P.nc_cap;
    a.lg_stride = P.lg_stride;
    a.nchunk = P.nchunk;
    a.total_chunks = P.total_chunks;
    a.nstat = P.nstat;
    a.score_log2 = P.score_log2;
    return a;
}

SelectArgs select_args(const Plan& P, const int32_t* seq_lens, int32_t* block_idx, int32_t* n_sel,
                       float* block_scores, void* ws) {
    SelectArgs a;
    memset(&a, 0, sizeof a);
    a.seq_lens = seq_lens;
    a.logits = ws_at<float>(ws, P.off_logits);
    a.stats = ws_at<float2>(ws, P.off_stats);
    a.bscores = ws_at<float>(ws, P.off_bscores);
    a.block_scores = block_scores;
    a.block_idx = block_idx;
    a.n_sel = n_sel;
    a.err = ws_at<uint32_t>(ws, P.off_err);
    a.cnt = ws_at<int>(ws, P.off_sel_cnt);
    a.Hkv = P.Hkv;
    a.G = P.G;
    a.Gp = P.Gp;
    a.l = P.l;
    a.s = P.s;
    a.BS = P.BS;
    a.n_init = P.n_init;
    a.n_local = P.n_local;
    a.top_k = P.top_k;
    a.sel_cap = P.sel_cap;
    a.T_cap = P.T_cap;
    a.nc_cap = P.nc_cap;
    a.nb_cap = P.nb_cap;
    a.lg_stride = P.lg_stride;
    a.nstat = P.nstat;
    a.key_words = (int64_t)P.select_keys;
    a.ring = P.select_ring;
    a.parts = P.select_parts;
    a.part_windows = P.select_part_windows;
    return a;
}

// Scoring then selection, chained on the stream.
// The TMA descriptor of a compressed-key array, re-encoded only when the array changes.
struct CkMapCache {
    CUtensorMap map;
    MapKey key;
};

bsa_status_t do_select(const Plan& P, const void* q, const void* ck, const int32_t* seq_lens,
                       int32_t* block_idx, int32_t* n_sel, float* block_scores, void* ws,
                       cudaStream_t st, CkMapCache* cache = nullptr) {
    ScoreArgs sa = score_args(P, q, ck, seq_lens, ws);
    static thread_local CkMapCache own;
    CkMapCache& c = cache ? *cache : own;
    if (P.dtype == BSA_BF16 && P.nc_cap > 0 &&
        !encode_kv_map_cached(&c.map, &c.key, ck, (uint64_t)P.pairs * P.nc_cap, P.D, 64))
        return BSA_ERR_CUDA;
    cudaError_t e = launch_score(P, sa, &c.map, st);
    if (e != cudaSuccess) return BSA_ERR_CUDA;
    SelectArgs la = select_args(P, seq_lens, block_idx, n_sel, block_scores, ws);
    return from_cuda(launch_select(P, la, st));
}

DecodeArgs decode_args(const Plan& P, const int32_t* seq_lens, const int32_t* block_idx,
                       const int32_t* n_sel, void* ws) {
    DecodeArgs a;
    memset(&a, 0, sizeof a);
    a.seq_lens = seq_lens;
    a.block_idx = block_idx;
    a.n_sel = n_sel;
    a.err = ws_at<uint32_t>(ws, P.off_err);
    a.cnt = ws_at<int>(ws, P.off_dec_cnt);
    a.part_ml = ws_at<float2>(ws, P.off_part_ml);
    a.part_acc = ws_at<float>(ws, P.off_part_acc);
    a.Hq = P.Hq;
    a.Hkv = P.Hkv;
    a.G = P.G;
    a.Gp = P.Gp;
    a.BS = P.BS;
    a.sel_cap = P.sel_cap;
    a.pairs = P.pairs;
    a.T_cap = P.T_cap;
    a.splits = P.dec_splits;
    a.bpc = P.dec_bpc;
    a.slots = P.dec_slots;
    a.ctas = P.dec_ctas;
    a.stage_tokens = P.stage_tokens;
    a.scale_log2 = P.scale_log2;
    return a;
}

// TMA descriptors of the layers' caches (bf16 path only).
// (Each entry point keeps its descriptors, with the tensors they were encoded for, per thread.)
struct KVMapCache {
    KVMaps maps;
    MapKey k[BSA_MAX_LAYERS], v[BSA_MAX_LAYERS];
};

bsa_status_t make_maps(const Plan& P, const DecodeArgs& a, int layers, KVMapCache* c) {
    if (P.dtype != BSA_BF16) return BSA_OK;
    const uint64_t rows = (uint64_t)P.pairs * (uint64_t)P.T_cap;
    for (int i = 0; i < layers; ++i) {
        if (!encode_kv_map_cached(&c->maps.k[i], &c->k[i], a.k[i], rows, P.D, P.stage_tokens) ||
            !encode_kv_map_cached(&c->maps.v[i], &c->v[i], a.v[i], rows, P.D, P.stage_tokens))
            return BSA_ERR_CUDA;
    }
    return BSA_OK;
}

// TMA descriptors of the fused step: compressed keys, K and V in boxes of 64 rows.
struct StepMapCache {
    StepMaps maps;
    MapKey ck, k, v;
};

StepArgs step_args(const Plan& P, const void* q, const void* f, const int32_t* seq_lens,
                   int32_t* block_idx, int32_t* n_sel, float* block_scores, void* out, float* lse,
                   void* ws) {
    StepArgs a;
    memset(&a, 0, sizeof a);
    a.q = q;
    a.f = f;
    a.seq_lens = seq_lens;
    a.block_idx = block_idx;
    a.n_sel = n_sel;
    a.block_scores = block_scores;
    a.out = out;
    a.lse = lse;
    a.err = ws_at<uint32_t>(ws, P.off_err);
    a.Hq = P.Hq;
    a.Hkv = P.Hkv;
    a.G = P.G;
    a.l = P.l;
    a.s = P.s;
    a.BS = P.BS;
    a.n_init = P.n_init;
    a.n_local = P.n_local;
    a.top_k = P.top_k;
    a.sel_cap = P.sel_cap;
    a.pairs = P.pairs;
    a.T_cap = P.T_cap;
    a.nc_cap = P.nc_cap;
    a.nb_cap = P.nb_cap;
    a.nch_cap = P.step_nch_cap;
    a.key_words = P.step_key_words;
    a.tmem_cols = P.step_tmem_cols;
    a.score_log2 = P.score_log2;
    a.scale_log2 = P.scale_log2;
    return a;
}

bsa_status_t do_step_fused(const Plan& P, const void* q, const void* k_cache, const void* v_cache,
                           const void* ck, const int32_t* seq_lens, int32_t* block_idx, int32_t* n_sel,
                           float* block_scores, void* out, float* lse, void* ws, cudaStream_t st) {
    static thread_local StepMapCache c;
    if (!encode_kv_map_cached(&c.maps.ck, &c.ck, ck, (uint64_t)P.pairs * P.nc_cap, P.D, 64) ||
        !encode_kv_map_cached(&c.maps.k, &c.k, k_cache, (uint64_t)P.pairs * P.T_cap, P.D, 64) ||
        !encode_kv_map_cached(&c.maps.v, &c.v, v_cache, (uint64_t)P.pairs * P.T_cap, P.D, 64))
        return BSA_ERR_CUDA;
    const StepArgs a = step_args(P, q, nullptr, seq_lens, block_idx, n_sel, block_scores, out, lse, ws);
    return from_cuda(launch_step(P, a, &c.maps, st));
}

bsa_status_t do_append(const Plan& P, void* k_cache, void* v_cache, const void* k_new,
                       const void* v_new, int32_t* seq_lens, void* ck, void* ws, cudaStream_t st) {
    AppendArgs a;
    memset(&a, 0, sizeof a);
    a.k = k_cache;
    a.v = v_cache;
    a.k_new = k_new;
    a.v_new = v_new;
    a.seq_lens = seq_lens;
    a.ck = ck;
    a.err = ws ? ws_at<uint32_t>(ws, P.off_err) : nullptr;
    a.Hkv = P.Hkv;
    a.D = P.D;
    a.l = P.l;
    a.s = P.s;
    a.T_cap = P.T_cap;
    a.nc_cap = P.nc_cap;
    return from_cuda(launch_append(P, a, st));
}

}  // namespace
}  // namespace bsa

using namespace bsa;

extern "C" {

const char* bsa_status_string(bsa_status_t s) {
    switch (s) {
        case BSA_OK: return "BSA_OK";
        case BSA_ERR_INVALID_ARG: return "BSA_ERR_INVALID_ARG";
        case BSA_ERR_UNSUPPORTED: return "BSA_ERR_UNSUPPORTED";
        case BSA_ERR_WORKSPACE: return "BSA_ERR_WORKSPACE";
        case BSA_ERR_CUDA: return "BSA_ERR_CUDA";
        case BSA_ERR_DEVICE_CHECK: return "BSA_ERR_DEVICE_CHECK";
    }
    return "BSA_ERR_UNKNOWN";
}

int32_t bsa_abi_version(void) { return BSA_ABI_VERSION; }

bsa_status_t bsa_check_params(const bsa_params_t* params) {
    Plan P;
    return make_plan(params, &P);
}

bsa_status_t bsa_get_sizes(const bsa_params_t* params, bsa_sizes_t* sizes) {
    if (!sizes) return BSA_ERR_INVALID_ARG;
    Plan P;
    bsa_status_t st = make_plan(params, &P);
    if (st != BSA_OK) return st;
    sizes->nc_cap = P.nc_cap;
    sizes->nb_cap = P.nb_cap;
    sizes->sel_cap = P.sel_cap;
    sizes->group = P.G;
    sizes->workspace_bytes = P.ws_bytes;
    return BSA_OK;
}

size_t bsa_workspace_size(const bsa_params_t* params) {
    Plan P;
    return make_plan(params, &P) == BSA_OK ? P.ws_bytes : 0;
}

bsa_status_t bsa_workspace_init(const bsa_params_t* params, void* ws, size_t ws_bytes,
                                cudaStream_t stream) {
    Plan P;
    bsa_status_t st = make_plan(params, &P);
    if (st != BSA_OK) return st;
    if ((st = check_ws(P, ws, ws_bytes)) != BSA_OK) return st;
    // the error word and both counter arrays are contiguous at the front
    return from_cuda(cudaMemsetAsync(ws, 0, P.off_logits, stream));
}

bsa_status_t bsa_compress_keys(const bsa_params_t* params, const void* k_cache,
                               const int32_t* seq_lens, void* ck, cudaStream_t stream) {
    Plan P;
    bsa_status_t st = make_plan(params, &P);
    if (st != BSA_OK) return st;
    if (!ok16(k_cache) || !ok4(seq_lens)) return BSA_ERR_INVALID_ARG;
    if (P.nc_cap > 0 && !ok16(ck)) return BSA_ERR_INVALID_ARG;  // no window fits: ck may be empty
    CompressArgs a;
    memset(&a, 0, sizeof a);
    a.k = k_cache;
    a.ck = ck;
    a.seq_lens = seq_lens;
    a.err = nullptr;
    a.Hkv = P.Hkv;
    a.D = P.D;
    a.l = P.l;
    a.s = P.s;
    a.T_cap = P.T_cap;
    a.nc_cap = P.nc_cap;
    if (P.nc_cap == 0) return BSA_OK;
    return from_cuda(launch_compress_keys(P, a, stream));
}

bsa_status_t bsa_compress_append(const bsa_params_t* params, void* k_cache, void* v_cache,
                                 const void* k_new, const void* v_new, int32_t* seq_lens, void* ck,
                                 void* ws, size_t ws_bytes, cudaStream_t stream) {
    Plan P;
    bsa_status_t st = make_plan(params, &P);
    if (st != BSA_OK) return st;
    if (!ok16(k_cache) || !ok16(v_cache) || !ok16(k_new) || !ok16(v_new) || !ok4(seq_lens))
        return BSA_ERR_INVALID_ARG;
    if (P.nc_cap > 0 && !ok16(ck)) return BSA_ERR_INVALID_ARG;
    if (ws && (st = check_ws(P, ws, ws_bytes)) != BSA_OK) return st;
    return do_append(P, k_cache, v_cache, k_new, v_new, seq_lens, ck, ws, stream);
}

bsa_status_t bsa_select_blocks(const bsa_params_t* params, const void* q, const void* ck,
                               const int32_t* seq_lens, int32_t* block_idx, int32_t* n_sel,
                               float* block_scores, void* ws, size_t ws_bytes,
                               cudaStream_t stream) {
    Plan P;
    bsa_status_t st = make_plan(params, &P);
    if (st != BSA_OK) return st;
    if (!ok16(q) || !ok4(seq_lens) || !ok4(block_idx) || !ok4(n_sel)) return BSA_ERR_INVALID_ARG;
    if (P.nc_cap > 0 && !ok16(ck)) return BSA_ERR_INVALID_ARG;
    if (block_scores && !ok4(block_scores)) return BSA_ERR_INVALID_ARG;
    if ((st = check_ws(P, ws, ws_bytes)) != BSA_OK) return st;
    return do_select(P, q, ck, seq_lens, block_idx, n_sel, block_scores, ws, stream);
}

bsa_status_t bsa_select_blocks_forecast(const bsa_params_t* params, const void* f, const void* ck,
                                        const int32_t* seq_lens, int32_t* block_idx, int32_t* n_sel,
                                        float* block_scores, void* ws, size_t ws_bytes,
                                        cudaStream_t stream) {
    Plan P;
    bsa_status_t st = make_plan(params, &P);
    if (st != BSA_OK) return st;
    if (!ok16(f) || !ok4(seq_lens) || !ok4(block_idx) || !ok4(n_sel)) return BSA_ERR_INVALID_ARG;
    if (P.nc_cap > 0 && !ok16(ck)) return BSA_ERR_INVALID_ARG;
    if (block_scores && !ok4(block_scores)) return BSA_ERR_INVALID_ARG;
    if ((st = check_ws(P, ws, ws_bytes)) != BSA_OK) return st;
    // one scoring head per group: the plan of a problem with Hq = Hkv, whose workspace is a prefix
    // of this one's (same counters, smaller score and partial arrays)
    bsa_params_t pf = *params;
    pf.num_q_heads = pf.num_kv_heads;
    Plan F;
    if ((st = make_plan(&pf, &F)) != BSA_OK) return st;
    if (F.ws_bytes > P.ws_bytes || F.off_logits != P.off_logits) return BSA_ERR_UNSUPPORTED;
    ScoreArgs sa = score_args(F, f, ck, seq_lens, ws);
    sa.raw = 1;
    sa.score_log2 = 1.f;  // the raw dot products
    static thread_local CUtensorMap ck_map;
    static thread_local MapKey ck_key;
    if (F.dtype == BSA_BF16 && F.nc_cap > 0 &&
        !encode_kv_map_cached(&ck_map, &ck_key, ck, (uint64_t)F.pairs * F.nc_cap, F.D, 64))
        return BSA_ERR_CUDA;
    if (launch_score(F, sa, &ck_map, stream) != cudaSuccess) return BSA_ERR_CUDA;
    SelectArgs la = select_args(F, seq_lens, block_idx, n_sel, block_scores, ws);
    la.raw = 1;
    return from_cuda(launch_select(F, la, stream));
}

bsa_status_t bsa_sparse_decode_layers(const bsa_params_t* params, int32_t num_layers,
                                      const void* const* q, const void* const* k_caches,
                                      const void* const* v_caches, const int32_t* seq_lens,
                                      const int32_t* block_idx, const int32_t* n_sel,
                                      void* const* outs, float* const* lses, void* ws,
                                      size_t ws_bytes, cudaStream_t stream) {
    Plan P;
    bsa_status_t st = make_plan(params, &P);
    if (st != BSA_OK) return st;
    if (num_layers < 1 || num_layers > P.layers) return BSA_ERR_INVALID_ARG;
    if (!q || !k_caches || !v_caches || !outs) return BSA_ERR_INVALID_ARG;
    if (!ok4(seq_lens) || !ok4(block_idx) || !ok4(n_sel)) return BSA_ERR_INVALID_ARG;
    if ((st = check_ws(P, ws, ws_bytes)) != BSA_OK) return st;
    DecodeArgs a = decode_args(P, seq_lens, block_idx, n_sel, ws);
    for (int i = 0; i < num_layers; ++i) {
        if (!ok16(q[i]) || !ok16(k_caches[i]) || !ok16(v_caches[i]) || !ok16(outs[i]))
            return BSA_ERR_INVALID_ARG;
        float* lse = lses ? lses[i] : nullptr;
        if (lse && !ok4(lse)) return BSA_ERR_INVALID_ARG;
        a.q[i] = q[i];
        a.k[i] = k_caches[i];
        a.v[i] = v_caches[i];
        a.out[i] = outs[i];
        a.lse[i] = lse;
    }
    static thread_local KVMapCache maps;
    if ((st = make_maps(P, a, num_layers, &maps)) != BSA_OK) return st;
    return from_cuda(launch_decode(P, a, &maps.maps, num_layers, stream));
}

bsa_status_t bsa_decode_step_anchored(const bsa_params_t* params, int32_t num_layers,
                                      const int32_t* anchors, int32_t num_anchors,
                                      const void* const* q, const void* const* k_caches,
                                      const void* const* v_caches, const void* const* cks,
                                      const int32_t* seq_lens, int32_t* block_idx, int32_t* n_sel,
                                      void* const* outs, float* const* lses, void* ws,
                                      size_t ws_bytes, cudaStream_t stream) {
    Plan P;
    bsa_status_t st = make_plan(params, &P);
    if (st != BSA_OK) return st;
    if (num_layers < 1 || num_layers > P.layers) return BSA_ERR_INVALID_ARG;
    if (!anchors || num_anchors < 1 || num_anchors > num_layers || anchors[0] != 0)
        return BSA_ERR_INVALID_ARG;
    for (int i = 1; i < num_anchors; ++i)
        if (anchors[i] <= anchors[i - 1] || anchors[i] >= num_layers) return BSA_ERR_INVALID_ARG;
    if (!q || !k_caches || !v_caches || !cks || !outs) return BSA_ERR_INVALID_ARG;
    if (!ok4(seq_lens) || !ok4(block_idx) || !ok4(n_sel)) return BSA_ERR_INVALID_ARG;
    for (int l = 0; l < num_layers; ++l) {
        if (!ok16(q[l]) || !ok16(k_caches[l]) || !ok16(v_caches[l]) || !ok16(outs[l]))
            return BSA_ERR_INVALID_ARG;
        if (lses && lses[l] && !ok4(lses[l])) return BSA_ERR_INVALID_ARG;
    }
    for (int i = 0; i < num_anchors; ++i)
        if (P.nc_cap > 0 && !ok16(cks[anchors[i]])) return BSA_ERR_INVALID_ARG;
    if ((st = check_ws(P, ws, ws_bytes)) != BSA_OK) return st;
    // one descriptor cache per anchor position, so a steady schedule never re-encodes
    static thread_local CkMapCache ck_cache[BSA_MAX_LAYERS];
    static thread_local KVMapCache kv_cache[BSA_MAX_LAYERS];
    const size_t idx_stride = (size_t)P.pairs * P.sel_cap;
    for (int i = 0; i < num_anchors; ++i) {
        const int a0 = anchors[i], a1 = i + 1 < num_anchors ? anchors[i + 1] : num_layers;
        int32_t* bi = block_idx + (size_t)i * idx_stride;
        int32_t* ns = n_sel + (size_t)i * P.pairs;
        if ((st = do_select(P, q[a0], cks[a0], seq_lens, bi, ns, nullptr, ws, stream, &ck_cache[i])) !=
            BSA_OK)
            return st;
        DecodeArgs da = decode_args(P, seq_lens, bi, ns, ws);
        for (int l = a0; l < a1; ++l) {
            da.q[l - a0] = q[l];
            da.k[l - a0] = k_caches[l];
            da.v[l - a0] = v_caches[l];
            da.out[l - a0] = outs[l];
            da.lse[l - a0] = lses ? lses[l] : nullptr;
        }
        if ((st = make_maps(P, da, a1 - a0, &kv_cache[i])) != BSA_OK) return st;
        if ((st = from_cuda(launch_decode(P, da, &kv_cache[i].maps, a1 - a0, stream))) != BSA_OK)
            return st;
    }
    return BSA_OK;
}

bsa_status_t bsa_sparse_decode(const bsa_params_t* params, const void* q, const void* k_cache,
                               const void* v_cache, const int32_t* seq_lens,
                               const int32_t* block_idx, const int32_t* n_sel, void* out,
                               float* lse, void* ws, size_t ws_bytes, cudaStream_t stream) {
    const void* qs[1] = {q};
    const void* ks[1] = {k_cache};
    const void* vs[1] = {v_cache};
    void* os[1] = {out};
    float* ls[1] = {lse};
    return bsa_sparse_decode_layers(params, 1, qs, ks, vs, seq_lens, block_idx, n_sel, os, ls, ws,
                                    ws_bytes, stream);
}

}  // extern "C"

namespace bsa {
namespace {
// bsa_decode_step and bsa_decode_step_fused: `mode` 0 picks the path, 1 requires the fused one.
bsa_status_t decode_step(int mode, const bsa_params_t* params, const void* q, void* k_cache,
                         void* v_cache, void* ck, const void* k_new, const void* v_new,
                         int32_t* seq_lens, int32_t* block_idx, int32_t* n_sel, float* block_scores,
                         void* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t stream) {
    Plan P;
    bsa_status_t st = make_plan(params, &P);
    if (st != BSA_OK) return st;
    if (mode == 1 && !P.step_fused) return BSA_ERR_UNSUPPORTED;
    const bool append = k_new != nullptr && v_new != nullptr;
    if ((k_new == nullptr) != (v_new == nullptr)) return BSA_ERR_INVALID_ARG;
    if (!ok16(q) || !ok16(k_cache) || !ok16(v_cache) || !ok16(out) || !ok4(seq_lens) ||
        !ok4(block_idx) || !ok4(n_sel))
        return BSA_ERR_INVALID_ARG;
    if (P.nc_cap > 0 && !ok16(ck)) return BSA_ERR_INVALID_ARG;
    if (append && (!ok16(k_new) || !ok16(v_new))) return BSA_ERR_INVALID_ARG;
    if ((block_scores && !ok4(block_scores)) || (lse && !ok4(lse))) return BSA_ERR_INVALID_ARG;
    if ((st = check_ws(P, ws, ws_bytes)) != BSA_OK) return st;
    if (append) {
        st = do_append(P, k_cache, v_cache, k_new, v_new, seq_lens, ck, ws, stream);
        if (st != BSA_OK) return st;
    }
    if (mode == 1 || P.step_preferred)
        return do_step_fused(P, q, k_cache, v_cache, ck, seq_lens, block_idx, n_sel, block_scores, out,
                             lse, ws, stream);
    if ((st = do_select(P, q, ck, seq_lens, block_idx, n_sel, block_scores, ws, stream)) != BSA_OK)
        return st;
    DecodeArgs da = decode_args(P, seq_lens, block_idx, n_sel, ws);
    da.q[0] = q;
    da.k[0] = k_cache;
    da.v[0] = v_cache;
    da.out[0] = out;
    da.lse[0] = lse;
    static thread_local KVMapCache maps;
    if ((st = make_maps(P, da, 1, &maps)) != BSA_OK) return st;
    return from_cuda(launch_decode(P, da, &maps.maps, 1, stream));
}
}  // namespace
}  // namespace bsa

extern "C" {

bsa_status_t bsa_decode_step(const bsa_params_t* params, const void* q, void* k_cache,
                             void* v_cache, void* ck, const void* k_new, const void* v_new,
                             int32_t* seq_lens, int32_t* block_idx, int32_t* n_sel,
                             float* block_scores, void* out, float* lse, void* ws,
                             size_t ws_bytes, cudaStream_t stream) {
    return decode_step(0, params, q, k_cache, v_cache, ck, k_new, v_new, seq_lens, block_idx, n_sel,
                       block_scores, out, lse, ws, ws_bytes, stream);
}

bsa_status_t bsa_decode_step_fused(const bsa_params_t* params, const void* q, void* k_cache,
                                   void* v_cache, void* ck, const void* k_new, const void* v_new,
                                   int32_t* seq_lens, int32_t* block_idx, int32_t* n_sel,
                                   float* block_scores, void* out, float* lse, void* ws,
                                   size_t ws_bytes, cudaStream_t stream) {
    return decode_step(1, params, q, k_cache, v_cache, ck, k_new, v_new, seq_lens, block_idx, n_sel,
                       block_scores, out, lse, ws, ws_bytes, stream);
}

bsa_status_t bsa_decode_step_lookahead(const bsa_params_t* params, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* block_idx,
                                       const int32_t* n_sel, const void* f, const void* ck_next,
                                       const int32_t* seq_lens, int32_t* block_idx_next,
                                       int32_t* n_sel_next, float* block_scores_next, void* out,
                                       float* lse, void* ws, size_t ws_bytes, cudaStream_t stream) {
    Plan P;
    bsa_status_t st = make_plan(params, &P);
    if (st != BSA_OK) return st;
    if (!P.step_fused) return BSA_ERR_UNSUPPORTED;
    if (!ok16(q) || !ok16(k_cache) || !ok16(v_cache) || !ok16(f) || !ok16(ck_next) || !ok16(out) ||
        !ok4(seq_lens) || !ok4(block_idx) || !ok4(n_sel) || !ok4(block_idx_next) || !ok4(n_sel_next))
        return BSA_ERR_INVALID_ARG;
    if ((block_scores_next && !ok4(block_scores_next)) || (lse && !ok4(lse))) return BSA_ERR_INVALID_ARG;
    // the next layer's selection must not overwrite the blocks this layer reads
    const size_t idx_bytes = (size_t)P.pairs * P.sel_cap * sizeof(int32_t), ns_bytes = (size_t)P.pairs * sizeof(int32_t);
    auto overlap = [](const void* a, size_t na, const void* b, size_t nb) {
        const char *x = static_cast<const char*>(a), *y = static_cast<const char*>(b);
        return x < y + nb && y < x + na;
    };
    if (overlap(block_idx, idx_bytes, block_idx_next, idx_bytes) || overlap(block_idx, idx_bytes, n_sel_next, ns_bytes) ||
        overlap(n_sel, ns_bytes, block_idx_next, idx_bytes) || overlap(n_sel, ns_bytes, n_sel_next, ns_bytes))
        return BSA_ERR_INVALID_ARG;
    if ((st = check_ws(P, ws, ws_bytes)) != BSA_OK) return st;
    static thread_local StepMapCache c;
    if (!encode_kv_map_cached(&c.maps.ck, &c.ck, ck_next, (uint64_t)P.pairs * P.nc_cap, P.D, 64) ||
        !encode_kv_map_cached(&c.maps.k, &c.k, k_cache, (uint64_t)P.pairs * P.T_cap, P.D, 64) ||
        !encode_kv_map_cached(&c.maps.v, &c.v, v_cache, (uint64_t)P.pairs * P.T_cap, P.D, 64))
        return BSA_ERR_CUDA;
    StepArgs a = step_args(P, q, f, seq_lens, block_idx_next, n_sel_next, block_scores_next, out, lse, ws);
    a.in_idx = block_idx;
    a.in_nsel = n_sel;
    a.score_log2 = 1.f;  // the raw dot products
    return from_cuda(launch_step(P, a, &c.maps, stream));
}

}  // extern "C"

namespace bsa {
namespace {
// Prefill: argument checks and the kernels' arguments; `select` also checks the selection
// kernel's shared memory.
bsa_status_t prefill_args(const bsa_params_t* params, int32_t chunk, const void* q, const int32_t* seq_lens,
                          const int32_t* block_idx, const int32_t* n_sel, void* out, float* lse, void* ws,
                          size_t ws_bytes, bool select, Plan* P, PrefillArgs* a, size_t* smem) {
    bsa_status_t st = make_plan(params, P);
    if (st != BSA_OK) return st;
    if (P->dtype != BSA_BF16 || P->D != 128 || (P->G != 2 && P->G != 4) || P->BS != 64 || P->l != 32 ||
        P->s != 16)
        return BSA_ERR_UNSUPPORTED;
    if (chunk < 1 || chunk > P->T_cap) return BSA_ERR_INVALID_ARG;
    if (!ok16(q) || !ok16(out) || !ok4(seq_lens) || !ok4(block_idx) || !ok4(n_sel) || (lse && !ok4(lse)))
        return BSA_ERR_INVALID_ARG;
    if ((st = check_ws(*P, ws, ws_bytes)) != BSA_OK) return st;
    *smem = select ? prefill_select_smem_bytes(P->G, P->nc_cap, P->nb_cap, P->sel_cap) : 1;
    if (*smem == 0) return BSA_ERR_UNSUPPORTED;
    memset(a, 0, sizeof *a);
    a->q = q;
    a->seq_lens = seq_lens;
    a->block_idx = const_cast<int32_t*>(block_idx);
    a->n_sel = const_cast<int32_t*>(n_sel);
    a->out = out;
    a->lse = lse;
    a->err = ws_at<uint32_t>(ws, P->off_err);
    a->chunk = chunk;
    a->tiles_cap = (chunk + P->BS - 1) / P->BS + 1;
    a->Hq = P->Hq;
    a->Hkv = P->Hkv;
    a->G = P->G;
    a->n_init = P->n_init;
    a->n_local = P->n_local;
    a->top_k = P->top_k;
    a->sel_cap = P->sel_cap;
    a->pairs = P->pairs;
    a->BS = P->BS;
    a->l = P->l;
    a->s = P->s;
    a->T_cap = P->T_cap;
    a->nc_cap = P->nc_cap;
    a->nb_cap = P->nb_cap;
    a->score_log2 = P->score_log2;
    a->scale_log2 = P->scale_log2;
    if ((int64_t)P->pairs * a->tiles_cap > 0x7fffffffLL / 2) return BSA_ERR_UNSUPPORTED;
    return BSA_OK;
}
struct PrefillMapCache {
    CUtensorMap ck, k, v;
    MapKey kck, kk, kv;
};
}  // namespace
}  // namespace bsa

extern "C" {

}  // extern "C"

namespace bsa {
namespace {
// CLSA: the plan of the token scorer (windows of one token over the index layer's keys).
bsa_status_t clsa_plan(const bsa_params_t* params, Plan* P, Plan* F) {
    bsa_status_t st = make_plan(params, P);
    if (st != BSA_OK) return st;
    if (P->dtype != BSA_BF16) return BSA_ERR_UNSUPPORTED;
    bsa_params_t pt = *params;
    pt.cmp_kernel = 1;
    pt.cmp_stride = 1;
    if ((st = make_plan(&pt, F)) != BSA_OK) return st;
    const int64_t tok_cap = (int64_t)P->sel_cap * P->BS;
    if (tok_cap > 0x7fffffff / 2 || token_topk_smem_bytes(F->T_cap, F->nstat, F->Gp) == 0) return BSA_ERR_UNSUPPORTED;
    return BSA_OK;
}
}  // namespace
}  // namespace bsa

extern "C" {

size_t bsa_clsa_workspace_size(const bsa_params_t* params) {
    Plan P, F;
    return clsa_plan(params, &P, &F) == BSA_OK ? F.ws_bytes : 0;
}

bsa_status_t bsa_decode_step_clsa(const bsa_params_t* params, int32_t num_layers, const void* const* q,
                                  const void* const* k_caches, const void* const* v_caches,
                                  const int32_t* seq_lens, int32_t* tok_idx, int32_t* n_tok, void* const* outs,
                                  float* const* lses, void* ws, size_t ws_bytes, cudaStream_t stream) {
    Plan P, F;
    bsa_status_t st = clsa_plan(params, &P, &F);
    if (st != BSA_OK) return st;
    if (!q || !k_caches || !v_caches || !outs) return BSA_ERR_INVALID_ARG;
    if (num_layers < 1 || num_layers > BSA_MAX_LAYERS || num_layers > P.layers) return BSA_ERR_INVALID_ARG;
    if (!ok4(seq_lens) || !ok4(tok_idx) || !ok4(n_tok)) return BSA_ERR_INVALID_ARG;
    TokenLayers L;
    memset(&L, 0, sizeof L);
    for (int i = 0; i < num_layers; ++i) {
        if (!ok16(q[i]) || !ok16(k_caches[i]) || !ok16(v_caches[i]) || !ok16(outs[i])) return BSA_ERR_INVALID_ARG;
        if (lses && lses[i] && !ok4(lses[i])) return BSA_ERR_INVALID_ARG;
        L.q[i] = q[i];
        L.k[i] = k_caches[i];
        L.v[i] = v_caches[i];
        L.out[i] = outs[i];
        L.lse[i] = lses ? lses[i] : nullptr;
    }
    if ((st = check_ws(F, ws, ws_bytes)) != BSA_OK) return st;
    // token scoring of the index layer (layer 0): its K cache is the scorer's "compressed keys"
    ScoreArgs sa = score_args(F, q[0], k_caches[0], seq_lens, ws);
    static thread_local CUtensorMap k_map;
    static thread_local MapKey k_key;
    if (!encode_kv_map_cached(&k_map, &k_key, k_caches[0], (uint64_t)F.pairs * F.nc_cap, F.D, 64))
        return BSA_ERR_CUDA;
    if (launch_score(F, sa, &k_map, stream) != cudaSuccess) return BSA_ERR_CUDA;
    TokenArgs a;
    memset(&a, 0, sizeof a);
    a.seq_lens = seq_lens;
    a.logits = ws_at<float>(ws, F.off_logits);
    a.stats = ws_at<float2>(ws, F.off_stats);
    a.tok_idx = tok_idx;
    a.n_tok = n_tok;
    a.err = ws_at<uint32_t>(ws, F.off_err);
    a.Hq = P.Hq;
    a.Hkv = P.Hkv;
    a.G = P.G;
    a.pairs = P.pairs;
    a.n_init_tok = P.n_init * P.BS;
    a.n_local_tok = P.n_local * P.BS;
    a.top_k_tok = P.top_k * P.BS;
    a.tok_cap = P.sel_cap * P.BS;
    a.T_cap = F.T_cap;
    a.lg_stride = F.lg_stride;
    a.nstat = F.nstat;
    a.scale_log2 = P.scale_log2;
    if (launch_token_topk(a, F.Gp, token_topk_smem_bytes(F.T_cap, F.nstat, F.Gp), stream) != cudaSuccess)
        return BSA_ERR_CUDA;
    return from_cuda(launch_token_decode(a, L, num_layers, P.D, stream));
}

int32_t bsa_prefill_tiles(int32_t chunk, int32_t block_size) {
    return chunk < 1 || block_size < 1 ? 0 : (chunk + block_size - 1) / block_size + 1;
}

bsa_status_t bsa_prefill(const bsa_params_t* params, int32_t chunk, const void* q, const void* k_cache,
                         const void* v_cache, const void* ck, const int32_t* seq_lens, int32_t* block_idx,
                         int32_t* n_sel, void* out, float* lse, void* ws, size_t ws_bytes, cudaStream_t stream) {
    Plan P;
    PrefillArgs a;
    size_t smem = 0;
    bsa_status_t st = prefill_args(params, chunk, q, seq_lens, block_idx, n_sel, out, lse, ws, ws_bytes, true, &P,
                                   &a, &smem);
    if (st != BSA_OK) return st;
    if (!ok16(k_cache) || !ok16(v_cache) || (P.nc_cap > 0 && !ok16(ck))) return BSA_ERR_INVALID_ARG;
    static thread_local PrefillMapCache c;
    if ((P.nc_cap > 0 &&
         !encode_kv_map_cached(&c.ck, &c.kck, ck, (uint64_t)P.pairs * P.nc_cap, P.D, 128)) ||
        !encode_kv_map_cached(&c.k, &c.kk, k_cache, (uint64_t)P.pairs * P.T_cap, P.D, 64) ||
        !encode_kv_map_cached(&c.v, &c.kv, v_cache, (uint64_t)P.pairs * P.T_cap, P.D, 64))
        return BSA_ERR_CUDA;
    const int64_t items = (int64_t)P.pairs * a.tiles_cap;
    const int ctas = (int)(items < kNumSMs ? items : kNumSMs);
    cudaError_t e = launch_prefill_select(a, &c.ck, smem, ctas, stream);
    if (e != cudaSuccess) return BSA_ERR_CUDA;
    return from_cuda(launch_prefill_attend(a, &c.k, &c.v, stream));
}

bsa_status_t bsa_prefill_attend(const bsa_params_t* params, int32_t chunk, const void* q, const void* k_cache,
                                const void* v_cache, const int32_t* seq_lens, const int32_t* block_idx,
                                const int32_t* n_sel, void* out, float* lse, void* ws, size_t ws_bytes,
                                cudaStream_t stream) {
    Plan P;
    PrefillArgs a;
    size_t smem = 0;
    bsa_status_t st = prefill_args(params, chunk, q, seq_lens, block_idx, n_sel, out, lse, ws, ws_bytes, false, &P,
                                   &a, &smem);
    if (st != BSA_OK) return st;
    if (!ok16(k_cache) || !ok16(v_cache)) return BSA_ERR_INVALID_ARG;
    static thread_local PrefillMapCache c;
    if (!encode_kv_map_cached(&c.k, &c.kk, k_cache, (uint64_t)P.pairs * P.T_cap, P.D, 64) ||
        !encode_kv_map_cached(&c.v, &c.kv, v_cache, (uint64_t)P.pairs * P.T_cap, P.D, 64))
        return BSA_ERR_CUDA;
    return from_cuda(launch_prefill_attend(a, &c.k, &c.v, stream));
}

bsa_status_t bsa_decode_step_info(const bsa_params_t* params, int32_t append, int32_t* fused,
                                  int32_t* launches) {
    Plan P;
    bsa_status_t st = make_plan(params, &P);
    if (st != BSA_OK) return st;
    if (fused) *fused = P.step_preferred;
    // fused: the step kernel; chained: scoring, selection, attention (+ combine for bf16)
    const int32_t n = P.step_preferred ? 1 : (P.dtype == BSA_BF16 ? 4 : 3);
    if (launches) *launches = n + (append ? 1 : 0);
    return BSA_OK;
}

bsa_status_t bsa_read_device_error(void* ws, size_t ws_bytes, uint32_t* flags,
                                   cudaStream_t stream) {
    if (!flags) return BSA_ERR_INVALID_ARG;
    if (!ws || ws_bytes < sizeof(uint32_t) || !is_aligned(ws, kAlign)) return BSA_ERR_WORKSPACE;
    uint32_t v = 0;
    if (cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
        return BSA_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, sizeof v, stream) != cudaSuccess) return BSA_ERR_CUDA;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return BSA_ERR_CUDA;
    *flags = v;
    return v ? BSA_ERR_DEVICE_CHECK : BSA_OK;
}

}  // extern "C"

// ============================================================ decode without a caller workspace
// For callers that cannot allocate device memory: the sparse attention's split partials and
// completion counters live in a fixed array of this library instead of a caller's workspace.
#include <mutex>

namespace bsa {
namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)4 << 20;  // BSA_NOALLOC_SCRATCH_BYTES
static_assert(kNoAllocScratchBytes == BSA_NOALLOC_SCRATCH_BYTES, "header and library agree");
constexpr int kNoAllocMaxDevices = 64;

// Zero when the library's device code is loaded; every call re-zeroes its counter region.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of the scratch on the current device, looked up once per device (with that
// device current: the lookup may load this library's device code onto it).
bsa_status_t noalloc_scratch(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return BSA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress((void**)&p, g_noalloc_scratch) != cudaSuccess || !p)
            return BSA_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return BSA_OK;
}

// The decode part of the workspace layout (error word, counters, partials), packed from offset 0.
Plan noalloc_layout(const Plan& P) {
    Plan V = P;
    size_t off = 0;
    V.off_err = off;
    off = align_up(off + sizeof(uint32_t));
    V.off_dec_cnt = off;
    off = align_up(off + (size_t)P.layers * P.pairs * sizeof(int));
    V.off_part_ml = off;
    off = align_up(off + (size_t)P.layers * P.pairs * P.dec_slots * P.Gp * sizeof(float2));
    V.off_part_acc = off;
    off = align_up(off + (size_t)P.layers * P.pairs * P.dec_slots * P.Gp * P.D * sizeof(float));
    V.ws_bytes = off;
    return V;
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status_t bsa_sparse_decode_noalloc(const bsa_params_t* params, const void* q,
                                                  const void* k_cache, const void* v_cache,
                                                  const int32_t* seq_lens,
                                                  const int32_t* block_idx, const int32_t* n_sel,
                                                  void* out, float* lse, uint32_t* device_error,
                                                  cudaStream_t stream) {
    // one layer is attended: the scratch is laid out for one, whatever num_layers says
    if (!params) return BSA_ERR_INVALID_ARG;
    bsa_params_t one = *params;
    one.num_layers = 1;
    Plan P;
    bsa_status_t st = make_plan(&one, &P);
    if (st != BSA_OK) return st;
    if (!ok16(q) || !ok16(k_cache) || !ok16(v_cache) || !ok16(out) || !ok4(seq_lens) ||
        !ok4(block_idx) || !ok4(n_sel))
        return BSA_ERR_INVALID_ARG;
    if ((lse && !ok4(lse)) || (device_error && !ok4(device_error))) return BSA_ERR_INVALID_ARG;
    const Plan V = noalloc_layout(P);
    if (V.ws_bytes > kNoAllocScratchBytes) return BSA_ERR_WORKSPACE;  // before any CUDA call
    // the scratch used is the current device's: the stream must belong to that device
    if (stream != 0 && stream != cudaStreamLegacy && stream != cudaStreamPerThread) {
        int cur = -1, sdev = -1;
        if (cudaGetDevice(&cur) != cudaSuccess || cudaStreamGetDevice(stream, &sdev) != cudaSuccess)
            return BSA_ERR_CUDA;
        if (sdev != cur) return BSA_ERR_INVALID_ARG;
    }
    void* scratch = nullptr;
    if ((st = noalloc_scratch(&scratch)) != BSA_OK) return st;
    // error word and counters must start at zero: clear them on the stream, ahead of the kernel
    if (cudaMemsetAsync(scratch, 0, V.off_part_ml, stream) != cudaSuccess) return BSA_ERR_CUDA;
    DecodeArgs a = decode_args(V, seq_lens, block_idx, n_sel, scratch);
    if (device_error) a.err = device_error;
    a.q[0] = q;
    a.k[0] = k_cache;
    a.v[0] = v_cache;
    a.out[0] = out;
    a.lse[0] = lse;
    static thread_local KVMapCache maps;
    if ((st = make_maps(P, a, 1, &maps)) != BSA_OK) return st;
    return from_cuda(launch_decode(P, a, &maps.maps, 1, stream));
}
