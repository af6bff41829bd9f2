// Internal declarations of libbsa: launch plan, workspace layout, kernel argument blocks and
// small PTX helpers for sm_100a. Nothing here is part of the C ABI (include/bsa.h is).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "bsa.h"

namespace bsa {

constexpr int kMaxG = 8;         // query heads per kv head handled by one mma tile (N = 8)
constexpr int kScoreWarps = 8;   // warps per scoring CTA
constexpr int kDecodeWarps = 4;  // warps per decode CTA
constexpr int kMaxNbCap = 32768; // selection blocks per sequence (shared-memory key array)
constexpr int kMaxCombineSlots = 1024;  // splits * Gp handled by the decode combine

// ------------------------------------------------------------------------------------------------
// Launch plan: every size and workspace offset derived from bsa_params_t. The same function feeds
// bsa_workspace_size and the launches, so the two always agree.
struct Plan {
    int B, Hq, Hkv, G, Gp, D, l, s, BS, n_init, n_local, top_k, sel_cap, layers, dtype;
    int64_t T_cap, nc_cap, nb_cap;
    int64_t lg_stride;  // windows per pair in the window-term array (nc_cap rounded up to 4: 16 B)
    int pairs;
    float scale_log2;  // attention scale * log2(e): softmax evaluated with exp2
    float score_log2;  // (1 / tau) * log2(e)
    // scoring: 64-row chunks of compressed keys spread evenly over a persistent grid; softmax
    // statistics per chunk
    int64_t nchunk, total_chunks, nstat;
    int score_ctas;
    // selection: pairs * select_parts CTAs, each scoring select_part_windows windows
    int select_parts, select_part_windows;
    size_t select_keys;  // words of the block-key array at the front of its shared memory
    size_t select_smem;  // dynamic shared memory of the selection kernel
    int select_ring;     // one-part selection: 16 KB window-term stages in flight (0: general kernel)
    // decode: grid = layers * pairs * dec_splits CTAs of kDecodeWarps warps, dec_bpc blocks each
    int dec_splits, dec_bpc;
    int dec_ctas, dec_slots;  // bf16: persistent CTAs; partial slots per (layer, pair)
    int stage_tokens;  // bf16 decode pipeline stage: 64, 32 or 16 tokens (divides BS)
    // fused step (bf16): one CTA per pair (a persistent grid walks the pairs); 0 when the shape is
    // outside what that kernel handles, and the step then chains the separate kernels
    int step_fused, step_ctas, step_sgp, step_nch_cap, step_key_words;
    int step_preferred;  // bsa_decode_step takes the fused path (enough pairs to fill the SMs)
    uint32_t step_tmem_cols;
    size_t step_smem;
    // workspace layout (bytes)
    size_t off_err, off_sel_cnt, off_dec_cnt, off_logits, off_stats, off_bscores, off_part_ml,
        off_part_acc;
    size_t ws_bytes;
};

struct CompressArgs {
    const void* k;
    void* ck;
    const int32_t* seq_lens;
    uint32_t* err;  // may be null
    int Hkv, D, l, s, windows_per_cta;
    int64_t T_cap, nc_cap;
};

struct AppendArgs {
    void* k;
    void* v;
    const void* k_new;
    const void* v_new;
    int32_t* seq_lens;
    void* ck;
    uint32_t* err;  // may be null
    int Hkv, D, l, s;
    int64_t T_cap, nc_cap;
};

struct ScoreArgs {
    const void* q;
    const void* ck;
    const int32_t* seq_lens;
    uint32_t* err;
    float* logits;        // [pairs][lg_stride][Gp] window terms: exp2(x - chunk max), or raw x
    float2* stats;        // [pairs][nstat][Gp] (max, sum of exp2(x - max)) per chunk and head
    int B, Hq, Hkv, G, Gp, l, s;
    int64_t T_cap, nc_cap, lg_stride, nchunk, total_chunks, nstat;
    float score_log2;
    int raw;  // Forecast indexer: store the raw scores x (no exp2, no statistics)
};

struct SelectArgs {
    const int32_t* seq_lens;
    const float* logits;
    const float2* stats;
    float* bscores;       // [pairs][nb_cap] block scores (workspace)
    float* block_scores;  // caller's copy, may be null
    int32_t* block_idx;
    int32_t* n_sel;
    uint32_t* err;
    int* cnt;             // [pairs] completion counters
    int Hkv, G, Gp, l, s, BS, n_init, n_local, top_k, sel_cap;
    int64_t T_cap, nc_cap, nb_cap, lg_stride, nstat, key_words;
    int parts, part_windows;
    int ring;  // one-part kernel: window-term stages in flight
    int raw;   // Forecast indexer: the stored scores are the window scores (weight 1, no statistics)
};

// TMA descriptors of the K and V caches of every layer (bf16 path): 2-D views
// [B*Hkv*T_cap rows][D columns], boxes of 64 columns x stage_tokens rows, 128-byte swizzle.
struct alignas(64) KVMaps {
    CUtensorMap k[BSA_MAX_LAYERS];
    CUtensorMap v[BSA_MAX_LAYERS];
};

struct DecodeArgs {
    const void* q[BSA_MAX_LAYERS];
    const void* k[BSA_MAX_LAYERS];
    const void* v[BSA_MAX_LAYERS];
    void* out[BSA_MAX_LAYERS];
    float* lse[BSA_MAX_LAYERS];
    const int32_t* seq_lens;
    const int32_t* block_idx;
    const int32_t* n_sel;
    uint32_t* err;
    int* cnt;           // [layers * pairs]
    float2* part_ml;    // [layers * pairs][splits][Gp] (max, denominator) in log2 units
    float* part_acc;    // [layers * pairs][splits][Gp][D] unnormalised numerators
    int Hq, Hkv, G, Gp, BS, sel_cap, pairs;
    int64_t T_cap;
    int splits, bpc;   // fp32 path: CTA = (layer, pair, split) of bpc blocks
    int slots;         // partial slots per (layer, pair) in the workspace
    int ctas;          // bf16 path: persistent CTAs sharing the (layer, pair, block) slots evenly
    int stage_tokens;  // tokens per pipeline stage (bf16 path): 64, 32 or 16, dividing BS
    float scale_log2;
};

// The fused step: scoring, block reduction, top-k and attention of each (batch, kv head) pair in
// one CTA, its window terms held in tensor memory.
struct StepArgs {
    const void* q;         // [B][Hq][D] queries: the attention heads, and the scoring heads unless f
    const void* f;         // Forecast indexer: [B][Hkv][D] scoring vectors (raw scores), or null
    // lookahead (with f): this layer's blocks, chosen beforehand ([pairs][sel_cap], [pairs]); the
    // selection then goes to the next layer (block_idx, n_sel, from the next layer's compressed keys)
    const int32_t* in_idx;
    const int32_t* in_nsel;
    const int32_t* seq_lens;
    int32_t* block_idx;    // [pairs][sel_cap]
    int32_t* n_sel;        // [pairs]
    float* block_scores;   // [pairs][nb_cap] or null
    void* out;             // [B][Hq][D]
    float* lse;            // [B][Hq] or null
    uint32_t* err;
    int Hq, Hkv, G, l, s, BS, n_init, n_local, top_k, sel_cap, pairs;
    int64_t T_cap, nc_cap, nb_cap;
    int nch_cap, key_words;
    uint32_t tmem_cols;
    float score_log2, scale_log2;
};
// Block-sparse prefill of a chunk of `chunk` queries per sequence (positions T - chunk .. T - 1).
struct PrefillArgs {
    const void* q;          // [B][chunk][Hq][D]
    const int32_t* seq_lens;
    int32_t* block_idx;     // [pairs][tiles_cap][sel_cap] per query tile
    int32_t* n_sel;         // [pairs][tiles_cap]
    void* out;              // [B][chunk][Hq][D]
    float* lse;             // [B][chunk][Hq] or null
    uint32_t* err;
    int chunk, tiles_cap, Hq, Hkv, G, n_init, n_local, top_k, sel_cap, pairs, BS, l, s;
    int64_t T_cap, nc_cap, nb_cap;
    float score_log2, scale_log2;
};
cudaError_t launch_prefill_select(const PrefillArgs& a, const CUtensorMap* ck_map, size_t smem, int ctas,
                                  cudaStream_t st);
cudaError_t launch_prefill_attend(const PrefillArgs& a, const CUtensorMap* k_map, const CUtensorMap* v_map,
                                  cudaStream_t st);
// Dynamic shared memory of the prefill selection kernel, or 0 when it does not fit one CTA.
size_t prefill_select_smem_bytes(int G, int64_t nc_cap, int64_t nb_cap, int sel_cap);

// Token-level shared index (CLSA): the window terms and statistics of the token scorer, the token
// lists, and the layers that attend them.
struct TokenArgs {
    const int32_t* seq_lens;
    const float* logits;    // [pairs][lg_stride][Gp] window terms of the token scorer (one token per window)
    const float2* stats;    // [pairs][nstat][Gp]
    int32_t* tok_idx;       // [pairs][tok_cap] ascending, -1 padded
    int32_t* n_tok;         // [pairs]
    uint32_t* err;
    int Hq, Hkv, G, pairs, n_init_tok, n_local_tok, top_k_tok, tok_cap;
    int64_t T_cap, lg_stride, nstat;
    float scale_log2;
};
struct TokenLayers {
    const void* q[BSA_MAX_LAYERS];
    const void* k[BSA_MAX_LAYERS];
    const void* v[BSA_MAX_LAYERS];
    void* out[BSA_MAX_LAYERS];
    float* lse[BSA_MAX_LAYERS];
};
cudaError_t launch_token_topk(const TokenArgs& a, int Gp, size_t smem, cudaStream_t st);
cudaError_t launch_token_decode(const TokenArgs& a, const TokenLayers& L, int layers, int D, cudaStream_t st);
size_t token_topk_smem_bytes(int64_t T_cap, int64_t nstat, int Gp);

// TMA descriptors of the step: compressed keys (boxes of 64 rows), K and V (boxes of 32 rows).
struct alignas(64) StepMaps {
    CUtensorMap ck, k, v;
};

// Launchers (one per kernel family); they pick the template instance from the plan's dtype/D.
cudaError_t launch_compress_keys(const Plan& p, const CompressArgs& a, cudaStream_t st);
cudaError_t launch_append(const Plan& p, const AppendArgs& a, cudaStream_t st);
cudaError_t launch_score(const Plan& p, const ScoreArgs& a, const CUtensorMap* ck_map,
                         cudaStream_t st);
cudaError_t launch_select(const Plan& p, const SelectArgs& a, cudaStream_t st);
cudaError_t launch_decode(const Plan& p, const DecodeArgs& a, const KVMaps* maps, int layers,
                          cudaStream_t st);
cudaError_t launch_step(const Plan& p, const StepArgs& a, const StepMaps* maps, cudaStream_t st);
// Shared-memory bytes of the fused step kernel (dynamic part) for a parameter set, or 0 when its
// layout does not fit one CTA.
size_t step_smem_bytes(int D, int sgp, int G, int nch_cap, int key_words, int sel_cap);
// Encode a 2-D bf16 TMA descriptor over rows x D elements (128-byte swizzle, box 64 x box_rows).
bool encode_kv_map(CUtensorMap* map, const void* base, uint64_t rows, int D, int box_rows);

// The arguments `map` was last encoded for: calls with the same tensor skip the encode.
struct MapKey {
    const void* base = nullptr;
    uint64_t rows = 0;
    int D = 0, box = 0;
};
inline bool encode_kv_map_cached(CUtensorMap* map, MapKey* key, const void* base, uint64_t rows,
                                 int D, int box_rows) {
    if (base && key->base == base && key->rows == rows && key->D == D && key->box == box_rows)
        return true;
    key->base = nullptr;
    if (!encode_kv_map(map, base, rows, D, box_rows)) return false;
    key->base = base;
    key->rows = rows;
    key->D = D;
    key->box = box_rows;
    return true;
}

// Raise a kernel's dynamic shared-memory limit once per device (and size), not on every launch.
template <auto Kernel>
inline cudaError_t ensure_smem(size_t smem) {
    static int done[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
    if (dev >= 0 && dev < 64 && done[dev] >= (int)smem) return cudaSuccess;
    const cudaError_t e =
        cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = (int)smem;
    return e;
}

// Launch with programmatic dependent launch allowed: the kernel may start while the previous
// kernel in the stream drains; every kernel here waits (griddepcontrol.wait) before touching
// memory that an earlier kernel writes.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ------------------------------------------------------------------------------------------------
// Device helpers
#ifdef __CUDACC__

// A thread group that synchronises as one: the whole CTA (bar 0: __syncthreads) or the first `nt`
// threads of the CTA behind named barrier `bar`. tid is the thread's index inside the group.
struct Grp {
    int tid, nt, bar;
    __device__ __forceinline__ void sync() const {
        if (bar == 0) __syncthreads();
        else asm volatile("bar.sync %0, %1;" ::"r"(bar), "r"(nt) : "memory");
    }
};

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 128-bit streaming load: read-only for the kernel's lifetime, no L1 allocation, 256-byte L2
// prefetch granule (rows of the caches are 256 bytes at d = 128 bf16).
__device__ __forceinline__ uint4 ld_stream(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Loads that bypass L1 (data written by other CTAs of the same grid).
__device__ __forceinline__ float ld_cg(const float* p) { return __ldcg(p); }
__device__ __forceinline__ float2 ld_cg(const float2* p) { return __ldcg(p); }
__device__ __forceinline__ float4 ld_cg(const float4* p) { return __ldcg(p); }
__device__ __forceinline__ int ld_cg(const int* p) { return __ldcg(p); }

__device__ __forceinline__ uint32_t u4_get(const uint4& v, int i) {
    return i == 0 ? v.x : (i == 1 ? v.y : (i == 2 ? v.z : v.w));
}

// D[16x8] += A[16x16] * B[16x8], bf16 inputs, fp32 accumulate (warp-wide).
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose an 8x8 matrix of 16-bit elements held one 32-bit register per lane.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Two floats -> packed bf16x2 (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

// Running (max, sum exp2(x - max)) of a stream of log2-domain values. The roundings are spelled
// out (explicit mul / fma) so that every kernel merging the same statistics in the same order gets
// the same bits, whatever contraction the compiler would pick in each context.
__device__ __forceinline__ void online_add(float& m, float& s, float x) {
    float mn = fmaxf(m, x);
    s = __fadd_rn(__fmul_rn(s, exp2f(m - mn)), exp2f(x - mn));
    m = mn;
}
__device__ __forceinline__ void online_merge(float& m, float& s, float m2, float s2) {
    float mn = fmaxf(m, m2);
    if (mn == -INFINITY) {
        m = mn;
        s = 0.f;
        return;
    }
    s = __fmaf_rn(s2, exp2f(m2 - mn), __fmul_rn(s, exp2f(m - mn)));
    m = mn;
}

// A window's group score S = sum over the group's heads h < G of e[h] * w[h], in head order, with
// the roundings spelled out: the selection kernels and the fused step give the same bits.
template <int GP>
__device__ __forceinline__ float group_sum(const float* e, const float* w, int G) {
    float acc = __fmul_rn(e[0], w[0]);
#pragma unroll
    for (int h = 1; h < GP; ++h)
        if (h < G) acc = __fmaf_rn(e[h], w[h], acc);
    return acc;
}

// ---- shared-memory barriers and TMA (sm_90+ instructions, used on sm_100a)
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// Arrival that counts `count` times (one warp standing for several expected arrivals).
__device__ __forceinline__ void mbar_arrive_cnt(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Wait for the phase with the given parity to complete; gives up after `limit` polls (returns
// false) so that no wait can run forever.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit) {
    for (uint32_t it = 0; it < limit; ++it) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
            " selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(done)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (done) return true;
    }
    return false;
}
// 2-D tiled TMA load of one box into shared memory, completing on `bar` (transaction bytes).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// L2 policy for data read once by a stream (it should not push out data that other kernels reread).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
// 2-D tiled TMA load with an L2 cache policy.
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, int x, int y,
                                                 uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(map), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}
// 2-D tiled TMA prefetch of one box into L2 (no shared memory, no barrier): a cache hint only, so
// it may run before the data's producer has finished (loads that follow still see what it wrote).
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap* map, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(map), "r"(x), "r"(y)
                 : "memory");
}
// 1-D bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// ---- tensor memory (TMEM, 512 columns x 128 lanes of 32 bits per SM), used here as storage
// next to shared memory. Warp w of a CTA reaches lanes 32 * (w % 4) .. 32 * (w % 4) + 31; an address
// is (lane << 16) | column. Allocation is per CTA by one warp, in powers of two of >= 32 columns.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_fence_before_sync() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_fence_after_sync() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Lane i of the warp stores v[0..N) to columns taddr.col .. +N of TMEM lane taddr.lane + i (warp-wide).
template <int N>
__device__ __forceinline__ void tmem_st(uint32_t taddr, const float (&v)[N]) {
    static_assert(N == 2 || N == 4 || N == 8 || N == 16 || N == 32, "x2, x4, x8, x16 or x32");
    const uint32_t* u = reinterpret_cast<const uint32_t*>(v);
    if constexpr (N == 2) {
        asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1, %2};" ::"r"(taddr), "r"(u[0]), "r"(u[1])
                     : "memory");
    } else if constexpr (N == 4) {
        asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr), "r"(u[0]),
                     "r"(u[1]), "r"(u[2]), "r"(u[3])
                     : "memory");
    } else if constexpr (N == 8) {
        asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                     "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7])
                     : "memory");
    } else if constexpr (N == 16) {
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
            "%13, %14, %15, %16};" ::"r"(taddr),
            "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]), "r"(u[8]),
            "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]), "r"(u[15])
            : "memory");
    } else {
        asm volatile(
            "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
            "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, "
            "%32};" ::"r"(taddr),
            "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]), "r"(u[8]),
            "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]), "r"(u[15]), "r"(u[16]),
            "r"(u[17]), "r"(u[18]), "r"(u[19]), "r"(u[20]), "r"(u[21]), "r"(u[22]), "r"(u[23]), "r"(u[24]),
            "r"(u[25]), "r"(u[26]), "r"(u[27]), "r"(u[28]), "r"(u[29]), "r"(u[30]), "r"(u[31])
            : "memory");
    }
}
// Lane i of the warp loads columns taddr.col .. +N of TMEM lane taddr.lane + i into v (warp-wide;
// complete after tmem_wait_ld).
template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float (&v)[N]) {
    static_assert(N == 2 || N == 4 || N == 8 || N == 16 || N == 32, "x2, x4, x8, x16 or x32");
    uint32_t* u = reinterpret_cast<uint32_t*>(v);
    if constexpr (N == 2) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(u[0]), "=r"(u[1]) : "r"(taddr)
                     : "memory");
    } else if constexpr (N == 4) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3])
                     : "r"(taddr)
                     : "memory");
    } else if constexpr (N == 8) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]),
                       "=r"(u[7])
                     : "r"(taddr)
                     : "memory");
    } else if constexpr (N == 16) {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
            "%14, %15}, [%16];"
            : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
              "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
            : "r"(taddr)
            : "memory");
    } else {
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
            "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
            : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
              "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15]),
              "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]),
              "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
            : "r"(taddr)
            : "memory");
    }
}

// Order-preserving map of an fp32 score onto uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t order_key(float f) {
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

#endif  // __CUDACC__

}  // namespace bsa
