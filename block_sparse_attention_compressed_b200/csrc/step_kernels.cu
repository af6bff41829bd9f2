// The fused decode step: for each (batch, kv-head) pair, in one CTA,
//   scoring    logits x[j][h] = q_h . K~_j / tau of every complete window against the group's query
//              heads, per 64-window chunk its maximum m and e = exp2(x - m) (page "SparDA: Sparse
//              Decoupled Attention for Efficient Long-Context LLM Inference", Indexer Training,
//              Eq. 6; raw scores f . K~_j for the Forecast indexer, SparDA Architecture, Eq. 4);
//   reduction  S[j] = sum_h softmax_h[j], max-pooled onto the blocks ("Fine-grained supervision");
//   selection  top-k blocks (ties to the lower index) united with the init and local blocks
//              (Theoretical Foundation, Eq. 1);
//   attention  exact softmax attention of the group's heads over the selected blocks' tokens
//              (SparDA Architecture, Eq. 5), written straight to O and LSE.
//
// Layout of the work on a B200 SM: one CTA per SM walks pairs c, c + grid, ... Two producer warps
// stream 16 KB stages through an 8-slot shared-memory ring with TMA tensor copies (128-byte
// swizzle, L2 evict-first): first the pair's compressed-key chunks (64 rows), then, for every
// 64-token unit of its selected blocks, a K stage and a V stage. Eight consumer warps run the
// contractions on the tensor cores (mma.m16n8k16). The window terms e of the whole pair (131 KB at 128K tokens, G = 4) stay in
// tensor memory (TMEM, tcgen05.st / tcgen05.ld): the selection then needs no global-memory round
// trip at all, and the init and local blocks, which every selection contains, stream into the ring
// while the top-k runs. One CTA attends all of a pair's blocks, so there are no split partials and
// no combine pass.
//
// Stage bookkeeping: a global stage counter k runs over the CTA's lifetime on every warp; stage k
// uses slot k % 8 and is issued by producer k % 2. Chunk c of a pair (stage k0 + c) is scored by
// warp (c / 2) % 4 + 4 (c % 2): the two warps of TMEM lane quarter (c / 2) % 4 write the tile of
// chunks 2p, 2p + 1 there, one block per lane; attention unit i (stages kd + 2i for K and kd + 2i + 1 for V) is consumed by the four
// warps of group i % 2, 16 tokens each. Slots therefore have one consumer per phase, and a CTA-wide
// barrier separates the phases, so no warp waits on a slot two phases ahead of its last use.
#include "bsa_internal.cuh"
#include "tiles.cuh"
#include "topk.cuh"

namespace bsa {
namespace {

constexpr int kStepConsumers = 8;
constexpr int kStepScorers = 4;  // TMEM lane quarters: tile p of a pair goes to quarter p % 4
constexpr int kStepProducers = 2;
constexpr int kStepThreads = (kStepConsumers + kStepProducers) * 32;
constexpr int kStepSlots = 8;
constexpr uint32_t kSlotBytes = 16384;
constexpr int kUnitTokens = 64;               // tokens per attention unit (one K and one V stage)
constexpr uint32_t kBox = 64 * 128;             // one 64-row, 64-column box (compressed keys, K or V)
constexpr uint32_t kEmptyCount = 4;             // arrivals that free a slot: an attention unit's warps
constexpr int kConsumerBar = 1;               // named barrier of the consumer warps
constexpr int kHandBar = 2;                   // consumers + producers: the selection is handed over
constexpr int kPairBar0 = 3;                  // 3..6: the two scoring warps of a TMEM lane quarter
constexpr int kTopkBar = 7;                   // lookahead: the four warps that select the next layer's blocks
constexpr uint32_t kStepWaitPolls = 1u << 26;
constexpr int kPrefetchChunks = 16;           // compressed-key chunks prefetched into L2 at start-up
static_assert(kStepSlots % (2 * kStepScorers) == 0, "a scoring slot serves one consumer warp");
static_assert(kStepSlots % 4 == 0, "an attention slot serves one group of four warps");
static_assert(kStepSlots % kStepProducers == 0, "a slot is refilled by one producer");

struct StepStage {
    int tok0;    // first token of an attention unit
    int nvalid;  // its tokens below the sequence length
};

// Per-pair geometry, computed identically by every warp.
struct PairGeo {
    int64_t T;
    int nc, nb, nch, init_end, chi;
    bool ok;
};
__device__ __forceinline__ PairGeo pair_geo(const StepArgs& a, int pair) {
    PairGeo g;
    const int64_t T = a.seq_lens[pair / a.Hkv];
    g.ok = T >= 0 && T <= a.T_cap;
    g.T = g.ok ? T : 0;
    g.nc = (int)(g.T < a.l ? 0 : (g.T - a.l) / a.s + 1);
    g.nb = (int)((g.T + a.BS - 1) / a.BS);
    g.nch = (g.nc + 63) / 64;
    g.init_end = min(a.n_init, g.nb);
    g.chi = max(max(g.nb - a.n_local, 0), g.init_end);
    return g;
}
// Attention units of block b: kUnitTokens tokens each, the last one cut at T.
__device__ __forceinline__ int block_units(int64_t T, int b, int BS) {
    const int64_t rem = T - (int64_t)b * BS;
    const int64_t n = rem < BS ? rem : BS;
    return (int)((n + kUnitTokens - 1) / kUnitTokens);
}

// Lookahead: the attention units of the blocks given for this layer (entries outside [0, nb), such
// as the -1 padding, are skipped).
__device__ __forceinline__ int given_units(const StepArgs& a, const PairGeo& pg, int pair) {
    const int nin = min(max(a.in_nsel[pair], 0), a.sel_cap);
    int nu = 0;
    for (int i = 0; i < nin; ++i) {
        const int blk = a.in_idx[(size_t)pair * a.sel_cap + i];
        if (blk >= 0 && blk < pg.nb) nu += block_units(pg.T, blk, a.BS);
    }
    return nu;
}

__device__ __forceinline__ bool aborted(const volatile int* s_abort) { return *s_abort != 0; }

// SGP: scoring heads padded to a power of two (1 for the Forecast indexer's one vector); RAW: the
// stored window terms are the raw scores (no softmax, weight 1). LA (lookahead, with RAW): the
// Forecast vectors score the NEXT layer's compressed keys (maps.ck) and choose that layer's blocks
// (into block_idx / n_sel), while this layer attends the blocks chosen for it beforehand (in_idx /
// in_nsel, maps.k / maps.v): those stream right behind the chunks, and once the block maxima are
// taken four warps run the top-k while the other four attend.
template <int D, int SGP, bool RAW, bool LA>
__global__ void __launch_bounds__(kStepThreads, 1)
    step_kernel(const StepArgs a, const __grid_constant__ StepMaps maps) {
    static_assert(!LA || (RAW && SGP == 1), "lookahead selection scores one Forecast vector");
    extern __shared__ uint8_t dsm_raw[];
    __shared__ __align__(8) uint64_t full[kStepSlots], empty[kStepSlots];
    __shared__ StepStage meta[kStepSlots];
    __shared__ TopkSmem tk;
    __shared__ uint32_t s_tmem;
    __shared__ int s_nsel, s_ndec;
    __shared__ volatile int s_abort;
    constexpr int NB = D / 64;
    constexpr int KS = D / 16;
    constexpr int MT = D / 16;

    // dynamic shared memory: ring | keys (aliased by the end-of-pair merge) | chunk statistics |
    // chunk weights | last window's terms per chunk | transposition staging | selection
    // (offsetting the __shared__ array, not rounding an integer, keeps every pointer below in the
    // shared window: the compiler then emits shared-memory loads and stores, not generic ones)
    uint8_t* ring = dsm_raw + ((1024u - (smem_u32(dsm_raw) & 1023u)) & 1023u);
    uint8_t* p = ring + kStepSlots * kSlotBytes;
    uint32_t* keys = reinterpret_cast<uint32_t*>(p);
    float* merge = reinterpret_cast<float*>(p);
    const size_t keys_bytes = (size_t)a.key_words * 4;
    const size_t merge_bytes = (size_t)(2 * kStepConsumers * kMaxG + kStepConsumers * a.G * D) * 4;
    const size_t region = keys_bytes > merge_bytes ? keys_bytes : merge_bytes;
    p += (region + 15) & ~size_t(15);
    float2* stats = reinterpret_cast<float2*>(p);
    p += (size_t)a.nch_cap * SGP * sizeof(float2);
    float* wt = reinterpret_cast<float*>(p);
    p += (size_t)a.nch_cap * SGP * sizeof(float);
    float* lastE = reinterpret_cast<float*>(p);
    p += (size_t)a.nch_cap * SGP * sizeof(float);
    float* staging = reinterpret_cast<float*>(p);
    p += (size_t)kStepScorers * 2 * 128 * SGP * sizeof(float);
    int32_t* sel = reinterpret_cast<int32_t*>(p);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s2 = 0; s2 < kStepSlots; ++s2) {
            mbar_init(&full[s2], 1);
            mbar_init(&empty[s2], kEmptyCount);
        }
        mbar_fence_init();
        s_abort = 0;
    }
    if (warp == 0) tmem_alloc(&s_tmem, a.tmem_cols);
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t tbase = s_tmem;
    pdl_trigger();
    if (warp >= kStepConsumers && (int)blockIdx.x < a.pairs) {
        // while the previous kernel finishes, the first compressed-key chunks of this CTA's first
        // pair stream into L2 (a prefetch reads nothing into the CTA, so it needs no dependency;
        // the chunk count comes from the capacity, since the sequence lengths may not be final)
        const int nbox = min(kPrefetchChunks, (int)((a.nc_cap + 63) / 64)) * NB;
        for (int e = (warp - kStepConsumers) * 32 + lane; e < nbox; e += kStepProducers * 32)
            tma_prefetch_2d(&maps.ck, 64 * (e % NB), (int)((int64_t)blockIdx.x * a.nc_cap + 64 * (e / NB)));
    }
    pdl_wait();

    if (warp >= kStepConsumers) {
        // ------------------------------------------------------------------------ producers
        const int pw = warp - kStepConsumers;
        const uint64_t pol = l2_evict_first_policy();
        int64_t last_k[kStepSlots];  // last stage issued into each slot, + 1 (0: none)
#pragma unroll
        for (int s2 = 0; s2 < kStepSlots; ++s2) last_k[s2] = 0;
        // waits until slot kk % S may be refilled; on a wait that runs out the CTA stops streaming
        auto claim = [&](int64_t kk) -> int {
            const int slot = (int)(kk % kStepSlots);
            if (kk >= kStepSlots && !aborted(&s_abort) &&
                !mbar_wait(&empty[slot], (uint32_t)((kk / kStepSlots) - 1) & 1u, kStepWaitPolls)) {
                atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                s_abort = 1;
            }
            return slot;
        };
        int64_t k = 0;
        for (int pair = blockIdx.x; pair < a.pairs; pair += gridDim.x) {
            const PairGeo pg = pair_geo(a, pair);
            const int64_t kd = k + pg.nch;  // first attention stage of the pair
            // the attention units of block blk, numbered from i: unit i is stage kd + 2i (its K
            // rows) and kd + 2i + 1 (its V rows); stages numbered in [j_lo, j_hi) are issued
            auto issue_block = [&](int blk, int& i, int j_lo, int j_hi) {
                const int nu = block_units(pg.T, blk, a.BS);
                for (int u = 0; u < nu; ++u, ++i) {
                    const int64_t tok0 = (int64_t)blk * a.BS + (int64_t)u * kUnitTokens;
                    const int y = (int)((int64_t)pair * a.T_cap + tok0);
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const int j = 2 * i + t;
                        const int64_t kk = kd + j;
                        if (j < j_lo || j >= j_hi || (int)(kk % kStepProducers) != pw) continue;
                        const int slot = claim(kk);
                        if (aborted(&s_abort)) continue;
                        meta[slot].tok0 = (int)tok0;
                        meta[slot].nvalid = (int)min((int64_t)kUnitTokens, pg.T - tok0);
                        uint8_t* dst = ring + (size_t)slot * kSlotBytes;
                        mbar_arrive_expect_tx(&full[slot], NB * kBox);
#pragma unroll
                        for (int bi = 0; bi < NB; ++bi)
                            tma_load_2d_hint(dst + bi * kBox, t == 0 ? &maps.k : &maps.v, 64 * bi, y, &full[slot], pol);
                        last_k[slot] = kk + 1;
                    }
                }
            };
            if (lane == 0) {
                // the pair's compressed-key chunks
                for (int c = 0; c < pg.nch; ++c) {
                    const int64_t kk = k + c;
                    if ((int)(kk % kStepProducers) != pw) continue;
                    const int slot = claim(kk);
                    if (aborted(&s_abort)) continue;
                    uint8_t* dst = ring + (size_t)slot * kSlotBytes;
                    mbar_arrive_expect_tx(&full[slot], NB * kBox);
                    const int y = (int)((int64_t)pair * a.nc_cap + 64 * c);
#pragma unroll
                    for (int bi = 0; bi < NB; ++bi)
                        tma_load_2d_hint(dst + bi * kBox, &maps.ck, 64 * bi, y, &full[slot], pol);
                    last_k[slot] = kk + 1;
                }
                int j = 0;
                if constexpr (LA) {
                    // this layer's blocks are known: all their stages follow the chunks
                    const int nin = min(max(a.in_nsel[pair], 0), a.sel_cap);
                    for (int i = 0; i < nin; ++i) {
                        const int blk = a.in_idx[(size_t)pair * a.sel_cap + i];
                        if (blk >= 0 && blk < pg.nb) issue_block(blk, j, 0, INT32_MAX);
                    }
                } else {
                    // the init and local blocks are in every selection: their first stages load
                    // while the consumers select (as many as the ring holds without waiting for them)
                    for (int b = 0; b < pg.init_end; ++b) issue_block(b, j, 0, kStepSlots);
                    for (int b = pg.chi; b < pg.nb; ++b) issue_block(b, j, 0, kStepSlots);
                }
            }
            __syncwarp();
            if constexpr (!LA) {
                asm volatile("bar.sync %0, %1;" ::"r"(kHandBar), "r"(kStepThreads) : "memory");
                if (lane == 0) {
                    // the rest: init / local stages beyond the ring, then the top-k blocks
                    int j = 0;
                    for (int b = 0; b < pg.init_end; ++b) issue_block(b, j, kStepSlots, INT32_MAX);
                    for (int b = pg.chi; b < pg.nb; ++b) issue_block(b, j, kStepSlots, INT32_MAX);
                    const int top_end = s_nsel - (pg.nb - pg.chi);
                    for (int i = pg.init_end; i < top_end; ++i) issue_block(sel[i], j, 0, INT32_MAX);
                }
                __syncwarp();
                k = kd + s_ndec;
            } else {
                k = kd + 2 * given_units(a, pg, pair);
            }
        }
        // copies still in flight land before the CTA exits (all of them, on the normal path, have
        // been consumed already)
        if (lane == 0) {
            for (int s2 = 0; s2 < kStepSlots; ++s2) {
                if (last_k[s2] > 0 && !mbar_wait(&full[s2], (uint32_t)((last_k[s2] - 1) / kStepSlots) & 1u, kStepWaitPolls))
                    atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------------ consumers
        const int w = warp;
        const Grp grp{(int)threadIdx.x, kStepConsumers * 32, kConsumerBar};
        const int g = lane >> 2, tq = lane & 3;
        const int GS = RAW ? 1 : a.G;  // scoring heads
        const uint32_t tq_addr = tbase + ((32u * (uint32_t)(w & 3)) << 16);  // this warp's TMEM lanes
        SelectArgs sa;
        memset(&sa, 0, sizeof sa);
        sa.n_init = a.n_init;
        sa.n_local = a.n_local;
        sa.top_k = a.top_k;
        sa.sel_cap = a.sel_cap;
        const int L_w = a.l / a.s;  // windows of one block: BS = 4s, l = s or 2s
        // waits for stage kk's data; after a wait that runs out the CTA finishes without waiting
        auto await_stage = [&](int64_t kk) -> int {
            const int slot = (int)(kk % kStepSlots);
            if (!aborted(&s_abort) && !mbar_wait(&full[slot], (uint32_t)(kk / kStepSlots) & 1u, kStepWaitPolls)) {
                if (lane == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                s_abort = 1;
            }
            return slot;
        };
        int64_t k = 0;
        for (int pair = blockIdx.x; pair < a.pairs; pair += gridDim.x) {
            const PairGeo pg = pair_geo(a, pair);
            const int b = pair / a.Hkv, kvh = pair - b * a.Hkv;
            if (!pg.ok && threadIdx.x == 0 && kvh == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_SEQ_LEN);
            uint32_t qa[KS][2];  // attention B operand: the group's query heads
            load_q_frag<D>(qa, reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint16_t*>(a.q) +
                                                                 ((size_t)b * a.Hq + (size_t)kvh * a.G + g) * D),
                           g < a.G, tq);
            uint32_t qf_raw[RAW ? KS : 1][2];  // the pair's Forecast vector (Forecast indexer)
            if constexpr (RAW)
                load_q_frag<D>(qf_raw, reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint16_t*>(a.f) +
                                                                         (size_t)pair * D),
                               g == 0, tq);
            // scoring B operand: the group's query heads, or the Forecast vector
            const uint32_t(&qs)[KS][2] = *reinterpret_cast<const uint32_t(*)[KS][2]>(RAW ? &qf_raw[0][0] : &qa[0][0]);

            topk_prepare(tk, grp);  // the top-k's bins, cleared while the first chunks load
            if (LA && grp.tid == 0) s_ndec = 2 * given_units(a, pg, pair);  // read after the scoring's barrier
            // ---- scoring: tiles of two 64-window chunks. Chunk 2p of tile p is scored by warp p % 4 and
            // chunk 2p + 1 by warp p % 4 + 4, the two warps of TMEM lane quarter p % 4; they meet at a
            // named barrier and the first stores the tile, one block per lane: lane i holds block
            // 32p + i, its four windows 128p + 4i .. + 3 with every head (4 * SGP columns).
            const bool h0 = 2 * tq < GS, h1 = 2 * tq + 1 < GS;
            const int qd = w & 3, half = w >> 2;
            for (int p = qd; 2 * p < pg.nch; p += kStepScorers) {
                float* stg = staging + (qd * 2 + ((p / kStepScorers) & 1)) * 128 * SGP;  // double-buffered
                const int c = 2 * p + half;
                if (c < pg.nch) {
                    const int slot = await_stage(k + c);
                    float cc[4][4];
                    score_chunk<D>(ring + (size_t)slot * kSlotBytes, qs, cc, lane);
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cnt(&empty[slot], kEmptyCount);  // one warp stands for four
                    const int nrows = min(64, pg.nc - 64 * c);
                    float x[4][4];
#pragma unroll
                    for (int r = 0; r < 4; ++r)
#pragma unroll
                        for (int e = 0; e < 4; ++e) x[r][e] = __fmul_rn(cc[r][e], a.score_log2);  // rounded here in every kernel
                    if constexpr (!RAW) {
                        // the chunk's maximum per head, then e = exp2(x - max) and its sum
                        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            if (16 * r + g < nrows) {
                                m0 = fmaxf(m0, x[r][0]);
                                m1 = fmaxf(m1, x[r][1]);
                            }
                            if (16 * r + g + 8 < nrows) {
                                m0 = fmaxf(m0, x[r][2]);
                                m1 = fmaxf(m1, x[r][3]);
                            }
                        }
#pragma unroll
                        for (int off = 4; off < 32; off <<= 1) {
                            m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, off));
                            m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, off));
                        }
                        float s0 = 0.f, s1 = 0.f;
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const int lra = 16 * r + g, lrb = lra + 8;
                            if (lra < nrows) {
                                x[r][0] = exp2f(x[r][0] - m0);
                                x[r][1] = exp2f(x[r][1] - m1);
                                s0 += x[r][0];
                                s1 += x[r][1];
                            } else {
                                x[r][0] = x[r][1] = 0.f;
                            }
                            if (lrb < nrows) {
                                x[r][2] = exp2f(x[r][2] - m0);
                                x[r][3] = exp2f(x[r][3] - m1);
                                s0 += x[r][2];
                                s1 += x[r][3];
                            } else {
                                x[r][2] = x[r][3] = 0.f;
                            }
                        }
#pragma unroll
                        for (int off = 4; off < 32; off <<= 1) {
                            s0 += __shfl_xor_sync(0xffffffffu, s0, off);
                            s1 += __shfl_xor_sync(0xffffffffu, s1, off);
                        }
                        if (g == 0) {
                            if (h0) stats[c * SGP + 2 * tq] = make_float2(m0, s0);
                            if (h1) stats[c * SGP + 2 * tq + 1] = make_float2(m1, s1);
                        }
                    }
                    // the chunk's rows into the tile's staging rows 64 * half ..
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int lra = 64 * half + 16 * r + g, lrb = lra + 8;
                        if (2 * tq < SGP) {
                            stg[lra * SGP + 2 * tq] = x[r][0];
                            stg[lrb * SGP + 2 * tq] = x[r][2];
                        }
                        if (2 * tq + 1 < SGP) {
                            stg[lra * SGP + 2 * tq + 1] = x[r][1];
                            stg[lrb * SGP + 2 * tq + 1] = x[r][3];
                        }
                    }
                    __syncwarp();
                    if (lane < SGP) lastE[c * SGP + lane] = stg[(64 * half + 63) * SGP + lane];
                }
                asm volatile("bar.sync %0, %1;" ::"r"(kPairBar0 + qd), "r"(64) : "memory");
                if (half == 0) {
                    // lane i: rows 4i .. 4i + 3 of the tile (block 32p + i), all heads
                    float v[4 * SGP];
#pragma unroll
                    for (int e = 0; e < 4 * SGP; ++e) v[e] = stg[4 * lane * SGP + e];
                    tmem_st<4 * SGP>(tq_addr + (uint32_t)((p / kStepScorers) * 4 * SGP), v);
                }
            }
            k += pg.nch;
            tmem_wait_st();
            tmem_fence_before_sync();
            grp.sync();
            tmem_fence_after_sync();

            // ---- selection: weights, block maxima, top-k
            if constexpr (!RAW) {
                if (w < a.G) {
                    // head w's softmax normaliser (M, Z) from the chunk statistics, then one weight
                    // per chunk, w[c] = exp2(m_c - M) / Z
                    float m = -INFINITY, sum = 0.f;
                    for (int c = lane; c < pg.nch; c += 32) {
                        const float2 sv = stats[c * SGP + w];
                        online_merge(m, sum, sv.x, sv.y);
                    }
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) {
                        const float mo = __shfl_xor_sync(0xffffffffu, m, off);
                        const float so = __shfl_xor_sync(0xffffffffu, sum, off);
                        online_merge(m, sum, mo, so);
                    }
                    // the lanes' merges round in different orders: all take lane 0's (M, Z), as
                    // the selection kernels do
                    m = __shfl_sync(0xffffffffu, m, 0);
                    sum = __shfl_sync(0xffffffffu, sum, 0);
                    const float iz = sum > 0.f ? 1.f / sum : 0.f;
                    for (int c = lane; c < pg.nch; c += 32) wt[c * SGP + w] = exp2f(stats[c * SGP + w].x - m) * iz;
                }
            } else {
                for (int c = grp.tid; c < pg.nch; c += grp.nt) wt[c] = 1.f;
            }
            grp.sync();
            // block maxima, one block per lane: tile p of quarter p % 4 (warps w and w + 4 split the
            // quarter's tiles, TB tiles per TMEM load). Block b = 32p + i covers windows 4b .. 4b + 3,
            // and 4b - 1 when l = 2s: the previous lane's last window (lane 0: the previous tile's,
            // from the chunk's last terms).
            uint32_t kand = 0xffffffffu, kor = 0u;
            constexpr int TB = 1;  // tiles per TMEM load (two loads in flight)
            constexpr int LW = TB * 4 * SGP;
            const int nbt = (pg.nb + 31) / 32;  // tiles holding blocks
            const int qq = w & 3;
            const int nq = nbt > qq ? (nbt - qq + 3) / 4 : 0;
            const int i_lo = w < 4 ? 0 : (nq + 1) / 2, i_hi = w < 4 ? (nq + 1) / 2 : nq;
            // one tile group's maxima from its TMEM terms
            auto tile_maxima = [&](const float (&v)[LW], int i0) {
#pragma unroll
                for (int u = 0; u < TB; ++u) {
                    if (i0 + u >= i_hi) break;
                    const int p = qq + 4 * (i0 + u);
                    const int j0 = 128 * p + 4 * lane;  // the lane's first window
                    float mx = -INFINITY, last = -INFINITY;
                    if (j0 < pg.nc) {
                        float wc[SGP];  // the chunk's weights, loaded once
#pragma unroll
                        for (int h = 0; h < SGP; ++h) wc[h] = wt[(j0 >> 6) * SGP + h];
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
                            const float sv = j0 + jj < pg.nc ? group_sum<SGP>(v + u * 4 * SGP + jj * SGP, wc, GS) : -INFINITY;
                            mx = fmaxf(mx, sv);
                            if (jj == 3) last = sv;
                        }
                    }
                    if (L_w == 2) {
                        float prev = __shfl_up_sync(0xffffffffu, last, 1);
                        if (lane == 0)
                            prev = p > 0 && 128 * p - 1 < pg.nc
                                       ? group_sum<SGP>(lastE + (2 * p - 1) * SGP, wt + (2 * p - 1) * SGP, GS)
                                       : -INFINITY;
                        mx = fmaxf(mx, prev);
                    }
                    const int blk = 32 * p + lane;
                    if (blk < pg.nb) {
                        const uint32_t key = order_key(mx);
                        keys[blk] = key;
                        if (blk >= pg.init_end && blk < pg.chi) {
                            kand &= key;
                            kor |= key;
                        }
                        if (a.block_scores) a.block_scores[(size_t)pair * a.nb_cap + blk] = mx;
                    }
                }
            };
            // TMEM loads double-buffered: the next group's load is in flight while this one's
            // maxima are taken (only tiles that hold scored windows are loaded)
            auto scored = [&](int i0) { return i0 < i_hi && 2 * (qq + 4 * i0) < pg.nch; };
            float va[LW], vb[LW];
            if (scored(i_lo)) tmem_ld<LW>(tq_addr + (uint32_t)(i_lo * 4 * SGP), va);
            for (int i0 = i_lo; i0 < i_hi; i0 += 2 * TB) {
                tmem_wait_ld();
                if (scored(i0 + TB)) tmem_ld<LW>(tq_addr + (uint32_t)((i0 + TB) * 4 * SGP), vb);
                tile_maxima(va, i0);
                if (i0 + TB >= i_hi) break;
                tmem_wait_ld();
                if (scored(i0 + 2 * TB)) tmem_ld<LW>(tq_addr + (uint32_t)((i0 + 2 * TB) * 4 * SGP), va);
                tile_maxima(vb, i0 + TB);
            }
            tmem_wait_ld();
            if (a.block_scores)
                for (int64_t blk = pg.nb + grp.tid; blk < a.nb_cap; blk += grp.nt)
                    a.block_scores[(size_t)pair * a.nb_cap + blk] = -INFINITY;
            publish_andor(tk, kand, kor, grp);
            grp.sync();

            // attention: units i0, i0 + di, ... of this pair's blocks (stages kd + 2i for the K rows
            // and kd + 2i + 1 for the V rows), 16 tokens per warp: the K stage gives the scores and
            // probabilities, the V stage the numerators
            AttnState<D> as;
            as.reset();
            auto attend_units = [&](int64_t kd, int n_dec, int i0, int di) {
                const int r0 = 16 * (w & 3);
                for (int i = i0; 2 * i < n_dec; i += di) {
                    const int ks_ = await_stage(kd + 2 * i);
                    const StepStage md = meta[ks_];
                    PFrag pf;
                    if (r0 < md.nvalid)
                        pf = attn_scores16<D>(ring + (size_t)ks_ * kSlotBytes, kBox, r0, md.nvalid, qa, a.scale_log2, as, lane);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[ks_]);
                    const int vs_ = await_stage(kd + 2 * i + 1);
                    if (r0 < md.nvalid) attn_accum16<D>(ring + (size_t)vs_ * kSlotBytes, kBox, r0, md.nvalid, pf, as, lane);
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&empty[vs_]);
                }
            };
            if constexpr (LA) {
                // warps 0-3 choose the next layer's blocks while warps 4-7 attend this layer's
                // (all its units, in order: a slot is always refilled for the same four warps)
                const int n_dec = s_ndec;
                if (w < 4) {
                    const Grp ga{(int)threadIdx.x, 4 * 32, kTopkBar};
                    topk_union(sa, pg.nb, keys, tk, false, ga, sel, &s_nsel);
                    ga.sync();
                    for (int i = ga.tid; i < a.sel_cap; i += ga.nt) a.block_idx[(size_t)pair * a.sel_cap + i] = sel[i];
                    if (ga.tid == 0) a.n_sel[pair] = s_nsel;
                } else {
                    attend_units(k, n_dec, 0, 1);
                }
                k += n_dec;
            } else {
                topk_union(sa, pg.nb, keys, tk, true, grp, sel, &s_nsel);
                grp.sync();
                for (int i = grp.tid; i < a.sel_cap; i += grp.nt) a.block_idx[(size_t)pair * a.sel_cap + i] = sel[i];
                if (grp.tid == 0) {
                    const int nsel = s_nsel;
                    a.n_sel[pair] = nsel;
                    // attention units: one per selected block at BS = 64, else counted block by block
                    int nu = nsel;
                    if (a.BS != kUnitTokens) {
                        nu = 0;
                        for (int blk = 0; blk < pg.init_end; ++blk) nu += block_units(pg.T, blk, a.BS);
                        for (int blk = pg.chi; blk < pg.nb; ++blk) nu += block_units(pg.T, blk, a.BS);
                        for (int i = pg.init_end; i < nsel - (pg.nb - pg.chi); ++i) nu += block_units(pg.T, sel[i], a.BS);
                    }
                    s_ndec = 2 * nu;
                }
                asm volatile("bar.sync %0, %1;" ::"r"(kHandBar), "r"(kStepThreads) : "memory");
                // units i of group i % 2
                const int n_dec = s_ndec;
                attend_units(k, n_dec, w >> 2, 2);
                k += n_dec;
            }

            // ---- the eight warps' states merge into O and LSE (the merge area lies over the keys,
            // which the lookahead's top-k may still be using)
            if constexpr (LA) grp.sync();
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                as.lsum[0] += __shfl_xor_sync(0xffffffffu, as.lsum[0], off);
                as.lsum[1] += __shfl_xor_sync(0xffffffffu, as.lsum[1], off);
            }
            float* mM = merge;                                // [warp][kMaxG]
            float* mL = merge + kStepConsumers * kMaxG;       // [warp][kMaxG]
            float* mA = merge + 2 * kStepConsumers * kMaxG;  // [warp][G][D]
            const int hh0 = 2 * tq, hh1 = 2 * tq + 1;
            if (g == 0) {
                if (hh0 < a.G) {
                    mM[w * kMaxG + hh0] = as.m[0];
                    mL[w * kMaxG + hh0] = as.lsum[0];
                }
                if (hh1 < a.G) {
                    mM[w * kMaxG + hh1] = as.m[1];
                    mL[w * kMaxG + hh1] = as.lsum[1];
                }
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int d0 = 16 * mt + g;
                if (hh0 < a.G) {
                    mA[(w * a.G + hh0) * D + d0] = as.acc[mt][0];
                    mA[(w * a.G + hh0) * D + d0 + 8] = as.acc[mt][2];
                }
                if (hh1 < a.G) {
                    mA[(w * a.G + hh1) * D + d0] = as.acc[mt][1];
                    mA[(w * a.G + hh1) * D + d0 + 8] = as.acc[mt][3];
                }
            }
            grp.sync();
            __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out) + ((size_t)b * a.Hq + (size_t)kvh * a.G) * D;
            float* lse = a.lse ? a.lse + (size_t)b * a.Hq + (size_t)kvh * a.G : nullptr;
            for (int e = grp.tid; e < a.G * D; e += grp.nt) {
                const int h = e / D, dd = e - h * D;
                float M = -INFINITY;
#pragma unroll
                for (int ww = 0; ww < kStepConsumers; ++ww) M = fmaxf(M, mM[ww * kMaxG + h]);
                float num = 0.f, den = 0.f;
                if (M != -INFINITY) {
#pragma unroll
                    for (int ww = 0; ww < kStepConsumers; ++ww) {
                        const float f = exp2f(mM[ww * kMaxG + h] - M);
                        num = fmaf(f, mA[(ww * a.G + h) * D + dd], num);
                        den = fmaf(f, mL[ww * kMaxG + h], den);
                    }
                }
                out[h * D + dd] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
                if (dd == 0 && lse) lse[h] = den > 0.f ? (M + log2f(den)) * 0.69314718055994531f : -INFINITY;
            }
            grp.sync();  // the merge area (over the keys) is free for the next pair
        }
    }
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 0) tmem_dealloc(tbase, a.tmem_cols);
}

template <int D, int SGP, bool RAW, bool LA>
cudaError_t launch_step_k(const Plan& p, const StepArgs& a, const StepMaps* maps, cudaStream_t st) {
    if (a.pairs <= 0) return cudaSuccess;
    cudaError_t e = ensure_smem<step_kernel<D, SGP, RAW, LA>>(p.step_smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(step_kernel<D, SGP, RAW, LA>, dim3((unsigned)p.step_ctas), dim3(kStepThreads), p.step_smem,
                      st, a, *maps);
}

template <int D>
cudaError_t launch_step_d(const Plan& p, const StepArgs& a, const StepMaps* maps, cudaStream_t st) {
    if (a.in_idx) return launch_step_k<D, 1, true, true>(p, a, maps, st);
    if (a.f) return launch_step_k<D, 1, true, false>(p, a, maps, st);
    switch (p.step_sgp) {
        case 1: return launch_step_k<D, 1, false, false>(p, a, maps, st);
        case 2: return launch_step_k<D, 2, false, false>(p, a, maps, st);
        case 4: return launch_step_k<D, 4, false, false>(p, a, maps, st);
        default: return launch_step_k<D, 8, false, false>(p, a, maps, st);
    }
}

}  // namespace

size_t step_smem_bytes(int D, int sgp, int G, int nch_cap, int key_words, int sel_cap) {
    const size_t keys_bytes = (size_t)key_words * 4;
    const size_t merge_bytes = (size_t)(2 * kStepConsumers * kMaxG + kStepConsumers * G * D) * 4;
    const size_t region = keys_bytes > merge_bytes ? keys_bytes : merge_bytes;
    size_t bytes = 1024 + (size_t)kStepSlots * kSlotBytes + ((region + 15) & ~size_t(15));
    bytes += (size_t)nch_cap * sgp * (sizeof(float2) + 2 * sizeof(float));
    bytes += (size_t)kStepScorers * 2 * 128 * sgp * sizeof(float);
    bytes += (size_t)sel_cap * sizeof(int32_t);
    // the static part (ring barriers, stage records, top-k scratch) shares the 227 KB of a CTA
    const size_t limit = 227 * 1024 - sizeof(TopkSmem) - 1024;
    return bytes <= limit ? bytes : 0;
}

cudaError_t launch_step(const Plan& p, const StepArgs& a, const StepMaps* maps, cudaStream_t st) {
    return p.D == 128 ? launch_step_d<128>(p, a, maps, st) : launch_step_d<64>(p, a, maps, st);
}

}  // namespace bsa
