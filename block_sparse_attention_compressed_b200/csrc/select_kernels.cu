// Block selection: group scoring, block reduction and top-k (page "SparDA: Sparse Decoupled
// Attention for Efficient Long-Context LLM Inference": Indexer Training, Eq. 6 for the score of a
// GQA group; "Fine-grained supervision" for the max-pool onto the block grid; Theoretical
// Foundation, Eq. 1 and SparDA Architecture, Eq. 4 for the union with init/local blocks and f_top;
// SparDA Architecture, "Compact Forecast Indexer" for the raw-score mode).
//
// Two kernels chained with programmatic dependent launch:
//
// score (persistent): the 64-row chunks of all pairs' compressed keys are shared evenly by the CTAs,
//   so all finish together. For each chunk it computes the group's logits x[j][h] = q_h . K~_j / tau
//   (log2 units), takes the chunk's maximum m per head and writes e = exp2(x - m) to the workspace
//   with the chunk's per-head (m, sum e). (Raw-score mode, one Forecast vector per group: x itself.)
//   bf16: a producer warp streams the chunks into a ring of shared-memory stages with 2-D TMA
//   tensor copies (128-byte swizzle) completing on mbarriers; four consumer warps take whole
//   chunks in turn and run the contraction on the tensor cores (mma.m16n8k16 with ldmatrix
//   operands: rows are M, the G heads padded to 8 are N, head_dim is K). fp32: FMA dot products,
//   one warp per row.
//
// select: merges the chunk statistics into each head's softmax normaliser (M, Z) and one weight per
//   (chunk, head), w = exp2(m - M) / Z, so that S[j] = sum_h e[j][h] w[c(j)][h] = sum_h softmax_h[j];
//   max-pools S onto the blocks and runs the top-k: radix digits over order-preserving uint32 keys
//   (a wide first digit, then 8 bits), an exact ranking of the k-th key's bucket, ties toward the
//   lower block index, then the ascending union with the init and local blocks.
//   select_single_kernel (one CTA per pair) streams the pair's e rows into a shared-memory ring
//   with 1-D bulk copies and takes the block maxima with warp shuffles; select_kernel (pairs x
//   parts CTAs, for few pairs) splits the windows, and the last part of a pair to finish
//   (completion counter, no waiting) runs the top-k.
#include "bsa_internal.cuh"
#include "tiles.cuh"
#include "topk.cuh"

namespace bsa {
namespace {

constexpr int kScoreThreads = kScoreWarps * 32;
constexpr int kSelectThreads = 512;


__device__ __forceinline__ int64_t num_windows(int64_t T, int l, int s) {
    return T < l ? 0 : (T - l) / s + 1;
}
// Last window overlapping block b (before clamping to the window count).
__device__ __forceinline__ int64_t last_window(int64_t b, int BS, int s) {
    return (b * BS + BS - 1) / s;
}
// Smallest block whose first overlapping window is >= j.
__device__ __forceinline__ int64_t first_block_from(int64_t j, int BS, int l, int s) {
    return j <= 0 ? 0 : ((int64_t)s * (j - 1) + l + BS - 1) / BS;
}
// First and last window overlapping block b, in 32 bits (token indices stay below 2^31).
__device__ __forceinline__ uint32_t first_window32(uint32_t b, uint32_t BS, uint32_t l, uint32_t s) {
    const uint32_t tok0 = b * BS;
    return tok0 >= l ? (tok0 - l) / s + 1 : 0;
}
__device__ __forceinline__ uint32_t last_window32(uint32_t b, uint32_t BS, uint32_t s) {
    return (b * BS + BS - 1) / s;
}

__device__ __forceinline__ void report_lengths(const ScoreArgs& a) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        for (int b = 0; b < a.B; ++b) {
            const int T = a.seq_lens[b];
            if (T < 0 || T > a.T_cap) atomicOr(a.err, (uint32_t)BSA_DEVERR_SEQ_LEN);
        }
    }
}

// ================================================================================ score kernels
constexpr int kScoreConsumers = 4;
constexpr int kScoreTmaThreads = (kScoreConsumers + 1) * 32;
constexpr int kScoreMaxStages = 8;
static_assert(kScoreMaxStages % kScoreConsumers == 0, "slots are owned by one consumer warp each");
constexpr uint32_t kScoreWaitPolls = 1u << 26;

struct ScoreStage {
    int pair;
    int row0;   // first window of the chunk
    int nrows;  // windows of the chunk below the pair's window count; -1 ends the stream
};

// Consumer warp w takes stages w, w + 4, ...: a whole 64-row chunk per warp, its four 16-row groups
// as independent mma chains, so four chunks are in compute at once while the producer keeps the
// rest of the ring loading. The stage count must be a multiple of the consumer count: then slot
// st only ever serves warp st % 4, which waits on it one phase at a time. (A slot shared by two
// warps lets one of them wait two phases ahead, where the parity test cannot tell the phases
// apart and passes on a slot whose copy is still in flight.)
template <int D>
__global__ void __launch_bounds__(kScoreTmaThreads, 3)
    score_tma_kernel(const ScoreArgs a, const __grid_constant__ CUtensorMap ck_map, const int nstages) {
    extern __shared__ uint8_t dsm_raw[];
    __shared__ __align__(8) uint64_t full[kScoreMaxStages], empty[kScoreMaxStages];
    __shared__ ScoreStage meta[kScoreMaxStages];
    constexpr int NB = D / 64;  // 64-column boxes per row
    constexpr int KS = D / 16;  // k-steps
    const uint32_t box_bytes = 64u * 128u;
    const uint32_t stage_bytes = NB * box_bytes;
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    const int C = (int)gridDim.x;
    const int64_t c_lo = (int64_t)blockIdx.x * a.total_chunks / C;
    const int64_t c_hi = (int64_t)(blockIdx.x + 1) * a.total_chunks / C;
    if (threadIdx.x == 0) {
        for (int s2 = 0; s2 < nstages; ++s2) {
            mbar_init(&full[s2], 1);
            mbar_init(&empty[s2], 1);
        }
        mbar_fence_init();
    }
    __syncthreads();
    pdl_trigger();
    pdl_wait();
    report_lengths(a);

    if (warp == kScoreConsumers) {
        if (lane == 0) {
            // the compressed keys are read once: keep the window terms (reread by the
            // selection) in L2 rather than them
            const uint64_t ck_policy = l2_evict_first_policy();
            int k = 0, cur_pair = -1;
            int64_t nc = 0;
            bool ok = true;
            auto claim = [&](int kk) -> int {
                const int st = kk % nstages;
                if (kk >= nstages && !mbar_wait(&empty[st], ((kk / nstages) - 1) & 1, kScoreWaitPolls)) {
                    atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                    ok = false;
                }
                return st;
            };
            for (int64_t chunk = c_lo; chunk < c_hi && ok; ++chunk) {
                const int pair = (int)(chunk / a.nchunk);
                const int64_t row0 = (chunk - (int64_t)pair * a.nchunk) * 64;
                if (pair != cur_pair) {
                    cur_pair = pair;
                    const int64_t T = a.seq_lens[pair / a.Hkv];
                    nc = (T >= 0 && T <= a.T_cap) ? num_windows(T, a.l, a.s) : 0;
                }
                if (row0 >= nc) continue;  // past the sequence: nothing to score
                const int st = claim(k);
                if (!ok) break;
                meta[st].pair = pair;
                meta[st].row0 = (int)row0;
                meta[st].nrows = (int)min((int64_t)64, nc - row0);
                uint8_t* dst = ring + (size_t)st * stage_bytes;
                mbar_arrive_expect_tx(&full[st], stage_bytes);
                const int y = (int)((int64_t)pair * a.nc_cap + row0);
#pragma unroll
                for (int bi = 0; bi < NB; ++bi)
                    tma_load_2d_hint(dst + bi * box_bytes, &ck_map, 64 * bi, y, &full[st], ck_policy);
                ++k;
            }
            // end-of-stream markers, one per consumer warp (each waits on its own stages only)
            for (int w = 0; w < kScoreConsumers && ok; ++w) {
                const int st = claim(k);
                if (!ok) break;
                meta[st].nrows = -1;
                mbar_arrive(&full[st]);
                ++k;
            }
        }
    } else {
        const bool h0 = 2 * tq < a.G, h1 = 2 * tq + 1 < a.G;
        uint32_t qf[KS][2];
        int q_pair = -1;
        for (int k = warp;; k += kScoreConsumers) {
            const int st = k % nstages;
            if (!mbar_wait(&full[st], (k / nstages) & 1, kScoreWaitPolls)) {
                if (lane == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                break;
            }
            const ScoreStage md = meta[st];
            if (md.nrows < 0) break;
            if (md.pair != q_pair) {
                // q as the B operand: lane (g, tq) holds head g, d = 16ks + 2tq (+1, +8, +9)
                q_pair = md.pair;
                const int b = md.pair / a.Hkv, kvh = md.pair - b * a.Hkv;
                load_q_frag<D>(qf, reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint16_t*>(a.q) +
                                                                     ((size_t)b * a.Hq + (size_t)kvh * a.G + g) * D),
                               g < a.G, tq);
            }
            float c[4][4];
            score_chunk<D>(ring + (size_t)st * stage_bytes, qf, c, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);  // the data is in registers: refill the slot
            if (a.raw) {
                // Forecast indexer: the raw scores are the window scores
                float* lgr = a.logits + (size_t)md.pair * a.lg_stride * a.Gp;
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int lra = 16 * r + g, lrb = lra + 8;
                    if (lra < md.nrows) {
                        const int64_t ra = md.row0 + lra;
                        if (h1) *reinterpret_cast<float2*>(lgr + ra * a.Gp + 2 * tq) =
                            make_float2(c[r][0] * a.score_log2, c[r][1] * a.score_log2);
                        else if (h0) lgr[ra * a.Gp + 2 * tq] = c[r][0] * a.score_log2;
                    }
                    if (lrb < md.nrows) {
                        const int64_t rb = md.row0 + lrb;
                        if (h1) *reinterpret_cast<float2*>(lgr + rb * a.Gp + 2 * tq) =
                            make_float2(c[r][2] * a.score_log2, c[r][3] * a.score_log2);
                        else if (h0) lgr[rb * a.Gp + 2 * tq] = c[r][2] * a.score_log2;
                    }
                }
                continue;
            }
            // the chunk's maximum per head first, then e = exp2(x - max) is stored and summed: the
            // selection only rescales each chunk's e by one weight per head
            float x[4][4];
            float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
#pragma unroll
                for (int e = 0; e < 4; ++e) x[r][e] = __fmul_rn(c[r][e], a.score_log2);  // rounded here in every kernel
                if (16 * r + g < md.nrows) {
                    m0 = fmaxf(m0, x[r][0]);
                    m1 = fmaxf(m1, x[r][1]);
                }
                if (16 * r + g + 8 < md.nrows) {
                    m0 = fmaxf(m0, x[r][2]);
                    m1 = fmaxf(m1, x[r][3]);
                }
            }
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {  // over the 8 row groups (lanes with equal tq)
                m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, off));
                m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, off));
            }
            float* lg = a.logits + (size_t)md.pair * a.lg_stride * a.Gp;
            float s0 = 0.f, s1 = 0.f;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int lra = 16 * r + g, lrb = lra + 8;
                const int64_t ra = md.row0 + lra, rb = md.row0 + lrb;
                if (lra < md.nrows) {
                    const float e0 = exp2f(x[r][0] - m0), e1 = exp2f(x[r][1] - m1);
                    if (h1) *reinterpret_cast<float2*>(lg + ra * a.Gp + 2 * tq) = make_float2(e0, e1);
                    else if (h0) lg[ra * a.Gp + 2 * tq] = e0;
                    s0 += e0;
                    s1 += e1;
                }
                if (lrb < md.nrows) {
                    const float e2 = exp2f(x[r][2] - m0), e3 = exp2f(x[r][3] - m1);
                    if (h1) *reinterpret_cast<float2*>(lg + rb * a.Gp + 2 * tq) = make_float2(e2, e3);
                    else if (h0) lg[rb * a.Gp + 2 * tq] = e2;
                    s0 += e2;
                    s1 += e3;
                }
            }
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                s0 += __shfl_xor_sync(0xffffffffu, s0, off);
                s1 += __shfl_xor_sync(0xffffffffu, s1, off);
            }
            if (g == 0) {
                float2* dst = a.stats + ((size_t)md.pair * a.nstat + md.row0 / 64) * a.Gp;
                if (h0) dst[2 * tq] = make_float2(m0, s0);
                if (h1) dst[2 * tq + 1] = make_float2(m1, s1);
            }
        }
    }
}

// fp32: plain FMA dot products (fp32 inputs keep fp32 accuracy); a warp per chunk takes kRowU rows
// at a time, lanes splitting d.
constexpr int kRowU = 8;
template <int D>
__global__ void __launch_bounds__(kScoreThreads, 2) score_f32_kernel(ScoreArgs a) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
    const int64_t W = (int64_t)gridDim.x * kScoreWarps;
    const int64_t w = (int64_t)blockIdx.x * kScoreWarps + (threadIdx.x >> 5);
    const int64_t c_lo = w * a.total_chunks / W, c_hi = (w + 1) * a.total_chunks / W;
    pdl_trigger();
    pdl_wait();
    report_lengths(a);
    // the warp's chunk: x staged in shared memory, written out as e = exp2(x - max) at the end
    __shared__ float s_x[kScoreWarps][64 * kMaxG];
    __shared__ float s_m[kScoreWarps][kMaxG];
    float* sx = s_x[threadIdx.x >> 5];
    float* sm = s_m[threadIdx.x >> 5];
    int cur_pair = -1;
    int64_t nc = 0;
    float qv[kMaxG][E];
    for (int64_t chunk = c_lo; chunk < c_hi; ++chunk) {
        const int pair = (int)(chunk / a.nchunk);
        const int64_t ci = chunk - (int64_t)pair * a.nchunk;
        if (pair != cur_pair) {
            cur_pair = pair;
            const int b = pair / a.Hkv, kvh = pair - b * a.Hkv;
            const int64_t T = a.seq_lens[b];
            nc = (T >= 0 && T <= a.T_cap) ? num_windows(T, a.l, a.s) : 0;
            const float* qb = reinterpret_cast<const float*>(a.q) + ((size_t)b * a.Hq + (size_t)kvh * a.G) * D;
#pragma unroll
            for (int h = 0; h < kMaxG; ++h)
#pragma unroll
                for (int e = 0; e < E; ++e) qv[h][e] = h < a.G ? qb[h * D + lane * E + e] : 0.f;
        }
        const int64_t r0 = ci * 64, r1 = min(r0 + 64, nc);
        if (r0 >= r1) continue;
        const float* ckp = reinterpret_cast<const float*>(a.ck) + (size_t)pair * a.nc_cap * D;
        float* lg = a.logits + (size_t)pair * a.lg_stride * a.Gp;
        float m[kMaxG], s[kMaxG];
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) {
            m[h] = -INFINITY;
            s[h] = 0.f;
        }
        // rows in groups of kRowU, their loads in flight together
        for (int64_t rg = r0; rg < r1; rg += kRowU) {
            float kv[kRowU][E];
#pragma unroll
            for (int u = 0; u < kRowU; ++u)
#pragma unroll
                for (int e = 0; e < E; ++e)
                    kv[u][e] = rg + u < r1 ? __ldg(ckp + (rg + u) * D + lane * E + e) : 0.f;
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) {
                if (h >= a.G) break;
                float p[kRowU];
#pragma unroll
                for (int u = 0; u < kRowU; ++u) {
                    p[u] = 0.f;
#pragma unroll
                    for (int e = 0; e < E; ++e) p[u] = fmaf(qv[h][e], kv[u][e], p[u]);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                    for (int u = 0; u < kRowU; ++u) p[u] += __shfl_xor_sync(0xffffffffu, p[u], off);
#pragma unroll
                for (int u = 0; u < kRowU; ++u) {
                    if (rg + u < r1) {
                        const float x = p[u] * a.score_log2;
                        if (lane == h) sx[(rg + u - r0) * a.Gp + h] = x;
                        online_add(m[h], s[h], x);
                    }
                }
            }
        }
        float2* st = a.stats + ((size_t)pair * a.nstat + ci) * a.Gp;
#pragma unroll
        for (int h = 0; h < kMaxG; ++h)
            if (h < a.G && lane == h) {
                st[h] = make_float2(m[h], s[h]);
                sm[h] = m[h];
            }
        __syncwarp();
        // the chunk's rows, coalesced: e = exp2(x - max) (0 in the padding heads), or the raw
        // scores x for the Forecast indexer
        const int nvals = (int)(r1 - r0) * a.Gp;
        for (int e = lane; e < nvals; e += 32) {
            const int h = e % a.Gp;
            lg[r0 * a.Gp + e] = h < a.G ? (a.raw ? sx[e] : exp2f(sx[e] - sm[h])) : 0.f;
        }
        __syncwarp();
    }
}

// ============================================================================== select kernel
template <int GP>
struct LogitRow {
    float v[GP];
};
template <int GP>
__device__ __forceinline__ LogitRow<GP> load_row(const float* p) {
    LogitRow<GP> r;
    if constexpr (GP == 1) {
        r.v[0] = __ldcg(p);
    } else if constexpr (GP == 2) {
        const float2 t = __ldcg(reinterpret_cast<const float2*>(p));
        r.v[0] = t.x;
        r.v[1] = t.y;
    } else {
#pragma unroll
        for (int q = 0; q < GP / 4; ++q) {
            const float4 t = __ldcg(reinterpret_cast<const float4*>(p) + q);
            r.v[4 * q] = t.x;
            r.v[4 * q + 1] = t.y;
            r.v[4 * q + 2] = t.z;
            r.v[4 * q + 3] = t.w;
        }
    }
    return r;
}

// S[j - j0] = sum over the group's heads of e[j][h] * w[j / 64][h] for windows j in [j0, j1), where
// e = exp2(x - chunk max) is what the scorer stored and w[c][h] = exp2(chunk max - M_h) / Z_h (the
// .x of the chunk's staged statistics), kU rows per thread in flight.
template <int GP>
__device__ void window_scores(const float* lg, int64_t j0, int64_t j1, int G, const float2* wt, float* S) {
    constexpr int kU = GP <= 4 ? 16 : 8;
    const int tid = threadIdx.x, NT = blockDim.x;
    for (int64_t base = j0; base < j1; base += (int64_t)NT * kU) {
        LogitRow<GP> r[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t j = base + (int64_t)u * NT + tid;
            if (j < j1) r[u] = load_row<GP>(lg + j * GP);
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int64_t j = base + (int64_t)u * NT + tid;
            if (j < j1) {
                const float2* w = wt + (j >> 6) * GP;
                float wx[GP];
#pragma unroll
                for (int h = 0; h < GP; ++h) wx[h] = w[h].x;
                S[j - j0] = group_sum<GP>(r[u].v, wx, G);
            }
        }
    }
}


// grid = pairs * parts. Part p of a pair scores windows [p*PW, p*PW + PW) and owns the blocks whose
// first overlapping window falls in that range (the last part with windows also owns the blocks
// past the last window, which score -inf).
template <int GP>
__global__ void __launch_bounds__(kSelectThreads, 1) select_kernel(SelectArgs a) {
    extern __shared__ uint32_t s_dyn[];  // [key_words] keys, then [PW + W_max] window scores
    __shared__ float sM[kMaxG], sInvZ[kMaxG];
    __shared__ TopkSmem tk;
    __shared__ int s_last;
    const int pair = blockIdx.x / a.parts, part = blockIdx.x - pair * a.parts;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float* S = reinterpret_cast<float*>(s_dyn + a.key_words);
    pdl_trigger();
    pdl_wait();
    const int64_t T = a.seq_lens[pair / a.Hkv];
    const bool ok = T >= 0 && T <= a.T_cap;
    const int64_t nc = ok ? num_windows(T, a.l, a.s) : 0;
    const int64_t nb = ok ? (T + a.BS - 1) / a.BS : 0;
    const int64_t parts_used = nc > 0 ? (nc + a.part_windows - 1) / a.part_windows : 1;
    float* bs = a.bscores + (size_t)pair * a.nb_cap;

    if (part < parts_used) {
        // softmax normaliser of every head from the chunk statistics: one parallel round of
        // loads into shared memory (aliasing the key array, unused until the top-k), then warp h
        // merges head h, and every chunk's weight per head replaces its maximum
        float2* s_st = reinterpret_cast<float2*>(s_dyn);  // 2 * nstat * Gp <= key_words
        {
            const int64_t nch = (nc + 63) / 64;
            const float2* st = a.stats + (size_t)pair * a.nstat * a.Gp;
            for (int64_t e = tid; e < nch * a.Gp; e += kSelectThreads) s_st[e] = ld_cg(st + e);
            __syncthreads();
            if (warp < a.G) {
                float m = -INFINITY, s = 0.f;
                for (int64_t c = lane; c < nch; c += 32) {
                    const float2 v = s_st[c * a.Gp + warp];
                    online_merge(m, s, v.x, v.y);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    const float mo = __shfl_xor_sync(0xffffffffu, m, off);
                    const float so = __shfl_xor_sync(0xffffffffu, s, off);
                    online_merge(m, s, mo, so);
                }
                if (lane == 0) {
                    sM[warp] = m;
                    sInvZ[warp] = s > 0.f ? 1.f / s : 0.f;
                }
            }
            __syncthreads();
            for (int64_t e = tid; e < nch * a.Gp; e += kSelectThreads) {
                const int h = (int)(e % a.Gp);
                s_st[e].x = h < a.G ? (a.raw ? 1.f : exp2f(s_st[e].x - sM[h]) * sInvZ[h]) : 0.f;
            }
            __syncthreads();
        }
        const int64_t j0 = (int64_t)part * a.part_windows;
        const int64_t j1 = min(j0 + a.part_windows, nc);
        const int64_t b_lo = first_block_from(j0, a.BS, a.l, a.s);
        const int64_t b_hi =
            part == parts_used - 1 ? nb : min(first_block_from(j1, a.BS, a.l, a.s), nb);
        const int64_t jend = b_hi > b_lo ? min(last_window(b_hi - 1, a.BS, a.s) + 1, nc) : j0;
        if (jend > j0) {
            const float* lg = a.logits + (size_t)pair * a.lg_stride * a.Gp;
            window_scores<GP>(lg, j0, jend, a.G, s_st, S);
        }
        __syncthreads();
        const int j0i = (int)j0, nci = (int)nc;
        for (int b = (int)b_lo + tid; b < (int)b_hi; b += kSelectThreads) {
            float best = -INFINITY;
            const int jlo = (int)first_window32(b, a.BS, a.l, a.s);
            const int jhi = min((int)last_window32(b, a.BS, a.s), nci - 1);
            for (int j = jlo; j <= jhi; ++j) best = fmaxf(best, S[j - j0i]);
            bs[b] = best;
            if (a.block_scores) a.block_scores[(size_t)pair * a.nb_cap + b] = best;
        }
    }
    if (part == 0 && a.block_scores)
        for (int64_t b = nb + tid; b < a.nb_cap; b += kSelectThreads)
            a.block_scores[(size_t)pair * a.nb_cap + b] = -INFINITY;

    // the last part of the pair runs the top-k over all its block scores
    __threadfence();
    __syncthreads();
    if (tid == 0) {
        const int prev = atomicAdd(a.cnt + pair, 1);
        s_last = (prev == a.parts - 1);
        if (s_last) atomicExch(a.cnt + pair, 0);  // ready for the next launch
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    for (int64_t b = tid; b < nb; b += kSelectThreads) s_dyn[b] = order_key(ld_cg(bs + b));
    const Grp cta{(int)threadIdx.x, (int)blockDim.x, 0};
    topk_prepare(tk, cta);
    __syncthreads();
    topk_union(a, (int)nb, s_dyn, tk, false, cta, a.block_idx + (size_t)pair * a.sel_cap, a.n_sel + pair);
}

// One CTA per pair, when there are enough pairs to fill the GPU: the pair's stored e rows stream
// into a ring of 16 KB shared-memory stages with 1-D bulk copies (the first stages are issued as
// soon as the scores are complete, before the sequence length is read, sized by the row capacity),
// while the chunk statistics turn into one weight per (chunk, head). S[j] is then evaluated from
// shared memory; when the whole row fits the ring and blocks start on window boundaries, the block
// maxima are taken with warp shuffles in the same pass, straight into the key array. The top-k
// follows, with no completion counter.
constexpr int kRingStage = 16 * 1024;
constexpr int kMaxRing = 8;

template <int GP>
__global__ void __launch_bounds__(kSelectThreads, 1) select_single_kernel(SelectArgs a) {
    extern __shared__ __align__(128) uint8_t s_raw[];
    __shared__ __align__(8) uint64_t full[kMaxRing];
    __shared__ TopkSmem tk;
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(s_raw) + 127) & ~uintptr_t(127));
    uint32_t* keys = reinterpret_cast<uint32_t*>(ring + (size_t)a.ring * kRingStage);
    float* S = reinterpret_cast<float*>(keys + a.key_words);
    // [nstat][GP] chunk weights, 16-byte aligned (one vector per chunk when GP = 4)
    float* wt = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(S + a.part_windows) + 15) & ~uintptr_t(15));
    const int pair = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int R = a.ring;
    if (tid == 0) {
        for (int r = 0; r < R; ++r) mbar_init(&full[r], 1);
        mbar_fence_init();
    }
    __syncthreads();
    pdl_trigger();
    pdl_wait();
    constexpr int PW = kRingStage / (GP * 4);  // windows per stage
    const uint8_t* src = reinterpret_cast<const uint8_t*>(a.logits + (size_t)pair * a.lg_stride * GP);
    // thread 0: windows [r*PW, r*PW + PW) below `limit` into ring slot r % R
    auto issue = [&](int r, int64_t limit) {
        const int64_t w0 = (int64_t)r * PW;
        const int64_t wn = min((int64_t)PW, limit - w0);
        const uint32_t bytes = ((uint32_t)wn * GP * 4 + 15u) & ~15u;  // inside the padded row
        uint64_t* bar = &full[r % R];
        mbar_arrive_expect_tx(bar, bytes);
        bulk_load(ring + (size_t)(r % R) * kRingStage, src + (size_t)w0 * GP * 4, bytes, bar);
    };
    // the sequence length and, in warp h < G, head h's chunk statistics (lane l: chunks l + 32u of
    // the row capacity) in one round of loads, requested before the bulk copies so that they do not
    // queue behind them
    constexpr int kStatU = 4;
    const float2* sth = a.stats + (size_t)pair * a.nstat * GP + warp;  // [chunk][GP], head `warp`
    float2 sv[kStatU];
    if (warp < a.G && !a.raw) {
#pragma unroll
        for (int u = 0; u < kStatU; ++u) {
            const int64_t c = lane + 32 * u;
            if (c < a.nstat) sv[u] = ld_cg(sth + c * GP);
        }
    }
    const int64_t T = a.seq_lens[pair / a.Hkv];
    __syncthreads();  // every load above has been issued
    const int cap_pieces = (int)((a.lg_stride + PW - 1) / PW);
    const int n_pre = min(cap_pieces, R);
    if (tid == 0)
        for (int r = 0; r < n_pre; ++r) issue(r, a.lg_stride);
    const bool ok = T >= 0 && T <= a.T_cap;
    const int nc = ok ? (int)num_windows(T, a.l, a.s) : 0;
    const int nb = ok ? (int)((T + a.BS - 1) / a.BS) : 0;
    const int npieces = (nc + PW - 1) / PW;
    const int nch = (nc + 63) / 64;
    // warp h merges head h's chunk statistics into its normaliser (M_h, Z_h), which every lane
    // then holds, and weighs the head's chunks: w[c][h] = exp2(m_c - M_h) / Z_h
    if (warp < a.G) {
        if (a.raw) {
            // Forecast indexer: the stored raw scores are the window scores
            for (int c = lane; c < nch; c += 32) wt[c * GP + warp] = 1.f;
        } else {
            float m = -INFINITY, sum = 0.f;
#pragma unroll
            for (int u = 0; u < kStatU; ++u)
                if (lane + 32 * u < nch) online_merge(m, sum, sv[u].x, sv[u].y);
            for (int c = lane + 32 * kStatU; c < nch; c += 32) {  // rows longer than 8192 windows
                const float2 v = ld_cg(sth + (int64_t)c * GP);
                online_merge(m, sum, v.x, v.y);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float mo = __shfl_xor_sync(0xffffffffu, m, off);
                const float so = __shfl_xor_sync(0xffffffffu, sum, off);
                online_merge(m, sum, mo, so);
            }
            // the lanes' merges round in different orders: every lane takes lane 0's (M, Z), as
            // the multi-part kernel does
            m = __shfl_sync(0xffffffffu, m, 0);
            sum = __shfl_sync(0xffffffffu, sum, 0);
            const float iz = sum > 0.f ? 1.f / sum : 0.f;
#pragma unroll
            for (int u = 0; u < kStatU; ++u)
                if (lane + 32 * u < nch) wt[(lane + 32 * u) * GP + warp] = exp2f(sv[u].x - m) * iz;
            for (int c = lane + 32 * kStatU; c < nch; c += 32)
                wt[c * GP + warp] = exp2f(ld_cg(sth + (int64_t)c * GP).x - m) * iz;
        }
    }
    __syncthreads();
    // S[j] = sum_h e[j][h] * w[j / 64][h], for window j at index i of the stage in slot `slot`
    auto window_score = [&](int slot, int i, int j) -> float {
        const float* lg = reinterpret_cast<const float*>(ring + (size_t)slot * kRingStage) + (size_t)i * GP;
        const float* w = wt + (j >> 6) * GP;
        float x[GP];
        if constexpr (GP == 1) {
            x[0] = lg[0];
        } else if constexpr (GP == 2) {
            const float2 t = *reinterpret_cast<const float2*>(lg);
            x[0] = t.x;
            x[1] = t.y;
        } else {
#pragma unroll
            for (int q = 0; q < GP / 4; ++q) {
                const float4 t = reinterpret_cast<const float4*>(lg)[q];
                x[4 * q] = t.x;
                x[4 * q + 1] = t.y;
                x[4 * q + 2] = t.z;
                x[4 * q + 3] = t.w;
            }
        }
        return group_sum<GP>(x, w, a.G);
    };
    // blocks start on window boundaries: block b's windows are [rb - (L - 1), rb + r - 1], with
    // r = BS / s a power of two up to 32 and L = l / s in {1, 2}
    const int r_w = a.BS / a.s, L_w = a.l / a.s;
    const bool shuffle_max = a.BS % a.s == 0 && a.l % a.s == 0 && r_w >= 1 && r_w <= 32 &&
                             (r_w & (r_w - 1)) == 0 && (L_w == 1 || L_w == 2) && nc > 0;
    bool keys_done = false;
    uint32_t kand = 0xffffffffu, kor = 0u;  // over the candidate keys this thread writes
    if (npieces <= R) {
        // every stage needed is in flight from the start: wait for all that were issued
        // (a wait that runs out is reported; the pass then reads whatever the ring holds, so that
        // every thread takes the same path to the barriers below)
        bool waited = true;
        for (int r = 0; r < n_pre && waited; ++r) waited = mbar_wait(&full[r], 0, kScoreWaitPolls);
        if (!waited) atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
        if (shuffle_max) {
            // warp w takes a contiguous run of 32-window tiles: lane l scores window 32t + l (the
            // stages are contiguous in shared memory, so window j sits at index j of slot 0); the
            // lanes then take running maxima over groups of r lanes, and lane r*i adds window
            // 32t + r*i - 1 when L = 2 (lane 31 of the previous tile for i = 0)
            const int lsh = __ffs(r_w) - 1;  // log2(r)
            const int bsh = 5 - lsh;          // log2(blocks per tile)
            const int bpt = 1 << bsh;
            const int tiles = (nb + bpt - 1) >> bsh;
            const int nw = kSelectThreads / 32;
            const int t_lo = (int)((int64_t)warp * tiles / nw), t_hi = (int)((int64_t)(warp + 1) * tiles / nw);
            // S of window j = 32t + lane (the tile's windows share one chunk, so GP = 4 reads its
            // weights as one broadcast vector)
            auto S_at = [&](int j) -> float {
                const int jj = min(j, nc - 1);
                float v;
                if constexpr (GP == 4) {
                    const float4 e = reinterpret_cast<const float4*>(ring)[jj];
                    const float4 w = reinterpret_cast<const float4*>(wt)[jj >> 6];
                    const float ev[4] = {e.x, e.y, e.z, e.w}, wv[4] = {w.x, w.y, w.z, w.w};
                    v = group_sum<4>(ev, wv, a.G);
                } else {
                    v = window_score(0, jj, jj);
                }
                return j < nc ? v : -INFINITY;
            };
            // four tiles at a time, their shared-memory reads in flight together
            constexpr int kTileU = 4;
            float prev = t_lo > 0 ? S_at(32 * t_lo - 32 + lane) : -INFINITY;
            const int clo = cand_begin(a, nb), chi = cand_end(a, nb);
            for (int t0 = t_lo; t0 < t_hi; t0 += kTileU) {
                // the tiles' chains side by side: reads, then each shuffle step for all tiles
                float cur[kTileU], m[kTileU];
#pragma unroll
                for (int u = 0; u < kTileU; ++u) {
                    cur[u] = t0 + u < t_hi ? S_at(32 * (t0 + u) + lane) : -INFINITY;
                    m[u] = cur[u];
                }
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    if (off < r_w) {
#pragma unroll
                        for (int u = 0; u < kTileU; ++u) m[u] = fmaxf(m[u], __shfl_down_sync(0xffffffffu, m[u], off));
                    }
                }
                if (L_w == 2) {
#pragma unroll
                    for (int u = 0; u < kTileU; ++u) {
                        const float before = __shfl_up_sync(0xffffffffu, cur[u], 1);
                        const float last_prev = __shfl_sync(0xffffffffu, u == 0 ? prev : cur[u > 0 ? u - 1 : 0], 31);
                        m[u] = fmaxf(m[u], lane == 0 ? last_prev : before);
                    }
                }
#pragma unroll
                for (int u = 0; u < kTileU; ++u) {
                    const int b = ((t0 + u) << bsh) + (lane >> lsh);
                    if ((lane & (r_w - 1)) == 0 && t0 + u < t_hi && b < nb) {
                        const uint32_t key = order_key(m[u]);
                        keys[b] = key;
                        if (b >= clo && b < chi) {
                            kand &= key;
                            kor |= key;
                        }
                        if (a.block_scores) a.block_scores[(size_t)pair * a.nb_cap + b] = m[u];
                    }
                }
                prev = cur[kTileU - 1];
            }
            keys_done = true;
        } else {
            for (int j = tid; j < nc; j += kSelectThreads) S[j] = window_score(0, j, j);
        }
    } else {
        for (int r = 0; r < npieces; ++r) {
            // every thread leaves the loop together when a wait runs out (barriers follow)
            const bool got = mbar_wait(&full[r % R], (r / R) & 1, kScoreWaitPolls);
            if (!__syncthreads_and(got)) {
                if (tid == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                break;
            }
            const int w0 = r * PW, wn = min(PW, nc - w0);
            for (int i = tid; i < wn; i += kSelectThreads) S[w0 + i] = window_score(r % R, i, w0 + i);
            __syncthreads();  // the slot has been read by everyone
            if (tid == 0 && r + R < npieces) {
                fence_proxy_async_smem();
                issue(r + R, nc);
            }
        }
    }
    if (!keys_done) {  // uniform: the window scores S are complete once every thread is here
        __syncthreads();
        // block scores: the maximum of S over the complete windows overlapping each block
        const int clo = cand_begin(a, nb), chi = cand_end(a, nb);
        for (int b = tid; b < nb; b += kSelectThreads) {
            float best = -INFINITY;
            const int jlo = (int)first_window32(b, a.BS, a.l, a.s);
            const int jhi = min((int)last_window32(b, a.BS, a.s), nc - 1);
            for (int j = jlo; j <= jhi; ++j) best = fmaxf(best, S[j]);
            const uint32_t key = order_key(best);
            keys[b] = key;
            if (b >= clo && b < chi) {
                kand &= key;
                kor |= key;
            }
            if (a.block_scores) a.block_scores[(size_t)pair * a.nb_cap + b] = best;
        }
    }
    if (a.block_scores)
        for (int64_t b = nb + tid; b < a.nb_cap; b += kSelectThreads)
            a.block_scores[(size_t)pair * a.nb_cap + b] = -INFINITY;
    const Grp cta{(int)threadIdx.x, (int)blockDim.x, 0};
    publish_andor(tk, kand, kor, cta);
    topk_prepare(tk, cta);
    __syncthreads();
    topk_union(a, nb, keys, tk, true, cta, a.block_idx + (size_t)pair * a.sel_cap, a.n_sel + pair);
}

int sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

template <typename K>
cudaError_t launch_score_f32(K kernel, const ScoreArgs& a, cudaStream_t st) {
    if (a.total_chunks == 0) return cudaSuccess;
    int per_sm = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kScoreThreads, 0);
    if (e != cudaSuccess) return e;
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)per_sm * sm_count();
    const int64_t need = (a.total_chunks + kScoreWarps - 1) / kScoreWarps;  // >= 1 chunk per warp
    if (grid > need) grid = need;
    return launch_pdl(kernel, dim3((unsigned)grid), dim3(kScoreThreads), 0, st, a);
}

template <int D>
cudaError_t launch_score_tma(const Plan& p, const ScoreArgs& a, const CUtensorMap* ck_map,
                             cudaStream_t st) {
    if (a.total_chunks == 0) return cudaSuccess;
    const size_t stage_bytes = (size_t)(D / 64) * 64 * 128;
    // a multiple of the consumer count, so that every slot belongs to one consumer warp
    int nstages = (int)((100 * 1024) / stage_bytes);
    if (nstages > kScoreMaxStages) nstages = kScoreMaxStages;
    nstages -= nstages % kScoreConsumers;
    if (nstages < kScoreConsumers) nstages = kScoreConsumers;
    const size_t smem = 1024 + (size_t)nstages * stage_bytes;
    cudaError_t e = ensure_smem<score_tma_kernel<D>>(smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(score_tma_kernel<D>, dim3((unsigned)p.score_ctas), dim3(kScoreTmaThreads),
                      smem, st, a, *ck_map, nstages);
}

template <int GP>
cudaError_t launch_select_k(const Plan& p, const SelectArgs& a, cudaStream_t st) {
    if (p.select_ring > 0) {
        const size_t smem = 128 + (size_t)p.select_ring * kRingStage +
                            (p.select_keys + (size_t)p.select_part_windows + 4 + (size_t)p.nstat * p.Gp) *
                                sizeof(uint32_t);
        cudaError_t e = ensure_smem<select_single_kernel<GP>>(smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(select_single_kernel<GP>, dim3((unsigned)p.pairs), dim3(kSelectThreads),
                          smem, st, a);
    }
    if (p.select_smem > 48 * 1024) {
        cudaError_t e = ensure_smem<select_kernel<GP>>(p.select_smem);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(select_kernel<GP>, dim3((unsigned)(p.pairs * p.select_parts)),
                      dim3(kSelectThreads), p.select_smem, st, a);
}

}  // namespace

cudaError_t launch_score(const Plan& p, const ScoreArgs& a, const CUtensorMap* ck_map,
                         cudaStream_t st) {
    if (p.dtype == BSA_BF16)
        return p.D == 128 ? launch_score_tma<128>(p, a, ck_map, st) : launch_score_tma<64>(p, a, ck_map, st);
    return p.D == 128 ? launch_score_f32(score_f32_kernel<128>, a, st)
                      : launch_score_f32(score_f32_kernel<64>, a, st);
}

cudaError_t launch_select(const Plan& p, const SelectArgs& a, cudaStream_t st) {
    switch (p.Gp) {
        case 1: return launch_select_k<1>(p, a, st);
        case 2: return launch_select_k<2>(p, a, st);
        case 4: return launch_select_k<4>(p, a, st);
        default: return launch_select_k<8>(p, a, st);
    }
}

}  // namespace bsa
