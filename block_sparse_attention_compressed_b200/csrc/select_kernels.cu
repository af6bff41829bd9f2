// Block selection: group scoring, block reduction and top-k (page "SparDA: Sparse Decoupled
// Attention for Efficient Long-Context LLM Inference": Indexer Training, Eq. 6 for the score of a
// GQA group; "Fine-grained supervision" for the max-pool onto the block grid; Theoretical
// Foundation, Eq. 1 and SparDA Architecture, Eq. 4 for the union with init/local blocks and f_top).
//
// Two kernels chained with programmatic dependent launch:
//
// score (persistent): the 64-row chunks of all pairs' compressed keys are shared evenly by the CTAs,
//   so all finish together. It computes the group's logits x[j][h] = q_h . K~_j / tau (log2 units)
//   and writes them to the workspace with each chunk's per-head (max, sum exp2(x - max)).
//   bf16: a producer warp streams the chunks into a ring of shared-memory stages with 2-D TMA
//   tensor copies (128-byte swizzle) completing on mbarriers; four consumer warps take whole
//   chunks in turn and run the contraction on the tensor cores (mma.m16n8k16 with ldmatrix
//   operands: rows are M, the G heads padded to 8 are N, head_dim is K). fp32: FMA dot products,
//   one warp per row.
//
// select (pairs x parts CTAs): merges the chunk statistics into each head's softmax normaliser,
//   turns the logits of its part of the windows into S[j] = sum_h softmax_h[j], max-pools S onto
//   the blocks it owns and writes the block scores. The last part of a pair to finish (completion
//   counter, no waiting) runs the top-k: an 8-bit radix select over order-preserving uint32 keys,
//   ties resolved toward the lower block index by an ordered scan, then the ascending union with
//   the init and local blocks.
#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int kScoreThreads = kScoreWarps * 32;
constexpr int kSelectThreads = 512;

// Block-wide exclusive scan of one int per thread (contiguous, in thread order).
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarps ? s_warp[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, w, off);
            if (lane >= off) w += y;
        }
        if (lane < nwarps) s_warp[lane] = w;
    }
    __syncthreads();
    const int base = warp > 0 ? s_warp[warp - 1] : 0;
    *total = s_warp[nwarps - 1];
    __syncthreads();  // s_warp may be reused right after
    return base + x - v;
}

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
__device__ __forceinline__ void flush_stats(float2* dst, float m0, float s0, float m1, float s1,
                                            int g, int tq, int G) {
    // combine the 8 row groups (lanes with equal tq), then lanes g == 0 publish heads 2tq, 2tq+1
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        float mo = __shfl_xor_sync(0xffffffffu, m0, off), so = __shfl_xor_sync(0xffffffffu, s0, off);
        online_merge(m0, s0, mo, so);
        mo = __shfl_xor_sync(0xffffffffu, m1, off);
        so = __shfl_xor_sync(0xffffffffu, s1, off);
        online_merge(m1, s1, mo, so);
    }
    if (g == 0) {
        if (2 * tq < G) dst[2 * tq] = make_float2(m0, s0);
        if (2 * tq + 1 < G) dst[2 * tq + 1] = make_float2(m1, s1);
    }
}

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
__global__ void __launch_bounds__(kScoreTmaThreads, 2)
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
            // the compressed keys are read once: keep the window logits (reread by the
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
        const int mi = lane >> 3, ri = lane & 7;
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
                const uint32_t* qs = reinterpret_cast<const uint32_t*>(
                    reinterpret_cast<const uint16_t*>(a.q) + ((size_t)b * a.Hq + (size_t)kvh * a.G + g) * D);
#pragma unroll
                for (int ks = 0; ks < KS; ++ks) {
                    qf[ks][0] = g < a.G ? qs[8 * ks + tq] : 0u;
                    qf[ks][1] = g < a.G ? qs[8 * ks + 4 + tq] : 0u;
                }
            }
            const uint8_t* cst = ring + (size_t)st * stage_bytes;
            float c[4][4];
#pragma unroll
            for (int r = 0; r < 4; ++r) c[r][0] = c[r][1] = c[r][2] = c[r][3] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
                for (int r = 0; r < 4; ++r) {  // four independent 16-row groups
                    const int row = 16 * r + ri + 8 * (mi & 1);
                    const int ch = (ks & 3) * 2 + (mi >> 1);
                    uint32_t af[4];
                    ldmatrix_x4(af, smem_u32(cst + (ks >> 2) * box_bytes + row * 128 + ((ch ^ (row & 7)) << 4)));
                    mma_bf16_16816(c[r], af[0], af[1], af[2], af[3], qf[ks][0], qf[ks][1]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);  // the data is in registers: refill the slot
            float* lg = a.logits + (size_t)md.pair * a.lg_stride * a.Gp;
            float m0 = -INFINITY, s0 = 0.f, m1 = -INFINITY, s1 = 0.f;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const float x0 = c[r][0] * a.score_log2, x1 = c[r][1] * a.score_log2;
                const float x2 = c[r][2] * a.score_log2, x3 = c[r][3] * a.score_log2;
                const int lra = 16 * r + g, lrb = lra + 8;
                const int64_t ra = md.row0 + lra, rb = md.row0 + lrb;
                if (lra < md.nrows) {
                    if (h1) *reinterpret_cast<float2*>(lg + ra * a.Gp + 2 * tq) = make_float2(x0, x1);
                    else if (h0) lg[ra * a.Gp + 2 * tq] = x0;
                    if (h0) online_add(m0, s0, x0);
                    if (h1) online_add(m1, s1, x1);
                }
                if (lrb < md.nrows) {
                    if (h1) *reinterpret_cast<float2*>(lg + rb * a.Gp + 2 * tq) = make_float2(x2, x3);
                    else if (h0) lg[rb * a.Gp + 2 * tq] = x2;
                    if (h0) online_add(m0, s0, x2);
                    if (h1) online_add(m1, s1, x3);
                }
            }
            flush_stats(a.stats + ((size_t)md.pair * a.nstat + md.row0 / 64) * a.Gp, m0, s0, m1, s1, g, tq, a.G);
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
                        if (lane == h) lg[(rg + u) * a.Gp + h] = x;
                        online_add(m[h], s[h], x);
                    }
                }
            }
        }
        float2* st = a.stats + ((size_t)pair * a.nstat + ci) * a.Gp;
#pragma unroll
        for (int h = 0; h < kMaxG; ++h)
            if (h < a.G && lane == h) st[h] = make_float2(m[h], s[h]);
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

// S[j - j0] = sum over the group's heads of exp2(x[j][h] - M_h) / Z_h for windows j in [j0, j1),
// kU rows per thread in flight.
template <int GP>
__device__ void window_scores(const float* lg, int64_t j0, int64_t j1, int G, const float* sM,
                              const float* sInvZ, float* S) {
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
                float acc = 0.f;
#pragma unroll
                for (int h = 0; h < GP; ++h)
                    if (h < G) acc += exp2f(r[u].v[h] - sM[h]) * sInvZ[h];
                S[j - j0] = acc;
            }
        }
    }
}

// Top-k of the candidate blocks [init_end, local_begin) by score (ties: lower index first), united
// with the init and local blocks, written ascending. keys[] (shared) holds the nb block keys and
// is overwritten. Each thread keeps its contiguous segment of up to kKeysPerThread candidate keys
// in registers for the radix passes (larger candidate sets are streamed from shared memory).
constexpr int kKeysPerThread = 8;

__device__ void topk_union(const SelectArgs& a, int pair, int nb, uint32_t* keys) {
    __shared__ int s_warp[32];
    __shared__ int hist[256];
    __shared__ uint32_t s_prefix;
    __shared__ int s_need, s_bcnt, s_bn;
    __shared__ uint32_t s_and[32], s_or[32];
    __shared__ uint32_t s_bkey[32];
    __shared__ int s_bidx[32], s_btake[32];
    const int tid = threadIdx.x, NT = blockDim.x, lane = tid & 31;
    const int init_end = min(a.n_init, nb);
    const int local_begin = max(nb - a.n_local, 0);
    const int clo = init_end, chi = max(local_begin, init_end);
    const int ncand = chi - clo;
    const int kk = min(a.top_k, ncand);
    const bool take_all = (kk == ncand);
    const int per = (ncand + NT - 1) / NT;  // contiguous segment of each thread
    const int seg_lo = clo + tid * per, seg_hi = min(seg_lo + per, chi);
    const bool in_regs = per <= kKeysPerThread;
    uint32_t kr[kKeysPerThread];
#pragma unroll
    for (int e = 0; e < kKeysPerThread; ++e) kr[e] = (in_regs && seg_lo + e < seg_hi) ? keys[seg_lo + e] : 0u;

    uint32_t thr = 0xffffffffu;  // keys > thr are taken, plus the first `need` keys == thr
    int need = 0;
    // Early finish: once the digit bucket that holds the k-th key has at most 32 keys, one warp
    // ranks them exactly (score descending, block ascending); then the candidates taken are those
    // above the bucket plus the bucket keys ranked below `need`.
    bool exact = false;
    uint32_t emask = 0u, eprefix = 0u;
    int ebn = 0;
    if (kk > 0 && !take_all) {
        // bytes that every candidate shares need no histogram pass: start at the first byte in
        // which two candidates differ (block-wide AND / OR of the keys)
        uint32_t kand = 0xffffffffu, kor = 0u;
        if (in_regs) {
#pragma unroll
            for (int e = 0; e < kKeysPerThread; ++e) {
                if (seg_lo + e < seg_hi) {
                    kand &= kr[e];
                    kor |= kr[e];
                }
            }
        } else {
            for (int i = seg_lo; i < seg_hi; ++i) {
                kand &= keys[i];
                kor |= keys[i];
            }
        }
        kand = __reduce_and_sync(0xffffffffu, kand);
        kor = __reduce_or_sync(0xffffffffu, kor);
        if (lane == 0) {
            s_and[tid >> 5] = kand;
            s_or[tid >> 5] = kor;
        }
        __syncthreads();
        kand = 0xffffffffu;
        kor = 0u;
        for (int w = 0; w < (NT >> 5); ++w) {
            kand &= s_and[w];
            kor |= s_or[w];
        }
        const uint32_t diff = kand ^ kor;  // bits in which some candidates differ
        int top = 24;
        while (top > 0 && (diff >> top) == 0u) top -= 8;
        uint32_t prefix = top < 24 ? (kand & (0xffffffffu << (top + 8))) : 0u;
        uint32_t mask = top < 24 ? (0xffffffffu << (top + 8)) : 0u;
        need = kk;
        for (int shift = top; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += NT) hist[i] = 0;
            if (tid == 0) s_bn = 0;
            __syncthreads();
            // warp-aggregated histogram (keys of a warp often share a digit): one atomic per
            // distinct digit per warp; all of a thread's keys are processed independently
            if (in_regs) {
                uint32_t dg[kKeysPerThread];
#pragma unroll
                for (int e = 0; e < kKeysPerThread; ++e) {
                    const bool live = seg_lo + e < seg_hi && (kr[e] & mask) == prefix;
                    dg[e] = live ? ((kr[e] >> shift) & 255u) : 256u;
                }
#pragma unroll
                for (int e = 0; e < kKeysPerThread; ++e) {
                    const uint32_t peers = __match_any_sync(0xffffffffu, dg[e]);
                    if (dg[e] < 256u && lane == __ffs(peers) - 1) atomicAdd(&hist[dg[e]], __popc(peers));
                }
            } else {
                for (int i0 = 0; i0 < per; ++i0) {
                    const int i = seg_lo + i0;
                    const uint32_t u = i < seg_hi ? keys[i] : 0u;
                    const uint32_t d = (i < seg_hi && (u & mask) == prefix) ? ((u >> shift) & 255u) : 256u;
                    const uint32_t peers = __match_any_sync(0xffffffffu, d);
                    if (d < 256u && lane == __ffs(peers) - 1) atomicAdd(&hist[d], __popc(peers));
                }
            }
            __syncthreads();
            if (tid < 32) {
                // lane L owns digits 255-8L .. 248-8L, scanned from the top
                int c[8], sum = 0;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    c[k] = hist[255 - 8 * tid - k];
                    sum += c[k];
                }
                int incl = sum;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    int y = __shfl_up_sync(0xffffffffu, incl, off);
                    if (tid >= off) incl += y;
                }
                const int excl = incl - sum;
                if (excl < need && need <= incl) {
                    int acc = excl;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        if (acc < need && acc + c[k] >= need) {
                            s_prefix = prefix | ((uint32_t)(255 - 8 * tid - k) << shift);
                            s_need = need - acc;
                            s_bcnt = c[k];
                        }
                        acc += c[k];
                    }
                }
            }
            __syncthreads();
            prefix = s_prefix;
            need = s_need;
            mask |= 255u << shift;
            if (in_regs && shift > 0 && s_bcnt <= 32) {
                exact = true;
                break;
            }
        }
        thr = prefix;
        if (exact) {
            emask = mask;
            eprefix = prefix;
#pragma unroll
            for (int e = 0; e < kKeysPerThread; ++e) {
                if (seg_lo + e < seg_hi && (kr[e] & mask) == prefix) {
                    const int slot = atomicAdd(&s_bn, 1);
                    s_bkey[slot] = kr[e];
                    s_bidx[slot] = seg_lo + e;
                }
            }
            __syncthreads();
            ebn = s_bn;
            if (tid < 32) {
                const uint32_t key = tid < ebn ? s_bkey[tid] : 0u;
                const int idx = tid < ebn ? s_bidx[tid] : 0x7fffffff;
                int rank = 0;
                for (int j = 0; j < ebn; ++j) {
                    const uint32_t kj = s_bkey[j];
                    const int ij = s_bidx[j];
                    rank += (kj > key || (kj == key && ij < idx));
                }
                if (tid < ebn) s_btake[tid] = rank < need ? idx : -1;
            }
            __syncthreads();
        }
    }
    if (exact) {
        // above the bucket, or ranked within it
#pragma unroll
        for (int e = 0; e < kKeysPerThread; ++e) {
            if (seg_lo + e < seg_hi) {
                const uint32_t mk = kr[e] & emask;
                bool take = mk > eprefix;
                if (mk == eprefix)
                    for (int j = 0; j < ebn; ++j) take |= s_btake[j] == seg_lo + e;
                keys[seg_lo + e] = take ? 1u : 0u;
            }
        }
    } else {
        // mark the taken candidates in index order (equal keys: lowest block first)
        int cnt = 0;
        if (in_regs) {
#pragma unroll
            for (int e = 0; e < kKeysPerThread; ++e) cnt += (seg_lo + e < seg_hi && kr[e] == thr);
        } else {
            for (int i = seg_lo; i < seg_hi; ++i) cnt += (keys[i] == thr);
        }
        int tot;
        int r = block_exclusive_scan(cnt, s_warp, &tot);
        if (in_regs) {
#pragma unroll
            for (int e = 0; e < kKeysPerThread; ++e) {
                if (seg_lo + e < seg_hi) {
                    const uint32_t u = kr[e];
                    const bool take = take_all || u > thr || (u == thr && r < need);
                    r += (u == thr);
                    keys[seg_lo + e] = take ? 1u : 0u;
                }
            }
        } else {
            for (int i = seg_lo; i < seg_hi; ++i) {
                const uint32_t u = keys[i];
                const bool take = take_all || u > thr || (u == thr && r < need);
                r += (u == thr);
                keys[i] = take ? 1u : 0u;
            }
        }
    }
    __syncthreads();
    // union with init and local blocks, emitted in ascending block order
    int32_t* out = a.block_idx + (size_t)pair * a.sel_cap;
    {
        const int per2 = (nb + NT - 1) / NT;
        const int lo = tid * per2, hi = min(lo + per2, nb);
        int cnt = 0;
        for (int i = lo; i < hi; ++i) cnt += (i < init_end || i >= local_begin || keys[i] != 0u);
        int total;
        int pos = block_exclusive_scan(cnt, s_warp, &total);
        for (int i = lo; i < hi; ++i)
            if (i < init_end || i >= local_begin || keys[i] != 0u) out[pos++] = i;
        for (int i = total + tid; i < a.sel_cap; i += NT) out[i] = -1;
        if (tid == 0) a.n_sel[pair] = total;
    }
}

// grid = pairs * parts. Part p of a pair scores windows [p*PW, p*PW + PW) and owns the blocks whose
// first overlapping window falls in that range (the last part with windows also owns the blocks
// past the last window, which score -inf).
template <int GP>
__global__ void __launch_bounds__(kSelectThreads, 1) select_kernel(SelectArgs a) {
    extern __shared__ uint32_t s_dyn[];  // [key_words] keys, then [PW + W_max] window scores
    __shared__ float sM[kMaxG], sInvZ[kMaxG];
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
        // merges head h
        {
            const int64_t nch = (nc + 63) / 64;
            float2* s_st = reinterpret_cast<float2*>(s_dyn);  // 2 * nstat * Gp <= key_words
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
        }
        const int64_t j0 = (int64_t)part * a.part_windows;
        const int64_t j1 = min(j0 + a.part_windows, nc);
        const int64_t b_lo = first_block_from(j0, a.BS, a.l, a.s);
        const int64_t b_hi =
            part == parts_used - 1 ? nb : min(first_block_from(j1, a.BS, a.l, a.s), nb);
        const int64_t jend = b_hi > b_lo ? min(last_window(b_hi - 1, a.BS, a.s) + 1, nc) : j0;
        if (jend > j0) {
            const float* lg = a.logits + (size_t)pair * a.lg_stride * a.Gp;
            window_scores<GP>(lg, j0, jend, a.G, sM, sInvZ, S);
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
    __syncthreads();
    topk_union(a, pair, (int)nb, s_dyn);
}

// One CTA per pair, when there are enough pairs to fill the GPU: the pair's logits stream into a
// ring of 16 KB shared-memory stages with 1-D bulk copies (all stages in flight at once, while the
// chunk statistics are merged), S[j] is evaluated from shared memory, the block maxima go straight
// to the key array and the top-k follows, with no completion counter.
constexpr int kRingStage = 16 * 1024;
constexpr int kMaxRing = 8;

template <int GP>
__global__ void __launch_bounds__(kSelectThreads, 1) select_single_kernel(SelectArgs a) {
    extern __shared__ __align__(128) uint8_t s_raw[];
    __shared__ __align__(8) uint64_t full[kMaxRing];
    __shared__ float sM[kMaxG], sInvZ[kMaxG];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(s_raw) + 127) & ~uintptr_t(127));
    uint32_t* keys = reinterpret_cast<uint32_t*>(ring + (size_t)a.ring * kRingStage);
    float* S = reinterpret_cast<float*>(keys + a.key_words);
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
    const int64_t T = a.seq_lens[pair / a.Hkv];
    const bool ok = T >= 0 && T <= a.T_cap;
    const int nc = ok ? (int)num_windows(T, a.l, a.s) : 0;
    const int nb = ok ? (int)((T + a.BS - 1) / a.BS) : 0;
    constexpr int PW = kRingStage / (GP * 4);  // windows per stage
    const int npieces = (nc + PW - 1) / PW;
    const uint8_t* src = reinterpret_cast<const uint8_t*>(a.logits + (size_t)pair * a.lg_stride * GP);
    auto issue = [&](int r) {  // thread 0: stage r of the pair's logits into ring slot r % R
        const int w0 = r * PW, wn = min(PW, nc - w0);
        const uint32_t bytes = ((uint32_t)wn * GP * 4 + 15u) & ~15u;  // inside the padded row
        uint64_t* bar = &full[r % R];
        mbar_arrive_expect_tx(bar, bytes);
        bulk_load(ring + (size_t)(r % R) * kRingStage, src + (size_t)w0 * GP * 4, bytes, bar);
    };
    if (tid == 0)
        for (int r = 0; r < npieces && r < R; ++r) issue(r);

    // softmax normaliser of every head from the chunk statistics (staged in the key array)
    {
        const int nch = (nc + 63) / 64;
        float2* s_st = reinterpret_cast<float2*>(keys);  // 2 * nstat * Gp <= key_words
        const float2* st = a.stats + (size_t)pair * a.nstat * GP;
        for (int e = tid; e < nch * GP; e += kSelectThreads) s_st[e] = ld_cg(st + e);
        __syncthreads();
        if (warp < a.G) {
            float m = -INFINITY, sum = 0.f;
            for (int c = lane; c < nch; c += 32) {
                const float2 v = s_st[c * GP + warp];
                online_merge(m, sum, v.x, v.y);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const float mo = __shfl_xor_sync(0xffffffffu, m, off);
                const float so = __shfl_xor_sync(0xffffffffu, sum, off);
                online_merge(m, sum, mo, so);
            }
            if (lane == 0) {
                sM[warp] = m;
                sInvZ[warp] = sum > 0.f ? 1.f / sum : 0.f;
            }
        }
        __syncthreads();
    }
    float M[GP], iz[GP];
#pragma unroll
    for (int h = 0; h < GP; ++h) {
        M[h] = h < a.G ? sM[h] : 0.f;
        iz[h] = h < a.G ? sInvZ[h] : 0.f;
    }
    // S[j] = sum_h exp2(x[j][h] - M_h) / Z_h for window j at index i of the stage in slot `slot`
    auto window_score = [&](int slot, int i) -> float {
        const float* lg = reinterpret_cast<const float*>(ring + (size_t)slot * kRingStage);
        float x[GP];
        if constexpr (GP == 1) {
            x[0] = lg[i];
        } else if constexpr (GP == 2) {
            const float2 t = reinterpret_cast<const float2*>(lg)[i];
            x[0] = t.x;
            x[1] = t.y;
        } else {
#pragma unroll
            for (int q = 0; q < GP / 4; ++q) {
                const float4 t = reinterpret_cast<const float4*>(lg + (size_t)i * GP)[q];
                x[4 * q] = t.x;
                x[4 * q + 1] = t.y;
                x[4 * q + 2] = t.z;
                x[4 * q + 3] = t.w;
            }
        }
        float acc = 0.f;
#pragma unroll
        for (int h = 0; h < GP; ++h)
            if (h < a.G) acc += exp2f(x[h] - M[h]) * iz[h];
        return acc;
    };
    if (npieces <= R) {
        // every stage is in flight from the start: wait for all, then one pass over the windows
        bool waited = true;
        for (int r = 0; r < npieces && waited; ++r) waited = mbar_wait(&full[r], 0, kScoreWaitPolls);
        if (!waited) {
            if (tid == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
        } else {
            for (int j = tid; j < nc; j += kSelectThreads) S[j] = window_score(j / PW, j % PW);
        }
    } else {
        for (int r = 0; r < npieces; ++r) {
            if (!mbar_wait(&full[r % R], (r / R) & 1, kScoreWaitPolls)) {
                if (tid == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                break;
            }
            const int w0 = r * PW, wn = min(PW, nc - w0);
            for (int i = tid; i < wn; i += kSelectThreads) S[w0 + i] = window_score(r % R, i);
            __syncthreads();  // the slot has been read by everyone
            if (tid == 0 && r + R < npieces) {
                fence_proxy_async_smem();
                issue(r + R);
            }
        }
    }
    __syncthreads();
    // block scores: the maximum of S over the complete windows overlapping each block
    for (int b = tid; b < nb; b += kSelectThreads) {
        float best = -INFINITY;
        const int jlo = (int)first_window32(b, a.BS, a.l, a.s);
        const int jhi = min((int)last_window32(b, a.BS, a.s), nc - 1);
        for (int j = jlo; j <= jhi; ++j) best = fmaxf(best, S[j]);
        keys[b] = order_key(best);
        if (a.block_scores) a.block_scores[(size_t)pair * a.nb_cap + b] = best;
    }
    if (a.block_scores)
        for (int64_t b = nb + tid; b < a.nb_cap; b += kSelectThreads)
            a.block_scores[(size_t)pair * a.nb_cap + b] = -INFINITY;
    __syncthreads();
    topk_union(a, pair, nb, keys);
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
                            (p.select_keys + (size_t)p.select_part_windows) * sizeof(uint32_t);
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
