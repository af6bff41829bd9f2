// Block selection: group scoring, block reduction and top-k (page "SparDA: Sparse Decoupled
// Attention for Efficient Long-Context LLM Inference": Indexer Training, Eq. 6 for the score of a
// GQA group; "Fine-grained supervision" for the max-pool onto the block grid; Theoretical
// Foundation, Eq. 1 and SparDA Architecture, Eq. 4 for the union with init/local blocks and f_top).
//
// One kernel, grid = pairs * items CTAs (pair-major). Each CTA scores a contiguous slice of the
// pair's compressed keys against the group's G query heads and writes log2-domain logits plus the
// slice's per-head (max, sum exp2) to the workspace. The last CTA of a pair to finish (completion
// counter, no waiting) merges the per-slice statistics into each head's softmax normaliser,
// evaluates S[j] = sum_h softmax_h[j] on the fly, max-pools onto blocks and runs the selection.
//
// bf16 path: the contraction q . K~_j runs on the tensor cores with mma.m16n8k16: compressed-key
// rows are the M dimension (16 per tile), the group's heads are N (padded to 8), head_dim is K.
// Because a dot product does not care about the order of its terms, each lane feeds the A operand
// straight from its own 16-byte global loads (no shared-memory staging, no shuffles) and the q
// operand is permuted the same way once per CTA.
#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int kScoreThreads = kScoreWarps * 32;

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

// Selection for one pair, run by a whole CTA after every slice of the pair is scored.
__device__ void select_pair(const ScoreArgs& a, int pair, int64_t T, int64_t nc, bool ok,
                            uint32_t* keys) {
    __shared__ float sM[kMaxG], sInvZ[kMaxG];
    __shared__ int s_warp[32];
    __shared__ int hist[256];
    __shared__ uint32_t s_prefix;
    __shared__ int s_need;
    const int tid = threadIdx.x, NT = blockDim.x;
    const int64_t nb = ok ? (T + a.BS - 1) / a.BS : 0;

    // 1. softmax normaliser of every head from the per-slice (max, sum) pairs
    if (tid < a.G) {
        const float2* st = a.stats + (size_t)pair * a.items * a.Gp + tid;
        float M = -INFINITY;
        for (int it = 0; it < a.items; ++it) M = fmaxf(M, ld_cg(st + (size_t)it * a.Gp).x);
        float Z = 0.f;
        if (M != -INFINITY) {
            for (int it = 0; it < a.items; ++it) {
                float2 ms = ld_cg(st + (size_t)it * a.Gp);
                if (ms.x != -INFINITY) Z += ms.y * exp2f(ms.x - M);
            }
        }
        sM[tid] = M;
        sInvZ[tid] = Z > 0.f ? 1.f / Z : 0.f;
    }
    __syncthreads();

    // 2. block scores: max over the complete windows overlapping the block of sum_h p_h[j]
    const float* lg = a.logits + (size_t)pair * a.nc_cap * a.Gp;
    for (int64_t bb = tid; bb < a.nb_cap; bb += NT) {
        float best = -INFINITY;
        if (bb < nb && nc > 0) {
            const int64_t tok0 = bb * a.BS;
            const int64_t jlo = tok0 >= a.l ? (tok0 - a.l) / a.s + 1 : 0;
            const int64_t jhi = min((tok0 + a.BS - 1) / a.s, nc - 1);
            for (int64_t j = jlo; j <= jhi; ++j) {
                const float* row = lg + j * a.Gp;
                float S = 0.f;
                for (int h = 0; h < a.G; ++h) S += exp2f(ld_cg(row + h) - sM[h]) * sInvZ[h];
                best = fmaxf(best, S);
            }
        }
        if (a.block_scores) a.block_scores[(size_t)pair * a.nb_cap + bb] = best;
        keys[bb] = order_key(best);
    }
    __syncthreads();

    // 3. top-k among the candidates [init_end, local_begin): radix select of the k-th key
    const int64_t init_end = min((int64_t)a.n_init, nb);
    const int64_t local_begin = max(nb - (int64_t)a.n_local, (int64_t)0);
    const int64_t clo = init_end, chi = max(local_begin, init_end);
    const int64_t ncand = chi - clo;
    const int kk = (int)min((int64_t)a.top_k, ncand);
    const bool take_all = (kk == ncand);
    uint32_t thr = 0xffffffffu;  // keys > thr are taken, plus the first `need` keys == thr
    int need = 0;
    if (kk > 0 && !take_all) {
        uint32_t prefix = 0, mask = 0;
        need = kk;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = tid; i < 256; i += NT) hist[i] = 0;
            __syncthreads();
            for (int64_t i = clo + tid; i < chi; i += NT) {
                const uint32_t u = keys[i];
                if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1);
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
                        }
                        acc += c[k];
                    }
                }
            }
            __syncthreads();
            prefix = s_prefix;
            need = s_need;
            mask |= 255u << shift;
        }
        thr = prefix;
    }

    // 4. mark the taken candidates in index order (equal keys: lowest block first)
    {
        const int64_t per = (ncand + NT - 1) / NT;
        const int64_t lo = clo + tid * per, hi = min(lo + per, chi);
        int cnt = 0;
        for (int64_t i = lo; i < hi; ++i) cnt += (keys[i] == thr);
        int tot;
        int r = block_exclusive_scan(cnt, s_warp, &tot);
        for (int64_t i = lo; i < hi; ++i) {
            const uint32_t u = keys[i];
            const bool take = take_all || u > thr || (u == thr && r < need);
            r += (u == thr);
            keys[i] = take ? 1u : 0u;
        }
    }
    __syncthreads();

    // 5. union with init and local blocks, emitted in ascending block order
    int32_t* out = a.block_idx + (size_t)pair * a.sel_cap;
    {
        const int64_t per = (nb + NT - 1) / NT;
        const int64_t lo = tid * per, hi = min(lo + per, nb);
        int cnt = 0;
        for (int64_t i = lo; i < hi; ++i)
            cnt += (i < init_end || i >= local_begin || keys[i] != 0u);
        int total;
        int pos = block_exclusive_scan(cnt, s_warp, &total);
        for (int64_t i = lo; i < hi; ++i)
            if (i < init_end || i >= local_begin || keys[i] != 0u) out[pos++] = (int32_t)i;
        for (int i = total + tid; i < a.sel_cap; i += NT) out[i] = -1;
        if (tid == 0) a.n_sel[pair] = total;
    }
}

// Merge the warps' (max, sum) per head, publish the slice statistics, and let the last CTA of the
// pair run the selection.
__device__ void finish_slice(const ScoreArgs& a, int pair, int item, int64_t T, int64_t nc, bool ok,
                             float (*s_wm)[kMaxG], float (*s_ws)[kMaxG], uint32_t* keys) {
    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x < a.G) {
        float m = -INFINITY, s = 0.f;
        for (int w = 0; w < kScoreWarps; ++w) online_merge(m, s, s_wm[w][threadIdx.x], s_ws[w][threadIdx.x]);
        a.stats[((size_t)pair * a.items + item) * a.Gp + threadIdx.x] = make_float2(m, s);
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int prev = atomicAdd(a.cnt + pair, 1);
        s_last = (prev == a.items - 1);
        if (s_last) atomicExch(a.cnt + pair, 0);  // ready for the next launch
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    select_pair(a, pair, T, nc, ok, keys);
}

__device__ __forceinline__ void seq_info(const ScoreArgs& a, int b, int pair, int item, int64_t& T,
                                         int64_t& nc, bool& ok) {
    T = a.seq_lens[b];
    ok = T >= 0 && T <= a.T_cap;
    if (!ok && item == 0 && threadIdx.x == 0 && pair % a.Hkv == 0)
        atomicOr(a.err, (uint32_t)BSA_DEVERR_SEQ_LEN);
    nc = (ok && T >= a.l) ? (T - a.l) / a.s + 1 : 0;
}

// ---------------------------------------------------------------------------------- bf16 path
template <int D>
struct KTile {
    static constexpr int NI = D / 32;  // 16-byte chunks a lane holds per row (chunks tq + 4i)
    uint4 a[NI], b[NI];                // rows r+g and r+g+8 of the tile
};

template <int D>
__device__ __forceinline__ void load_ktile(KTile<D>& t, const uint16_t* ckp, int64_t r, int64_t r1,
                                           int g, int tq) {
    const int64_t ra = r + g, rb = r + g + 8;
#pragma unroll
    for (int i = 0; i < KTile<D>::NI; ++i) {
        const int col = (tq + 4 * i) * 8;
        t.a[i] = ra < r1 ? ld_stream(ckp + ra * D + col) : make_uint4(0, 0, 0, 0);
        t.b[i] = rb < r1 ? ld_stream(ckp + rb * D + col) : make_uint4(0, 0, 0, 0);
    }
}

template <int D>
__global__ void __launch_bounds__(kScoreThreads, 2) score_select_bf16_kernel(ScoreArgs a) {
    extern __shared__ uint32_t s_keys[];
    __shared__ float s_wm[kScoreWarps][kMaxG], s_ws[kScoreWarps][kMaxG];
    constexpr int NI = D / 32;
    const int pair = blockIdx.x / a.items, item = blockIdx.x - pair * a.items;
    const int b = pair / a.Hkv, kvh = pair - b * a.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;

    // q as the B operand: lane (g, tq) holds head g, chunks tq + 4i -- the same d positions its
    // own key loads cover. q is never written by this library, so it is read before the wait.
    uint32_t qf[NI][4];
    {
        const uint16_t* qh =
            reinterpret_cast<const uint16_t*>(a.q) + ((size_t)b * a.Hq + (size_t)kvh * a.G + g) * D;
#pragma unroll
        for (int i = 0; i < NI; ++i) {
            uint4 v = g < a.G ? *reinterpret_cast<const uint4*>(qh + (tq + 4 * i) * 8)
                              : make_uint4(0, 0, 0, 0);
            qf[i][0] = v.x;
            qf[i][1] = v.y;
            qf[i][2] = v.z;
            qf[i][3] = v.w;
        }
    }
    pdl_trigger();
    pdl_wait();
    int64_t T, nc;
    bool ok;
    seq_info(a, b, pair, item, T, nc, ok);

    const int64_t r0 = ((int64_t)item * kScoreWarps + warp) * a.rows_per_warp;
    const int64_t r1 = min(r0 + (int64_t)a.rows_per_warp, nc);
    const uint16_t* ckp = reinterpret_cast<const uint16_t*>(a.ck) + (size_t)pair * a.nc_cap * D;
    float* lg = a.logits + (size_t)pair * a.nc_cap * a.Gp;
    const bool h0 = 2 * tq < a.G, h1 = 2 * tq + 1 < a.G;
    float m0 = -INFINITY, s0 = 0.f, m1 = -INFINITY, s1 = 0.f;

    KTile<D> cur, nxt;
    if (r0 < r1) load_ktile<D>(cur, ckp, r0, r1, g, tq);
    for (int64_t r = r0; r < r1; r += 16) {
        if (r + 16 < r1) load_ktile<D>(nxt, ckp, r + 16, r1, g, tq);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < NI; ++i) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                mma_bf16_16816(c, u4_get(cur.a[i], 2 * hh), u4_get(cur.b[i], 2 * hh),
                               u4_get(cur.a[i], 2 * hh + 1), u4_get(cur.b[i], 2 * hh + 1),
                               qf[i][2 * hh], qf[i][2 * hh + 1]);
            }
        }
        const float x0 = c[0] * a.score_log2, x1 = c[1] * a.score_log2;
        const float x2 = c[2] * a.score_log2, x3 = c[3] * a.score_log2;
        const int64_t ra = r + g, rb = r + g + 8;
        if (ra < r1) {
            if (h1) *reinterpret_cast<float2*>(lg + ra * a.Gp + 2 * tq) = make_float2(x0, x1);
            else if (h0) lg[ra * a.Gp + 2 * tq] = x0;
            if (h0) online_add(m0, s0, x0);
            if (h1) online_add(m1, s1, x1);
        }
        if (rb < r1) {
            if (h1) *reinterpret_cast<float2*>(lg + rb * a.Gp + 2 * tq) = make_float2(x2, x3);
            else if (h0) lg[rb * a.Gp + 2 * tq] = x2;
            if (h0) online_add(m0, s0, x2);
            if (h1) online_add(m1, s1, x3);
        }
        cur = nxt;
    }
    // combine the 8 row-groups (lanes with equal tq)
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        float mo = __shfl_xor_sync(0xffffffffu, m0, off), so = __shfl_xor_sync(0xffffffffu, s0, off);
        online_merge(m0, s0, mo, so);
        mo = __shfl_xor_sync(0xffffffffu, m1, off);
        so = __shfl_xor_sync(0xffffffffu, s1, off);
        online_merge(m1, s1, mo, so);
    }
    if (g == 0) {
        if (h0) {
            s_wm[warp][2 * tq] = m0;
            s_ws[warp][2 * tq] = s0;
        }
        if (h1) {
            s_wm[warp][2 * tq + 1] = m1;
            s_ws[warp][2 * tq + 1] = s1;
        }
    }
    finish_slice(a, pair, item, T, nc, ok, s_wm, s_ws, s_keys);
}

// ---------------------------------------------------------------------------------- fp32 path
// Plain FMA dot products (fp32 inputs keep fp32 accuracy); one warp per row, lanes split d.
template <int D>
__global__ void __launch_bounds__(kScoreThreads, 2) score_select_f32_kernel(ScoreArgs a) {
    extern __shared__ uint32_t s_keys[];
    __shared__ float s_wm[kScoreWarps][kMaxG], s_ws[kScoreWarps][kMaxG];
    constexpr int E = D / 32;
    const int pair = blockIdx.x / a.items, item = blockIdx.x - pair * a.items;
    const int b = pair / a.Hkv, kvh = pair - b * a.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    float qv[kMaxG][E];
    const float* qbase = reinterpret_cast<const float*>(a.q) + ((size_t)b * a.Hq + (size_t)kvh * a.G) * D;
#pragma unroll
    for (int h = 0; h < kMaxG; ++h)
#pragma unroll
        for (int e = 0; e < E; ++e) qv[h][e] = h < a.G ? qbase[h * D + lane * E + e] : 0.f;
    pdl_trigger();
    pdl_wait();
    int64_t T, nc;
    bool ok;
    seq_info(a, b, pair, item, T, nc, ok);

    const int64_t r0 = ((int64_t)item * kScoreWarps + warp) * a.rows_per_warp;
    const int64_t r1 = min(r0 + (int64_t)a.rows_per_warp, nc);
    const float* ckp = reinterpret_cast<const float*>(a.ck) + (size_t)pair * a.nc_cap * D;
    float* lg = a.logits + (size_t)pair * a.nc_cap * a.Gp;
    float m[kMaxG], s[kMaxG];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
        m[h] = -INFINITY;
        s[h] = 0.f;
    }
    for (int64_t r = r0; r < r1; ++r) {
        float kv[E];
#pragma unroll
        for (int e = 0; e < E; ++e) kv[e] = __ldg(ckp + r * D + lane * E + e);
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) {
            if (h >= a.G) break;
            float p = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) p = fmaf(qv[h][e], kv[e], p);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
            const float x = p * a.score_log2;
            if (lane == h) lg[r * a.Gp + h] = x;
            online_add(m[h], s[h], x);
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) {
            if (h < a.G) {
                s_wm[warp][h] = m[h];
                s_ws[warp][h] = s[h];
            }
        }
    }
    finish_slice(a, pair, item, T, nc, ok, s_wm, s_ws, s_keys);
}

template <typename K>
cudaError_t launch_with_smem(K kernel, const Plan& p, const ScoreArgs& a, cudaStream_t st) {
    if (p.score_smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)p.score_smem);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(kernel, dim3((unsigned)(p.pairs * p.score_items)), dim3(kScoreThreads),
                      p.score_smem, st, a);
}

}  // namespace

cudaError_t launch_score_select(const Plan& p, const ScoreArgs& a, cudaStream_t st) {
    if (p.dtype == BSA_BF16)
        return p.D == 128 ? launch_with_smem(score_select_bf16_kernel<128>, p, a, st)
                          : launch_with_smem(score_select_bf16_kernel<64>, p, a, st);
    return p.D == 128 ? launch_with_smem(score_select_f32_kernel<128>, p, a, st)
                      : launch_with_smem(score_select_f32_kernel<64>, p, a, st);
}

}  // namespace bsa
