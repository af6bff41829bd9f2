// Token-level shared index (page "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing",
// CLSA abstract: one indexer computes a token-level top-k once and every layer reuses it). The
// indexer is the base selector at token granularity (page "SparDA: Sparse Decoupled Attention for
// Efficient Long-Context LLM Inference", Indexer Training, Eq. 6, with every key as its own window):
// S[t] = sum over the group's heads of softmax_t(q_h . K_t / tau) over the index layer's tokens; the
// first n_init * BS and last n_local * BS tokens are always taken and top_k * BS more by score (ties
// to the lower token), written ascending (Theoretical Foundation, Eq. 1, with blocks of one token).
//
// The scoring is the compressed-key scorer run with windows of one token on the index layer's K
// cache (its window terms e = exp2(x - chunk max) and per-chunk statistics land in the workspace).
// token_topk_kernel (a CTA per pair) weighs the terms into S[t], keeps the keys in shared memory and
// runs the shared top-k; token_decode_kernel (a CTA per (layer, pair)) gathers the taken tokens'
// K and V rows with cp.async into a swizzled three-stage ring and attends them on the tensor cores
// with the decode tiles, merging its four warps straight into O and LSE.
#include "bsa_internal.cuh"
#include "tiles.cuh"
#include "topk.cuh"

namespace bsa {
namespace {

constexpr int kTkThreads = 1024;

template <int GP>
__global__ void __launch_bounds__(kTkThreads, 1) token_topk_kernel(const TokenArgs a) {
    extern __shared__ uint8_t dsm_raw[];
    __shared__ TopkSmem tk;
    uint32_t* keys = reinterpret_cast<uint32_t*>(dsm_raw);                        // [T_cap]
    float* wts = reinterpret_cast<float*>(keys + ((a.T_cap + 3) & ~int64_t(3)));  // [nstat][GP]
    const int pair = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const Grp cta{tid, kTkThreads, 0};
    pdl_trigger();
    pdl_wait();
    const int b = pair / a.Hkv;
    int64_t T = a.seq_lens[b];
    if (T < 0 || T > a.T_cap) {
        if (tid == 0 && pair % a.Hkv == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_SEQ_LEN);
        T = T < 0 ? 0 : a.T_cap;
    }
    const int n = (int)T;
    const int nch = (n + 63) / 64;
    topk_prepare(tk, cta);
    // each head's softmax normaliser (M, Z) from the chunk statistics, then one weight per
    // (chunk, head): w = exp2(m_c - M) / Z
    if (warp < a.G) {
        const float2* st = a.stats + (size_t)pair * a.nstat * GP;
        float m = -INFINITY, sum = 0.f;
        for (int c = lane; c < nch; c += 32) {
            const float2 sv = st[(size_t)c * GP + warp];
            online_merge(m, sum, sv.x, sv.y);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float mo = __shfl_xor_sync(0xffffffffu, m, off);
            const float so = __shfl_xor_sync(0xffffffffu, sum, off);
            online_merge(m, sum, mo, so);
        }
        m = __shfl_sync(0xffffffffu, m, 0);
        sum = __shfl_sync(0xffffffffu, sum, 0);
        const float iz = sum > 0.f ? 1.f / sum : 0.f;
        for (int c = lane; c < nch; c += 32) wts[c * GP + warp] = exp2f(st[(size_t)c * GP + warp].x - m) * iz;
    }
    __syncthreads();
    // token scores S[t] = sum_h e[t][h] w[chunk][h], as order keys
    const float* lg = a.logits + (size_t)pair * a.lg_stride * GP;
    for (int t = tid; t < n; t += kTkThreads) {
        float e[GP];
        if constexpr (GP >= 4) {
#pragma unroll
            for (int h4 = 0; h4 < GP; h4 += 4) {
                const float4 v = *reinterpret_cast<const float4*>(lg + (size_t)t * GP + h4);
                e[h4] = v.x;
                e[h4 + 1] = v.y;
                e[h4 + 2] = v.z;
                e[h4 + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int h = 0; h < GP; ++h) e[h] = lg[(size_t)t * GP + h];
        }
        keys[t] = order_key(group_sum<GP>(e, wts + (t >> 6) * GP, a.G));
    }
    __syncthreads();
    SelectArgs sa;
    memset(&sa, 0, sizeof sa);
    sa.n_init = a.n_init_tok;
    sa.n_local = a.n_local_tok;
    sa.top_k = a.top_k_tok;
    sa.sel_cap = a.tok_cap;
    topk_union(sa, n, keys, tk, false, cta, a.tok_idx + (size_t)pair * a.tok_cap, a.n_tok + pair);
}

// ---------------------------------------------------------------------------- token attention
constexpr int kTdWarps = 4;
constexpr int kTdStages = 3;
constexpr uint32_t kTdBox = 64u * 128u;  // 64 rows x 128 bytes

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int D>
__global__ void __launch_bounds__(kTdWarps * 32) token_decode_kernel(const TokenArgs a, TokenLayers L) {
    constexpr int NB = D / 64;
    constexpr uint32_t kStage = 2u * NB * kTdBox;  // K and V of 64 tokens
    extern __shared__ uint8_t dsm_raw[];
    uint8_t* ring = dsm_raw + ((1024u - (smem_u32(dsm_raw) & 1023u)) & 1023u);
    float* merge = reinterpret_cast<float*>(ring + kTdStages * kStage);
    const int layer = blockIdx.x / a.pairs, pair = blockIdx.x - layer * a.pairs;
    const int b = pair / a.Hkv, kvh = pair - b * a.Hkv;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31, g = lane >> 2, tq = lane & 3;
    pdl_trigger();
    pdl_wait();
    const int n = min(max(a.n_tok[pair], 0), a.tok_cap);
    const int64_t T = min(max((int64_t)a.seq_lens[b], (int64_t)0), a.T_cap);
    const int32_t* idx = a.tok_idx + (size_t)pair * a.tok_cap;
    const uint16_t* kc = reinterpret_cast<const uint16_t*>(L.k[layer]) + (size_t)pair * a.T_cap * D;
    const uint16_t* vc = reinterpret_cast<const uint16_t*>(L.v[layer]) + (size_t)pair * a.T_cap * D;
    const int units = (n + 63) / 64;
    // stage u: row r of unit u is token idx[64u + r] (zero rows past the list or outside 0 .. T-1)
    auto issue = [&](int u) {
        if (u < units) {
            const uint32_t st = smem_u32(ring + (size_t)(u % kTdStages) * kStage);
            for (int e = tid; e < 64 * NB * 8; e += kTdWarps * 32) {
                const int r = e / (NB * 8), bi = (e / 8) % NB, ch = e % 8;
                const int i = 64 * u + r;
                const int tok = i < n ? idx[i] : -1;
                const bool ok = tok >= 0 && tok < T;
                const size_t off = (size_t)(ok ? tok : 0) * D + bi * 64 + ch * 8;
                const uint32_t d = st + (uint32_t)(bi * kTdBox + r * 128 + ((ch ^ (r & 7)) << 4));
                cp_async16(d, kc + off, ok);
                cp_async16(d + NB * kTdBox, vc + off, ok);
            }
        }
        cp_async_commit();
    };
    uint32_t qa[D / 16][2];
    load_q_frag<D>(qa, reinterpret_cast<const uint32_t*>(reinterpret_cast<const uint16_t*>(L.q[layer]) +
                                                         ((size_t)b * a.Hq + (size_t)kvh * a.G + g) * D),
                   g < a.G, tq);
    AttnState<D> as;
    as.reset();
    issue(0);
    issue(1);
    for (int u = 0; u < units; ++u) {
        issue(u + 2);
        cp_async_wait<2>();
        __syncthreads();
        uint8_t* kst = ring + (size_t)(u % kTdStages) * kStage;
        const int nvalid = min(64, n - 64 * u);
        if (16 * w < nvalid) attend16<D>(kst, kst + NB * kTdBox, kTdBox, 16 * w, nvalid, qa, a.scale_log2, as, lane);
        __syncthreads();  // the stage is refilled by the next iteration's issue
    }
    cp_async_wait<0>();
    // the four warps' states into O and LSE
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        as.lsum[0] += __shfl_xor_sync(0xffffffffu, as.lsum[0], off);
        as.lsum[1] += __shfl_xor_sync(0xffffffffu, as.lsum[1], off);
    }
    float* mM = merge;                           // [warp][kMaxG]
    float* mL = merge + kTdWarps * kMaxG;        // [warp][kMaxG]
    float* mA = merge + 2 * kTdWarps * kMaxG;    // [warp][G][D]
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
    for (int mt = 0; mt < D / 16; ++mt) {
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
    __syncthreads();
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(L.out[layer]) + ((size_t)b * a.Hq + (size_t)kvh * a.G) * D;
    float* lse = L.lse[layer] ? L.lse[layer] + (size_t)b * a.Hq + (size_t)kvh * a.G : nullptr;
    for (int e = tid; e < a.G * D; e += kTdWarps * 32) {
        const int h = e / D, dd = e - h * D;
        float M = -INFINITY;
#pragma unroll
        for (int ww = 0; ww < kTdWarps; ++ww) M = fmaxf(M, mM[ww * kMaxG + h]);
        float num = 0.f, den = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int ww = 0; ww < kTdWarps; ++ww) {
                const float f = exp2f(mM[ww * kMaxG + h] - M);
                num = fmaf(f, mA[(ww * a.G + h) * D + dd], num);
                den = fmaf(f, mL[ww * kMaxG + h], den);
            }
        }
        out[h * D + dd] = __float2bfloat16_rn(den > 0.f ? num / den : 0.f);
        if (dd == 0 && lse) lse[h] = den > 0.f ? (M + log2f(den)) * 0.69314718055994531f : -INFINITY;
    }
}

}  // namespace

size_t token_topk_smem_bytes(int64_t T_cap, int64_t nstat, int Gp) {
    const size_t bytes = (size_t)((T_cap + 3) & ~int64_t(3)) * 4 + (size_t)nstat * Gp * 4;
    const size_t limit = 227 * 1024 - sizeof(TopkSmem) - 256;
    return bytes <= limit ? bytes : 0;
}

size_t token_decode_smem_bytes(int D, int G) {
    return 1024 + (size_t)kTdStages * 2 * (D / 64) * kTdBox + (size_t)(2 * kTdWarps * kMaxG + kTdWarps * G * D) * 4;
}

cudaError_t launch_token_topk(const TokenArgs& a, int Gp, size_t smem, cudaStream_t st) {
    if (a.pairs <= 0) return cudaSuccess;
    switch (Gp) {
        case 1: {
            cudaError_t e = ensure_smem<token_topk_kernel<1>>(smem);
            return e != cudaSuccess ? e : launch_pdl(token_topk_kernel<1>, dim3((unsigned)a.pairs), dim3(kTkThreads), smem, st, a);
        }
        case 2: {
            cudaError_t e = ensure_smem<token_topk_kernel<2>>(smem);
            return e != cudaSuccess ? e : launch_pdl(token_topk_kernel<2>, dim3((unsigned)a.pairs), dim3(kTkThreads), smem, st, a);
        }
        case 4: {
            cudaError_t e = ensure_smem<token_topk_kernel<4>>(smem);
            return e != cudaSuccess ? e : launch_pdl(token_topk_kernel<4>, dim3((unsigned)a.pairs), dim3(kTkThreads), smem, st, a);
        }
        default: {
            cudaError_t e = ensure_smem<token_topk_kernel<8>>(smem);
            return e != cudaSuccess ? e : launch_pdl(token_topk_kernel<8>, dim3((unsigned)a.pairs), dim3(kTkThreads), smem, st, a);
        }
    }
}

cudaError_t launch_token_decode(const TokenArgs& a, const TokenLayers& L, int layers, int D, cudaStream_t st) {
    const int64_t ctas = (int64_t)layers * a.pairs;
    if (ctas <= 0) return cudaSuccess;
    const size_t smem = token_decode_smem_bytes(D, a.G);
    if (D == 128) {
        cudaError_t e = ensure_smem<token_decode_kernel<128>>(smem);
        return e != cudaSuccess ? e : launch_pdl(token_decode_kernel<128>, dim3((unsigned)ctas), dim3(kTdWarps * 32), smem, st, a, L);
    }
    cudaError_t e = ensure_smem<token_decode_kernel<64>>(smem);
    return e != cudaSuccess ? e : launch_pdl(token_decode_kernel<64>, dim3((unsigned)ctas), dim3(kTdWarps * 32), smem, st, a, L);
}

}  // namespace bsa
