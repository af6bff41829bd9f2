// Sparse attention over the selected blocks (page "SparDA: Sparse Decoupled Attention for Efficient
// Long-Context LLM Inference", SparDA Architecture, Eq. 5: O = Attn(Q, K[B], V[B])), with the
// shared-index mode of the pages "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (first abstract) and "CoSA: Accelerating Long-Context Inference via Proxy-Kernel Co-Designed
// Sparse Attention" (second abstract): several layers attended with one layer's selection.
//
// Split-KV flash decoding. grid = layers * pairs * splits CTAs; CTA `split` of a (layer, pair)
// owns blocks [split*bpc, (split+1)*bpc) of the pair's selection, its warps take those blocks
// round-robin and run an online softmax (fp32, exp2 domain) over 16-token sub-tiles. The warps'
// partial states are merged in shared memory and written to the workspace; the last CTA of the
// (layer, pair) to finish (completion counter, no waiting) combines all splits into O and LSE.
//
// bf16 path, per 16-token sub-tile, all on the tensor cores with mma.m16n8k16:
//   S^T[tok][head] = K_tile[tok][:] . q^T   (tokens are M, the G heads padded to 8 are N); each
//       lane feeds the A operand from its own 16-byte global loads, q permuted to match;
//   O^T[d][head] += V_tile^T[d][tok] . P^T[tok][head]   (d is M, tokens are K): the V operand is
//       built from two token rows per register with PRMT, P^T comes from the S^T accumulators via
//       movmatrix.trans. P is split as P_hi + P_lo (both bf16) so that the products keep ~16
//       significant bits of the fp32 probabilities.
// K and V rows at or past the sequence length are never loaded (zero fill) and masked to -inf.
#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int kDecodeThreads = kDecodeWarps * 32;

// Shared-memory image of the warps' states, merged by the whole CTA.
template <int D>
struct DecodeSmem {
    float m[kDecodeWarps][kMaxG];
    float l[kDecodeWarps][kMaxG];
    float acc[kDecodeWarps][kMaxG][D];
};

template <typename T>
__device__ __forceinline__ void store_out(T* p, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* p, float v) {
    *p = __float2bfloat16_rn(v);
}

// CTA merge of the warp states, split partial write, and the cross-split combine by the last CTA.
template <typename T, int D>
__device__ void finish_split(const DecodeArgs& a, int layer, int pair, int lp, int split,
                             DecodeSmem<D>& sm) {
    __shared__ int s_last;
    __syncthreads();
    const int G = a.G, NT = blockDim.x;
    float2* pml = a.part_ml + ((size_t)lp * a.splits + split) * a.Gp;
    float* pacc = a.part_acc + ((size_t)lp * a.splits + split) * a.Gp * D;
    for (int e = threadIdx.x; e < G * D; e += NT) {
        const int h = e / D, dd = e - h * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, sm.m[w][h]);
        float num = 0.f, den = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kDecodeWarps; ++w) {
                const float f = exp2f(sm.m[w][h] - M);
                num = fmaf(f, sm.acc[w][h][dd], num);
                den = fmaf(f, sm.l[w][h], den);
            }
        }
        pacc[h * D + dd] = num;
        if (dd == 0) pml[h] = make_float2(M, den);
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int prev = atomicAdd(a.cnt + lp, 1);
        s_last = (prev == a.splits - 1);
        if (s_last) atomicExch(a.cnt + lp, 0);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // Combine the splits: per head the global max M and denominator, per split a scale factor
    // exp2(m_s - M) (shared memory), then every (head, d) element sums its scaled numerators with
    // the loads of kU splits in flight.
    __shared__ float2 s_ml[kMaxCombineSlots];
    __shared__ float s_M[kMaxG], s_den[kMaxG];
    const int S = a.splits;
    const float2* ml0 = a.part_ml + (size_t)lp * S * a.Gp;
    const float* acc0 = a.part_acc + (size_t)lp * S * a.Gp * D;
    for (int e = threadIdx.x; e < S * a.Gp; e += NT) s_ml[e] = ld_cg(ml0 + e);  // one round
    __syncthreads();
    if (threadIdx.x < G) {
        const int h = threadIdx.x;
        float M = -INFINITY;
        for (int s2 = 0; s2 < S; ++s2) M = fmaxf(M, s_ml[s2 * a.Gp + h].x);
        float den = 0.f;
        for (int s2 = 0; s2 < S; ++s2) {
            const float2 ml = s_ml[s2 * a.Gp + h];
            const float f = M == -INFINITY ? 0.f : exp2f(ml.x - M);
            den = fmaf(f, ml.y, den);
            s_ml[s2 * a.Gp + h].x = f;  // becomes the split's scale factor
        }
        s_M[h] = M;
        s_den[h] = den;
    }
    __syncthreads();
    const int b = pair / a.Hkv, kvh = pair - b * a.Hkv;
    T* out = reinterpret_cast<T*>(a.out[layer]) + ((size_t)b * a.Hq + (size_t)kvh * G) * D;
    float* lse = a.lse[layer] ? a.lse[layer] + (size_t)b * a.Hq + (size_t)kvh * G : nullptr;
    constexpr int kU = 8;
    for (int e = threadIdx.x; e < G * D; e += NT) {
        const int h = e / D, dd = e - h * D;
        float num = 0.f;
        for (int s0 = 0; s0 < S; s0 += kU) {
            float v[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u)
                v[u] = s0 + u < S ? ld_cg(acc0 + ((size_t)(s0 + u) * a.Gp + h) * D + dd) : 0.f;
#pragma unroll
            for (int u = 0; u < kU; ++u)
                if (s0 + u < S) num = fmaf(s_ml[(s0 + u) * a.Gp + h].x, v[u], num);
        }
        const float den = s_den[h];
        store_out<T>(out + h * D + dd, den > 0.f ? num / den : 0.f);
        if (dd == 0 && lse)
            lse[h] = den > 0.f ? (s_M[h] + log2f(den)) * 0.69314718055994531f : -INFINITY;
    }
}

// Which blocks this CTA owns, and the sequence facts every warp needs.
struct SplitInfo {
    int64_t T, nb;
    int beg, end;
    bool ok;
};

__device__ __forceinline__ SplitInfo split_info(const DecodeArgs& a, int layer, int pair, int split) {
    SplitInfo si;
    const int b = pair / a.Hkv;
    si.T = a.seq_lens[b];
    si.ok = si.T >= 0 && si.T <= a.T_cap;
    const bool reporter = layer == 0 && split == 0 && threadIdx.x == 0;
    if (!si.ok && reporter && pair % a.Hkv == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_SEQ_LEN);
    int ns = a.n_sel[pair];
    if (ns < 0 || ns > a.sel_cap) {
        if (reporter) atomicOr(a.err, (uint32_t)BSA_DEVERR_N_SEL);
        ns = ns < 0 ? 0 : a.sel_cap;
    }
    if (!si.ok) ns = 0;
    si.nb = si.ok ? (si.T + a.BS - 1) / a.BS : 0;
    si.beg = split * a.bpc;
    si.end = min(si.beg + a.bpc, ns);
    return si;
}

// -------------------------------------------------------------------------------------- bf16 path
template <int D>
struct KVTile {
    static constexpr int NI = D / 32;   // key chunks per lane per row (chunks tq + 4i)
    static constexpr int NCV = D / 64;  // value chunks per lane per token (chunks g, g + 8)
    uint4 ka[NI], kb[NI];               // key rows base+g, base+g+8
    uint4 v[4][NCV];                    // value rows base+2tq, +2tq+1, +2tq+8, +2tq+9
};

template <int D>
__device__ __forceinline__ void load_kvtile(KVTile<D>& t, const uint16_t* kp, const uint16_t* vp,
                                            int64_t base, int64_t T, int g, int tq) {
    const int64_t ra = base + g, rb = base + g + 8;
#pragma unroll
    for (int i = 0; i < KVTile<D>::NI; ++i) {
        const int col = (tq + 4 * i) * 8;
        t.ka[i] = ra < T ? ld_stream(kp + ra * D + col) : make_uint4(0, 0, 0, 0);
        t.kb[i] = rb < T ? ld_stream(kp + rb * D + col) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int64_t row = base + 2 * tq + (r & 1) + (r >> 1) * 8;
#pragma unroll
        for (int i = 0; i < KVTile<D>::NCV; ++i) {
            const int col = (g + 8 * i) * 8;
            t.v[r][i] = row < T ? ld_stream(vp + row * D + col) : make_uint4(0, 0, 0, 0);
        }
    }
}

template <int D>
__device__ __forceinline__ void attend_tile(const KVTile<D>& t, const uint32_t (&qf)[D / 32][4],
                                            int64_t base, int64_t T, float sl, int g, float (&m)[2],
                                            float (&lsum)[2], float (&acc)[D / 16][4]) {
    constexpr int NI = D / 32, MT = D / 16;
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < NI; ++i)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
            mma_bf16_16816(c, u4_get(t.ka[i], 2 * hh), u4_get(t.kb[i], 2 * hh),
                           u4_get(t.ka[i], 2 * hh + 1), u4_get(t.kb[i], 2 * hh + 1),
                           qf[i][2 * hh], qf[i][2 * hh + 1]);
    const bool va = base + g < T, vb = base + g + 8 < T;
    const float x0 = va ? c[0] * sl : -INFINITY, x1 = va ? c[1] * sl : -INFINITY;
    const float x2 = vb ? c[2] * sl : -INFINITY, x3 = vb ? c[3] * sl : -INFINITY;
    float t0 = fmaxf(x0, x2), t1 = fmaxf(x1, x3);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, off));
        t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, off));
    }
    const float mn0 = fmaxf(m[0], t0), mn1 = fmaxf(m[1], t1);
    const float al0 = mn0 == -INFINITY ? 1.f : exp2f(m[0] - mn0);
    const float al1 = mn1 == -INFINITY ? 1.f : exp2f(m[1] - mn1);
    const float ref0 = mn0 == -INFINITY ? 0.f : mn0, ref1 = mn1 == -INFINITY ? 0.f : mn1;
    const float p0 = exp2f(x0 - ref0), p2 = exp2f(x2 - ref0);
    const float p1 = exp2f(x1 - ref1), p3 = exp2f(x3 - ref1);
    m[0] = mn0;
    m[1] = mn1;
    lsum[0] = lsum[0] * al0 + (p0 + p2);
    lsum[1] = lsum[1] * al1 + (p1 + p3);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        acc[mt][0] *= al0;
        acc[mt][1] *= al1;
        acc[mt][2] *= al0;
        acc[mt][3] *= al1;
    }
    // P^T operand: rows of the S^T accumulator are tokens, columns heads; transpose 8x8 pieces
    const uint32_t hi0 = pack_bf16x2(p0, p1), hi1 = pack_bf16x2(p2, p3);
    const uint32_t lo0 = pack_bf16x2(p0 - bf16_lo(hi0), p1 - bf16_hi(hi0));
    const uint32_t lo1 = pack_bf16x2(p2 - bf16_lo(hi1), p3 - bf16_hi(hi1));
    const uint32_t bh0 = movmatrix_trans(hi0), bh1 = movmatrix_trans(hi1);
    const uint32_t bl0 = movmatrix_trans(lo0), bl1 = movmatrix_trans(lo1);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int ci = mt / 4, comp = mt % 4;
        const uint32_t r0 = u4_get(t.v[0][ci], comp), r1 = u4_get(t.v[1][ci], comp);
        const uint32_t r2 = u4_get(t.v[2][ci], comp), r3 = u4_get(t.v[3][ci], comp);
        const uint32_t a0 = prmt(r0, r1, 0x5410u), a1 = prmt(r0, r1, 0x7632u);
        const uint32_t a2 = prmt(r2, r3, 0x5410u), a3 = prmt(r2, r3, 0x7632u);
        mma_bf16_16816(acc[mt], a0, a1, a2, a3, bh0, bh1);
        mma_bf16_16816(acc[mt], a0, a1, a2, a3, bl0, bl1);
    }
}

template <int D>
__global__ void __launch_bounds__(kDecodeThreads, 2) decode_bf16_kernel(DecodeArgs a) {
    __shared__ DecodeSmem<D> sm;
    constexpr int NI = D / 32, MT = D / 16;
    const int split = blockIdx.x % a.splits, lp = blockIdx.x / a.splits;
    const int layer = lp / a.pairs, pair = lp - layer * a.pairs;
    const int b = pair / a.Hkv, kvh = pair - b * a.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;

    uint32_t qf[NI][4];
    {
        const uint16_t* qh = reinterpret_cast<const uint16_t*>(a.q[layer]) +
                             ((size_t)b * a.Hq + (size_t)kvh * a.G + g) * D;
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
    const SplitInfo si = split_info(a, layer, pair, split);
    const uint16_t* kp = reinterpret_cast<const uint16_t*>(a.k[layer]) + (size_t)pair * a.T_cap * D;
    const uint16_t* vp = reinterpret_cast<const uint16_t*>(a.v[layer]) + (size_t)pair * a.T_cap * D;
    const int32_t* ip = a.block_idx + (size_t)pair * a.sel_cap;

    float m[2] = {-INFINITY, -INFINITY}, lsum[2] = {0.f, 0.f};
    float acc[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;

    // The warp's work: its blocks (round-robin within the split) x 16-token sub-tiles, walked
    // with the next sub-tile's loads in flight while the current one is computed.
    const int sub_per_block = a.BS / 16;
    int my_blk = -1;  // lane j holds the warp's j-th block index
    {
        const int i = si.beg + warp + lane * kDecodeWarps;
        if (lane * kDecodeWarps + warp < a.bpc && i < si.end) {
            const int v = ip[i];
            if (v >= 0 && v < si.nb) my_blk = v;
            else if (v >= si.nb) atomicOr(a.err, (uint32_t)BSA_DEVERR_BLOCK_IDX);
        }
    }
    const int n_units = ((a.bpc + kDecodeWarps - 1) / kDecodeWarps) * sub_per_block;
    auto unit_base = [&](int u) -> int64_t {  // token base of a unit, or -1 when it has no token
        const int blk = __shfl_sync(0xffffffffu, my_blk, u / sub_per_block);
        if (blk < 0) return -1;
        const int64_t base = (int64_t)blk * a.BS + (u % sub_per_block) * 16;
        return base < si.T ? base : -1;
    };
    auto next_unit = [&](int u, int64_t& base) -> int {
        for (++u; u < n_units; ++u) {
            base = unit_base(u);
            if (base >= 0) return u;
        }
        return n_units;
    };
    // Two tile buffers in ping-pong (no register copy waits on a pending load).
    KVTile<D> ta, tb;
    int64_t base_a = -1, base_b = -1;
    int ua = next_unit(-1, base_a);
    if (ua < n_units) load_kvtile<D>(ta, kp, vp, base_a, si.T, g, tq);
    while (ua < n_units) {
        const int ub = next_unit(ua, base_b);
        if (ub < n_units) load_kvtile<D>(tb, kp, vp, base_b, si.T, g, tq);
        attend_tile<D>(ta, qf, base_a, si.T, a.scale_log2, g, m, lsum, acc);
        if (ub >= n_units) break;
        ua = next_unit(ub, base_a);
        if (ua < n_units) load_kvtile<D>(ta, kp, vp, base_a, si.T, g, tq);
        attend_tile<D>(tb, qf, base_b, si.T, a.scale_log2, g, m, lsum, acc);
    }

#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        lsum[0] += __shfl_xor_sync(0xffffffffu, lsum[0], off);
        lsum[1] += __shfl_xor_sync(0xffffffffu, lsum[1], off);
    }
    const int h0 = 2 * tq, h1 = 2 * tq + 1;
    if (g == 0) {
        if (h0 < a.G) {
            sm.m[warp][h0] = m[0];
            sm.l[warp][h0] = lsum[0];
        }
        if (h1 < a.G) {
            sm.m[warp][h1] = m[1];
            sm.l[warp][h1] = lsum[1];
        }
    }
    // accumulator (mt, row g / g+8) <-> d = (mt/4)*64 + 8g + 2(mt%4) + {0, 1}
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int d0 = (mt / 4) * 64 + 8 * g + 2 * (mt % 4);
        if (h0 < a.G) {
            sm.acc[warp][h0][d0] = acc[mt][0];
            sm.acc[warp][h0][d0 + 1] = acc[mt][2];
        }
        if (h1 < a.G) {
            sm.acc[warp][h1][d0] = acc[mt][1];
            sm.acc[warp][h1][d0 + 1] = acc[mt][3];
        }
    }
    finish_split<__nv_bfloat16, D>(a, layer, pair, lp, split, sm);
}

// -------------------------------------------------------------------------------------- fp32 path
// One token at a time per warp; lanes split d, warp reductions form the dot products.
template <int D>
__global__ void __launch_bounds__(kDecodeThreads) decode_f32_kernel(DecodeArgs a) {
    __shared__ DecodeSmem<D> sm;
    constexpr int E = D / 32;
    const int split = blockIdx.x % a.splits, lp = blockIdx.x / a.splits;
    const int layer = lp / a.pairs, pair = lp - layer * a.pairs;
    const int b = pair / a.Hkv, kvh = pair - b * a.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    float qv[kMaxG][E];
    const float* qb = reinterpret_cast<const float*>(a.q[layer]) + ((size_t)b * a.Hq + (size_t)kvh * a.G) * D;
#pragma unroll
    for (int h = 0; h < kMaxG; ++h)
#pragma unroll
        for (int e = 0; e < E; ++e) qv[h][e] = h < a.G ? qb[h * D + lane * E + e] : 0.f;
    pdl_trigger();
    pdl_wait();
    const SplitInfo si = split_info(a, layer, pair, split);
    const float* kp = reinterpret_cast<const float*>(a.k[layer]) + (size_t)pair * a.T_cap * D;
    const float* vp = reinterpret_cast<const float*>(a.v[layer]) + (size_t)pair * a.T_cap * D;
    const int32_t* ip = a.block_idx + (size_t)pair * a.sel_cap;

    float m[kMaxG], l[kMaxG], acc[kMaxG][E];
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[h][e] = 0.f;
    }
    for (int i = si.beg + warp; i < si.end; i += kDecodeWarps) {
        const int blk = ip[i];
        if (blk < 0) continue;
        if (blk >= si.nb) {
            if (lane == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_BLOCK_IDX);
            continue;
        }
        const int64_t t0 = (int64_t)blk * a.BS, t1 = min(t0 + a.BS, si.T);
        for (int64_t tok = t0; tok < t1; ++tok) {
            float kv[E], vv[E];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                kv[e] = __ldg(kp + tok * D + lane * E + e);
                vv[e] = __ldg(vp + tok * D + lane * E + e);
            }
#pragma unroll
            for (int h = 0; h < kMaxG; ++h) {
                if (h >= a.G) break;
                float p = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) p = fmaf(qv[h][e], kv[e], p);
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
                const float x = p * a.scale_log2;
                const float mn = fmaxf(m[h], x);
                const float al = exp2f(m[h] - mn);
                const float w = exp2f(x - mn);
                l[h] = l[h] * al + w;
#pragma unroll
                for (int e = 0; e < E; ++e) acc[h][e] = fmaf(w, vv[e], acc[h][e] * al);
                m[h] = mn;
            }
        }
    }
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
        if (h < a.G) {
            if (lane == 0) {
                sm.m[warp][h] = m[h];
                sm.l[warp][h] = l[h];
            }
#pragma unroll
            for (int e = 0; e < E; ++e) sm.acc[warp][h][lane * E + e] = acc[h][e];
        }
    }
    finish_split<float, D>(a, layer, pair, lp, split, sm);
}

template <typename K>
cudaError_t launch_decode_k(K kernel, const Plan& p, const DecodeArgs& a, int layers, cudaStream_t st) {
    const int64_t grid = (int64_t)layers * p.pairs * p.dec_splits;
    if (grid <= 0) return cudaSuccess;
    if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
    return launch_pdl(kernel, dim3((unsigned)grid), dim3(kDecodeThreads), 0, st, a);
}

}  // namespace

cudaError_t launch_decode(const Plan& p, const DecodeArgs& a, int layers, cudaStream_t st) {
    if (p.dtype == BSA_BF16)
        return p.D == 128 ? launch_decode_k(decode_bf16_kernel<128>, p, a, layers, st)
                          : launch_decode_k(decode_bf16_kernel<64>, p, a, layers, st);
    return p.D == 128 ? launch_decode_k(decode_f32_kernel<128>, p, a, layers, st)
                      : launch_decode_k(decode_f32_kernel<64>, p, a, layers, st);
}

}  // namespace bsa
