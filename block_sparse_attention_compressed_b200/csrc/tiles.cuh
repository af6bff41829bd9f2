// Per-warp tensor-core tiles shared by the scoring, sparse-attention and fused step kernels: the
// contraction of a 64-row chunk of compressed keys with the group's query heads (page "SparDA:
// Sparse Decoupled Attention for Efficient Long-Context LLM Inference", Indexer Training, Eq. 6:
// the logits q_h . K~_j), and the online-softmax update of one warp's 16 tokens of a K/V stage
// (SparDA Architecture, Eq. 5). Operands sit in shared memory as 2-D TMA boxes of 64 bf16 columns
// (128-byte rows, 128-byte swizzle); the G heads of a group, padded to 8, are the mma N dimension.
#pragma once

#include "bsa_internal.cuh"

namespace bsa {
namespace {

// q (or a Forecast vector) of head g as the mma B operand: lane (g, tq) holds d = 16ks + 2tq (+1)
// and 16ks + 8 + 2tq (+9). `row` points at head g's D bf16 values; `valid` is false for padding
// heads (their fragments are zero).
template <int D>
__device__ __forceinline__ void load_q_frag(uint32_t (&qf)[D / 16][2], const uint32_t* row, bool valid,
                                            int tq) {
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        qf[ks][0] = valid ? row[8 * ks + tq] : 0u;
        qf[ks][1] = valid ? row[8 * ks + 4 + tq] : 0u;
    }
}

// c[r] = rows 16r..16r+15 of a 64-row chunk times the B operand: lane (g, tq) receives rows
// 16r + g (c[r][0..1]) and 16r + g + 8 (c[r][2..3]) for heads 2tq, 2tq + 1. The chunk is D / 64
// boxes of 64 rows x 128 bytes; the four row groups run as independent mma chains.
template <int D>
__device__ __forceinline__ void score_chunk(const uint8_t* cst, const uint32_t (&qf)[D / 16][2],
                                            float (&c)[4][4], int lane) {
    constexpr uint32_t box_bytes = 64u * 128u;
    const int mi = lane >> 3, ri = lane & 7;
#pragma unroll
    for (int r = 0; r < 4; ++r) c[r][0] = c[r][1] = c[r][2] = c[r][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {  // four independent 16-row groups
            const int row = 16 * r + ri + 8 * (mi & 1);
            const int ch = (ks & 3) * 2 + (mi >> 1);
            uint32_t af[4];
            ldmatrix_x4(af, smem_u32(cst + (ks >> 2) * box_bytes + row * 128 + ((ch ^ (row & 7)) << 4)));
            mma_bf16_16816(c[r], af[0], af[1], af[2], af[3], qf[ks][0], qf[ks][1]);
        }
    }
}

// One warp's online-softmax state over the tokens it has attended: per head pair (2tq, 2tq + 1)
// the running max m and denominator lsum (log2 domain), and the numerators O^T (d = 16mt + g,
// 16mt + g + 8 in acc[mt][0..1] / acc[mt][2..3]).
template <int D>
struct AttnState {
    float m[2], lsum[2];
    float acc[D / 16][4];
    __device__ __forceinline__ void reset() {
        m[0] = m[1] = -INFINITY;
        lsum[0] = lsum[1] = 0.f;
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt) acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
    }
};

// The bf16 hi + lo parts of a warp's probabilities P^T (16 tokens x the heads), as mma B operands.
struct PFrag {
    uint32_t bh0, bh1, bl0, bl1;
};

// K half of the online-softmax update for tokens r0..r0+15 (K rows at kst, D / 64 boxes of
// box_bytes; the first nvalid - r0 tokens are below the sequence length): S^T = K q^T on the tensor
// cores, the running max / denominator and the numerators' rescale in fp32 / exp2, and P^T for the
// V half (from the S^T accumulators by movmatrix, split as bf16 hi + lo so the products keep
// about 16 significant bits).
template <int D>
__device__ __forceinline__ PFrag attn_scores16(const uint8_t* kst, uint32_t box_bytes, int r0, int nvalid,
                                               const uint32_t (&qf)[D / 16][2], float scale_log2,
                                               AttnState<D>& s, int lane) {
    constexpr int KS = D / 16, MT = D / 16;
    const int mi = lane >> 3, ri = lane & 7, g = lane >> 2;
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
        const int row = r0 + ri + 8 * (mi & 1);
        const int ch = (ks & 3) * 2 + (mi >> 1);
        uint32_t af[4];
        ldmatrix_x4(af, smem_u32(kst + (ks >> 2) * box_bytes + row * 128 + ((ch ^ (row & 7)) << 4)));
        mma_bf16_16816(c, af[0], af[1], af[2], af[3], qf[ks][0], qf[ks][1]);
    }
    const float sl = scale_log2;
    const bool va = r0 + g < nvalid, vb = r0 + g + 8 < nvalid;
    const float x0 = va ? c[0] * sl : -INFINITY, x1 = va ? c[1] * sl : -INFINITY;
    const float x2 = vb ? c[2] * sl : -INFINITY, x3 = vb ? c[3] * sl : -INFINITY;
    float t0 = fmaxf(x0, x2), t1 = fmaxf(x1, x3);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, off));
        t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, off));
    }
    const float mn0 = fmaxf(s.m[0], t0), mn1 = fmaxf(s.m[1], t1);
    const float al0 = mn0 == -INFINITY ? 1.f : exp2f(s.m[0] - mn0);
    const float al1 = mn1 == -INFINITY ? 1.f : exp2f(s.m[1] - mn1);
    const float ref0 = mn0 == -INFINITY ? 0.f : mn0, ref1 = mn1 == -INFINITY ? 0.f : mn1;
    const float p0 = exp2f(x0 - ref0), p2 = exp2f(x2 - ref0);
    const float p1 = exp2f(x1 - ref1), p3 = exp2f(x3 - ref1);
    s.m[0] = mn0;
    s.m[1] = mn1;
    s.lsum[0] = s.lsum[0] * al0 + (p0 + p2);
    s.lsum[1] = s.lsum[1] * al1 + (p1 + p3);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        s.acc[mt][0] *= al0;
        s.acc[mt][1] *= al1;
        s.acc[mt][2] *= al0;
        s.acc[mt][3] *= al1;
    }
    // P^T operand from the S^T accumulators (8x8 transposes), hi + lo bf16 parts
    const uint32_t hi0 = pack_bf16x2(p0, p1), hi1 = pack_bf16x2(p2, p3);
    const uint32_t lo0 = pack_bf16x2(p0 - bf16_lo(hi0), p1 - bf16_hi(hi0));
    const uint32_t lo1 = pack_bf16x2(p2 - bf16_lo(hi1), p3 - bf16_hi(hi1));
    PFrag pf;
    pf.bh0 = movmatrix_trans(hi0);
    pf.bh1 = movmatrix_trans(hi1);
    pf.bl0 = movmatrix_trans(lo0);
    pf.bl1 = movmatrix_trans(lo1);
    return pf;
}

// V half: O^T += V^T P^T for tokens r0..r0+15 (V rows at vst), V^T fragments straight from the
// swizzled stage (ldmatrix.trans). V rows at or past nvalid are zeroed in shared memory first
// (they may hold anything, and 0 * NaN would poison the sums).
template <int D>
__device__ __forceinline__ void attn_accum16(uint8_t* vst, uint32_t box_bytes, int r0, int nvalid, const PFrag& pf,
                                             AttnState<D>& s, int lane) {
    constexpr int NB = D / 64, MT = D / 16;
    const int mi = lane >> 3, ri = lane & 7;
    if (r0 + 16 > nvalid) {
        for (int e = lane; e < 16 * NB * 8; e += 32) {
            const int row = r0 + e / (NB * 8), bi = (e / 8) % NB, ch = e % 8;
            if (row >= nvalid)
                *reinterpret_cast<uint4*>(vst + bi * box_bytes + row * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
        __syncwarp();
    }
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
        const int row = r0 + ri + 8 * (mi >> 1);
        const int ch = 2 * mt + (mi & 1);
        uint32_t af[4];
        ldmatrix_x4_trans(af, smem_u32(vst + (ch >> 3) * box_bytes + row * 128 + (((ch & 7) ^ (row & 7)) << 4)));
        mma_bf16_16816(s.acc[mt], af[0], af[1], af[2], af[3], pf.bh0, pf.bh1);
        mma_bf16_16816(s.acc[mt], af[0], af[1], af[2], af[3], pf.bl0, pf.bl1);
    }
}

// Both halves for a stage holding K and V of the same tokens.
template <int D>
__device__ __forceinline__ void attend16(uint8_t* kst, uint8_t* vst, uint32_t box_bytes, int r0, int nvalid,
                                         const uint32_t (&qf)[D / 16][2], float scale_log2,
                                         AttnState<D>& s, int lane) {
    const PFrag pf = attn_scores16<D>(kst, box_bytes, r0, nvalid, qf, scale_log2, s, lane);
    attn_accum16<D>(vst, box_bytes, r0, nvalid, pf, s, lane);
}

}  // namespace
}  // namespace bsa
