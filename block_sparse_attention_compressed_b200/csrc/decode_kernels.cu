// Sparse attention over the selected blocks (page "SparDA: Sparse Decoupled Attention for Efficient
// Long-Context LLM Inference", SparDA Architecture, Eq. 5: O = Attn(Q, K[B], V[B])), with the
// shared-index mode of the pages "HySparse2: Hybrid Sparse Attention with Two-Level KV Sharing"
// (first abstract) and "CoSA: Accelerating Long-Context Inference via Proxy-Kernel Co-Designed
// Sparse Attention" (second abstract): several layers attended with one layer's selection.
//
// Split-KV flash decoding: partial softmax states (fp32, exp2 domain; per head the max m, the
// denominator l and the numerators acc) over disjoint parts of a pair's selected blocks, merged
// into O and LSE at the end.
//
// bf16 path (TMA pipeline, persistent): the layers * pairs * SEL_cap block slots are shared evenly
// by the CTAs; a (layer, pair) run inside a CTA's share is a segment with one partial. One producer
// warp walks the share and issues 2-D TMA tensor copies (128-byte swizzle, L2 evict-first) of each
// 16..64-token stage of K and V into a ring of shared-memory stages, completing on per-stage
// mbarriers; four consumer warps each take 16 tokens of a stage and run, on the tensor cores
// (mma.m16n8k16, operands from ldmatrix):
//   S^T[tok][head] = K[tok][:] . q^T          (tokens are M, the G heads padded to 8 are N)
//   O^T[d][head] += V^T[d][tok] . P^T[tok][head]  (d is M; V^T via ldmatrix.trans; P^T from the
//       S^T accumulators via movmatrix.trans, split as bf16 hi + lo so the products keep ~16
//       significant bits of the fp32 probabilities)
// then release the stage. Bytes in flight are set by the ring size, not by registers. Tokens at or
// past the sequence length are masked to -inf and their V rows zeroed in shared memory. At the end
// of a segment the warps merge their states and write its partial; combine_kernel merges each
// (layer, pair)'s partials in segment order once the grid has finished.
// fp32 path: grid = layers * pairs * splits CTAs, a split of bpc blocks each; the warps take groups
// of consecutive tokens in turn (FMA dot products, warp reductions), merge in shared memory, and
// the last split of a (layer, pair) to finish (completion counter, no waiting) combines them.
#include "bsa_internal.cuh"
#include "tiles.cuh"

namespace bsa {
namespace {

constexpr int kDecodeThreads = kDecodeWarps * 32;

// Shared-memory image of the warps' states: m and l per (warp, head), numerators per
// (warp, head, d) packed for the problem's G heads.
struct MergeView {
    float* m;    // [kDecodeWarps][kMaxG]
    float* l;    // [kDecodeWarps][kMaxG]
    float* acc;  // [kDecodeWarps][G][D]
    __device__ __forceinline__ float& M(int w, int h) const { return m[w * kMaxG + h]; }
    __device__ __forceinline__ float& L(int w, int h) const { return l[w * kMaxG + h]; }
};
__host__ __device__ constexpr size_t merge_bytes(int G, int D) {
    return sizeof(float) * (2 * kDecodeWarps * kMaxG + (size_t)kDecodeWarps * G * D);
}

template <typename T>
__device__ __forceinline__ void store_out(T* p, float v);
template <>
__device__ __forceinline__ void store_out<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16* p, float v) {
    *p = __float2bfloat16_rn(v);
}

// The threads that merge a split: the whole CTA (bar_id 0, __syncthreads) or a named-barrier
// group of `nthreads` threads (the consumer warps of the persistent kernel).
struct Group {
    int tid, nthreads, bar_id;
    __device__ __forceinline__ void sync() const {
        if (bar_id == 0) __syncthreads();
        else asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(nthreads) : "memory");
    }
};

template <typename T, int D>
__device__ void combine_partials(const DecodeArgs& a, int layer, int pair, int lp, int S,
                                 float2* s_ml, const Group gp);

// Merge of the warp states, split partial write, and the cross-split combine by the last split of
// the (layer, pair) to finish (fp32 path).
template <typename T, int D>
__device__ void finish_split(const DecodeArgs& a, int layer, int pair, int lp, int slot, int nslots,
                             const MergeView sm, float2* s_ml /* nslots * Gp */, const Group gp) {
    __shared__ int s_last;
    gp.sync();
    const int G = a.G, NT = gp.nthreads;
    float2* pml = a.part_ml + ((size_t)lp * a.slots + slot) * a.Gp;
    float* pacc = a.part_acc + ((size_t)lp * a.slots + slot) * a.Gp * D;
    for (int e = gp.tid; e < G * D; e += NT) {
        const int h = e / D, dd = e - h * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, sm.M(w, h));
        float num = 0.f, den = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kDecodeWarps; ++w) {
                const float f = exp2f(sm.M(w, h) - M);
                num = fmaf(f, sm.acc[(w * G + h) * D + dd], num);
                den = fmaf(f, sm.L(w, h), den);
            }
        }
        pacc[h * D + dd] = num;
        if (dd == 0) pml[h] = make_float2(M, den);
    }
    __threadfence();
    gp.sync();
    if (gp.tid == 0) {
        const int prev = atomicAdd(a.cnt + lp, 1);
        s_last = (prev == nslots - 1);
        if (s_last) atomicExch(a.cnt + lp, 0);
    }
    gp.sync();
    if (!s_last) return;
    __threadfence();
    combine_partials<T, D>(a, layer, pair, lp, nslots, s_ml, gp);
}

// Combine the S partials of a (layer, pair) into O and LSE: per head the global max M and
// denominator, per partial a scale factor exp2(m_s - M) (shared memory), then every (head, d)
// element sums its scaled numerators with the loads of kU partials in flight.
template <typename T, int D>
__device__ void combine_partials(const DecodeArgs& a, int layer, int pair, int lp, int S,
                                 float2* s_ml /* S * Gp */, const Group gp) {
    __shared__ float s_M[kMaxG], s_den[kMaxG];
    const int G = a.G, NT = gp.nthreads;
    const float2* ml0 = a.part_ml + (size_t)lp * a.slots * a.Gp;
    const float* acc0 = a.part_acc + (size_t)lp * a.slots * a.Gp * D;
    for (int e = gp.tid; e < S * a.Gp; e += NT) s_ml[e] = ld_cg(ml0 + e);  // one round
    gp.sync();
    if (gp.tid < G) {
        const int h = gp.tid;
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
    gp.sync();
    const int b = pair / a.Hkv, kvh = pair - b * a.Hkv;
    T* out = reinterpret_cast<T*>(a.out[layer]) + ((size_t)b * a.Hq + (size_t)kvh * G) * D;
    float* lse = a.lse[layer] ? a.lse[layer] + (size_t)b * a.Hq + (size_t)kvh * G : nullptr;
    constexpr int kU = 8;
    for (int e = gp.tid; e < G * D; e += NT) {
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

// bf16 path: merge of the consumer warps' states into partial `slot` of a (layer, pair). The
// partials are combined by a second kernel once the whole grid has finished, so no fence or
// completion count is needed here.
template <int D>
__device__ void write_partial(const DecodeArgs& a, int lp, int slot, const MergeView sm,
                              const Group gp) {
    gp.sync();
    const int G = a.G, NT = gp.nthreads;
    float2* pml = a.part_ml + ((size_t)lp * a.slots + slot) * a.Gp;
    float* pacc = a.part_acc + ((size_t)lp * a.slots + slot) * a.Gp * D;
    for (int e = gp.tid; e < G * D; e += NT) {
        const int h = e / D, dd = e - h * D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, sm.M(w, h));
        float num = 0.f, den = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kDecodeWarps; ++w) {
                const float f = exp2f(sm.M(w, h) - M);
                num = fmaf(f, sm.acc[(w * G + h) * D + dd], num);
                den = fmaf(f, sm.L(w, h), den);
            }
        }
        pacc[h * D + dd] = num;
        if (dd == 0) pml[h] = make_float2(M, den);
    }
    gp.sync();  // the merge area is free for the next segment
}

// Which blocks this CTA owns, and the sequence facts every warp needs.
struct SplitInfo {
    int64_t T, nb;
    int ns;        // selected blocks of the pair (clamped to [0, SEL_cap]; 0 for a bad length)
    int beg, end;  // this split's blocks [beg, end) (fp32 path)
    bool ok;
};

// `lead` is true for exactly one thread of the CTA that handles the split (it reports errors).
__device__ __forceinline__ SplitInfo split_info(const DecodeArgs& a, int layer, int pair, int split,
                                                bool lead) {
    SplitInfo si;
    const int b = pair / a.Hkv;
    si.T = a.seq_lens[b];
    si.ok = si.T >= 0 && si.T <= a.T_cap;
    const bool reporter = layer == 0 && split == 0 && lead;
    if (!si.ok && reporter && pair % a.Hkv == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_SEQ_LEN);
    int ns = a.n_sel[pair];
    if (ns < 0 || ns > a.sel_cap) {
        if (reporter) atomicOr(a.err, (uint32_t)BSA_DEVERR_N_SEL);
        ns = ns < 0 ? 0 : a.sel_cap;
    }
    if (!si.ok) ns = 0;
    si.ns = ns;
    si.nb = si.ok ? (si.T + a.BS - 1) / a.BS : 0;
    si.beg = split * a.bpc;
    si.end = min(si.beg + a.bpc, ns);
    return si;
}

// -------------------------------------------------------------------------------------- bf16 path
constexpr int kConsumerWarps = 4;
constexpr int kTmaThreads = (kConsumerWarps + 1) * 32;  // + one producer warp
constexpr int kMaxStages = 8;
constexpr uint32_t kWaitPolls = 1u << 26;  // far beyond any legitimate wait; then give up
constexpr uint32_t kQSlot = 1024;          // bytes per stage for q of the group (G * D * 2 <= 2048)
constexpr int kCombineThreads = 256;
constexpr int kTokU = 4;  // fp32 path: tokens per warp step (BS is a multiple of 16)

enum : int { kStageFirst = 1, kStageLast = 2, kStageEnd = 4 };

struct StageMeta {
    int tok0;    // first token of the stage within the sequence
    int nvalid;  // tokens of the stage below the sequence length (0: flush-only stage)
    int lp;      // layer * pairs + pair
    int seg;     // this CTA's segment of the (layer, pair): partial slot
    int nseg;    // segments (CTAs) the (layer, pair) spans
    int flags;   // kStageFirst: q of this pair is in the stage; kStageLast: segment ends; kStageEnd
};

// CTA (of C) whose share [c*N/C, (c+1)*N/C) of the N block slots holds slot x.
__device__ __forceinline__ int cta_of_slot(int64_t x, int64_t N, int C) {
    return (int)(((x + 1) * C + N - 1) / N - 1);
}

// Persistent: the N = layers * pairs * SEL_cap block slots are shared evenly by C CTAs; CTA c walks
// slots [c*N/C, (c+1)*N/C). The producer lane streams every stage of its slots through the ring
// without draining; where its range crosses from one (layer, pair) to the next, the consumer warps
// flush the segment (merge into the segment's partial) behind a named barrier while the next
// stages are already loading. combine_kernel then merges each (layer, pair)'s partials.
template <int D>
__global__ void __launch_bounds__(kTmaThreads, 2)
    decode_tma_kernel(const DecodeArgs a, const __grid_constant__ KVMaps maps, const int nstages,
                      const int64_t n_slots) {
    extern __shared__ uint8_t dsm_raw[];
    __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages];
    __shared__ StageMeta meta[kMaxStages];
    constexpr int NB = D / 64;     // 64-column boxes per row
    constexpr int KS = D / 16;     // k-steps of S^T = K q^T
    constexpr int MT = D / 16;     // m-tiles of O^T
    const int ST = a.stage_tokens;
    const uint32_t box_bytes = (uint32_t)ST * 128u;
    const uint32_t kv_bytes = 2u * NB * box_bytes;
    const uint32_t stage_bytes = kv_bytes + kQSlot * ((a.G * D * 2 + kQSlot - 1) / kQSlot);
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
    float* mbase = reinterpret_cast<float*>(ring + (size_t)nstages * stage_bytes);
    const MergeView sm{mbase, mbase + kDecodeWarps * kMaxG, mbase + 2 * kDecodeWarps * kMaxG};

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
    const bool producer = warp == kConsumerWarps;
    const int C = (int)gridDim.x;
    const int64_t x_lo = (int64_t)blockIdx.x * n_slots / C, x_hi = (int64_t)(blockIdx.x + 1) * n_slots / C;

    if (threadIdx.x == 0) {
        for (int s2 = 0; s2 < nstages; ++s2) {
            mbar_init(&full[s2], 1);
            mbar_init(&empty[s2], kConsumerWarps);
        }
        mbar_fence_init();
    }
    __syncthreads();
    pdl_trigger();
    pdl_wait();

    if (producer) {
        if (lane == 0) {
            // the selected K/V rows are read once: keep the partials (reread by the combine) in L2
            const uint64_t kv_policy = l2_evict_first_policy();
            const int sub_per_block = a.BS / ST;
            int k = 0;
            bool ok = true;
            // claims ring slot k (waiting for the consumers to release it)
            auto claim = [&](int kk) -> int {
                const int st = kk % nstages;
                if (kk >= nstages && !mbar_wait(&empty[st], ((kk / nstages) - 1) & 1, kWaitPolls)) {
                    atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                    ok = false;
                }
                return st;
            };
            int q_lp = -1;  // (layer, pair) whose q the consumers hold
            for (int64_t x = x_lo; x < x_hi && ok;) {
                const int lp = (int)(x / a.sel_cap);
                const int64_t seg_end = min((int64_t)(lp + 1) * a.sel_cap, x_hi);
                const int layer = lp / a.pairs, pair = lp - layer * a.pairs;
                const int c_first = cta_of_slot((int64_t)lp * a.sel_cap, n_slots, C);
                const int c_last = cta_of_slot((int64_t)(lp + 1) * a.sel_cap - 1, n_slots, C);
                const int seg = (int)blockIdx.x - c_first, nseg = c_last - c_first + 1;
                // blocks [i_lo, i_hi) of the pair's selection fall in this CTA's share
                SplitInfo si = split_info(a, layer, pair, 0, seg == 0);
                const int i_lo = (int)(x - (int64_t)lp * a.sel_cap);
                const int i_hi = min((int)(seg_end - (int64_t)lp * a.sel_cap), si.ns);
                x = seg_end;
                const int64_t row_base = (int64_t)pair * a.T_cap;
                const int b = pair / a.Hkv, kvh = pair - b * a.Hkv;
                const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(a.q[layer]) +
                                      ((size_t)b * a.Hq + (size_t)kvh * a.G) * D * 2;
                bool first = lp != q_lp;
                int issued = 0;
                const int32_t* ip = a.block_idx + (size_t)pair * a.sel_cap;
                for (int i = i_lo; i < i_hi && ok; ++i) {
                    const int blk = ip[i];
                    if (blk < 0) continue;
                    if (blk >= si.nb) {
                        atomicOr(a.err, (uint32_t)BSA_DEVERR_BLOCK_IDX);
                        continue;
                    }
                    for (int sub = 0; sub < sub_per_block && ok; ++sub) {
                        const int64_t tok0 = (int64_t)blk * a.BS + (int64_t)sub * ST;
                        if (tok0 >= si.T) break;
                        const int st = claim(k);
                        if (!ok) break;
                        // is this the segment's last stage? (look ahead for another valid stage)
                        bool more = tok0 + ST < si.T && sub + 1 < sub_per_block;
                        for (int i2 = i + 1; i2 < i_hi && !more; ++i2) {
                            const int b2 = ip[i2];
                            more = b2 >= 0 && b2 < si.nb;
                        }
                        meta[st].tok0 = (int)tok0;
                        meta[st].nvalid = (int)min((int64_t)ST, si.T - tok0);
                        meta[st].lp = lp;
                        meta[st].seg = seg;
                        meta[st].nseg = nseg;
                        meta[st].flags = (first ? kStageFirst : 0) | (more ? 0 : kStageLast);
                        uint8_t* dst = ring + (size_t)st * stage_bytes;
                        const uint32_t qb = first ? (uint32_t)(a.G * D * 2) : 0u;
                        mbar_arrive_expect_tx(&full[st], kv_bytes + qb);
                        const int y = (int)(row_base + tok0);
#pragma unroll
                        for (int bi = 0; bi < NB; ++bi)
                            tma_load_2d_hint(dst + bi * box_bytes, &maps.k[layer], 64 * bi, y, &full[st], kv_policy);
#pragma unroll
                        for (int bi = 0; bi < NB; ++bi)
                            tma_load_2d_hint(dst + (NB + bi) * box_bytes, &maps.v[layer], 64 * bi, y, &full[st],
                                             kv_policy);
                        if (first) {
                            bulk_load(dst + kv_bytes, qsrc, qb, &full[st]);
                            q_lp = lp;
                        }
                        first = false;
                        ++issued;
                        ++k;
                    }
                }
                if (ok && issued == 0) {
                    // nothing to attend: a flush-only stage so the consumers publish an empty part
                    const int st = claim(k);
                    if (!ok) break;
                    meta[st].tok0 = 0;
                    meta[st].nvalid = 0;
                    meta[st].lp = lp;
                    meta[st].seg = seg;
                    meta[st].nseg = nseg;
                    meta[st].flags = kStageLast;
                    mbar_arrive(&full[st]);
                    ++k;
                }
            }
            if (ok) {
                const int st = claim(k);
                if (ok) {
                    meta[st].flags = kStageEnd;
                    mbar_arrive(&full[st]);
                }
            }
        }
    } else {
        const int r0 = 16 * warp;
        const Group gp{(int)threadIdx.x, kConsumerWarps * 32, 1};
        uint32_t qf[KS][2];
        AttnState<D> as;
        as.reset();
        for (int k = 0;; ++k) {
            const int st = k % nstages;
            if (!mbar_wait(&full[st], (k / nstages) & 1, kWaitPolls)) {
                if (lane == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                break;
            }
            const StageMeta md = meta[st];
            if (md.flags & kStageEnd) break;
            uint8_t* kst = ring + (size_t)st * stage_bytes;
            uint8_t* vst = kst + NB * box_bytes;
            if (md.flags & kStageFirst) {
                // q as the B operand: lane (g, tq) holds head g, d = 16ks + 2tq (+1, +8, +9)
                load_q_frag<D>(qf, reinterpret_cast<const uint32_t*>(kst + kv_bytes) + g * (D / 2), g < a.G, tq);
            }
            if (r0 < md.nvalid) attend16<D>(kst, vst, box_bytes, r0, md.nvalid, qf, a.scale_log2, as, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[st]);  // the ring slot may be refilled now
            if (md.flags & kStageLast) {
                // publish this warp's state of the item, then merge the item's split as a group
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    as.lsum[0] += __shfl_xor_sync(0xffffffffu, as.lsum[0], off);
                    as.lsum[1] += __shfl_xor_sync(0xffffffffu, as.lsum[1], off);
                }
                const int h0 = 2 * tq, h1 = 2 * tq + 1;
                if (g == 0) {
                    if (h0 < a.G) {
                        sm.M(warp, h0) = as.m[0];
                        sm.L(warp, h0) = as.lsum[0];
                    }
                    if (h1 < a.G) {
                        sm.M(warp, h1) = as.m[1];
                        sm.L(warp, h1) = as.lsum[1];
                    }
                }
                // accumulator (mt, row g / g+8) <-> d = 16 mt + g (+8)
                float* w0 = sm.acc + (warp * a.G + h0) * D;
                float* w1 = w0 + D;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    const int d0 = 16 * mt + g;
                    if (h0 < a.G) {
                        w0[d0] = as.acc[mt][0];
                        w0[d0 + 8] = as.acc[mt][2];
                    }
                    if (h1 < a.G) {
                        w1[d0] = as.acc[mt][1];
                        w1[d0 + 8] = as.acc[mt][3];
                    }
                }
                write_partial<D>(a, md.lp, md.seg, sm, gp);
                as.reset();
            }
        }
    }
}

// -------------------------------------------------------------------------------------- fp32 path
// One token at a time per warp; lanes split d, warp reductions form the dot products.
template <int D>
__global__ void __launch_bounds__(kDecodeThreads) decode_f32_kernel(DecodeArgs a) {
    __shared__ float s_m[kDecodeWarps * kMaxG], s_l[kDecodeWarps * kMaxG];
    __shared__ float s_acc[kDecodeWarps * kMaxG * D];
    const MergeView sm{s_m, s_l, s_acc};
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
    const SplitInfo si = split_info(a, layer, pair, split, threadIdx.x == 0);
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
    // The split's tokens, in groups of kTokU consecutive tokens of one block, are dealt to the
    // warps in turn; a group's K and V rows are loaded together and its softmax update is one step.
    const int gpb = a.BS / kTokU;  // groups per block
    const int ngroups = (si.end > si.beg ? si.end - si.beg : 0) * gpb;
    for (int gi = warp; gi < ngroups; gi += kDecodeWarps) {
        const int i = si.beg + gi / gpb;
        const int blk = ip[i];
        if (blk < 0) continue;
        if (blk >= si.nb) {
            if (lane == 0 && gi % gpb == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_BLOCK_IDX);
            continue;
        }
        const int64_t t0 = (int64_t)blk * a.BS + (int64_t)(gi % gpb) * kTokU;
        if (t0 >= si.T) continue;
        float kv[kTokU][E], vv[kTokU][E];
#pragma unroll
        for (int u = 0; u < kTokU; ++u) {
            const bool in = t0 + u < si.T;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                kv[u][e] = in ? __ldg(kp + (t0 + u) * D + lane * E + e) : 0.f;
                vv[u][e] = in ? __ldg(vp + (t0 + u) * D + lane * E + e) : 0.f;
            }
        }
#pragma unroll
        for (int h = 0; h < kMaxG; ++h) {
            if (h >= a.G) break;
            float x[kTokU];
#pragma unroll
            for (int u = 0; u < kTokU; ++u) {
                float p = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) p = fmaf(qv[h][e], kv[u][e], p);
                x[u] = p;
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                for (int u = 0; u < kTokU; ++u) x[u] += __shfl_xor_sync(0xffffffffu, x[u], off);
            float gmax = -INFINITY;
#pragma unroll
            for (int u = 0; u < kTokU; ++u) {
                x[u] = t0 + u < si.T ? x[u] * a.scale_log2 : -INFINITY;
                gmax = fmaxf(gmax, x[u]);
            }
            const float mn = fmaxf(m[h], gmax);
            const float al = exp2f(m[h] - mn);  // m[h] = -inf first: al = 0
            float wsum = 0.f, w[kTokU];
#pragma unroll
            for (int u = 0; u < kTokU; ++u) {
                w[u] = exp2f(x[u] - mn);
                wsum += w[u];
            }
            l[h] = l[h] * al + wsum;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                float t = acc[h][e] * al;
#pragma unroll
                for (int u = 0; u < kTokU; ++u) t = fmaf(w[u], vv[u][e], t);
                acc[h][e] = t;
            }
            m[h] = mn;
        }
    }
#pragma unroll
    for (int h = 0; h < kMaxG; ++h) {
        if (h < a.G) {
            if (lane == 0) {
                sm.M(warp, h) = m[h];
                sm.L(warp, h) = l[h];
            }
#pragma unroll
            for (int e = 0; e < E; ++e) sm.acc[(warp * a.G + h) * D + lane * E + e] = acc[h][e];
        }
    }
    __shared__ float2 s_ml[kMaxCombineSlots];
    finish_split<float, D>(a, layer, pair, lp, split, a.splits, sm, s_ml,
                           Group{(int)threadIdx.x, (int)blockDim.x, 0});
}

template <typename K>
cudaError_t launch_decode_k(K kernel, const Plan& p, const DecodeArgs& a, int layers, cudaStream_t st) {
    const int64_t grid = (int64_t)layers * p.pairs * p.dec_splits;
    if (grid <= 0) return cudaSuccess;
    if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
    return launch_pdl(kernel, dim3((unsigned)grid), dim3(kDecodeThreads), 0, st, a);
}

// bf16 path: one CTA per (layer, pair) merges, in segment order, the partials of the CTAs whose
// shares cover it, once the attention grid has finished.
// Every thread owns one head and four consecutive d values, and merges their partials in segment
// order with the (max, sum) and 16-byte numerator loads of up to kCombineU partials in flight
// together: one round of memory latency for the usual handful of partials, and no block barrier.
constexpr int kCombineU = 8;
static_assert(kCombineThreads * 4 >= kMaxG * 128, "one thread per head and four d values");

template <int D>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const DecodeArgs a, const int64_t n_slots,
                                                                  const int C) {
    pdl_trigger();
    pdl_wait();
    constexpr int Q = D / 4;  // groups of four d values per head
    const int lp = blockIdx.x;
    const int G = a.G;
    if ((int)threadIdx.x >= G * Q) return;
    const int h = (int)threadIdx.x / Q, dd = ((int)threadIdx.x - h * Q) * 4;
    const int layer = lp / a.pairs, pair = lp - layer * a.pairs;
    const int c_first = cta_of_slot((int64_t)lp * a.sel_cap, n_slots, C);
    const int c_last = cta_of_slot((int64_t)(lp + 1) * a.sel_cap - 1, n_slots, C);
    const int S = c_last - c_first + 1;
    const float2* ml0 = a.part_ml + (size_t)lp * a.slots * a.Gp + h;
    const float* acc0 = a.part_acc + (size_t)lp * a.slots * a.Gp * D + (size_t)h * D + dd;
    const int b = pair / a.Hkv, kvh = pair - b * a.Hkv;
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out[layer]) +
                         ((size_t)b * a.Hq + (size_t)kvh * G + h) * D + dd;
    float M = -INFINITY, den = 0.f;
    float num[4] = {0.f, 0.f, 0.f, 0.f};
    for (int s0 = 0; s0 < S; s0 += kCombineU) {
        float2 ml[kCombineU];
        float4 ac[kCombineU];
#pragma unroll
        for (int u = 0; u < kCombineU; ++u) {
            const bool in = s0 + u < S;
            const size_t slot = (size_t)(s0 + u) * a.Gp;
            ml[u] = in ? ld_cg(ml0 + slot) : make_float2(-INFINITY, 0.f);
            ac[u] = in ? ld_cg(reinterpret_cast<const float4*>(acc0 + slot * D)) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < kCombineU; ++u) {
            if (ml[u].x == -INFINITY) continue;  // an empty partial
            const float Mn = fmaxf(M, ml[u].x);
            const float fo = exp2f(M - Mn), fn = exp2f(ml[u].x - Mn);
            den = den * fo + ml[u].y * fn;
            num[0] = num[0] * fo + ac[u].x * fn;
            num[1] = num[1] * fo + ac[u].y * fn;
            num[2] = num[2] * fo + ac[u].z * fn;
            num[3] = num[3] * fo + ac[u].w * fn;
            M = Mn;
        }
    }
    float o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) o[k] = den > 0.f ? num[k] / den : 0.f;
    if ((reinterpret_cast<uintptr_t>(out) & 7u) == 0u) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(o[0], o[1]), hi = __floats2bfloat162_rn(o[2], o[3]);
        uint2 v;
        v.x = *reinterpret_cast<uint32_t*>(&lo);
        v.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(out) = v;
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) store_out<__nv_bfloat16>(out + k, o[k]);
    }
    if (dd == 0 && a.lse[layer]) {
        float* lse = a.lse[layer] + (size_t)b * a.Hq + (size_t)kvh * G + h;
        *lse = den > 0.f ? (M + log2f(den)) * 0.69314718055994531f : -INFINITY;
    }
}

template <int D>
cudaError_t launch_decode_tma(const Plan& p, const DecodeArgs& a, const KVMaps* maps, int layers,
                              cudaStream_t st) {
    const int64_t n_slots = (int64_t)layers * p.pairs * p.sel_cap;
    if (n_slots <= 0) return cudaSuccess;
    // the plan's CTA count covers num_layers layers; fewer layers get proportionally fewer CTAs
    int64_t ctas = (int64_t)p.dec_ctas * layers / p.layers;
    if (ctas < 1) ctas = 1;
    const size_t qslot = kQSlot * (((size_t)a.G * D * 2 + kQSlot - 1) / kQSlot);
    const size_t stage_bytes = (size_t)2 * (D / 64) * a.stage_tokens * 128 + qslot;
    // two CTAs per SM: ~112 KB each, of which the merge and combine scratch take a few KB
    const size_t scratch = merge_bytes(a.G, D);
    const size_t budget = 112 * 1024 - 1024 - scratch;
    int nstages = (int)(budget / stage_bytes);
    if (nstages < 2) nstages = 2;
    if (nstages > kMaxStages) nstages = kMaxStages;
    const size_t smem = 1024 + (size_t)nstages * stage_bytes + scratch;
    cudaError_t e = ensure_smem<decode_tma_kernel<D>>(smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(decode_tma_kernel<D>, dim3((unsigned)ctas), dim3(kTmaThreads), smem, st, a, *maps,
                   nstages, n_slots);
    if (e != cudaSuccess) return e;
    const int64_t lps = (int64_t)layers * p.pairs;
    return launch_pdl(combine_kernel<D>, dim3((unsigned)lps), dim3(kCombineThreads), 0, st, a, n_slots,
                      (int)ctas);
}

}  // namespace

cudaError_t launch_decode(const Plan& p, const DecodeArgs& a, const KVMaps* maps, int layers,
                          cudaStream_t st) {
    if (p.dtype == BSA_BF16)
        return p.D == 128 ? launch_decode_tma<128>(p, a, maps, layers, st)
                          : launch_decode_tma<64>(p, a, maps, layers, st);
    return p.D == 128 ? launch_decode_k(decode_f32_kernel<128>, p, a, layers, st)
                      : launch_decode_k(decode_f32_kernel<64>, p, a, layers, st);
}

bool encode_kv_map(CUtensorMap* map, const void* base, uint64_t rows, int D, int box_rows) {
    typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static EncodeFn encode = nullptr;
    if (!encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !fn)
            return false;
        encode = reinterpret_cast<EncodeFn>(fn);
    }
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace bsa
