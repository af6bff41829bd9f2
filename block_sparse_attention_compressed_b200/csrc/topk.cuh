// Top-k block selection shared by the selection kernels and the fused step kernel: the k largest
// block scores among the candidates (ties toward the lower block index), united with the init and
// local blocks and written in ascending order (page "SparDA: Sparse Decoupled Attention for Efficient
// Long-Context LLM Inference", Theoretical Foundation, Eq. 1; SparDA Architecture, Eq. 4, f_top).
// Every routine runs on a thread group: a whole CTA (barrier 0) or a named-barrier group of warps.
#pragma once

#include "bsa_internal.cuh"

namespace bsa {
namespace {

// Exclusive scan over a thread group of one int per thread (contiguous, in thread order), with one
// barrier:
// every warp scans its own values, publishes its total, and then scans all the warps' totals
// itself. With `reuse`, s_warp may be written again as soon as it returns.
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int* total, const Grp& gp,
                                                    bool reuse = true) {
    const int lane = gp.tid & 31, warp = gp.tid >> 5, nwarps = gp.nt >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    gp.sync();
    int w = lane < nwarps ? s_warp[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, w, off);
        if (lane >= off) w += y;
    }
    const int base = warp > 0 ? __shfl_sync(0xffffffffu, w, warp - 1) : 0;
    *total = __shfl_sync(0xffffffffu, w, nwarps - 1);
    if (reuse) gp.sync();
    return base + x - v;
}

// Top-k of the candidate blocks [init_end, local_begin) by score (ties: lower index first), united
// with the init and local blocks, written ascending. keys[] (shared) holds the nb block keys and
// may be overwritten. Each thread owns a contiguous segment of the candidates, kept in registers
// when it has at most kKeysPerThread of them (larger candidate sets are streamed from shared
// memory).
//
// The k-th largest key is located by radix digits below the bits that all candidates share: a
// first digit of up to kFirstDigitBits bits (one histogram bin per value, found with a two-level
// descending scan), then 8-bit digits. When that bucket holds exactly the number of keys still
// needed, all of them are taken with those above it. Otherwise, as soon as the bucket has at most
// kExactMax keys, they are gathered and each is ranked exactly against the others (score
// descending, block ascending) by its own team of threads; the taken candidates are those above
// the bucket plus the bucket keys ranked below the number still needed. Otherwise the ties at the
// final key value are taken in block order. Thread groups have kExactMax threads or more.
constexpr int kKeysPerThread = 8;
constexpr int kFirstDigitBits = 12;
constexpr int kExactMax = 128;
constexpr int kHistBins = 1 << kFirstDigitBits;

// Bin d* (scanning digits from the top) at which the running count of hist reaches `need`; the
// winning thread publishes the digit, the count still needed inside it and the bin's size.
__device__ __forceinline__ void find_digit_from_top(const int* hist, int nbins, int need, int* s_warp,
                                                    int* s_digit, int* s_need, int* s_bcnt, const Grp& gp) {
    const int tid = gp.tid, NT = gp.nt, lane = tid & 31, warp = tid >> 5;
    const int per_t = (nbins + NT - 1) / NT;  // bins per thread, descending from the top
    int c = 0, h8[16];
    // 8 or 16 bins per thread: bins [nbins - P(t+1), nbins - Pt) in 16-byte loads, top bin first
    const int P = (per_t == 16 && nbins == 16 * NT) ? 16 : ((per_t == 8 && nbins == 8 * NT) ? 8 : 0);
    const bool vec = P != 0;
    if (vec) {
        const int4* p = reinterpret_cast<const int4*>(hist + nbins - P * (tid + 1));
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (q < P / 4) {
                const int4 v = p[P / 4 - 1 - q];
                h8[4 * q] = v.w;
                h8[4 * q + 1] = v.z;
                h8[4 * q + 2] = v.y;
                h8[4 * q + 3] = v.x;
            } else {
                h8[4 * q] = h8[4 * q + 1] = h8[4 * q + 2] = h8[4 * q + 3] = 0;
            }
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) c += h8[k];
    } else {
        for (int k = 0; k < per_t; ++k) {
            const int d = nbins - 1 - (tid * per_t + k);
            if (d >= 0) c += hist[d];
        }
    }
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) s_warp[warp] = incl;
    if (tid == 0) {
        // found by exactly one thread below when the bins hold `need` keys or more; the defaults
        // (no exact bucket ranking) stand otherwise
        *s_digit = 0;
        *s_need = need;
        *s_bcnt = 0x7fffffff;
    }
    gp.sync();
    // totals of the warps before this one (a warp scan over the per-warp totals)
    int wt = lane < (NT >> 5) ? s_warp[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, wt, off);
        if (lane >= off) wt += y;
    }
    const int base = __shfl_sync(0xffffffffu, wt, (warp + 31) & 31) * (warp > 0);
    const int excl = base + incl - c;
    if (excl < need && need <= excl + c) {
        int acc = excl;
        if (vec) {
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                if (k < P && acc < need && acc + h8[k] >= need) {
                    *s_digit = nbins - 1 - (tid * P + k);
                    *s_need = need - acc;
                    *s_bcnt = h8[k];
                }
                acc += h8[k];
            }
        } else {
            for (int k = 0; k < per_t; ++k) {
                const int d = nbins - 1 - (tid * per_t + k);
                if (d < 0) break;
                const int cd = hist[d];
                if (acc < need && acc + cd >= need) {
                    *s_digit = d;
                    *s_need = need - acc;
                    *s_bcnt = cd;
                }
                acc += cd;
            }
        }
    }
    gp.sync();
}

// The top-k's shared memory, declared by each selection kernel.
struct TopkSmem {
    int warp[32];
    __align__(16) int hist[kHistBins];
    int digit, need, bcnt, bn;
    uint32_t kand[32], kor[32];                 // each warp's AND / OR of candidate keys
    __align__(16) uint32_t bkey[kExactMax];     // 0 pads: below every real key
    __align__(16) int bidx[kExactMax];
};

// Candidate blocks [init_end(nb), cand_end(nb)): neither init nor local.
__device__ __forceinline__ int cand_begin(const SelectArgs& a, int nb) { return min(a.n_init, nb); }
__device__ __forceinline__ int cand_end(const SelectArgs& a, int nb) {
    return max(max(nb - a.n_local, 0), min(a.n_init, nb));
}

// Clears the first digit's bins and the exact bucket; a barrier must follow before topk_union.
__device__ __forceinline__ void topk_prepare(TopkSmem& t, const Grp& gp) {
    for (int i = gp.tid; i < kHistBins / 4; i += gp.nt)
        reinterpret_cast<int4*>(t.hist)[i] = make_int4(0, 0, 0, 0);
    for (int i = gp.tid; i < kExactMax; i += gp.nt) t.bkey[i] = 0u;
    if (gp.tid == 0) t.bn = 0;
}

// Publishes a warp's AND / OR of the candidate keys it wrote (identity values when none).
__device__ __forceinline__ void publish_andor(TopkSmem& t, uint32_t kand, uint32_t kor, const Grp& gp) {
    kand = __reduce_and_sync(0xffffffffu, kand);
    kor = __reduce_or_sync(0xffffffffu, kor);
    if ((gp.tid & 31) == 0) {
        t.kand[gp.tid >> 5] = kand;
        t.kor[gp.tid >> 5] = kor;
    }
}

// `andor_ready`: every warp has published the AND / OR of the candidate keys it wrote (then no
// pass over the keys is needed for them). topk_prepare and a barrier come before the call.
__device__ void topk_union(const SelectArgs& a, int nb, uint32_t* keys, TopkSmem& t, bool andor_ready,
                           const Grp& gp, int32_t* out, int32_t* n_out) {
    int* s_warp = t.warp;
    int* hist = t.hist;
    uint32_t* s_bkey = t.bkey;
    int* s_bidx = t.bidx;
    const int tid = gp.tid, NT = gp.nt;
    const int init_end = cand_begin(a, nb);
    const int clo = init_end, chi = cand_end(a, nb);
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
    bool exact = false, whole = false;
    uint32_t emask = 0u, eprefix = 0u;
    if (kk > 0 && !take_all) {
        // bits that every candidate shares need no histogram pass (block-wide AND / OR)
        if (!andor_ready) {
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
                // keys in shared memory: a strided walk (consecutive lanes, consecutive words)
                for (int i = clo + tid; i < chi; i += NT) {
                    kand &= keys[i];
                    kor |= keys[i];
                }
            }
            publish_andor(t, kand, kor, gp);
            gp.sync();
        }
        uint32_t kand = 0xffffffffu, kor = 0u;
        for (int w = 0; w < (NT >> 5); ++w) {
            kand &= t.kand[w];
            kor |= t.kor[w];
        }
        const uint32_t diff = kand ^ kor;  // bits in which some candidates differ
        uint32_t prefix = kand, mask = 0xffffffffu;
        need = kk;
        if (diff != 0u) {
            int hi = 31 - __clz(diff);
            mask = hi < 31 ? (0xffffffffu << (hi + 1)) : 0u;
            prefix = kand & mask;
            int width = min(kFirstDigitBits, hi + 1);
            for (bool first = true;; first = false) {
                const int shift = hi - width + 1;
                const int nbins = 1 << width;
                const uint32_t dmask = (uint32_t)nbins - 1u;
                if (!first) {
                    for (int i = tid; i < nbins; i += NT) hist[i] = 0;
                    gp.sync();
                }
                if (in_regs) {
#pragma unroll
                    for (int e = 0; e < kKeysPerThread; ++e)
                        if (seg_lo + e < seg_hi && (kr[e] & mask) == prefix) atomicAdd(&hist[(kr[e] >> shift) & dmask], 1);
                } else {
                    for (int i = clo + tid; i < chi; i += NT) {
                        const uint32_t u = keys[i];
                        if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & dmask], 1);
                    }
                }
                gp.sync();
                find_digit_from_top(hist, nbins, need, s_warp, &t.digit, &t.need, &t.bcnt, gp);
                prefix |= (uint32_t)t.digit << shift;
                need = t.need;
                mask |= dmask << shift;
                if (in_regs && t.bcnt == need) {
                    whole = true;  // the bucket holds exactly the keys still needed: all are taken
                    break;
                }
                if (shift == 0) break;  // every bit decided: the bucket's keys are all equal
                if (in_regs && t.bcnt <= kExactMax) {
                    exact = true;
                    break;
                }
                gp.sync();  // everyone has read the bins before they are cleared
                hi = shift - 1;
                width = min(8, hi + 1);
            }
        }
        thr = prefix;
        if (exact || whole) {
            emask = mask;
            eprefix = prefix;
        }
    }

    if (in_regs) {
        // taken flags of the thread's own candidates
        bool fl[kKeysPerThread];
        if (whole) {
            // the keys above the k-th key's bucket, and the whole bucket
#pragma unroll
            for (int e = 0; e < kKeysPerThread; ++e) fl[e] = seg_lo + e < seg_hi && (kr[e] & emask) >= eprefix;
        } else if (exact) {
#pragma unroll
            for (int e = 0; e < kKeysPerThread; ++e) {
                if (seg_lo + e < seg_hi && (kr[e] & emask) == eprefix) {
                    const int slot = atomicAdd(&t.bn, 1);
                    if (slot < kExactMax) {  // always, when the keys' AND / OR are those published
                        s_bkey[slot] = kr[e];
                        s_bidx[slot] = seg_lo + e;
                    }
                }
            }
            gp.sync();
            const int ebn = min(t.bn, kExactMax);
            const uint4* bk4 = reinterpret_cast<const uint4*>(s_bkey);
            const int4* bi4 = reinterpret_cast<const int4*>(s_bidx);
            // entries of the bucket ahead of key u at block idx (four per 16-byte read; the zero
            // pads never count), over the quads q0, q0 + dq, ...
            auto ahead = [&](uint32_t u, int idx, int q0, int dq) {
                int rank = 0;
                for (int q = q0; q < (ebn + 3) / 4; q += dq) {
                    const uint4 kq = bk4[q];
                    const int4 iq = bi4[q];
                    rank += (kq.x > u || (kq.x == u && iq.x < idx)) + (kq.y > u || (kq.y == u && iq.y < idx)) +
                            (kq.z > u || (kq.z == u && iq.z < idx)) + (kq.w > u || (kq.w == u && iq.w < idx));
                }
                return rank;
            };
            {
                // each entry is ranked by a team of NT / kExactMax consecutive lanes, which marks it
                // taken or not in keys[] at its block (its owner may hold several entries)
                const int team = NT / kExactMax;  // 1, 2, 4 or 8 (NT = 128 .. 1024)
                const int j = tid / team, r = tid - j * team;
                int rank = j < ebn ? ahead(s_bkey[j], s_bidx[j], r, team) : 0;
                for (int off = 1; off < team; off <<= 1) rank += __shfl_xor_sync(0xffffffffu, rank, off);
                if (j < ebn && r == 0) keys[s_bidx[j]] = rank < need ? 1u : 0u;
                gp.sync();
#pragma unroll
                for (int e = 0; e < kKeysPerThread; ++e) {
                    fl[e] = false;
                    if (seg_lo + e < seg_hi) {
                        const uint32_t mk = kr[e] & emask;
                        fl[e] = mk > eprefix || (mk == eprefix && keys[seg_lo + e] == 1u);
                    }
                }
            }
        } else if (take_all || kk == 0) {
#pragma unroll
            for (int e = 0; e < kKeysPerThread; ++e) fl[e] = take_all && seg_lo + e < seg_hi;
        } else {
            // keys above thr, and the first `need` keys equal to thr in block order
            int cnt = 0;
#pragma unroll
            for (int e = 0; e < kKeysPerThread; ++e) cnt += (seg_lo + e < seg_hi && kr[e] == thr);
            int tot;
            int r = block_exclusive_scan(cnt, s_warp, &tot, gp);
#pragma unroll
            for (int e = 0; e < kKeysPerThread; ++e) {
                fl[e] = false;
                if (seg_lo + e < seg_hi) {
                    const uint32_t u = kr[e];
                    fl[e] = u > thr || (u == thr && r < need);
                    r += (u == thr);
                }
            }
        }
        // union: init blocks, the taken candidates in block order, then the local blocks
        int cnt = 0;
#pragma unroll
        for (int e = 0; e < kKeysPerThread; ++e) cnt += fl[e];
        int taken;
        int pos = init_end + block_exclusive_scan(cnt, s_warp, &taken, gp, false);
#pragma unroll
        for (int e = 0; e < kKeysPerThread; ++e)
            if (fl[e]) out[pos++] = seg_lo + e;
        for (int i = tid; i < init_end; i += NT) out[i] = i;
        const int n_loc = nb - chi;
        for (int i = tid; i < n_loc; i += NT) out[init_end + taken + i] = chi + i;
        const int total = init_end + taken + n_loc;
        for (int i = total + tid; i < a.sel_cap; i += NT) out[i] = -1;
        if (tid == 0) *n_out = total;
        return;
    }

    // streamed candidates (keys in shared memory): the warps walk 32-block chunks, lane l taking
    // block 32c + l, so every read is conflict-free; block order comes from per-chunk counts
    // (ballots) and a scan over the chunks. The bins are free now and hold those counts.
    {
        const int lane = tid & 31, warp = tid >> 5, nwarps = NT >> 5;
        const int nch = (nb + 31) / 32;
        const unsigned lt = (1u << lane) - 1u;
        int* eqc = hist;                   // [nch] keys equal to thr, then their exclusive prefix
        int* tkc = hist + kHistBins / 2;   // [nch] blocks in the union, then their exclusive prefix
        // in-place exclusive prefix over arr[0 .. n), in chunk order; returns the total
        auto chunk_scan = [&](int* arr, int n) -> int {
            const int cpt = (n + NT - 1) / NT;
            const int lo = tid * cpt, hi = min(lo + cpt, n);
            int sum = 0;
            for (int c = lo; c < hi; ++c) sum += arr[c];
            int tot;
            int base = block_exclusive_scan(sum, s_warp, &tot, gp);
            for (int c = lo; c < hi; ++c) {
                const int v = arr[c];
                arr[c] = base;
                base += v;
            }
            gp.sync();
            return tot;
        };
        for (int c = warp; c < nch; c += nwarps) {
            const int i = 32 * c + lane;
            const bool eq = i >= clo && i < chi && keys[i] == thr;
            const unsigned m = __ballot_sync(0xffffffffu, eq);
            if (lane == 0) eqc[c] = __popc(m);
        }
        gp.sync();
        chunk_scan(eqc, nch);
        // taken flags into keys[] (1 / 0): init and local blocks, candidates above thr, and the
        // first `need` candidates equal to thr in block order
        for (int c = warp; c < nch; c += nwarps) {
            const int i = 32 * c + lane;
            const bool cand = i >= clo && i < chi;
            const uint32_t u = cand ? keys[i] : 0u;
            const unsigned m = __ballot_sync(0xffffffffu, cand && u == thr);
            const int r = eqc[c] + __popc(m & lt);  // candidates equal to thr before block i
            const bool fl = i < nb && (!cand || (kk > 0 && (take_all || u > thr || (u == thr && r < need))));
            const unsigned fm = __ballot_sync(0xffffffffu, fl);
            if (lane == 0) tkc[c] = __popc(fm);
            if (i < nb) keys[i] = fl ? 1u : 0u;
        }
        gp.sync();
        const int total = chunk_scan(tkc, nch);
        for (int c = warp; c < nch; c += nwarps) {
            const int i = 32 * c + lane;
            const bool fl = i < nb && keys[i] != 0u;
            const unsigned fm = __ballot_sync(0xffffffffu, fl);
            if (fl) out[tkc[c] + __popc(fm & lt)] = i;
        }
        for (int i = total + tid; i < a.sel_cap; i += NT) out[i] = -1;
        if (tid == 0) *n_out = total;
    }
}

}  // namespace
}  // namespace bsa
