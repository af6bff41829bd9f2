// Block-sparse prefill of a chunk of queries (page "SparDA: Sparse Decoupled Attention for
// Efficient Long-Context LLM Inference", Theoretical Foundation, Eq. 1 and the prefill workload of
// its Efficiency Results; the selection is made per query tile, as the tile-level operations of the
// page "CoSA: Accelerating Long-Context Inference via Proxy-Kernel Co-Designed Sparse Attention",
// Kascade abstract, suggest). The chunk's C queries of sequence b sit at positions T - C .. T - 1
// (T = seq_lens[b]; their keys and values are already in the cache, the compressed keys formed).
// Query tile r is the chunk's positions inside block r. For each (tile, kv head):
//   scores     S[j] = sum over the tile's positions p and the group's heads h of
//              softmax_j(q_{p,h} . K~_j / tau) over the windows complete before block r begins
//              (Indexer Training, Eq. 6, summed over the tile);
//   selection  the block maxima of S and the top-k union of Eq. 1 among blocks 0 .. r;
//   attention  each query attends the selected blocks' tokens at or before its position (Eq. 5).
//
// Selection kernel (tcgen05): a persistent CTA per SM takes (pair, tile) items. Its tile rows are
// the R = 64 * G (position, head) pairs of the tile, K-major in shared memory with the 128-byte
// swizzle; the compressed keys stream through a ring of 128-window stages by TMA. The tensor cores
// run two passes over the windows: pass 1, rows x windows (M = 128 rows per MMA, N = 128 windows),
// gives each row its softmax maximum and sum (one row per TMEM lane: no cross-thread reduction);
// pass 2, windows x rows (M = 128 windows, N = R), gives each window the sum over the rows of its
// probability (one window per TMEM lane). The accumulators live in tensor memory (two 256-column
// buffers), read back with tcgen05.ld by four epilogue warps; one warp issues the TMA copies and one
// thread the MMAs (tcgen05.mma, completion through tcgen05.commit on shared-memory barriers).
//
// Attention kernel (mma.m16n8k16): a CTA per (pair, tile, pair of heads), four warps of 16 query
// positions per head; the selected blocks' K and V rows stream through a TMA ring.
#include "bsa_internal.cuh"
#include "topk.cuh"

namespace bsa {
namespace {

// ------------------------------------------------------------------------------ tcgen05 helpers
// Shared-memory matrix descriptor of a K-major operand in the 128-byte swizzle: rows of 64 bf16
// (128 bytes), 8-row groups 1024 bytes apart (leading offset unused for this layout).
__device__ __forceinline__ uint64_t umma_desc_k_sw128(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | (1ull << 16) | (64ull << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor: bf16 x bf16 -> fp32, both operands K-major, M x N.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
// D (TMEM) = A * B^T (+ D when acc), issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}
// `bar` receives one arrival when every MMA this thread issued so far has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// ------------------------------------------------------------------------------ selection kernel
constexpr int kPsWarps = 6;             // producer, MMA issuer, four epilogue warps
constexpr int kPsThreads = kPsWarps * 32;
constexpr int kPsSlots = 3;             // compressed-key stages in flight
constexpr int kPsChunk = 128;           // windows per stage
constexpr uint32_t kPsSlotBytes = 2u * kPsChunk * 128u;  // two 64-column boxes of 128 rows
constexpr int kPsEpiBar = 1;            // named barrier of the epilogue warps
constexpr uint32_t kPsPolls = 1u << 26;

// One (pair, tile) item, computed identically by every role.
struct PsItem {
    int pair, b, kvh, ti;
    int64_t T, t0, r;
    int nc, nch;  // windows complete before block r; 128-window stages
    bool live;
};
__device__ __forceinline__ PsItem ps_item(const PrefillArgs& a, int g) {
    PsItem it;
    it.pair = g / a.tiles_cap;
    it.ti = g - it.pair * a.tiles_cap;
    it.b = it.pair / a.Hkv;
    it.kvh = it.pair - it.b * a.Hkv;
    it.T = a.seq_lens[it.b];
    const bool ok = it.T >= a.chunk && it.T <= a.T_cap;
    it.t0 = it.T - a.chunk;
    it.r = it.t0 / a.BS + it.ti;
    it.live = ok && it.r <= (it.T - 1) / a.BS;
    const int64_t start = (int64_t)a.BS * it.r;
    int64_t nc = start < a.l ? 0 : (start - a.l) / a.s + 1;
    if (nc > a.nc_cap) nc = a.nc_cap;
    it.nc = it.live ? (int)nc : 0;
    it.nch = (it.nc + kPsChunk - 1) / kPsChunk;
    return it;
}

// R: rows of a tile (64 positions x G heads, 128 or 256).
template <int R>
__global__ void __launch_bounds__(kPsThreads, 1)
    prefill_select_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap ck_map) {
    static_assert(R == 128 || R == 256, "tiles of 128 or 256 rows");
    constexpr int MB = R / 128;                 // 128-row blocks of pass 1
    extern __shared__ uint8_t dsm_raw[];
    __shared__ __align__(8) uint64_t full[kPsSlots], empty[kPsSlots], accf[2], acce[2], qready;
    __shared__ TopkSmem tk;
    __shared__ uint32_t s_tmem;
    __shared__ int s_nsel;
    uint8_t* qt = dsm_raw + ((1024u - (smem_u32(dsm_raw) & 1023u)) & 1023u);  // 2 boxes x R rows x 128 B
    uint8_t* ring = qt + 2 * R * 128;
    float2* stats = reinterpret_cast<float2*>(ring + kPsSlots * kPsSlotBytes);  // [R] (max, 1/sum), log2 domain
    float* S = reinterpret_cast<float*>(stats + R);                            // [nc_cap] window scores
    uint32_t* keys = reinterpret_cast<uint32_t*>(S + ((a.nc_cap + 3) & ~int64_t(3)));  // [nb_cap]
    int32_t* sel = reinterpret_cast<int32_t*>(keys + ((a.nb_cap + 3) & ~int64_t(3)));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kPsSlots; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&accf[i], 1);
            mbar_init(&acce[i], 4);
        }
        mbar_init(&qready, 128);
        mbar_fence_init();
    }
    if (warp == 1) tmem_alloc(&s_tmem, 512);
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t tbase = s_tmem;
    pdl_trigger();
    pdl_wait();
    const int items = a.pairs * a.tiles_cap;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            int64_t k = 0;
            bool stop = false;
            for (int g = blockIdx.x; g < items && !stop; g += gridDim.x) {
                const PsItem it = ps_item(a, g);
                for (int pass = 0; pass < 2 && !stop; ++pass)
                    for (int c = 0; c < it.nch; ++c, ++k) {
                        const int slot = (int)(k % kPsSlots);
                        if (k >= kPsSlots && !mbar_wait(&empty[slot], (uint32_t)((k / kPsSlots) - 1) & 1u, kPsPolls)) {
                            atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                            stop = true;
                            break;
                        }
                        uint8_t* dst = ring + (size_t)slot * kPsSlotBytes;
                        mbar_arrive_expect_tx(&full[slot], kPsSlotBytes);
                        const int y = (int)((int64_t)it.pair * a.nc_cap + (int64_t)kPsChunk * c);
                        tma_load_2d_hint(dst, &ck_map, 0, y, &full[slot], pol);
                        tma_load_2d_hint(dst + kPsChunk * 128, &ck_map, 64, y, &full[slot], pol);
                    }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int64_t k = 0, n = 0;
            uint32_t qphase = 0;
            bool stop = false;
            const uint32_t qt_a = smem_u32(qt), ring_a = smem_u32(ring);
            for (int g = blockIdx.x; g < items && !stop; g += gridDim.x) {
                const PsItem it = ps_item(a, g);
                if (!it.live) continue;
                if (!mbar_wait(&qready, qphase, kPsPolls)) {
                    atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                    break;
                }
                qphase ^= 1u;
                for (int pass = 0; pass < 2 && !stop; ++pass)
                    for (int c = 0; c < it.nch; ++c, ++k, ++n) {
                        const int slot = (int)(k % kPsSlots), buf = (int)(n & 1);
                        if (!mbar_wait(&full[slot], (uint32_t)(k / kPsSlots) & 1u, kPsPolls) ||
                            (n >= 2 && !mbar_wait(&acce[buf], (uint32_t)((n >> 1) - 1) & 1u, kPsPolls))) {
                            atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                            stop = true;
                            break;
                        }
                        tmem_fence_after_sync();
                        const uint32_t st_a = ring_a + (uint32_t)slot * kPsSlotBytes;
                        const uint32_t d0 = tbase + (uint32_t)(buf * 256);
                        if (pass == 0) {
                            // rows x windows: D[row][window] for each 128-row block
                            for (int mb = 0; mb < MB; ++mb)
                                for (int ks = 0; ks < 8; ++ks) {
                                    const uint32_t off = (uint32_t)((ks & 3) * 32);
                                    umma_bf16(d0 + (uint32_t)(mb * 128),
                                              umma_desc_k_sw128(qt_a + (uint32_t)((ks >> 2) * R * 128 + mb * 128 * 128) + off),
                                              umma_desc_k_sw128(st_a + (uint32_t)((ks >> 2) * kPsChunk * 128) + off),
                                              umma_idesc_bf16(128, kPsChunk), ks > 0);
                                }
                        } else {
                            // windows x rows: D[window][row]
                            for (int ks = 0; ks < 8; ++ks) {
                                const uint32_t off = (uint32_t)((ks & 3) * 32);
                                umma_bf16(d0, umma_desc_k_sw128(st_a + (uint32_t)((ks >> 2) * kPsChunk * 128) + off),
                                          umma_desc_k_sw128(qt_a + (uint32_t)((ks >> 2) * R * 128) + off),
                                          umma_idesc_bf16(128, R), ks > 0);
                            }
                        }
                        umma_commit(&empty[slot]);
                        umma_commit(&accf[buf]);
                    }
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue warps
        const int et = threadIdx.x - 64;                    // 0..127
        const Grp grp{et, 128, kPsEpiBar};
        const int quarter = warp & 3;                       // TMEM lanes 32 * quarter ..
        const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
        SelectArgs sa;
        memset(&sa, 0, sizeof sa);
        sa.n_init = a.n_init;
        sa.n_local = a.n_local;
        sa.top_k = a.top_k;
        sa.sel_cap = a.sel_cap;
        int64_t n = 0;
        bool dead = false;
        const float sl = a.score_log2;
        for (int g = blockIdx.x; g < items; g += gridDim.x) {
            const PsItem it = ps_item(a, g);
            int32_t* oidx = a.block_idx + (size_t)g * a.sel_cap;
            if (!it.live || dead) {
                for (int i = et; i < a.sel_cap; i += 128) oidx[i] = -1;
                if (et == 0) a.n_sel[g] = 0;
                continue;
            }
            topk_prepare(tk, grp);
            // the tile's rows into shared memory (row = position-in-block * G + head), K-major with
            // the 128-byte swizzle; rows outside the chunk are zero
            const int G = a.G;
            for (int e = et; e < R * 16; e += 128) {
                const int row = e >> 4, ch = e & 15;
                const int cpos = row / G, h = row - cpos * G;
                const int64_t p = (int64_t)a.BS * it.r + cpos;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (row < 64 * G && p >= it.t0 && p < it.T)
                    v = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.q) +
                                                        (((size_t)it.b * a.chunk + (size_t)(p - it.t0)) * a.Hq +
                                                         (size_t)it.kvh * G + h) * 128 + ch * 8);
                *reinterpret_cast<uint4*>(qt + (ch >> 3) * R * 128 + row * 128 + (((ch & 7) ^ (row & 7)) << 4)) = v;
            }
            fence_proxy_async_smem();
            mbar_arrive(&qready);
            // ---- pass 1: each thread's rows (one per 128-row block): softmax maximum and sum
            float m[MB], z[MB];
#pragma unroll
            for (int mb = 0; mb < MB; ++mb) m[mb] = -INFINITY, z[mb] = 0.f;
            for (int c = 0; c < it.nch; ++c, ++n) {
                const int buf = (int)(n & 1);
                if (!dead && !mbar_wait(&accf[buf], (uint32_t)(n >> 1) & 1u, kPsPolls)) {
                    if (lane == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                    dead = true;
                }
                tmem_fence_after_sync();
#pragma unroll
                for (int mb = 0; mb < MB; ++mb) {
#pragma unroll
                    for (int pc = 0; pc < kPsChunk / 32; ++pc) {
                        float v[32];
                        tmem_ld<32>(tbase + lane_off + (uint32_t)(buf * 256 + mb * 128 + pc * 32), v);
                        tmem_wait_ld();
                        const int j0 = kPsChunk * c + 32 * pc;
                        const int nv = min(32, it.nc - j0);  // valid windows of this piece
                        float mx = -INFINITY;
#pragma unroll
                        for (int e = 0; e < 32; ++e) {
                            v[e] *= sl;
                            if (e < nv) mx = fmaxf(mx, v[e]);
                        }
                        if (nv > 0) {
                            const float mn = fmaxf(m[mb], mx);
                            float acc = 0.f;
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (e < nv) acc += exp2f(v[e] - mn);
                            z[mb] = (m[mb] == -INFINITY ? 0.f : z[mb] * exp2f(m[mb] - mn)) + acc;
                            m[mb] = mn;
                        }
                    }
                }
                tmem_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce[buf]);
            }
#pragma unroll
            for (int mb = 0; mb < MB; ++mb) {
                const int row = mb * 128 + 32 * quarter + lane;
                const int cpos = row / G;
                const int64_t p = (int64_t)a.BS * it.r + cpos;
                const bool valid = row < 64 * G && p >= it.t0 && p < it.T && z[mb] > 0.f;
                stats[row] = valid ? make_float2(m[mb], 1.f / z[mb]) : make_float2(0.f, 0.f);
            }
            grp.sync();
            // ---- pass 2: each thread's window of every stage: the sum over the rows of exp2(x - max) / sum
            for (int c = 0; c < it.nch; ++c, ++n) {
                const int buf = (int)(n & 1);
                if (!dead && !mbar_wait(&accf[buf], (uint32_t)(n >> 1) & 1u, kPsPolls)) {
                    if (lane == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                    dead = true;
                }
                tmem_fence_after_sync();
                float acc = 0.f;
#pragma unroll 1
                for (int pc = 0; pc < R / 32; ++pc) {
                    float v[32];
                    tmem_ld<32>(tbase + lane_off + (uint32_t)(buf * 256 + pc * 32), v);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float2 st = stats[32 * pc + e];
                        if (st.y > 0.f) acc += exp2f(v[e] * sl - st.x) * st.y;
                    }
                }
                tmem_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce[buf]);
                const int j = kPsChunk * c + 32 * quarter + lane;
                if (j < it.nc) S[j] = acc;
            }
            grp.sync();
            // ---- block maxima over blocks 0 .. r: block b's windows are 4b - 1 .. 4b + 3
            const int nb = (int)it.r + 1;
            for (int bb = et; bb < nb; bb += 128) {
                float mx = -INFINITY;
                for (int j = max(4 * bb - 1, 0); j <= 4 * bb + 3 && j < it.nc; ++j) mx = fmaxf(mx, S[j]);
                keys[bb] = order_key(mx);
            }
            grp.sync();
            topk_union(sa, nb, keys, tk, false, grp, sel, &s_nsel);
            grp.sync();
            for (int i = et; i < a.sel_cap; i += 128) oidx[i] = sel[i];
            if (et == 0) a.n_sel[g] = s_nsel;
            grp.sync();  // sel, keys and stats are rewritten by the next item
        }
    }
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 1) tmem_dealloc(tbase, 512);
}

// ------------------------------------------------------------------------------ attention kernel
constexpr int kPaWarps = 8;              // two heads x four warps of 16 positions
constexpr int kPaThreads = (kPaWarps + 1) * 32;
constexpr int kPaSlots = 4;              // K + V block stages in flight
constexpr uint32_t kPaBox = 64u * 128u;  // 64 rows x 64 columns
constexpr uint32_t kPaStage = 4u * kPaBox;  // K (two boxes) and V (two boxes) of one 64-token block
constexpr uint32_t kPaPolls = 1u << 26;

__global__ void __launch_bounds__(kPaThreads, 1)
    prefill_attend_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap k_map,
                          const __grid_constant__ CUtensorMap v_map) {
    extern __shared__ uint8_t dsm_raw[];
    __shared__ __align__(8) uint64_t full[kPaSlots], empty[kPaSlots];
    uint8_t* ring = dsm_raw + ((1024u - (smem_u32(dsm_raw) & 1023u)) & 1023u);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // item: (pair, tile, head pair)
    const int hp_n = (a.G + 1) / 2;
    const int item = blockIdx.x;
    const int hp = item % hp_n;
    const int g = item / hp_n;  // pair * tiles_cap + tile
    const int pair = g / a.tiles_cap, ti = g - pair * a.tiles_cap;
    const int b = pair / a.Hkv, kvh = pair - b * a.Hkv;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kPaSlots; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kPaWarps);
        }
        mbar_fence_init();
    }
    __syncthreads();
    pdl_trigger();
    pdl_wait();
    const int64_t T = a.seq_lens[b];
    const bool ok = T >= a.chunk && T <= a.T_cap;
    const int64_t t0 = T - a.chunk, r = t0 / a.BS + ti;
    const bool live = ok && r <= (T - 1) / a.BS;
    const int nsel = live ? min(max(a.n_sel[g], 0), a.sel_cap) : 0;
    const int32_t* idx = a.block_idx + (size_t)g * a.sel_cap;

    if (warp == kPaWarps) {
        // ---- producer: the selected blocks' K and V rows
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            int kk = 0;  // stages issued (entries outside blocks 0 .. r are skipped by every warp alike)
            for (int i = 0; i < nsel; ++i) {
                const int blk = idx[i];
                if (blk < 0 || blk > r) continue;
                const int slot = kk % kPaSlots;
                if (kk >= kPaSlots && !mbar_wait(&empty[slot], (uint32_t)((kk / kPaSlots) - 1) & 1u, kPaPolls)) {
                    atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                    break;
                }
                uint8_t* dst = ring + (size_t)slot * kPaStage;
                mbar_arrive_expect_tx(&full[slot], kPaStage);
                const int y = (int)((int64_t)pair * a.T_cap + (int64_t)blk * a.BS);
                tma_load_2d_hint(dst, &k_map, 0, y, &full[slot], pol);
                tma_load_2d_hint(dst + kPaBox, &k_map, 64, y, &full[slot], pol);
                tma_load_2d_hint(dst + 2 * kPaBox, &v_map, 0, y, &full[slot], pol);
                tma_load_2d_hint(dst + 3 * kPaBox, &v_map, 64, y, &full[slot], pol);
                ++kk;
            }
        }
        return;
    }
    // ---- consumers: warp w takes head 2 hp + (w >> 2), positions 16 (w & 3) .. + 15 of the tile
    const int h = 2 * hp + (warp >> 2);
    const bool hvalid = h < a.G;
    const int g8 = lane >> 2, tq = lane & 3;
    const int prow0 = 16 * (warp & 3);            // first position (within the block) of the warp
    const int64_t blk_start = (int64_t)a.BS * r;
    // positions of this thread's two rows (g8 and g8 + 8 of the warp's 16)
    const int64_t pa = blk_start + prow0 + g8, pb = pa + 8;
    const bool va = live && hvalid && pa >= t0 && pa < T, vb = live && hvalid && pb >= t0 && pb < T;
    // Q fragments (A operand, rows g8 / g8 + 8, columns 16 ks + 2 tq (+1), + 8)
    uint32_t qf[8][4];
    {
        const uint16_t* q16 = reinterpret_cast<const uint16_t*>(a.q);
        const size_t hq = (size_t)kvh * a.G + (hvalid ? h : 0);
        const uint32_t* ra = va ? reinterpret_cast<const uint32_t*>(q16 + (((size_t)b * a.chunk + (size_t)(pa - t0)) * a.Hq + hq) * 128) : nullptr;
        const uint32_t* rb = vb ? reinterpret_cast<const uint32_t*>(q16 + (((size_t)b * a.chunk + (size_t)(pb - t0)) * a.Hq + hq) * 128) : nullptr;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
            qf[ks][0] = ra ? ra[8 * ks + tq] : 0u;
            qf[ks][1] = rb ? rb[8 * ks + tq] : 0u;
            qf[ks][2] = ra ? ra[8 * ks + 4 + tq] : 0u;
            qf[ks][3] = rb ? rb[8 * ks + 4 + tq] : 0u;
        }
    }
    float o[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
    const float sl = a.scale_log2;
    const int mi = lane >> 3, ri = lane & 7;
    bool dead = false;
    int ns_ = 0;  // stages consumed
    for (int i = 0; i < nsel; ++i) {
        const int blk = idx[i];
        if (blk < 0 || blk > r) continue;
        const int slot = ns_ % kPaSlots;
        if (!dead && !mbar_wait(&full[slot], (uint32_t)(ns_ / kPaSlots) & 1u, kPaPolls)) {
            if (lane == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
            dead = true;
        }
        const uint8_t* kst = ring + (size_t)slot * kPaStage;
        const uint8_t* vst = kst + 2 * kPaBox;
        // S = Q K^T: 16 rows x 64 keys (eight 8-key tiles), fp32
        float sc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {  // two 8-key tiles per ldmatrix.x4
                const int key = 16 * np + ri + 8 * (mi >> 1);
                const int ch = (ks & 3) * 2 + (mi & 1);
                uint32_t bf[4];
                ldmatrix_x4(bf, smem_u32(kst + (ks >> 2) * kPaBox + key * 128 + ((ch ^ (key & 7)) << 4)));
                mma_bf16_16816(sc[2 * np], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], bf[0], bf[1]);
                mma_bf16_16816(sc[2 * np + 1], qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3], bf[2], bf[3]);
            }
        }
        // causal mask on the tile's own block; scale to the log2 domain
        const int64_t kbase = (int64_t)blk * a.BS;
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int64_t key = kbase + 8 * nt + 2 * tq + (e & 1);
                const int64_t pos = (e < 2) ? pa : pb;
                const float x = (key <= pos && key < T) ? sc[nt][e] * sl : -INFINITY;
                sc[nt][e] = x;
                mx[e >> 1] = fmaxf(mx[e >> 1], x);
            }
        }
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 1));
            mx[rr] = fmaxf(mx[rr], __shfl_xor_sync(0xffffffffu, mx[rr], 2));
        }
        float alpha[2], ref[2];
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
            const float mn = fmaxf(mrow[rr], mx[rr]);
            alpha[rr] = mn == -INFINITY ? 1.f : exp2f(mrow[rr] - mn);
            ref[rr] = mn == -INFINITY ? 0.f : mn;
            mrow[rr] = mn;
        }
        float ps[2] = {0.f, 0.f};
        // P as the A operand of P V (four 16-key steps), split into bf16 hi + lo parts so that the
        // products keep about 16 significant bits
        uint32_t pf[4][4], pl[4][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const float p0 = exp2f(sc[nt][0] - ref[0]), p1 = exp2f(sc[nt][1] - ref[0]);
            const float p2 = exp2f(sc[nt][2] - ref[1]), p3 = exp2f(sc[nt][3] - ref[1]);
            ps[0] += p0 + p1;
            ps[1] += p2 + p3;
            const int kq = nt >> 1, hi = nt & 1;
            const uint32_t h01 = pack_bf16x2(p0, p1), h23 = pack_bf16x2(p2, p3);
            pf[kq][2 * hi] = h01;
            pf[kq][2 * hi + 1] = h23;
            pl[kq][2 * hi] = pack_bf16x2(p0 - bf16_lo(h01), p1 - bf16_hi(h01));
            pl[kq][2 * hi + 1] = pack_bf16x2(p2 - bf16_lo(h23), p3 - bf16_hi(h23));
        }
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) lrow[rr] = lrow[rr] * alpha[rr] + ps[rr];
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            o[nt][0] *= alpha[0];
            o[nt][1] *= alpha[0];
            o[nt][2] *= alpha[1];
            o[nt][3] *= alpha[1];
        }
        // O += P V: V^T fragments from the swizzled V rows (ldmatrix.trans)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
            for (int dp = 0; dp < 8; ++dp) {  // two 8-column tiles of d per ldmatrix.x4
                const int key = 16 * kk + ri + 8 * (mi & 1);
                const int ch = 2 * dp + (mi >> 1);
                uint32_t vf[4];
                ldmatrix_x4_trans(vf, smem_u32(vst + (ch >> 3) * kPaBox + key * 128 + (((ch & 7) ^ (key & 7)) << 4)));
                mma_bf16_16816(o[2 * dp], pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3], vf[0], vf[1]);
                mma_bf16_16816(o[2 * dp + 1], pf[kk][0], pf[kk][1], pf[kk][2], pf[kk][3], vf[2], vf[3]);
                mma_bf16_16816(o[2 * dp], pl[kk][0], pl[kk][1], pl[kk][2], pl[kk][3], vf[0], vf[1]);
                mma_bf16_16816(o[2 * dp + 1], pl[kk][0], pl[kk][1], pl[kk][2], pl[kk][3], vf[2], vf[3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
        ++ns_;
    }
    // row sums across the quad, then O / l
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        lrow[rr] += __shfl_xor_sync(0xffffffffu, lrow[rr], 1);
        lrow[rr] += __shfl_xor_sync(0xffffffffu, lrow[rr], 2);
    }
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out);
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
        const bool v = rr == 0 ? va : vb;
        if (!v) continue;
        const int64_t pos = rr == 0 ? pa : pb;
        const size_t row = ((size_t)b * a.chunk + (size_t)(pos - t0)) * a.Hq + (size_t)kvh * a.G + h;
        const float inv = lrow[rr] > 0.f ? 1.f / lrow[rr] : 0.f;
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
            const int d0 = 8 * nt + 2 * tq;
            const uint32_t pk = pack_bf16x2(o[nt][2 * rr] * inv, o[nt][2 * rr + 1] * inv);
            *reinterpret_cast<uint32_t*>(out + row * 128 + d0) = pk;
        }
        if (a.lse && tq == 0)
            a.lse[row] = lrow[rr] > 0.f ? (mrow[rr] + log2f(lrow[rr])) * 0.69314718055994531f : -INFINITY;
    }
}

}  // namespace

size_t prefill_select_smem_bytes(int G, int64_t nc_cap, int64_t nb_cap, int sel_cap) {
    const int R = 64 * G;
    size_t bytes = 1024 + (size_t)2 * R * 128 + (size_t)kPsSlots * kPsSlotBytes + (size_t)R * sizeof(float2);
    bytes += (size_t)((nc_cap + 3) & ~int64_t(3)) * 4 + (size_t)((nb_cap + 3) & ~int64_t(3)) * 4 + (size_t)sel_cap * 4;
    const size_t limit = 227 * 1024 - sizeof(TopkSmem) - 256;
    return bytes <= limit ? bytes : 0;
}

size_t prefill_attend_smem_bytes() { return 1024 + (size_t)kPaSlots * kPaStage; }

cudaError_t launch_prefill_select(const PrefillArgs& a, const CUtensorMap* ck_map, size_t smem, int ctas,
                                  cudaStream_t st) {
    if (a.pairs <= 0 || ctas <= 0) return cudaSuccess;
    if (a.G == 2) {
        cudaError_t e = ensure_smem<prefill_select_kernel<128>>(smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(prefill_select_kernel<128>, dim3((unsigned)ctas), dim3(kPsThreads), smem, st, a, *ck_map);
    }
    cudaError_t e = ensure_smem<prefill_select_kernel<256>>(smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(prefill_select_kernel<256>, dim3((unsigned)ctas), dim3(kPsThreads), smem, st, a, *ck_map);
}

cudaError_t launch_prefill_attend(const PrefillArgs& a, const CUtensorMap* k_map, const CUtensorMap* v_map,
                                  cudaStream_t st) {
    const int64_t items = (int64_t)a.pairs * a.tiles_cap * ((a.G + 1) / 2);
    if (items <= 0) return cudaSuccess;
    const size_t smem = prefill_attend_smem_bytes();
    cudaError_t e = ensure_smem<prefill_attend_kernel>(smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(prefill_attend_kernel, dim3((unsigned)items), dim3(kPaThreads), smem, st, a, *k_map, *v_map);
}

}  // namespace bsa
