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
// buffers), read back with tcgen05.ld by eight epilogue warps, two per TMEM lane quarter, each
// taking half of the columns; one warp issues the TMA copies and one thread the MMAs (tcgen05.mma,
// completion through tcgen05.commit on shared-memory barriers).
//
// Attention kernel (tcgen05): a CTA per (pair, tile) holds the tile's R rows in shared memory as
// 128-row halves; the selected blocks' K and V rows stream through a TMA ring. For each block one
// thread issues S = Q K^T (M = 128 rows, N = 64 keys) into a double-buffered TMEM accumulator per
// half; eight warps per half read it back (two threads per row, 32 scores each), take the online
// softmax in the log2 domain and write P as bf16 over S in TMEM; the same thread then issues
// O += P V (A = P from TMEM, N = 128, V read MN-major from its TMA rows) into a TMEM accumulator.
// The issuing thread takes whichever is ready first, S of a later block or P V of a half whose P is
// written, so the tensor cores work while the softmax runs. A row's
// reference maximum moves only when the block maximum exceeds it by more than 8 (log2), so P stays
// below 2^8 and O is rescaled in TMEM rarely; O / sum is exact either way.
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

// 2^x by the special-function unit (PTX ex2.approx.ftz: relative error about 2^-22, results below
// 2^-126 flushed to zero, 2^-inf = 0).
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ------------------------------------------------------------------------------ selection kernel
constexpr int kPsEpiWarps = 8;          // two groups of four epilogue warps
constexpr int kPsEpiThreads = kPsEpiWarps * 32;
constexpr int kPsWarps = 2 + kPsEpiWarps;  // producer, MMA issuer, epilogue
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
    float2* part = reinterpret_cast<float2*>(ring + kPsSlots * kPsSlotBytes);  // [2][128] (max, sum) per group
    float* mz = reinterpret_cast<float*>(part + 256);  // [R] max + log2(sum) of each row, log2 domain
    float* S = mz + R;                                 // [nc_cap] window scores
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
            mbar_init(&acce[i], kPsEpiWarps);
        }
        mbar_init(&qready, kPsEpiThreads);
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
        // Group eg (warps 2 + 4 eg .. 5 + 4 eg) reads NL = R / 2 columns of each accumulator: in
        // pass 1 the windows of its half (R = 128) or all 128 windows of row block eg (R = 256); in
        // pass 2 the rows eg NL .. eg NL + NL - 1.
        constexpr int NL = R / 2;
        const int et = threadIdx.x - 64;                    // 0 .. 255
        const int eg = et >> 7;
        const Grp grp{et, kPsEpiThreads, kPsEpiBar};
        const int quarter = warp & 3;                       // TMEM lanes 32 * quarter ..
        const int ml = 32 * quarter + lane;                 // this thread's TMEM lane
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
                for (int i = et; i < a.sel_cap; i += kPsEpiThreads) oidx[i] = -1;
                if (et == 0) a.n_sel[g] = 0;
                continue;
            }
            topk_prepare(tk, grp);
            // the tile's rows into shared memory (row = position-in-block * G + head), K-major with
            // the 128-byte swizzle; rows outside the chunk are zero
            const int G = a.G;
            for (int e = et; e < R * 16; e += kPsEpiThreads) {
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
            // ---- pass 1: the softmax maximum and sum of row (R = 256: eg * 128 +) ml over the
            // group's windows
            float m = -INFINITY, z = 0.f;
            for (int c = 0; c < it.nch; ++c, ++n) {
                const int buf = (int)(n & 1);
                if (!dead && !mbar_wait(&accf[buf], (uint32_t)(n >> 1) & 1u, kPsPolls)) {
                    if (lane == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                    dead = true;
                }
                tmem_fence_after_sync();
                float v[NL];
#pragma unroll
                for (int pc = 0; pc < NL / 32; ++pc)
                    tmem_ld<32>(tbase + lane_off + (uint32_t)(buf * 256 + eg * NL + pc * 32),
                                *reinterpret_cast<float(*)[32]>(v + 32 * pc));
                tmem_wait_ld();
                tmem_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce[buf]);
                const int nv = min(NL, it.nc - (kPsChunk * c + (R == 128 ? eg * NL : 0)));  // valid windows
                if (nv > 0) {
                    float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int e = 0; e < NL; ++e)
                        if (e < nv) mq[e & 3] = fmaxf(mq[e & 3], v[e]);
                    const float mn = fmaxf(m, fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3])) * sl);  // sl > 0
                    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int e = 0; e < NL; ++e)
                        if (e < nv) acc[e & 3] += ex2_ftz(fmaf(v[e], sl, -mn));
                    z = (m == -INFINITY ? 0.f : z * ex2_ftz(m - mn)) + ((acc[0] + acc[1]) + (acc[2] + acc[3]));
                    m = mn;
                }
            }
            part[eg * 128 + ml] = make_float2(m, z);
            grp.sync();
            // merge the groups' halves (R = 128) and form max + log2(sum) per row; zero the scores
            for (int row = et; row < R; row += kPsEpiThreads) {
                float2 mzr = part[row];
                if (R == 128) {
                    const float2 o = part[128 + row];
                    const float mn = fmaxf(mzr.x, o.x);
                    if (mn != -INFINITY)
                        mzr = make_float2(mn, (mzr.y > 0.f ? mzr.y * exp2f(mzr.x - mn) : 0.f) +
                                                  (o.y > 0.f ? o.y * exp2f(o.x - mn) : 0.f));
                }
                const int64_t p = (int64_t)a.BS * it.r + row / G;
                const bool valid = row < 64 * G && p >= it.t0 && p < it.T && mzr.y > 0.f;
                mz[row] = valid ? mzr.x + log2f(mzr.y) : INFINITY;  // a row outside the chunk adds 0
            }
            for (int j = et; j < it.nc; j += kPsEpiThreads) S[j] = 0.f;
            grp.sync();
            // ---- pass 2: window kPsChunk c + ml of each stage: the sum over the group's rows of
            // exp2(x - max - log2 sum); the two groups' sums meet in S (0 + a + b is exact in either order)
            for (int c = 0; c < it.nch; ++c, ++n) {
                const int buf = (int)(n & 1);
                if (!dead && !mbar_wait(&accf[buf], (uint32_t)(n >> 1) & 1u, kPsPolls)) {
                    if (lane == 0) atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                    dead = true;
                }
                tmem_fence_after_sync();
                float v[NL];
#pragma unroll
                for (int pc = 0; pc < NL / 32; ++pc)
                    tmem_ld<32>(tbase + lane_off + (uint32_t)(buf * 256 + eg * NL + pc * 32),
                                *reinterpret_cast<float(*)[32]>(v + 32 * pc));
                tmem_wait_ld();
                tmem_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acce[buf]);
                const float4* mz4 = reinterpret_cast<const float4*>(mz + eg * NL);
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int e4 = 0; e4 < NL / 4; ++e4) {
                    const float4 w = mz4[e4];
                    acc[0] += ex2_ftz(fmaf(v[4 * e4], sl, -w.x));
                    acc[1] += ex2_ftz(fmaf(v[4 * e4 + 1], sl, -w.y));
                    acc[2] += ex2_ftz(fmaf(v[4 * e4 + 2], sl, -w.z));
                    acc[3] += ex2_ftz(fmaf(v[4 * e4 + 3], sl, -w.w));
                }
                const int j = kPsChunk * c + ml;
                if (j < it.nc) atomicAdd(&S[j], (acc[0] + acc[1]) + (acc[2] + acc[3]));
            }
            grp.sync();
            // ---- block maxima over blocks 0 .. r: block b's windows are 4b - 1 .. 4b + 3
            const int nb = (int)it.r + 1;
            for (int bb = et; bb < nb; bb += kPsEpiThreads) {
                float mx = -INFINITY;
                for (int j = max(4 * bb - 1, 0); j <= 4 * bb + 3 && j < it.nc; ++j) mx = fmaxf(mx, S[j]);
                keys[bb] = order_key(mx);
            }
            grp.sync();
            topk_union(sa, nb, keys, tk, false, grp, sel, &s_nsel);
            grp.sync();
            for (int i = et; i < a.sel_cap; i += kPsEpiThreads) oidx[i] = sel[i];
            if (et == 0) a.n_sel[g] = s_nsel;
            grp.sync();  // sel, keys, mz and S are rewritten by the next item
        }
    }
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 1) tmem_dealloc(tbase, 512);
}

// ------------------------------------------------------------------------------ attention kernel
constexpr int kPaSlots = 4;                    // K + V block stages in flight
constexpr uint32_t kPaBox = 64u * 128u;        // 64 rows x 64 columns of bf16
constexpr uint32_t kPaStage = 4u * kPaBox;     // K (two boxes) and V (two boxes) of one 64-token block
constexpr uint32_t kPaPolls = 1u << 26;
constexpr float kPaHeadroom = 8.f;             // log2 growth of a row maximum absorbed without rescaling O

// Shared-memory descriptor of an MN-major operand in the 128-byte swizzle: 64 values of the N
// dimension per 128-byte row, one row per K index, 8-row groups 1024 bytes apart and the next 64
// values of N `lbo` bytes further (V as the B operand of P V: N = d, K = keys).
__device__ __forceinline__ uint64_t umma_desc_mn_sw128(uint32_t saddr, uint32_t lbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) | (64ull << 32) |
           (1ull << 46) | (2ull << 61);
}
// P V: bf16 x bf16 -> fp32, M = 128 rows, N = 128 values of d, A (P, in TMEM) K-major, B (V) MN-major.
constexpr uint32_t kPaIdescPV = umma_idesc_bf16(128, 128) | (1u << 16);
// D (TMEM) = A (TMEM: row i in lane i, two bf16 per 32-bit column) * B^T (+ D when acc).
__device__ __forceinline__ void umma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t bdesc, uint32_t idesc,
                                             uint32_t acc) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(tmem_d),
        "r"(tmem_a), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}
// Non-blocking test of a barrier phase (true once the phase with the given parity has completed).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// H: 128-row halves of the tile (G = 2: one; G = 4: two). Warp 0 issues the TMA copies, warp 1
// allocates tensor memory; one thread per half issues that half's MMAs (warp 1 for half 0, warp
// 2 + 8H for half 1); warps 2 .. 2 + 8H - 1 run the softmax of half (warp - 2) / 8, two threads per
// tile row (its TMEM lane), 32 scores each.
template <int H>
__global__ void __launch_bounds__((2 + 9 * H - 1) * 32, 1)
    prefill_attend_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap k_map,
                          const __grid_constant__ CUtensorMap v_map) {
    constexpr int R = 128 * H;
    extern __shared__ uint8_t dsm_raw[];
    __shared__ __align__(8) uint64_t full_k[kPaSlots], full_v[kPaSlots], empty[kPaSlots], qready, fin;
    __shared__ __align__(8) uint64_t s_full[H][2], p_full[H][2], o_done[H];
    __shared__ float xm[2][H][2][128];  // [block parity][half][column group][row]: partial maxima
    __shared__ uint32_t s_tmem;
    uint8_t* qt = dsm_raw + ((1024u - (smem_u32(dsm_raw) & 1023u)) & 1023u);  // 2 boxes x R rows x 128 B
    uint8_t* ring = qt + 2 * R * 128;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.x;  // pair * tiles_cap + tile
    const int pair = g / a.tiles_cap, ti = g - pair * a.tiles_cap;
    const int b = pair / a.Hkv, kvh = pair - b * a.Hkv;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kPaSlots; ++i) {
            mbar_init(&full_k[i], 1);
            mbar_init(&full_v[i], 1);
            mbar_init(&empty[i], H);  // one release per half
        }
        mbar_init(&qready, 256 * H);
        mbar_init(&fin, H);
        for (int h = 0; h < H; ++h) {
            for (int u = 0; u < 2; ++u) {
                mbar_init(&s_full[h][u], 1);
                mbar_init(&p_full[h][u], 8);
            }
            mbar_init(&o_done[h], 1);
        }
        mbar_fence_init();
    }
    if (warp == 1) tmem_alloc(&s_tmem, 256 * H);
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    // TMEM columns: S of half h, buffer u at 64 (2h + u); O of half h at 128 H + 128 h
    const uint32_t tbase = s_tmem;
    pdl_trigger();
    pdl_wait();
    const int64_t T = a.seq_lens[b];
    const bool ok = T >= a.chunk && T <= a.T_cap;
    const int64_t t0 = T - a.chunk, r = t0 / a.BS + ti;
    const bool live = ok && r <= (T - 1) / a.BS;
    const int nsel = live ? min(max(a.n_sel[g], 0), a.sel_cap) : 0;
    const int32_t* idx = a.block_idx + (size_t)g * a.sel_cap;
    // entries outside blocks 0 .. r are skipped by every role alike; j counts the others

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int j = 0;
            for (int i = 0; i < nsel; ++i) {
                const int blk = idx[i];
                if (blk < 0 || blk > r) continue;
                const int slot = j % kPaSlots;
                if (j >= kPaSlots && !mbar_wait(&empty[slot], (uint32_t)((j / kPaSlots) - 1) & 1u, kPaPolls)) {
                    atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                    break;
                }
                uint8_t* dst = ring + (size_t)slot * kPaStage;
                const int y = (int)((int64_t)pair * a.T_cap + (int64_t)blk * a.BS);
                mbar_arrive_expect_tx(&full_k[slot], 2 * kPaBox);
                tma_load_2d(dst, &k_map, 0, y, &full_k[slot]);
                tma_load_2d(dst + kPaBox, &k_map, 64, y, &full_k[slot]);
                mbar_arrive_expect_tx(&full_v[slot], 2 * kPaBox);
                tma_load_2d(dst + 2 * kPaBox, &v_map, 0, y, &full_v[slot]);
                tma_load_2d(dst + 3 * kPaBox, &v_map, 64, y, &full_v[slot]);
                ++j;
            }
            // every copy issued has landed before the CTA ends (they already have, unless a wait gave up)
            for (int jj = max(j - kPaSlots, 0); jj < j; ++jj)
                if (!mbar_wait(&full_k[jj % kPaSlots], (uint32_t)(jj / kPaSlots) & 1u, kPaPolls) ||
                    !mbar_wait(&full_v[jj % kPaSlots], (uint32_t)(jj / kPaSlots) & 1u, kPaPolls)) {
                    atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                    break;
                }
        }
    } else if (warp == 1 || warp == 2 + 8 * H) {
        // ---------------------------------------------------------------- MMA issuers
        // One thread per half takes whichever is ready first: S of its next block (the K landed;
        // the half's TMEM buffer is free once its P V of two blocks back is issued: that P V needed
        // the softmax to have read the S, and it reads the P written over it before the later S, in
        // issue order) or P V of its next block (the half's P written, the V landed). Each half
        // releases a K/V stage after its P V of that block (the commit fires when its MMAs complete).
        if (lane == 0) {
            const int h = warp == 1 ? 0 : 1;
            int n = 0;
            for (int i = 0; i < nsel; ++i) {
                const int blk = idx[i];
                n += (blk >= 0 && blk <= r) ? 1 : 0;
            }
            const uint32_t qt_a = smem_u32(qt), ring_a = smem_u32(ring);
            const uint32_t q_a = qt_a + (uint32_t)(h * 128 * 128);
            const uint32_t d_o = tbase + (uint32_t)(128 * H + 128 * h);
            int ns = 0, npv = 0;
            bool stop = n > 0 && !mbar_wait(&qready, 0, kPaPolls);
            uint32_t idle = 0;
            while (!stop && npv < n) {
                bool progress = false;
                if (ns < n && ns <= npv + 1 && mbar_test(&full_k[ns % kPaSlots], (uint32_t)(ns / kPaSlots) & 1u)) {
                    tmem_fence_after_sync();
                    const uint32_t k_a = ring_a + (uint32_t)(ns % kPaSlots) * kPaStage;
                    const uint32_t d = tbase + (uint32_t)(64 * (2 * h + (ns & 1)));
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t off = (uint32_t)((ks & 3) * 32);
                        umma_bf16(d, umma_desc_k_sw128(q_a + (uint32_t)((ks >> 2) * R * 128) + off),
                                  umma_desc_k_sw128(k_a + (uint32_t)((ks >> 2) * kPaBox) + off),
                                  umma_idesc_bf16(128, 64), ks > 0);
                    }
                    umma_commit(&s_full[h][ns & 1]);
                    ++ns;
                    progress = true;
                }
                const int j = npv;
                // P of block j sits in S buffer j & 1; its barrier completes once per two blocks, and
                // the softmax cannot write P of block j + 2 before S of block j + 2, which waits for
                // this P V
                if (j < ns && mbar_test(&p_full[h][j & 1], (uint32_t)(j >> 1) & 1u) &&
                    mbar_test(&full_v[j % kPaSlots], (uint32_t)(j / kPaSlots) & 1u)) {
                    tmem_fence_after_sync();
                    const uint32_t v_a = ring_a + (uint32_t)(j % kPaSlots) * kPaStage + 2 * kPaBox;
                    const uint32_t pa = tbase + (uint32_t)(64 * (2 * h + (j & 1)));  // P over S of block j
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)  // 16 keys (8 columns of P) per MMA
                        umma_bf16_ts(d_o, pa + (uint32_t)(kk * 8),
                                     umma_desc_mn_sw128(v_a + (uint32_t)(kk * 2048), kPaBox), kPaIdescPV,
                                     (j > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&o_done[h]);
                    umma_commit(&empty[j % kPaSlots]);
                    npv = j + 1;
                    progress = true;
                }
                if (progress) idle = 0;
                else if (++idle > 4 * kPaPolls) stop = true;
            }
            if (stop) atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
            // every MMA issued has completed before the tensor memory is released
            umma_commit(&fin);
            if (!mbar_wait(&fin, 0, kPaPolls)) atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
        }
    } else {
        // ---------------------------------------------------------------- softmax warps
        // Row m of half h is shared by the threads of column groups cg = 0 and 1 (scores 32 cg ..
        // 32 cg + 31, O columns 64 cg .. 64 cg + 63), lane m % 32 of two warps that reach the same
        // TMEM lanes; the pair exchanges its maxima (and at the end its sums) through shared memory
        // behind a named barrier of its 64 threads, so both take the same rescaling decisions.
        const int sw = warp - 2;
        const int h = sw >> 3, cg = (sw >> 2) & 1;      // half, column group
        const int quarter = warp & 3;                   // TMEM lanes 32 * quarter ..
        const int m = 32 * quarter + lane;              // row within the half (TMEM lane)
        const int row = 128 * h + m;                    // tile row: position-in-block * G + head
        const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
        const uint32_t pair_bar = (uint32_t)(1 + 4 * h + quarter);
        const int G = a.G;
        // the tile's rows into shared memory, K-major with the 128-byte swizzle; rows outside the
        // chunk are zero
        if (live) {
            for (int e = threadIdx.x - 64; e < R * 16; e += 256 * H) {
                const int rr = e >> 4, ch = e & 15;
                const int cp = rr / G, hh = rr - cp * G;
                const int64_t p = (int64_t)a.BS * r + cp;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (rr < 64 * G && p >= t0 && p < T)
                    v = *reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(a.q) +
                                                        (((size_t)b * a.chunk + (size_t)(p - t0)) * a.Hq +
                                                         (size_t)kvh * G + hh) * 128 + ch * 8);
                *reinterpret_cast<uint4*>(qt + (ch >> 3) * R * 128 + rr * 128 + (((ch & 7) ^ (rr & 7)) << 4)) = v;
            }
            fence_proxy_async_smem();
        }
        mbar_arrive(&qready);
        const int cpos = row / G, hd = row - cpos * G;
        const int64_t pos = (int64_t)a.BS * r + cpos;
        const bool valid = live && row < 64 * G && pos >= t0 && pos < T;
        const float sl = a.scale_log2;
        const uint32_t t_o = tbase + lane_off + (uint32_t)(128 * H + 128 * h + 64 * cg);
        float m_used = -INFINITY, lsum = 0.f;  // log2-domain reference maximum and (partial) sum of the row
        bool dead = false;
        int j = 0;
        for (int i = 0; i < nsel; ++i) {
            const int blk = idx[i];
            if (blk < 0 || blk > r) continue;
            const int u = j & 1;
            if (!dead && !mbar_wait(&s_full[h][u], (uint32_t)(j >> 1) & 1u, kPaPolls)) {
                atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                dead = true;
            }
            tmem_fence_after_sync();
            float x[32];
            tmem_ld<32>(tbase + lane_off + (uint32_t)(64 * (2 * h + u) + 32 * cg), x);
            tmem_wait_ld();
            // causal mask inside the tile's own block
            if (blk == r) {
#pragma unroll
                for (int c = 0; c < 32; ++c) x[c] = 32 * cg + c <= cpos ? x[c] : -INFINITY;
            }
            float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int c = 0; c < 32; ++c) mq[c & 3] = fmaxf(mq[c & 3], x[c]);
            const float pm = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
            xm[u][h][cg][m] = pm;
            asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
            const float mx = fmaxf(pm, xm[u][h][cg ^ 1][m]) * sl;  // log2 domain (sl > 0)
            // the reference maximum moves (and O and the sum are rescaled) only when the row's
            // maximum exceeds it by more than the headroom: P stays below 2^8
            const bool need = mx > m_used + kPaHeadroom;
            if (__any_sync(0xffffffffu, need)) {
                const float mn = need ? mx : m_used;
                const float alpha = m_used == -INFINITY ? 0.f : ex2_ftz(m_used - mn);
                if (j > 0) {
                    // O holds P V of blocks 0 .. j - 1 once the last of them has completed
                    if (!dead && !mbar_wait(&o_done[h], (uint32_t)(j - 1) & 1u, kPaPolls)) {
                        atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                        dead = true;
                    }
                    tmem_fence_after_sync();
#pragma unroll 1
                    for (int cc = 0; cc < 2; ++cc) {
                        float o[32];
                        tmem_ld<32>(t_o + (uint32_t)(32 * cc), o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] *= alpha;
                        tmem_st<32>(t_o + (uint32_t)(32 * cc), o);
                    }
                    tmem_wait_st();
                }
                lsum *= alpha;
                m_used = mn;
            }
            uint32_t pk[16];
            float ps[4] = {0.f, 0.f, 0.f, 0.f};
            const float nref = m_used == -INFINITY ? 0.f : -m_used;  // a row with no finite score so far
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float p0 = ex2_ftz(fmaf(x[2 * c], sl, nref)), p1 = ex2_ftz(fmaf(x[2 * c + 1], sl, nref));
                ps[(2 * c) & 3] += p0;
                ps[(2 * c + 1) & 3] += p1;
                pk[c] = pack_bf16x2(p0, p1);
            }
            lsum += (ps[0] + ps[1]) + (ps[2] + ps[3]);
            // P over the row's S in TMEM (keys 32 cg .. 32 cg + 31 -> columns 16 cg .. 16 cg + 15; both
            // threads of the row have read their S before the pair barrier above)
            tmem_st<16>(tbase + lane_off + (uint32_t)(64 * (2 * h + u) + 16 * cg), *reinterpret_cast<float(*)[16]>(pk));
            tmem_wait_st();
            tmem_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[h][u]);
            ++j;
        }
        // ---- the row's sum from both threads (in the maxima buffer the last block did not use),
        // then O / sum
        xm[j & 1][h][cg][m] = lsum;
        asm volatile("bar.sync %0, 64;" ::"r"(pair_bar) : "memory");
        lsum += xm[j & 1][h][cg ^ 1][m];
        const size_t orow = ((size_t)b * a.chunk + (size_t)(valid ? pos - t0 : 0)) * a.Hq + (size_t)kvh * G + hd;
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(a.out) + orow * 128 + 64 * cg;
        if (j > 0) {
            if (!dead && !mbar_wait(&o_done[h], (uint32_t)(j - 1) & 1u, kPaPolls)) {
                atomicOr(a.err, (uint32_t)BSA_DEVERR_TIMEOUT);
                dead = true;
            }
            tmem_fence_after_sync();
            const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
#pragma unroll 1
            for (int cc = 0; cc < 2; ++cc) {
                float o[32];
                tmem_ld<32>(t_o + (uint32_t)(32 * cc), o);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        *reinterpret_cast<uint4*>(out + 32 * cc + 8 * q4) =
                            make_uint4(pack_bf16x2(o[8 * q4] * inv, o[8 * q4 + 1] * inv),
                                       pack_bf16x2(o[8 * q4 + 2] * inv, o[8 * q4 + 3] * inv),
                                       pack_bf16x2(o[8 * q4 + 4] * inv, o[8 * q4 + 5] * inv),
                                       pack_bf16x2(o[8 * q4 + 6] * inv, o[8 * q4 + 7] * inv));
                }
            }
        } else if (valid) {
            for (int q4 = 0; q4 < 8; ++q4) *reinterpret_cast<uint4*>(out + 8 * q4) = make_uint4(0, 0, 0, 0);
        }
        if (valid && cg == 0 && a.lse)
            a.lse[orow] = lsum > 0.f ? (m_used + log2f(lsum)) * 0.69314718055994531f : -INFINITY;
    }
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 1) tmem_dealloc(tbase, 256 * H);
}

}  // namespace

size_t prefill_select_smem_bytes(int G, int64_t nc_cap, int64_t nb_cap, int sel_cap) {
    const int R = 64 * G;
    size_t bytes = 1024 + (size_t)2 * R * 128 + (size_t)kPsSlots * kPsSlotBytes + 256 * sizeof(float2) + (size_t)R * 4;
    bytes += (size_t)((nc_cap + 3) & ~int64_t(3)) * 4 + (size_t)((nb_cap + 3) & ~int64_t(3)) * 4 + (size_t)sel_cap * 4;
    const size_t limit = 227 * 1024 - sizeof(TopkSmem) - 256;
    return bytes <= limit ? bytes : 0;
}

size_t prefill_attend_smem_bytes(int G) {
    const int H = G > 2 ? 2 : 1;
    return 1024 + (size_t)2 * 128 * H * 128 + (size_t)kPaSlots * kPaStage;
}

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
    const int64_t items = (int64_t)a.pairs * a.tiles_cap;
    if (items <= 0) return cudaSuccess;
    const size_t smem = prefill_attend_smem_bytes(a.G);
    if (a.G == 2) {
        cudaError_t e = ensure_smem<prefill_attend_kernel<1>>(smem);
        if (e != cudaSuccess) return e;
        return launch_pdl(prefill_attend_kernel<1>, dim3((unsigned)items), dim3(10 * 32), smem, st, a, *k_map, *v_map);
    }
    cudaError_t e = ensure_smem<prefill_attend_kernel<2>>(smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(prefill_attend_kernel<2>, dim3((unsigned)items), dim3(19 * 32), smem, st, a, *k_map, *v_map);
}

}  // namespace bsa
