// Compressed keys (page "SparDA: Sparse Decoupled Attention for Efficient Long-Context LLM
// Inference", Theoretical Foundation, Eq. 2): K~_j = mean of K over rows [s*j, s*j + l).
//
// Both kernels form each window sum in fp64 and round the mean once to the element type
// (round to nearest even). With bf16 or fp32 inputs of ordinary magnitude the fp64 sum of l <= 2^20
// values is exact, so the stored value is the correctly rounded mean.
#include "bsa_internal.cuh"

namespace bsa {
namespace {

template <typename T>
struct Elem;
template <>
struct Elem<float> {
    static constexpr int kPerChunk = 4;  // elements per 16-byte chunk
    __device__ static void widen(const uint4& v, double (&o)[4]) {
        o[0] = __uint_as_float(v.x);
        o[1] = __uint_as_float(v.y);
        o[2] = __uint_as_float(v.z);
        o[3] = __uint_as_float(v.w);
    }
    __device__ static uint4 narrow(const double (&o)[4]) {
        return make_uint4(__float_as_uint(__double2float_rn(o[0])),
                          __float_as_uint(__double2float_rn(o[1])),
                          __float_as_uint(__double2float_rn(o[2])),
                          __float_as_uint(__double2float_rn(o[3])));
    }
};
template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kPerChunk = 8;
    __device__ static void widen(const uint4& v, double (&o)[8]) {
        o[0] = bf16_lo(v.x);
        o[1] = bf16_hi(v.x);
        o[2] = bf16_lo(v.y);
        o[3] = bf16_hi(v.y);
        o[4] = bf16_lo(v.z);
        o[5] = bf16_hi(v.z);
        o[6] = bf16_lo(v.w);
        o[7] = bf16_hi(v.w);
    }
    __device__ static uint32_t pack(double lo, double hi) {
        uint32_t a = __bfloat16_as_ushort(__double2bfloat16(lo));
        uint32_t b = __bfloat16_as_ushort(__double2bfloat16(hi));
        return a | (b << 16);
    }
    __device__ static uint4 narrow(const double (&o)[8]) {
        return make_uint4(pack(o[0], o[1]), pack(o[2], o[3]), pack(o[4], o[5]), pack(o[6], o[7]));
    }
};

// Mean of rows [row0, row0 + l) of one 16-byte chunk column; `coherent` loads bypass L1 (rows
// written earlier by this same kernel).
template <typename T, bool kCoherent>
__device__ __forceinline__ uint4 window_mean(const T* src, int64_t row_stride, int l) {
    constexpr int E = Elem<T>::kPerChunk;
    double acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.0;
    for (int r = 0; r < l; ++r) {
        const T* p = src + (int64_t)r * row_stride;
        uint4 v = kCoherent ? __ldcg(reinterpret_cast<const uint4*>(p)) : ld_stream(p);
        double w[E];
        Elem<T>::widen(v, w);
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] += w[e];
    }
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = acc[e] / (double)l;
    return Elem<T>::narrow(acc);
}

// grid = (pairs, ceil(nc_cap / windows_per_cta)); thread = (window, 16-byte chunk column).
template <typename T, int D>
__global__ void __launch_bounds__(256) compress_keys_kernel(CompressArgs a) {
    constexpr int CH = D * (int)sizeof(T) / 16;
    const int pair = blockIdx.x;
    const int b = pair / a.Hkv;
    const int64_t j = (int64_t)blockIdx.y * a.windows_per_cta + threadIdx.x / CH;
    const int c = threadIdx.x % CH;
    pdl_wait();
    pdl_trigger();
    const int64_t Tb = a.seq_lens[b];
    if (Tb < 0 || Tb > a.T_cap) {
        if (a.err && blockIdx.y == 0 && threadIdx.x == 0 && pair % a.Hkv == 0)
            atomicOr(a.err, (uint32_t)BSA_DEVERR_SEQ_LEN);
        return;
    }
    const int64_t nc = Tb < a.l ? 0 : (Tb - a.l) / a.s + 1;
    if (threadIdx.x >= a.windows_per_cta * CH || j >= nc) return;
    const T* src = reinterpret_cast<const T*>(a.k) + ((int64_t)pair * a.T_cap + j * a.s) * D +
                   c * Elem<T>::kPerChunk;
    uint4 m = window_mean<T, false>(src, D, a.l);
    T* dst = reinterpret_cast<T*>(a.ck) + ((int64_t)pair * a.nc_cap + j) * D + c * Elem<T>::kPerChunk;
    *reinterpret_cast<uint4*>(dst) = m;
}

// grid = B; one CTA appends the new row of every kv head of sequence b, completes the window
// that the new row closes, then advances seq_lens[b] (no other CTA touches that sequence).
template <typename T, int D>
__global__ void __launch_bounds__(256) append_kernel(AppendArgs a) {
    constexpr int E = Elem<T>::kPerChunk;
    constexpr int CH = D / E;
    const int b = blockIdx.x;
    pdl_wait();
    pdl_trigger();
    const int64_t Tb = a.seq_lens[b];
    if (Tb < 0 || Tb >= a.T_cap) {
        if (a.err && threadIdx.x == 0)
            atomicOr(a.err, (uint32_t)(Tb == a.T_cap ? BSA_DEVERR_CAPACITY : BSA_DEVERR_SEQ_LEN));
        return;
    }
    const int work = a.Hkv * CH;
    for (int e = threadIdx.x; e < work; e += blockDim.x) {
        const int h = e / CH, c = e % CH;
        const int64_t pair = (int64_t)b * a.Hkv + h;
        const uint4 kv = *reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(a.k_new) +
                                                         pair * D + c * E);
        const uint4 vv = *reinterpret_cast<const uint4*>(reinterpret_cast<const T*>(a.v_new) +
                                                         pair * D + c * E);
        const int64_t off = (pair * a.T_cap + Tb) * D + c * E;
        *reinterpret_cast<uint4*>(reinterpret_cast<T*>(a.k) + off) = kv;
        *reinterpret_cast<uint4*>(reinterpret_cast<T*>(a.v) + off) = vv;
    }
    const int64_t Tn = Tb + 1;
    __syncthreads();  // the new rows are visible to the whole CTA from here on
    if (Tn >= a.l && (Tn - a.l) % a.s == 0) {
        const int64_t j = (Tn - a.l) / a.s;
        for (int e = threadIdx.x; e < work; e += blockDim.x) {
            const int h = e / CH, c = e % CH;
            const int64_t pair = (int64_t)b * a.Hkv + h;
            const T* src = reinterpret_cast<const T*>(a.k) + (pair * a.T_cap + j * a.s) * D + c * E;
            uint4 m = window_mean<T, true>(src, D, a.l);
            T* dst = reinterpret_cast<T*>(a.ck) + (pair * a.nc_cap + j) * D + c * E;
            *reinterpret_cast<uint4*>(dst) = m;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) a.seq_lens[b] = (int32_t)Tn;
}

template <typename T, int D>
cudaError_t launch_compress_t(const Plan& p, CompressArgs a, cudaStream_t st) {
    constexpr int CH = D * (int)sizeof(T) / 16;
    a.windows_per_cta = 256 / CH;
    const int64_t ny = (p.nc_cap + a.windows_per_cta - 1) / a.windows_per_cta;
    if (ny == 0) return cudaSuccess;
    if (ny > 65535) return cudaErrorInvalidConfiguration;
    return launch_pdl(compress_keys_kernel<T, D>, dim3(p.pairs, (unsigned)ny), dim3(256), 0, st, a);
}

template <typename T, int D>
cudaError_t launch_append_t(const Plan& p, const AppendArgs& a, cudaStream_t st) {
    return launch_pdl(append_kernel<T, D>, dim3(p.B), dim3(256), 0, st, a);
}

}  // namespace

cudaError_t launch_compress_keys(const Plan& p, const CompressArgs& a, cudaStream_t st) {
    if (p.dtype == BSA_BF16)
        return p.D == 128 ? launch_compress_t<__nv_bfloat16, 128>(p, a, st)
                          : launch_compress_t<__nv_bfloat16, 64>(p, a, st);
    return p.D == 128 ? launch_compress_t<float, 128>(p, a, st)
                      : launch_compress_t<float, 64>(p, a, st);
}

cudaError_t launch_append(const Plan& p, const AppendArgs& a, cudaStream_t st) {
    if (p.dtype == BSA_BF16)
        return p.D == 128 ? launch_append_t<__nv_bfloat16, 128>(p, a, st)
                          : launch_append_t<__nv_bfloat16, 64>(p, a, st);
    return p.D == 128 ? launch_append_t<float, 128>(p, a, st) : launch_append_t<float, 64>(p, a, st);
}

}  // namespace bsa
