// meanpool.cu -- averaging initialisation of GQA key/value heads (sm_100a).
//
// "Grouped-Query Attention" (llm-arch-kb), section 2 "Uptraining recipe
// (averaging-init)": each of the G new key (and value) projection heads is the
// mean of the H/G original MHA heads assigned to its group.  Here, for every
// element e of a head's [d_h, d] projection,
//     out[g, e] = (((0 + W[g*r, e]) + W[g*r+1, e]) + ... + W[g*r+r-1, e]) / r
// in IEEE binary64 (ascending head order, correctly rounded division), then one
// round-to-nearest-even to the storage type.  Every step is a correctly
// rounded IEEE operation in a fixed order, so the result is bit-exact with
// that definition.  When r is a power of two the division is a multiplication
// by 1/r: both are exact in binary64 here (the sums of bf16 or fp32 values are
// far above the subnormal range), so the bits are the same and the FP64 pipe
// is spared the division sequence.
//
// Streaming kernel: each thread produces 16 bytes of one output head from r
// independent 16-byte loads (one per input head of its group); K and V are
// handled by the same launch.  HBM-bound: reads 2*H*n and writes 2*G*n
// elements.
//
// The same kernels also build the two alternatives the pages set against the
// mean (section 2 "Uptraining recipe": picking one head per group; section 4:
// a weighted average over a group's heads with per-head weights):
//   MODE_SELECT:   out[g] = W[g*r + sel]                (a copy, exact)
//   MODE_WEIGHTED: out[g] = sum_j w[g*r + j] * W[g*r + j], binary64 products
//                  and sums in ascending j, one rounding.
#include "common.cuh"
#include "gqa.h"
#include "internal.h"

namespace gqa {

namespace {

enum { MODE_MEAN = 0, MODE_SELECT = 1, MODE_WEIGHTED = 2 };

__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_stream(uint4 *p, uint4 v) {
    asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

// acc += wt * v (wt = 1 adds v itself: the product is then exact)
__device__ __forceinline__ void add_bf16x8(double *acc, uint4 v, double wt, bool weighted) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const double lo = (double)__uint_as_float(w[k] << 16);  // exact bf16 -> f32 -> f64
        const double hi = (double)__uint_as_float(w[k] & 0xffff0000u);
        acc[2 * k] = __dadd_rn(acc[2 * k], weighted ? __dmul_rn(wt, lo) : lo);
        acc[2 * k + 1] = __dadd_rn(acc[2 * k + 1], weighted ? __dmul_rn(wt, hi) : hi);
    }
}

__device__ __forceinline__ uint32_t bf16_bits(double x) {
    return (uint32_t)__bfloat16_as_ushort(__double2bfloat16(x));  // nearest-even
}

// 16-byte vectors: bf16 -> 8 elements per vector, fp32 -> 4.
template <bool BF16, int MODE>
__global__ void __launch_bounds__(256) meanpool_vec(const uint4 *__restrict__ wk,
                                                    const uint4 *__restrict__ wv, uint4 *ok,
                                                    uint4 *ov, int r, long long n_vec,
                                                    long long out_vec, const float *wts, int sel,
                                                    unsigned *status) {
    const long long total = 2 * out_vec;
    const double dr = (double)r, inv_r = 1.0 / dr;
    const bool pow2 = (r & (r - 1)) == 0;
    auto mean = [&](double a) { return pow2 ? __dmul_rn(a, inv_r) : __ddiv_rn(a, dr); };
    const int H = (int)(r * (out_vec / n_vec));
    {   // L2 hint for this thread's first vectors, before the wait for the work ahead
        // (addresses only: the values are read after the wait)
        const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
        if (idx < total) {
            const bool is_v = idx >= out_vec;
            const long long v = is_v ? idx - out_vec : idx;
            const long long g = v / n_vec, e = v - g * n_vec;
            if (g * r + r <= H) {
                const uint4 *src = (is_v ? wv : wk) + (g * r) * n_vec + e;
                for (int j = 0; j < r; ++j)
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(src + (long long)j * n_vec));
            }
        }
    }
    pdl_wait_primary();       // inputs written by the work before this kernel are visible
    pdl_launch_dependents();  // the next kernel may set up while this one streams
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const bool is_v = idx >= out_vec;
        const long long v = is_v ? idx - out_vec : idx;
        const long long g = v / n_vec, e = v - g * n_vec;
        if (!index_ok(g * r + r <= H && (MODE != MODE_SELECT || sel < r), status)) continue;
        const uint4 *src = (is_v ? wv : wk) + (g * r) * n_vec + e;
        const float *wg = MODE == MODE_WEIGHTED ? wts + (is_v ? H : 0) + g * r : nullptr;
        if constexpr (MODE == MODE_SELECT) {  // one head of the group, unchanged
            st_stream((is_v ? ov : ok) + v, ld_stream(src + (long long)sel * n_vec));
        } else if constexpr (BF16) {
            double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            for (int j = 0; j < r; ++j)
                add_bf16x8(acc, ld_stream(src + (long long)j * n_vec), MODE == MODE_WEIGHTED ? (double)wg[j] : 1.0,
                           MODE == MODE_WEIGHTED);
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const double a0 = MODE == MODE_MEAN ? mean(acc[2 * k]) : acc[2 * k];
                const double a1 = MODE == MODE_MEAN ? mean(acc[2 * k + 1]) : acc[2 * k + 1];
                o[k] = bf16_bits(a0) | (bf16_bits(a1) << 16);
            }
            st_stream((is_v ? ov : ok) + v, make_uint4(o[0], o[1], o[2], o[3]));
        } else {
            double acc[4] = {0, 0, 0, 0};
            for (int j = 0; j < r; ++j) {
                const uint4 x = ld_stream(src + (long long)j * n_vec);
                const double f[4] = {(double)__uint_as_float(x.x), (double)__uint_as_float(x.y),
                                     (double)__uint_as_float(x.z), (double)__uint_as_float(x.w)};
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    acc[k] = __dadd_rn(acc[k], MODE == MODE_WEIGHTED ? __dmul_rn((double)wg[j], f[k]) : f[k]);
            }
            uint4 o;
            uint32_t *ow = &o.x;
#pragma unroll
            for (int k = 0; k < 4; ++k)
                ow[k] = __float_as_uint(__double2float_rn(MODE == MODE_MEAN ? mean(acc[k]) : acc[k]));
            st_stream((is_v ? ov : ok) + v, o);
        }
    }
}

// Element-wise variant for sizes or addresses that are not 16-byte multiples.
template <bool BF16, int MODE>
__global__ void __launch_bounds__(256) meanpool_scalar(const void *wk, const void *wv, void *ok,
                                                       void *ov, int r, long long n,
                                                       long long out_n, const float *wts, int sel,
                                                       unsigned *status) {
    pdl_wait_primary();
    pdl_launch_dependents();
    const long long total = 2 * out_n;
    const double dr = (double)r, inv_r = 1.0 / dr;
    const bool pow2 = (r & (r - 1)) == 0;
    auto mean = [&](double a) { return pow2 ? __dmul_rn(a, inv_r) : __ddiv_rn(a, dr); };
    const int H = (int)(r * (out_n / n));
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const bool is_v = idx >= out_n;
        const long long v = is_v ? idx - out_n : idx;
        const long long g = v / n, e = v - g * n;
        if (!index_ok(g * r + r <= H && (MODE != MODE_SELECT || sel < r), status)) continue;
        const float *wg = MODE == MODE_WEIGHTED ? wts + (is_v ? H : 0) + g * r : nullptr;
        double acc = 0.0;
        if constexpr (BF16) {
            const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(is_v ? wv : wk) + g * r * n + e;
            if constexpr (MODE == MODE_SELECT) {
                static_cast<__nv_bfloat16 *>(is_v ? ov : ok)[v] = src[(long long)sel * n];
            } else {
                for (int j = 0; j < r; ++j) {
                    const double x = (double)__bfloat162float(src[(long long)j * n]);
                    acc = __dadd_rn(acc, MODE == MODE_WEIGHTED ? __dmul_rn((double)wg[j], x) : x);
                }
                static_cast<__nv_bfloat16 *>(is_v ? ov : ok)[v] =
                    __double2bfloat16(MODE == MODE_MEAN ? mean(acc) : acc);
            }
        } else {
            const float *src = static_cast<const float *>(is_v ? wv : wk) + g * r * n + e;
            if constexpr (MODE == MODE_SELECT) {
                static_cast<float *>(is_v ? ov : ok)[v] = src[(long long)sel * n];
            } else {
                for (int j = 0; j < r; ++j) {
                    const double x = (double)src[(long long)j * n];
                    acc = __dadd_rn(acc, MODE == MODE_WEIGHTED ? __dmul_rn((double)wg[j], x) : x);
                }
                static_cast<float *>(is_v ? ov : ok)[v] =
                    __double2float_rn(MODE == MODE_MEAN ? mean(acc) : acc);
            }
        }
    }
}

// Launched as programmatic dependents: the kernels ask L2 for their first
// inputs (a hint) and then wait for the work ahead of them on the stream
// before they read or write anything.
cudaLaunchConfig_t pdl_config(unsigned blocks, int threads, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    return cfg;
}
void pdl_attr(cudaLaunchConfig_t &cfg, cudaLaunchAttribute (&attr)[1]) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
}

template <int MODE>
cudaError_t launch_mode(const void *wk, const void *wv, void *ok, void *ov, int H, int G, long long n, bool bf16,
                        bool aligned, int num_sms, const float *wts, int sel, unsigned *status,
                        cudaStream_t st) {
    const int r = H / G;
    const int per_vec = bf16 ? 8 : 4;
    const long long out_elems = (long long)G * n;
    const int threads = 256;
    const long long cap = (long long)num_sms * 16;
    if (aligned && n % per_vec == 0) {
        const long long n_vec = n / per_vec, out_vec = (long long)G * n_vec;
        long long blocks = (2 * out_vec + threads - 1) / threads;
        if (blocks > cap) blocks = cap;
        auto kern = bf16 ? meanpool_vec<true, MODE> : meanpool_vec<false, MODE>;
        cudaLaunchConfig_t cfg = pdl_config((unsigned)blocks, threads, st);
        cudaLaunchAttribute attr[1];
        pdl_attr(cfg, attr);
        cudaError_t le = cudaLaunchKernelEx(&cfg, kern, static_cast<const uint4 *>(wk), static_cast<const uint4 *>(wv),
                                            static_cast<uint4 *>(ok), static_cast<uint4 *>(ov), r, n_vec, out_vec, wts,
                                            sel, status);
        if (le != cudaSuccess) return le;
    } else {
        long long blocks = (2 * out_elems + threads - 1) / threads;
        if (blocks > cap) blocks = cap;
        auto kern = bf16 ? meanpool_scalar<true, MODE> : meanpool_scalar<false, MODE>;
        cudaLaunchConfig_t cfg = pdl_config((unsigned)blocks, threads, st);
        cudaLaunchAttribute attr[1];
        pdl_attr(cfg, attr);
        cudaError_t le = cudaLaunchKernelEx(&cfg, kern, wk, wv, ok, ov, r, n, out_elems, wts, sel, status);
        if (le != cudaSuccess) return le;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_meanpool(const void *wk, const void *wv, void *ok, void *ov, int H, int G, long long n,
                            int dtype, int num_sms, unsigned *status, cudaStream_t st) {
    return launch_init_heads(wk, wv, ok, ov, H, G, n, dtype, 0, nullptr, 0, num_sms, status, st);
}

cudaError_t launch_init_heads(const void *wk, const void *wv, void *ok, void *ov, int H, int G, long long n,
                              int dtype, int mode, const float *weights, int select, int num_sms,
                              unsigned *status, cudaStream_t st) {
    const bool bf16 = dtype == GQA_BF16;
    const bool aligned = ((reinterpret_cast<uintptr_t>(wk) | reinterpret_cast<uintptr_t>(wv) |
                           reinterpret_cast<uintptr_t>(ok) | reinterpret_cast<uintptr_t>(ov)) &
                          15) == 0;
    if ((long long)G * n == 0) return cudaSuccess;
    switch (mode) {
        case MODE_SELECT:
            return launch_mode<MODE_SELECT>(wk, wv, ok, ov, H, G, n, bf16, aligned, num_sms, weights, select, status, st);
        case MODE_WEIGHTED:
            return launch_mode<MODE_WEIGHTED>(wk, wv, ok, ov, H, G, n, bf16, aligned, num_sms, weights, select, status, st);
        default:
            return launch_mode<MODE_MEAN>(wk, wv, ok, ov, H, G, n, bf16, aligned, num_sms, weights, select, status, st);
    }
}

}  // namespace gqa
