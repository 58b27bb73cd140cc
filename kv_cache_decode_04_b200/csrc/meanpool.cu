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
// that definition.
//
// Streaming kernel: each thread produces 16 bytes of one output head from r
// independent 16-byte loads (one per input head of its group); K and V are
// handled by the same launch.  HBM-bound: reads 2*H*n and writes 2*G*n
// elements.
#include "common.cuh"
#include "gqa.h"
#include "internal.h"

namespace gqa {

namespace {

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

__device__ __forceinline__ void add_bf16x8(double *acc, uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float lo = __uint_as_float(w[k] << 16);          // exact bf16 -> f32
        const float hi = __uint_as_float(w[k] & 0xffff0000u);
        acc[2 * k] = __dadd_rn(acc[2 * k], (double)lo);
        acc[2 * k + 1] = __dadd_rn(acc[2 * k + 1], (double)hi);
    }
}

__device__ __forceinline__ uint32_t bf16_bits(double x) {
    return (uint32_t)__bfloat16_as_ushort(__double2bfloat16(x));  // nearest-even
}

// 16-byte vectors: bf16 -> 8 elements per vector, fp32 -> 4.
template <bool BF16>
__global__ void __launch_bounds__(256) meanpool_vec(const uint4 *__restrict__ wk,
                                                    const uint4 *__restrict__ wv, uint4 *ok,
                                                    uint4 *ov, int r, long long n_vec,
                                                    long long out_vec) {
    const long long total = 2 * out_vec;
    const double dr = (double)r;
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const bool is_v = idx >= out_vec;
        const long long v = is_v ? idx - out_vec : idx;
        const long long g = v / n_vec, e = v - g * n_vec;
        const uint4 *src = (is_v ? wv : wk) + (g * r) * n_vec + e;
        if (BF16) {
            double acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            for (int j = 0; j < r; ++j) add_bf16x8(acc, ld_stream(src + (long long)j * n_vec));
            uint32_t o[4];
#pragma unroll
            for (int k = 0; k < 4; ++k)
                o[k] = bf16_bits(__ddiv_rn(acc[2 * k], dr)) |
                       (bf16_bits(__ddiv_rn(acc[2 * k + 1], dr)) << 16);
            st_stream((is_v ? ov : ok) + v, make_uint4(o[0], o[1], o[2], o[3]));
        } else {
            double acc[4] = {0, 0, 0, 0};
            for (int j = 0; j < r; ++j) {
                const uint4 x = ld_stream(src + (long long)j * n_vec);
                acc[0] = __dadd_rn(acc[0], (double)__uint_as_float(x.x));
                acc[1] = __dadd_rn(acc[1], (double)__uint_as_float(x.y));
                acc[2] = __dadd_rn(acc[2], (double)__uint_as_float(x.z));
                acc[3] = __dadd_rn(acc[3], (double)__uint_as_float(x.w));
            }
            uint4 o;
            o.x = __float_as_uint(__double2float_rn(__ddiv_rn(acc[0], dr)));
            o.y = __float_as_uint(__double2float_rn(__ddiv_rn(acc[1], dr)));
            o.z = __float_as_uint(__double2float_rn(__ddiv_rn(acc[2], dr)));
            o.w = __float_as_uint(__double2float_rn(__ddiv_rn(acc[3], dr)));
            st_stream((is_v ? ov : ok) + v, o);
        }
    }
}

// Element-wise variant for sizes or addresses that are not 16-byte multiples.
template <bool BF16>
__global__ void __launch_bounds__(256) meanpool_scalar(const void *wk, const void *wv, void *ok,
                                                       void *ov, int r, long long n,
                                                       long long out_n) {
    const long long total = 2 * out_n;
    const double dr = (double)r;
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const bool is_v = idx >= out_n;
        const long long v = is_v ? idx - out_n : idx;
        const long long g = v / n, e = v - g * n;
        double acc = 0.0;
        if (BF16) {
            const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(is_v ? wv : wk) + g * r * n + e;
            for (int j = 0; j < r; ++j) acc = __dadd_rn(acc, (double)__bfloat162float(src[(long long)j * n]));
            static_cast<__nv_bfloat16 *>(is_v ? ov : ok)[v] = __double2bfloat16(__ddiv_rn(acc, dr));
        } else {
            const float *src = static_cast<const float *>(is_v ? wv : wk) + g * r * n + e;
            for (int j = 0; j < r; ++j) acc = __dadd_rn(acc, (double)src[(long long)j * n]);
            static_cast<float *>(is_v ? ov : ok)[v] = __double2float_rn(__ddiv_rn(acc, dr));
        }
    }
}

}  // namespace

cudaError_t launch_meanpool(const void *wk, const void *wv, void *ok, void *ov, int H, int G,
                            long long n, int dtype, int num_sms, cudaStream_t st) {
    const int r = H / G;
    const bool bf16 = dtype == GQA_BF16;
    const int esz = bf16 ? 2 : 4;
    const int per_vec = 16 / esz;
    const bool aligned = ((reinterpret_cast<uintptr_t>(wk) | reinterpret_cast<uintptr_t>(wv) |
                           reinterpret_cast<uintptr_t>(ok) | reinterpret_cast<uintptr_t>(ov)) &
                          15) == 0;
    const long long out_elems = (long long)G * n;
    if (out_elems == 0) return cudaSuccess;
    const int threads = 256;
    if (aligned && n % per_vec == 0) {
        const long long n_vec = n / per_vec, out_vec = (long long)G * n_vec;
        long long blocks = (2 * out_vec + threads - 1) / threads;
        const long long cap = (long long)num_sms * 16;
        if (blocks > cap) blocks = cap;
        if (bf16)
            meanpool_vec<true><<<(unsigned)blocks, threads, 0, st>>>(
                static_cast<const uint4 *>(wk), static_cast<const uint4 *>(wv), static_cast<uint4 *>(ok),
                static_cast<uint4 *>(ov), r, n_vec, out_vec);
        else
            meanpool_vec<false><<<(unsigned)blocks, threads, 0, st>>>(
                static_cast<const uint4 *>(wk), static_cast<const uint4 *>(wv), static_cast<uint4 *>(ok),
                static_cast<uint4 *>(ov), r, n_vec, out_vec);
    } else {
        long long blocks = (2 * out_elems + threads - 1) / threads;
        const long long cap = (long long)num_sms * 16;
        if (blocks > cap) blocks = cap;
        if (bf16)
            meanpool_scalar<true><<<(unsigned)blocks, threads, 0, st>>>(wk, wv, ok, ov, r, n, out_elems);
        else
            meanpool_scalar<false><<<(unsigned)blocks, threads, 0, st>>>(wk, wv, ok, ov, r, n, out_elems);
    }
    return cudaGetLastError();
}

}  // namespace gqa
