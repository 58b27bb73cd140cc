// api.cu -- the extern "C" boundary of libgqa.so (declared in include/gqa.h).
//
// Host-side only: argument validation, TMA tensor-map encoding, the device
// status word, and the kernel launches.  No device memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>
#include <random>

#include "gqa.h"
#include "internal.h"

namespace gqa {
__device__ unsigned g_status_word;  // bits: see common.cuh
}

namespace {

thread_local char t_err[512] = "";

int fail(int code, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_err, sizeof t_err, fmt, ap);
    va_end(ap);
    return code;
}

int fail_cuda(cudaError_t e, const char *what) {
    cudaGetLastError();  // clear a non-sticky error
    return fail(GQA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool misaligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; }

constexpr int kMaxDevices = 64;

struct DeviceInfo {
    bool ready = false;
    int num_sms = 0;
    unsigned *status = nullptr;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Per-device facts, set up once per device with that device current.
int device_info(DeviceInfo **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return fail_cuda(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(GQA_ERR_UNSUPPORTED, "device ordinal %d", dev);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.ready) {
        cudaDeviceProp prop;
        e = cudaGetDeviceProperties(&prop, dev);
        if (e != cudaSuccess) return fail_cuda(e, "cudaGetDeviceProperties");
        if (prop.major != 10)
            return fail(GQA_ERR_UNSUPPORTED, "libgqa is built for sm_100a; device %d is sm_%d%d", dev,
                        prop.major, prop.minor);
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, gqa::g_status_word);
        if (e != cudaSuccess) return fail_cuda(e, "cudaGetSymbolAddress(status word)");
        d.num_sms = prop.multiProcessorCount;
        d.status = static_cast<unsigned *>(p);
        d.ready = true;
    }
    *out = &d;
    return GQA_OK;
}

uint64_t wait_timeout_ns() {
    static uint64_t v = [] {
        const char *s = getenv("GQA_WAIT_TIMEOUT_NS");
        const unsigned long long x = s ? strtoull(s, nullptr, 10) : 0ull;
        return x ? (uint64_t)x : (uint64_t)2000000000ull;  // 2 s
    }();
    return v;
}

// Tags for the split-K projections' block counters: nonzero, below 2^32, and
// different from one call to the next.
unsigned long long next_tag() {
    static std::atomic<unsigned> t{(unsigned)std::random_device{}()};
    unsigned v;
    do {
        v = t.fetch_add(1, std::memory_order_relaxed) + 1;
    } while (v == 0);
    return v;
}

int forced_splits() {
    const char *s = getenv("GQA_DECODE_CTAS");
    return s ? atoi(s) : 0;
}

// ------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int get_encoder(EncodeTiledFn *fn) {
    static EncodeTiledFn cached = nullptr;
    static std::once_flag once;
    static cudaError_t err = cudaSuccess;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) cached = reinterpret_cast<EncodeTiledFn>(p);
    });
    if (!cached) return fail(GQA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(err));
    *fn = cached;
    return GQA_OK;
}

// bf16 tensor of `rank` dims (innermost first), 128-byte swizzled boxes.
int make_tmap_bf16(CUtensorMap *m, const void *base, int rank, const cuuint64_t *dims,
                   const cuuint64_t *strides_bytes, const cuuint32_t *box) {
    EncodeTiledFn enc;
    int rc = get_encoder(&enc);
    if (rc) return rc;
    cuuint32_t elem[5] = {1, 1, 1, 1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base), dims,
                     strides_bytes, box, elem, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(GQA_ERR_CUDA, "cuTensorMapEncodeTiled failed (CUresult %d)", (int)r);
    return GQA_OK;
}

int check_dims(int B, int H, int G, int d_h) {
    if (B <= 0 || H <= 0 || G <= 0 || d_h <= 0)
        return fail(GQA_ERR_INVALID, "dimensions must be positive (B=%d H=%d G=%d d_h=%d)", B, H, G, d_h);
    if (H % G != 0) return fail(GQA_ERR_INVALID, "G=%d must divide H=%d", G, H);
    return GQA_OK;
}

}  // namespace

int gqa::set_error(int code, const char *msg) { return fail(code, "%s", msg); }

extern "C" {

int gqa_version(void) { return 101; }

const char *gqa_last_error_string(void) { return t_err; }

uint64_t gqa_kv_cache_bytes(int G, int d_h, int L, int elem_bytes) {
    if (G <= 0 || d_h <= 0 || L <= 0 || elem_bytes <= 0) return 0;
    return 2ull * (uint64_t)G * (uint64_t)d_h * (uint64_t)L * (uint64_t)elem_bytes;
}

size_t gqa_decode_workspace_bytes(int B, int H, int G, int d_h, int T_cap, gqa_dtype dt) {
    if (check_dims(B, H, G, d_h) || T_cap <= 0) return 0;
    if (dt != GQA_BF16 && dt != GQA_F32) return 0;
    DeviceInfo *d = nullptr;
    if (device_info(&d)) return 0;
    return gqa::decode_layout(B, H, G, d_h, T_cap, dt, d->num_sms, forced_splits()).total;
}

// warm: let the split kernels warm L2 with their first tiles before the work
// ahead of them on the stream has finished (see decode_common.cuh).
static int decode_impl(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens,
                       float scale, void *out, int B, int H, int G, int d_h, int T_cap, int window,
                       gqa_dtype dt, void *workspace, size_t workspace_bytes, gqa_stream_t stream,
                       bool warm = true) {
    t_err[0] = 0;
    int rc = check_dims(B, H, G, d_h);
    if (window < 0) return fail(GQA_ERR_INVALID, "window must be >= 0 (0: no window)");
    if (rc) return rc;
    if (T_cap <= 0) return fail(GQA_ERR_INVALID, "T_cap must be positive");
    if (!q || !k_cache || !v_cache || !seqlens || !out) return fail(GQA_ERR_INVALID, "null tensor pointer");
    if (!std::isfinite(scale)) return fail(GQA_ERR_INVALID, "scale must be finite");
    if (dt != GQA_BF16 && dt != GQA_F32) return fail(GQA_ERR_UNSUPPORTED, "dtype %d", (int)dt);
    if (d_h != 64 && d_h != 128) return fail(GQA_ERR_UNSUPPORTED, "d_h=%d (built: 64, 128)", d_h);
    const int r = H / G;
    if (dt == GQA_BF16 && r > 64) return fail(GQA_ERR_UNSUPPORTED, "bf16 decode needs H/G <= 64 (got %d)", r);
    if ((long long)B * G * T_cap >= (1ll << 31))
        return fail(GQA_ERR_UNSUPPORTED, "B*G*T_cap must be below 2^31 rows");
    if (B > 8192) return fail(GQA_ERR_UNSUPPORTED, "B=%d above 8192", B);
    if (misaligned(q, 16) || misaligned(k_cache, 16) || misaligned(v_cache, 16) || misaligned(out, 16) ||
        misaligned(seqlens, 4))
        return fail(GQA_ERR_ALIGN, "q, k_cache, v_cache and out must be 16-byte aligned");
    if (gqa::decode_smem_bytes(B, H, G, d_h, dt) > 227u * 1024u)
        return fail(GQA_ERR_UNSUPPORTED, "shape needs more shared memory than a CTA has (B or H/G too large)");
    DeviceInfo *d = nullptr;
    rc = device_info(&d);
    if (rc) return rc;
    const gqa::DecodeLayout L = gqa::decode_layout(B, H, G, d_h, T_cap, dt, d->num_sms, forced_splits());
    if (!workspace || workspace_bytes < L.total)
        return fail(GQA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", L.total,
                    workspace ? workspace_bytes : (size_t)0);
    if (misaligned(workspace, 256)) return fail(GQA_ERR_ALIGN, "workspace must be 256-byte aligned");

    CUtensorMap tmk, tmv;
    memset(&tmk, 0, sizeof tmk);
    memset(&tmv, 0, sizeof tmv);
    if (dt == GQA_BF16) {
        const cuuint64_t dims[2] = {(cuuint64_t)d_h, (cuuint64_t)B * G * T_cap};
        const cuuint64_t strides[1] = {(cuuint64_t)d_h * 2};
        const cuuint32_t box[2] = {64, 64};
        rc = make_tmap_bf16(&tmk, k_cache, 2, dims, strides, box);
        if (rc) return rc;
        rc = make_tmap_bf16(&tmv, v_cache, 2, dims, strides, box);
        if (rc) return rc;
    }
    gqa::DecodeArgs a = {};
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.seqlens = seqlens;
    a.out = out;
    a.scale = scale;
    a.B = B;
    a.H = H;
    a.G = G;
    a.d_h = d_h;
    a.T_cap = T_cap;
    a.dtype = dt;
    a.workspace = workspace;
    a.workspace_bytes = workspace_bytes;
    a.status = d->status;
    a.timeout_ns = wait_timeout_ns();
    a.num_sms = d->num_sms;
    a.force_ctas = forced_splits();
    a.window = window;
    a.warm = warm ? 1 : 0;
    cudaError_t e = gqa::launch_decode(a, &tmk, &tmv, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail_cuda(e, "decode launch");
    return GQA_OK;
}

int gqa_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens,
               float scale, void *out, int B, int H, int G, int d_h, int T_cap, gqa_dtype dt,
               void *workspace, size_t workspace_bytes, gqa_stream_t stream) {
    return decode_impl(q, k_cache, v_cache, seqlens, scale, out, B, H, G, d_h, T_cap, 0, dt, workspace,
                       workspace_bytes, stream);
}

int gqa_decode_window(const void *q, const void *k_cache, const void *v_cache, const int32_t *seqlens,
                      float scale, void *out, int B, int H, int G, int d_h, int T_cap, int window,
                      gqa_dtype dt, void *workspace, size_t workspace_bytes, gqa_stream_t stream) {
    return decode_impl(q, k_cache, v_cache, seqlens, scale, out, B, H, G, d_h, T_cap, window, dt, workspace,
                       workspace_bytes, stream);
}

static int prefill_impl(const void *q, const void *k, const void *v, void *out, int B, int S, int H, int G,
                        int d_h, float scale, int window, gqa_dtype dt, gqa_stream_t stream) {
    t_err[0] = 0;
    int rc = check_dims(B, H, G, d_h);
    if (window < 0) return fail(GQA_ERR_INVALID, "window must be >= 0 (0: no window)");
    if (rc) return rc;
    if (S <= 0) return fail(GQA_ERR_INVALID, "S must be positive");
    if (!q || !k || !v || !out) return fail(GQA_ERR_INVALID, "null tensor pointer");
    if (!std::isfinite(scale) || !(scale > 0.f))
        return fail(GQA_ERR_INVALID, "prefill scale must be finite and positive");
    if (dt != GQA_BF16) return fail(GQA_ERR_UNSUPPORTED, "prefill supports bf16 only");
    if (d_h != 64 && d_h != 128) return fail(GQA_ERR_UNSUPPORTED, "prefill d_h=%d (built: 64, 128)", d_h);
    if ((long long)B * S * H >= (1ll << 31)) return fail(GQA_ERR_UNSUPPORTED, "B*S*H must be below 2^31");
    if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(out, 16))
        return fail(GQA_ERR_ALIGN, "q, k, v and out must be 16-byte aligned");
    DeviceInfo *d = nullptr;
    rc = device_info(&d);
    if (rc) return rc;
    // 4-D views (innermost first): q [d_h, H, S, B], k/v [d_h, G, S, B].  Boxes of
    // [64 dims x 1 head x 128 positions x 1 sequence]; positions past S read as zero.
    CUtensorMap tmq, tmk, tmv;
    {
        const cuuint64_t dims[4] = {(cuuint64_t)d_h, (cuuint64_t)H, (cuuint64_t)S, (cuuint64_t)B};
        const cuuint64_t strides[3] = {(cuuint64_t)d_h * 2, (cuuint64_t)H * d_h * 2,
                                       (cuuint64_t)S * H * d_h * 2};
        const cuuint32_t box[4] = {64, 1, 128, 1};
        rc = make_tmap_bf16(&tmq, q, 4, dims, strides, box);
        if (rc) return rc;
    }
    {
        const cuuint64_t dims[4] = {(cuuint64_t)d_h, (cuuint64_t)G, (cuuint64_t)S, (cuuint64_t)B};
        const cuuint64_t strides[3] = {(cuuint64_t)d_h * 2, (cuuint64_t)G * d_h * 2,
                                       (cuuint64_t)S * G * d_h * 2};
        const cuuint32_t box[4] = {64, 1, 128, 1};
        rc = make_tmap_bf16(&tmk, k, 4, dims, strides, box);
        if (rc) return rc;
        rc = make_tmap_bf16(&tmv, v, 4, dims, strides, box);
        if (rc) return rc;
    }
    gqa::PrefillArgs a = {};
    a.q = q;
    a.k = k;
    a.v = v;
    a.out = out;
    a.scale = scale;
    a.B = B;
    a.S = S;
    a.H = H;
    a.G = G;
    a.d_h = d_h;
    a.status = d->status;
    a.timeout_ns = wait_timeout_ns();
    a.num_sms = d->num_sms;
    a.window = window;
    cudaError_t e = gqa::launch_prefill(a, &tmq, &tmk, &tmv, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail_cuda(e, "prefill launch");
    return GQA_OK;
}

int gqa_prefill_causal(const void *q, const void *k, const void *v, void *out, int B, int S, int H, int G,
                       int d_h, float scale, gqa_dtype dt, gqa_stream_t stream) {
    return prefill_impl(q, k, v, out, B, S, H, G, d_h, scale, 0, dt, stream);
}

int gqa_prefill_causal_window(const void *q, const void *k, const void *v, void *out, int B, int S, int H,
                              int G, int d_h, float scale, int window, gqa_dtype dt, gqa_stream_t stream) {
    return prefill_impl(q, k, v, out, B, S, H, G, d_h, scale, window, dt, stream);
}

static int init_heads_impl(const void *WK, const void *WV, void *WK_out, void *WV_out, int H, int G, int d_h,
                           int d, int mode, const float *weights, int select, gqa_dtype dt, gqa_stream_t stream) {
    t_err[0] = 0;
    if (mode != GQA_INIT_MEAN && mode != GQA_INIT_SELECT && mode != GQA_INIT_WEIGHTED)
        return fail(GQA_ERR_INVALID, "unknown init mode %d", mode);
    if (mode == GQA_INIT_SELECT && (G <= 0 || H % G != 0 || select < 0 || select >= H / G))
        return fail(GQA_ERR_INVALID, "select must index a head inside its group (0 <= select < H/G)");
    if (mode == GQA_INIT_WEIGHTED && (!weights || misaligned(weights, 4)))
        return fail(GQA_ERR_INVALID, "weighted init needs 2*H device float weights");
    if (H <= 0 || G <= 0 || d_h <= 0 || d <= 0)
        return fail(GQA_ERR_INVALID, "dimensions must be positive (H=%d G=%d d_h=%d d=%d)", H, G, d_h, d);
    if (H % G != 0) return fail(GQA_ERR_INVALID, "G=%d must divide H=%d", G, H);
    if (!WK || !WV || !WK_out || !WV_out) return fail(GQA_ERR_INVALID, "null tensor pointer");
    if (dt != GQA_BF16 && dt != GQA_F32) return fail(GQA_ERR_UNSUPPORTED, "dtype %d", (int)dt);
    const size_t esz = dt == GQA_BF16 ? 2 : 4;
    if (misaligned(WK, esz) || misaligned(WV, esz) || misaligned(WK_out, esz) || misaligned(WV_out, esz))
        return fail(GQA_ERR_ALIGN, "tensors must be aligned to their element size");
    const long long n = (long long)d_h * d;
    // the outputs must not overlap the inputs
    const char *ik = static_cast<const char *>(WK), *iv = static_cast<const char *>(WV);
    const char *okp = static_cast<const char *>(WK_out), *ovp = static_cast<const char *>(WV_out);
    const long long in_b = (long long)H * n * esz, out_b = (long long)G * n * esz;
    auto overlap = [](const char *a, long long na, const char *b, long long nb) {
        return a < b + nb && b < a + na;
    };
    if (overlap(ik, in_b, okp, out_b) || overlap(ik, in_b, ovp, out_b) || overlap(iv, in_b, okp, out_b) ||
        overlap(iv, in_b, ovp, out_b) || overlap(okp, out_b, ovp, out_b))
        return fail(GQA_ERR_INVALID, "output tensors overlap an input or each other");
    DeviceInfo *d_ = nullptr;
    int rc = device_info(&d_);
    if (rc) return rc;
    cudaError_t e = gqa::launch_init_heads(WK, WV, WK_out, WV_out, H, G, n, dt, mode, weights, select,
                                           d_->num_sms, d_->status, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail_cuda(e, "init-heads launch");
    return GQA_OK;
}

int gqa_meanpool_kv(const void *WK, const void *WV, void *WK_out, void *WV_out, int H, int G, int d_h,
                    int d, gqa_dtype dt, gqa_stream_t stream) {
    return init_heads_impl(WK, WV, WK_out, WV_out, H, G, d_h, d, GQA_INIT_MEAN, nullptr, 0, dt, stream);
}

int gqa_init_kv_heads(const void *WK, const void *WV, void *WK_out, void *WV_out, int H, int G, int d_h,
                      int d, int mode, const float *head_weights, int select, gqa_dtype dt,
                      gqa_stream_t stream) {
    return init_heads_impl(WK, WV, WK_out, WV_out, H, G, d_h, d, mode, head_weights, select, dt, stream);
}

size_t gqa_project_workspace_bytes(int ncols, int d) {
    if (ncols <= 0 || d <= 0) return 0;
    DeviceInfo *dev = nullptr;
    if (device_info(&dev)) return 0;
    return gqa::proj_workspace_bytes(ncols, d, dev->num_sms);
}

static int check_proj_workspace(void *workspace, size_t bytes, int ncols, int d, int num_sms) {
    if (!workspace) return GQA_OK;
    const size_t need = gqa::proj_workspace_bytes(ncols, d, num_sms);
    if (bytes < need)
        return fail(GQA_ERR_WORKSPACE, "projection workspace of %zu bytes needed, %zu given", need, bytes);
    if (misaligned(workspace, 256)) return fail(GQA_ERR_ALIGN, "workspace must be 256-byte aligned");
    return GQA_OK;
}

// warm: the column kernel asks L2 for its first weight tiles before the wait
// for the work ahead of it (a hint).  The layer step turns it on: its Q/K/V
// projection follows the previous step's W_O projection, which leaves most
// SMs idle, and the 7B-shaped step went from 70.5 to 69.6 us.  Back to back
// with itself, as in repeated standalone calls, it was slower (12.0 against
// 11.7 us), so gqa_qkv_append leaves it off.
static int qkv_append_impl(const void *h, const void *W_Q, const void *W_K, const void *W_V, void *q_out,
                           void *k_cache, void *v_cache, const int32_t *seqlens, int32_t *seqlens_out, int B,
                           int d, int H, int G, int d_h, int T_cap, gqa_dtype dt, void *workspace,
                           size_t workspace_bytes, gqa_stream_t stream, bool warm) {
    t_err[0] = 0;
    int rc = check_dims(B, H, G, d_h);
    if (rc) return rc;
    if (d <= 0 || T_cap <= 0) return fail(GQA_ERR_INVALID, "d and T_cap must be positive");
    if (!h || !W_Q || !W_K || !W_V || !q_out || !k_cache || !v_cache || !seqlens)
        return fail(GQA_ERR_INVALID, "null tensor pointer");
    if (dt != GQA_BF16) return fail(GQA_ERR_UNSUPPORTED, "qkv_append supports bf16 only");
    if (d_h != 64 && d_h != 128) return fail(GQA_ERR_UNSUPPORTED, "d_h=%d (built: 64, 128)", d_h);
    if (d % 128 != 0) return fail(GQA_ERR_UNSUPPORTED, "d=%d must be a multiple of 128", d);
    if (seqlens_out && seqlens_out < seqlens + B && seqlens < seqlens_out + B)
        return fail(GQA_ERR_INVALID, "seqlens_out must not overlap seqlens");
    if ((long long)B * G * T_cap * d_h >= (1ll << 40)) return fail(GQA_ERR_UNSUPPORTED, "cache too large");
    if (misaligned(W_Q, 16) || misaligned(W_K, 16) || misaligned(W_V, 16) || misaligned(h, 16) ||
        misaligned(q_out, 2) || misaligned(k_cache, 2) || misaligned(v_cache, 2) || misaligned(seqlens, 4) ||
        misaligned(seqlens_out, 4))
        return fail(GQA_ERR_ALIGN, "weights and h must be 16-byte aligned");
    DeviceInfo *dev = nullptr;
    rc = device_info(&dev);
    if (rc) return rc;
    rc = check_proj_workspace(workspace, workspace_bytes, (H + 2 * G) * d_h, d, dev->num_sms);
    if (rc) return rc;
    CUtensorMap tq, tk, tv;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)H * d_h, (cuuint64_t)d};
        const cuuint64_t strides[1] = {(cuuint64_t)H * d_h * 2};
        const cuuint32_t box[2] = {64, 128};
        rc = make_tmap_bf16(&tq, W_Q, 2, dims, strides, box);
        if (rc) return rc;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)G * d_h, (cuuint64_t)d};
        const cuuint64_t strides[1] = {(cuuint64_t)G * d_h * 2};
        const cuuint32_t box[2] = {64, 128};
        rc = make_tmap_bf16(&tk, W_K, 2, dims, strides, box);
        if (rc) return rc;
        rc = make_tmap_bf16(&tv, W_V, 2, dims, strides, box);
        if (rc) return rc;
    }
    CUtensorMap th;  // h [B, d]: boxes of 32 sequences x 64 features (rows past B read as 0)
    {
        const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)B};
        const cuuint64_t strides[1] = {(cuuint64_t)d * 2};
        const cuuint32_t box[2] = {64, 32};
        rc = make_tmap_bf16(&th, h, 2, dims, strides, box);
        if (rc) return rc;
    }
    gqa::QkvArgs a = {};
    a.h = h;
    a.q_out = q_out;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.seqlens = seqlens;
    a.seqlens_out = seqlens_out;
    a.B = B;
    a.d = d;
    a.H = H;
    a.G = G;
    a.d_h = d_h;
    a.T_cap = T_cap;
    a.status = dev->status;
    a.timeout_ns = wait_timeout_ns();
    a.workspace = workspace;
    a.num_sms = dev->num_sms;
    a.tag = next_tag();
    a.warm = warm ? 1 : 0;
    cudaError_t e = gqa::launch_qkv_append(a, &tq, &tk, &tv, &th, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail_cuda(e, "qkv_append launch");
    return GQA_OK;
}

int gqa_qkv_append(const void *h, const void *W_Q, const void *W_K, const void *W_V, void *q_out,
                   void *k_cache, void *v_cache, const int32_t *seqlens, int32_t *seqlens_out, int B, int d,
                   int H, int G, int d_h, int T_cap, gqa_dtype dt, void *workspace, size_t workspace_bytes,
                   gqa_stream_t stream) {
    return qkv_append_impl(h, W_Q, W_K, W_V, q_out, k_cache, v_cache, seqlens, seqlens_out, B, d, H, G, d_h,
                           T_cap, dt, workspace, workspace_bytes, stream, false);
}

int gqa_out_project(const void *x, const void *W, void *out, int B, int K, int N, gqa_dtype dt,
                    void *workspace, size_t workspace_bytes, gqa_stream_t stream) {
    t_err[0] = 0;
    if (B <= 0 || K <= 0 || N <= 0) return fail(GQA_ERR_INVALID, "B, K and N must be positive");
    if (!x || !W || !out) return fail(GQA_ERR_INVALID, "null tensor pointer");
    if (dt != GQA_BF16) return fail(GQA_ERR_UNSUPPORTED, "out_project supports bf16 only");
    if (K % 128 != 0 || N % 64 != 0)
        return fail(GQA_ERR_UNSUPPORTED, "K must be a multiple of 128 and N of 64 (K=%d N=%d)", K, N);
    if (misaligned(x, 16) || misaligned(W, 16) || misaligned(out, 2))
        return fail(GQA_ERR_ALIGN, "x and W must be 16-byte aligned");
    DeviceInfo *dev = nullptr;
    int rc = device_info(&dev);
    if (rc) return rc;
    rc = check_proj_workspace(workspace, workspace_bytes, N, K, dev->num_sms);
    if (rc) return rc;
    CUtensorMap tw, tx;
    {
        const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)K};
        const cuuint64_t strides[1] = {(cuuint64_t)N * 2};
        const cuuint32_t box[2] = {64, 128};
        rc = make_tmap_bf16(&tw, W, 2, dims, strides, box);
        if (rc) return rc;
    }
    {
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)B};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {64, 32};
        rc = make_tmap_bf16(&tx, x, 2, dims, strides, box);
        if (rc) return rc;
    }
    cudaError_t e = gqa::launch_out_project(x, out, B, K, N, dev->status, wait_timeout_ns(), workspace,
                                            dev->num_sms, next_tag(), &tw, &tx,
                                            reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail_cuda(e, "out_project launch");
    return GQA_OK;
}

static size_t align256_host(size_t x) { return (x + 255) & ~size_t(255); }

// The projections' split-K region of the layer workspace: the larger of the
// Q/K/V projection's and W_O's (they run one after the other), or 0 when the
// shape takes the column-block kernel.
static size_t layer_proj_bytes(int d, int H, int G, int d_h) {
    DeviceInfo *dev = nullptr;
    if (device_info(&dev)) return 0;
    const size_t a = gqa::proj_workspace_bytes((H + 2 * G) * d_h, d, dev->num_sms);
    const size_t b = gqa::proj_workspace_bytes(d, H * d_h, dev->num_sms);
    if (!a || !b) return 0;
    return align256_host(a > b ? a : b);
}

size_t gqa_layer_decode_workspace_bytes(int B, int d, int H, int G, int d_h, int T_cap, gqa_dtype dt) {
    const size_t dec = gqa_decode_workspace_bytes(B, H, G, d_h, T_cap, dt);
    if (!dec || d <= 0) return 0;
    return 2 * align256_host((size_t)B * H * d_h * 2) + layer_proj_bytes(d, H, G, d_h) + dec;
}

int gqa_layer_decode_step(const void *h, const void *W_Q, const void *W_K, const void *W_V, const void *W_O,
                          void *k_cache, void *v_cache, const int32_t *seqlens, int32_t *seqlens_out,
                          float scale, int window, void *out, int B, int d, int H, int G, int d_h, int T_cap,
                          gqa_dtype dt, void *workspace, size_t workspace_bytes, gqa_stream_t stream) {
    t_err[0] = 0;
    if (!seqlens_out) return fail(GQA_ERR_INVALID, "the layer step needs seqlens_out (lengths after the append)");
    const size_t need = gqa_layer_decode_workspace_bytes(B, d, H, G, d_h, T_cap, dt);
    if (!need) return decode_impl(nullptr, nullptr, nullptr, nullptr, scale, nullptr, B, H, G, d_h, T_cap, window, dt,
                                  nullptr, 0, stream);
    if (!workspace || workspace_bytes < need)
        return fail(GQA_ERR_WORKSPACE, "layer workspace of %zu bytes needed, %zu given", need,
                    workspace ? workspace_bytes : (size_t)0);
    if (misaligned(workspace, 256)) return fail(GQA_ERR_ALIGN, "workspace must be 256-byte aligned");
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const size_t qbytes = align256_host((size_t)B * H * d_h * 2);
    const size_t pbytes = layer_proj_bytes(d, H, G, d_h);
    void *q = ws, *attn = ws + qbytes;
    void *pws = pbytes ? ws + 2 * qbytes : nullptr;  // split-K projections, when the shape allows them
    uint8_t *dws = ws + 2 * qbytes + pbytes;
    // 1. q = h W_Q; k, v appended at seqlens[b]
    int rc = qkv_append_impl(h, W_Q, W_K, W_V, q, k_cache, v_cache, seqlens, seqlens_out, B, d, H, G, d_h,
                             T_cap, dt, pws, pbytes, stream, true);
    if (rc) return rc;
    // 2. attention over the cache including the new token.  No early L2 warm-up
    //    here: the projection before it streams its weights to the end, and
    //    warming the cache then competes with that stream (70.9 against 70.3 us
    //    per 7B-shaped step, measured).
    rc = decode_impl(q, k_cache, v_cache, seqlens_out, scale, attn, B, H, G, d_h, T_cap, window, dt, dws,
                     workspace_bytes - 2 * qbytes - pbytes, stream, false);
    if (rc) return rc;
    // 3. concatenated heads times W_O
    return gqa_out_project(attn, W_O, out, B, H * d_h, d, dt, pws, pbytes, stream);
}

int gqa_selftest_wait_timeout(uint64_t limit_ns, int *waited, gqa_stream_t stream) {
    t_err[0] = 0;
    if (limit_ns == 0 || limit_ns > 10000000000ull)
        return fail(GQA_ERR_INVALID, "limit_ns must be in (0, 1e10]");
    if (misaligned(waited, 4)) return fail(GQA_ERR_ALIGN, "waited must be 4-byte aligned");
    DeviceInfo *dev = nullptr;
    int rc = device_info(&dev);
    if (rc) return rc;
    cudaError_t e = gqa::launch_wait_timeout_selftest(dev->status, limit_ns, waited,
                                                      reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail_cuda(e, "self-test launch");
    return GQA_OK;
}

int gqa_get_status(gqa_stream_t stream) {
    t_err[0] = 0;
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail_cuda(e, "cudaStreamSynchronize");
    DeviceInfo *d = nullptr;
    int rc = device_info(&d);
    if (rc) return rc;
    unsigned word = 0;
    e = cudaMemcpy(&word, d->status, sizeof word, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return fail_cuda(e, "reading the status word");
    if (word) {
        const unsigned zero = 0;
        e = cudaMemcpy(d->status, &zero, sizeof zero, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return fail_cuda(e, "clearing the status word");
    }
    if (word & 4u) return fail(GQA_ERR_INDEX, "an index check of the debug build failed (the access was skipped)");
    if (word & 2u) return fail(GQA_ERR_TIMEOUT, "a device-side wait ran out of time");
    if (word & 1u) return fail(GQA_ERR_SEQLEN, "a seqlens entry was outside [0, T_cap] (clamped)");
    return GQA_OK;
}

}  // extern "C"
