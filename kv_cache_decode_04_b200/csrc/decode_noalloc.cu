// decode_noalloc.cu -- gqa_decode without a caller-provided workspace.
//
// gqa_decode needs device scratch for its per-split partial results, which
// the caller normally allocates.  Some callers cannot allocate device memory:
// a plug-in running inside a host runtime that has already reserved the whole
// device memory budget for its own allocator, or a serving loop that must not
// allocate after start-up because an allocation could stall it or fail.  For
// them gqa_decode_noalloc uses a scratch array compiled into this library
// instead.  It forwards to gqa_decode unchanged, so results are the same.
//
// The array below lives in every GPU that loads the library, until the
// process exits.  In host code its name is only a host-side stand-in, never a
// device address: the device address is obtained once per device with
// cudaGetSymbolAddress, with that device current, on the first call made on
// that device (make that first call before any stream capture).  Every call
// on a device shares the one array; two calls whose kernels overlap on the
// GPU (different streams, no ordering between them) race on it.  The array
// keeps the last call's contents; nothing in it has to start at zero, because
// each call writes every record it later reads.
#include <cuda_runtime.h>

#include <mutex>

#include "gqa.h"
#include "internal.h"

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[GQA_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDev = 64;
std::mutex g_mu;
void *g_scratch_ptr[kMaxDev] = {};

// Device address of the scratch array on the current device (set up once).
int scratch_address(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return gqa::set_error(GQA_ERR_CUDA, cudaGetErrorString(e));
    if (dev < 0 || dev >= kMaxDev) return gqa::set_error(GQA_ERR_UNSUPPORTED, "device ordinal out of range");
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_decode_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return gqa::set_error(GQA_ERR_CUDA, "cudaGetSymbolAddress of the static decode scratch failed");
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return GQA_OK;
}

}  // namespace

extern "C" int gqa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                  const int32_t *seqlens, float scale, void *out, int B, int H, int G,
                                  int d_h, int T_cap, gqa_dtype dt, gqa_stream_t stream) {
    const size_t need = gqa_decode_workspace_bytes(B, H, G, d_h, T_cap, dt);
    if (need == 0)  // invalid shape or no usable device: gqa_decode reports why
        return gqa_decode(q, k_cache, v_cache, seqlens, scale, out, B, H, G, d_h, T_cap, dt, nullptr, 0,
                          stream);
    if (need > (size_t)GQA_DECODE_NOALLOC_SCRATCH_BYTES)
        return gqa::set_error(GQA_ERR_WORKSPACE,
                              "this shape needs more decode scratch than the library's static "
                              "array holds (GQA_DECODE_NOALLOC_SCRATCH_BYTES); use gqa_decode with a "
                              "caller-allocated workspace");
    void *ws = nullptr;
    const int rc = scratch_address(&ws);
    if (rc) return rc;
    return gqa_decode(q, k_cache, v_cache, seqlens, scale, out, B, H, G, d_h, T_cap, dt, ws,
                      (size_t)GQA_DECODE_NOALLOC_SCRATCH_BYTES, stream);
}
