// internal.h -- launchers shared between the C-ABI layer and the kernel files.
// Not installed; the public interface is include/gqa.h.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gqa {

// Split-KV decode: one pass over equal shares of the cache tiles, then a
// combine pass.  Partial records live in the caller's workspace.
struct DecodeArgs {
    const void *q;
    const void *k_cache;
    const void *v_cache;
    const int32_t *seqlens;
    void *out;
    float scale;
    int B, H, G, d_h, T_cap;
    int dtype;  // gqa_dtype
    void *workspace;
    size_t workspace_bytes;
    unsigned *status;
    uint64_t timeout_ns;
    int num_sms;
    int force_ctas;  // >0: use this many split CTAs (tests of the split logic)
    int window;      // >0: sliding window of the last `window` cached positions
    int warm;        // nonzero: the split kernels warm L2 with their first tiles early
};

// Workspace layout, all offsets 256-byte aligned.  The first 256 bytes are a
// header that carries the completion-flag generation from one call to the
// next; it sits at offset 0 for every shape, so calls of different shapes can
// share a workspace.
struct DecodeLayout {
    int ctas;          // split CTAs of the first kernel
    long long n_rec;   // partial records: ctas + B*G
    size_t off_hdr, off_cu, off_ml, off_o, off_flag, total;
};

DecodeLayout decode_layout(int B, int H, int G, int d_h, int T_cap, int dtype, int num_sms,
                           int force_ctas);
size_t decode_smem_bytes(int B, int H, int G, int d_h, int dtype);
// Split kernel + combine.  tmk/tmv ([B*G*T_cap, d_h], boxes of [64 x 64])
// for every bf16 call.
cudaError_t launch_decode(const DecodeArgs &a, const CUtensorMap *tmk, const CUtensorMap *tmv,
                          cudaStream_t stream);

// Prefill (tcgen05).  Tensor maps over q, k, v built by the caller.
struct PrefillArgs {
    const void *q, *k, *v;
    void *out;
    float scale;
    int B, S, H, G, d_h;
    unsigned *status;
    uint64_t timeout_ns;
    int num_sms;
    int window;  // >0: query s sees keys s-window < t <= s
};
cudaError_t launch_prefill(const PrefillArgs &a, const CUtensorMap *tmq, const CUtensorMap *tmk,
                           const CUtensorMap *tmv, cudaStream_t stream);

// One decode token's Q/K/V projections and the KV-cache append.
struct QkvArgs {
    const void *h;
    void *q_out, *k_cache, *v_cache;
    const int32_t *seqlens;
    int32_t *seqlens_out;
    int B, d, H, G, d_h, T_cap;
    unsigned *status;
    uint64_t timeout_ns;
    void *workspace;         // null: one CTA per 64-column block; else the split-K kernel
    int num_sms;
    unsigned long long tag;  // nonzero, < 2^32: this call's tag for the split-K block counters
    int warm;                // nonzero: the column kernel asks L2 for its first weight tiles early
};
cudaError_t launch_qkv_append(const QkvArgs &a, const CUtensorMap *tq, const CUtensorMap *tk,
                              const CUtensorMap *tv, const CUtensorMap *th, cudaStream_t stream);

cudaError_t launch_out_project(const void *x, void *out, int B, int K, int N, unsigned *status,
                               uint64_t timeout_ns, void *workspace, int num_sms, unsigned long long tag,
                               const CUtensorMap *tw, const CUtensorMap *tx, cudaStream_t stream);

// Workspace of the split-K projection kernel for ncols output columns and a
// reduction over d (0 when the shape is not supported).
size_t proj_workspace_bytes(int ncols, int d, int num_sms);

// One CTA waits on an mbarrier nothing arrives at, with the bounded wait.
cudaError_t launch_wait_timeout_selftest(unsigned *status, uint64_t limit_ns, int *waited,
                                         cudaStream_t stream);

// Records `msg` as the calling thread's last error and returns `code`.
int set_error(int code, const char *msg);

// Mean-pool init, and its select-one-head / weighted-average alternatives
// (mode 0, 1, 2; weights [2H] device floats for mode 2, K's then V's).
cudaError_t launch_meanpool(const void *wk, const void *wv, void *ok, void *ov, int H, int G,
                            long long n, int dtype, int num_sms, unsigned *status, cudaStream_t stream);
cudaError_t launch_init_heads(const void *wk, const void *wv, void *ok, void *ov, int H, int G,
                              long long n, int dtype, int mode, const float *weights, int select,
                              int num_sms, unsigned *status, cudaStream_t stream);

}  // namespace gqa
