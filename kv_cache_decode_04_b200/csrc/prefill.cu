// prefill.cu -- causal GQA prefill on the 5th-generation tensor cores (sm_100a).
//
// What is computed ("Grouped-Query Attention", llm-arch-kb, section 3
// "Reference implementation"): for each sequence b, position s and query head
// i with g = i / (H/G),
//     out[b,s,i] = sum_{t <= s} softmax_t(scale * q[b,s,i] . k[b,t,g]) v[b,t,g].
// GQA does not reduce the flops of this step (each query head still scores
// every key), so QK^T and PV are dense tensor-core contractions here.
//
// One CTA = 128 query positions x 2 query heads of the same group: both heads
// read the same K/V tiles, which each load therefore serves twice.  When H/G
// is odd, the last head of each group gets a CTA of its own (one head; the
// second softmax warpgroup idles), so any group size works, H/G = 1 (MHA)
// included.
//   warp 8      TMA producer: Q tiles once, then [128 x d_h] K and V tiles of
//               the group through 2-stage rings (128-byte swizzle).
//   warp 9      allocates 512 tensor-memory columns; one lane issues every
//               tcgen05.mma:  S_h = Q_h K_j^T  (fp32 in TMEM, 128 cols each)
//                             O_h += P_h V_j   (P read from TMEM, fp32 O in TMEM)
//   warps 0-3   softmax + epilogue for head 0 (one thread per query row =
//   warps 4-7   one TMEM lane), head 1.  While one group runs its softmax the
//               tensor core works on the other head's MMAs.
//   warps 10-11 idle (they complete the third warpgroup for the register split).
// d_h is 64 or 128 (a template parameter).
// TMEM columns: [0,128) S0/P0, [128,256) S1/P1, [256,256+d_h) O0, [384,384+d_h) O1.
// P (bf16) overwrites the first 64 columns of its S block after S is read.
// Online softmax in the base-2 domain; the running max is only moved (and O
// rescaled in TMEM) when it grows by more than 8, so p <= 2^8: the result is
// the same because numerator and denominator use the same stale maximum.
// Only KV tiles j <= query tile are visited; the diagonal tile is masked
// (key > query -> -inf).
#include <climits>

#include "common.cuh"
#include "gqa.h"
#include "internal.h"
#include "tc.cuh"

namespace gqa {

namespace {

constexpr int kBM = 128;                 // query rows per tile
constexpr int kBN = 128;                 // keys per KV tile
constexpr int kHalf = 128 * 64 * 2;      // one [128 rows x 64 bf16] swizzled box
constexpr int kThreads = 384;           // 3 warpgroups
// Register split (setmaxnreg): the launch gives every thread kLaunchRegs; the
// TMA/MMA warpgroup then drops to kLowRegs and the two softmax warpgroups rise
// to kHighRegs.  2*128*kHighRegs + 128*kLowRegs must not exceed
// 384*kLaunchRegs, or an .inc would wait for registers that never come; the
// launcher checks the compiled register count against this before launching.
constexpr int kLaunchRegs = 168;
constexpr int kLowRegs = 136;
constexpr int kHighRegs = 184;
static_assert(2 * 128 * kHighRegs + 128 * kLowRegs <= kThreads * kLaunchRegs, "register split");
constexpr uint32_t kTmemCols = 512;

// Shared memory of the d_h = D kernel: Q0, Q1, K stages 0-1, V stages 0-1
// ([128 x D] bf16 tiles of D/64 swizzled boxes each), then the barriers.
template <int D>
struct PLay {
    static constexpr int HALVES = D / 64;
    static constexpr int TILE = HALVES * kHalf;  // [128 x D] bf16
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = 2 * TILE;
    static constexpr int OFF_V = 4 * TILE;
    static constexpr int OFF_BAR = 6 * TILE;
    static constexpr size_t SMEM = 1024 + OFF_BAR + 256;
};

struct PrefillParams {
    void *out;
    unsigned *status;
    float scale_log2;
    int B, S, H, G, r, n_qt;
    unsigned long long timeout_ns;
    int window;  // > 0: query s sees keys s - window < t <= s
};

__device__ __forceinline__ void tma_load_4d(void *dst, const void *tmap, uint64_t *bar, int x, int y,
                                            int z, int w, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w),
        "l"(policy)
        : "memory");
}

// Packed pairs of fp32 (Blackwell's paired FMA/ADD datapath).
__device__ __forceinline__ uint64_t f32x2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void f32x2_unpack(uint64_t v, float &a, float &b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f32x2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f32x2_add(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// 2^x for a pair of fp32 values on the FMA and integer pipes instead of the
// special-function unit, which the exponentials of a tile would otherwise keep
// as busy as the tensor core.  x = j + f with j = round(x) (the 1.5 * 2^23
// rounding trick) and f in [-1/2, 1/2]; 2^f is a degree-3 polynomial whose
// coefficients are a Remez (minimax) fit of the relative error over that
// interval, max relative error 7.5e-5 (P is rounded to bf16, 2^-9, after
// this); 2^j enters as j added to the exponent field.  x is clamped at -125
// first, so the exponent cannot underflow: x = -inf (a masked key) gives
// 2^-125 instead of 0, which no bf16 P or fp32 row sum can tell apart.
__device__ __forceinline__ uint64_t exp2_poly_x2(uint64_t x2) {
    float x0, x1;
    f32x2_unpack(x2, x0, x1);
    const uint64_t x = f32x2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
    constexpr float kRound = 12582912.f;  // 1.5 * 2^23
    const uint64_t t = f32x2_add(x, f32x2_pack(kRound, kRound));
    const uint64_t j = f32x2_add(t, f32x2_pack(-kRound, -kRound));
    float j0, j1;
    f32x2_unpack(j, j0, j1);
    const uint64_t f = f32x2_add(x, f32x2_pack(-j0, -j1));
    uint64_t q = f32x2_fma(f, f32x2_pack(0.05517167f, 0.05517167f), f32x2_pack(0.24261113f, 0.24261113f));
    q = f32x2_fma(q, f, f32x2_pack(0.69326097f, 0.69326097f));
    q = f32x2_fma(q, f, f32x2_pack(0.99992806f, 0.99992806f));
    float q0, q1, t0, t1;
    f32x2_unpack(q, q0, q1);
    f32x2_unpack(t, t0, t1);
    // the low bits of t hold j (t = 1.5 * 2^23 + j); shifting them into the
    // exponent field drops the 1.5 * 2^23 part, whose low 9 bits are zero
    const int r0 = (int)(__float_as_uint(t0) << 23) + (int)__float_as_uint(q0);
    const int r1 = (int)(__float_as_uint(t1) << 23) + (int)__float_as_uint(q1);
    return f32x2_pack(__int_as_float(r0), __int_as_float(r1));
}

// Pairs, out of every 8 of a row's 64 score pairs per tile, whose 2^x runs on
// the FMA pipe (exp2_poly_x2) instead of the special-function unit.
#ifndef GQA_PREFILL_EXP_POLY_OF_8
#define GQA_PREFILL_EXP_POLY_OF_8 0
#endif
constexpr int kExpPolyOf8 = GQA_PREFILL_EXP_POLY_OF_8;

// Warp-uniform bounded wait: every lane polls; the warp agrees on the result.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, uint64_t limit) {
    const bool ok = mbar_wait(bar, parity, limit);
    return __all_sync(0xffffffffu, ok);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_causal_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                          const __grid_constant__ CUtensorMap tmv, const PrefillParams p) {
    using Lay = PLay<D>;
    constexpr int HALVES = Lay::HALVES, kTile = Lay::TILE;
    constexpr int kOffQ = Lay::OFF_Q, kOffK = Lay::OFF_K, kOffV = Lay::OFF_V;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Lay::OFF_BAR);
    uint64_t *bar_q = bars + 0;
    uint64_t *k_full = bars + 1;   // [2]
    uint64_t *k_empty = bars + 3;  // [2]
    uint64_t *v_full = bars + 5;   // [2]
    uint64_t *v_empty = bars + 7;  // [2]
    uint64_t *s_full = bars + 9;   // [2] one per head
    uint64_t *p_ready = bars + 11; // [2]
    uint64_t *o_done = bars + 13;
    uint64_t *drain = bars + 14;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 15);
    int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
    volatile int *vabort = abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // work unit: heaviest query tiles (most KV tiles) first; heads 2u, 2u+1 of the
    // group, or head r-1 alone when r is odd
    const int pairs = (p.r + 1) >> 1;
    const int per_qt = p.B * p.G * pairs;
    const int qt = p.n_qt - 1 - (int)(blockIdx.x / per_qt);
    const int rem = (int)(blockIdx.x % per_qt);
    const int b = rem / (p.G * pairs);
    const int g = (rem / pairs) % p.G;
    const int pr = rem % pairs;
    const int h0 = g * p.r + 2 * pr;
    const int nh = min(2, p.r - 2 * pr);  // heads of this CTA (1 or 2)
    // the debug build's check of the unit's indices (uniform over the CTA: all
    // threads leave before any barrier or tensor memory is set up)
    if (!index_ok(qt >= 0 && b < p.B && g < p.G && nh >= 1 && h0 + nh <= p.H, p.status)) return;
    const int s0 = qt * kBM;
    // KV tiles j_lo..qt: with a sliding window of W keys the tiles wholly below the
    // first row's window (keys < s0 - W + 1) are skipped.
    const int j_lo = p.window > 0 ? max(0, s0 - p.window + 1) / kBN : 0;
    const int n_kv = qt - j_lo + 1;
    // Rows that see few keys carry P as two bf16 terms (see the softmax below).
    const bool split_p = qt == 0 || (p.window > 0 && p.window <= 256);

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 1);
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], 1);
            mbar_init(&s_full[s], 1);
            mbar_init(&p_ready[s], 128);
        }
        mbar_init(o_done, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 9) tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp >= 8) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kLowRegs));
      if (warp == 8) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmq);
            tma_prefetch_desc(&tmk);
            tma_prefetch_desc(&tmv);
            const uint64_t pol_q = l2_policy_evict_first();
            const uint64_t pol_kv = l2_policy_evict_last();
            mbar_arrive_expect_tx(bar_q, nh * kTile);
            for (int hh = 0; hh < nh; ++hh)
                for (int half = 0; half < HALVES; ++half)
                    tma_load_4d(sm + kOffQ + hh * kTile + half * kHalf, &tmq, bar_q, half * 64, h0 + hh, s0,
                                b, pol_q);
            for (int jj = 0; jj < n_kv; ++jj) {
                const int j = j_lo + jj;
                const int st = jj & 1;
                const uint32_t ph = (jj >> 1) & 1;
                if (*vabort || !mbar_wait(&k_empty[st], ph ^ 1, p.timeout_ns)) {
                    set_status(p.status, STATUS_TIMEOUT);
                    *vabort = 1;
                    break;
                }
                mbar_arrive_expect_tx(&k_full[st], kTile);
                for (int half = 0; half < HALVES; ++half)
                    tma_load_4d(sm + kOffK + st * kTile + half * kHalf, &tmk, &k_full[st], half * 64, g, j * kBN,
                                b, pol_kv);
                if (*vabort || !mbar_wait(&v_empty[st], ph ^ 1, p.timeout_ns)) {
                    set_status(p.status, STATUS_TIMEOUT);
                    *vabort = 1;
                    break;
                }
                mbar_arrive_expect_tx(&v_full[st], kTile);
                for (int half = 0; half < HALVES; ++half)
                    tma_load_4d(sm + kOffV + st * kTile + half * kHalf, &tmv, &v_full[st], half * 64, g, j * kBN,
                                b, pol_kv);
            }
        }
        __syncwarp();
      } else if (warp == 9) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = tc::idesc_bf16(128, 128, false, false);
            constexpr uint32_t idesc_o = tc::idesc_bf16(128, D, false, true);
            const uint32_t q_addr = smem_u32(sm + kOffQ), k_addr = smem_u32(sm + kOffK),
                           v_addr = smem_u32(sm + kOffV);
            bool issued = false, ok = true;
            // The waits for P spin (test_wait) rather than suspend: a suspended thread
            // resumed ~600 cycles after the softmax published P, and that delay sat on
            // every tile's critical path.
            auto wait = [&](uint64_t *bar, uint32_t par, bool spin = false) {
                if (!ok || *vabort ||
                    !(spin ? mbar_wait_spin(bar, par, p.timeout_ns) : mbar_wait(bar, par, p.timeout_ns))) {
                    if (ok) set_status(p.status, STATUS_TIMEOUT);
                    ok = false;
                    *vabort = 1;
                }
                return ok;
            };
            // Descriptors are built from one base per operand; a K-step only moves the
            // start address (low word, 16-byte units).  The loops stay rolled so the
            // issuing warp needs few registers.
            const uint64_t dq = tc::sdesc_sw128(q_addr, 16, 1024);
            const uint64_t dk = tc::sdesc_sw128(k_addr, 16, 1024);
            const uint64_t dv = tc::sdesc_sw128(v_addr, kHalf, 1024);
            // S_h = Q_h K^T: D/16 K-steps of 16 over d_h (64-wide swizzled boxes)
            auto issue_s = [&](int hh, int ks) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
                    tc::mma_ss(tmem + hh * 128, dq + ((hh * kTile) >> 4) + off, dk + ((ks * kTile) >> 4) + off,
                               idesc_s, kk > 0 ? 1u : 0u);
                }
            };
            // O_h += P_h V: 8 K-steps of 16 keys; V is MN-major (d_h contiguous).  On
            // the first query tile a second pass adds P_lo (TMEM columns 64..127).
            auto issue_pv = [&](int hh, int vs, bool acc) {
                const int passes = split_p ? 2 : 1;
#pragma unroll 1
                for (int ps = 0; ps < passes; ++ps)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        tc::mma_ts(tmem + 256 + hh * 128, tmem + hh * 128 + ps * 64 + kk * 8,
                                   dv + ((vs * kTile + kk * 2048) >> 4), idesc_o,
                                   (acc || ps > 0 || kk > 0) ? 1u : 0u);
            };
            const bool two = nh == 2;
            if (wait(bar_q, 0) && wait(&k_full[0], 0)) {
                issue_s(0, 0);
                tc::commit(&s_full[0]);
                if (two) {
                    issue_s(1, 0);
                    tc::commit(&s_full[1]);
                }
                tc::commit(&k_empty[0]);
                issued = true;
                for (int j = 0; j < n_kv && ok; ++j) {  // j counts visited tiles
                    const int st = j & 1;
                    const uint32_t ph = (j >> 1) & 1;
                    const int st2 = (j + 1) & 1;
                    const uint32_t ph2 = ((j + 1) >> 1) & 1;
                    if (!wait(&v_full[st], ph) || !wait(&p_ready[0], j & 1, true)) break;
                    tc::fence_after();
                    issue_pv(0, st, j > 0);
                    if (j + 1 < n_kv) {
                        if (!wait(&k_full[st2], ph2)) break;
                        issue_s(0, st2);
                        tc::commit(&s_full[0]);
                    }
                    if (two) {
                        if (!wait(&p_ready[1], j & 1, true)) break;
                        tc::fence_after();
                        issue_pv(1, st, j > 0);
                    }
                    tc::commit(&v_empty[st]);
                    if (j + 1 < n_kv) {
                        if (two) {
                            issue_s(1, st2);
                            tc::commit(&s_full[1]);
                        }
                        tc::commit(&k_empty[st2]);
                    }
                }
                tc::commit(o_done);
            }
            if (issued && !ok) {  // let MMAs already issued finish before TMEM is freed
                tc::commit(drain);
                mbar_wait(drain, 0, p.timeout_ns);
            }
        }
        __syncwarp();
      }
      // warps 10 and 11: spare members of the TMA/MMA warpgroup
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kHighRegs));
        // ------------------------------------------------ softmax + epilogue
        const int hh = warp >> 2;                 // head of the pair
        const int t = threadIdx.x & 127;          // query row in the tile = TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + hh * 128;
        const uint32_t tO = tmem + lane_off + 256 + hh * 128;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        // first key this row may see under a sliding window (none below it)
        const int key_lo = p.window > 0 ? s0 + t - p.window + 1 : INT_MIN;
        const int my_kv = hh < nh ? n_kv : 0;  // a one-head CTA's second warpgroup has no work
        for (int jj = 0; jj < my_kv; ++jj) {
            const int j = j_lo + jj;  // KV tile index
            const bool aborted = __any_sync(0xffffffffu, *vabort != 0);  // warp-uniform
            if (aborted || !warp_wait(&s_full[hh], jj & 1, p.timeout_ns)) {
                if (lane == 0) set_status(p.status, STATUS_TIMEOUT);
                *vabort = 1;
                ok = false;
                break;
            }
            tc::fence_after();
            uint32_t sr[4][32];
            const bool diag = (j == qt);
            // a tile holding keys below some row's window start
            const bool lo_tile = p.window > 0 && j * kBN < s0 + kBM - p.window;
            // keys after the query row, or before its window, are masked
            auto mask_chunk = [&](int c) {
                if (diag || lo_tile) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int key = j * kBN + c * 32 + e;
                        if ((diag && key > s0 + t) || key < key_lo) sr[c][e] = __float_as_uint(-INFINITY);
                    }
                }
            };
#pragma unroll
            for (int c = 0; c < 4; ++c) tc::ld32(tS + c * 32, sr[c]);
            tc::wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                tc::hold32(sr[c]);
                mask_chunk(c);
            }
            // Row maximum of the raw scores (the scale is positive), with eight
            // independent partial maxima instead of one 128-long chain.
            float mx8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) mx8[i] = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 32; ++e) mx8[e & 7] = fmaxf(mx8[e & 7], __uint_as_float(sr[c][e]));
            // P = 2^(s * scale_log2 - m) in bf16 pairs over the first 64 columns of
            // this S block; the exponent argument is formed two at a time (packed
            // fp32 FMA) and the row sum kept in four packed partial sums.
            // Rows of the first query tile see at most 128 keys, too few for the bf16
            // rounding of P to average out; there P is carried as P_hi + P_lo (two bf16
            // terms, about 16 significant bits), P_lo in columns 64..127.
            // A row that has seen no key yet (m = -inf) has only -inf scores: p = 0.
            // Returns the row sum of the unrounded p.
            const uint64_t sc2 = f32x2_pack(p.scale_log2, p.scale_log2);
            auto exp_pass = [&](float mrun) -> float {
                const float mu = mrun == -INFINITY ? 0.f : mrun;
                const uint64_t nm2 = f32x2_pack(-mu, -mu);
                uint64_t rs2[4] = {0ull, 0ull, 0ull, 0ull};
                if (!split_p) {
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        uint32_t pk[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const uint64_t x2 = f32x2_fma(f32x2_pack(__uint_as_float(sr[c4][2 * e]),
                                                                     __uint_as_float(sr[c4][2 * e + 1])), sc2, nm2);
                            float p0, p1;
                            if ((e & 7) < kExpPolyOf8) {
                                f32x2_unpack(exp2_poly_x2(x2), p0, p1);
                            } else {
                                float x0, x1;
                                f32x2_unpack(x2, x0, x1);
                                p0 = fast_exp2(x0);
                                p1 = fast_exp2(x1);
                            }
                            rs2[e & 3] = f32x2_add(rs2[e & 3], f32x2_pack(p0, p1));
                            pk[e] = pack_bf16x2(p0, p1);
                        }
                        tc::st16(tS + c4 * 16, pk);
                    }
                } else {  // first query tile: P_hi to columns 0..63, P_lo to 64..127
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
#pragma unroll
                        for (int e4 = 0; e4 < 4; ++e4) {
                            uint32_t ph[4], pl[4];
#pragma unroll
                            for (int e1 = 0; e1 < 4; ++e1) {
                                const int e = e4 * 4 + e1;
                                const float p0 = fast_exp2(fmaf(__uint_as_float(sr[c4][2 * e]), p.scale_log2, -mu));
                                const float p1 = fast_exp2(fmaf(__uint_as_float(sr[c4][2 * e + 1]), p.scale_log2, -mu));
                                rs2[e1] = f32x2_add(rs2[e1], f32x2_pack(p0, p1));
                                ph[e1] = pack_bf16x2(p0, p1);
                                const float2 h = unpack_bf16x2(ph[e1]);
                                pl[e1] = pack_bf16x2(p0 - h.x, p1 - h.y);
                            }
                            tc::st4(tS + c4 * 16 + e4 * 4, ph);
                            tc::st4(tS + 64 + c4 * 16 + e4 * 4, pl);
                        }
                    }
                }
                float sum = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float a0, a1;
                    f32x2_unpack(rs2[i], a0, a1);
                    sum += a0 + a1;
                }
                return sum;
            };
            const float mx = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                   fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7]))) * p.scale_log2;
            float alpha = 1.f;
            bool rescale = false;
            if (jj == 0) {
                m = mx;  // -inf when a sliding window hides this tile from the row
            } else {
                const float mn = fmaxf(m, mx);
                const bool need = mn > m + 8.f;
                rescale = __any_sync(0xffffffffu, need);
                if (need) {
                    alpha = fast_exp2(m - mn);
                    m = mn;
                    l *= alpha;
                }
            }
            const float rs = exp_pass(m);
            if (rescale) {  // O was last written by the P.V of tile j-1, complete by now
#pragma unroll 1
                for (int c = 0; c < D / 16; ++c) {
                    uint32_t orow[16];
                    tc::ld16(tO + c * 16, orow);
                    tc::wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) orow[e] = __float_as_uint(__uint_as_float(orow[e]) * alpha);
                    tc::st16(tO + c * 16, orow);
                }
            }
            l += rs;
            tc::wait_st();
            tc::fence_before();
            mbar_arrive(&p_ready[hh]);
        }
        // epilogue: O / l -> bf16 -> out[b, s0 + t, h0 + hh, :]
        const bool go = __all_sync(0xffffffffu, ok && *vabort == 0);
        if (hh >= nh) {
            // no head: nothing to store
        } else if (go && warp_wait(o_done, 0, p.timeout_ns)) {
            tc::fence_after();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            const int s = s0 + t;
            __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.out) +
                                 (((size_t)b * p.S + s) * p.H + h0 + hh) * D;
#pragma unroll 1
            for (int c = 0; c < D / 16; ++c) {
                uint32_t orow[16];
                tc::ld16(tO + c * 16, orow);
                tc::wait_ld();
                uint32_t pk[8];
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    pk[e] = pack_bf16x2(__uint_as_float(orow[2 * e]) * inv, __uint_as_float(orow[2 * e + 1]) * inv);
                if (s < p.S) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst + c * 16);
                    d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
        } else if (lane == 0) {
            set_status(p.status, STATUS_TIMEOUT);
        }
    }
    tc::fence_before();
    __syncthreads();
    if (warp == 9) {
        tc::fence_after();
        tc::tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

template <int D>
struct PrefillTag {};

template <int D>
cudaError_t run_prefill(const PrefillParams &p, long long grid, const CUtensorMap *tmq, const CUtensorMap *tmk,
                        const CUtensorMap *tmv, cudaStream_t st) {
    constexpr size_t smem = PLay<D>::SMEM;
    cudaError_t e = once_per_device<PrefillTag<D>>([] {
        cudaFuncAttributes fa;
        cudaError_t r = cudaFuncGetAttributes(&fa, prefill_causal_kernel<D>);
        if (r != cudaSuccess) return r;
        if (fa.numRegs != kLaunchRegs) return cudaErrorInvalidKernelImage;  // register split would not hold
        return cudaFuncSetAttribute(prefill_causal_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)smem);
    });
    if (e != cudaSuccess) return e;
    prefill_causal_kernel<D><<<(unsigned)grid, kThreads, smem, st>>>(*tmq, *tmk, *tmv, p);
    return cudaGetLastError();
}

cudaError_t launch_prefill(const PrefillArgs &a, const CUtensorMap *tmq, const CUtensorMap *tmk,
                           const CUtensorMap *tmv, cudaStream_t st) {
    PrefillParams p = {};
    p.out = a.out;
    p.status = a.status;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.B = a.B;
    p.S = a.S;
    p.H = a.H;
    p.G = a.G;
    p.r = a.H / a.G;
    p.n_qt = (a.S + kBM - 1) / kBM;
    p.window = a.window;
    p.timeout_ns = a.timeout_ns;
    const long long grid = (long long)p.n_qt * a.B * a.G * ((p.r + 1) / 2);
    if (grid <= 0 || grid >= (1ll << 31)) return cudaErrorInvalidConfiguration;
    if (a.d_h == 64) return run_prefill<64>(p, grid, tmq, tmk, tmv, st);
    if (a.d_h == 128) return run_prefill<128>(p, grid, tmq, tmk, tmv, st);
    return cudaErrorInvalidValue;
}

}  // namespace gqa
