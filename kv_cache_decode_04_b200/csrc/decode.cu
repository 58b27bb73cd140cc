// decode.cu -- GQA decode over a [B, G, T_cap, d_h] KV cache (sm_100a).
//
// What is computed ("Grouped-Query Attention", llm-arch-kb, sections 1-3):
// for every sequence b and query head i, with g = i / (H/G),
//     out[b,i] = sum_{t < T_b} softmax_t(scale * q[b,i] . K[b,g,t]) V[b,g,t].
// Every cached key and value is read once per decode step; the H/G query
// heads of a group share the one K/V head, so a K/V tile staged in shared
// memory serves all of them.
//
// How (split-KV, two kernels):
//   1. decode_split_*: the cache tiles of all (b, g) segments are laid end to
//      end and cut into gridDim.x equal shares; CTA c takes share c.  A share
//      may cover the tail of one segment and the head of the next.  For each
//      piece (the part of one segment inside one share) the CTA emits a
//      partial record (running max m, sum l, unnormalised output o) per query
//      head, at record index c + segment (distinct for all pieces: two pieces
//      with equal c + segment would need an earlier CTA to hold a later
//      segment).
//   2. decode_combine: for each (b, i) merges the records of its segment:
//      M = max m_c, L = sum 2^(m_c - M) l_c, out = sum 2^(m_c - M) o_c / L.
//   Groups of 16 or more query heads take the tcgen05 split kernel of
//   decode_tc.cu instead of decode_split_bf16; both write the same records.
//   Softmax runs in the base-2 domain on scores pre-multiplied by
//   scale*log2(e), which leaves the result unchanged.
//
// bf16 path: a producer warp streams [64 x d_h] K and V tiles with TMA
// (128-byte swizzle) through a 2-stage mbarrier ring (two CTAs per SM); four
// consumer warps run warp-level bf16 tensor-core MMAs (scores, then P.V with P
// rounded to bf16) and an fp32 online softmax; query rows are padded to 16 per
// MMA tile.
// fp32 path: CUDA-core fp32 arithmetic throughout (no TF32).
#include <atomic>
#include <cstdlib>
#include <chrono>
#include <random>

#include "common.cuh"
#include "decode_common.cuh"
#include "gqa.h"
#include "internal.h"

namespace gqa {

namespace {

constexpr int kTileF32 = 32;    // tokens per tile, fp32 path
constexpr int kStages = 2;      // TMA ring depth per CTA
constexpr int kCtasPerSm = 2;   // resident split CTAs per SM (2 x 2 stages in flight)
constexpr int kCWarps = 4;      // consumer warps
constexpr int kThreads = (kCWarps + 1) * 32;
constexpr int kThreadsF32 = 128;

using dec::attended_len;
using dec::build_tile_prefix;
using dec::clamp_len;
using dec::Cursor;
using dec::cursor_next;
using dec::cursor_seek;
using dec::DecodeParams;
using dec::kHalfBytes;
using dec::kSplitPMaxLen;
using dec::kTile;
using dec::publish_flag;
using dec::publish_prefix;
using dec::wait_flag;

__device__ __forceinline__ void named_bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ uint32_t ld_u32(const __nv_bfloat16 *p) {
    return *reinterpret_cast<const uint32_t *>(p);
}

// Byte offset of (token, dim) inside a stage buffer of [64 x D] bf16 made of
// D/64 boxes of [64 tokens x 64 dims] with the TMA 128-byte swizzle: the
// 16-byte chunk index inside a 128-byte row is XORed with (row mod 8).
__device__ __forceinline__ uint32_t swz(int tok, int dim) {
    return (uint32_t)((dim >> 6) * kHalfBytes + tok * 128 + ((((dim & 63) >> 3) ^ (tok & 7)) << 4) +
                      ((dim & 7) << 1));
}

// ----------------------------------------------------------------- bf16

// RR: rows of the cross-slice reduction buffer per 16-row head tile (the
// group's H/G heads when they are fewer than 16, so the buffer shrinks).
template <int D, int NMT, int STAGES, int RR>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    decode_split_bf16(const __grid_constant__ CUtensorMap tmk,
                      const __grid_constant__ CUtensorMap tmv, const DecodeParams p) {
    constexpr int HALVES = D / 64;
    constexpr int KV_BYTES = kTile * D * 2;
    constexpr int STAGE_BYTES = 2 * KV_BYTES;
    constexpr int NSL = kCWarps / NMT;  // token slices of a tile
    constexpr int TPS = kTile / NSL;    // tokens per slice
    constexpr int ROWF = D + 2;         // reduction row: m, l, o[D]
    constexpr int RED_FLOATS = NSL > 1 ? NSL * NMT * RR * ROWF : 0;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~uintptr_t(1023));
    uint8_t *stages = smem;
    float *red = reinterpret_cast<float *>(smem + STAGES * STAGE_BYTES);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES + RED_FLOATS * 4);
    uint64_t *empty = full + STAGES;
    int *abort_flag = reinterpret_cast<int *>(empty + STAGES);
    int *cu = abort_flag + 1;
    int *scratch = cu + p.B + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kCWarps);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kCWarps) {
        if (lane == 0) {
            tma_prefetch_desc(&tmk);
            tma_prefetch_desc(&tmv);
        }
        // 8 tiles (4 ring fills): graph-replayed A/Bs put 8 ahead of 2, 4, 12 and
        // 16 on the 7B- and 70B-shaped steps, and level with none on long rows
        dec::warm_first_tiles<kTile>(p, lane, 8, D * 2);
    }
    pdl_wait_primary();  // inputs written by the kernels before this one are visible
    const unsigned long long gen = dec::call_generation(p);
    const int W = build_tile_prefix<kTile>(p, cu, scratch, blockIdx.x == 0);
    publish_prefix(p, cu, gen);
    pdl_launch_dependents();

    const long long C = gridDim.x;
    const int u_begin = (int)((long long)blockIdx.x * W / C);
    const int u_end = (int)((long long)(blockIdx.x + 1) * W / C);
    if (u_begin >= u_end) return;
    volatile int *vabort = abort_flag;

    if (warp == kCWarps) {  // ---------------- producer: TMA ring
        if (lane == 0) {
            const uint64_t pol = l2_policy_evict_first();
            Cursor c;
            cursor_seek(cu, p.B, p.G, u_begin, c);
            for (int u = u_begin, it = 0; u < u_end; ++u, ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                if (*vabort || !mbar_wait(&empty[s], ph ^ 1, p.timeout_ns)) {
                    set_status(p.status, STATUS_TIMEOUT);
                    *vabort = 1;
                    break;
                }
                uint8_t *kdst = stages + s * STAGE_BYTES;
                uint8_t *vdst = kdst + KV_BYTES;
                mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
                const int Tb = clamp_len(p.seqlens[c.b], p.T_cap);
                const int start = Tb - attended_len(Tb, p);
                const int row = (c.b * p.G + c.g) * p.T_cap + start + c.j * kTile;
                // the tile starts inside its (b, g) segment of the cache
                const bool row_ok = index_ok(c.b < p.B && c.g < p.G && start + c.j * kTile < p.T_cap, p.status);
#pragma unroll
                for (int h = 0; h < HALVES; ++h) {
                    // (a skipped tile leaves the barrier short of its bytes: the
                    // consumers' bounded wait then ends the CTA)
                    if (!row_ok) break;
                    tma_load_2d(kdst + h * kHalfBytes, &tmk, &full[s], h * 64, row, pol);
                    tma_load_2d(vdst + h * kHalfBytes, &tmv, &full[s], h * 64, row, pol);
                }
                cursor_next(cu, p.B, p.G, c);
            }
        }
        return;
    }

    // ---------------- consumers
    const int mt = warp % NMT, sl = warp / NMT;
    const int g8 = lane >> 2, q4 = lane & 3;
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(p.q);

    uint32_t qa[D / 16][4];
    float o[D / 8][4];
    float m_a = -INFINITY, m_b = -INFINITY, l_a = 0.f, l_b = 0.f;
    int cur_bg = -1;
    bool dead = false;  // a wait ran out: keep joining barriers, skip the work

    Cursor c;
    cursor_seek(cu, p.B, p.G, u_begin, c);
    for (int u = u_begin, it = 0; u < u_end; ++u, ++it) {
        const int b = c.b, bg = c.b * p.G + c.g;
        const int seq_len = attended_len(p.seqlens[b], p);  // tiles start at T_b - seq_len
        const int n_valid = min(kTile, seq_len - c.j * kTile);
        if (bg != cur_bg) {  // first tile of a piece: this group's queries
            cur_bg = bg;
            const int hl_a = mt * 16 + g8, hl_b = hl_a + 8;
            const __nv_bfloat16 *qb = qg + ((size_t)b * p.H + (size_t)c.g * p.r) * D;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
                const int col = kk * 16 + 2 * q4;
                qa[kk][0] = hl_a < p.r ? ld_u32(qb + (size_t)hl_a * D + col) : 0u;
                qa[kk][1] = hl_b < p.r ? ld_u32(qb + (size_t)hl_b * D + col) : 0u;
                qa[kk][2] = hl_a < p.r ? ld_u32(qb + (size_t)hl_a * D + col + 8) : 0u;
                qa[kk][3] = hl_b < p.r ? ld_u32(qb + (size_t)hl_b * D + col + 8) : 0u;
            }
#pragma unroll
            for (int nn = 0; nn < D / 8; ++nn) o[nn][0] = o[nn][1] = o[nn][2] = o[nn][3] = 0.f;
            m_a = m_b = -INFINITY;
            l_a = l_b = 0.f;
        }
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!dead && (*vabort || !mbar_wait(&full[s], ph, p.timeout_ns))) {
            dead = true;
            *vabort = 1;
            set_status(p.status, STATUS_TIMEOUT);
        }
        if (!dead) {
            const uint32_t kbase = smem_u32(stages + s * STAGE_BYTES);
            const uint32_t vbase = kbase + KV_BYTES;
#pragma unroll
            for (int step = 0; step < TPS / 16; ++step) {
                const int row0 = sl * TPS + step * 16;
                if (row0 >= n_valid) break;
                if (row0 + 16 > n_valid) {
                    // rows past the end of the sequence: zero V so 0 * (garbage) stays 0
                    for (int idx = lane; idx < 16 * HALVES * 8; idx += 32) {
                        const int rr = row0 + idx / (HALVES * 8);
                        const int rem = idx % (HALVES * 8);
                        if (rr >= n_valid) {
                            const uint32_t a = vbase + (rem >> 3) * kHalfBytes + rr * 128 + (rem & 7) * 16;
                            asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};" ::"r"(a), "r"(0u)
                                         : "memory");
                        }
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                // S[16 heads x 16 tokens] = q . K^T
                float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
                {
                    const int tok = row0 + ((lane >> 4) << 3) + (lane & 7);
                    const int dsel = ((lane >> 3) & 1) << 3;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(kbase + swz(tok, kk * 16 + dsel), b0, b1, b2, b3);
                        mma_16816(sc[0], qa[kk], b0, b1);
                        mma_16816(sc[1], qa[kk], b2, b3);
                    }
                }
                // scale into the log2 domain, mask tokens past the end
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int tok = row0 + nt * 8 + 2 * q4 + (e & 1);
                        const float v = sc[nt][e] * p.scale_log2;
                        sc[nt][e] = tok < n_valid ? v : -INFINITY;
                    }
                float mx_a = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
                float mx_b = fmaxf(fmaxf(sc[0][2], sc[0][3]), fmaxf(sc[1][2], sc[1][3]));
                mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 1));
                mx_a = fmaxf(mx_a, __shfl_xor_sync(0xffffffffu, mx_a, 2));
                mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 1));
                mx_b = fmaxf(mx_b, __shfl_xor_sync(0xffffffffu, mx_b, 2));
                const float mn_a = fmaxf(m_a, mx_a), mn_b = fmaxf(m_b, mx_b);
                const float mu_a = mn_a == -INFINITY ? 0.f : mn_a;
                const float mu_b = mn_b == -INFINITY ? 0.f : mn_b;
                const float al_a = fast_exp2(m_a - mu_a), al_b = fast_exp2(m_b - mu_b);
                m_a = mn_a;
                m_b = mn_b;
                uint32_t pa[4];
                float ps_a = 0.f, ps_b = 0.f;
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    pa[2 * nt + 0] = pack_bf16x2(fast_exp2(sc[nt][0] - mu_a), fast_exp2(sc[nt][1] - mu_a));
                    pa[2 * nt + 1] = pack_bf16x2(fast_exp2(sc[nt][2] - mu_b), fast_exp2(sc[nt][3] - mu_b));
                    const float2 fa = unpack_bf16x2(pa[2 * nt + 0]);
                    const float2 fb = unpack_bf16x2(pa[2 * nt + 1]);
                    ps_a += fa.x + fa.y;
                    ps_b += fb.x + fb.y;
                }
                l_a = l_a * al_a + ps_a;
                l_b = l_b * al_b + ps_b;
#pragma unroll
                for (int nn = 0; nn < D / 8; ++nn) {
                    o[nn][0] *= al_a;
                    o[nn][1] *= al_a;
                    o[nn][2] *= al_b;
                    o[nn][3] *= al_b;
                }
                // O[16 x D] += P[16 x 16] . V[16 x D].  For short sequences the bf16
                // rounding of P does not average out; there P is carried as two bf16
                // terms P_hi + P_lo (about 16 significant bits).
                const bool split_p = seq_len <= kSplitPMaxLen;
                uint32_t pl[4] = {0u, 0u, 0u, 0u};
                if (split_p) {
                    // the row sum takes the same P_hi + P_lo the products use, so that
                    // numerator and denominator agree (with P_hi alone it would be off
                    // by the rounding of P, ~2^-9 relative on short sequences)
                    float ls_a = 0.f, ls_b = 0.f;
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        const float2 ha = unpack_bf16x2(pa[2 * nt + 0]);
                        const float2 hb = unpack_bf16x2(pa[2 * nt + 1]);
                        pl[2 * nt + 0] = pack_bf16x2(fast_exp2(sc[nt][0] - mu_a) - ha.x,
                                                     fast_exp2(sc[nt][1] - mu_a) - ha.y);
                        pl[2 * nt + 1] = pack_bf16x2(fast_exp2(sc[nt][2] - mu_b) - hb.x,
                                                     fast_exp2(sc[nt][3] - mu_b) - hb.y);
                        const float2 la = unpack_bf16x2(pl[2 * nt + 0]);
                        const float2 lb = unpack_bf16x2(pl[2 * nt + 1]);
                        ls_a += la.x + la.y;
                        ls_b += lb.x + lb.y;
                    }
                    l_a += ls_a;
                    l_b += ls_b;
                }
                {
                    const int tok = row0 + (((lane >> 3) & 1) << 3) + (lane & 7);
                    const int dsel = (lane >> 4) << 3;
                    if (!split_p) {
#pragma unroll
                        for (int n2 = 0; n2 < D / 16; ++n2) {
                            uint32_t b0, b1, b2, b3;
                            ldsm_x4_t(vbase + swz(tok, n2 * 16 + dsel), b0, b1, b2, b3);
                            mma_16816(o[2 * n2], pa, b0, b1);
                            mma_16816(o[2 * n2 + 1], pa, b2, b3);
                        }
                    } else {
#pragma unroll
                        for (int n2 = 0; n2 < D / 16; ++n2) {
                            uint32_t b0, b1, b2, b3;
                            ldsm_x4_t(vbase + swz(tok, n2 * 16 + dsel), b0, b1, b2, b3);
                            mma_16816(o[2 * n2], pa, b0, b1);
                            mma_16816(o[2 * n2 + 1], pa, b2, b3);
                            mma_16816(o[2 * n2], pl, b0, b1);
                            mma_16816(o[2 * n2 + 1], pl, b2, b3);
                        }
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        cursor_next(cu, p.B, p.G, c);
        const bool piece_end = (u + 1 == u_end) || (c.b * p.G + c.g != bg);
        if (!piece_end) continue;

        // ---------------- emit this piece's partial record
        float la = l_a, lb = l_b;
        la += __shfl_xor_sync(0xffffffffu, la, 1);
        la += __shfl_xor_sync(0xffffffffu, la, 2);
        lb += __shfl_xor_sync(0xffffffffu, lb, 1);
        lb += __shfl_xor_sync(0xffffffffu, lb, 2);
        const long long rec = (long long)blockIdx.x + bg;
        const bool rec_ok = index_ok(rec < p.n_rec, p.status);
        if (!rec_ok) dead = true;
        if (NSL == 1) {
            const int hl_a = mt * 16 + g8, hl_b = hl_a + 8;
            if (!dead && hl_a < p.r) {
                float *dst = p.ws_o + (rec * p.r + hl_a) * D;
#pragma unroll
                for (int nn = 0; nn < D / 8; ++nn)
                    *reinterpret_cast<float2 *>(dst + nn * 8 + 2 * q4) = make_float2(o[nn][0], o[nn][1]);
                if (q4 == 0) p.ws_ml[rec * p.r + hl_a] = make_float2(m_a, la);
            }
            if (!dead && hl_b < p.r) {
                float *dst = p.ws_o + (rec * p.r + hl_b) * D;
#pragma unroll
                for (int nn = 0; nn < D / 8; ++nn)
                    *reinterpret_cast<float2 *>(dst + nn * 8 + 2 * q4) = make_float2(o[nn][2], o[nn][3]);
                if (q4 == 0) p.ws_ml[rec * p.r + hl_b] = make_float2(m_b, lb);
            }
            __threadfence();
            named_bar_sync(1, kCWarps * 32);
            if (tid == 0 && !dead) publish_flag(&p.ws_flag[1 + rec], gen);
        } else {
            // rows g8 and g8+8 of this warp's head tile; rows >= RR are past H/G
            float *ra = red + ((sl * NMT + mt) * RR + g8) * ROWF;
            float *rb = ra + 8 * ROWF;
            if (g8 < RR) {
                if (q4 == 0) {
                    ra[0] = m_a;
                    ra[1] = la;
                }
#pragma unroll
                for (int nn = 0; nn < D / 8; ++nn) {
                    ra[2 + nn * 8 + 2 * q4] = o[nn][0];
                    ra[3 + nn * 8 + 2 * q4] = o[nn][1];
                }
            }
            if (g8 + 8 < RR) {
                if (q4 == 0) {
                    rb[0] = m_b;
                    rb[1] = lb;
                }
#pragma unroll
                for (int nn = 0; nn < D / 8; ++nn) {
                    rb[2 + nn * 8 + 2 * q4] = o[nn][2];
                    rb[3 + nn * 8 + 2 * q4] = o[nn][3];
                }
            }
            named_bar_sync(1, kCWarps * 32);
            const int rows = min(p.r, NMT * 16);
            for (int idx = tid; idx < rows * D; idx += kCWarps * 32) {
                const int hl = idx / D, col = idx - hl * D;
                const int mtr = hl >> 4, rr = hl & 15;
                float M = -INFINITY;
#pragma unroll
                for (int k = 0; k < NSL; ++k) M = fmaxf(M, red[((k * NMT + mtr) * RR + rr) * ROWF]);
                float acc = 0.f, L = 0.f;
#pragma unroll
                for (int k = 0; k < NSL; ++k) {
                    const float *row = red + ((k * NMT + mtr) * RR + rr) * ROWF;
                    const float w = fast_exp2(row[0] - M);
                    acc += w * row[2 + col];
                    L += w * row[1];
                }
                if (!dead) {
                    p.ws_o[(rec * p.r + hl) * D + col] = acc;
                    if (col == 0) p.ws_ml[rec * p.r + hl] = make_float2(M, L);
                }
            }
            __threadfence();
            named_bar_sync(1, kCWarps * 32);
            if (tid == 0 && !dead) publish_flag(&p.ws_flag[1 + rec], gen);
        }
    }
}

// ----------------------------------------------------------------- fp32

template <int D>
__global__ void __launch_bounds__(kThreadsF32)
    decode_split_f32(const DecodeParams p) {
    constexpr int KS = D + 1;  // padded row stride (bank spread)
    extern __shared__ float sm32[];
    float *Ks = sm32;                  // [32][KS]
    float *Vs = Ks + kTileF32 * KS;    // [32][KS]
    float *ps = Vs + kTileF32 * KS;    // [4 warps][32]
    float *qs = ps + 4 * 32;           // [r][D]
    float *st_o = qs + p.r * D;        // [r][D]
    float *st_m = st_o + p.r * D;      // [r]
    float *st_l = st_m + p.r;          // [r]
    int *cu = reinterpret_cast<int *>(st_l + p.r);
    int *scratch = cu + p.B + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    pdl_wait_primary();  // inputs written by the kernels before this one are visible
    const unsigned long long gen = dec::call_generation(p);
    const int W = build_tile_prefix<kTileF32>(p, cu, scratch, blockIdx.x == 0);
    publish_prefix(p, cu, gen);
    pdl_launch_dependents();
    const long long C = gridDim.x;
    const int u_begin = (int)((long long)blockIdx.x * W / C);
    const int u_end = (int)((long long)(blockIdx.x + 1) * W / C);
    if (u_begin >= u_end) return;
    const float *qg = static_cast<const float *>(p.q);

    int cur_bg = -1;
    Cursor c;
    cursor_seek(cu, p.B, p.G, u_begin, c);
    for (int u = u_begin; u < u_end; ++u) {
        const int b = c.b, bg = c.b * p.G + c.g;
        const int seq_len = attended_len(p.seqlens[b], p);
        const int t0 = clamp_len(p.seqlens[b], p.T_cap) - seq_len + c.j * kTileF32;
        const int n_valid = min(kTileF32, seq_len - c.j * kTileF32);
        if (bg != cur_bg) {
            cur_bg = bg;
            const float *qb = qg + ((size_t)b * p.H + (size_t)c.g * p.r) * D;
            for (int i = tid; i < p.r * D; i += blockDim.x) {
                qs[i] = qb[i];
                st_o[i] = 0.f;
            }
            for (int i = tid; i < p.r; i += blockDim.x) {
                st_m[i] = -INFINITY;
                st_l[i] = 0.f;
            }
        }
        const size_t base = ((size_t)bg * p.T_cap + t0) * D;
        const bool seg_ok = index_ok(b < p.B && t0 >= 0 && t0 + n_valid <= p.T_cap, p.status);
        for (int i = tid; i < kTileF32 * D; i += blockDim.x) {
            const int row = i / D, col = i - row * D;
            const bool ok = row < n_valid && seg_ok;
            Ks[row * KS + col] = ok ? p.k32[base + i] : 0.f;
            Vs[row * KS + col] = ok ? p.v32[base + i] : 0.f;
        }
        __syncthreads();
        for (int hl = warp; hl < p.r; hl += 4) {
            float s = -INFINITY;
            if (lane < n_valid) {
                float acc = 0.f;
                for (int k = 0; k < D; ++k) acc = fmaf(qs[hl * D + k], Ks[lane * KS + k], acc);
                s = acc * p.scale_log2;
            }
            float mx = s;
#pragma unroll
            for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float m_old = st_m[hl];
            const float m_new = fmaxf(m_old, mx);  // finite: token 0 of a tile is valid
            const float alpha = fast_exp2(m_old - m_new);
            const float pr = fast_exp2(s - m_new);
            float sum = pr;
#pragma unroll
            for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
            ps[warp * 32 + lane] = pr;
            __syncwarp();
            for (int col = lane; col < D; col += 32) {
                float acc = st_o[hl * D + col] * alpha;
                for (int t = 0; t < n_valid; ++t) acc = fmaf(ps[warp * 32 + t], Vs[t * KS + col], acc);
                st_o[hl * D + col] = acc;
            }
            __syncwarp();
            if (lane == 0) {
                st_m[hl] = m_new;
                st_l[hl] = st_l[hl] * alpha + sum;
            }
            __syncwarp();
        }
        __syncthreads();
        cursor_next(cu, p.B, p.G, c);
        const bool piece_end = (u + 1 == u_end) || (c.b * p.G + c.g != bg);
        if (piece_end) {
            const long long rec = (long long)blockIdx.x + bg;
            if (index_ok(rec < p.n_rec, p.status)) {
                for (int i = tid; i < p.r * D; i += blockDim.x) p.ws_o[rec * p.r * D + i] = st_o[i];
                for (int i = tid; i < p.r; i += blockDim.x)
                    p.ws_ml[rec * p.r + i] = make_float2(st_m[i], st_l[i]);
                __threadfence();
                __syncthreads();
                if (tid == 0) publish_flag(&p.ws_flag[1 + rec], gen);
            }
        }
    }
}

// ----------------------------------------------------------------- combine

// One CTA of NW warps per output row (b, i).  It runs alongside the split
// kernel (a programmatic dependent launched early) and waits only for what it
// reads: the tile prefix, then each record of its segment, through the
// completion flags the split kernel publishes.  Warp w merges records w,
// w + NW, ... of the row's segment, issuing the loads of up to kCombBatch
// records at once and keeping a running (max, sum, o); the warps' results are
// then merged in a fixed order (deterministic results).  NW is 16, 8 or 4
// (see run_combine).
constexpr int kCombBatch = 8;

// One block per SM is all the launch bounds ask for, so the compiler keeps
// the merge loop in registers (94 at d_h = 128, no spills).  Left to its own
// choice it fitted the 16-warp combine into 64 registers with 136 bytes of
// spills, and that combine then also fitted next to the tcgen05 split kernel
// on every SM, where its polling slowed the split: graph-timed, the G = 2
// long-context step took 99-104 us that way against 89-90 us with these
// bounds (7B-shaped step: 47.6 us either way).
template <int D, bool BF16_OUT, int NW>
__global__ void __launch_bounds__(NW * 32, 1) decode_combine(const DecodeParams p, int C) {
    constexpr int PER = D / 32;
    __shared__ float red_m[NW], red_l[NW];
    __shared__ int red_bad[NW];
    __shared__ __align__(16) float red_o[NW][D];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = blockIdx.x;  // b*H + h
    const int b = (int)(row / p.H), h = (int)(row % p.H);
    const int g = h / p.r, hl = h - g * p.r;
    const int bg = b * p.G + g;
    float acc[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) acc[k] = 0.f;
    float M = -INFINITY, L = 0.f;
    const unsigned long long gen = dec::call_generation(p);
    const bool pre_ok = __all_sync(0xffffffffu, wait_flag(&p.ws_flag[0], gen, p.timeout_ns));  // tile prefix
    if (threadIdx.x == 0) {
        // Count this CTA as started: its read of the header is behind it.  The
        // last CTA to count stores this call's generation for the next call (all
        // CTAs have derived theirs by then), so the store is off the grid's tail.
        // The count was zeroed before the prefix flag; a CTA that never saw that
        // flag does not count itself (the grid then never completes the count)
        // and invalidates the header.  A wait that runs out later marks the
        // count bad and invalidates the header itself (below), so the next call
        // starts from a fresh random generation rather than one that flags left
        // by this call could match.
        if (!pre_ok) {
            p.ws_hdr[dec::HDR_CHECK] = 0ull;
        } else {
            const unsigned long long prev = atomicAdd(&p.ws_hdr[dec::HDR_DONE], 1ull);
            if ((prev & 0xffffffffull) == (unsigned long long)gridDim.x - 1) {
                if (prev >> 32) {
                    p.ws_hdr[dec::HDR_CHECK] = 0ull;
                } else {
                    p.ws_hdr[dec::HDR_EPOCH] = gen;
                    p.ws_hdr[dec::HDR_CHECK] = gen ^ dec::kHdrMagic;
                }
            }
        }
    }
    bool ok = pre_ok;
    const int *cu = p.ws_cu;
    const int ntb = ok ? (cu[b + 1] - cu[b]) / p.G : 0;
    if (ntb > 0) {
        const long long W = cu[p.B];
        const long long s0 = cu[b] + (long long)g * ntb, s1 = s0 + ntb;
        const int c_lo = (int)(((s0 + 1) * C - 1) / W);
        const int c_hi = (int)((s1 * C - 1) / W);
        const int n = c_hi - c_lo + 1;
        // With fewer tiles than CTAs some shares are empty; those CTAs wrote no record.
        const bool may_skip = W < C;
        auto has_record = [&](int i) {
            const int c = c_lo + i;
            return i < n && !(may_skip && (long long)c * W / C == (long long)(c + 1) * W / C) &&
                   index_ok(c_lo >= 0 && (long long)c + bg < p.n_rec, p.status);
        };
        for (int i0 = warp; i0 < n && ok; i0 += NW * kCombBatch) {
#pragma unroll 1
            for (int j = 0; j < kCombBatch; ++j) {  // the batch's records are complete
                const int i = i0 + j * NW;
                if (has_record(i))
                    ok &= __all_sync(0xffffffffu, wait_flag(&p.ws_flag[1 + (long long)c_lo + i + bg], gen,
                                                            p.timeout_ns));
            }
            if (!ok) break;
            float2 ml[kCombBatch];
            float v[kCombBatch][PER];
#pragma unroll
            for (int j = 0; j < kCombBatch; ++j) {
                const int i = i0 + j * NW;
                ml[j] = make_float2(-INFINITY, 0.f);
#pragma unroll
                for (int k = 0; k < PER; ++k) v[j][k] = 0.f;
                if (!has_record(i)) continue;
                const long long rec = (long long)c_lo + i + bg;
                ml[j] = p.ws_ml[rec * p.r + hl];
                const float *src = p.ws_o + (rec * p.r + hl) * D + lane * PER;
                if constexpr (PER == 4) {
                    const float4 t = *reinterpret_cast<const float4 *>(src);
                    v[j][0] = t.x;
                    v[j][1] = t.y;
                    v[j][2] = t.z;
                    v[j][3] = t.w;
                } else {
                    const float2 t = *reinterpret_cast<const float2 *>(src);
                    v[j][0] = t.x;
                    v[j][1] = t.y;
                }
            }
#pragma unroll
            for (int j = 0; j < kCombBatch; ++j) {
                const float Mn = fmaxf(M, ml[j].x);
                if (Mn == -INFINITY) continue;  // nothing seen yet
                const float a = fast_exp2(M - Mn), w = fast_exp2(ml[j].x - Mn);
                L = L * a + w * ml[j].y;
#pragma unroll
                for (int k = 0; k < PER; ++k) acc[k] = acc[k] * a + w * v[j][k];
                M = Mn;
            }
        }
    }
    if (!ok && lane == 0) set_status(p.status, STATUS_TIMEOUT);
    if (lane == 0) red_bad[warp] = (pre_ok ? 0 : 2) | (ok ? 0 : 1);
#pragma unroll
    for (int k = 0; k < PER; ++k) red_o[warp][lane * PER + k] = acc[k];
    if (lane == 0) {
        red_m[warp] = M;
        red_l[warp] = L;
    }
    __syncthreads();
    pdl_launch_dependents();  // the next decode's split kernel may start its prologue
    if (warp != 0) return;
    if (lane == 0 && pre_ok) {
        int bad = 0;
#pragma unroll
        for (int w = 0; w < NW; ++w) bad |= red_bad[w];
        if (bad) {  // a record wait ran out: no valid header from this call
            atomicAdd(&p.ws_hdr[dec::HDR_DONE], 1ull << 32);
            __threadfence();
            p.ws_hdr[dec::HDR_CHECK] = 0ull;
        }
    }
    float Mt = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) Mt = fmaxf(Mt, red_m[w]);
    float Lt = 0.f;
#pragma unroll
    for (int k = 0; k < PER; ++k) acc[k] = 0.f;
    if (Mt != -INFINITY) {
#pragma unroll
        for (int w = 0; w < NW; ++w) {
            const float f = fast_exp2(red_m[w] - Mt);  // 0 for a warp that merged nothing
            Lt = fmaf(f, red_l[w], Lt);
#pragma unroll
            for (int k = 0; k < PER; ++k) acc[k] = fmaf(f, red_o[w][lane * PER + k], acc[k]);
        }
    }
    const float inv = Lt > 0.f ? 1.f / Lt : 0.f;
#pragma unroll
    for (int k = 0; k < PER; ++k) acc[k] *= inv;
    if constexpr (BF16_OUT) {
        __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(p.out) + row * D + lane * PER;
        if constexpr (PER == 4)
            *reinterpret_cast<uint2 *>(dst) =
                make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]));
        else
            *reinterpret_cast<uint32_t *>(dst) = pack_bf16x2(acc[0], acc[1]);
    } else {
        float *dst = static_cast<float *>(p.out) + row * D + lane * PER;
        if constexpr (PER == 4)
            *reinterpret_cast<float4 *>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        else
            *reinterpret_cast<float2 *>(dst) = make_float2(acc[0], acc[1]);
    }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Raises a kernel's dynamic shared-memory limit once per device (the
// attribute persists); one instance per kernel through the Tag parameter.
template <typename Tag, typename Kern>
cudaError_t set_smem_once(Kern kern, size_t smem) {
    static std::atomic<int> done[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const bool cached = dev >= 0 && dev < 64;
    if (cached && done[dev].load(std::memory_order_acquire) >= (int)smem) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess && cached) {
        int cur = done[dev].load();
        while (cur < (int)smem && !done[dev].compare_exchange_weak(cur, (int)smem)) {
        }
    }
    return e;
}

template <int D, int NMT, int STAGES, int RR>
struct Bf16Tag {};
template <int D>
struct F32Tag {};

int bf16_nmt(int r) { return r <= 16 ? 1 : (r <= 32 ? 2 : 4); }

// Ring depth and reduction rows for a group of r query heads: groups of at
// most 4 heads use 4-row reduction buffers.
int bf16_stages(int r) { (void)r; return kStages; }
int bf16_red_rows(int r) { return r <= 4 ? 4 : 16; }

size_t smem_bf16(int D, int nmt, int B, int stages, int rr) {
    const int nsl = kCWarps / nmt;
    const size_t red = nsl > 1 ? (size_t)nsl * nmt * rr * (D + 2) * 4 : 0;
    return 1024 + (size_t)stages * 2 * kTile * D * 2 + red + 2 * (size_t)stages * 8 + 4 +
           (size_t)(B + 1) * 4 + 32 * 4;
}

size_t smem_f32(int D, int r, int B) {
    return ((size_t)2 * kTileF32 * (D + 1) + 4 * 32 + 2 * (size_t)r * D + 2 * r) * 4 +
           (size_t)(B + 1) * 4 + 32 * 4;
}

template <int D, int NMT, int STAGES, int RR>
cudaError_t run_bf16(const DecodeParams &p, const CUtensorMap *tmk, const CUtensorMap *tmv,
                     int ctas, cudaStream_t st) {
    const size_t smem = smem_bf16(D, NMT, p.B, STAGES, RR);
    auto kern = decode_split_bf16<D, NMT, STAGES, RR>;
    cudaError_t e = set_smem_once<Bf16Tag<D, NMT, STAGES, RR>>(kern, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(ctas), dim3(kThreads), smem, st, *tmk, *tmv, p);
}

template <int D>
cudaError_t run_f32(const DecodeParams &p, int ctas, cudaStream_t st) {
    const size_t smem = smem_f32(D, p.r, p.B);
    auto kern = decode_split_f32<D>;
    cudaError_t e = set_smem_once<F32Tag<D>>(kern, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(ctas), dim3(kThreadsF32), smem, st, p);
}

template <int D, bool BF16_OUT, int NW>
struct CombineTag {};

template <int D, bool BF16_OUT, int NW>
cudaError_t run_combine_nw(const DecodeParams &p, int ctas, cudaStream_t st) {
    // The split kernels before it run with (nearly) all of an SM's shared
    // memory; asking for the same carveout here spares every call an L1/shared
    // memory reconfiguration of the SMs between the two kernels.
    cudaError_t e = once_per_device<CombineTag<D, BF16_OUT, NW>>([] {
        return cudaFuncSetAttribute(decode_combine<D, BF16_OUT, NW>, cudaFuncAttributePreferredSharedMemoryCarveout,
                                    (int)cudaSharedmemCarveoutMaxShared);
    });
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((long long)p.B * p.H));
    cfg.blockDim = dim3(NW * 32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_combine<D, BF16_OUT, NW>, p, ctas);
}

template <int D, bool BF16_OUT>
cudaError_t run_combine(const DecodeParams &p, int ctas, cudaStream_t st) {
    // Records of one row: about CTAs per segment + 1.
    // Wide CTAs (16 warps, one per SM by registers) only when the rows are few
    // enough to fit one wave and have records for the extra warps.
    const long long segs = (long long)p.B * p.G, rows = (long long)p.B * p.H;
    const long long recs = ((long long)ctas + segs - 1) / segs + 1;
    if (rows <= 148 && recs > 16) return run_combine_nw<D, BF16_OUT, 16>(p, ctas, st);
    if (rows <= 3 * 148 && recs > 8) return run_combine_nw<D, BF16_OUT, 8>(p, ctas, st);
    return run_combine_nw<D, BF16_OUT, 4>(p, ctas, st);
}

// Seeds for the completion-flag generation (see dec::call_generation), used
// when a workspace's header is not valid: unique per call in this process and
// started from a random 64-bit base, so that flags left in reused memory (by
// this or another process) do not match.
unsigned long long next_seed() {
    static std::atomic<unsigned long long> gen{[] {
        std::random_device rd;
        const unsigned long long t =
            (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count();
        return ((unsigned long long)rd() << 32 ^ (unsigned long long)rd()) ^ (t * 0x9E3779B97F4A7C15ull);
    }()};
    return gen.fetch_add(1, std::memory_order_relaxed) + 1;
}

}  // namespace

DecodeLayout decode_layout(int B, int H, int G, int d_h, int T_cap, int dtype, int num_sms,
                           int force_ctas) {
    DecodeLayout L = {};
    const int r = H / G;
    const int tile = dtype == GQA_BF16 ? kTile : kTileF32;
    const long long max_tiles = (long long)B * G * ((T_cap + tile - 1) / tile);
    const bool tc = dtype == GQA_BF16 && dec::tc_eligible(r, d_h, B);
    long long ctas = force_ctas > 0 ? force_ctas
                                    : (long long)num_sms * (dtype == GQA_BF16 && !tc ? kCtasPerSm : 1);
    if (ctas > max_tiles) ctas = max_tiles;
    if (ctas < 1) ctas = 1;
    L.ctas = (int)ctas;
    L.n_rec = ctas + (long long)B * G;
    L.off_hdr = 0;
    L.off_cu = 256;
    L.off_ml = L.off_cu + align256((size_t)(B + 1) * 4);
    L.off_o = L.off_ml + align256((size_t)L.n_rec * r * sizeof(float2));
    L.off_flag = L.off_o + align256((size_t)L.n_rec * r * d_h * sizeof(float));
    L.total = L.off_flag + align256((size_t)(1 + L.n_rec) * sizeof(unsigned long long));
    return L;
}

size_t decode_smem_bytes(int B, int H, int G, int d_h, int dtype) {
    const int r = H / G;
    if (dtype == GQA_BF16 && dec::tc_eligible(r, d_h, B)) return dec::tc_smem_bytes(d_h, B);
    return dtype == GQA_BF16 ? smem_bf16(d_h, bf16_nmt(r), B, bf16_stages(r), bf16_red_rows(r))
                             : smem_f32(d_h, r, B);
}

cudaError_t launch_decode(const DecodeArgs &a, const CUtensorMap *tmk, const CUtensorMap *tmv,
                          cudaStream_t st) {
    const DecodeLayout L = decode_layout(a.B, a.H, a.G, a.d_h, a.T_cap, a.dtype, a.num_sms, a.force_ctas);
    uint8_t *ws = static_cast<uint8_t *>(a.workspace);
    DecodeParams p = {};
    p.q = a.q;
    p.seqlens = a.seqlens;
    p.out = a.out;
    p.ws_cu = reinterpret_cast<int *>(ws + L.off_cu);
    p.ws_ml = reinterpret_cast<float2 *>(ws + L.off_ml);
    p.ws_o = reinterpret_cast<float *>(ws + L.off_o);
    p.k32 = static_cast<const float *>(a.k_cache);
    p.v32 = static_cast<const float *>(a.v_cache);
    p.status = a.status;
    p.scale_log2 = a.scale * 1.4426950408889634f;
    p.B = a.B;
    p.H = a.H;
    p.G = a.G;
    p.r = a.H / a.G;
    p.T_cap = a.T_cap;
    p.timeout_ns = a.timeout_ns;
    p.window = a.window;
    p.warm = a.warm;
    p.ws_flag = reinterpret_cast<unsigned long long *>(ws + L.off_flag);
    p.ws_hdr = reinterpret_cast<unsigned long long *>(ws + L.off_hdr);
    p.n_rec = L.n_rec;
#ifdef GQA_DEBUG
    // Test hook of the debug build only: declare one record fewer than a call
    // over full-length sequences writes (its highest record index is
    // n_rec - 2: the last CTA's last piece), so the index check on that record
    // fires; the skipped record would still have been inside the workspace.
    if (getenv("GQA_DEBUG_DECLARE_FEWER_RECORDS")) p.n_rec = L.n_rec - 2;
#endif
    p.seed = next_seed();
    cudaError_t e;
    if (a.dtype == GQA_BF16) {
        const int nmt = bf16_nmt(p.r);
        if (dec::tc_eligible(p.r, a.d_h, a.B)) {
            e = dec::run_split_tc(p, tmk, tmv, a.d_h, L.ctas, st);
        } else if (a.d_h == 128)
            e = p.r <= 4  ? run_bf16<128, 1, kStages, 4>(p, tmk, tmv, L.ctas, st)
              : nmt == 1  ? run_bf16<128, 1, kStages, 16>(p, tmk, tmv, L.ctas, st)
              : nmt == 2  ? run_bf16<128, 2, kStages, 16>(p, tmk, tmv, L.ctas, st)
                          : run_bf16<128, 4, kStages, 16>(p, tmk, tmv, L.ctas, st);
        else
            e = p.r <= 4  ? run_bf16<64, 1, kStages, 4>(p, tmk, tmv, L.ctas, st)
              : nmt == 1  ? run_bf16<64, 1, kStages, 16>(p, tmk, tmv, L.ctas, st)
              : nmt == 2  ? run_bf16<64, 2, kStages, 16>(p, tmk, tmv, L.ctas, st)
                          : run_bf16<64, 4, kStages, 16>(p, tmk, tmv, L.ctas, st);
        if (e != cudaSuccess) return e;
        return a.d_h == 128 ? run_combine<128, true>(p, L.ctas, st) : run_combine<64, true>(p, L.ctas, st);
    }
    e = a.d_h == 128 ? run_f32<128>(p, L.ctas, st) : run_f32<64>(p, L.ctas, st);
    if (e != cudaSuccess) return e;
    return a.d_h == 128 ? run_combine<128, false>(p, L.ctas, st) : run_combine<64, false>(p, L.ctas, st);
}

}  // namespace gqa
