"""Pins for the fp64 oracle: each check ties it to something other than itself.

Sources (page title, section):
  KB  = "Grouped-Query Attention" (llm-arch-kb): s1 Premise, s2 Derivation,
        s3 Reference implementation.
  CA  = "GQA: Training Generalized Multi-Query Transformer Models from
        Multi-Head Checkpoints" (crackai.dev): How It Works, Key Takeaways.
  AIU = "Grouped-Query Attention" (AI Understanding guide): FAQ.
  MQ  = "Multi-Query and Grouped-Query Attention" (praveentn.live).

Kinds of pin: worked values printed on the pages (tests/golden), closed forms,
invariants (G=H is MHA, G=1 is MQA, GQA is MHA on repeat-interleaved K/V),
an independent library routine (torch SDPA in float64), and a 60-digit
decimal brute force on tiny inputs.
"""
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import gqa_inputs as gi
import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _records(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


# ----------------------------------------------------------------- KV bytes

def test_kv_cache_bytes_worked_values():
    """KB s1 and s2 print the per-token and total cache sizes for Llama 2 70B."""
    recs = list(_records("kv_cache_worked_values.txt"))
    assert len(recs) == 2
    for rec in recs:
        H, G, d_h, L, eb, per_tok = map(int, rec[1:7])
        assert oracle.kv_cache_bytes(G, d_h, L, eb) == per_tok
        rest = list(map(int, rec[7:]))
        for T, total in zip(rest[::2], rest[1::2]):
            assert oracle.kv_cache_bytes(G, d_h, L, eb) * T == total
    # 2.5 MiB and 320 KiB per token, as the pages also say
    assert oracle.kv_cache_bytes(64, 128, 80, 2) == int(2.5 * 2**20)
    assert oracle.kv_cache_bytes(8, 128, 80, 2) == 320 * 2**10


def test_kv_cache_bytes_closed_forms():
    """CA How It Works: MHA 2*H*d_h, MQA 2*d_h, GQA 2*G*d_h scalars per token."""
    for H, d_h in [(32, 128), (64, 128), (8, 64)]:
        assert oracle.kv_cache_bytes(H, d_h, 1, 1) == 2 * H * d_h          # MHA
        assert oracle.kv_cache_bytes(1, d_h, 1, 1) == 2 * d_h              # MQA
        # KB s2: MHA stores 2*H*d_h = 2*d scalars with d = H*d_h
        assert oracle.kv_cache_bytes(H, d_h, 1, 1) == 2 * (H * d_h)
    for H, G, factor in (map(int, r) for r in _records("head_ratios.txt")):
        mha = oracle.kv_cache_bytes(H, 128, 80, 2)
        gqa = oracle.kv_cache_bytes(G, 128, 80, 2)
        assert mha == factor * gqa


# ----------------------------------------------------------------- group map

@pytest.mark.parametrize("H,G", [(8, 2), (32, 8), (64, 8), (32, 1), (32, 32), (12, 4),
                                 (32, 2), (32, 4), (32, 16), (6, 3)])
def test_group_map_is_repeat_interleave(H, G):
    """KB s2 g(i)=ceil(iG/H) must agree with KB s3's repeat_interleave broadcast."""
    r = H // G
    via_sketch = torch.arange(G).repeat_interleave(r)  # KV head seen by each query head
    got = [oracle.group_of_head(i, H, G) for i in range(H)]
    assert got == via_sketch.tolist()
    # contiguous groups of H/G heads, every group used
    assert sorted(set(got)) == list(range(G))
    assert all(got.count(g) == r for g in range(G))


def test_group_map_llama2_70b():
    """CA Key Takeaways: 64 query heads and 8 KV heads form 8 groups of 8."""
    got = [oracle.group_of_head(i, 64, 8) for i in range(64)]
    assert [got.count(g) for g in range(8)] == [8] * 8
    assert got[:8] == [0] * 8 and got[-8:] == [7] * 8


# ----------------------------------------------------------------- decode

def _sdpa_decode(x):
    """Library reference: torch SDPA in float64, one sequence at a time."""
    outs = []
    for b in range(x.B):
        n = int(x.seqlens[b])
        q = x.q[b:b + 1].double()[:, :, None, :]                    # [1,H,1,d]
        k = x.k_cache[b:b + 1, :, :n].double()                     # [1,G,n,d]
        v = x.v_cache[b:b + 1, :, :n].double()
        outs.append(F.scaled_dot_product_attention(q, k, v, scale=x.scale,
                                                   enable_gqa=True)[:, :, 0, :])
    return torch.cat(outs, 0)


@pytest.mark.parametrize("B,H,G,d_h,T,dtype,ragged", [
    (1, 8, 2, 64, 128, torch.float32, None),
    (2, 8, 8, 32, 50, torch.float32, None),
    (3, 16, 1, 16, 37, torch.bfloat16, (1, 37)),
    (2, 12, 4, 8, 70, torch.bfloat16, (5, 70)),
    (4, 32, 8, 128, 300, torch.bfloat16, (100, 300)),
])
def test_decode_matches_sdpa_fp64(B, H, G, d_h, T, dtype, ragged):
    x = gi.decode_inputs(B, H, G, d_h, T, dtype, seed=1, ragged=ragged)
    got = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    ref = _sdpa_decode(x)
    assert torch.isfinite(got).all()     # NaN padding past seqlens is never read
    assert (got - ref).abs().max().item() < 1e-12


def test_decode_G_eq_H_is_per_head_mha():
    """KB s1/CA: G = H is MHA (each query head owns its K/V head)."""
    x = gi.decode_inputs(2, 8, 8, 16, 40, torch.bfloat16, seed=2, ragged=(3, 40))
    gqa = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    mha = oracle.mha_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    assert torch.equal(gqa, mha)


def test_decode_is_mha_on_repeat_interleaved_kv():
    """KB s3: broadcasting each KV head to H/G query heads gives GQA from MHA."""
    for G in (1, 2, 4):
        x = gi.decode_inputs(2, 8, G, 16, 33, torch.bfloat16, seed=3, ragged=(1, 33))
        r = 8 // G
        k_rep = np.repeat(x.k_cache.float().numpy(), r, axis=1)
        v_rep = np.repeat(x.v_cache.float().numpy(), r, axis=1)
        gqa = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
        mha = oracle.mha_decode(x.q, torch.from_numpy(k_rep), torch.from_numpy(v_rep),
                                x.seqlens, x.scale)
        assert torch.equal(gqa, mha)


def test_decode_G1_is_mqa():
    """MQ 'The asymmetric cut': with one shared K/V, heads differ only by q."""
    x = gi.decode_inputs(1, 4, 1, 16, 20, torch.float32, seed=4)
    q = x.q.clone()
    q[0, 3] = q[0, 1]                     # two heads with the same query
    out = oracle.gqa_decode(q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    assert torch.equal(out[0, 3], out[0, 1])
    # and each head equals single-head attention against the one KV head
    for i in range(4):
        one = oracle.mha_decode(q[:, i:i + 1], x.k_cache, x.v_cache, x.seqlens, x.scale)
        assert torch.equal(one[0, 0], out[0, i])


def test_decode_closed_forms():
    x = gi.decode_inputs(2, 4, 2, 8, 16, torch.float64, seed=5, seqlens=[16, 9])
    # q = 0: uniform softmax, output = mean of the valid values
    out = oracle.gqa_decode(torch.zeros_like(x.q), x.k_cache, x.v_cache, x.seqlens, x.scale)
    for b, n in enumerate([16, 9]):
        for i in range(4):
            mean = x.v_cache[b, i // 2, :n].mean(0)
            assert (out[b, i] - mean).abs().max() < 1e-14
    # scale = 0 gives the same
    out0 = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, 0.0)
    assert (out0 - out).abs().max() < 1e-14
    # one cached token: output is that value exactly
    out1 = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, [1, 1], x.scale)
    for i in range(4):
        assert torch.equal(out1[:, i], x.v_cache[:, i // 2, 0])
    # constant values: output is that constant
    vc = torch.full_like(x.v_cache, 0.375)
    outc = oracle.gqa_decode(x.q, x.k_cache, vc, x.seqlens, x.scale)
    assert (outc - 0.375).abs().max() < 1e-15
    # empty cache: zero row (reading of an empty softmax)
    oute = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, [0, 9], x.scale)
    assert torch.equal(oute[0], torch.zeros_like(oute[0]))
    # a dominant key: q aligned with key j and large gives v_j
    q = torch.zeros_like(x.q)
    q[0, 0] = 60.0 * x.k_cache[0, 0, 5] / x.k_cache[0, 0, 5].norm()
    outd = oracle.gqa_decode(q, x.k_cache, x.v_cache, x.seqlens, 1.0)
    assert (outd[0, 0] - x.v_cache[0, 0, 5]).abs().max() < 1e-6


def test_decode_permutation_and_linearity():
    """Softmax attention is invariant to cache order and linear in V."""
    x = gi.decode_inputs(1, 8, 2, 16, 24, torch.float64, seed=6)
    perm = torch.randperm(24, generator=torch.Generator().manual_seed(0))
    a = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    b = oracle.gqa_decode(x.q, x.k_cache[:, :, perm], x.v_cache[:, :, perm], x.seqlens, x.scale)
    assert (a - b).abs().max() < 1e-14
    c = oracle.gqa_decode(x.q, x.k_cache, 3.0 * x.v_cache + 1.0, x.seqlens, x.scale)
    assert (c - (3.0 * a + 1.0)).abs().max() < 1e-13


def _decimal_attention(qv, keys, vals, scale):
    """Brute force at 60 digits: exp without max subtraction, plain sums."""
    getcontext().prec = 60
    sc = Decimal(repr(scale))
    e = []
    for k in keys:
        s = sum(Decimal(repr(a)) * Decimal(repr(b)) for a, b in zip(qv, k)) * sc
        e.append(s.exp())
    den = sum(e)
    return [float(sum(ei * Decimal(repr(v[c])) for ei, v in zip(e, vals)) / den)
            for c in range(len(vals[0]))]


def test_decode_decimal_brute_force():
    x = gi.decode_inputs(2, 4, 2, 4, 6, torch.float32, seed=7, seqlens=[6, 3])
    out = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    for b in range(2):
        n = int(x.seqlens[b])
        for i in range(4):
            g = i // 2
            ref = _decimal_attention(x.q[b, i].double().tolist(),
                                     x.k_cache[b, g, :n].double().tolist(),
                                     x.v_cache[b, g, :n].double().tolist(), x.scale)
            assert max(abs(u - v) for u, v in zip(out[b, i].tolist(), ref)) < 1e-14


def test_decode_rows_subset_matches_full():
    x = gi.decode_inputs(3, 8, 2, 16, 30, torch.bfloat16, seed=8, ragged=(1, 30))
    full = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    rows = [0, 5, 9, 23, 17]
    part = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, rows=rows)
    assert torch.equal(part, full.reshape(-1, 16)[rows])


# ----------------------------------------------------------------- prefill

def _sdpa_prefill(x):
    q = x.q.double().permute(0, 2, 1, 3)
    k = x.k.double().permute(0, 2, 1, 3)
    v = x.v.double().permute(0, 2, 1, 3)
    o = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=x.scale,
                                       enable_gqa=True)
    return o.permute(0, 2, 1, 3)


@pytest.mark.parametrize("B,S,H,G,d_h", [(1, 17, 4, 2, 8), (2, 64, 8, 2, 32),
                                         (1, 40, 6, 3, 16), (2, 33, 4, 4, 16),
                                         (1, 50, 8, 1, 16)])
def test_prefill_matches_sdpa_fp64(B, S, H, G, d_h):
    x = gi.prefill_inputs(B, S, H, G, d_h, torch.bfloat16, seed=9)
    got = oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale)
    assert (got - _sdpa_prefill(x)).abs().max().item() < 1e-12


def test_prefill_first_row_and_last_row():
    x = gi.prefill_inputs(2, 24, 8, 2, 16, torch.bfloat16, seed=10)
    out = oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale)
    # row 0 sees only key 0: output is v_0 of its group
    for i in range(8):
        assert torch.equal(out[:, 0, i], x.v[:, 0, i // 4].double())
    # last row equals decode over the whole sequence (K/V moved to [B,G,T,d])
    dec = oracle.gqa_decode(x.q[:, -1], x.k.permute(0, 2, 1, 3), x.v.permute(0, 2, 1, 3),
                            [24, 24], x.scale)
    assert torch.equal(out[:, -1], dec)


def test_prefill_is_causal():
    """Changing keys/values after position s leaves row s unchanged."""
    x = gi.prefill_inputs(1, 20, 4, 2, 8, torch.float32, seed=11)
    a = oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale)
    k2, v2 = x.k.clone(), x.v.clone()
    k2[:, 12:] = torch.randn_like(k2[:, 12:])
    v2[:, 12:] = 1e3
    b = oracle.gqa_prefill_causal(x.q, k2, v2, x.scale)
    assert torch.equal(a[:, :12], b[:, :12])
    assert not torch.equal(a[:, 12:], b[:, 12:])


def test_prefill_rows_subset_matches_full():
    x = gi.prefill_inputs(2, 16, 4, 2, 8, torch.bfloat16, seed=12)
    full = oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale)
    rows = [0, 7, 64, 127, 100]
    part = oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale, rows=rows)
    assert torch.equal(part, full.reshape(-1, 8)[rows])


# ----------------------------------------------------------------- mean-pool

def test_meanpool_G_eq_H_is_identity():
    wk, _ = gi.meanpool_inputs(8, 4, 16, seed=13)
    assert torch.equal(oracle.meanpool(wk, 8).view(torch.int16), wk.view(torch.int16))


def test_meanpool_integer_coded_exact():
    """KB s2 averaging-init: group g's head is the mean of its H/G original heads.
    Integer-coded heads make every mean exact, so indexing errors show directly."""
    H, G, n1, n2 = 16, 4, 3, 5
    # W[i, e] = 16*i + (e mod 16): distinct per head, all below 256, so exact in bf16
    e = torch.arange(n1 * n2, dtype=torch.float64).reshape(n1, n2) % 16
    W = 16.0 * torch.arange(H, dtype=torch.float64)[:, None, None] + e[None]
    Wb = W.to(torch.bfloat16)
    assert torch.equal(Wb.double(), W)
    mean = oracle.meanpool_mean(Wb, G)
    r = H // G
    for g in range(G):
        exp = sum(W[g * r + j] for j in range(r)) / r
        assert torch.equal(mean[g], exp)


def test_meanpool_G1_is_mean_of_all_heads():
    wk, _ = gi.meanpool_inputs(8, 4, 8, dtype=torch.float32, seed=14)
    mean = oracle.meanpool_mean(wk, 1)
    assert (mean[0] - wk.double().mean(0)).abs().max() < 1e-16


def test_meanpool_parameter_saving():
    """KB s2: GQA saves 2 d^2 (1 - G/H) K/V parameters per layer, with d_h = d/H."""
    for H, G, d in [(64, 8, 8192), (32, 8, 4096), (16, 1, 1024)]:
        d_h = d // H
        mha = 2 * H * d_h * d
        gqa = 2 * G * d_h * d
        assert mha - gqa == 2 * d * d * (H - G) // H
    wk, wv = gi.meanpool_inputs(16, 4, 64, seed=15)  # d = 64, H = 16, d_h = 4
    outk, outv = oracle.meanpool(wk, 4), oracle.meanpool(wv, 4)
    saved = (wk.numel() + wv.numel()) - (outk.numel() + outv.numel())
    assert saved == 2 * 64 * 64 * (1 - 4 / 16)


# ----------------------------------------------------------------- rounding

def test_round_bf16_ties_and_specials():
    cases = [
        (1.0 + 2 ** -8, 1.0),                        # tie, even mantissa stays
        (1.0 + 3 * 2 ** -8, 1.0 + 2 ** -6),          # tie, odd mantissa rounds up
        (1.0 + 2 ** -8 + 2 ** -30, 1.0 + 2 ** -7),   # just above the tie
        (-(1.0 + 2 ** -8), -1.0),
        (2.0 ** -133, 2.0 ** -133),                  # smallest subnormal
        (2.0 ** -134, 0.0),                          # tie between 0 and it: even is 0
        (1.5 * 2.0 ** -134, 2.0 ** -133),
        (float.fromhex("0x1.fefp127"), float.fromhex("0x1.fep127")),  # max finite
        (float.fromhex("0x1.ffp127"), float("inf")),  # max + half ulp ties to 2^128
        (float("inf"), float("inf")),
        (0.0, 0.0),
    ]
    xs = torch.tensor([c[0] for c in cases], dtype=torch.float64)
    got = oracle.round_to(xs, torch.bfloat16).double().tolist()
    for (x, want), g in zip(cases, got):
        assert g == want, (x, g, want)
    assert math.isnan(oracle.round_to(torch.tensor([float("nan")]), torch.bfloat16).item())


def test_round_bf16_matches_brute_force_nearest():
    """Brute force: among all finite bf16 values pick the nearest, ties to even."""
    all_bits = torch.arange(0, 0x7F80, dtype=torch.int32).to(torch.int16)
    grid = all_bits.view(torch.bfloat16).double()                       # ascending
    gen = torch.Generator().manual_seed(16)
    xs = torch.cat([torch.randn(4000, generator=gen, dtype=torch.float64) * 10.0 ** e
                    for e in (-40, -20, -3, 0, 3, 20, 37)]).abs()
    got = oracle.round_to(xs, torch.bfloat16).view(torch.int16).to(torch.int32)
    idx = torch.searchsorted(grid, xs).clamp(1, grid.numel() - 1)
    lo, hi = grid[idx - 1], grid[idx]
    pick_hi = (xs - lo > hi - xs) | ((xs - lo == hi - xs) & (idx % 2 == 0))
    exp_bits = torch.where(pick_hi, idx, idx - 1)
    assert torch.equal(got, exp_bits.to(torch.int32))


def test_round_bf16_matches_torch_on_binary32_values():
    """On values already in binary32 the double rounding issue cannot arise, so
    torch's float32 -> bfloat16 conversion (nearest-even) is a valid reference."""
    gen = torch.Generator().manual_seed(17)
    xf = torch.randn(100000, generator=gen) * 3.0
    got = oracle.round_to(xf.double(), torch.bfloat16)
    assert torch.equal(got.view(torch.int16), xf.to(torch.bfloat16).view(torch.int16))


def test_round_f32():
    xs = torch.tensor([1.0 + 2 ** -24, 1.0 + 3 * 2 ** -24, 1e-45, 3.5e38], dtype=torch.float64)
    got = oracle.round_to(xs, torch.float32)
    assert got[0].item() == 1.0 and got[1].item() == 1.0 + 2 ** -22
    assert got[2].item() == 2 ** -149 and math.isinf(got[3].item())


def test_row_selection_rejects_out_of_range():
    x = gi.decode_inputs(1, 4, 2, 8, 8, torch.float32, seed=18)
    with pytest.raises(IndexError):
        oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, rows=[4])
    p = gi.prefill_inputs(1, 4, 2, 1, 8, torch.float32, seed=18)
    with pytest.raises(IndexError):
        oracle.gqa_prefill_causal(p.q, p.k, p.v, p.scale, rows=[-1])


# ----------------------------------------------------------------- projections

def test_project_matches_torch_matmul_fp64():
    x = gi.qkv_inputs(5, 64, 4, 2, 16, 4, seed=19)
    got = oracle.project(x.h, x.W_Q)
    assert (got - x.h.double() @ x.W_Q.double()).abs().max() < 1e-12


def test_project_one_hot_rows_pick_weight_rows():
    d, N = 32, 48
    W = torch.randn(d, N, generator=torch.Generator().manual_seed(20)).to(torch.bfloat16)
    h = torch.eye(d, dtype=torch.float64)[[3, 0, 31]]
    assert torch.equal(oracle.project(h, W), W.double()[[3, 0, 31]])


def test_qkv_append_grows_cache_by_2Gdh_scalars_per_token():
    """KB s1/s2: one key and one value vector per KV head per token, i.e. the
    closed form 2*G*d_h scalars; positions other than T_b stay as they were."""
    x = gi.qkv_inputs(3, 64, 8, 2, 16, 5, seed=21, seqlens=[0, 4, 5])
    q, k, v, kc, vc, sl, app = oracle.qkv_append(x.h, x.W_Q, x.W_K, x.W_V, x.k_cache, x.v_cache,
                                                 x.seqlens)
    assert app.tolist() == [True, True, False] and sl.tolist() == [1, 5, 5]
    changed = ((kc != x.k_cache.double()).any(-1).sum() + (vc != x.v_cache.double()).any(-1).sum())
    per_token_scalars = oracle.kv_cache_bytes(2, 16, 1, 1)
    assert int(changed) * 16 == 2 * per_token_scalars            # two appends, G vectors each
    assert q.shape == (3, 8, 16) and k.shape == (3, 2, 16)        # K/V GEMM is G/H of Q's
    assert torch.equal(kc[0, :, 0], k[0]) and torch.equal(vc[1, :, 4], v[1])


def test_qkv_append_values_are_the_head_split_projections():
    """KB s1: q = h W_Q split into H heads of d_h (head i = columns i*d_h ..),
    k and v = h W_K, h W_V split into G heads, each written at position T_b of
    its own sequence and KV head; checked against an fp64 torch matmul."""
    B, d, H, G, d_h, T = 3, 48, 6, 3, 8, 7
    x = gi.qkv_inputs(B, d, H, G, d_h, T, seed=31, seqlens=[0, 3, 6])
    q, k, v, kc, vc, sl, app = oracle.qkv_append(x.h, x.W_Q, x.W_K, x.W_V, x.k_cache, x.v_cache,
                                                 x.seqlens)
    h = x.h.double()
    tol = dict(rtol=1e-12, atol=1e-12)
    torch.testing.assert_close(q, (h @ x.W_Q.double()).view(B, H, d_h), **tol)
    torch.testing.assert_close(k, (h @ x.W_K.double()).view(B, G, d_h), **tol)
    torch.testing.assert_close(v, (h @ x.W_V.double()).view(B, G, d_h), **tol)
    for b, t in enumerate([0, 3, 6]):
        for g in range(G):
            assert torch.equal(kc[b, g, t], k[b, g]) and torch.equal(vc[b, g, t], v[b, g])
    assert sl.tolist() == [1, 4, 7]


# ----------------------------------------------------------------- sliding window

def _band_sdpa_prefill(x, W):
    """SDPA in float64 with an explicit band mask: key t visible to s iff s-W < t <= s."""
    S = x.S
    s = torch.arange(S)[:, None]
    t = torch.arange(S)[None, :]
    mask = (t <= s) & (t > s - W)
    q = x.q.double().permute(0, 2, 1, 3)
    k = x.k.double().permute(0, 2, 1, 3)
    v = x.v.double().permute(0, 2, 1, 3)
    o = F.scaled_dot_product_attention(q, k, v, attn_mask=mask, scale=x.scale, enable_gqa=True)
    return o.permute(0, 2, 1, 3)


@pytest.mark.parametrize("W", [1, 5, 16, 40])
def test_prefill_window_matches_band_masked_sdpa(W):
    x = gi.prefill_inputs(2, 40, 8, 2, 16, torch.bfloat16, seed=22 + W)
    got = oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale, window=W)
    assert (got - _band_sdpa_prefill(x, W)).abs().max() < 1e-12


def test_prefill_window_limits():
    x = gi.prefill_inputs(1, 30, 4, 2, 8, torch.float32, seed=23)
    full = oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale)
    assert torch.equal(oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale, window=30), full)
    assert torch.equal(oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale, window=1000), full)
    one = oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale, window=1)
    for i in range(4):                       # W = 1: every query sees only itself
        assert torch.equal(one[0, :, i], x.v[0, :, i // 2].double())


def test_decode_window_is_decode_on_the_last_W_positions():
    x = gi.decode_inputs(3, 8, 2, 16, 50, torch.bfloat16, seed=24, seqlens=[50, 7, 23])
    W = 10
    got = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, window=W)
    for b, T in enumerate([50, 7, 23]):
        lo = max(0, T - W)
        ref = oracle.gqa_decode(x.q[b:b + 1], x.k_cache[b:b + 1, :, lo:T], x.v_cache[b:b + 1, :, lo:T],
                                [T - lo], x.scale)
        assert torch.equal(got[b], ref[0])
    assert torch.equal(oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, window=50),
                       oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale))


# ----------------------------------------------------------------- init variants

def test_init_select_picks_one_head_per_group():
    """KB s2: the alternative of picking a single head from each group."""
    wk, _ = gi.meanpool_inputs(16, 4, 8, seed=25)
    for sel in range(4):
        got = oracle.init_heads(wk, 4, "select", select=sel)
        assert torch.equal(got.view(torch.int16), wk[sel::4].view(torch.int16))


def test_init_weighted_special_cases():
    """Weighted averaging (KB s4): 1/r weights give the mean (exact for r a power
    of two), one-hot weights give selection, doubling the weights doubles the result."""
    wk, _ = gi.meanpool_inputs(16, 4, 8, seed=26, std=0.5)
    H, G, r = 16, 4, 4
    mean = oracle.meanpool(wk, G)
    assert torch.equal(oracle.init_heads(wk, G, "weighted", weights=[1 / r] * H).view(torch.int16),
                       mean.view(torch.int16))
    onehot = [1.0 if i % r == 2 else 0.0 for i in range(H)]
    assert torch.equal(oracle.init_heads(wk, G, "weighted", weights=onehot).view(torch.int16),
                       oracle.init_heads(wk, G, "select", select=2).view(torch.int16))
    wts = torch.rand(H, generator=torch.Generator().manual_seed(27)).double()
    a = oracle.init_heads(wk, G, "weighted", weights=wts, out_dtype=torch.float32)
    b = oracle.init_heads(wk, G, "weighted", weights=2 * wts, out_dtype=torch.float32)
    assert torch.equal(2 * a, b)
    ref = torch.stack([sum(float(wts[g * r + j]) * wk[g * r + j].double() for j in range(r)) for g in range(G)])
    assert (a.double() - ref).abs().max() < 1e-6


def test_layer_step_with_identity_output_projection_is_the_attention():
    """With W_O = I (d = H*d_h) the layer output is the attention output itself."""
    H, G, d_h = 4, 2, 32
    d = H * d_h
    x = gi.qkv_inputs(2, d, H, G, d_h, 9, seed=28, seqlens=[3, 8])
    eye = torch.eye(d, dtype=torch.bfloat16)
    out, sl = oracle.layer_decode_step(x.h, x.W_Q, x.W_K, x.W_V, eye, x.k_cache, x.v_cache,
                                       x.seqlens, d_h ** -0.5)
    q, k, v, kc, vc, sl2, _ = oracle.qkv_append(x.h, x.W_Q, x.W_K, x.W_V, x.k_cache, x.v_cache,
                                                x.seqlens)
    st = torch.bfloat16
    attn = oracle.gqa_decode(oracle.round_to(q, st), oracle.round_to(kc, st), oracle.round_to(vc, st),
                             sl2, d_h ** -0.5)
    assert torch.equal(out, oracle.round_to(attn, st).double().reshape(2, d))
    assert sl.tolist() == [4, 9]


def test_layer_step_output_is_concatenated_heads_times_W_O():
    """KB s2 / s3: the layer output is the H heads' attention outputs laid side
    by side ([B, H*d_h], head i at columns i*d_h ..) times W_O [H*d_h, d]; a
    non-square W_O fixes the orientation.  Checked with an fp64 torch matmul."""
    B, H, G, d_h, d = 2, 4, 2, 16, 40
    x = gi.qkv_inputs(B, d, H, G, d_h, 9, seed=32, seqlens=[2, 7])
    W_O = (torch.randn(H * d_h, d, generator=torch.Generator().manual_seed(33)) * 0.1).to(torch.bfloat16)
    out, sl = oracle.layer_decode_step(x.h, x.W_Q, x.W_K, x.W_V, W_O, x.k_cache, x.v_cache,
                                       x.seqlens, d_h ** -0.5)
    q, k, v, kc, vc, sl2, _ = oracle.qkv_append(x.h, x.W_Q, x.W_K, x.W_V, x.k_cache, x.v_cache,
                                                x.seqlens)
    st = torch.bfloat16
    attn = oracle.gqa_decode(oracle.round_to(q, st), oracle.round_to(kc, st), oracle.round_to(vc, st),
                             sl2, d_h ** -0.5)
    concat = torch.cat([oracle.round_to(attn, st)[:, i].double() for i in range(H)], dim=1)
    assert out.shape == (B, d)
    torch.testing.assert_close(out, concat @ W_O.double(), rtol=1e-12, atol=1e-12)
    assert sl.tolist() == [3, 8]
