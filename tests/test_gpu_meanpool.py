"""Mean-pool init through the C ABI vs the oracle: bit-exact (same binary64
operations in the same order, one nearest-even rounding)."""
import pytest
import torch

import gqa_inputs as gi
import oracle

pytestmark = pytest.mark.gpu


def bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def run(gqa, wk, wv, G):
    ok, ov = gqa.meanpool_kv(wk.cuda(), wv.cuda(), G)
    gqa.get_status()
    return ok.cpu(), ov.cpu()


def test_meanpool_full_workload_bit_exact(gqa):
    """W_K, W_V [64, 128, 8192] bf16 ~ N(0, 0.02) into 8 groups."""
    wk, wv = gi.workload_inputs("meanpool_init")
    ok, ov = run(gqa, wk, wv, 8)
    assert torch.equal(bits(ok), bits(oracle.meanpool(wk, 8)))
    assert torch.equal(bits(ov), bits(oracle.meanpool(wv, 8)))


@pytest.mark.parametrize("H,G,d_h,d", [(8, 2, 4, 16), (12, 4, 3, 5), (16, 16, 8, 8),
                                       (32, 1, 8, 24), (6, 2, 7, 9), (64, 8, 128, 64)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_meanpool_shapes_bit_exact(gqa, H, G, d_h, d, dtype):
    wk, wv = gi.meanpool_inputs(H, d_h, d, dtype=dtype, seed=H * 31 + d, std=0.5)
    ok, ov = run(gqa, wk, wv, G)
    assert torch.equal(bits(ok), bits(oracle.meanpool(wk, G)))
    assert torch.equal(bits(ov), bits(oracle.meanpool(wv, G)))


def test_meanpool_integer_coded(gqa):
    H, G = 16, 4
    e = torch.arange(8 * 16, dtype=torch.float32).reshape(8, 16) % 16
    W = (16.0 * torch.arange(H, dtype=torch.float32)[:, None, None] + e[None]).to(torch.bfloat16)
    ok, ov = run(gqa, W, W.flip(0).contiguous(), G)
    r = H // G
    for g in range(G):
        exp = sum(W[g * r + j].double() for j in range(r)) / r
        assert torch.equal(ok[g].double(), oracle.round_to(exp, torch.bfloat16).double())


def _same_bits_or_both_nan(a, b):
    nan = torch.isnan(a.float())
    return torch.equal(nan, torch.isnan(b.float())) and torch.equal(bits(a)[~nan], bits(b)[~nan])


def _bf16_mix(kind, H, n, seed):
    """bf16 [H, n] inputs over the whole bf16 range, by kind."""
    gen = torch.Generator().manual_seed(seed)
    z = torch.randn(H, n, generator=gen, dtype=torch.float64)
    if kind == "wide":  # exponents spread over 2^-40 .. 2^40 per element: the sums round
        x = z * torch.exp2(torch.randint(-40, 40, (H, n), generator=gen).double())
    elif kind == "edge":  # exponent spreads of 0..15 per group, full mantissas, a few negatives
        base = torch.randint(20, 200, (1, n), generator=gen)
        ex = base + torch.randint(0, 16, (H, n), generator=gen)
        mant = torch.randint(0, 128, (H, n), generator=gen).double()
        mant[:, ::2] = 127
        sign = torch.where(torch.rand(H, n, generator=gen, dtype=torch.float64) < 0.1, -1.0, 1.0)
        x = sign * (1 + mant / 128) * torch.exp2(ex.double() - 127)
    else:  # "special": zeros, subnormals, +-inf, NaN, near-overflow values, cancelling pairs
        x = z.clone()
        u = torch.rand(H, n, generator=gen, dtype=torch.float64)
        x[u < 0.01] = 0.0
        x[(u >= 0.01) & (u < 0.02)] = float("inf")
        x[(u >= 0.02) & (u < 0.025)] = float("-inf")
        x[(u >= 0.025) & (u < 0.03)] = float("nan")
        x[(u >= 0.03) & (u < 0.04)] = 1e-39
        x[(u >= 0.04) & (u < 0.05)] = 3.3e38
        x[1::2, ::3] = -x[0::2, ::3][: x[1::2, ::3].shape[0]]
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("H,G", [(64, 8), (48, 4), (8, 8), (64, 1), (12, 4)])
@pytest.mark.parametrize("kind", ["wide", "edge", "special"])
def test_meanpool_extreme_values_bit_exact(gqa, H, G, kind):
    """Exponent spreads that make the binary64 sums round, full mantissas,
    zeros, subnormals, +-inf, NaN, near-overflow values and cancelling pairs:
    every output keeps the bits of the binary64 mean (NaN stays NaN)."""
    d_h, d = 16, 64
    wk = _bf16_mix(kind, H, d_h * d, seed=H * 7 + G).view(H, d_h, d)
    wv = _bf16_mix(kind, H, d_h * d, seed=H * 7 + G + 1).view(H, d_h, d)
    ok, ov = run(gqa, wk, wv, G)
    assert _same_bits_or_both_nan(ok, oracle.meanpool(wk, G))
    assert _same_bits_or_both_nan(ov, oracle.meanpool(wv, G))


def test_meanpool_unaligned_views(gqa):
    """Element offsets that break 16-byte alignment take the element-wise kernel."""
    H, G, d_h, d = 8, 2, 5, 7
    base = torch.randn(2 * H * d_h * d + 3, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    dev = base.cuda()
    n = H * d_h * d
    wk = dev[1:1 + n].view(H, d_h, d)
    wv = dev[2 + n:2 + 2 * n].view(H, d_h, d)
    ok, ov = gqa.meanpool_kv(wk, wv, G)
    gqa.get_status()
    assert torch.equal(bits(ok.cpu()), bits(oracle.meanpool(wk.cpu(), G)))
    assert torch.equal(bits(ov.cpu()), bits(oracle.meanpool(wv.cpu(), G)))


# ------------------------------------------------------------ the alternatives to the mean

@pytest.mark.parametrize("H,G,d_h,d", [(64, 8, 128, 64), (12, 4, 3, 5), (16, 1, 8, 24)])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_init_select_and_weighted_bit_exact(gqa, H, G, d_h, d, dtype):
    wk, wv = gi.meanpool_inputs(H, d_h, d, dtype=dtype, seed=H + 3 * d, std=0.5)
    r = H // G
    for sel in sorted({0, r - 1}):
        ok, ov = gqa.init_kv_heads(wk.cuda(), wv.cuda(), G, mode="select", select=sel)
        gqa.get_status()
        assert torch.equal(bits(ok.cpu()), bits(oracle.init_heads(wk, G, "select", select=sel)))
        assert torch.equal(bits(ov.cpu()), bits(oracle.init_heads(wv, G, "select", select=sel)))
    w = torch.rand(2, H, generator=torch.Generator().manual_seed(H)) + 0.1
    ok, ov = gqa.init_kv_heads(wk.cuda(), wv.cuda(), G, mode="weighted", head_weights=w.cuda())
    gqa.get_status()
    assert torch.equal(bits(ok.cpu()), bits(oracle.init_heads(wk, G, "weighted", weights=w[0].double())))
    assert torch.equal(bits(ov.cpu()), bits(oracle.init_heads(wv, G, "weighted", weights=w[1].double())))
    # the mean through the same entry point equals gqa_meanpool_kv's
    ok, ov = gqa.init_kv_heads(wk.cuda(), wv.cuda(), G, mode="mean")
    gqa.get_status()
    assert torch.equal(bits(ok.cpu()), bits(oracle.meanpool(wk, G)))


def test_init_rejects_bad_selection(gqa):
    wk, wv = gi.meanpool_inputs(8, 4, 8, seed=1)
    with pytest.raises(gqa.GQAError):
        gqa.init_kv_heads(wk.cuda(), wv.cuda(), 2, mode="select", select=4)
    with pytest.raises(gqa.GQAError):
        gqa.init_kv_heads(wk.cuda(), wv.cuda(), 2, mode="weighted")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_meanpool_reads_what_the_kernel_before_wrote(gqa, dtype):
    """The mean-pool kernels start as programmatic dependents and touch only
    addresses before they wait: weights written by the kernel launched just
    before them (here a torch elementwise kernel, alternating between two
    contents) must be the ones they average."""
    H, G, d_h, d = 16, 4, 64, 256
    wk, wv = gi.meanpool_inputs(H, d_h, d, dtype=dtype, seed=5, std=0.5)
    wk2, wv2 = gi.meanpool_inputs(H, d_h, d, dtype=dtype, seed=6, std=0.5)
    dk, dv = torch.empty_like(wk).cuda(), torch.empty_like(wv).cuda()
    srcs = [(wk.cuda(), wv.cuda()), (wk2.cuda(), wv2.cuda())]
    outs = []
    for i in range(6):
        sk, sv = srcs[i % 2]
        torch.mul(sv, 1, out=dv)   # an elementwise kernel writes the inputs ...
        torch.mul(sk, 1, out=dk)
        outs.append(gqa.meanpool_kv(dk, dv, G))  # ... and the mean-pool follows at once
    gqa.get_status()
    for i, (ok, ov) in enumerate(outs):
        k, v = (wk, wv) if i % 2 == 0 else (wk2, wv2)
        assert torch.equal(bits(ok.cpu()), bits(oracle.meanpool(k, G))), i
        assert torch.equal(bits(ov.cpu()), bits(oracle.meanpool(v, G))), i
