"""Tolerances for comparing kernel outputs (as stored) with the fp64 oracle.

bf16 inputs with fp32 accumulation: max abs error 2e-3 and max relative error
1e-2; fp32 inputs: 1e-5 for both.  Two readings are used:

* ``assert_strict``: max_i |d_i| <= atol AND max_i |d_i| / max_i |ref_i| <= rtol
  (normwise relative).  Used at the benchmark workloads, whose outputs are
  small averages (|out| << 1).
* ``assert_close``: |d_i| <= atol + rtol * |ref_i| for every i.  Used in the
  sweeps, where a short sequence makes |out| ~ 1 and rounding the output to
  bf16 alone moves it by up to 2^-9 |out| > 2e-3.
Every value must be finite.
"""
import torch

TOL = {torch.bfloat16: (2e-3, 1e-2), torch.float32: (1e-5, 1e-5)}


def errors(got, ref):
    got = got.detach().double().cpu()
    ref = ref.detach().double().cpu()
    d = (got - ref).abs()
    if d.numel() == 0:
        return 0.0, 0.0
    maxabs = d.max().item()
    refmax = ref.abs().max().item()
    return maxabs, (maxabs / refmax if refmax > 0 else maxabs)


def assert_strict(got, ref, dtype):
    atol, rtol = TOL[dtype]
    g = got.detach().double().cpu()
    assert torch.isfinite(g).all(), "non-finite output"
    maxabs, normrel = errors(got, ref)
    assert maxabs <= atol and normrel <= rtol, (maxabs, normrel)
    return maxabs, normrel


def assert_close(got, ref, dtype):
    atol, rtol = TOL[dtype]
    g = got.detach().double().cpu()
    r = ref.detach().double().cpu()
    assert torch.isfinite(g).all(), "non-finite output"
    d = (g - r).abs()
    bad = d > atol + rtol * r.abs()
    assert not bad.any(), "max excess %g at %s" % ((d - atol - rtol * r.abs()).max().item(),
                                                   bad.nonzero()[:4].tolist())
    return errors(got, ref)


def assert_close_plus(got, ref, dtype, extra):
    """assert_close with an extra per-element allowance ``extra`` (>= 0), for
    outputs computed through intermediates stored in bf16: the kernel rounds
    its fp32 intermediate and the oracle its fp64 one, and near a rounding
    boundary the two land one bf16 step apart, which later steps carry on."""
    atol, rtol = TOL[dtype]
    g = got.detach().double().cpu()
    r = ref.detach().double().cpu()
    assert torch.isfinite(g).all(), "non-finite output"
    d = (g - r).abs()
    bound = atol + rtol * r.abs() + extra.double().cpu()
    assert not (d > bound).any(), "max excess %g" % (d - bound).max().item()
    return errors(got, ref)


def assert_rows(got, ref, dtype, strict_below=0.5):
    """Row by row (rows of the last dimension): rows whose max |ref| is below
    ``strict_below`` get the strict form (max abs <= atol and max abs / max |ref|
    <= rtol, over the row); the others, whose O(1) values bf16 storage alone
    moves by more than atol, get the per-element form.  Returns the number of
    rows checked in the strict form."""
    atol, rtol = TOL[dtype]
    g = got.detach().double().cpu().reshape(-1, got.shape[-1])
    r = ref.detach().double().cpu().reshape(-1, ref.shape[-1])
    assert torch.isfinite(g).all(), "non-finite output"
    d = (g - r).abs()
    rmax = r.abs().amax(dim=1)
    dmax = d.amax(dim=1)
    strict = rmax < strict_below
    bad_strict = strict & ((dmax > atol) | (dmax > rtol * rmax))
    assert not bad_strict.any(), "strict rows failing: %s (max abs %s, row max %s)" % (
        bad_strict.nonzero()[:4].flatten().tolist(), dmax[bad_strict][:4].tolist(),
        rmax[bad_strict][:4].tolist())
    loose = ~strict
    if loose.any():
        excess = (d[loose] - atol - rtol * r[loose].abs()).amax().item()
        assert excess <= 0, "per-element rows: max excess %g" % excess
    return int(strict.sum())


def full_rows(S, H, seed, n_random, b_edge=1, head_edge=37):
    """Sampled (b, s, head) rows of a [2, S, H] prefill: both ends of every 128-row
    tile of one (b, head), plus n_random seeded random rows."""
    picks = {(0, 0, 0), (1, S - 1, H - 1)}
    for t in range(0, S, 128):
        picks.add((b_edge, t, head_edge))
        picks.add((b_edge, min(S - 1, t + 127), head_edge))
    gen = torch.Generator().manual_seed(seed)
    while len(picks) < 2 + 2 * ((S + 127) // 128) + n_random:
        b, s, i = (int(torch.randint(0, n, (1,), generator=gen)) for n in (2, S, H))
        picks.add((b, s, i))
    return sorted(picks)
