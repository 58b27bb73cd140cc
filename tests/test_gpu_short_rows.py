"""Rows over few keys: within one bf16 step of the fp64 value.

Rows that attend over at most 128 keys in prefill (the first query tile),
or 256 cached positions in decode, carry P as two bf16 terms (P_hi + P_lo,
about 16 significant bits) because the rounding of a one-term P does not
average out over so few keys.  Their outputs, O(1) in size, are then fixed
up to the final rounding to bf16: every element must be within one bf16
step (2^-8 relative) of the fp64 value, plus 1e-4 absolute for cancelling
sums.  This is tighter than the bf16 tolerance's per-element form (1e-2
relative), which a mismatch between the P of the products and the P of the
row sum (2^-9 relative, once present in the warp-MMA decode kernel) passed.
"""
import pytest
import torch

import gqa_inputs as gi
import oracle

pytestmark = pytest.mark.gpu


def assert_one_step(got, ref):
    g = got.detach().double().cpu()
    r = ref.detach().double().cpu()
    assert torch.isfinite(g).all()
    d = (g - r).abs()
    bound = 2.0 ** -8 * r.abs() + 1e-4
    assert not (d > bound).any(), "max excess %g (max |d| %g)" % ((d - bound).max().item(), d.max().item())


@pytest.mark.parametrize("H,G", [(16, 4), (32, 2), (8, 8)])  # warp MMA (r 4, 1) and tcgen05 (r 16)
@pytest.mark.parametrize("d_h", [64, 128])
def test_decode_short_caches(gqa, H, G, d_h):
    x = gi.decode_inputs(7, H, G, d_h, 256, torch.bfloat16, seed=970 + H + d_h,
                         seqlens=[1, 2, 3, 17, 64, 129, 256])
    out = gqa.decode(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.cuda(), x.scale)
    gqa.get_status()
    assert_one_step(out, oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale))


@pytest.mark.parametrize("H,G,d_h", [(8, 2, 128), (6, 6, 64), (4, 1, 128)])
def test_prefill_first_tile_rows(gqa, H, G, d_h):
    x = gi.prefill_inputs(2, 128, H, G, d_h, torch.bfloat16, seed=980 + H + d_h)
    out = gqa.prefill_causal(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.scale)
    gqa.get_status()
    assert_one_step(out, oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale))
