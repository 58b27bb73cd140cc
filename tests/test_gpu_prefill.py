"""Causal GQA prefill (tcgen05) through the C ABI vs the fp64 oracle.

Ordered from one CTA (one 128-row query tile, diagonal KV tile only) up to the
full B=2, S=8192, H=64, G=8 workload (sampled rows).  Ragged S (not a multiple
of the 128-row tile) and several group sizes are covered.
"""
import pytest
import torch

import gqa_inputs as gi
import oracle
from parity import assert_close, assert_rows, full_rows

pytestmark = pytest.mark.gpu


def run(gqa, x):
    out = gqa.prefill_causal(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.scale)
    gqa.get_status()
    return out.cpu()


@pytest.mark.parametrize("B,S,H,G", [
    (1, 128, 2, 1),      # one CTA, diagonal tile only
    (1, 256, 2, 1),      # two query tiles, one and two KV tiles
    (1, 384, 4, 2),
    (2, 200, 8, 2),      # ragged: 200 = 128 + 72
    (1, 1, 2, 1),        # a single position
    (1, 129, 4, 1),      # one row past a tile
    (2, 77, 16, 2),      # r = 8
    (1, 1000, 8, 4),     # r = 2
    (1, 640, 32, 1),     # r = 32 (MQA-like)
])
def test_prefill_small(gqa, B, S, H, G):
    x = gi.prefill_inputs(B, S, H, G, 128, torch.bfloat16, seed=S + 7 * H)
    got = run(gqa, x)
    ref = oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale)
    assert_close(got, ref, torch.bfloat16)


@pytest.mark.parametrize("B,S,H,G,d_h", [
    (1, 300, 4, 4, 128),     # G = H: MHA, every CTA holds one head
    (2, 200, 6, 6, 64),      # MHA at d_h = 64, ragged S
    (1, 384, 6, 2, 128),     # r = 3: one pair and one lone head per group
    (2, 257, 10, 2, 128),    # r = 5, ragged S
    (1, 640, 8, 1, 64),      # G = 1: MQA at d_h = 64
    (1, 128, 2, 1, 64),      # one CTA at d_h = 64
    (2, 777, 8, 2, 64),      # r = 4 at d_h = 64, ragged S
    (1, 1, 3, 1, 64),        # a single position, r = 3
])
def test_prefill_group_sizes_and_head_dims(gqa, B, S, H, G, d_h):
    x = gi.prefill_inputs(B, S, H, G, d_h, torch.bfloat16, seed=S + 13 * H + d_h)
    got = run(gqa, x)
    ref = oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale)
    assert_close(got, ref, torch.bfloat16)


@pytest.mark.parametrize("H,G,d_h", [(8, 2, 128), (6, 2, 64), (4, 1, 128)])
def test_prefill_gqa_equals_mha_on_repeated_kv(gqa, H, G, d_h):
    """The page's broadcast identity on the GPU: GQA prefill equals MHA prefill
    (G = H) on K/V repeat-interleaved H/G times along the head axis, bit for
    bit, since each query head sees the same K/V values in the same order."""
    x = gi.prefill_inputs(1, 300, H, G, d_h, torch.bfloat16, seed=40 + H + d_h)
    gqa_out = run(gqa, x)
    r = H // G
    xr = gi.PrefillInputs(x.q, x.k.repeat_interleave(r, dim=2).contiguous(),
                          x.v.repeat_interleave(r, dim=2).contiguous(), x.scale, 1, 300, H, H, d_h)
    mha_out = run(gqa, xr)
    assert torch.equal(gqa_out, mha_out)
    assert_close(gqa_out, oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale), torch.bfloat16)


def test_prefill_deterministic(gqa):
    x = gi.prefill_inputs(1, 512, 8, 2, 128, torch.bfloat16, seed=3)
    assert torch.equal(run(gqa, x), run(gqa, x))


def test_prefill_last_row_matches_decode(gqa):
    """Last prefill row over S keys equals one decode step over the same K/V."""
    x = gi.prefill_inputs(2, 300, 8, 2, 128, torch.bfloat16, seed=5)
    pre = run(gqa, x)
    kc = x.k.permute(0, 2, 1, 3).contiguous()
    vc = x.v.permute(0, 2, 1, 3).contiguous()
    dec = gqa.decode(x.q[:, -1].contiguous().cuda(), kc.cuda(), vc.cuda(),
                     torch.tensor([300, 300], dtype=torch.int32, device="cuda"), x.scale).cpu()
    ref = oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale)[:, -1]
    assert_close(pre[:, -1], ref, torch.bfloat16)
    assert_close(dec, ref, torch.bfloat16)


def test_causal_prefill_full_workload(gqa):
    """B=2, S=8192, H=64, G=8, d_h=128: 1,154 sampled rows (every tile edge of one
    (b, head) and 1,024 random rows), strict form on every row whose output stays
    below 0.5 in magnitude."""
    x = gi.workload_inputs("causal_prefill")
    got = run(gqa, x)
    assert torch.isfinite(got.float()).all()
    S, H = 8192, 64
    picks = full_rows(S, H, seed=11, n_random=1024)
    assert len(picks) >= 1024 + 128
    rows = [(b * S + s) * H + i for b, s, i in picks]
    ref = oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale, rows=rows)
    n_strict = assert_rows(got.reshape(-1, 128)[rows], ref, torch.bfloat16)
    assert n_strict >= 0.95 * len(rows), n_strict  # all but the first few positions
