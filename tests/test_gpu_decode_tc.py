"""Decode for groups of 16 or more query heads (the tcgen05 split kernel)
through the C ABI vs the fp64 oracle on the same seeded inputs.

Covers what the group-size sweep in test_gpu_decode.py does not reach:
many pieces per CTA (the double-buffered query rows in tensor memory cycle
through several phases), shares that start mid-segment, a score that jumps mid-sequence (the
running maximum moves and O is rescaled in tensor memory), a negative scale,
two softmax warps with a partly filled second warp (H/G = 48), and sequences
longer than the short-sequence P_hi + P_lo threshold of 256 positions.
"""
import pytest
import torch

import gqa_inputs as gi
import oracle
from parity import assert_close

pytestmark = pytest.mark.gpu


def run_decode(gqa, x, window=0):
    q, k, v = x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda()
    sl = x.seqlens.to(torch.int32).cuda()
    out = gqa.decode(q, k, v, sl, x.scale, window=window)
    gqa.get_status()
    return out.cpu()


def check(gqa, x, window=0):
    got = run_decode(gqa, x, window)
    ref = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, window=window)
    assert_close(got, ref, torch.bfloat16)
    return got


@pytest.mark.parametrize("H,G", [(32, 1), (32, 2), (48, 1), (64, 2)])
def test_many_short_pieces_per_cta(gqa, H, G):
    """40 sequences of 1..700 positions: most CTAs hold several segments."""
    x = gi.decode_inputs(40, H, G, 128, 700, torch.bfloat16, seed=700 + H + G, ragged=(1, 700))
    check(gqa, x)


@pytest.mark.parametrize("ctas", [1, 2, 5, 33, 1000])
def test_forced_split_counts(gqa, monkeypatch, ctas):
    """One CTA walks every segment (eight query-tile loads); more CTAs than tiles."""
    monkeypatch.setenv("GQA_DECODE_CTAS", str(ctas))
    x = gi.decode_inputs(6, 32, 2, 128, 600, torch.bfloat16, seed=710,
                         seqlens=[600, 1, 0, 257, 64, 130])
    check(gqa, x)


@pytest.mark.parametrize("d_h", [64, 128])
def test_score_jump_rescales_output(gqa, d_h):
    """Position 900 of sequence 0 is planted with K = 4 q[head 5]: head 5's
    score there is far above everything before it, so its running maximum
    moves by more than the lazy threshold after many tiles; other heads keep
    theirs.  Sequence 1 gets the jump at its last position."""
    x = gi.decode_inputs(2, 32, 1, d_h, 1500, torch.bfloat16, seed=720, seqlens=[1500, 1201])
    x.k_cache[0, 0, 900] = (4.0 * x.q[0, 5].float()).to(torch.bfloat16)
    x.k_cache[1, 0, 1200] = (4.0 * x.q[1, 7].float()).to(torch.bfloat16)
    got = check(gqa, x)
    # the planted position dominates head 5: its output is close to V[900]
    assert torch.allclose(got[0, 5].float(), x.v_cache[0, 0, 900].float(), atol=0.05)


def test_negative_scale(gqa):
    x = gi.decode_inputs(3, 32, 1, 128, 500, torch.bfloat16, seed=730, seqlens=[500, 77, 300],
                         scale=-0.125)
    check(gqa, x)


def test_long_sequences_past_split_threshold(gqa):
    """Lengths on both sides of 256 and tile boundaries, NaN padding after them."""
    x = gi.decode_inputs(8, 32, 2, 128, 2000, torch.bfloat16, seed=740,
                         seqlens=[256, 257, 2000, 1023, 1024, 1025, 63, 1999])
    check(gqa, x)


@pytest.mark.parametrize("W", [1, 100, 256, 1000])
def test_window(gqa, W):
    x = gi.decode_inputs(5, 32, 1, 128, 1500, torch.bfloat16, seed=750 + W,
                         seqlens=[1500, 20, 999, 1000, 1])
    check(gqa, x, window=W)


def test_mqa_equals_per_head_mha(gqa):
    """G = 1 (MQA) against MHA on the one K/V head repeated H times: the
    tensor-core path against the warp-MMA path on the same data."""
    x = gi.decode_inputs(3, 32, 1, 128, 800, torch.bfloat16, seed=760, seqlens=[800, 300, 45])
    got = run_decode(gqa, x)
    xr = gi.DecodeInputs(x.q, x.k_cache.repeat_interleave(32, dim=1).contiguous(),
                         x.v_cache.repeat_interleave(32, dim=1).contiguous(), x.seqlens,
                         x.scale, 3, 32, 32, 128, 800)
    mha = run_decode(gqa, xr)
    ref = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    assert_close(got, ref, torch.bfloat16)
    assert_close(mha, ref, torch.bfloat16)


@pytest.mark.parametrize("B", [2000, 2400])
def test_large_batches_near_the_shared_memory_bound(gqa, B):
    """The per-sequence prefix lives in shared memory next to the ring: B = 2000
    still fits the tensor-core kernel, B = 2400 takes the warp-MMA kernel."""
    x = gi.decode_inputs(B, 16, 1, 128, 40, torch.bfloat16, seed=770 + B, ragged=(0, 40))
    check(gqa, x)


def test_one_workspace_alternating_shapes(gqa):
    """Completion flags left in a workspace by one call never satisfy the next:
    two shapes (the tensor-core and the warp-MMA split kernel) take turns on
    one buffer, each call checked against the oracle."""
    xa = gi.decode_inputs(3, 32, 1, 128, 700, torch.bfloat16, seed=780, seqlens=[700, 5, 333])
    xb = gi.decode_inputs(4, 16, 4, 128, 500, torch.bfloat16, seed=781, seqlens=[1, 500, 64, 0])
    refs = [oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale) for x in (xa, xb)]
    dev = [(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.to(torch.int32).cuda(), x.scale)
           for x in (xa, xb)]
    need = max(gqa.decode_workspace_bytes(3, 32, 1, 128, 700), gqa.decode_workspace_bytes(4, 16, 4, 128, 500))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    for i in range(6):
        q, k, v, sl, scale = dev[i % 2]
        got = gqa.decode(q, k, v, sl, scale, workspace=ws)
        gqa.get_status()
        assert_close(got.cpu(), refs[i % 2], torch.bfloat16)


def test_deterministic_across_streams(gqa):
    """Every merge (slices of a piece, pieces of a segment) runs in a fixed
    order, so repeated calls give the same bits, whatever the timing."""
    x = gi.decode_inputs(5, 32, 1, 128, 3000, torch.bfloat16, seed=790, ragged=(1, 3000))
    q, k, v = x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda()
    sl = x.seqlens.to(torch.int32).cuda()
    first = gqa.decode(q, k, v, sl, x.scale).clone()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        outs = [gqa.decode(q, k, v, sl, x.scale, stream=s) for _ in range(3)]
    s.synchronize()
    gqa.get_status()
    for o in outs:
        assert torch.equal(o, first)
