"""GQA decode through the C ABI vs the fp64 oracle on the same seeded inputs.

Sweeps cover d_h in {64, 128}, group sizes H/G from 1 (MHA) to 64, ragged
lengths (0, 1, tile boundaries 63/64/65, non-multiples), NaN-poisoned cache
padding, split counts from 1 to more CTAs than tiles, fp32 and bf16.  The
benchmark workloads run at full size: every row for the 7B-shaped step,
sampled rows for the 70B-shaped ragged step and the 131072-token G sweep.
"""
import math

import pytest
import torch

import gqa_inputs as gi
import oracle
from parity import assert_close, assert_strict

pytestmark = pytest.mark.gpu


def run_decode(gqa, x, stream=None):
    q, k, v = x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda()
    sl = x.seqlens.to(torch.int32).cuda()
    out = gqa.decode(q, k, v, sl, x.scale, stream=stream)
    gqa.get_status()
    return out.cpu()


def test_tiny_fp32_workload(gqa):
    x = gi.workload_inputs("tiny_decode_fp32")
    assert x.scale == 1.0 / 8.0
    got = run_decode(gqa, x)
    ref = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    assert_strict(got, ref, torch.float32)


@pytest.mark.parametrize("d_h", [64, 128])
@pytest.mark.parametrize("r", [1, 2, 4, 8, 12, 16, 24, 32, 64])
def test_bf16_group_sizes(gqa, d_h, r):
    G = 2
    x = gi.decode_inputs(6, r * G, G, d_h, 200, torch.bfloat16, seed=100 + r,
                         seqlens=[200, 1, 64, 65, 0, 137])
    got = run_decode(gqa, x)
    ref = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    assert_close(got, ref, torch.bfloat16)
    assert torch.equal(got[4], torch.zeros_like(got[4]))  # empty cache row


@pytest.mark.parametrize("d_h", [64, 128])
@pytest.mark.parametrize("r", [1, 3, 8])
def test_f32_sweep(gqa, d_h, r):
    G = 3
    x = gi.decode_inputs(4, r * G, G, d_h, 97, torch.float32, seed=200 + r,
                         seqlens=[97, 1, 33, 64])
    got = run_decode(gqa, x)
    ref = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    assert_close(got, ref, torch.float32)


@pytest.mark.parametrize("ctas", [1, 2, 3, 7, 50, 1000])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_forced_split_counts(gqa, monkeypatch, ctas, dtype):
    """Shares that start mid-segment and span several segments."""
    monkeypatch.setenv("GQA_DECODE_CTAS", str(ctas))
    x = gi.decode_inputs(5, 16, 4, 128, 300, dtype, seed=300, seqlens=[300, 1, 0, 129, 64])
    got = run_decode(gqa, x)
    ref = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    assert_close(got, ref, dtype)


def test_seqlens_out_of_range_are_clamped_and_flagged(gqa):
    x = gi.decode_inputs(3, 8, 2, 64, 100, torch.bfloat16, seed=400, seqlens=[100, 50, 10],
                         nan_pad=False)
    q, k, v = x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda()
    sl = torch.tensor([130, -5, 10], dtype=torch.int32, device="cuda")
    out = gqa.decode(q, k, v, sl, x.scale)
    with pytest.raises(gqa.GQAError) as ei:
        gqa.get_status()
    assert ei.value.code == -7
    gqa.get_status()  # cleared
    ref = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, [100, 0, 10], x.scale)
    assert_close(out.cpu(), ref, torch.bfloat16)


def test_deterministic_and_stream_ordered(gqa):
    x = gi.decode_inputs(4, 32, 8, 128, 1000, torch.bfloat16, seed=500, ragged=(1, 1000))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a = run_decode(gqa, x, stream=s)
        b = run_decode(gqa, x, stream=s)
    assert torch.equal(a, b)


def test_gqa_equals_mha_on_repeated_kv(gqa):
    """The page's broadcast identity, on the GPU: G heads shared by H/G query
    heads gives the MHA result on K/V repeated H/G times."""
    x = gi.decode_inputs(2, 16, 4, 128, 256, torch.bfloat16, seed=600, seqlens=[256, 77])
    got = run_decode(gqa, x)
    xr = gi.DecodeInputs(x.q, x.k_cache.repeat_interleave(4, dim=1).contiguous(),
                         x.v_cache.repeat_interleave(4, dim=1).contiguous(), x.seqlens,
                         x.scale, 2, 16, 16, 128, 256)
    mha = run_decode(gqa, xr)
    ref = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    assert_close(got, ref, torch.bfloat16)
    assert_close(mha, ref, torch.bfloat16)


# ------------------------------------------------------------ full-size workloads

def test_llama2_7b_decode_full(gqa):
    """B=16, H=32, G=8, d_h=128, T=4096, bf16: every output row."""
    x = gi.workload_inputs("llama2_7b_decode")
    got = run_decode(gqa, x)
    ref = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    assert_strict(got, ref, torch.bfloat16)


def test_llama2_70b_ragged_decode_full(gqa):
    """B=32, H=64, G=8, d_h=128, T_b uniform in [1024, 8192], NaN padding."""
    x = gi.workload_inputs("llama2_70b_ragged_decode")
    assert int(x.seqlens.min()) >= 1024 and int(x.seqlens.max()) <= 8192
    got = run_decode(gqa, x)
    assert torch.isfinite(got.float()).all()
    gen = torch.Generator().manual_seed(1)
    rows = sorted(set(torch.randint(0, 32 * 64, (192,), generator=gen).tolist()
                      + [0, 63, 64, 32 * 64 - 1]))
    ref = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, rows=rows)
    assert_strict(got.reshape(-1, 128)[rows], ref, torch.bfloat16)


@pytest.mark.parametrize("G", [1, 2, 4, 8, 16, 32])
def test_long_context_decode_full(gqa, G):
    """B=4, H=32, d_h=128, T=131072: sampled rows of sequences 0 and 3."""
    x = gi.decode_inputs(4, 32, G, 128, 131072, torch.bfloat16, seed=0, device="cuda")
    out = gqa.decode(x.q, x.k_cache, x.v_cache, x.seqlens.cuda(), x.scale)
    gqa.get_status()
    out = out.cpu()
    assert torch.isfinite(out.float()).all()
    r = 32 // G
    for b in (0, 3):
        heads = sorted({h for h in (0, r - 1, r, 31, (7 * b + 5) % 32, (11 * b + 17) % 32)
                        if h < 32})
        kb = x.k_cache[b:b + 1].cpu()
        vb = x.v_cache[b:b + 1].cpu()
        ref = oracle.gqa_decode(x.q[b:b + 1].cpu(), kb, vb, x.seqlens[b:b + 1], x.scale,
                                rows=heads)
        assert_strict(out[b, heads], ref, torch.bfloat16)
        del kb, vb


@pytest.mark.parametrize("H,G", [(32, 8), (32, 1)])
def test_cuda_graph_replay_matches_eager(gqa, H, G):
    """bench.py times decode steps replayed from a CUDA graph: the captured calls
    (programmatic-dependent launches, completion flags from fresh call
    generations at capture time) must give the eager calls' bits on every
    replay, also with other work between replays."""
    x = gi.decode_inputs(6, H, G, 128, 900, torch.bfloat16, seed=800 + G, ragged=(1, 900))
    q, k, v = x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda()
    sl = x.seqlens.to(torch.int32).cuda()
    eager = gqa.decode(q, k, v, sl, x.scale).clone()
    out = torch.empty_like(q)
    ws = torch.empty(gqa.decode_workspace_bytes(6, H, G, 128, 900, q.dtype), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        gqa.decode(q, k, v, sl, x.scale, out=out, workspace=ws)
    torch.cuda.synchronize()
    graph, s = torch.cuda.CUDAGraph(), torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=s):
        for _ in range(3):
            gqa.decode(q, k, v, sl, x.scale, out=out, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    for i in range(4):
        out.zero_()
        gqa.decode(q, k, v, sl, x.scale)  # another call (other workspace) between replays
        graph.replay()
        torch.cuda.synchronize()
        gqa.get_status()
        assert torch.equal(out, eager), "replay %d" % i


@pytest.mark.parametrize("H,G,d_h,dtype", [
    (32, 8, 128, torch.bfloat16),   # warp-MMA split kernel (4 heads per group)
    (32, 1, 128, torch.bfloat16),   # tcgen05 split kernel (32 heads per group)
    (8, 2, 64, torch.float32),      # fp32 split kernel
])
def test_single_call_graph_replay_with_changing_inputs(gqa, H, G, d_h, dtype):
    """One decode call captured in a CUDA graph and replayed once per step, as a
    serving loop does: q and seqlens change in place before every replay, and
    eager calls on the same workspace run between replays.  Each replay must
    give, bit for bit, what an eager call on the same inputs gives.  (Frozen
    kernel arguments must not let a replay accept the partial results its
    previous replay left in the workspace.)"""
    B, T = 6, 900
    x = gi.decode_inputs(B, H, G, d_h, T, dtype, seed=850 + G, nan_pad=False)
    q, k, v = x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda()
    sl = x.seqlens.to(torch.int32).cuda()
    out = torch.empty_like(q)
    ws = torch.empty(gqa.decode_workspace_bytes(B, H, G, d_h, T, dtype), dtype=torch.uint8,
                     device="cuda")
    gqa.decode(q, k, v, sl, x.scale, out=out, workspace=ws)
    torch.cuda.synchronize()
    graph, s = torch.cuda.CUDAGraph(), torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=s):
        gqa.decode(q, k, v, sl, x.scale, out=out, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    gen = torch.Generator().manual_seed(851)
    for i in range(8):
        q.copy_(torch.randn(q.shape, generator=gen).to(dtype))
        lens = torch.randint(0, T + 1, (B,), generator=gen, dtype=torch.int32)
        if i % 3 == 0:
            lens[0] = 0
        sl.copy_(lens)
        graph.replay()
        got = out.clone()
        ref = gqa.decode(q, k, v, sl, x.scale)  # its own workspace
        if i % 2:  # an eager call on the graph's workspace between replays
            other = gqa.decode(q, k, v, sl, x.scale * 0.5, workspace=ws)
            ref2 = gqa.decode(q, k, v, sl, x.scale * 0.5)
            torch.cuda.synchronize()
            assert torch.equal(other, ref2), "eager call on the shared workspace, step %d" % i
        torch.cuda.synchronize()
        gqa.get_status()
        assert torch.equal(got, ref), "replay %d" % i


@pytest.mark.parametrize("fill", ["zeros", "random", "ones"])
def test_workspace_initial_contents_do_not_matter(gqa, fill):
    """The workspace needs no initialisation: fresh zeros, random bytes, or a
    fill whose header words look like flags all give the same bits."""
    x = gi.decode_inputs(4, 32, 8, 128, 500, torch.bfloat16, seed=860, ragged=(1, 500))
    q, k, v = x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda()
    sl = x.seqlens.to(torch.int32).cuda()
    ref = gqa.decode(q, k, v, sl, x.scale)
    n = gqa.decode_workspace_bytes(4, 32, 8, 128, 500, torch.bfloat16)
    if fill == "zeros":
        ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    elif fill == "ones":
        ws = torch.full((n,), 1, dtype=torch.uint8, device="cuda")
    else:
        g = torch.Generator(device="cuda").manual_seed(861)
        ws = torch.randint(0, 256, (n,), generator=g, dtype=torch.uint8, device="cuda")
    for _ in range(3):
        out = gqa.decode(q, k, v, sl, x.scale, workspace=ws)
        gqa.get_status()
        assert torch.equal(out, ref)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_largest_batch(gqa, dtype):
    """B = 8192, the largest batch the calls take: the tile prefix over 8192
    lengths (chunked over the block's threads), shares that cross hundreds of
    sequences, and empty caches among them."""
    gen = torch.Generator().manual_seed(8192)
    seqlens = torch.randint(0, 17, (8192,), generator=gen).tolist()
    x = gi.decode_inputs(8192, 8, 2, 64, 16, dtype, seed=8192, seqlens=seqlens)
    got = run_decode(gqa, x)
    ref = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale)
    assert_close(got, ref, dtype)
    empty = [b for b, t in enumerate(seqlens) if t == 0]
    assert empty and torch.equal(got[empty], torch.zeros_like(got[empty]))
