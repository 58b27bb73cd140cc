"""Fused Q/K/V projection + KV-cache append (gqa_qkv_append) vs the oracle.

q and the appended k/v rows are compared with the fp64 oracle (bf16 inputs,
fp32 accumulation, one rounding: the bf16 tolerance); every other cache
position must be bit-identical to its input, and seqlens_out = seqlens + 1
except for full caches, which get no append and flag GQA_ERR_SEQLEN.

Two kernels can run a projection: the column-block kernel and the split-K
kernel (with a workspace).  GQA_PROJ_KERNEL, read on every call, forces one,
so each test runs both.
"""
import pytest
import torch

import gqa_inputs as gi
import oracle
from parity import assert_close

pytestmark = pytest.mark.gpu


def _workspace(gqa, x):
    n = gqa.project_workspace_bytes((x.H + 2 * x.G) * x.d_h, x.d)
    return torch.empty(n, dtype=torch.uint8, device="cuda")


KERNELS = ["column", "split"]


def run_and_check(gqa, x, expect_full=False, split=False):
    kc, vc = x.k_cache.cuda(), x.v_cache.cuda()
    q, sl_out = gqa.qkv_append(x.h.cuda(), x.W_Q.cuda(), x.W_K.cuda(), x.W_V.cuda(), kc, vc,
                               x.seqlens.cuda(), workspace=_workspace(gqa, x) if split else None)
    if expect_full:
        with pytest.raises(gqa.GQAError) as ei:
            gqa.get_status()
        assert ei.value.code == -7
    else:
        gqa.get_status()
    rq, rk, rv, rkc, rvc, rsl, appended = oracle.qkv_append(x.h, x.W_Q, x.W_K, x.W_V, x.k_cache,
                                                            x.v_cache, x.seqlens)
    assert_close(q.cpu(), rq, torch.bfloat16)
    assert torch.equal(sl_out.cpu(), rsl)
    kc, vc = kc.cpu(), vc.cpu()
    for b in range(x.B):
        t = int(x.seqlens[b])
        touched = torch.zeros(x.T_cap, dtype=torch.bool)
        if appended[b]:
            touched[t] = True
            assert_close(kc[b, :, t], rk[b], torch.bfloat16)
            assert_close(vc[b, :, t], rv[b], torch.bfloat16)
        # every other position is untouched, bit for bit
        assert torch.equal(kc[b][:, ~touched].view(torch.int16), x.k_cache[b][:, ~touched].view(torch.int16))
        assert torch.equal(vc[b][:, ~touched].view(torch.int16), x.v_cache[b][:, ~touched].view(torch.int16))


@pytest.mark.parametrize("B,d,H,G,d_h,T,seqlens", [
    (3, 256, 4, 2, 64, 16, [0, 5, 15]),
    (16, 512, 8, 2, 128, 32, list(range(0, 32, 2))),
    (33, 256, 8, 8, 64, 10, [i % 10 for i in range(33)]),   # two launches, G = H (MHA)
    (5, 128, 32, 1, 128, 4, [3, 0, 1, 2, 3]),                # MQA
])
@pytest.mark.parametrize("kernel", KERNELS)
def test_qkv_append_small(gqa, monkeypatch, B, d, H, G, d_h, T, seqlens, kernel):
    monkeypatch.setenv("GQA_PROJ_KERNEL", kernel)
    x = gi.qkv_inputs(B, d, H, G, d_h, T, seed=B + d, seqlens=seqlens)
    run_and_check(gqa, x, split=kernel == "split")


@pytest.mark.parametrize("kernel", KERNELS)
def test_qkv_append_full_cache_is_not_written(gqa, monkeypatch, kernel):
    monkeypatch.setenv("GQA_PROJ_KERNEL", kernel)
    x = gi.qkv_inputs(4, 256, 8, 2, 64, 6, seed=3, seqlens=[6, 2, 6, 5])
    run_and_check(gqa, x, expect_full=True, split=kernel == "split")


@pytest.mark.parametrize("kernel", KERNELS)
def test_qkv_append_llama2_7b_full(gqa, monkeypatch, kernel):
    """B=16, d=4096, H=32, G=8, d_h=128, T_cap=4096 (last free slot)."""
    monkeypatch.setenv("GQA_PROJ_KERNEL", kernel)
    x = gi.workload_inputs("qkv_append_llama2_7b")
    run_and_check(gqa, x, split=kernel == "split")


def test_split_k_is_deterministic_and_graph_replayable(gqa, monkeypatch):
    """The split-K kernel adds a block's partial sums in slot order whichever CTA
    finishes last, and resets the block counters for the next call: repeated
    calls, and one call captured in a CUDA graph and replayed with h changed in
    place, give the bits of eager calls."""
    # 48 column blocks: each is split over three CTAs on a 148-SM part
    monkeypatch.setenv("GQA_PROJ_KERNEL", "split")
    x = gi.qkv_inputs(16, 4096, 16, 4, 128, 8, seed=21, seqlens=[3] * 16)
    h, wq, wk, wv = x.h.cuda(), x.W_Q.cuda(), x.W_K.cuda(), x.W_V.cuda()
    kc, vc, sl = x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.cuda()
    ws = _workspace(gqa, x)
    q = torch.empty((16, 16, 128), dtype=torch.bfloat16, device="cuda")
    sl_out = torch.empty_like(sl)
    ref = [gqa.qkv_append(h, wq, wk, wv, kc, vc, sl, workspace=ws)[0].clone() for _ in range(3)]
    assert torch.equal(ref[0], ref[1]) and torch.equal(ref[0], ref[2])
    gqa.qkv_append(h, wq, wk, wv, kc, vc, sl, q_out=q, seqlens_out=sl_out, workspace=ws)
    torch.cuda.synchronize()
    graph, s = torch.cuda.CUDAGraph(), torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.graph(graph, stream=s):
        gqa.qkv_append(h, wq, wk, wv, kc, vc, sl, q_out=q, seqlens_out=sl_out, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    gen = torch.Generator().manual_seed(22)
    for i in range(4):
        h.copy_(torch.randn(h.shape, generator=gen).to(torch.bfloat16))
        graph.replay()
        got = q.clone()
        eager_split = gqa.qkv_append(h, wq, wk, wv, kc.clone(), vc.clone(), sl,
                                     workspace=_workspace(gqa, x))[0]
        monkeypatch.setenv("GQA_PROJ_KERNEL", "column")
        eager = gqa.qkv_append(h, wq, wk, wv, kc.clone(), vc.clone(), sl)[0]
        monkeypatch.setenv("GQA_PROJ_KERNEL", "split")
        torch.cuda.synchronize()
        gqa.get_status()
        assert torch.equal(got, eager_split), "replay %d" % i
        assert_close(got.cpu(), eager.cpu().double(), torch.bfloat16)


def test_qkv_then_decode_sees_the_new_token(gqa):
    """After the append, decode over seqlens_out attends over the new key/value."""
    x = gi.qkv_inputs(2, 256, 8, 2, 128, 40, seed=9, seqlens=[10, 39])
    kc, vc = x.k_cache.cuda(), x.v_cache.cuda()
    q, sl_out = gqa.qkv_append(x.h.cuda(), x.W_Q.cuda(), x.W_K.cuda(), x.W_V.cuda(), kc, vc,
                               x.seqlens.cuda())
    out = gqa.decode(q, kc, vc, sl_out, 128 ** -0.5)
    gqa.get_status()
    ref = oracle.gqa_decode(q.cpu(), kc.cpu(), vc.cpu(), sl_out.cpu(), 128 ** -0.5)
    assert_close(out.cpu(), ref, torch.bfloat16)
    assert sl_out.cpu().tolist() == [11, 40]


def test_append_then_decode_chain_across_tile_boundaries(gqa):
    """Twenty append -> decode rounds back to back on one stream, each decode over the
    lengths the append before it has just written (seqlens_out), starting one
    position short of a 64-token tile boundary: every round must see its new token."""
    x = gi.qkv_inputs(2, 256, 8, 2, 128, 160, seed=21, seqlens=[63, 127])
    kc, vc = x.k_cache.cuda(), x.v_cache.cuda()
    h, wq, wk, wv = x.h.cuda(), x.W_Q.cuda(), x.W_K.cuda(), x.W_V.cuda()
    sl = x.seqlens.cuda()
    outs, qs, lens = [], [], []
    for _ in range(20):
        q, sl_out = gqa.qkv_append(h, wq, wk, wv, kc, vc, sl)
        outs.append(gqa.decode(q, kc, vc, sl_out, 128 ** -0.5))
        qs.append(q)
        lens.append(sl_out)
        sl = sl_out
    gqa.get_status()
    kc_c, vc_c = kc.cpu(), vc.cpu()
    for i, (out, q, L) in enumerate(zip(outs, qs, lens)):
        assert L.cpu().tolist() == [64 + i, 128 + i]
        ref = oracle.gqa_decode(q.cpu(), kc_c, vc_c, L.cpu(), 128 ** -0.5)
        assert_close(out.cpu(), ref, torch.bfloat16)
