"""Sliding-window decode and prefill (gqa_decode_window, gqa_prefill_causal_window)
vs the fp64 oracle's windowed forms."""
import pytest
import torch

import gqa_inputs as gi
import oracle
from parity import assert_close, assert_rows, assert_strict, full_rows

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("W", [1, 7, 64, 100, 5000])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_window(gqa, W, dtype):
    x = gi.decode_inputs(6, 16, 4, 128, 300, dtype, seed=700 + W, seqlens=[300, 1, 0, 65, 129, 250])
    out = gqa.decode(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.cuda(), x.scale,
                     window=W)
    gqa.get_status()
    ref = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, window=W)
    assert_close(out.cpu(), ref, dtype)


@pytest.mark.parametrize("ctas", [3, 1000])
def test_decode_window_forced_splits(gqa, monkeypatch, ctas):
    monkeypatch.setenv("GQA_DECODE_CTAS", str(ctas))
    x = gi.decode_inputs(4, 32, 8, 64, 700, torch.bfloat16, seed=710, ragged=(1, 700))
    out = gqa.decode(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.cuda(), x.scale,
                     window=200)
    gqa.get_status()
    ref = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, window=200)
    assert_close(out.cpu(), ref, torch.bfloat16)


@pytest.mark.parametrize("S,W", [(200, 1), (700, 100), (700, 128), (700, 129), (1024, 256),
                                 (1024, 300), (1000, 1000), (640, 4096)])
def test_prefill_window(gqa, S, W):
    x = gi.prefill_inputs(1, S, 8, 2, 128, torch.bfloat16, seed=S + W)
    out = gqa.prefill_causal(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.scale, window=W)
    gqa.get_status()
    ref = oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale, window=W)
    assert_close(out.cpu(), ref, torch.bfloat16)


@pytest.mark.parametrize("S,W,H,G,d_h", [
    (1024, 257, 8, 2, 128),  # one key past the two-term-P threshold (W <= 256)
    (500, 130, 6, 2, 64),    # r = 3 (a lone head per group) at d_h = 64
    (300, 64, 4, 4, 64),     # G = H (MHA) with a window inside one tile
    (777, 200, 10, 2, 128),  # r = 5, ragged S
])
def test_prefill_window_group_sizes_and_head_dims(gqa, S, W, H, G, d_h):
    x = gi.prefill_inputs(1, S, H, G, d_h, torch.bfloat16, seed=S + W + d_h)
    out = gqa.prefill_causal(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.scale, window=W)
    gqa.get_status()
    ref = oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale, window=W)
    assert_close(out.cpu(), ref, torch.bfloat16)


def test_prefill_window_4096_full_workload(gqa):
    """B=2, S=8192, H=64, G=8 with a 4096-key window: every tile edge of one
    (b, head) and 1,024 random rows; strict form on rows below 0.5."""
    x = gi.workload_inputs("causal_prefill")
    out = gqa.prefill_causal(x.q.cuda(), x.k.cuda(), x.v.cuda(), x.scale, window=4096).cpu()
    gqa.get_status()
    S, H = 8192, 64
    picks = full_rows(S, H, seed=12, n_random=1024, b_edge=0, head_edge=9)
    rows = [(b * S + s) * H + i for b, s, i in picks]
    ref = oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale, rows=rows, window=4096)
    n_strict = assert_rows(out.reshape(-1, 128)[rows], ref, torch.bfloat16)
    assert n_strict >= 0.95 * len(rows), n_strict


def test_decode_window_4096_ragged_workload(gqa):
    """B=32, H=64, G=8, T_b in [1024, 8192] with the last 4096 positions attended."""
    x = gi.workload_inputs("llama2_70b_ragged_decode")
    out = gqa.decode(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.cuda(), x.scale,
                     window=4096).cpu()
    gqa.get_status()
    rows = list(range(0, 32 * 64, 7))
    ref = oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, rows=rows, window=4096)
    assert_strict(out.reshape(-1, 128)[rows], ref, torch.bfloat16)
