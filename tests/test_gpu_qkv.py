"""Fused Q/K/V projection + KV-cache append (gqa_qkv_append) vs the oracle.

q and the appended k/v rows are compared with the fp64 oracle (bf16 inputs,
fp32 accumulation, one rounding: the bf16 tolerance); every other cache
position must be bit-identical to its input, and seqlens_out = seqlens + 1
except for full caches, which get no append and flag GQA_ERR_SEQLEN.
"""
import pytest
import torch

import gqa_inputs as gi
import oracle
from parity import assert_close

pytestmark = pytest.mark.gpu


def run_and_check(gqa, x, expect_full=False):
    kc, vc = x.k_cache.cuda(), x.v_cache.cuda()
    q, sl_out = gqa.qkv_append(x.h.cuda(), x.W_Q.cuda(), x.W_K.cuda(), x.W_V.cuda(), kc, vc,
                               x.seqlens.cuda())
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
def test_qkv_append_small(gqa, B, d, H, G, d_h, T, seqlens):
    x = gi.qkv_inputs(B, d, H, G, d_h, T, seed=B + d, seqlens=seqlens)
    run_and_check(gqa, x)


def test_qkv_append_full_cache_is_not_written(gqa):
    x = gi.qkv_inputs(4, 256, 8, 2, 64, 6, seed=3, seqlens=[6, 2, 6, 5])
    run_and_check(gqa, x, expect_full=True)


def test_qkv_append_llama2_7b_full(gqa):
    """B=16, d=4096, H=32, G=8, d_h=128, T_cap=4096 (last free slot)."""
    x = gi.workload_inputs("qkv_append_llama2_7b")
    run_and_check(gqa, x)


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
