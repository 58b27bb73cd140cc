"""Output projection (gqa_out_project) and the whole-layer decode step
(gqa_layer_decode_step: append, attend, project) vs the fp64 oracle.

The layer stores q and the attention output in bf16 between its steps; the
oracle rounds at the same points, but from fp64 instead of fp32 values, so an
element close to a rounding boundary can end one bf16 step (2^-8 relative)
apart on the two sides.  The layer test therefore allows, on top of the bf16
tolerance, two such steps per attention element carried through W_O:
2 * 2^-8 * (|attn| @ |W_O|).  The steps themselves are tested without it.
"""
import pytest
import torch

import gqa_inputs as gi
import oracle
from parity import assert_close, assert_close_plus

pytestmark = pytest.mark.gpu


def _carry(x, W_O, scale, window):
    """2 * 2^-8 * (|attn| @ |W_O|): two bf16 steps of every attention element carried by W_O."""
    q, k, v, kc, vc, sl, _ = oracle.qkv_append(x.h, x.W_Q, x.W_K, x.W_V, x.k_cache, x.v_cache, x.seqlens)
    st = torch.bfloat16
    attn = oracle.gqa_decode(oracle.round_to(q, st), oracle.round_to(kc, st), oracle.round_to(vc, st),
                             sl, scale, window=window)
    return 2 * 2.0 ** -8 * (attn.abs().reshape(x.B, -1) @ W_O.double().abs())


@pytest.mark.parametrize("B,K,N", [(1, 128, 64), (16, 4096, 4096), (33, 256, 192), (20, 512, 640)])
def test_out_project(gqa, B, K, N):
    gen = torch.Generator().manual_seed(B + K + N)
    x = torch.randn(B, K, generator=gen).to(torch.bfloat16)
    W = (torch.randn(K, N, generator=gen) * K ** -0.5).to(torch.bfloat16)
    out = gqa.out_project(x.cuda(), W.cuda())
    gqa.get_status()
    assert_close(out.cpu(), oracle.project(x, W), torch.bfloat16)


@pytest.mark.parametrize("B,d,H,G,d_h,T,seqlens,window", [
    (3, 256, 4, 2, 64, 40, [0, 17, 39], 0),
    (4, 512, 8, 2, 128, 100, [99, 1, 50, 64], 0),
    (2, 512, 8, 8, 64, 300, [299, 150], 100),
])
def test_layer_decode_step_small(gqa, B, d, H, G, d_h, T, seqlens, window):
    x = gi.qkv_inputs(B, d, H, G, d_h, T, seed=B * d + T, seqlens=seqlens)
    gen = torch.Generator().manual_seed(7)
    W_O = (torch.randn(H * d_h, d, generator=gen) * (H * d_h) ** -0.5).to(torch.bfloat16)
    kc, vc = x.k_cache.cuda(), x.v_cache.cuda()
    out, sl = gqa.layer_decode_step(x.h.cuda(), x.W_Q.cuda(), x.W_K.cuda(), x.W_V.cuda(), W_O.cuda(),
                                    kc, vc, x.seqlens.cuda(), scale=d_h ** -0.5, window=window)
    gqa.get_status()
    ref, rsl = oracle.layer_decode_step(x.h, x.W_Q, x.W_K, x.W_V, W_O, x.k_cache, x.v_cache,
                                        x.seqlens, d_h ** -0.5, window=window)
    assert torch.equal(sl.cpu(), rsl)
    assert_close_plus(out.cpu(), ref, torch.bfloat16, _carry(x, W_O, d_h ** -0.5, window))


def test_layer_decode_step_llama2_7b(gqa):
    """B=16, d=4096, H=32, G=8, d_h=128, T_cap=4096, one free slot per sequence."""
    x = gi.workload_inputs("qkv_append_llama2_7b")
    gen = torch.Generator().manual_seed(8)
    W_O = (torch.randn(4096, 4096, generator=gen) * 4096 ** -0.5).to(torch.bfloat16)
    out, sl = gqa.layer_decode_step(x.h.cuda(), x.W_Q.cuda(), x.W_K.cuda(), x.W_V.cuda(), W_O.cuda(),
                                    x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.cuda())
    gqa.get_status()
    ref, rsl = oracle.layer_decode_step(x.h, x.W_Q, x.W_K, x.W_V, W_O, x.k_cache, x.v_cache,
                                        x.seqlens, 128 ** -0.5)
    assert torch.equal(sl.cpu(), rsl)
    assert_close_plus(out.cpu(), ref, torch.bfloat16, _carry(x, W_O, 128 ** -0.5, 0))
