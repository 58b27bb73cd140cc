"""Output projection (gqa_out_project) and the whole-layer decode step
(gqa_layer_decode_step: append, attend, project) vs the fp64 oracle.

The layer stores q and the attention output in bf16 between its steps, and
the oracle rounds at the same two points (from fp64 values instead of fp32
ones).  Where the two sides land one bf16 step apart on an intermediate, the
step carries through W_O; such flips are rare (the fp32 and fp64 values differ
by ~1e-7 relative against a 2^-8 step) and of random sign, so their carry is
far below the tolerance and no allowance is added: the layer is held to the
same bound as the kernels it is made of, the strict normwise form at the
benchmark shape.  A negative control checks that this bound is tight enough
to catch a wrong layer: against an oracle layer whose W_O has two heads'
blocks of rows swapped (a head-order mistake, planted on the host side), the
same GPU output must fail it.
"""
import pytest
import torch

import gqa_inputs as gi
import oracle
from parity import assert_close, assert_strict, errors

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,K,N", [(1, 128, 64), (16, 4096, 4096), (33, 256, 192), (20, 512, 640),
                                   (16, 4096, 1024)])
@pytest.mark.parametrize("kernel", ["default", "column", "split"])
def test_out_project(gqa, monkeypatch, B, K, N, kernel):
    """Both projection kernels (GQA_PROJ_KERNEL forces one), and the default
    choice with a workspace: split-K for few column blocks (N = 64, 192, 640,
    1024 on 148 SMs), column blocks for N = 4096."""
    if kernel == "default":
        monkeypatch.delenv("GQA_PROJ_KERNEL", raising=False)
    else:
        monkeypatch.setenv("GQA_PROJ_KERNEL", kernel)
    gen = torch.Generator().manual_seed(B + K + N)
    x = torch.randn(B, K, generator=gen).to(torch.bfloat16)
    W = (torch.randn(K, N, generator=gen) * K ** -0.5).to(torch.bfloat16)
    ws = None
    if kernel != "column":
        ws = torch.empty(gqa.project_workspace_bytes(N, K), dtype=torch.uint8, device="cuda")
    out = gqa.out_project(x.cuda(), W.cuda(), workspace=ws)
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
    # short caches give O(1) outputs, where bf16 storage alone exceeds 2e-3:
    # the per-element form |d| <= 2e-3 + 1e-2 |ref|
    assert_close(out.cpu(), ref, torch.bfloat16)


def _swap_head_blocks(W_O, d_h, a, b):
    w = W_O.clone()
    w[a * d_h:(a + 1) * d_h], w[b * d_h:(b + 1) * d_h] = W_O[b * d_h:(b + 1) * d_h], W_O[a * d_h:(a + 1) * d_h]
    return w


def test_layer_decode_step_llama2_7b(gqa):
    """B=16, d=4096, H=32, G=8, d_h=128, T_cap=4096, one free slot per sequence:
    strict bound (max abs <= 2e-3 and max abs / max |ref| <= 1e-2) on every
    output, and the negative control."""
    x = gi.workload_inputs("qkv_append_llama2_7b")
    gen = torch.Generator().manual_seed(8)
    W_O = (torch.randn(4096, 4096, generator=gen) * 4096 ** -0.5).to(torch.bfloat16)
    out, sl = gqa.layer_decode_step(x.h.cuda(), x.W_Q.cuda(), x.W_K.cuda(), x.W_V.cuda(), W_O.cuda(),
                                    x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.cuda())
    gqa.get_status()
    out = out.cpu()
    ref, rsl = oracle.layer_decode_step(x.h, x.W_Q, x.W_K, x.W_V, W_O, x.k_cache, x.v_cache,
                                        x.seqlens, 128 ** -0.5)
    assert torch.equal(sl.cpu(), rsl)
    assert_strict(out, ref, torch.bfloat16)
    # negative control: the oracle layer with heads 0 and 1 of W_O swapped
    bad, _ = oracle.layer_decode_step(x.h, x.W_Q, x.W_K, x.W_V, _swap_head_blocks(W_O, 128, 0, 1),
                                      x.k_cache, x.v_cache, x.seqlens, 128 ** -0.5)
    with pytest.raises(AssertionError):
        assert_strict(out, bad, torch.bfloat16)
    maxabs, normrel = errors(out, bad)
    assert normrel > 2e-2, (maxabs, normrel)  # fails by a wide margin, not at the edge
