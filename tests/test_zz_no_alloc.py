"""gqa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a plug-in whose host runtime owns the whole device memory
budget, or a serving loop that must not allocate once it runs) cannot give
gqa_decode a workspace; this entry point uses the library's built-in scratch
array instead.  The tests call it through the C ABI, twice in a row on the
same inputs, and compare each output with gqa_decode's (with its own
workspace) bit for bit: both run the same kernels with the same split count,
so any difference would be a wrong offset or grid.  Two shapes alternate on
the shared array, and the device memory in use must not change across the
calls (nothing is allocated).  This file runs last so that a run stopping at
the first failure has already run every other test, and it passes both alone
in a fresh process and after the rest of the suite.
"""
import ctypes

import pytest
import torch

import gqa_inputs as gi

pytestmark = pytest.mark.gpu


def _call_noalloc(gqa, q, k, v, sl, scale, out):
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = gqa.GQA_BF16 if q.dtype == torch.bfloat16 else gqa.GQA_F32
    B, H, d_h = q.shape
    _, G, T_cap, _ = k.shape
    return gqa.lib.gqa_decode_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), sl.data_ptr(),
                                      float(scale), out.data_ptr(), B, H, G, d_h, T_cap, code, s)


def _device_bytes_in_use():
    torch.cuda.synchronize()
    free, total = torch.cuda.mem_get_info()
    return total - free, torch.cuda.memory_allocated(), torch.cuda.memory_reserved()


SHAPES = [
    (torch.bfloat16, 16, 32, 8, 128, 4096, None),       # 7B-shaped decode step
    (torch.bfloat16, 6, 32, 2, 64, 700, (1, 700)),      # ragged, d_h 64, 16 heads per group
    (torch.float32, 2, 8, 2, 64, 300, (1, 300)),
]


def _inputs(dtype, B, H, G, d_h, T, ragged, seed):
    x = gi.decode_inputs(B, H, G, d_h, T, dtype, seed=seed, ragged=ragged)
    return x, x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.to(torch.int32).cuda()


@pytest.mark.parametrize("dtype,B,H,G,d_h,T,ragged", SHAPES)
def test_noalloc_matches_gqa_decode_twice(gqa, dtype, B, H, G, d_h, T, ragged):
    x, q, k, v, sl = _inputs(dtype, B, H, G, d_h, T, ragged, seed=91)
    ref = gqa.decode(q, k, v, sl, x.scale)
    gqa.get_status()
    outs = [torch.full_like(q, float("nan")) for _ in range(2)]
    _call_noalloc(gqa, q, k, v, sl, x.scale, torch.empty_like(q))  # first call on the device: set-up
    gqa.get_status()
    before = _device_bytes_in_use()
    for out in outs:
        rc = _call_noalloc(gqa, q, k, v, sl, x.scale, out)
        assert rc == 0, gqa.lib.gqa_last_error_string().decode()
    gqa.get_status()
    assert _device_bytes_in_use() == before, "device memory in use changed across the calls"
    for out in outs:
        assert torch.equal(out, ref)


def test_noalloc_two_shapes_back_to_back(gqa):
    """Calls of two different shapes alternate on the one scratch array, queued
    back to back on one stream without a synchronisation between them."""
    a = _inputs(*SHAPES[0], seed=92)
    b = _inputs(*SHAPES[1], seed=93)
    refs = []
    for x, q, k, v, sl in (a, b):
        refs.append(gqa.decode(q, k, v, sl, x.scale))
    gqa.get_status()
    outs = [torch.full_like((a, b)[i % 2][1], float("nan")) for i in range(4)]
    before = _device_bytes_in_use()
    for i, out in enumerate(outs):
        x, q, k, v, sl = (a, b)[i % 2]
        assert _call_noalloc(gqa, q, k, v, sl, x.scale, out) == 0
    gqa.get_status()
    assert _device_bytes_in_use() == before, "device memory in use changed across the calls"
    for i, out in enumerate(outs):
        assert torch.equal(out, refs[i % 2]), "call %d" % i


def test_noalloc_rejects_shapes_beyond_its_scratch(gqa):
    limit = 8 << 20
    B, H, G, d_h, T = 512, 64, 8, 128, 1024    # ~17 MiB of partial records
    need = gqa.decode_workspace_bytes(B, H, G, d_h, T, torch.bfloat16)
    assert need > limit
    dummy = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    p = dummy.data_ptr()
    rc = gqa.lib.gqa_decode_noalloc(p, p, p, p, 0.1, p, B, H, G, d_h, T, gqa.GQA_BF16,
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == -5
    assert "scratch" in gqa.lib.gqa_last_error_string().decode()
