"""gqa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a plug-in whose host runtime owns the whole device memory
budget, or a serving loop that must not allocate once it runs) cannot give
gqa_decode a workspace; this entry point uses the library's built-in scratch
array instead.  The test calls it through the C ABI, twice in a row on the
same inputs, and checks each output against gqa_decode's (with its own
workspace) within the decode tolerance.  It runs last so that a run stopping at
the first failure has already run every other test, and it passes both alone
in a fresh process and after the rest of the suite.
"""
import ctypes

import pytest
import torch

import gqa_inputs as gi
from parity import assert_close

pytestmark = pytest.mark.gpu


def _call_noalloc(gqa, q, k, v, sl, scale, out):
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    code = gqa.GQA_BF16 if q.dtype == torch.bfloat16 else gqa.GQA_F32
    B, H, d_h = q.shape
    _, G, T_cap, _ = k.shape
    return gqa.lib.gqa_decode_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), sl.data_ptr(),
                                      float(scale), out.data_ptr(), B, H, G, d_h, T_cap, code, s)


@pytest.mark.parametrize("dtype,B,H,G,d_h,T,ragged", [
    (torch.bfloat16, 16, 32, 8, 128, 4096, None),       # 7B-shaped decode step
    (torch.bfloat16, 6, 32, 2, 64, 700, (1, 700)),      # ragged, d_h 64, 16 heads per group
    (torch.float32, 2, 8, 2, 64, 300, (1, 300)),
])
def test_noalloc_matches_gqa_decode_twice(gqa, dtype, B, H, G, d_h, T, ragged):
    x = gi.decode_inputs(B, H, G, d_h, T, dtype, seed=91, ragged=ragged)
    q, k, v = x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda()
    sl = x.seqlens.to(torch.int32).cuda()
    ref = gqa.decode(q, k, v, sl, x.scale)
    gqa.get_status()
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        rc = _call_noalloc(gqa, q, k, v, sl, x.scale, out)
        assert rc == 0, gqa.lib.gqa_last_error_string().decode()
        gqa.get_status()
        assert_close(out.cpu(), ref.cpu().double(), dtype)


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
