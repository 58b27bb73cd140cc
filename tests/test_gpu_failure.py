"""Failure detection on the GPU without faulting or hanging it, and guard bands.

* A bounded wait that runs out (a barrier nothing arrives at) is reported as
  GQA_ERR_TIMEOUT by gqa_get_status, and the context stays usable: a decode
  right after it is still correct.
* Outputs written into the middle of sentinel-filled buffers leave every
  byte around them untouched (no out-of-range writes).
"""
import ctypes

import pytest
import torch

import gqa_inputs as gi
import oracle
from parity import assert_close

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_context_survives(gqa):
    gqa.get_status()  # start clean
    waited = torch.zeros(1, dtype=torch.int32, device="cuda")
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert gqa.lib.gqa_selftest_wait_timeout(50_000_000, waited.data_ptr(), s) == 0
    with pytest.raises(gqa.GQAError) as ei:
        gqa.get_status()
    assert ei.value.code == -6
    assert int(waited.item()) == 1
    gqa.get_status()  # the flag was cleared
    x = gi.decode_inputs(2, 8, 2, 64, 100, torch.bfloat16, seed=900, seqlens=[100, 37])
    out = gqa.decode(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.cuda(), x.scale)
    gqa.get_status()
    assert_close(out.cpu(), oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale),
                 torch.bfloat16)


def _guarded(shape, dtype, pad=4096):
    n = 1
    for v in shape:
        n *= v
    buf = torch.full((pad + n + pad,), -12345.0, dtype=torch.float32, device="cuda").to(dtype)
    return buf, buf[pad:pad + n].view(shape), pad


def _guards_intact(buf, pad, n):
    sentinel = torch.tensor(-12345.0).to(buf.dtype).item()
    return bool((buf[:pad] == sentinel).all()) and bool((buf[pad + n:] == sentinel).all())


def test_outputs_stay_inside_their_buffers(gqa):
    x = gi.decode_inputs(3, 16, 4, 128, 200, torch.bfloat16, seed=901, seqlens=[200, 0, 77])
    buf, out, pad = _guarded((3, 16, 128), torch.bfloat16)
    gqa.decode(x.q.cuda(), x.k_cache.cuda(), x.v_cache.cuda(), x.seqlens.cuda(), x.scale, out=out)
    gqa.get_status()
    assert _guards_intact(buf, pad, out.numel())
    p = gi.prefill_inputs(1, 200, 4, 2, 128, torch.bfloat16, seed=902)
    buf, out, pad = _guarded((1, 200, 4, 128), torch.bfloat16)
    gqa.prefill_causal(p.q.cuda(), p.k.cuda(), p.v.cuda(), p.scale, out=out)
    gqa.get_status()
    assert _guards_intact(buf, pad, out.numel())
    wk, wv = gi.meanpool_inputs(8, 4, 24, seed=903)
    bk, ok, pad = _guarded((2, 4, 24), torch.bfloat16)
    bv, ov, _ = _guarded((2, 4, 24), torch.bfloat16)
    gqa.meanpool_kv(wk.cuda(), wv.cuda(), 2, out_k=ok, out_v=ov)
    gqa.get_status()
    assert _guards_intact(bk, pad, ok.numel()) and _guards_intact(bv, pad, ov.numel())
