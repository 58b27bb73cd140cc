"""The C-ABI library: it loads, exports what include/gqa.h declares, and
rejects bad arguments on the host before touching a device (no GPU needed)."""
import ctypes
import os
import re

import kv_cache_decode_04_b200 as gqa
import oracle

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "gqa.h")


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"GQA_API\s+[\w\s\*]+?\b(gqa_\w+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(gqa.EXPORTS)


def test_library_exports_every_declared_symbol():
    pkg = os.path.dirname(gqa.LIB_PATH)
    for so in ("libgqa.so", "libgqa_debug.so"):  # release and index-checked builds
        lib = ctypes.CDLL(os.path.join(pkg, so))
        for name in declared_functions():
            assert hasattr(lib, name), (so, name)
        assert lib.gqa_version() == 101


def test_kv_cache_bytes_matches_oracle_and_pages():
    for G, d_h, L, eb in [(64, 128, 80, 2), (8, 128, 80, 2), (1, 128, 80, 2), (8, 64, 32, 4)]:
        assert gqa.kv_cache_bytes(G, d_h, L, eb) == oracle.kv_cache_bytes(G, d_h, L, eb)
    assert gqa.kv_cache_bytes(64, 128, 80, 2) == 2621440
    assert gqa.kv_cache_bytes(8, 128, 80, 2) == 327680
    assert gqa.kv_cache_bytes(0, 128, 80, 2) == 0


def _decode_rc(**kw):
    a = dict(q=16, k=16, v=16, sl=16, scale=0.125, out=16, B=1, H=8, G=2, d_h=64, T=128,
             dt=gqa.GQA_BF16, ws=256, wsb=1 << 20)
    a.update(kw)
    rc = gqa.lib.gqa_decode(a["q"], a["k"], a["v"], a["sl"], a["scale"], a["out"], a["B"],
                            a["H"], a["G"], a["d_h"], a["T"], a["dt"], a["ws"], a["wsb"], None)
    return rc, gqa.lib.gqa_last_error_string().decode()


def test_decode_rejects_bad_arguments_on_host():
    assert _decode_rc(G=3)[0] == -1                       # G does not divide H
    assert _decode_rc(B=0)[0] == -1
    assert _decode_rc(T=0)[0] == -1
    assert _decode_rc(q=None)[0] == -1
    assert _decode_rc(scale=float("nan"))[0] == -1
    assert _decode_rc(d_h=96)[0] == -2                     # not built
    assert _decode_rc(dt=7)[0] == -2
    assert _decode_rc(H=130, G=2)[0] == -2                 # bf16 group of 65 heads
    assert _decode_rc(B=8193)[0] == -2                     # above the largest batch built for
    assert _decode_rc(k=24)[0] == -3                       # misaligned
    rc, msg = _decode_rc(G=3)
    assert "divide" in msg


def test_prefill_and_meanpool_reject_bad_arguments_on_host():
    L = gqa.lib
    assert L.gqa_prefill_causal(16, 16, 16, 16, 1, 8, 8, 3, 128, 0.1, gqa.GQA_BF16, None) == -1
    assert L.gqa_prefill_causal(16, 16, 16, 16, 1, 8, 8, 2, 96, 0.1, gqa.GQA_BF16, None) == -2  # d_h not built
    assert L.gqa_prefill_causal(16, 16, 16, 16, 1, 8, 8, 2, 128, 0.1, gqa.GQA_F32, None) == -2
    assert L.gqa_prefill_causal(16, 16, 16, 16, 1, 0, 8, 2, 128, 0.1, gqa.GQA_BF16, None) == -1
    assert L.gqa_prefill_causal(16, 16, 16, 8, 1, 8, 8, 2, 128, 0.1, gqa.GQA_BF16, None) == -3
    assert L.gqa_meanpool_kv(16, 16, 16, 16, 8, 3, 4, 4, gqa.GQA_BF16, None) == -1
    assert L.gqa_meanpool_kv(None, 16, 16, 16, 8, 2, 4, 4, gqa.GQA_BF16, None) == -1
    # outputs overlapping the inputs
    assert L.gqa_meanpool_kv(1 << 20, 1 << 24, (1 << 20) + 64, 1 << 28, 8, 2, 4, 4,
                             gqa.GQA_BF16, None) == -1


def _qkv_rc(**kw):
    a = dict(h=1 << 20, wq=1 << 21, wk=1 << 22, wv=1 << 23, q=1 << 24, kc=1 << 25, vc=1 << 26,
             sl=1 << 27, slo=1 << 28, B=4, d=256, H=8, G=2, d_h=128, T=16, dt=gqa.GQA_BF16)
    a.update(kw)
    return gqa.lib.gqa_qkv_append(a["h"], a["wq"], a["wk"], a["wv"], a["q"], a["kc"], a["vc"], a["sl"], a["slo"],
                                  a["B"], a["d"], a["H"], a["G"], a["d_h"], a["T"], a["dt"], None, 0, None)


def test_projections_reject_bad_arguments_on_host():
    assert _qkv_rc(G=3) == -1                       # G does not divide H
    assert _qkv_rc(B=0) == -1
    assert _qkv_rc(d=0) == -1
    assert _qkv_rc(T=0) == -1
    assert _qkv_rc(h=None) == -1
    assert _qkv_rc(slo=(1 << 27) + 4) == -1        # seqlens_out overlaps seqlens
    assert _qkv_rc(dt=gqa.GQA_F32) == -2
    assert _qkv_rc(d_h=96) == -2
    assert _qkv_rc(d=200) == -2                     # d not a multiple of 128
    assert _qkv_rc(wq=(1 << 21) + 8) == -3          # weights must be 16-byte aligned
    assert _qkv_rc(G=3) == -1 and "divide" in gqa.lib.gqa_last_error_string().decode()
    L = gqa.lib
    x, w, o = 1 << 20, 1 << 24, 1 << 28
    assert L.gqa_out_project(x, w, o, 0, 256, 128, gqa.GQA_BF16, None, 0, None) == -1
    assert L.gqa_out_project(None, w, o, 4, 256, 128, gqa.GQA_BF16, None, 0, None) == -1
    assert L.gqa_out_project(x, w, o, 4, 256, 128, gqa.GQA_F32, None, 0, None) == -2
    assert L.gqa_out_project(x, w, o, 4, 200, 128, gqa.GQA_BF16, None, 0, None) == -2   # K % 128
    assert L.gqa_out_project(x, w, o, 4, 256, 96, gqa.GQA_BF16, None, 0, None) == -2    # N % 64
    assert L.gqa_out_project(x + 4, w, o, 4, 256, 128, gqa.GQA_BF16, None, 0, None) == -3
    # the layer step needs the post-append lengths
    assert L.gqa_layer_decode_step(x, w, w, w, w, o, o, x, None, 0.1, 0, o, 4, 256, 8, 2, 128, 16,
                                   gqa.GQA_BF16, None, 0, None) == -1
