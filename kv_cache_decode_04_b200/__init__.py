"""Grouped-query attention (GQA) on NVIDIA B200: Python binding of libgqa.so.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/gqa.h``.  Tensors are torch
CUDA tensors (torch provides device memory and streams); there is no CPU or
library fallback, and importing this module fails loudly when the compiled
library is missing.

Calls (same names as the C ABI, without the ``gqa_`` prefix):

* :func:`decode` -- one decode step over a [B, G, T_cap, d_h] KV cache.
* :func:`prefill_causal` -- causal attention over a whole prompt.
* :func:`meanpool_kv` -- averaging-init of G K/V heads from H MHA heads.
* :func:`kv_cache_bytes` -- KV-cache bytes per token, 2*G*d_h*L*elem_bytes.
* :func:`get_status` -- device-side status of earlier calls.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = ["decode", "decode_noalloc", "decode_workspace_bytes", "prefill_causal", "meanpool_kv",
           "qkv_append", "init_kv_heads", "out_project", "project_workspace_bytes", "layer_decode_step",
           "kv_cache_bytes", "get_status", "GQAError", "LIB_PATH", "lib"]

# GQA_LIB=debug selects libgqa_debug.so: the same kernels with device-side
# index checks compiled in (a failed check sets GQA_ERR_INDEX in the status word).
LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "libgqa_debug.so" if os.environ.get("GQA_LIB") == "debug" else "libgqa.so")

GQA_F32, GQA_BF16 = 0, 1
_ERRORS = {-1: "INVALID", -2: "UNSUPPORTED", -3: "ALIGN", -4: "CUDA", -5: "WORKSPACE",
           -6: "TIMEOUT", -7: "SEQLEN", -8: "INDEX"}

# Every symbol include/gqa.h declares.
EXPORTS = ("gqa_kv_cache_bytes", "gqa_decode_workspace_bytes", "gqa_decode",
           "gqa_decode_window", "gqa_decode_noalloc", "gqa_prefill_causal",
           "gqa_prefill_causal_window", "gqa_meanpool_kv", "gqa_init_kv_heads", "gqa_qkv_append",
           "gqa_out_project", "gqa_project_workspace_bytes", "gqa_layer_decode_workspace_bytes",
           "gqa_layer_decode_step",
           "gqa_selftest_wait_timeout", "gqa_get_status", "gqa_last_error_string", "gqa_version")


class GQAError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__("GQA_ERR_%s (%d): %s" % (_ERRORS.get(code, "?"), code, msg))
        self.code = code


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("%s is not built (expected at %s); run "
                          "`python kv_cache_decode_04_b200/build.py`%s"
                          % (os.path.basename(LIB_PATH), LIB_PATH,
                             " --debug" if "debug" in os.path.basename(LIB_PATH) else ""))
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.gqa_kv_cache_bytes.argtypes = [i32, i32, i32, i32]
    L.gqa_kv_cache_bytes.restype = ctypes.c_uint64
    L.gqa_decode_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32]
    L.gqa_decode_workspace_bytes.restype = sz
    L.gqa_decode.argtypes = [vp, vp, vp, vp, f32, vp, i32, i32, i32, i32, i32, i32, vp, sz, vp]
    L.gqa_decode.restype = i32
    L.gqa_decode_window.argtypes = [vp, vp, vp, vp, f32, vp, i32, i32, i32, i32, i32, i32, i32, vp,
                                    sz, vp]
    L.gqa_decode_window.restype = i32
    L.gqa_prefill_causal_window.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, i32, i32,
                                            vp]
    L.gqa_prefill_causal_window.restype = i32
    L.gqa_decode_noalloc.argtypes = [vp, vp, vp, vp, f32, vp, i32, i32, i32, i32, i32, i32, vp]
    L.gqa_decode_noalloc.restype = i32
    L.gqa_prefill_causal.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, i32, vp]
    L.gqa_prefill_causal.restype = i32
    L.gqa_meanpool_kv.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp]
    L.gqa_meanpool_kv.restype = i32
    L.gqa_qkv_append.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32,
                                 i32, vp, sz, vp]
    L.gqa_qkv_append.restype = i32
    L.gqa_init_kv_heads.argtypes = [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, i32, i32, vp]
    L.gqa_init_kv_heads.restype = i32
    L.gqa_out_project.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, sz, vp]
    L.gqa_out_project.restype = i32
    L.gqa_project_workspace_bytes.argtypes = [i32, i32]
    L.gqa_project_workspace_bytes.restype = sz
    L.gqa_layer_decode_workspace_bytes.argtypes = [i32, i32, i32, i32, i32, i32, i32]
    L.gqa_layer_decode_workspace_bytes.restype = sz
    L.gqa_layer_decode_step.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, f32, i32, vp, i32, i32,
                                        i32, i32, i32, i32, i32, vp, sz, vp]
    L.gqa_layer_decode_step.restype = i32
    L.gqa_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp, vp]
    L.gqa_selftest_wait_timeout.restype = i32
    L.gqa_get_status.argtypes = [vp]
    L.gqa_get_status.restype = i32
    L.gqa_last_error_string.argtypes = []
    L.gqa_last_error_string.restype = ctypes.c_char_p
    L.gqa_version.restype = i32
    return L


lib = _load()


def _check(rc):
    if rc != 0:
        raise GQAError(rc, lib.gqa_last_error_string().decode())


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return GQA_BF16
    if t.dtype == torch.float32:
        return GQA_F32
    raise TypeError("GQA tensors must be bfloat16 or float32, got %s" % t.dtype)


def _dev(t, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t.data_ptr()


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def kv_cache_bytes(G: int, d_h: int, L: int, elem_bytes: int) -> int:
    """KV-cache bytes per token: 2 * G * d_h * L * elem_bytes."""
    return int(lib.gqa_kv_cache_bytes(G, d_h, L, elem_bytes))


def decode_workspace_bytes(B, H, G, d_h, T_cap, dtype=torch.bfloat16) -> int:
    code = GQA_BF16 if dtype == torch.bfloat16 else GQA_F32
    n = int(lib.gqa_decode_workspace_bytes(B, H, G, d_h, T_cap, code))
    if n == 0:
        raise GQAError(-1, "invalid decode shape or device: " + lib.gqa_last_error_string().decode())
    return n


def decode(q, k_cache, v_cache, seqlens, scale=None, out=None, workspace=None, stream=None,
           window=0):
    """GQA decode: out[b,i] = softmax(scale q[b,i].K[b,g]^T over t < seqlens[b]) V[b,g].

    q [B,H,d_h]; k_cache, v_cache [B,G,T_cap,d_h]; seqlens [B] int32 (device);
    scale defaults to 1/sqrt(d_h).  window > 0 attends over the last
    ``window`` cached positions only.  Returns ``out`` [B,H,d_h].
    """
    B, H, d_h = q.shape
    Bk, G, T_cap, dk = k_cache.shape
    if Bk != B or dk != d_h or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch between q, k_cache and v_cache")
    if q.dtype != k_cache.dtype or q.dtype != v_cache.dtype:
        raise TypeError("q, k_cache and v_cache must share a dtype")
    if seqlens.dtype != torch.int32 or seqlens.numel() != B:
        raise ValueError("seqlens must be int32 [B]")
    code = _dtype_code(q)
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:  # (a given workspace's size is checked by the library)
        need = decode_workspace_bytes(B, H, G, d_h, T_cap, q.dtype)
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    rc = lib.gqa_decode_window(_dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                               _dev(seqlens, "seqlens"), float(scale), _dev(out, "out"), B, H, G,
                               d_h, T_cap, int(window), code, _dev(workspace, "workspace"),
                               workspace.numel(), _stream(stream))
    _check(rc)
    return out


def decode_noalloc(q, k_cache, v_cache, seqlens, scale=None, out=None, stream=None):
    """Same as :func:`decode`, with the library's built-in scratch instead of a workspace.

    For callers that cannot allocate device memory; see gqa_decode_noalloc in
    include/gqa.h for the size limit and the sharing rules of that scratch.
    """
    B, H, d_h = q.shape
    Bk, G, T_cap, dk = k_cache.shape
    if Bk != B or dk != d_h or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch between q, k_cache and v_cache")
    if q.dtype != k_cache.dtype or q.dtype != v_cache.dtype:
        raise TypeError("q, k_cache and v_cache must share a dtype")
    if seqlens.dtype != torch.int32 or seqlens.numel() != B:
        raise ValueError("seqlens must be int32 [B]")
    code = _dtype_code(q)
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    if out is None:
        out = torch.empty_like(q)
    rc = lib.gqa_decode_noalloc(_dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                                _dev(seqlens, "seqlens"), float(scale), _dev(out, "out"), B, H, G,
                                d_h, T_cap, code, _stream(stream))
    _check(rc)
    return out


def prefill_causal(q, k, v, scale=None, out=None, stream=None, window=0):
    """Causal GQA prefill: q [B,S,H,d_h], k/v [B,S,G,d_h] bf16 -> out [B,S,H,d_h].

    window > 0: query s sees keys s-window < t <= s only.
    """
    B, S, H, d_h = q.shape
    G = k.shape[2]
    if tuple(k.shape) != (B, S, G, d_h) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("shape mismatch between q, k and v")
    code = _dtype_code(q)
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    if out is None:
        out = torch.empty_like(q)
    rc = lib.gqa_prefill_causal_window(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"),
                                       B, S, H, G, d_h, float(scale), int(window), code,
                                       _stream(stream))
    _check(rc)
    return out


def meanpool_kv(wk, wv, G, out_k=None, out_v=None, stream=None):
    """Averaging init: [H,d_h,d] MHA K/V projections -> [G,d_h,d] group means."""
    H, d_h, d = wk.shape
    if tuple(wv.shape) != tuple(wk.shape) or wk.dtype != wv.dtype:
        raise ValueError("WK and WV must have the same shape and dtype")
    code = _dtype_code(wk)
    if out_k is None:
        out_k = torch.empty((G, d_h, d), dtype=wk.dtype, device=wk.device)
    if out_v is None:
        out_v = torch.empty((G, d_h, d), dtype=wk.dtype, device=wk.device)
    rc = lib.gqa_meanpool_kv(_dev(wk, "WK"), _dev(wv, "WV"), _dev(out_k, "WK_out"),
                             _dev(out_v, "WV_out"), H, int(G), d_h, d, code, _stream(stream))
    _check(rc)
    return out_k, out_v


GQA_INIT_MEAN, GQA_INIT_SELECT, GQA_INIT_WEIGHTED = 0, 1, 2


def init_kv_heads(wk, wv, G, mode="mean", head_weights=None, select=0, out_k=None, out_v=None,
                  stream=None):
    """G K/V heads from H MHA heads: mode "mean" (= meanpool_kv), "select" (head
    `select` of each group) or "weighted" (head_weights [2, H] device float32:
    K's weights then V's)."""
    H, d_h, d = wk.shape
    if tuple(wv.shape) != tuple(wk.shape) or wk.dtype != wv.dtype:
        raise ValueError("WK and WV must have the same shape and dtype")
    m = {"mean": GQA_INIT_MEAN, "select": GQA_INIT_SELECT, "weighted": GQA_INIT_WEIGHTED}[mode]
    code = _dtype_code(wk)
    if out_k is None:
        out_k = torch.empty((G, d_h, d), dtype=wk.dtype, device=wk.device)
    if out_v is None:
        out_v = torch.empty((G, d_h, d), dtype=wk.dtype, device=wk.device)
    wp = None
    if head_weights is not None:
        if head_weights.dtype != torch.float32 or head_weights.numel() != 2 * H:
            raise ValueError("head_weights must be float32 [2, H]")
        wp = _dev(head_weights, "head_weights")
    rc = lib.gqa_init_kv_heads(_dev(wk, "WK"), _dev(wv, "WV"), _dev(out_k, "WK_out"),
                               _dev(out_v, "WV_out"), H, int(G), d_h, d, m, wp, int(select), code,
                               _stream(stream))
    _check(rc)
    return out_k, out_v


def project_workspace_bytes(ncols: int, d: int) -> int:
    """Workspace of the split-K projection kernel: ncols output columns, d rows reduced."""
    n = int(lib.gqa_project_workspace_bytes(int(ncols), int(d)))
    if n == 0:
        raise GQAError(-1, "unsupported projection shape: " + lib.gqa_last_error_string().decode())
    return n


def _ws(workspace):
    if workspace is None:
        return None, 0
    return _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()


def qkv_append(h, W_Q, W_K, W_V, k_cache, v_cache, seqlens, q_out=None, seqlens_out=None,
               stream=None, workspace=None):
    """One decode token: q = h W_Q, and h W_K, h W_V appended to the KV cache.

    h [B, d]; W_Q [d, H*d_h]; W_K, W_V [d, G*d_h]; k_cache, v_cache
    [B, G, T_cap, d_h] (written in place at position seqlens[b]); seqlens [B]
    int32.  Returns (q_out [B, H, d_h], seqlens_out [B] = seqlens + 1).
    workspace (uint8, >= project_workspace_bytes((H + 2G) d_h, d)) selects the
    split-K kernel that spreads the weights over every SM.
    """
    B, d = h.shape
    _, G, T_cap, d_h = k_cache.shape
    H = W_Q.shape[1] // d_h
    if tuple(W_Q.shape) != (d, H * d_h) or tuple(W_K.shape) != (d, G * d_h) or \
            tuple(W_V.shape) != (d, G * d_h) or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("shape mismatch between h, the weights and the caches")
    code = _dtype_code(h)
    if q_out is None:
        q_out = torch.empty((B, H, d_h), dtype=h.dtype, device=h.device)
    if seqlens_out is None:
        seqlens_out = torch.empty_like(seqlens)
    rc = lib.gqa_qkv_append(_dev(h, "h"), _dev(W_Q, "W_Q"), _dev(W_K, "W_K"), _dev(W_V, "W_V"),
                            _dev(q_out, "q_out"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
                            _dev(seqlens, "seqlens"), _dev(seqlens_out, "seqlens_out"), B, d, H, G,
                            d_h, T_cap, code, *_ws(workspace), _stream(stream))
    _check(rc)
    return q_out, seqlens_out


def out_project(x, W, out=None, stream=None, workspace=None):
    """out = x W for x [B, K] (e.g. the concatenated heads [B, H*d_h]) and W [K, N].

    workspace (>= project_workspace_bytes(N, K)) selects the split-K kernel."""
    x2 = x.reshape(x.shape[0], -1)
    B, K = x2.shape
    if W.shape[0] != K:
        raise ValueError("x and W disagree on K")
    N = W.shape[1]
    if out is None:
        out = torch.empty((B, N), dtype=x.dtype, device=x.device)
    _check(lib.gqa_out_project(_dev(x2, "x"), _dev(W, "W"), _dev(out, "out"), B, K, N,
                               _dtype_code(x), *_ws(workspace), _stream(stream)))
    return out


def layer_decode_step(h, W_Q, W_K, W_V, W_O, k_cache, v_cache, seqlens, scale=None, window=0,
                      out=None, seqlens_out=None, workspace=None, stream=None):
    """One decode step of the attention layer: append, attend, project.

    Returns (out [B, d], seqlens_out)."""
    B, d = h.shape
    _, G, T_cap, d_h = k_cache.shape
    H = W_Q.shape[1] // d_h
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    if out is None:
        out = torch.empty((B, d), dtype=h.dtype, device=h.device)
    if seqlens_out is None:
        seqlens_out = torch.empty_like(seqlens)
    code = _dtype_code(h)
    if workspace is None:
        n = int(lib.gqa_layer_decode_workspace_bytes(B, d, H, G, d_h, T_cap, code))
        if n == 0:
            raise GQAError(-1, lib.gqa_last_error_string().decode())
        workspace = torch.empty(n, dtype=torch.uint8, device=h.device)
    rc = lib.gqa_layer_decode_step(_dev(h, "h"), _dev(W_Q, "W_Q"), _dev(W_K, "W_K"), _dev(W_V, "W_V"),
                                   _dev(W_O, "W_O"), _dev(k_cache, "k_cache"),
                                   _dev(v_cache, "v_cache"), _dev(seqlens, "seqlens"),
                                   _dev(seqlens_out, "seqlens_out"), float(scale), int(window),
                                   _dev(out, "out"), B, d, H, G, d_h, T_cap, code,
                                   _dev(workspace, "workspace"), workspace.numel(), _stream(stream))
    _check(rc)
    return out, seqlens_out


def get_status(stream=None):
    """Synchronise the stream and raise GQAError if a kernel flagged a device condition."""
    _check(lib.gqa_get_status(_stream(stream)))
