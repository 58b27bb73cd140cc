"""fp64 CPU oracle for grouped-query attention (GQA).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The CUDA library (``kv_cache_decode_04_b200``) never imports it, and
the two share no code; the only module both sides read is ``gqa_inputs``
(seeded input generators, no attention arithmetic).

The arithmetic lives in ``gqa_oracle.c`` (plain binary64 loops).  This module
only marshals torch/numpy arrays into it.  Sources followed, by page and
section:

* "Grouped-Query Attention" (llm-arch-kb), section 2 "Derivation": group map
  g(i) = ceil(i*G/H) over 1-indexed heads; averaging-init (mean of the heads of
  a group); KV-cache footprint of 2*G*d_h scalars per token per layer.
* same page, section 3 "Reference implementation": scale 1/sqrt(d_h), causal
  mask, softmax over keys, K/V shared by H/G query heads.
* same page, section 1 "Premise": decode reads every cached key and value.

Every function here is pinned by ``tests/test_oracle_*.py`` against values the
pages print, closed forms, invariants and an independent library routine.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gqa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

F64, F32, BF16 = 0, 1, 2

_lib = None


def build(force: bool = False) -> str:
    """Compile gqa_oracle.c into liboracle.so next to it (plain gcc, IEEE)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-D_GNU_SOURCE", "-o", tmp, _SRC,
           "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_long, ctypes.c_double
    lib.oracle_group_of_head.argtypes = [i32, i32, i32]
    lib.oracle_group_of_head.restype = i32
    lib.oracle_kv_cache_bytes.argtypes = [i32, i32, i32, i32]
    lib.oracle_kv_cache_bytes.restype = ctypes.c_uint64
    lib.oracle_default_threads.restype = i32
    lib.oracle_gqa_decode.argtypes = [vp, i32, vp, vp, i32, vp, dbl, vp,
                                      i32, i32, i32, i32, i32, vp, i64, i32, i32]
    lib.oracle_gqa_decode.restype = i32
    lib.oracle_mha_decode.argtypes = [vp, i32, vp, vp, i32, vp, dbl, vp,
                                      i32, i32, i32, i32, i32]
    lib.oracle_mha_decode.restype = i32
    lib.oracle_gqa_prefill_causal.argtypes = [vp, vp, vp, i32, dbl, vp, i32, i32,
                                              i32, i32, i32, vp, i64, i32, i32]
    lib.oracle_gqa_prefill_causal.restype = i32
    lib.oracle_meanpool.argtypes = [vp, i32, i32, i32, ctypes.c_size_t, vp]
    lib.oracle_meanpool.restype = i32
    lib.oracle_init_heads.argtypes = [vp, i32, i32, i32, ctypes.c_size_t, i32, vp, i32, vp]
    lib.oracle_init_heads.restype = i32
    lib.oracle_project.argtypes = [vp, i32, vp, i32, vp, i32, i32, i32]
    lib.oracle_project.restype = i32
    lib.oracle_round_bf16.argtypes = [vp, vp, ctypes.c_size_t]
    lib.oracle_round_bf16.restype = None
    lib.oracle_round_f32.argtypes = [vp, vp, ctypes.c_size_t]
    lib.oracle_round_f32.restype = None
    _lib = lib
    return lib


def default_threads() -> int:
    return int(_load().oracle_default_threads())


# ---------------------------------------------------------------- marshalling

def _as_host(x):
    """Return (contiguous CPU tensor kept alive, pointer, oracle dtype code)."""
    if isinstance(x, np.ndarray):
        x = torch.from_numpy(np.ascontiguousarray(x))
    x = x.detach().to("cpu").contiguous()
    if x.dtype == torch.float64:
        code = F64
    elif x.dtype == torch.float32:
        code = F32
    elif x.dtype == torch.bfloat16:
        code = BF16
    else:
        raise TypeError("oracle takes float64, float32 or bfloat16, got %s" % x.dtype)
    return x, x.data_ptr(), code


def _i32(x):
    t = torch.as_tensor(x).to("cpu", torch.int32).contiguous()
    return t, t.data_ptr()


def _rows(rows, limit):
    if rows is None:
        return None, None, 0
    t = torch.as_tensor(rows, dtype=torch.int64).reshape(-1).contiguous()
    if t.numel() and (int(t.min()) < 0 or int(t.max()) >= limit):
        raise IndexError("row index outside [0, %d)" % limit)
    return t, t.data_ptr(), t.numel()


# ---------------------------------------------------------------- public API

def group_of_head(i: int, H: int, G: int) -> int:
    """0-indexed KV group of 0-indexed query head i (g(i) = ceil(i*G/H), 1-indexed)."""
    return int(_load().oracle_group_of_head(int(i), int(H), int(G)))


def kv_cache_bytes(G: int, d_h: int, L: int, elem_bytes: int) -> int:
    """KV-cache bytes per token: 2 * G * d_h * L * elem_bytes."""
    return int(_load().oracle_kv_cache_bytes(int(G), int(d_h), int(L), int(elem_bytes)))


def gqa_decode(q, k_cache, v_cache, seqlens, scale, rows=None, nthreads=0, window=0):
    """fp64 GQA decode.

    q [B,H,d_h]; k_cache, v_cache [B,G,T_cap,d_h]; seqlens [B] ints.
    window > 0: attend over the last `window` cached positions only.
    Returns float64 [B,H,d_h], or [len(rows), d_h] for rows = flat (b*H + i).
    """
    lib = _load()
    qt, qp, qdt = _as_host(q)
    kt, kp, kdt = _as_host(k_cache)
    vt, vp_, vdt = _as_host(v_cache)
    if kdt != vdt:
        raise TypeError("K and V must share a dtype")
    B, H, d_h = qt.shape
    _, G, T_cap, _ = kt.shape
    st, sp = _i32(seqlens)
    rt, rp, nr = _rows(rows, B * H)
    out = torch.empty((nr, d_h) if rt is not None else (B, H, d_h), dtype=torch.float64)
    rc = lib.oracle_gqa_decode(qp, qdt, kp, vp_, kdt, sp, float(scale), out.data_ptr(),
                               B, H, G, d_h, T_cap, rp, nr, int(nthreads), int(window))
    if rc != 0:
        raise ValueError("oracle_gqa_decode failed (rc=%d)" % rc)
    return out


def mha_decode(q, k_cache, v_cache, seqlens, scale, nthreads=0):
    """fp64 per-head MHA decode: q [B,H,d_h]; K,V [B,H,T_cap,d_h]."""
    lib = _load()
    qt, qp, qdt = _as_host(q)
    kt, kp, kdt = _as_host(k_cache)
    vt, vp_, vdt = _as_host(v_cache)
    B, H, d_h = qt.shape
    T_cap = kt.shape[2]
    if kt.shape[1] != H:
        raise ValueError("MHA needs one K/V head per query head")
    st, sp = _i32(seqlens)
    out = torch.empty((B, H, d_h), dtype=torch.float64)
    rc = lib.oracle_mha_decode(qp, qdt, kp, vp_, kdt, sp, float(scale), out.data_ptr(),
                               B, H, d_h, T_cap, int(nthreads))
    if rc != 0:
        raise ValueError("oracle_mha_decode failed (rc=%d)" % rc)
    return out


def gqa_prefill_causal(q, k, v, scale, rows=None, nthreads=0, window=0):
    """fp64 causal GQA prefill.

    q [B,S,H,d_h]; k, v [B,S,G,d_h] (same dtype).  window > 0: query s sees
    keys s-window < t <= s.  Returns float64 [B,S,H,d_h], or [len(rows), d_h]
    for rows = flat ((b*S + s)*H + i).
    """
    lib = _load()
    qt, qp, qdt = _as_host(q)
    kt, kp, kdt = _as_host(k)
    vt, vp_, vdt = _as_host(v)
    if not (qdt == kdt == vdt):
        raise TypeError("q, k, v must share a dtype")
    B, S, H, d_h = qt.shape
    G = kt.shape[2]
    rt, rp, nr = _rows(rows, B * S * H)
    out = torch.empty((nr, d_h) if rt is not None else (B, S, H, d_h), dtype=torch.float64)
    rc = lib.oracle_gqa_prefill_causal(qp, kp, vp_, qdt, float(scale), out.data_ptr(),
                                       B, S, H, G, d_h, rp, nr, int(nthreads), int(window))
    if rc != 0:
        raise ValueError("oracle_gqa_prefill_causal failed (rc=%d)" % rc)
    return out


def meanpool_mean(W, G):
    """fp64 group means of W [H, ...] -> [G, ...] (ascending-head sum / count)."""
    lib = _load()
    wt, wp, wdt = _as_host(W)
    H = wt.shape[0]
    n = wt[0].numel() if H else 0
    out = torch.empty((G,) + tuple(wt.shape[1:]), dtype=torch.float64)
    rc = lib.oracle_meanpool(wp, wdt, H, int(G), n, out.data_ptr())
    if rc != 0:
        raise ValueError("oracle_meanpool failed (rc=%d)" % rc)
    return out


def round_to(x, dtype):
    """Round a float64 tensor once (nearest-even) to bfloat16 or float32."""
    lib = _load()
    xt = torch.as_tensor(x, dtype=torch.float64).contiguous()
    if dtype == torch.bfloat16:
        bits = torch.empty(xt.shape, dtype=torch.int16)
        lib.oracle_round_bf16(xt.data_ptr(), bits.data_ptr(), xt.numel())
        return bits.view(torch.bfloat16)
    if dtype == torch.float32:
        y = torch.empty(xt.shape, dtype=torch.float32)
        lib.oracle_round_f32(xt.data_ptr(), y.data_ptr(), xt.numel())
        return y
    raise TypeError("round_to supports bfloat16 and float32")


def meanpool(W, G, out_dtype=None):
    """Mean-pool init: group means of W [H,d_h,d] rounded once to out_dtype."""
    mean = meanpool_mean(W, G)
    return round_to(mean, out_dtype or W.dtype)


def project(h, W):
    """fp64 h @ W: h [B, d], W [d, N] -> [B, N] (plain ascending-k sums)."""
    lib = _load()
    ht, hp, hdt = _as_host(h)
    wt, wp, wdt = _as_host(W)
    B, d = ht.shape
    d2, N = wt.shape
    if d != d2:
        raise ValueError("h and W disagree on d")
    out = torch.empty((B, N), dtype=torch.float64)
    lib.oracle_project(hp, hdt, wp, wdt, out.data_ptr(), B, d, N)
    return out


def qkv_append(h, W_Q, W_K, W_V, k_cache, v_cache, seqlens):
    """One decode token's projections and the cache append.

    q = h @ W_Q -> [B, H, d_h]; k = h @ W_K, v = h @ W_V -> [B, G, d_h] (fp64),
    written at position seqlens[b] of each sequence's cache, which then holds
    one more token ("Grouped-Query Attention", section 1: the cache grows by
    one key and one value vector per token, head and layer).  A sequence whose
    cache is full (seqlens[b] >= T_cap) or whose length is negative gets no
    append and keeps its length.

    Returns (q, k, v, k_cache_after, v_cache_after, seqlens_after, appended)
    where the caches after are float64 copies with the new rows in place.
    """
    Bq, d = h.shape
    G, T_cap, d_h = k_cache.shape[1], k_cache.shape[2], k_cache.shape[3]
    H = W_Q.shape[1] // d_h
    q = project(h, W_Q).reshape(Bq, H, d_h)
    k = project(h, W_K).reshape(Bq, G, d_h)
    v = project(h, W_V).reshape(Bq, G, d_h)
    kc = torch.as_tensor(k_cache).detach().cpu().double().clone()
    vc = torch.as_tensor(v_cache).detach().cpu().double().clone()
    sl = torch.as_tensor(seqlens).to(torch.int64).cpu().clone()
    appended = torch.zeros(Bq, dtype=torch.bool)
    for b in range(Bq):
        t = int(sl[b])
        if 0 <= t < T_cap:
            kc[b, :, t, :] = k[b]
            vc[b, :, t, :] = v[b]
            sl[b] = t + 1
            appended[b] = True
    return q, k, v, kc, vc, sl.to(torch.int32), appended


def init_heads(W, G, mode, weights=None, select=0, out_dtype=None):
    """Alternatives to the mean-pool init, rounded once to out_dtype.

    mode "select": head `select` of each group; mode "weighted": sum of the
    group's heads times caller weights [H] (binary64, ascending head order).
    """
    lib = _load()
    wt, wp, wdt = _as_host(W)
    H = wt.shape[0]
    n = wt[0].numel() if H else 0
    out = torch.empty((G,) + tuple(wt.shape[1:]), dtype=torch.float64)
    m = {"select": 1, "weighted": 2}[mode]
    wts = torch.as_tensor(weights if weights is not None else [0.0] * H,
                          dtype=torch.float64).reshape(-1).contiguous()
    if wts.numel() != H:
        raise ValueError("need one weight per head")
    rc = lib.oracle_init_heads(wp, wdt, H, int(G), n, m, wts.data_ptr(), int(select), out.data_ptr())
    if rc != 0:
        raise ValueError("oracle_init_heads failed (rc=%d)" % rc)
    return round_to(out, out_dtype or W.dtype)


def layer_decode_step(h, W_Q, W_K, W_V, W_O, k_cache, v_cache, seqlens, scale, window=0):
    """One decode step of the attention layer ("Grouped-Query Attention",
    section 3's gqa() for one token): project and append (qkv_append), attend
    over the lengths after the append (gqa_decode), then the concatenated heads
    times W_O.  Values stored in bf16 between the steps are rounded to bf16 here
    at the same points: q, the appended k/v rows (the cache is bf16) and the
    attention output.  Returns (out float64 [B, d], seqlens_after)."""
    q, k, v, kc, vc, sl, app = qkv_append(h, W_Q, W_K, W_V, k_cache, v_cache, seqlens)
    st = torch.bfloat16
    qs = round_to(q, st)
    kcs, vcs = round_to(kc, st), round_to(vc, st)
    attn = gqa_decode(qs, kcs, vcs, sl, scale, window=window)
    B, H, d_h = attn.shape
    attn_s = round_to(attn, st).reshape(B, H * d_h)
    return project(attn_s, W_O), sl
