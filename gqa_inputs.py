"""Seeded synthetic inputs for the GQA decode / prefill / mean-pool workloads.

Both the fp64 oracle and the CUDA path are fed from here; this module holds no
attention arithmetic.  Every tensor comes from one CPU ``torch.Generator``
(default seed 0) in a fixed draw order: q, K, V, then seqlens (ragged decode);
W_K, W_V for the mean-pool.  Values are ``torch.randn`` in float32 times sigma,
then rounded to nearest-even into the storage dtype.  Cache positions at or
past ``seqlens[b]`` are filled with NaN so that a kernel reading them shows up.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

# Workloads, named by what they are (all sizes as stated for each).
WORKLOADS = {
    "tiny_decode_fp32": dict(kind="decode", B=1, H=8, G=2, d_h=64, T=128,
                             dtype=torch.float32, ragged=None),
    "llama2_7b_decode": dict(kind="decode", B=16, H=32, G=8, d_h=128, T=4096,
                             dtype=torch.bfloat16, ragged=None),
    "llama2_70b_ragged_decode": dict(kind="decode", B=32, H=64, G=8, d_h=128, T=8192,
                                     dtype=torch.bfloat16, ragged=(1024, 8192)),
    **{"long_ctx_decode_G%d" % g: dict(kind="decode", B=4, H=32, G=g, d_h=128, T=131072,
                                       dtype=torch.bfloat16, ragged=None)
       for g in (1, 2, 4, 8, 16, 32)},
    "causal_prefill": dict(kind="prefill", B=2, S=8192, H=64, G=8, d_h=128,
                           dtype=torch.bfloat16),
    "meanpool_init": dict(kind="meanpool", H=64, G=8, d_h=128, d=8192,
                          dtype=torch.bfloat16, std=0.02),
    # sliding-window variants (4096-key window)
    "causal_prefill_window4096": dict(kind="prefill", B=2, S=8192, H=64, G=8, d_h=128,
                                      dtype=torch.bfloat16, window=4096),
    "llama2_70b_ragged_decode_window4096": dict(kind="decode", B=32, H=64, G=8, d_h=128, T=8192,
                                                dtype=torch.bfloat16, ragged=(1024, 8192),
                                                window=4096),
    # one decode token's projections + cache append, Llama-2-7B shape (d = 4096)
    "qkv_append_llama2_7b": dict(kind="qkv", B=16, d=4096, H=32, G=8, d_h=128, T=4096,
                                 dtype=torch.bfloat16),
    # one decode step of the whole attention layer (append, attend, W_O), same shape
    "layer_decode_llama2_7b": dict(kind="layer", B=16, d=4096, H=32, G=8, d_h=128, T=4096,
                                   dtype=torch.bfloat16),
    # half-length prefill (150 MB of q/k/v/out, above the 126 MB L2) for profiler captures
    "causal_prefill_profile": dict(kind="prefill", B=1, S=4096, H=64, G=8, d_h=128,
                                   dtype=torch.bfloat16),
}

_CHUNK = 1 << 24  # draw at most this many normals at a time


def _randn(shape, gen, dtype, std=1.0):
    """randn in float32 (chunked, in draw order), scaled, rounded to dtype."""
    out = torch.empty(shape, dtype=dtype, device=gen.device)
    flat = out.view(-1)
    n = flat.numel()
    pos = 0
    while pos < n:
        m = min(_CHUNK, n - pos)
        x = torch.randn(m, generator=gen, dtype=torch.float32, device=gen.device)
        if std != 1.0:
            x.mul_(std)
        flat[pos:pos + m] = x.to(dtype)
        pos += m
    return out


@dataclass
class DecodeInputs:
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    seqlens: torch.Tensor
    scale: float
    B: int
    H: int
    G: int
    d_h: int
    T_cap: int


def decode_inputs(B, H, G, d_h, T_cap, dtype=torch.bfloat16, seed=0, ragged=None,
                  seqlens=None, nan_pad=True, scale=None, std=1.0, device="cpu"):
    """q [B,H,d_h], K/V [B,G,T_cap,d_h], seqlens [B] int32.

    ragged=(lo, hi): seqlens drawn uniform over the integers lo..hi inclusive
    after K and V.  An explicit ``seqlens`` list overrides it.  Otherwise every
    sequence holds T_cap tokens.  device="cuda" draws from torch's CUDA
    generator with the same seed and order (other values than on the CPU, same
    recipe), for inputs too large to draw on the host; seqlens stay on the CPU.
    """
    gen = torch.Generator(device=device).manual_seed(seed)
    q = _randn((B, H, d_h), gen, dtype, std)
    k = _randn((B, G, T_cap, d_h), gen, dtype, std)
    v = _randn((B, G, T_cap, d_h), gen, dtype, std)
    if seqlens is not None:
        sl = torch.as_tensor(seqlens, dtype=torch.int32).reshape(B)
    elif ragged is not None:
        lo, hi = ragged
        sl = torch.randint(lo, hi + 1, (B,), generator=gen, dtype=torch.int64,
                           device=gen.device).to(torch.int32).cpu()
    else:
        sl = torch.full((B,), T_cap, dtype=torch.int32)
    if nan_pad:
        for b in range(B):
            n = int(sl[b])
            if 0 <= n < T_cap:
                k[b, :, n:, :] = float("nan")
                v[b, :, n:, :] = float("nan")
    if scale is None:
        scale = 1.0 / math.sqrt(d_h)
    return DecodeInputs(q, k, v, sl, float(scale), B, H, G, d_h, T_cap)


@dataclass
class PrefillInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    scale: float
    B: int
    S: int
    H: int
    G: int
    d_h: int


def prefill_inputs(B, S, H, G, d_h, dtype=torch.bfloat16, seed=0, std=1.0):
    """q [B,S,H,d_h], k/v [B,S,G,d_h] token-major (CPU tensors); scale 1/sqrt(d_h)."""
    gen = torch.Generator().manual_seed(seed)
    q = _randn((B, S, H, d_h), gen, dtype, std)
    k = _randn((B, S, G, d_h), gen, dtype, std)
    v = _randn((B, S, G, d_h), gen, dtype, std)
    return PrefillInputs(q, k, v, 1.0 / math.sqrt(d_h), B, S, H, G, d_h)


def meanpool_inputs(H, d_h, d, dtype=torch.bfloat16, seed=0, std=0.02):
    """MHA projection weights W_K, W_V [H, d_h, d] (CPU tensors)."""
    gen = torch.Generator().manual_seed(seed)
    wk = _randn((H, d_h, d), gen, dtype, std)
    wv = _randn((H, d_h, d), gen, dtype, std)
    return wk, wv


@dataclass
class QkvInputs:
    h: torch.Tensor
    W_Q: torch.Tensor
    W_K: torch.Tensor
    W_V: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    seqlens: torch.Tensor
    B: int
    d: int
    H: int
    G: int
    d_h: int
    T_cap: int


def qkv_inputs(B, d, H, G, d_h, T_cap, dtype=torch.bfloat16, seed=0, seqlens=None):
    """h [B, d] ~ N(0, 1); W_Q [d, H*d_h], W_K/W_V [d, G*d_h] ~ N(0, d^-1/2) (so the
    projections are O(1)); caches [B, G, T_cap, d_h] ~ N(0, 1); seqlens default
    T_cap - 1 (one free slot).  Draw order: h, W_Q, W_K, W_V, K cache, V cache."""
    gen = torch.Generator().manual_seed(seed)
    h = _randn((B, d), gen, dtype)
    w_std = d ** -0.5
    wq = _randn((d, H * d_h), gen, dtype, w_std)
    wk = _randn((d, G * d_h), gen, dtype, w_std)
    wv = _randn((d, G * d_h), gen, dtype, w_std)
    kc = _randn((B, G, T_cap, d_h), gen, dtype)
    vc = _randn((B, G, T_cap, d_h), gen, dtype)
    if seqlens is None:
        sl = torch.full((B,), T_cap - 1, dtype=torch.int32)
    else:
        sl = torch.as_tensor(seqlens, dtype=torch.int32).reshape(B)
    return QkvInputs(h, wq, wk, wv, kc, vc, sl, B, d, H, G, d_h, T_cap)


def workload_inputs(name, seed=0):
    w = WORKLOADS[name]
    if w["kind"] == "decode":
        return decode_inputs(w["B"], w["H"], w["G"], w["d_h"], w["T"], w["dtype"], seed,
                             ragged=w["ragged"])
    if w["kind"] == "prefill":
        return prefill_inputs(w["B"], w["S"], w["H"], w["G"], w["d_h"], w["dtype"], seed)
    if w["kind"] in ("qkv", "layer"):
        return qkv_inputs(w["B"], w["d"], w["H"], w["G"], w["d_h"], w["T"], w["dtype"], seed)
    return meanpool_inputs(w["H"], w["d_h"], w["d"], w["dtype"], seed, w["std"])
