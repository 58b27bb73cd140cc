#!/usr/bin/env python
"""Benchmark of the GQA hot path on B200: decode, causal prefill, mean-pool init.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl reference] [--no-rows]

Prints ONE JSON line on rank 0.  The headline workload is the Llama-2-7B-shaped
decode step (B=16, H=32, G=8, d_h=128, T=4096, bf16): a step is one
``gqa_decode`` call (split-KV kernel + combine kernel) over freshly
device-resident inputs; ``value`` is achieved HBM bandwidth on the KV-cache
bytes the step must read (2 * sum_b T_b * G * d_h * 2 bytes), summed over all
ranks and divided by the max-over-ranks device time.  The other workloads are
measured the same way and reported under ``rows``.  Each rank runs its own
independent batch (weak scaling); no data crosses ranks.

``--impl reference`` times the fp64 CPU oracle (the only reference this
project has) on a bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import gqa_inputs as gi  # noqa: E402

METRIC = "GQA decode achieved HBM GB/s (% of peak) & attn-tokens/s; prefill TFLOP/s"
HEADLINE = "llama2_7b_decode"
ROW_WORKLOADS = ["tiny_decode_fp32", "llama2_70b_ragged_decode"] + \
    ["long_ctx_decode_G%d" % g for g in (1, 2, 4, 8, 16, 32)] + ["causal_prefill", "meanpool_init",
                                                                "qkv_append_llama2_7b",
                                                                "causal_prefill_window4096",
                                                                "llama2_70b_ragged_decode_window4096",
                                                                "layer_decode_llama2_7b"]

# dram__bytes_read.sum + dram__bytes_write.sum per launch of the dominant
# kernel, in bytes, each from one single-pass ncu capture of that kernel as it
# is now, on the full workload (the ncu summaries give the commands); for the
# layer step, the sum over its four kernels (Q/K/V projection, decode split,
# combine, W_O projection).  A workload missing here has no capture of its
# current kernel, and its traffic is reported as null.
NCU_TRAFFIC = {
    "llama2_7b_decode": 271878400,                     # warp-MMA split kernel
    "llama2_70b_ragged_decode": 658844672,
    "llama2_70b_ragged_decode_window4096": 462055936,
    "long_ctx_decode_G1": 271545088,                   # tcgen05 split kernel
    "long_ctx_decode_G2": 539985664,
    "long_ctx_decode_G4": 1079909120,                  # warp-MMA split kernel from here on
    "long_ctx_decode_G8": 2151690240,
    "long_ctx_decode_G16": 4299057152,
    "long_ctx_decode_G32": 8595744256,
    "causal_prefill": 734912768,
    "causal_prefill_window4096": 559403520,
    "meanpool_init": 274089216,
    "qkv_append_llama2_7b": 50491136,
    "layer_decode_llama2_7b": 357121280,
}

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# The spec figures the targets are stated against (context next to the measured peaks):
# ~8 TB/s of HBM3e and 2.25 PFLOP/s of dense bf16 per B200.
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ dist

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "gloo" if args.impl == "reference" else "nccl"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local) if backend == "nccl" else None)
    elif args.impl != "reference":
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples (every 200 ms) while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                   "-lms", "200"]
            uuid = getattr(torch.cuda.get_device_properties(self.dev), "uuid", None)
            if uuid:
                u = str(uuid)
                cmd += ["-i", u if u.startswith("GPU-") else "GPU-" + u]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


BAD_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


# ------------------------------------------------------------------ workloads

class Decode:
    kind = "decode"
    graphable = True  # a step is a pure function of the resident inputs

    def __init__(self, name, gqa, device="cuda"):
        w = gi.WORKLOADS[name]
        self.name, self.w, self.gqa = name, w, gqa
        big = w["B"] * w["G"] * w["T"] * w["d_h"] * 2 > (1 << 30)
        # multi-GiB caches are drawn on the device (same recipe, torch CUDA generator)
        x = gi.decode_inputs(w["B"], w["H"], w["G"], w["d_h"], w["T"], w["dtype"], seed=0,
                             ragged=w["ragged"], device="cuda" if big else "cpu")
        self.x = x
        self.q, self.k, self.v = x.q.to(device), x.k_cache.to(device), x.v_cache.to(device)
        self.sl = x.seqlens.to(torch.int32).to(device)
        self.out = torch.empty_like(self.q)
        self.ws = torch.empty(gqa.decode_workspace_bytes(x.B, x.H, x.G, x.d_h, x.T_cap, self.q.dtype),
                              dtype=torch.uint8, device=device)
        esz = self.q.element_size()
        self.window = w.get("window", 0)
        T_att = x.seqlens.clamp(0, x.T_cap)
        if self.window:
            T_att = T_att.clamp(max=self.window)
        self.sum_T = int(T_att.sum())                             # positions attended
        self.bytes = 2 * self.sum_T * x.G * x.d_h * esz           # K and V actually read
        self.flops = 4 * self.sum_T * x.H * x.d_h                 # q.k and p.v
        self.launches_per_step = 2
        self.dtype = "bf16" if self.q.dtype == torch.bfloat16 else "f32"

    def step(self, stream=None):
        self.gqa.decode(self.q, self.k, self.v, self.sl, self.x.scale, out=self.out,
                        workspace=self.ws, stream=stream, window=self.window)

    def config(self):
        x = self.x
        return {"workload": self.name, "B": x.B, "H": x.H, "G": x.G, "d_h": x.d_h, "T_cap": x.T_cap,
                "sum_T": self.sum_T, "ragged": self.w["ragged"] is not None, "window": self.window}

    def metric(self, seconds_per_step, n_ranks):
        gbs = n_ranks * self.bytes / seconds_per_step / 1e9
        return {"value": gbs, "unit": "GB/s",
                "attn_tokens_per_s": n_ranks * self.sum_T / seconds_per_step,
                "kv_bytes_per_step": self.bytes}

    def roofline(self, seconds_per_step, peaks, which, long_run=False):
        a = self.bytes / seconds_per_step / 1e9
        return {"bound": "hbm", "achieved": a, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": a / peaks["hbm_gbs"], "peak_source": which + " hbm_gbs",
                "peak_nominal": NOMINAL_PEAKS["hbm_gbs"], "frac_nominal": a / NOMINAL_PEAKS["hbm_gbs"],
                "traffic": NCU_TRAFFIC.get(self.name)}

    # e2e: host (pinned) inputs copied in, result read back, every step
    def e2e_setup(self):
        self.h = [t.cpu().pin_memory() for t in (self.q, self.k, self.v, self.sl)]
        self.h_out = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
        self.h2d = sum(t.numel() * t.element_size() for t in self.h)
        self.d2h = self.h_out.numel() * self.h_out.element_size()

    def e2e_step(self):
        for dst, src in zip((self.q, self.k, self.v, self.sl), self.h):
            dst.copy_(src, non_blocking=True)
        self.step()
        self.h_out.copy_(self.out, non_blocking=True)

    def oracle_sample(self, budget_s):
        """Oracle on whole output rows, enough of them for about budget_s seconds."""
        import oracle
        x = self.x
        rows_total = x.B * x.H
        gen = torch.Generator().manual_seed(7)
        order = torch.randperm(rows_total, generator=gen).tolist()
        k_host = x.k_cache if x.k_cache.device.type == "cpu" else None
        done, t_used, tokens = 0, 0.0, 0
        n = 1
        while done < rows_total and (done == 0 or t_used < budget_s):
            rows = order[done:done + n]
            if k_host is None:   # device-drawn cache: copy the slabs of one sequence
                b = rows[0] // x.H
                rows = [r for r in rows if r // x.H == b]
                kb, vb = x.k_cache[b:b + 1].cpu(), x.v_cache[b:b + 1].cpu()
                t0 = time.perf_counter()
                oracle.gqa_decode(x.q[b:b + 1].cpu(), kb, vb, x.seqlens[b:b + 1], x.scale,
                                  rows=[r % x.H for r in rows], window=self.window)
            else:
                t0 = time.perf_counter()
                oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, rows=rows,
                                  window=self.window)
            t_used += time.perf_counter() - t0
            tokens += sum(min(int(x.seqlens[r // x.H].clamp(0, x.T_cap)), self.window or x.T_cap)
                          for r in rows)
            done += len(rows)
            n = min(2 * n, 512)
        passes = 1
        if done == rows_total and k_host is not None:
            # the whole step took less than the budget: time further whole steps
            # until it is spent, so that the figure is not one short run
            while t_used < budget_s:
                t0 = time.perf_counter()
                oracle.gqa_decode(x.q, x.k_cache, x.v_cache, x.seqlens, x.scale, window=self.window)
                t_used += time.perf_counter() - t0
                passes += 1
            tokens *= passes
        # tokens here are (query head, key) pairs; convert to the step's KV bytes
        frac = tokens / (self.sum_T * x.H)
        sample = "%d of %d output rows (b, head), each over its whole cache" % (done, rows_total)
        if passes > 1:
            sample = "%d whole steps (all %d output rows (b, head), each over its whole cache)" % (passes, rows_total)
        return {"seconds": t_used, "fraction_of_step": frac, "sample": sample}


class Prefill:
    kind = "prefill"
    graphable = True

    def __init__(self, name, gqa, device="cuda"):
        w = gi.WORKLOADS[name]
        self.name, self.w, self.gqa = name, w, gqa
        x = gi.prefill_inputs(w["B"], w["S"], w["H"], w["G"], w["d_h"], w["dtype"], seed=0)
        self.x = x
        self.q, self.k, self.v = x.q.to(device), x.k.to(device), x.v.to(device)
        self.out = torch.empty_like(self.q)
        S = x.S
        self.window = w.get("window", 0)
        Wn = self.window if self.window else S
        pairs = sum(min(s + 1, Wn) for s in range(S))              # visible (query, key) pairs
        self.flops = 4 * x.B * x.H * x.d_h * pairs                 # QK^T + PV on visible pairs
        self.bytes = (self.q.numel() * 2 + self.k.numel() * 2 * 2 + self.out.numel() * 2)
        self.launches_per_step = 1
        self.dtype = "bf16"

    def step(self, stream=None):
        self.gqa.prefill_causal(self.q, self.k, self.v, self.x.scale, out=self.out, stream=stream,
                                window=self.window)

    def config(self):
        x = self.x
        return {"workload": self.name, "B": x.B, "S": x.S, "H": x.H, "G": x.G, "d_h": x.d_h,
                "causal_flops": self.flops, "window": self.window}

    def metric(self, sps, n_ranks):
        return {"value": n_ranks * self.flops / sps / 1e12, "unit": "TFLOP/s"}

    def roofline(self, sps, peaks, which, long_run=False):
        key = "bf16_tflops_sustained" if long_run else "bf16_tflops"
        a = self.flops / sps / 1e12
        return {"bound": "tensor", "achieved": a, "peak": peaks[key], "unit": "TFLOP/s",
                "frac": a / peaks[key], "peak_source": which + " " + key,
                "peak_nominal": NOMINAL_PEAKS["bf16_tflops"],
                "frac_nominal": a / NOMINAL_PEAKS["bf16_tflops"],
                "traffic": NCU_TRAFFIC.get(self.name)}

    def oracle_sample(self, budget_s):
        import oracle
        x = self.x
        gen = torch.Generator().manual_seed(7)
        total = x.B * x.S * x.H
        done, t_used, flops = 0, 0.0, 0
        n = 1
        while done < total and (done == 0 or t_used < budget_s):
            rows = torch.randint(0, total, (n,), generator=gen).tolist()
            t0 = time.perf_counter()
            oracle.gqa_prefill_causal(x.q, x.k, x.v, x.scale, rows=rows, window=self.window)
            t_used += time.perf_counter() - t0
            Wn = self.window if self.window else x.S
            flops += sum(4 * x.d_h * min((r // x.H) % x.S + 1, Wn) for r in rows)
            done += n
            n = min(2 * n, 1024)
        return {"seconds": t_used, "fraction_of_step": flops / self.flops,
                "sample": "%d random output rows (b, s, head), each over keys 0..s" % done}


class MeanPool:
    kind = "meanpool"
    graphable = True

    def __init__(self, name, gqa, device="cuda"):
        w = gi.WORKLOADS[name]
        self.name, self.w, self.gqa = name, w, gqa
        wk, wv = gi.meanpool_inputs(w["H"], w["d_h"], w["d"], w["dtype"], seed=0, std=w["std"])
        self.wk_h, self.wv_h = wk, wv
        self.wk, self.wv = wk.to(device), wv.to(device)
        G = w["G"]
        self.ok = torch.empty((G, w["d_h"], w["d"]), dtype=wk.dtype, device=device)
        self.ov = torch.empty_like(self.ok)
        self.bytes = 2 * (wk.numel() + self.ok.numel()) * wk.element_size()
        self.launches_per_step = 1
        self.dtype = "bf16"

    def step(self, stream=None):
        self.gqa.meanpool_kv(self.wk, self.wv, self.w["G"], out_k=self.ok, out_v=self.ov, stream=stream)

    def config(self):
        w = self.w
        return {"workload": self.name, "H": w["H"], "G": w["G"], "d_h": w["d_h"], "d": w["d"]}

    def metric(self, sps, n_ranks):
        return {"value": n_ranks * self.bytes / sps / 1e9, "unit": "GB/s"}

    def roofline(self, sps, peaks, which, long_run=False):
        a = self.bytes / sps / 1e9
        return {"bound": "hbm", "achieved": a, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": a / peaks["hbm_gbs"], "peak_source": which + " hbm_gbs",
                "peak_nominal": NOMINAL_PEAKS["hbm_gbs"], "frac_nominal": a / NOMINAL_PEAKS["hbm_gbs"],
                "traffic": NCU_TRAFFIC.get(self.name)}

    def oracle_sample(self, budget_s):
        import oracle
        t0 = time.perf_counter()
        oracle.meanpool(self.wk_h, self.w["G"])
        oracle.meanpool(self.wv_h, self.w["G"])
        return {"seconds": time.perf_counter() - t0, "fraction_of_step": 1.0,
                "sample": "the whole conversion (both W_K and W_V)"}


L2_ROTATE_BYTES = 256 << 20  # > 2x the 126 MB L2


def rotation(nbytes):
    """Copies of a weight set needed for the steps' working set to exceed L2."""
    return max(1, -(-L2_ROTATE_BYTES // max(1, nbytes)))


class QkvAppend:
    """One decode token's Q/K/V projections with the KV-cache append.

    The weights (48 MB for the 7B shape) would fit in L2, so step i reads copy
    i mod n of them, with n copies spanning more than twice the L2; every step
    writes the same k/v rows and q, so repeated steps are identical work."""
    kind = "qkv"
    graphable = True

    def __init__(self, name, gqa, device="cuda"):
        w = gi.WORKLOADS[name]
        self.name, self.w, self.gqa = name, w, gqa
        x = gi.qkv_inputs(w["B"], w["d"], w["H"], w["G"], w["d_h"], w["T"], w["dtype"], seed=0)
        self.x = x
        self.h = x.h.to(device)
        wbytes = sum(t.numel() * t.element_size() for t in (x.W_Q, x.W_K, x.W_V)) + self._extra_weight_bytes()
        self.n_sets = rotation(wbytes)
        self.sets = [tuple(t.to(device) for t in (x.W_Q, x.W_K, x.W_V)) for _ in range(self.n_sets)]
        self.wq, self.wk, self.wv = self.sets[0]
        self.i = 0
        self.weight_mb = wbytes / 1e6
        self.kc, self.vc = x.k_cache.to(device), x.v_cache.to(device)
        self.sl = x.seqlens.to(device)
        self.q = torch.empty((x.B, x.H, x.d_h), dtype=x.h.dtype, device=device)
        self.sl_out = torch.empty_like(self.sl)
        # split-K over every SM (the workspace holds the partial sums of split blocks)
        self.pws = torch.empty(gqa.project_workspace_bytes((x.H + 2 * x.G) * x.d_h, x.d), dtype=torch.uint8,
                               device=device)
        e = x.h.element_size()
        # weights read once, h read, q written, one k and one v row per KV head written
        self.bytes = (x.d * (x.H + 2 * x.G) * x.d_h + x.B * x.d + x.B * x.H * x.d_h
                      + 2 * x.B * x.G * x.d_h) * e
        self.launches_per_step = (x.B + 31) // 32
        self.dtype = "bf16"

    def _extra_weight_bytes(self):
        return 0

    def _next_set(self):
        ws = self.sets[self.i % self.n_sets]
        self.i += 1
        return ws

    def step(self, stream=None):
        wq, wk, wv = self._next_set()
        self.gqa.qkv_append(self.h, wq, wk, wv, self.kc, self.vc, self.sl,
                            q_out=self.q, seqlens_out=self.sl_out, stream=stream, workspace=self.pws)

    def config(self):
        x = self.x
        return {"workload": self.name, "B": x.B, "d": x.d, "H": x.H, "G": x.G, "d_h": x.d_h,
                "T_cap": x.T_cap,
                "l2": "weights rotate over %d copies of %.0f MB (> 126 MB L2), no flush"
                      % (self.n_sets, self.weight_mb)}

    def metric(self, sps, n_ranks):
        return {"value": n_ranks * self.bytes / sps / 1e9, "unit": "GB/s"}

    def roofline(self, sps, peaks, which, long_run=False):
        a = self.bytes / sps / 1e9
        return {"bound": "hbm", "achieved": a, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": a / peaks["hbm_gbs"], "peak_source": which + " hbm_gbs",
                "peak_nominal": NOMINAL_PEAKS["hbm_gbs"], "frac_nominal": a / NOMINAL_PEAKS["hbm_gbs"],
                "traffic": NCU_TRAFFIC.get(self.name)}

    def oracle_sample(self, budget_s):
        import oracle
        x = self.x
        t0 = time.perf_counter()
        oracle.qkv_append(x.h[:1], x.W_Q, x.W_K, x.W_V, x.k_cache[:1], x.v_cache[:1], x.seqlens[:1])
        return {"seconds": time.perf_counter() - t0, "fraction_of_step": 1.0 / x.B,
                "sample": "the projections and append of sequence 0 of %d" % x.B}


class LayerDecode(QkvAppend):
    """One decode step of the attention layer: append, attend over the cache, W_O."""
    kind = "layer"

    def __init__(self, name, gqa, device="cuda"):
        super().__init__(name, gqa, device)
        x = self.x
        gen = torch.Generator().manual_seed(1)
        D = x.H * x.d_h
        wo = (torch.randn(D, x.d, generator=gen) * D ** -0.5).to(x.h.dtype)
        self.wos = [wo.to(device) for _ in range(self.n_sets)]
        self.wo = self.wos[0]
        self.out = torch.empty((x.B, x.d), dtype=x.h.dtype, device=device)
        self.ws = torch.empty(int(gqa.lib.gqa_layer_decode_workspace_bytes(x.B, x.d, x.H, x.G, x.d_h,
                                                                             x.T_cap, gqa.GQA_BF16)),
                              dtype=torch.uint8, device=device)
        e = x.h.element_size()
        T_after = (x.seqlens.clamp(max=x.T_cap - 1) + 1).sum().item()
        # weights (Q, K, V, O) once, the cache over the lengths after the append, small tensors
        self.bytes = ((x.d * (x.H + 2 * x.G) * x.d_h + D * x.d) + 2 * T_after * x.G * x.d_h
                      + x.B * x.d * 2 + 2 * x.B * x.H * x.d_h + 2 * x.B * x.G * x.d_h) * e
        self.launches_per_step = 2 * ((x.B + 31) // 32) + 2

    def _extra_weight_bytes(self):
        x = self.x
        return x.H * x.d_h * x.d * x.h.element_size()  # W_O

    def step(self, stream=None):
        k = self.i % self.n_sets
        wq, wk, wv = self._next_set()
        self.gqa.layer_decode_step(self.h, wq, wk, wv, self.wos[k], self.kc, self.vc,
                                   self.sl, out=self.out, seqlens_out=self.sl_out,
                                   workspace=self.ws, stream=stream)

    def oracle_sample(self, budget_s):
        import oracle
        x = self.x
        t0 = time.perf_counter()
        oracle.layer_decode_step(x.h[:1], x.W_Q, x.W_K, x.W_V, self.wo.cpu(), x.k_cache[:1],
                                 x.v_cache[:1], x.seqlens[:1], x.d_h ** -0.5)
        return {"seconds": time.perf_counter() - t0, "fraction_of_step": 1.0 / x.B,
                "sample": "the whole layer step of sequence 0 of %d" % x.B}


def make(name, gqa):
    kind = gi.WORKLOADS[name]["kind"]
    return {"decode": Decode, "prefill": Prefill, "meanpool": MeanPool, "qkv": QkvAppend,
            "layer": LayerDecode}[kind](name, gqa)


# ------------------------------------------------------------------ timing

GRAPH_CHUNK = 50  # steps per captured CUDA graph


def _capture(wl, n):
    """A CUDA graph of n consecutive steps of wl (the same kernels, arguments
    and stream order as n eager calls), or None when capture fails."""
    if n <= 0:
        return None
    try:
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.graph(g, stream=s):
            for _ in range(n):
                wl.step()
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        return g
    except Exception:  # noqa: BLE001 -- any capture failure means: launch eagerly
        torch.cuda.synchronize()
        return None


def time_steps(wl, steps, warmup, world, clocks=None):
    """W untimed steps, then K steps between a barrier + synchronize on both
    sides, timed with CUDA events on the launching stream.  Returns seconds
    per step (max over ranks).  Workloads whose step is a pure function of
    resident inputs replay it from CUDA graphs of GRAPH_CHUNK steps (exactly
    K steps in all); wl.launch records which launch mode was timed."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        wl.step()
    torch.cuda.synchronize()
    graphs = None
    if getattr(wl, "graphable", False):
        full, rem = divmod(steps, GRAPH_CHUNK)
        g_full = _capture(wl, GRAPH_CHUNK) if full else None
        g_rem = _capture(wl, rem) if rem else None
        if (g_full is not None or not full) and (g_rem is not None or not rem):
            graphs = (g_full, full, g_rem)
            for g in (g_full, g_rem):  # one untimed replay of each: a graph's first launch is slow
                if g is not None:
                    g.replay()
            torch.cuda.synchronize()
    wl.launch = ("cuda_graph, %d steps per graph" % GRAPH_CHUNK) if graphs else "eager"
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx = clocks if clocks is not None else _Null()
    with ctx:
        ev0.record(stream)
        if graphs:
            g_full, full, g_rem = graphs
            for _ in range(full):
                g_full.replay()
            if g_rem is not None:
                g_rem.replay()
        else:
            for _ in range(steps):
                wl.step()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms, world)
    return ms / 1e3 / steps


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def steps_for(seconds_per_step, target_s, lo=5, hi=200000):
    return int(min(hi, max(lo, target_s / max(seconds_per_step, 1e-9))))


def probe_step_time(wl):
    wl.step()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for _ in range(3):
        wl.step()
    torch.cuda.synchronize()
    return (time.perf_counter() - t0) / 3


def run_e2e(wl, steps, world):
    wl.e2e_setup()
    for _ in range(2):
        wl.e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        wl.e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    sps = max_over_ranks(ev0.elapsed_time(ev1), world) / 1e3 / steps
    m = wl.metric(sps, world)
    return {"value": m["value"], "unit": m["unit"], "h2d_bytes_per_step": wl.h2d,
            "d2h_bytes_per_step": wl.d2h, "steps": steps, "ms_per_step": sps * 1e3}


def cpu_baseline(wl, budget_s):
    import oracle
    r = wl.oracle_sample(budget_s)
    sps_equiv = r["seconds"] / max(r["fraction_of_step"], 1e-30)   # seconds per whole step
    m = wl.metric(sps_equiv, 1)
    return {"value": m["value"], "unit": m["unit"], "cores": oracle.default_threads(),
            "kind": "oracle", "sample": r["sample"], "seconds": r["seconds"]}


# ------------------------------------------------------------------ main

def run_reference(args, world, rank):
    if rank != 0:
        return 0
    import oracle

    name = args.workload or HEADLINE
    wl = make_host_only(name)
    # the whole reference run stays within about a minute and a half of oracle time
    per_step = min(2.0, 90.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        wl.oracle_sample(per_step / 4)
    secs, frac = 0.0, 0.0
    samples = []
    for _ in range(args.steps):
        r = wl.oracle_sample(per_step)
        secs += r["seconds"]
        frac += r["fraction_of_step"]
        samples.append(r["sample"])
    sps = secs / frac
    m = wl.metric(sps, 1)
    line = {"impl": "reference", "metric": METRIC, "value": m["value"], "unit": m["unit"],
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": wl.config(),
            "cpu_baseline": {"value": m["value"], "unit": m["unit"], "kind": "oracle",
                             "cores": oracle.default_threads(),
                             "sample": "each step: " + samples[-1]},
            "e2e": {"value": m["value"], "unit": m["unit"], "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def make_host_only(name):
    """A workload object with host inputs only (the reference arm needs no GPU)."""
    kind = gi.WORKLOADS[name]["kind"]
    cls = {"decode": Decode, "prefill": Prefill, "meanpool": MeanPool, "qkv": QkvAppend,
           "layer": QkvAppend}[kind]
    obj = cls.__new__(cls)
    w = gi.WORKLOADS[name]
    obj.name, obj.w, obj.gqa = name, w, None
    obj.window = w.get("window", 0)
    if kind == "decode":
        x = gi.decode_inputs(w["B"], w["H"], w["G"], w["d_h"], w["T"], w["dtype"], seed=0,
                             ragged=w["ragged"])
        obj.x = x
        T_att = x.seqlens.clamp(0, x.T_cap)
        if obj.window:
            T_att = T_att.clamp(max=obj.window)
        obj.sum_T = int(T_att.sum())
        obj.bytes = 2 * obj.sum_T * x.G * x.d_h * x.q.element_size()
    elif kind == "prefill":
        x = gi.prefill_inputs(w["B"], w["S"], w["H"], w["G"], w["d_h"], w["dtype"], seed=0)
        obj.x = x
        Wn = obj.window if obj.window else x.S
        obj.flops = 4 * x.B * x.H * x.d_h * sum(min(s + 1, Wn) for s in range(x.S))
    elif kind in ("qkv", "layer"):
        x = gi.qkv_inputs(w["B"], w["d"], w["H"], w["G"], w["d_h"], w["T"], w["dtype"], seed=0)
        obj.x = x
        obj.bytes = (x.d * (x.H + 2 * x.G) * x.d_h + x.B * x.d + x.B * x.H * x.d_h
                     + 2 * x.B * x.G * x.d_h) * x.h.element_size()
    else:
        wk, wv = gi.meanpool_inputs(w["H"], w["d_h"], w["d"], w["dtype"], seed=0, std=w["std"])
        obj.wk_h, obj.wv_h = wk, wv
        obj.bytes = 2 * (wk.numel() + w["G"] * w["d_h"] * w["d"]) * wk.element_size()
    return obj


def measure_row(name, gqa, peaks, which, world, target_s=0.4):
    wl = make(name, gqa)
    sps0 = probe_step_time(wl)
    steps = steps_for(sps0, target_s)
    sps = time_steps(wl, steps, max(3, min(50, steps // 10)), world)
    row = {"config": dict(wl.config(), launch=wl.launch), "steps": steps, "ms_per_step": sps * 1e3,
           "dtype": wl.dtype}
    row.update(wl.metric(sps, world))
    row["roofline"] = wl.roofline(sps, peaks, which, long_run=sps * steps > 1.0)
    del wl
    torch.cuda.empty_cache()
    return row


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=100)
    ap.add_argument("--workload", default=None, choices=sorted(gi.WORKLOADS))
    ap.add_argument("--impl", default="gqa", choices=["gqa", "reference"])
    ap.add_argument("--no-rows", action="store_true", help="headline only")
    ap.add_argument("--oracle-budget", type=float, default=10.0)
    args = ap.parse_args()

    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        rc = run_reference(args, world, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc

    import kv_cache_decode_04_b200 as gqa  # fails loudly if libgqa.so is missing

    peaks, which = load_peaks()
    name = args.workload or HEADLINE
    wl = make(name, gqa)
    warmup = max(3, args.warmup)

    clocks = ClockSampler(local)
    sps = time_steps(wl, args.steps, warmup, world, clocks)
    csum = clocks.summary()
    remeasured = False
    if BAD_REASONS & set(csum["reasons"]):
        clocks = ClockSampler(local)
        sps = time_steps(wl, args.steps, warmup, world, clocks)
        csum = clocks.summary()
        remeasured = True
    m = wl.metric(sps, world)
    long_run = sps * args.steps > 1.0
    roof = wl.roofline(sps, peaks, which, long_run)
    e2e = run_e2e(wl, max(3, min(20, args.steps)), world) if hasattr(wl, "e2e_setup") else None

    line = {"metric": METRIC, "value": m["value"], "unit": m["unit"], "n_gpus": world,
            "steps": args.steps, "warmup": warmup, "ms_per_step": sps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": wl.dtype, "data": "synthetic",
            "config": dict(wl.config(), launch=wl.launch,
                           parallelism="replicas, one independent batch per rank",
                           l2="inputs larger than L2 (KV %.0f MB vs 126 MB L2), no flush"
                           % (getattr(wl, "bytes", 0) / 1e6)),
            "roofline": roof, "clocks": dict(csum, remeasured=remeasured),
            "gpu_launches": wl.launches_per_step * args.steps}
    for k in ("attn_tokens_per_s", "kv_bytes_per_step"):
        if k in m:
            line[k] = m[k]
    if e2e is not None:
        line["e2e"] = e2e
    if rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_baseline(wl, args.oracle_budget)
    del wl
    torch.cuda.empty_cache()

    if world == 1 and not args.no_rows and args.workload is None:
        rows = {}
        for rn in ROW_WORKLOADS:
            try:
                rows[rn] = measure_row(rn, gqa, peaks, which, world)
            except Exception as e:  # a row that cannot run is reported, not hidden
                rows[rn] = {"error": "%s: %s" % (type(e).__name__, e)}
        line["rows"] = rows

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
