"""Benchmark of the B200 scaled dot-product attention forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one sdpa_fwd() call on one batch of the headline workload (bf16
causal prefill, B=4, Hq=Hkv=16, L=S=2048, E=Ev=128): load, scores, logits,
online softmax, weighted sum, epilogue, with causal tile skipping.  Rank 0
prints ONE JSON line.  Inputs are seeded synthetic N(0,1) tensors; several
input sets rotate so that their total exceeds the 126 MB L2 and no step reads
its inputs from L2.  Under torchrun each rank runs its own copy of the
workload on its own GPU (independent problems, no collective on the data
path: weak scaling); time is the max over ranks.

At N=1 the line also carries the other workloads (fp32 small case, fp16
packed varlen, bf16 GQA decode, fp16 head_dim-96 prefill at two scales), each
with its own roofline, and the float64 CPU oracle timed on a bounded sample.

``--impl reference`` times the float64 CPU oracle on this host (the only
reference implementation there is), on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads as W  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
METRIC = "prefill TFLOP/s (% of dense peak); decode K/V GB/s (% of HBM peak)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# The sources each path's kernels are compiled from.
KERNEL_SOURCES = {
    "prefill_tcgen05": ["prefill_sm100.cu", "sm100_ptx.cuh", "exp2_poly.cuh", "common.cuh"],
    "decode_split": ["decode.cu", "common.cuh"],
    "decode_paged": ["decode.cu", "decode_paged.cu", "common.cuh"],
    "simt": ["simt.cu", "common.cuh"],
    "backward_simt": ["backward_simt.cu", "backward.cuh", "common.cuh"],
    "backward_tcgen05": ["backward_sm100.cu", "backward_simt.cu", "backward.cuh", "tma_host.cuh", "sm100_ptx.cuh",
                         "exp2_poly.cuh", "common.cuh"],
}


def kernel_source_hash(path: str = None) -> str:
    """Hash of the CUDA sources of one path (all sources when None), to tell
    whether stored ncu counters still describe the kernel being timed."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "scaled_dot_product_15_b200", "csrc")
    names = KERNEL_SOURCES.get(path) if path else None
    if names is None:
        names = [n for n in os.listdir(csrc) if n.endswith((".cu", ".cuh"))]
    for name in sorted(names):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def stored_traffic(workload: str, path: str):
    """DRAM bytes per launch of the path's dominant kernel from a committed
    ncu capture (profiles/traffic.json), if that kernel's sources have not
    changed since it was taken (else None)."""
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(tpath) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(workload)
    if not e or e.get("path") != path or e.get("kernel_sha") != kernel_source_hash(path):
        return None
    return e.get("traffic_bytes_per_launch")


# ----------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        "hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
        "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
        "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
        "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
        "hw_power_brake": "nvmlClocksEventReasonHwPowerBrakeSlowdown",
    }

    def __init__(self, device_index: int, interval: float = 0.005):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            uuid = None
            try:
                uuid = torch.cuda.get_device_properties(device_index).uuid
            except Exception:
                pass
            handle = None
            if uuid is not None:
                want = "GPU-" + str(uuid)
                for i in range(pynvml.nvmlDeviceGetCount()):
                    h = pynvml.nvmlDeviceGetHandleByIndex(i)
                    u = pynvml.nvmlDeviceGetUUID(h)
                    u = u.decode() if isinstance(u, bytes) else u
                    if u == want:
                        handle = h
            if handle is None:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.h = handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self._ok = False
        self.interval = interval
        self._t = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for name, attr in self.REASONS.items():
                    if r & getattr(nv, attr, 0):
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.interval)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()
            self._run_once()

    def _run_once(self):
        if not self.samples and self._ok:
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            except Exception:
                pass

    def summary(self):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        med = float(np.median(self.samples)) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ----------------------------------------------------------------- GPU arm


def _bytes_of(ts):
    return sum(t.numel() * t.element_size() for t in ts)


def make_sets(w: W.Workload, device):
    """Input sets for a workload: enough copies that their total exceeds L2."""
    q, k, v = W.make_inputs(w, device)
    set_bytes = _bytes_of((q, k, v))
    n = 1 if set_bytes > 2 * L2_BYTES else min(16, int(math.ceil(2.5 * L2_BYTES / set_bytes)))
    sets = [(q, k, v)]
    for i in range(1, n):
        # different memory, same values: L2 residency is what matters
        sets.append((q.clone(), k.clone(), v.clone()))
    return sets, set_bytes


def prepared_calls(w: W.Workload, sets, device):
    from scaled_dot_product_15_b200 import PreparedCall

    seqlens = W.workload_seqlens(w)
    calls = []
    for q, k, v in sets:
        if w.layout == "packed":
            cu = torch.tensor(W.cu_seqlens_of(seqlens), dtype=torch.int32, device=device)
            calls.append(PreparedCall(q, k, v, is_causal=w.mask == "block_diag_causal", cu_seqlens=cu,
                                      max_seqlen=max(seqlens), scale=w.scale))
        else:
            calls.append(PreparedCall(q, k, v, is_causal=w.mask == "causal", scale=w.scale,
                                      enable_gqa=w.Hq != w.Hkv))
    return calls


def time_device(calls, steps: int, warmup: int, dist_on: bool, sampler=None):
    """Warm up, then time exactly `steps` calls with CUDA events on the
    launching stream; per-call events give the kernels' average duration."""
    stream = torch.cuda.current_stream()
    launches = 0
    for i in range(warmup):
        calls[i % len(calls)]()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ctx = sampler if sampler is not None else _Null()
    with ctx:
        t0.record(stream)
        for i in range(steps):
            ev[i][0].record(stream)
            launches += calls[i % len(calls)]()
            ev[i][1].record(stream)
        t1.record(stream)
        torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    total_ms = t0.elapsed_time(t1)
    per = [a.elapsed_time(b) for a, b in ev]
    return total_ms, float(np.mean(per)), launches


class _Null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def time_e2e(w: W.Workload, sets, steps: int, warmup: int):
    """Same metric end to end: each step copies its inputs from pinned host
    memory, runs sdpa() through the public API, and reads out and lse back."""
    from scaled_dot_product_15_b200 import sdpa

    seqlens = W.workload_seqlens(w)
    q, k, v = sets[0]
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    dq, dk, dv = (torch.empty_like(t) for t in (q, k, v))
    cu = None
    if w.layout == "packed":
        cu = torch.tensor(W.cu_seqlens_of(seqlens), dtype=torch.int32, device=q.device)
    out_h = lse_h = None

    def step():
        nonlocal out_h, lse_h
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        if cu is not None:
            o, l_ = sdpa(dq, dk, dv, is_causal=True, cu_seqlens=cu, max_seqlen=max(seqlens), scale=w.scale)
        else:
            o, l_ = sdpa(dq, dk, dv, is_causal=w.mask == "causal", scale=w.scale, enable_gqa=w.Hq != w.Hkv)
        if out_h is None:
            out_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
            lse_h = torch.empty(l_.shape, dtype=l_.dtype, pin_memory=True)
        out_h.copy_(o, non_blocking=True)
        lse_h.copy_(l_, non_blocking=True)
        return o, l_

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        o, l_ = step()
    t1.record()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    h2d = _bytes_of((hq, hk, hv))
    d2h = _bytes_of((out_h, lse_h))
    return ms, h2d, d2h


def work_units(w: W.Workload):
    """(amount per call, unit, bound) of a workload's roofline."""
    if w.L == 1 and w.mask == "none":
        return W.kv_bytes(w), "GB/s", "hbm"
    return W.flops(w), "TFLOP/s", "tensor"


def rate(amount, ms, unit):
    if unit == "GB/s":
        return amount / (ms * 1e-3) / 1e9
    return amount / (ms * 1e-3) / 1e12


def roofline(w: W.Workload, kernel_ms: float, peaks, peak_src, path: str, sustained=False):
    amount, unit, bound = work_units(w)
    achieved = rate(amount, kernel_ms, unit)
    if bound == "hbm":
        peak = float(peaks["hbm_gbs"])
    else:
        peak = float(peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"])
        # fp16 dense rate equals bf16 on this tensor core; fp32 runs on FMA units
    return {"bound": bound, "achieved": round(achieved, 3), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4), "traffic": stored_traffic(w.name, path),
            "peak_source": f"of {peak_src}", "algorithmic_per_launch": amount}


def measure_workload(w: W.Workload, steps: int, warmup: int, peaks, peak_src, device, dist_on=False,
                     sampler=None):
    sets, set_bytes = make_sets(w, device)
    calls = prepared_calls(w, sets, device)
    total_ms, kernel_ms, launches = time_device(calls, steps, warmup, dist_on, sampler)
    amount, unit, _ = work_units(w)
    res = {
        "value": round(rate(amount, total_ms / steps, unit), 3),
        "unit": unit,
        "ms_per_step": round(total_ms / steps, 5),
        "path": calls[0].plan,
        "gpu_launches": launches,
        "roofline": roofline(w, kernel_ms, peaks, peak_src, calls[0].plan),
        "l2": (f"{len(sets)} rotating input sets of {set_bytes / 1e6:.1f} MB"
               + (" (all sets fit in L2: latency case)" if len(sets) * set_bytes < L2_BYTES else "")),
    }
    if w.layout == "packed":
        res["flops_exact"] = W.flops(w)
        res["segments"] = len(W.workload_seqlens(w))
    del calls, sets
    torch.cuda.empty_cache()
    return res, total_ms, kernel_ms, launches


def measure_backward(w: W.Workload, steps: int, warmup: int, peaks, peak_src, device):
    """The gradients of a prefill workload (sdpa_backward for a random output
    gradient, the forward's out and lse given), timed like the forward.
    Algorithmic work: 2.5x the forward's flops (five matrix products of the
    forward's size: S, dP, dV, dK, dQ)."""
    from scaled_dot_product_15_b200 import sdpa, sdpa_backward

    q, k, v = W.make_inputs(w, device)
    g = W.randn(tuple(q.shape), w.seed + 100, q.dtype).to(device)
    causal = w.mask == "causal"
    out, lse = sdpa(q, k, v, is_causal=causal, scale=w.scale)

    def call():
        sdpa_backward(q, k, v, out, lse, g, is_causal=causal, scale=w.scale)
        from scaled_dot_product_15_b200 import api

        return api.last_launch_count()

    total_ms, kernel_ms, launches = time_device([call], steps, warmup, False)
    from scaled_dot_product_15_b200.api import backward_plan

    path = backward_plan(q, k, v, g, mask_kind=1 if causal else 0)
    amount = 2.5 * W.flops(w)
    achieved = rate(amount, kernel_ms, "TFLOP/s")
    peak = float(peaks["bf16_tflops"])
    return {
        "value": round(rate(amount, total_ms / steps, "TFLOP/s"), 3),
        "unit": "TFLOP/s",
        "ms_per_step": round(total_ms / steps, 5),
        "path": path,
        "gpu_launches": launches,
        "roofline": {"bound": "tensor", "achieved": round(achieved, 3), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": stored_traffic(w.name + ":backward", path),
                     "peak_source": f"of {peak_src}", "algorithmic_per_launch": amount},
        "note": "gradients (dq, dk, dv) of this workload: row-dot, dK/dV and dQ kernels",
    }


PAGE_SIZE = 16


def paged_cache(k, v, page_size: int, pages_layout: str, seed: int):
    """A contiguous (B, Hkv, S, E) cache rewritten as a page pool: pages of
    ``page_size`` tokens, page i of the identity order stored at pool slot
    perm[i] for a seeded permutation, and the block table that undoes it.
    Returns (k_pages, v_pages, block_table int32 (B, S/page_size))."""
    B, Hkv, S, _ = k.shape
    n_pages = B * S // page_size
    perm = torch.randperm(n_pages, generator=torch.Generator().manual_seed(seed)).to(k.device)

    def pool(t):
        e = t.shape[-1]
        if pages_layout == "head_major":
            pages = t.reshape(B, Hkv, S // page_size, page_size, e).permute(0, 2, 1, 3, 4)
            pages = pages.reshape(n_pages, Hkv, page_size, e)
        else:
            pages = t.transpose(1, 2).reshape(n_pages, page_size, Hkv, e)
        out = torch.empty_like(pages)
        out[perm] = pages
        return out

    return pool(k), pool(v), perm.to(torch.int32).reshape(B, S // page_size).contiguous()


def measure_paged_decode(w: W.Workload, steps: int, warmup: int, peaks, peak_src, device,
                         pages_layout: str = "head_major"):
    """The decode workload with its key/value cache in pages of 16 tokens of a
    shared pool, the pages in shuffled order behind each row's block table
    (sdpa_decode_paged).  ``pages_layout``: "head_major" pools (num_pages,
    Hkv, 16, E), each head's 16 tokens of a page contiguous; "token_major"
    (num_pages, 16, Hkv, E).  Algorithmic bytes: the same K/V bytes as the
    contiguous decode (the block table adds 4 bytes per page)."""
    from scaled_dot_product_15_b200 import api, sdpa_decode_paged

    q, k, v = W.make_inputs(w, device)
    kp, vp, table = paged_cache(k, v, PAGE_SIZE, pages_layout, w.seed)
    del k, v
    torch.cuda.empty_cache()
    lens = torch.full((w.B,), w.S, dtype=torch.int32, device=device)
    out, lse = sdpa_decode_paged(q, kp, vp, table, lens, pages_layout=pages_layout)

    def call():
        sdpa_decode_paged(q, kp, vp, table, lens, pages_layout=pages_layout, out=out, lse=lse)
        return api.last_launch_count()

    total_ms, kernel_ms, launches = time_device([call], steps, warmup, False)
    amount = W.kv_bytes(w)
    achieved = rate(amount, kernel_ms, "GB/s")
    peak = float(peaks["hbm_gbs"])
    res = {
        "value": round(rate(amount, total_ms / steps, "GB/s"), 3),
        "unit": "GB/s",
        "ms_per_step": round(total_ms / steps, 5),
        "path": "decode_paged",
        "gpu_launches": launches,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 3), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": stored_traffic(w.name + f":paged{PAGE_SIZE}"
                                               + ("" if pages_layout == "head_major" else "_token_major"),
                                               "decode_paged"),
                     "peak_source": f"of {peak_src}", "algorithmic_per_launch": amount},
        "note": f"paged cache: {pages_layout} pages of {PAGE_SIZE} tokens in shuffled order, one block table per row",
    }
    del kp, vp, q, out, lse
    torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------------- CPU oracle


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info

        info = threadpool_info()
        return max([i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"] or [1])
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(w: W.Workload, seconds: float):
    """Run the float64 oracle on whole (batch, head) problems of the workload
    until `seconds` of CPU time have passed; returns (amount, unit, elapsed,
    description)."""
    from oracle import sdpa as ref_sdpa
    from oracle import sdpa_packed as ref_packed

    amount_unit = work_units(w)
    t0 = time.perf_counter()
    done = 0.0
    n_units = 0
    if w.layout == "packed":
        seqlens = W.workload_seqlens(w)
        q, k, v = W.make_inputs(w, "cpu")
        h = 0
        while (h == 0 or time.perf_counter() - t0 < seconds) and h < w.Hq:
            ref_packed(q, k, v, seqlens, causal=True, heads=[h], scale=w.scale)
            done += W.flops(w) / w.Hq
            h += 1
            n_units += 1
        desc = f"{n_units} of {w.Hq} heads of the packed batch"
    else:
        g = w.Hq // w.Hkv
        per_head = work_units(w)[0] / (w.B * w.Hq)
        b = 0
        while (b == 0 or time.perf_counter() - t0 < seconds) and b < w.B:
            qb, kb, vb = (W.make_slice(w, x, b) for x in ("q", "k", "v"))
            for h in range(w.Hq):
                ref_sdpa(qb[h][None, None], kb[h // g][None, None], vb[h // g][None, None],
                         is_causal=w.mask == "causal", scale=w.scale)
                done += per_head
                n_units += 1
                if time.perf_counter() - t0 >= seconds:
                    break
            b += 1
        desc = f"{n_units} of {w.B * w.Hq} (batch, query head) problems"
    el = time.perf_counter() - t0
    return done, amount_unit[1], el, desc


def cpu_baseline(w: W.Workload, seconds: float):
    amount, unit, el, desc = oracle_sample(w, seconds)
    return {"value": round(rate(amount, el * 1e3, unit), 6), "unit": unit, "cores": _blas_threads(),
            "kind": "oracle", "sample": f"{desc}, {el:.1f} s, float64 numpy"}


# ----------------------------------------------------------------- main


def max_over_ranks(x: float, device, dist_on: bool) -> float:
    """The largest of every rank's `x` (every rank gets it): the job is as
    slow as its slowest rank."""
    t = torch.tensor([x], dtype=torch.float64, device=device)
    if dist_on:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(amount_per_rank: float, ranks: int, max_ms_per_step: float, unit: str) -> float:
    """Whole-job throughput: the work of every rank over the slowest rank's
    time per step (weak scaling: each rank runs its own replica)."""
    return rate(amount_per_rank * ranks, max_ms_per_step, unit)


def dist_setup(n_gpus):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return ws, rank, local


def run_reference(args, ws, rank):
    if rank != 0:
        return
    w = W.WORKLOADS[args.workload]
    from oracle import sdpa as ref_sdpa

    amount_unit = work_units(w)
    per_step = min(args.ref_seconds, 150.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(w, 0.0)
    times, amounts, descs = [], [], []
    for _ in range(args.steps):
        amount, unit, el, desc = oracle_sample(w, per_step)
        times.append(el)
        amounts.append(amount)
        descs.append(desc)
    tot = sum(times)
    val = rate(sum(amounts), tot * 1e3, amount_unit[1])
    line = {
        "impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": amount_unit[1],
        "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(val, 6), "unit": amount_unit[1], "cores": _blas_threads(),
                         "kind": "oracle", "sample": f"per step: {descs[0]}"},
        "e2e": {"value": round(val, 6), "unit": amount_unit[1], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=W.HEADLINE, choices=sorted(W.WORKLOADS))
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-seconds", type=float, default=2.0, help="oracle seconds per reference step")
    ap.add_argument("--bare", action="store_true",
                    help="only run the workload's launches (for profilers); prints no bench line")
    ap.add_argument("--bare-backward", action="store_true",
                    help="time only the workload's backward (gradients) and print one short line (for profilers)")
    ap.add_argument("--bare-paged", action="store_true",
                    help="time only the decode workload over a paged cache and print one short line (for profilers)")
    ap.add_argument("--pages-layout", default="head_major", choices=["head_major", "token_major"],
                    help="with --bare-paged: the page pools' layout")
    ap.add_argument("--bare-batch", type=int, default=0,
                    help="with --bare / --bare-paged: use this batch size instead of the workload's "
                         "(smaller profiler captures)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, ws, rank)
        return

    ws, rank, local = dist_setup(args.gpus)
    dist_on = ws > 1
    device = torch.device("cuda", local)
    from scaled_dot_product_15_b200 import load_library

    load_library()
    peaks, peak_src = load_peaks()
    w = W.WORKLOADS[args.workload]
    if args.bare_backward:
        r = measure_backward(w, args.steps, args.warmup, peaks, peak_src, device)
        print(json.dumps({"bare_backward": w.name, "ms_per_step": r["ms_per_step"], "path": r["path"],
                          "launches": r["gpu_launches"]}))
        return
    if args.bare_paged:
        if args.bare_batch:
            import dataclasses

            w = dataclasses.replace(w, B=args.bare_batch)
        r = measure_paged_decode(w, args.steps, args.warmup, peaks, peak_src, device, args.pages_layout)
        print(json.dumps({"bare_paged": w.name, "ms_per_step": r["ms_per_step"], "path": r["path"],
                          "launches": r["gpu_launches"]}))
        return
    if args.bare:
        if args.bare_batch:
            import dataclasses

            w = dataclasses.replace(w, B=args.bare_batch)
        sets, _ = make_sets(w, device)
        calls = prepared_calls(w, sets, device)
        total_ms, kernel_ms, launches = time_device(calls, args.steps, args.warmup, dist_on)
        print(json.dumps({"bare": w.name, "ms_per_step": total_ms / args.steps, "launches": launches}))
        return
    sampler = ClockSampler(local)
    res, total_ms, kernel_ms, launches = measure_workload(w, args.steps, args.warmup, peaks, peak_src, device,
                                                         dist_on, sampler)
    max_ms = max_over_ranks(total_ms, device, dist_on)
    amount, unit, _ = work_units(w)
    value = job_rate(amount, ws, max_ms / args.steps, unit)
    e2e_ms, h2d, d2h = time_e2e(w, [W.make_inputs(w, device)], max(3, args.steps // 10), 3)
    e2e_value = job_rate(amount, ws, max_over_ranks(e2e_ms, device, dist_on), unit)

    extra = {}
    cpu = None
    if rank == 0 and ws == 1 and not args.no_extra:
        for name, ow in W.WORKLOADS.items():
            if name == w.name:
                continue
            try:
                r, *_ = measure_workload(ow, max(20, args.steps // 4), args.warmup, peaks, peak_src, device)
                extra[name] = r
            except Exception as e:  # report, never hide
                extra[name] = {"error": repr(e)}
        if w.mask == "causal" and w.L > 1:
            try:
                extra[w.name + ":backward"] = measure_backward(w, 5, 2, peaks, peak_src, device)
            except Exception as e:
                extra[w.name + ":backward"] = {"error": repr(e)}
        for name, ow in W.WORKLOADS.items():
            if ow.L == 1 and ow.mask == "none" and ow.layout != "packed":
                for lay, tag in (("head_major", ""), ("token_major", "_token_major")):
                    key = name + f":paged{PAGE_SIZE}{tag}"
                    try:
                        extra[key] = measure_paged_decode(ow, max(20, args.steps // 4), args.warmup, peaks,
                                                          peak_src, device, lay)
                    except Exception as e:
                        extra[key] = {"error": repr(e)}
    if rank == 0 and ws == 1:
        cpu = cpu_baseline(w, args.cpu_seconds)

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(value, 3),
            "unit": unit,
            "n_gpus": ws,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(max_ms / args.steps, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": w.dtype.replace("fp", "f").replace("bf16", "bf16"),
            "data": "synthetic: seeded iid N(0,1) inputs",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "L": w.L, "S": w.S, "E": w.E,
                       "Ev": w.Ev, "mask": w.mask, "parallelism": f"independent replicas x{ws}",
                       "l2": res["l2"], "path": res["path"]},
            "roofline": res["roofline"],
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 3), "unit": unit, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "clocks": sampler.summary(),
            "kernel_sha": kernel_source_hash(res["path"]),
            "workloads": extra,
        }
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
