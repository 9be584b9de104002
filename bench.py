#!/usr/bin/env python
"""Benchmark of the fused attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-extra]

A step is one call of the library's attention forward (``attn_fwd``) over one
batch of the workload, inputs resident in HBM.  Steps are timed with CUDA
events on the launching stream; a 256 MiB buffer is rewritten between steps
(outside the events) so every step starts with a cold L2.  Under torchrun each
rank runs the same per-GPU workload (weak scaling, no collective on the data
path); the barrier-bracketed timed region is reduced with MAX over ranks and
rank 0 prints one JSON line.

The default workload is the bf16 causal dot-product prefill (N=4, H=16,
L=S=2048, E=Ev=128); its throughput in TFLOP/s (2*(E+Ev) FLOPs per visible
query/key pair) is `value`.  The other reference workloads are measured too
and reported under "workloads" (TFLOP/s for prefill, KV-read GB/s for decode).

``--impl reference`` runs the reference arm: the float64 CPU oracle, timed on
the host cores on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synth import workloads as sw  # noqa: E402

METRIC = "attn fwd TFLOP/s (prefill), KV-read GB/s (decode), % of B200 roofline"
DEFAULT_WORKLOAD = "dot_causal_2k_bf16"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# fp32 FMA-pipe roofline of the exact-fp32 path: measured FFMA throughput per SM per
# clock on this B200 (a dependent-free FFMA stream, 4 warps per SM) x 2 flops x SMs x
# the maximum SM clock
FFMA_PER_CLK_SM = 122

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the
# dominant kernel from one ncu capture of the same kernel build, with the batch N
# of that capture; the traffic of these kernels grows in proportion to N, so a
# line at another N reports it scaled.  The capture command and counters are in
# profiles/.  Must be reset when the kernel changes.  Keyed by the line's label:
# a variant line (another mask, mode or key selection) has no entry, so null.
NCU_TRAFFIC_BYTES = {
    "dot_causal_2k_bf16": (132_508_416 + 11_135_232, 4),          # prefill_kernel<128,128,dot> (plain variant)
    "dot_causal_2k_bf16:backward": (453_969_920 + 291_908_608, 4),  # bwd_kernel<128,128> (--backward)
    # decode_partial_kernel<128,128>, two consumer groups (a batch-2 capture: 16 GB of cache at batch 32)
    "decode_sink_gqa_128k_bf16": (1_073_873_920 + 3_484_160, 2),
}


# ---------------------------------------------------------------------------
# algorithmic work
# ---------------------------------------------------------------------------

def row_pairs(r: sw.Recipe, rows) -> np.ndarray:
    """Visible keys of each query row in ``rows`` under r's mask kind (a bias does not change it)."""
    ip = np.asarray(rows, dtype=np.int64) + (r.S - r.L)
    if r.mask_kind == "none":
        return np.full(ip.size, r.S, dtype=np.int64)
    hi = np.minimum(r.S, ip + 1)
    if r.mask_kind == "causal":
        return np.maximum(0, hi)
    lo = np.minimum(np.maximum(0, ip - r.window + 1), np.maximum(hi, 0))
    n = np.maximum(0, hi - lo)
    if r.mask_kind == "streaming":
        n = n + np.maximum(0, np.minimum(r.keep, lo))  # kept initial keys below the window
    return n


def visible_pairs(r: sw.Recipe) -> int:
    """Number of (query, key) pairs the mask leaves visible, per (n, hq) (no keep bits or padding)."""
    return int(row_pairs(r, np.arange(r.L)).sum())


def visible_pairs_total(r: sw.Recipe) -> int:
    """Visible (query, key) pairs summed over the batch, per query head: the mask kind,
    then the keep bits and each batch's key padding."""
    ks, ke = sw.kv_ranges(r)
    keep = sw.keep_matrix(r)
    if keep is None and ks is None:
        return r.N * visible_pairs(r)
    ip = np.arange(r.L, dtype=np.int64) + (r.S - r.L)
    hi = np.full(r.L, r.S) if r.mask_kind == "none" else np.minimum(r.S, ip + 1)
    lo = np.maximum(0, ip - r.window + 1) if r.mask_kind == "window" else np.zeros(r.L, dtype=np.int64)
    starts = np.zeros(r.N, dtype=np.int64) if ks is None else ks.astype(np.int64)
    ends = np.full(r.N, r.S) if ke is None else ke.astype(np.int64)
    if keep is None:
        return int(sum(np.maximum(0, np.minimum(hi, e) - np.maximum(lo, b)).sum() for b, e in zip(starts, ends)))
    j = np.arange(r.S)[None, :]
    vis = keep & (j >= lo[:, None]) & (j < hi[:, None])
    csum = np.concatenate([np.zeros((r.L, 1), dtype=np.int64), np.cumsum(vis, axis=1)], axis=1)
    return int(sum((csum[:, e] - csum[:, b]).sum() for b, e in zip(starts, ends)))


def is_decode(r: sw.Recipe) -> bool:
    return r.dtype == "bf16" and (r.Hq // r.H) * r.L <= 16


def decode_keys(r: sw.Recipe) -> int:
    """Keys some query row can see: what a decode step has to read from the cache."""
    if r.mask_kind in ("none", "causal"):
        return r.S
    ip = np.arange(r.L, dtype=np.int64)[:, None] + (r.S - r.L)
    j = np.arange(r.S, dtype=np.int64)[None, :]
    d = ip - j
    seen = (d >= 0) & (d < r.window)
    if r.mask_kind == "streaming":
        seen |= (d >= 0) & (j < r.keep)
    return int(seen.any(axis=0).sum())


def work_units(r: sw.Recipe):
    """(amount, unit, roofline bound) of one step of workload r on one GPU."""
    if r.n_sel > 0:
        # listed-key decode: the gathered K and V rows plus the key lists themselves
        return r.N * r.H * r.n_sel * ((r.E + r.Ev) * 2 + 4), "GB/s", "hbm"
    if is_decode(r):
        kv_bytes = r.N * r.H * decode_keys(r) * (r.E + r.Ev) * 2
        return kv_bytes, "GB/s", "hbm"
    if r.backward:
        # S^T, dP^T, dV, dK and dQ products: 2 (3E + 2Ev) flops per visible pair
        return 2 * (3 * r.E + 2 * r.Ev) * visible_pairs_total(r) * r.Hq, "TFLOP/s", "tensor"
    if r.dtype == "f32":
        # exact fp32 on the FMA pipe; a bias mask cannot skip work, so its pairs are counted
        pairs = r.N * visible_pairs(r) if r.bias != "none" else visible_pairs_total(r)
        return 2 * (r.E + r.Ev) * pairs * r.Hq, "TFLOP/s", "fma"
    flops = 2 * (r.E + r.Ev) * visible_pairs_total(r) * r.Hq
    return flops, "TFLOP/s", "tensor"


def rate(amount: float, seconds: float, unit: str) -> float:
    return amount / seconds / (1e12 if unit == "TFLOP/s" else 1e9)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# clocks (NVML, read only)
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {
        0x0000000000000008: "hw_slowdown",
        0x0000000000000040: "hw_thermal_slowdown",
        0x0000000000000020: "sw_thermal_slowdown",
        0x0000000000000004: "sw_power_cap",
        0x0000000000000080: "hw_power_brake_slowdown",
    }

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001
            self.nvml = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
                mask = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml is not None:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.nvml is not None:
            self.t.join()

    def summary(self):
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def max_sm_mhz(device_index: int = 0) -> int:
    """The GPU's maximum SM clock (NVML, read only); 1965 MHz, the B200's, if NVML is unavailable."""
    try:
        import pynvml
        pynvml.nvmlInit()
        return int(pynvml.nvmlDeviceGetMaxClockInfo(pynvml.nvmlDeviceGetHandleByIndex(device_index),
                                                    pynvml.NVML_CLOCK_SM))
    except Exception:  # noqa: BLE001
        return 1965


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    return world, rank, local, pg


def barrier(pg):
    if pg is not None:
        pg.barrier()


def max_over_ranks(pg, value: float, device: str = "cuda") -> float:
    """Largest value over all ranks (the job's time is its slowest rank's)."""
    if pg is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_rate(amount_per_rank: float, world: int, secs_max: float, steps: int, unit: str) -> float:
    """Whole-job throughput: every rank runs its own full batch (weak scaling),
    so the work is world x per-rank work over the slowest rank's time."""
    return rate(amount_per_rank * world, secs_max / steps, unit)


def time_device(fn, steps, warmup, flush_buf, stream):
    """Sum of per-step CUDA-event times (seconds); L2 flushed before every step."""
    import torch
    for _ in range(warmup):
        flush_buf.fill_(1.0)
        fn()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for k in range(steps):
        flush_buf.fill_(float(k))
        starts[k].record(stream)
        fn()
        ends[k].record(stream)
    torch.cuda.synchronize()
    return sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / 1e3


def run_workload(name, steps, warmup, pg, flush_buf, peaks, peak_kind, clocks=False, label=None):
    import torch

    import attention_tiled_attn_b200 as attn
    from synth import gpu as sgpu

    r = sw.RECIPES[name]
    t = sgpu.generate_on_device(r)
    out = torch.empty((r.N, r.Hq, r.L, r.Ev), dtype=t["q"].dtype, device="cuda")
    lse = torch.empty((r.N, r.Hq, r.L), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    masks = dict(keep_first=r.keep, mask_bits=t["mask_bits"], kv_start=t["kv_start"], kv_end=t["kv_end"])
    if r.backward:
        # the forward's output and lse, and a seeded dout, are inputs of the timed backward
        attn.attn_fwd(t["q"], t["k"], t["v"], scale=r.scale, mode=r.mode, sink=t["sink"], mask_kind=r.mask_kind,
                      window=r.window, out=out, lse=lse, stream=stream, **masks)
        dout = torch.empty_like(out)
        sgpu.normal_into(dout, sw.stream_key(r.seed, sw.STREAM_DOUT))

    def step():
        if r.backward:
            attn.attn_bwd(t["q"], t["k"], t["v"], out, lse, dout, scale=r.scale, mode=r.mode, sink=t["sink"],
                          mask_kind=r.mask_kind, window=r.window, stream=stream, **masks)
            return
        if r.n_sel > 0:
            attn.attn_decode_indexed(t["q"], t["k"], t["v"], t["key_idx"], scale=r.scale, sink=t["sink"],
                                     mask_kind=r.mask_kind, window=r.window, bias=t["bias"], out=out, lse=lse,
                                     stream=stream)
            return
        attn.attn_fwd(t["q"], t["k"], t["v"], scale=r.scale, mode=r.mode, sink=t["sink"], mask_kind=r.mask_kind,
                      window=r.window, keep_first=r.keep, bias=t["bias"], out=out, lse=lse, stream=stream,
                      mask_bits=t["mask_bits"], kv_start=t["kv_start"], kv_end=t["kv_end"])

    amount, unit, bound = work_units(r)
    barrier(pg)
    torch.cuda.synchronize()
    sampler = ClockSampler(torch.cuda.current_device()) if clocks else None
    if sampler:
        sampler.__enter__()
    secs = time_device(step, steps, warmup, flush_buf, stream)
    if sampler:
        sampler.__exit__()
    torch.cuda.synchronize()
    barrier(pg)
    secs_max = max_over_ranks(pg, secs)
    status = attn.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after {name}")
    per_launch = secs / steps
    achieved = rate(amount, per_launch, unit)
    if bound == "tensor":
        peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        punit = "TFLOP/s"
    elif bound == "fma":
        props = torch.cuda.get_device_properties(torch.cuda.current_device())
        max_mhz = (sampler.max_mhz if sampler and sampler.max_mhz else None) or max_sm_mhz()
        peak = round(FFMA_PER_CLK_SM * 2 * props.multi_processor_count * max_mhz * 1e6 / 1e12, 2)
        punit = "TFLOP/s"
    else:
        peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        punit = "GB/s"
    key = label or (name + (":backward" if r.backward else "") + (f":select{r.n_sel}" if r.n_sel > 0 else ""))
    traffic = None
    if key in NCU_TRAFFIC_BYTES:
        t_bytes, t_n = NCU_TRAFFIC_BYTES[key]
        traffic = t_bytes * r.N // t_n
    res = {
        "recipe": r, "amount": amount, "unit": unit, "secs_max": secs_max, "secs": secs,
        "roofline": {"bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": punit,
                     "frac": round(achieved / peak, 4), "traffic": traffic,
                     "peak_source": ("derived: FFMA/clk/SM x 2 x SMs x max SM clock" if bound == "fma" else
                                     f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback")},
        # this library's kernels per step: backward = pre-pass + main; a bf16 prefill with a float
        # bias = keep-bit pre-pass + prefill; decode (combine fused) and the rest = one
        "launches_per_step": 2 if (r.backward or (r.bias != "none" and r.dtype == "bf16" and not is_decode(r)
                                                   and r.n_sel == 0 and r.mask_kind != "streaming")) else 1,
        "clocks": sampler.summary() if sampler else None,
        "tensors": t, "out": out, "lse": lse, "dout": dout if r.backward else None,
    }
    return res


def e2e_measure(res, steps, warmup):
    """Same metric through the public API with pinned host buffers: every step copies
    its inputs host->device, runs attn_fwd and reads the output back.  Steps are
    pipelined the way a caller streaming batches would run them: the host->device
    copies on one stream, the calls in order on another (they share the library's
    workspace), the device->host copies on a third, with two device copies of the
    inputs and outputs so that step k's input copy and step k-1's output copy overlap
    step k-1's and step k's compute."""
    import torch

    import attention_tiled_attn_b200 as attn
    r = res["recipe"]
    t = res["tensors"]
    if r.backward:
        return e2e_backward(res, steps, warmup)
    names = ("q", "k", "v", "key_idx") if r.n_sel > 0 else ("q", "k", "v")
    host = {k: t[k].cpu().pin_memory() for k in names}
    dev = [{k: torch.empty_like(t[k]) for k in names} for _ in range(2)]
    outs = [(torch.empty_like(res["out"]), torch.empty_like(res["lse"])) for _ in range(2)]
    out_host = [torch.empty(res["out"].shape, dtype=res["out"].dtype).pin_memory() for _ in range(2)]
    lse_host = [torch.empty(res["lse"].shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    h2d = sum(host[k].numel() * host[k].element_size() for k in host)
    d2h = out_host[0].numel() * out_host[0].element_size() + lse_host[0].numel() * 4
    ev = lambda: torch.cuda.Event()  # noqa: E731
    ran = [None, None]   # compute of the step that last used buffer set i (its inputs may be overwritten after)
    read = [None, None]  # output copy of the step that last used buffer set i (its outputs may be overwritten after)

    def step(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if ran[b] is not None:
                s_in.wait_event(ran[b])
            for k in names:
                dev[b][k].copy_(host[k], non_blocking=True)
            landed = ev()
            landed.record(s_in)
        with torch.cuda.stream(s_run):
            s_run.wait_event(landed)
            if read[b] is not None:
                s_run.wait_event(read[b])
            o, l = outs[b]
            if r.n_sel > 0:
                attn.attn_decode_indexed(dev[b]["q"], dev[b]["k"], dev[b]["v"], dev[b]["key_idx"], scale=r.scale,
                                         sink=t["sink"], mask_kind=r.mask_kind, window=r.window, bias=t["bias"],
                                         out=o, lse=l, stream=s_run)
            else:
                attn.attn_fwd(dev[b]["q"], dev[b]["k"], dev[b]["v"], scale=r.scale, mode=r.mode, sink=t["sink"],
                              mask_kind=r.mask_kind, window=r.window, keep_first=r.keep, bias=t["bias"], out=o,
                              lse=l, stream=s_run, mask_bits=t["mask_bits"], kv_start=t["kv_start"],
                              kv_end=t["kv_end"])
            ran[b] = ev()
            ran[b].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ran[b])
            out_host[b].copy_(o, non_blocking=True)
            lse_host[b].copy_(l, non_blocking=True)
            read[b] = ev()
            read[b].record(s_out)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    z = torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    s_run.wait_event(a)
    s_out.wait_event(a)
    for i in range(steps):
        step(i)
    s_in.wait_stream(s_run)
    s_in.wait_stream(s_out)
    z.record(s_in)
    torch.cuda.synchronize()
    secs = a.elapsed_time(z) / 1e3
    for k in list(host):
        del host[k]
    return {"value": round(rate(res["amount"], secs / steps, res["unit"]), 3), "unit": res["unit"],
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}, secs


def e2e_backward(res, steps, warmup):
    """The backward through the public API with pinned host buffers: every step copies
    q, k, v, out, lse and dout host->device, runs attn_bwd and reads dq, dk, dv back."""
    import torch

    import attention_tiled_attn_b200 as attn
    r = res["recipe"]
    t = res["tensors"]
    src = {"q": t["q"], "k": t["k"], "v": t["v"], "out": res["out"], "lse": res["lse"], "dout": res["dout"]}
    host = {k: x.cpu().pin_memory() for k, x in src.items()}
    dev = {k: torch.empty_like(x) for k, x in src.items()}
    stream = torch.cuda.current_stream()
    h2d = sum(x.numel() * x.element_size() for x in host.values())
    outs_host = None

    def step():
        nonlocal outs_host
        for k in host:
            dev[k].copy_(host[k], non_blocking=True)
        g = attn.attn_bwd(dev["q"], dev["k"], dev["v"], dev["out"], dev["lse"], dev["dout"], scale=r.scale,
                          mode=r.mode, sink=t["sink"], mask_kind=r.mask_kind, window=r.window, stream=stream,
                          keep_first=r.keep, mask_bits=t["mask_bits"], kv_start=t["kv_start"], kv_end=t["kv_end"])
        if outs_host is None:
            outs_host = [torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in g[:3]]
        for hbuf, x in zip(outs_host, g[:3]):
            hbuf.copy_(x, non_blocking=True)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    secs = a.elapsed_time(b) / 1e3
    d2h = sum(x.numel() * x.element_size() for x in outs_host)
    return {"value": round(rate(res["amount"], secs / steps, res["unit"]), 3), "unit": res["unit"],
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}, secs


def _oracle_cores():
    try:
        from threadpoolctl import threadpool_info
        return int(max([i.get("num_threads", 1) for i in threadpool_info()] + [1]))
    except Exception:  # noqa: BLE001
        return int(os.cpu_count() or 1)


class OracleSample:
    """Runs the float64 oracle (as it stands) on row blocks of one (n, hq) head
    of workload r, and converts the time into the workload's unit."""

    def __init__(self, r: sw.Recipe, n: int = 0, hq: int = 0, key_idx=None):
        from oracle import attention as orc
        self.orc, self.r, self.hq = orc, r, hq
        kvh = hq // r.group
        if r.n_sel > 0:  # the unit's key list (key_idx: the workload's lists, when already drawn)
            self.key_list = (sw.key_index_set(r) if key_idx is None else key_idx)[n, kvh]
        self.q = sw.tensor_slice_f64(r, "q", n, hq)
        self.k = sw.tensor_slice_f64(r, "k", n, kvh)
        self.v = sw.tensor_slice_f64(r, "v", n, kvh)
        s = sw.sink_logits(r)
        self.sink = None if s is None else float(s[hq])
        self.bias = sw.bias_matrix(r)
        amount, self.unit, _ = work_units(r)
        self.per_pair = amount / (r.N * r.Hq * max(1, visible_pairs(r)))

    def rows_amount(self, rows):
        r = self.r
        if r.backward:
            return work_units(r)[0] / (r.N * r.Hq) * rows.size / r.L
        if r.n_sel > 0:
            return work_units(r)[0] / (r.N * r.Hq) * rows.size / r.L
        return float(row_pairs(r, rows).sum()) * self.per_pair

    def run(self, rows):
        r = self.r
        if r.backward:
            # the oracle backward of this head (all L rows; it recomputes its forward); dout: seeded draws
            dout = np.random.default_rng(self.hq).standard_normal((1, 1, r.L, r.Ev))
            self.orc.attention_backward(self.q[None, None], self.k[None, None], self.v[None, None], dout,
                                        scale=r.scale, mode=r.mode,
                                        sink=None if self.sink is None else np.array([self.sink]),
                                        mask_kind=r.mask_kind, window=r.window, keep=r.keep)
            return self.rows_amount(np.arange(r.L))
        if r.n_sel > 0:
            # the index-set oracle on this head's L rows (decode: L is small); rows counts the work done
            self.orc.attention_over_index_set(
                self.q[None, None], self.k[None, None], self.v[None, None], self.key_list[None, None],
                scale=r.scale, sink=None if self.sink is None else np.array([self.sink]), mask_kind=r.mask_kind,
                window=r.window, bias=self.bias)
            return self.rows_amount(np.arange(r.L))
        for i0 in range(0, rows.size, 256):
            rr = rows[i0:i0 + 256]
            self.orc.attend_rows(self.q[rr], rr, self.k, self.v, r.L, scale=r.scale, mode=r.mode, sink=self.sink,
                                 mask_kind=r.mask_kind, window=r.window, keep=r.keep,
                                 bias_rows=None if self.bias is None else self.bias[rr])
        return self.rows_amount(rows)


def cpu_baseline(r: sw.Recipe, budget_s: float = 12.0, wall_limit_s: float = 40.0):
    """Oracle throughput on the host cores over a bounded sample: 256-row
    blocks of successive (n, hq) heads, last rows first (the heaviest under a
    causal mask), until budget_s of oracle compute or wall_limit_s of wall
    time (input regeneration included) is spent.  The rate counts compute
    time only."""
    done, secs, blocks, heads = 0.0, 0.0, 0, 0
    unit = work_units(r)[1]
    t_start = time.perf_counter()
    key_idx = sw.key_index_set(r)
    stop = False
    for n in range(r.N):
        for hq in range(r.Hq):
            smp = OracleSample(r, n, hq, key_idx)
            heads += 1
            for i1 in (range(r.L, 0, -r.L) if r.backward else range(r.L, 0, -256)):
                rows = np.arange(max(0, i1 - 256), i1)
                t0 = time.perf_counter()
                done += smp.run(rows)
                secs += time.perf_counter() - t0
                blocks += 1
                if secs > budget_s or time.perf_counter() - t_start > wall_limit_s:
                    stop = True
                    break
            if stop or time.perf_counter() - t_start > wall_limit_s:
                stop = True
                break
        if stop:
            break
    return {"value": round(rate(done, secs, unit), 6), "unit": unit, "cores": _oracle_cores(), "kind": "oracle",
            "sample": f"{blocks} x 256-row blocks from {heads} (n, hq) heads of {r.name} "
                      f"({secs:.1f} s of float64 numpy compute)"}


def ours(args):
    import torch
    world, rank, local, pg = dist_setup(args)
    peaks, peak_kind = load_peaks()
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    main = run_workload(args.workload, args.steps, args.warmup, pg, flush, peaks, peak_kind, clocks=True)
    r = main["recipe"]
    e2e, _ = e2e_measure(main, max(3, min(args.steps, 20)), 2)
    extra = {}
    if not args.no_extra:
        import dataclasses
        # every reference workload but the tiny fp32 parity case
        names = [n for n in sw.RECIPES if n != args.workload and n != "tiny_rbf_sink_causal_f32"]
        runs = []
        # steady-state control: the bench workload's kernel (dot, E=128) on one long
        # non-causal sequence, where per-item pipeline fill and drain are amortised
        base = sw.RECIPES[args.workload]
        if base.mode == "dot" and base.dtype == "bf16" and not is_decode(base):
            runs.append((args.workload + ":steady_state_noncausal_8k",
                         dataclasses.replace(base, N=1, L=8192, S=8192, mask_kind="none")))
            # a 10% random 0/-inf mask as packed keep bits and as the fp32 bias; ragged left padding
            runs.append((args.workload + ":keep_bits_random10", dataclasses.replace(base, keep_mask="random10")))
            runs.append((args.workload + ":bias_random10", dataclasses.replace(base, bias="random10")))
            runs.append((args.workload + ":left_pad_upto50", dataclasses.replace(base, pad_left=0.5)))
            runs.append((args.workload + ":backward", dataclasses.replace(base, backward=True)))
        for name in names:
            r0 = sw.RECIPES[name]
            runs.append((name, r0))
            # controls for the "RBF / sink within 10% of plain dot" comparison: same shapes and data
            if r0.mode == "rbf":
                runs.append((name + ":dot_control", dataclasses.replace(r0, mode="dot")))
                runs.append((name + ":backward", dataclasses.replace(r0, backward=True)))
            if r0.sink != "none":
                runs.append((name + ":no_sink_control", dataclasses.replace(r0, sink="none")))
            # the backward of the sink + GQA window workload (a 64-wide head dimension, groups of 8)
            if r0.mask_kind == "window" and not is_decode(r0):
                runs.append((name + ":backward", dataclasses.replace(r0, backward=True)))
            # StreamingLLM variant: 4 kept initial tokens plus the window (decode: a 4096-key window)
            if r0.mask_kind == "window":
                runs.append((name + ":streaming_keep4", dataclasses.replace(r0, mask_kind="streaming", keep=4)))
            elif is_decode(r0):
                runs.append((name + ":streaming_keep4_w4096",
                             dataclasses.replace(r0, mask_kind="streaming", window=4096, keep=4)))
                # exact attention over a 33x-sparse key selection (S/33 keys per KV head, random positions)
                runs.append((name + ":top_k_33x", dataclasses.replace(r0, n_sel=r0.S // 33)))
                # the RBF score on the same cache (key norms in the consumer warps), and one sequence
                # (N=1: 8 KV heads, each split over ~18 CTAs, so the combine merges many partials)
                runs.append((name + ":rbf", dataclasses.replace(r0, mode="rbf")))
                runs.append((name + ":batch1", dataclasses.replace(r0, N=1)))
        for label, rr in runs:
            base = sw.RECIPES[rr.name]
            sw.RECIPES[rr.name] = rr
            try:
                k = max(5, args.steps // 4)
                res = run_workload(rr.name, k, args.warmup, pg, flush, peaks, peak_kind, label=label)
            finally:
                sw.RECIPES[rr.name] = base
            extra[label] = {
                "value": round(job_rate(res["amount"], world, res["secs_max"], k, res["unit"]), 2),
                "unit": res["unit"], "ms_per_step": round(res["secs_max"] / k * 1e3, 4),
                "roofline_frac": res["roofline"]["frac"], "bound": res["roofline"]["bound"],
                "mode": rr.mode, "sink": rr.sink != "none", "mask": rr.mask_kind,
                **({"keys_listed_per_kv_head": rr.n_sel} if rr.n_sel > 0 else {}),
            }
            del res
            torch.cuda.empty_cache()
        for label in list(extra):
            if ":" in label:
                continue
            for ctl in (label + ":dot_control", label + ":no_sink_control"):
                if ctl in extra:
                    extra[label]["time_vs_" + ctl.split(":")[1]] = round(
                        extra[label]["ms_per_step"] / extra[ctl]["ms_per_step"], 4)
            if label + ":keep_bits_random10" in extra and label + ":bias_random10" in extra:
                extra[label + ":keep_bits_random10"]["time_vs_bias"] = round(
                    extra[label + ":keep_bits_random10"]["ms_per_step"] / extra[label + ":bias_random10"]["ms_per_step"],
                    4)
            if label + ":rbf" in extra and extra[label]["mode"] == "dot":
                extra[label + ":rbf"]["time_vs_dot"] = round(
                    extra[label + ":rbf"]["ms_per_step"] / extra[label]["ms_per_step"], 4)
            if label + ":top_k_33x" in extra:
                extra[label + ":top_k_33x"]["time_vs_dense"] = round(
                    extra[label + ":top_k_33x"]["ms_per_step"] / extra[label]["ms_per_step"], 4)
    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(job_rate(main["amount"], world, main["secs_max"], args.steps, main["unit"]), 3),
            "unit": main["unit"],
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(main["secs_max"] / args.steps * 1e3, 5),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16" if r.dtype == "bf16" else "f32",
            "data": "synthetic (seeded counter-based N(0,1) draws, see synth/workloads.py)",
            "config": {"workload": r.name, **({"keys_listed_per_kv_head": r.n_sel} if r.n_sel > 0 else {}),
                       "N": r.N, "Hq": r.Hq, "H": r.H, "L": r.L, "S": r.S, "E": r.E,
                       "Ev": r.Ev, "mode": r.mode, "mask": r.mask_kind, "window": r.window,
                       "sink": r.sink != "none", "scale": r.scale,
                       "parallelism": f"replicas x{world} (independent batches, no collective)",
                       "l2": "flushed: 256 MiB rewritten between timed steps, outside the events"},
            "roofline": main["roofline"],
            "cpu_baseline": cpu_baseline(r) if world == 1 else None,
            "e2e": e2e,
            "gpu_launches": main["launches_per_step"] * args.steps,
            "clocks": main["clocks"],
            "impl": "ours",
            "workloads": extra,
        }
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


# ---------------------------------------------------------------------------
# reference arm: the float64 oracle on the host cores
# ---------------------------------------------------------------------------

def reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    r = sw.RECIPES[args.workload]
    smp = OracleSample(r)
    # calibrate the per-step sample so that warmup + steps take ~90 s in total
    cal = np.arange(max(0, r.L - 64), r.L)
    t0 = time.perf_counter()
    smp.run(cal)
    per_row = (time.perf_counter() - t0) / cal.size
    rows_per_step = int(min(r.L, max(8, 90.0 / (args.steps + args.warmup) / max(per_row, 1e-9))))
    rows = np.arange(r.L - rows_per_step, r.L)
    for _ in range(args.warmup):
        smp.run(rows)
    done = 0.0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        done += smp.run(rows)
    secs = time.perf_counter() - t0
    value = rate(done, secs, smp.unit)
    sample = f"last {rows_per_step} rows of head (n=0, hq=0) of {r.name} per step, float64 numpy oracle"
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": smp.unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": r.name, **({"keys_listed_per_kv_head": r.n_sel} if r.n_sel > 0 else {}),
                   "N": r.N, "Hq": r.Hq, "H": r.H, "L": r.L, "S": r.S, "E": r.E,
                   "Ev": r.Ev, "mode": r.mode, "mask": r.mask_kind},
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 6), "unit": smp.unit, "cores": _oracle_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": smp.unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(sw.RECIPES))
    ap.add_argument("--no-extra", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch N (profiling captures of a smaller case)")
    ap.add_argument("--backward", action="store_true",
                    help="measure the backward pass (attn_bwd) of the workload instead of its forward")
    ap.add_argument("--select", type=int, default=None, metavar="K",
                    help="decode workloads: attend over K listed keys per KV head (attn_decode_indexed), "
                         "a random K-subset of the cache")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    import dataclasses
    if args.batch is not None:
        sw.RECIPES[args.workload] = dataclasses.replace(sw.RECIPES[args.workload], N=args.batch)
    if args.backward:
        rr = sw.RECIPES[args.workload]
        if rr.dtype != "bf16" or rr.bias != "none":
            raise SystemExit("--backward needs a bf16 workload without a bias")
        sw.RECIPES[args.workload] = dataclasses.replace(rr, backward=True)
    if args.select is not None:
        rr = sw.RECIPES[args.workload]
        if args.select < 1 or not is_decode(rr):
            raise SystemExit("--select needs K >= 1 and a decode-shaped bf16 workload")
        sw.RECIPES[args.workload] = dataclasses.replace(rr, n_sel=args.select)
    if args.impl == "reference":
        reference(args)
    else:
        ours(args)


if __name__ == "__main__":
    main()
