#!/usr/bin/env python
"""Benchmark of libg2attn on B200: useful attention TFLOP/s (prefill) and KV GB/s (decode).

One step = one pass of the prefill hot path over the 9B-shaped batched layer
pair (B=2, T=S=8192, H=16, Hkv=8, d=256, query_scale 1/16, softcap 50), the
largest single-GPU workload: the local layer (window 4096) and the global
layer, both through the C ABI. Useful FLOPs count 4*d per visible (query,
key, head) triple only. Inputs live in HBM; the L2 is flushed (a 512 MiB
write) between timed steps, outside the timed events.

Printed (rank 0, one JSON line): the contract keys, plus
  roofline      dominant kernel (prefill_fwd_sm100<256,2>, the CTA-pair kernel
                that d = 256 runs on) vs measured bf16 peak
  cpu_baseline  the fp64 oracle on the host cores: a bounded row sample of the
                step's workload, one thread on the tiny pair, the 27B decode
                (KV GB/s, tokens/s), the host's CPU model and core counts
  e2e           the same metric with pinned-host inputs and outputs copied
                inside the timed region
  clocks        nvidia-smi samples taken during the timed region
  layers        per-layer times of the step
  extra         2B pair, 27B decode (KV GB/s, tokens/s; linear, ring and paged
                caches), the 9B ragged varlen prefill (packed and paged K/V),
                the Gemma 3-shaped variant of the 2B pair (window 1024, no cap)
                and the gradients of the 27B-shaped pair (dense and as a packed
                batch of 8 sequences) and of the 2B-shaped pair at d = 256
                (useful backward TFLOP/s)

`--impl reference` times the fp64 oracle (the reference arm of this build)
on the host cores on bounded samples of the same workload.
Multi-GPU (torchrun): every rank runs its own replica (the units are
independent; there is no data-path collective); value = total useful FLOPs
of all ranks / max-over-ranks device time ("scaling": "weak"). `--gpus N`
must equal the launcher's WORLD_SIZE (1 without torchrun); otherwise the run
stops with an error instead of printing a line for another N.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from global_soft_capped_b200.inputs import (  # noqa: E402
    WORKLOADS, backward_inputs, decode_inputs, prefill_inputs, varlen_backward_inputs,
    varlen_inputs)

METRIC = "useful attention TFLOP/s (prefill) and KV GB/s (decode) vs B200 roofline"
WORKLOAD = "9b"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# work counts (host arithmetic on sizes only)
# ---------------------------------------------------------------------------
def visible_pairs(T, S, q_offset, window):
    """Number of visible (query row, key) pairs of one (batch, head)."""
    p = np.arange(T, dtype=np.int64) + q_offset
    hi = np.minimum(p, S - 1)
    lo = np.maximum(0, p - window + 1) if window > 0 else np.zeros_like(p)
    return int(np.sum(hi - lo + 1))


def prefill_flops(B, T, S, H, d, q_offset, window):
    return 4.0 * d * H * B * visible_pairs(T, S, q_offset, window)


def backward_flops(B, T, S, H, d, q_offset, window):
    """Useful FLOPs of the gradients: the five products S, dP, dV, dK, dQ,
    2d each, per visible (query, key, head) triple (2.5 x the forward)."""
    return 2.5 * prefill_flops(B, T, S, H, d, q_offset, window)


def varlen_flops(Ts, Ss, H, d, window):
    return sum(4.0 * d * H * visible_pairs(t, s, s - t, window) for t, s in zip(Ts, Ss))


def decode_kv_bytes(lengths, Hkv, d, window):
    rows = sum(min(L, window) if window > 0 else L for L in lengths)
    return rows * Hkv * d * 2 * 2  # K and V, bf16


def headline_config(world):
    """The `config` object of the bench line (identical in both arms)."""
    w = WORKLOADS[WORKLOAD]
    return {"workload": f"{WORKLOAD}_prefill_pair", "B": w.B, "T": w.T, "S": w.S, "H": w.H,
            "Hkv": w.Hkv, "d": w.d, "window_local": w.window_local,
            "query_scale": w.query_scale, "softcap": w.softcap,
            "global_batch": w.B * world, "seq_len": w.T,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "inputs (256 MiB) larger than L2; also flushed between steps by a 512 MiB "
                  "write outside the timed events"}


def step_flops_of(w):
    return sum(prefill_flops(w.B, w.T, w.S, w.H, w.d, 0, win) for win in (w.window_local, 0))


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return p, "measured"
    return PEAKS_FALLBACK, "fallback"


# CTA-group size of the d = 256 prefill kernel the library launches (pairs
# unless G2ATTN_PREFILL_PAIR=0 selects the single-CTA kernel).
KERNEL_CG = 1 if os.environ.get("G2ATTN_PREFILL_PAIR", "1").startswith("0") else 2


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("prefill_sm100.cuh", "common.cuh"):
        h.update(open(os.path.join(ROOT, "global_soft_capped_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key, units_now):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, scaled by units processed; None if the kernel source changed."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    try:
        rec = json.load(open(path)).get(kernel_key)
    except Exception:
        return None
    if not rec or rec.get("source_hash") != kernel_source_hash():
        return None
    return rec["bytes_per_launch"] * units_now / rec["units"]


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock, power and clock-event reasons sampled through NVML every 2 ms
    by a background thread; stop() keeps the samples taken inside the timed
    region (mark_begin / mark_end). Falls back to nvidia-smi at 100 ms."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device):
        self.device = device
        self.dev = device.index if device.index is not None else 0
        self.proc = None
        self.thread = None
        self.samples = []
        self.t0 = self.t1 = None
        self.path = os.path.join("/tmp", f"g2attn_clocks_{os.getpid()}.csv")

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.dev)

    def start(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.stop_flag = False
            get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons",
                                  getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons", None))

            def run():
                while not self.stop_flag:
                    t = time.perf_counter()
                    try:
                        sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                        rs = int(get_reasons(h)) if get_reasons else 0
                        self.samples.append((t, sm, pw, rs))
                    except Exception:
                        pass
                    time.sleep(0.002)
            self.thread = threading.Thread(target=run, daemon=True)
            self.thread.start()
            time.sleep(0.02)  # the sampler is running before the timed region starts
            return
        except Exception:
            self.thread = None
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def mark_begin(self):
        self.t0 = time.perf_counter()

    def mark_end(self):
        self.t1 = time.perf_counter()

    def stop(self):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=5)
            inside = [x for x in self.samples if self.t0 is not None and self.t0 <= x[0] <= self.t1]
            reasons = sorted({n for x in inside for bit, n in self.REASONS.items() if x[3] & bit})
            sms = [x[1] for x in inside]
            return {"sm_mhz": statistics.median(sms) if sms else None, "sm_max_mhz": self.max_mhz,
                    "sm_mhz_min": min(sms) if sms else None,
                    "power_w_median": round(statistics.median([x[2] for x in inside]), 1) if inside else None,
                    "samples_in_timed_region": len(inside), "sampler": "NVML every 2 ms",
                    "reasons": reasons}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock sampling unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sms, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm = float(parts[1])
                mx = float(parts[2])
                pw = float(parts[3]) if parts[3] not in ("[N/A]", "N/A") else 0.0
            except ValueError:
                continue
            if pw > 150.0:  # under load
                sms.append(sm)
            for n, flag in zip(names, parts[5:9]):
                if flag.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sms) if sms else None, "sm_max_mhz": mx,
                "samples_under_load": len(sms), "sampler": "nvidia-smi every 100 ms",
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def aggregate_over_ranks(total_ms, nsteps, step_flops, world, device):
    """Whole-job numbers of a replica run: every rank ran nsteps steps of
    step_flops each; the job time is the slowest rank's device time (max over
    ranks, one all-reduce). Returns (ms per step, TFLOP/s of all ranks)."""
    t = torch.tensor([float(total_ms)], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    ms_per_step = float(t.item()) / nsteps
    return ms_per_step, step_flops * world / (ms_per_step * 1e-3) / 1e12


def replica_seed(base_seed, rank):
    """Each replica draws its own inputs (independent units, no exchange)."""
    return base_seed + rank


def run_ours(args, rank, world, dev):
    import global_soft_capped_b200 as g2
    g2.load_library()
    w = WORKLOADS[WORKLOAD]
    q, k, v = prefill_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d, w.std, replica_seed(w.seed, rank))
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    outs = {lay: torch.empty_like(qd) for lay in ("local", "global")}
    lses = {lay: torch.empty((w.B, w.H, w.T), dtype=torch.float32, device=dev)
            for lay in ("local", "global")}
    windows = {"local": w.window_local, "global": 0}
    flops = {lay: prefill_flops(w.B, w.T, w.S, w.H, w.d, 0, windows[lay]) for lay in windows}
    step_flops = sum(flops.values())
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def layer(lay):
        g2.prefill(qd, kd, vd, query_scale=w.query_scale, softcap=w.softcap,
                   window=windows[lay], out=outs[lay], lse=lses[lay], stream=stream)

    for _ in range(args.warmup):
        layer("local")
        layer("global")
    torch.cuda.synchronize()

    nsteps = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nsteps)]
    clocks = ClockSampler(dev)
    clocks.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.mark_begin()
    t_wall = time.perf_counter()
    for i in range(nsteps):
        flush.zero_()
        ev[i][0].record(stream)
        layer("local")
        ev[i][1].record(stream)
        layer("global")
        ev[i][2].record(stream)
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    clocks.mark_end()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    loc = [ev[i][0].elapsed_time(ev[i][1]) for i in range(nsteps)]
    glo = [ev[i][1].elapsed_time(ev[i][2]) for i in range(nsteps)]
    total_ms = sum(loc) + sum(glo)
    ms_per_step, value = aggregate_over_ranks(total_ms, nsteps, step_flops, world, dev)

    pk, pk_kind = peaks()
    avg_loc, avg_glo = sum(loc) / nsteps, sum(glo) / nsteps
    ach = (flops["local"] + flops["global"]) / ((avg_loc + avg_glo) * 1e-3) / 1e12
    compulsory = 2 * (q.numel() + k.numel() + v.numel() + q.numel())
    roof = {"kernel": f"prefill_fwd_sm100<256,{KERNEL_CG}>", "bound": "tensor", "achieved": round(ach, 2),
            "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "frac": round(ach / pk["bf16_tflops"], 4),
            "peak_kind": f"{pk_kind} bf16 dense (burst; kernel timed alone)",
            "traffic": ncu_traffic(f"prefill_fwd_sm100<256,{KERNEL_CG}>/{WORKLOAD}_pair", 1.0),
            "traffic_unit": "bytes per launch (mean of the local and global launch)",
            "algorithmic": f"4*d*H*B per visible (query,key) pair; {step_flops / 1e12:.4f} TFLOP "
                           f"per step (two launches); compulsory bytes Q+K+V+O = {compulsory} "
                           f"per launch"}

    result = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": nsteps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded iid N(0,1) bf16)",
        "config": headline_config(world),
        "gpu_launches": 2 * nsteps,
        "wall_s_timed_region": round(t_wall, 3),
        "roofline": roof,
        "clocks": clk,
        "layers": {"local": {"ms": round(avg_loc, 5),
                             "tflops": round(flops["local"] / (avg_loc * 1e-3) / 1e12, 2)},
                   "global": {"ms": round(avg_glo, 5),
                              "tflops": round(flops["global"] / (avg_glo * 1e-3) / 1e12, 2)}},
    }

    # ---- e2e: pinned host inputs -> device -> both layers -> host outputs, every
    # step, pipelined over three streams with double-buffered device tensors:
    # the copy-in of step i+1 and the copy-out of step i-1 overlap step i's
    # kernels (PCIe carries both directions at once).
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    e2e_steps = max(3, min(nsteps, 50))
    s_in, s_run, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ins = [(qd, kd, vd), (torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd))]
    res_d = [(outs, lses),
             ({lay: torch.empty_like(qd) for lay in windows},
              {lay: torch.empty_like(lses[lay]) for lay in windows})]
    res_h = [({lay: torch.empty(q.shape, dtype=q.dtype).pin_memory() for lay in windows},
              {lay: torch.empty(tuple(lses[lay].shape), dtype=torch.float32).pin_memory()
               for lay in windows}) for _ in range(2)]
    total = e2e_steps + 2  # two untimed steps fill the pipeline
    ev_in = [torch.cuda.Event() for _ in range(total)]
    ev_run = [torch.cuda.Event() for _ in range(total)]
    ev_out = [torch.cuda.Event() for _ in range(total)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def e2e_step(i):
        b = i % 2
        (qb, kb, vb), (ob, lb), (ohb, lhb) = ins[b], res_d[b], res_h[b]
        if i >= 2:
            s_in.wait_event(ev_run[i - 2])   # step i-2's kernels have read buffer b
        with torch.cuda.stream(s_in):
            qb.copy_(qh, non_blocking=True)
            kb.copy_(kh, non_blocking=True)
            vb.copy_(vh, non_blocking=True)
            ev_in[i].record(s_in)
        s_run.wait_event(ev_in[i])
        if i >= 2:
            s_run.wait_event(ev_out[i - 2])  # step i-2's outputs have left buffer b
        for lay in ("local", "global"):
            g2.prefill(qb, kb, vb, query_scale=w.query_scale, softcap=w.softcap,
                       window=windows[lay], out=ob[lay], lse=lb[lay], stream=s_run)
        ev_run[i].record(s_run)
        s_out.wait_event(ev_run[i])
        with torch.cuda.stream(s_out):
            for lay in ("local", "global"):
                ohb[lay].copy_(ob[lay], non_blocking=True)
                lhb[lay].copy_(lb[lay], non_blocking=True)
            ev_out[i].record(s_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    e0.record(s_in)
    for i in range(2, total):
        e2e_step(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
    if world > 1:
        torch.distributed.all_reduce(e2e_t, op=torch.distributed.ReduceOp.MAX)
    e2e_ms = float(e2e_t.item())
    h2d = sum(t.numel() * t.element_size() for t in (q, k, v))
    d2h = sum(res_h[0][0][l].numel() * 2 + res_h[0][1][l].numel() * 4 for l in windows)
    result["e2e"] = {"value": round(step_flops * world / (e2e_ms * 1e-3) / 1e12, 3),
                     "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                     "ms_per_step": round(e2e_ms, 4),
                     "path": "pinned host q,k,v -> HBM -> g2attn_prefill x2 -> host out, lse; "
                             "every step, pipelined on three streams (copy-in of step i+1 and "
                             "copy-out of step i-1 overlap step i), double-buffered on the device",
                     "kernel_launches_per_step": 2}
    del ins, res_d, res_h

    if not args.no_extra:
        result["extra"] = extra_workloads(g2, dev, stream, flush)
    del flush
    return result


def time_launches(fn, flush, stream, reps=10, warm=3):
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts), min(ts)


def extra_workloads(g2, dev, stream, flush):
    pk, _ = peaks()
    res = {}
    # 2B pair, local and global reported separately
    w = WORKLOADS["2b"]
    q, k, v = (t.to(dev) for t in prefill_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d, w.std, w.seed))
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.T), dtype=torch.float32, device=dev)
    r9 = {}
    for lay, win in (("local", w.window_local), ("global", 0)):
        f = prefill_flops(w.B, w.T, w.S, w.H, w.d, 0, win)
        med, best = time_launches(lambda: g2.prefill(q, k, v, query_scale=w.query_scale,
                                                     softcap=w.softcap, window=win, out=out,
                                                     lse=lse, stream=stream), flush, stream)
        r9[lay] = {"ms": round(med, 4), "tflops": round(f / (med * 1e-3) / 1e12, 2),
                   "frac_bf16_peak": round(f / (med * 1e-3) / 1e12 / pk["bf16_tflops"], 4)}
    res["2b_prefill"] = r9
    del q, k, v, out, lse

    # Gemma 3-shaped variant of the 2B pair: window 1024, no soft-cap
    w = WORKLOADS["gemma3_2b"]
    q, k, v = (t.to(dev) for t in prefill_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d, w.std, w.seed))
    out = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.T), dtype=torch.float32, device=dev)
    rg = {}
    for lay, win in (("local", w.window_local), ("global", 0)):
        f = prefill_flops(w.B, w.T, w.S, w.H, w.d, 0, win)
        med, best = time_launches(lambda: g2.prefill(q, k, v, query_scale=w.query_scale,
                                                     softcap=w.softcap, window=win, out=out,
                                                     lse=lse, stream=stream), flush, stream)
        rg[lay] = {"ms": round(med, 4), "tflops": round(f / (med * 1e-3) / 1e12, 2),
                   "frac_bf16_peak": round(f / (med * 1e-3) / 1e12 / pk["bf16_tflops"], 4)}
    res["gemma3_2b_prefill"] = rg
    del q, k, v, out, lse

    # 27B decode
    w = WORKLOADS["27b_decode"]
    lengths, cu, q, k, v = decode_inputs(w.num_seqs, w.len_lo, w.len_hi, w.H, w.Hkv, w.d, w.std,
                                         w.seed)
    q, k, v, cu = q.to(dev), k.to(dev), v.to(dev), cu.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((q.shape[0], w.H), dtype=torch.float32, device=dev)
    ws = g2.decode_workspace(q.shape[0], w.H, w.d, max(lengths), dev)
    rd = {}
    for lay, win in (("local", w.window_local), ("global", 0)):
        nbytes = decode_kv_bytes(lengths, w.Hkv, w.d, win)
        med, best = time_launches(lambda: g2.decode(q, k, v, cu, max(lengths),
                                                    query_scale=w.query_scale, softcap=w.softcap,
                                                    window=win, out=out, lse=lse, workspace=ws,
                                                    stream=stream), flush, stream)
        gbs = nbytes / (med * 1e-3) / 1e9
        rd[lay] = {"ms": round(med, 4), "kv_GBps": round(gbs, 1),
                   "frac_hbm": round(gbs / pk["hbm_gbs"], 4),
                   "tokens_per_s": round(len(lengths) / (med * 1e-3), 1), "kv_bytes": nbytes}
    res["27b_decode"] = rd

    # the same decode from a ring cache (local layer, 4096 slots per sequence)
    # and from a paged cache (global layer, 64-row blocks in shuffled order)
    n, R, bs = len(lengths), w.window_local, 64
    Ls = torch.tensor(lengths, device=dev, dtype=torch.long)
    cul = cu.long()
    seq_of = torch.repeat_interleave(torch.arange(n, device=dev), Ls)
    pos = torch.arange(int(Ls.sum()), device=dev) - cul[:-1][seq_of]
    keep = pos >= (Ls[seq_of] - R)
    kr = torch.zeros((n * R,) + tuple(k.shape[1:]), dtype=k.dtype, device=dev)
    vr = torch.zeros_like(kr)
    kr[(seq_of * R + pos % R)[keep]] = k[keep]
    vr[(seq_of * R + pos % R)[keep]] = v[keep]
    kr, vr = kr.view(n, R, *k.shape[1:]), vr.view(n, R, *k.shape[1:])
    sl = Ls.to(torch.int32)
    nblk = (Ls + bs - 1) // bs
    total_blocks = int(nblk.sum())
    perm = torch.randperm(total_blocks, generator=torch.Generator().manual_seed(7)).to(dev)
    blk_start = torch.cumsum(nblk, 0) - nblk
    blk_of_row = perm[blk_start[seq_of] + pos // bs]
    kp = torch.zeros((total_blocks * bs,) + tuple(k.shape[1:]), dtype=k.dtype, device=dev)
    vp = torch.zeros_like(kp)
    kp[blk_of_row * bs + pos % bs] = k
    vp[blk_of_row * bs + pos % bs] = v
    kp, vp = kp.view(total_blocks, bs, *k.shape[1:]), vp.view(total_blocks, bs, *k.shape[1:])
    table = torch.full((n, int(nblk.max())), -1, dtype=torch.int32, device=dev)
    for s_ in range(n):
        table[s_, :int(nblk[s_])] = perm[int(blk_start[s_]):int(blk_start[s_] + nblk[s_])].int()
    del k, v
    rl = {}
    nbytes = decode_kv_bytes(lengths, w.Hkv, w.d, w.window_local)
    med, best = time_launches(lambda: g2.decode_ring(q, kr, vr, sl, w.window_local,
                                                     query_scale=w.query_scale,
                                                     softcap=w.softcap, out=out, lse=lse,
                                                     workspace=ws, stream=stream), flush, stream)
    gbs = nbytes / (med * 1e-3) / 1e9
    rl["ring_local"] = {"ms": round(med, 4), "kv_GBps": round(gbs, 1),
                        "frac_hbm": round(gbs / pk["hbm_gbs"], 4), "ring_slots": R}
    nbytes = decode_kv_bytes(lengths, w.Hkv, w.d, 0)
    med, best = time_launches(lambda: g2.decode_paged(q, kp, vp, table, sl, max(lengths),
                                                      query_scale=w.query_scale,
                                                      softcap=w.softcap, window=0, out=out,
                                                      lse=lse, workspace=ws, stream=stream),
                              flush, stream)
    gbs = nbytes / (med * 1e-3) / 1e9
    rl["paged_global"] = {"ms": round(med, 4), "kv_GBps": round(gbs, 1),
                          "frac_hbm": round(gbs / pk["hbm_gbs"], 4), "block_size": bs}
    res["27b_decode_cache_layouts"] = rl
    del q, kr, vr, kp, vp, out, lse, ws

    # 9B ragged packed prefill (16 sequences + chunked-prefill tail)
    w = WORKLOADS["9b_varlen"]
    Ts, Ss, cq, ck, q, k, v = varlen_inputs(w.num_seqs, w.len_lo, w.len_hi, w.H, w.Hkv, w.d,
                                            w.std, w.seed, tail_T=w.tail_T, tail_S=w.tail_S)
    q, k, v, cq, ck = q.to(dev), k.to(dev), v.to(dev), cq.to(dev), ck.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((w.H, q.shape[0]), dtype=torch.float32, device=dev)
    rv = {}
    for lay, win in (("local", w.window_local), ("global", 0)):
        f = varlen_flops(Ts, Ss, w.H, w.d, win)
        med, best = time_launches(lambda: g2.prefill_varlen(q, k, v, cq, ck, max(Ts), max(Ss),
                                                            query_scale=w.query_scale,
                                                            softcap=w.softcap, window=win,
                                                            out=out, lse=lse, stream=stream),
                                  flush, stream)
        rv[lay] = {"ms": round(med, 4), "tflops": round(f / (med * 1e-3) / 1e12, 2),
                   "frac_bf16_peak": round(f / (med * 1e-3) / 1e12 / pk["bf16_tflops"], 4)}
    res["9b_varlen"] = rv

    # the same packed queries with K/V in a paged cache (256-row blocks, shuffled)
    bs = 256
    Sl = torch.tensor(Ss, device=dev, dtype=torch.long)
    nblk = (Sl + bs - 1) // bs
    total_blocks = int(nblk.sum())
    perm = torch.randperm(total_blocks, generator=torch.Generator().manual_seed(9)).to(dev)
    seq_of = torch.repeat_interleave(torch.arange(len(Ss), device=dev), Sl)
    pos = torch.arange(int(Sl.sum()), device=dev) - ck.long()[:-1][seq_of]
    bstart = torch.cumsum(nblk, 0) - nblk
    dst = perm[bstart[seq_of] + pos // bs] * bs + pos % bs
    kp = torch.zeros((total_blocks * bs,) + tuple(k.shape[1:]), dtype=k.dtype, device=dev)
    vp = torch.zeros_like(kp)
    kp[dst] = k
    vp[dst] = v
    kp, vp = kp.view(total_blocks, bs, *k.shape[1:]), vp.view(total_blocks, bs, *k.shape[1:])
    table = torch.full((len(Ss), int(nblk.max())), -1, dtype=torch.int32, device=dev)
    for s_ in range(len(Ss)):
        table[s_, :int(nblk[s_])] = perm[int(bstart[s_]):int(bstart[s_] + nblk[s_])].int()
    sl = Sl.to(torch.int32)
    del k, v
    rp = {}
    for lay, win in (("local", w.window_local), ("global", 0)):
        f = varlen_flops(Ts, Ss, w.H, w.d, win)
        med, best = time_launches(lambda: g2.prefill_paged(q, kp, vp, cq, table, sl, max(Ts),
                                                           max(Ss), query_scale=w.query_scale,
                                                           softcap=w.softcap, window=win,
                                                           out=out, lse=lse, stream=stream),
                                  flush, stream)
        rp[lay] = {"ms": round(med, 4), "tflops": round(f / (med * 1e-3) / 1e12, 2),
                   "frac_bf16_peak": round(f / (med * 1e-3) / 1e12 / pk["bf16_tflops"], 4),
                   "block_size": bs}
    res["9b_varlen_paged_kv"] = rp
    del q, kp, vp, out, lse

    # gradients of the 27B-shaped (d = 128) and 2B-shaped (d = 256) layer pairs
    # (dq, dk, dv; three launches per call)
    for name in ("27b_backward", "2b_backward"):
        w = WORKLOADS[name]
        q, k, v, dout = (t.to(dev) for t in backward_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d,
                                                             w.std, w.seed))
        ws = g2.backward_workspace(w.B, w.T, w.H, dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        rb = {}
        for lay, win in (("local", w.window_local), ("global", 0)):
            out, lse = g2.prefill(q, k, v, query_scale=w.query_scale, softcap=w.softcap,
                                  window=win, stream=stream)
            f = backward_flops(w.B, w.T, w.S, w.H, w.d, 0, win)
            med, best = time_launches(
                lambda: g2.prefill_backward(q, k, v, out, lse, dout, query_scale=w.query_scale,
                                            softcap=w.softcap, window=win, workspace=ws, dq=dq,
                                            dk=dk, dv=dv, stream=stream), flush, stream)
            rb[lay] = {"ms": round(med, 4), "tflops": round(f / (med * 1e-3) / 1e12, 2),
                       "frac_bf16_peak": round(f / (med * 1e-3) / 1e12 / pk["bf16_tflops"], 4)}
        res[name] = rb
        del q, k, v, dout, dq, dk, dv, ws, out, lse

    # gradients of a 27B-shaped packed batch (8 sequences of 512-8192 tokens)
    w = WORKLOADS["27b_varlen_backward"]
    Ts, Ss, cq, ck, q, k, v, dout = varlen_backward_inputs(w.num_seqs, w.len_lo, w.len_hi, w.H,
                                                           w.Hkv, w.d, w.std, w.seed)
    q, k, v, dout, cq, ck = (t.to(dev) for t in (q, k, v, dout, cq, ck))
    n = g2.g2attn_varlen_backward_workspace_size(len(Ts), q.shape[0], w.H)
    ws = torch.empty(n, dtype=torch.uint8, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    rvb = {"tokens": int(sum(Ts))}
    for lay, win in (("local", w.window_local), ("global", 0)):
        out, lse = g2.prefill_varlen(q, k, v, cq, ck, max(Ts), max(Ss), query_scale=w.query_scale,
                                     softcap=w.softcap, window=win, stream=stream)
        f = 2.5 * varlen_flops(Ts, Ss, w.H, w.d, win)
        med, best = time_launches(
            lambda: g2.prefill_varlen_backward(q, k, v, out, lse, dout, cq, ck, max(Ts), max(Ss),
                                               query_scale=w.query_scale, softcap=w.softcap,
                                               window=win, workspace=ws, dq=dq, dk=dk, dv=dv,
                                               stream=stream), flush, stream)
        rvb[lay] = {"ms": round(med, 4), "tflops": round(f / (med * 1e-3) / 1e12, 2),
                    "frac_bf16_peak": round(f / (med * 1e-3) / 1e12 / pk["bf16_tflops"], 4)}
    res["27b_varlen_backward"] = rvb
    return res


# ---------------------------------------------------------------------------
# CPU baseline / reference arm: the fp64 oracle on the host cores
# ---------------------------------------------------------------------------
def host_info():
    """CPU model and core counts of the host the oracle runs on."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "os_cpu_count": os.cpu_count(),
            "affinity_cpus": len(os.sched_getaffinity(0))}


def _oracle_rows(oracle, q, k, v, w, nrows, rng):
    """The oracle on nrows query rows of each layer of workload w, spread
    uniformly over batch, positions and heads. Returns (seconds, useful FLOPs);
    the useful FLOPs of a row are 4*d*(visible keys of that row)."""
    t0 = time.perf_counter()
    useful = 0.0
    for win in (w.window_local, 0):
        b = rng.integers(0, w.B, nrows)
        pos = rng.integers(0, w.T, nrows)
        heads = rng.integers(0, w.H, nrows)
        rows = np.stack([b, pos, heads], 1).astype(np.int64)
        oracle.attn_rows(q, k, v, rows, query_scale=w.query_scale, softcap=w.softcap, window=win)
        vis = np.minimum(pos + 1, win) if win else pos + 1
        useful += float(np.sum(4.0 * w.d * vis))
    return time.perf_counter() - t0, useful


def _oracle_calibrate(oracle, q, k, v, w, target_s, rng):
    """Rows per layer for one sample of about target_s seconds."""
    threads = oracle.max_threads()
    n = max(threads, 8)
    dt, _ = _oracle_rows(oracle, q, k, v, w, n, rng)
    return int(max(threads, min(200000, n * target_s / max(dt, 1e-3))))


def cpu_baseline(target_s=15.0):
    """The fp64 oracle, as it stands, on the host cores (all the process may
    use): a bounded row sample of the step's workload (its value), one thread
    on the whole tiny pair, and the whole 27B decode in the GPU's units."""
    import oracle
    threads = len(os.sched_getaffinity(0))
    oracle.set_threads(threads)
    threads = oracle.max_threads()
    w = WORKLOADS[WORKLOAD]
    q, k, v = prefill_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d, w.std, w.seed)
    rng = np.random.default_rng(0)
    n = _oracle_calibrate(oracle, q, k, v, w, target_s, rng)
    dt, useful = _oracle_rows(oracle, q, k, v, w, n, rng)
    res = {"kind": "oracle", "cores": threads, "value": useful / dt / 1e12, "unit": "TFLOP/s",
           "sample": f"{2 * n} query rows (half local, half global) of the {WORKLOAD} pair, "
                     f"uniform batch, positions and heads",
           "seconds": round(dt, 2), "host": host_info()}

    # one thread, the whole tiny pair (B=1, T=S=256, H=4, Hkv=2, d=64)
    wt = WORKLOADS["tiny"]
    qt, kt, vt = prefill_inputs(wt.B, wt.T, wt.S, wt.H, wt.Hkv, wt.d, wt.std, wt.seed)
    oracle.set_threads(1)
    tiny = {"threads": oracle.max_threads()}
    tiny_useful = tiny_s = 0.0
    for lay, win in (("local", wt.window_local), ("global", 0)):
        t0 = time.perf_counter()
        oracle.attn(qt, kt, vt, query_scale=wt.query_scale, softcap=wt.softcap, window=win)
        tiny[f"{lay}_s"] = round(time.perf_counter() - t0, 4)
        tiny_s += tiny[f"{lay}_s"]
        tiny_useful += prefill_flops(wt.B, wt.T, wt.S, wt.H, wt.d, 0, win)
    tiny["gflops_per_s"] = round(tiny_useful / max(tiny_s, 1e-9) / 1e9, 3)
    oracle.set_threads(threads)
    res["tiny_pair_1_thread"] = tiny

    # the whole 27B decode (64 sequences), all threads, per layer
    wd = WORKLOADS["27b_decode"]
    lengths, cu, qd, kc, vc = decode_inputs(wd.num_seqs, wd.len_lo, wd.len_hi, wd.H, wd.Hkv,
                                            wd.d, wd.std, wd.seed)
    dec = {"sequences": len(lengths)}
    for lay, win in (("local", wd.window_local), ("global", 0)):
        t0 = time.perf_counter()
        oracle.decode(qd, kc, vc, cu, query_scale=wd.query_scale, softcap=wd.softcap, window=win)
        t = time.perf_counter() - t0
        nbytes = decode_kv_bytes(lengths, wd.Hkv, wd.d, win)
        dec[lay] = {"s": round(t, 3), "kv_GBps": round(nbytes / t / 1e9, 3),
                    "tokens_per_s": round(len(lengths) / t, 2)}
    res["27b_decode"] = dec
    return res


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle on the host cores, each step a
    bounded row sample of the step's workload (the same sample size every
    step), sized so that warm-up and timed steps end within a few minutes."""
    if rank != 0:
        return None
    import oracle
    threads = len(os.sched_getaffinity(0))
    oracle.set_threads(threads)
    threads = oracle.max_threads()
    w = WORKLOADS[WORKLOAD]
    q, k, v = prefill_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d, w.std, w.seed)
    rng = np.random.default_rng(0)
    total = args.warmup + args.steps
    per_step_s = min(10.0, max(0.05, 150.0 / max(total, 1)))
    n = _oracle_calibrate(oracle, q, k, v, w, per_step_s, rng)
    times, useful = [], 0.0
    for i in range(total):
        dt, u = _oracle_rows(oracle, q, k, v, w, n, rng)
        if i >= args.warmup:
            times.append(dt)
            useful += u
    value = useful / sum(times) / 1e12
    ms_per_step = 1e3 * sum(times) / len(times)
    sample = (f"{2 * n} query rows per step (half local, half global) of the {WORKLOAD} pair, "
              f"uniform batch, positions and heads")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded iid N(0,1) bf16)",
            "config": headline_config(world),
            "step": "one bounded sample of the workload (ms_per_step is the sample's time); "
                    "the whole two-layer step would take projected_ms_per_full_step",
            "projected_ms_per_full_step": step_flops_of(w) / (value * 1e12) * 1e3,
            "cpu_baseline": {"kind": "oracle", "cores": threads, "sample": sample,
                             "value": value, "unit": "TFLOP/s", "host": host_info()},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def run_single(args, dev):
    """One kernel case only (for profiling): `<workload>:<layer>`, layer local|global."""
    import global_soft_capped_b200 as g2
    g2.load_library()
    name, lay = args.single.split(":")
    w = WORKLOADS[name]
    win = w.window_local if lay == "local" else 0
    stream = torch.cuda.current_stream()
    if name == "27b_varlen_backward":
        Ts, Ss, cq, ck, q, k, v, dout = varlen_backward_inputs(w.num_seqs, w.len_lo, w.len_hi,
                                                               w.H, w.Hkv, w.d, w.std, w.seed)
        q, k, v, dout, cq, ck = (t.to(dev) for t in (q, k, v, dout, cq, ck))
        out, lse = g2.prefill_varlen(q, k, v, cq, ck, max(Ts), max(Ss), query_scale=w.query_scale,
                                     softcap=w.softcap, window=win, stream=stream)
        fn = lambda: g2.prefill_varlen_backward(q, k, v, out, lse, dout, cq, ck, max(Ts),
                                                max(Ss), query_scale=w.query_scale,
                                                softcap=w.softcap, window=win, stream=stream)
    elif name in ("27b_backward", "2b_backward"):
        q, k, v, dout = (t.to(dev) for t in backward_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d,
                                                             w.std, w.seed))
        out, lse = g2.prefill(q, k, v, query_scale=w.query_scale, softcap=w.softcap, window=win,
                              stream=stream)
        ws = g2.backward_workspace(w.B, w.T, w.H, dev)
        fn = lambda: g2.prefill_backward(q, k, v, out, lse, dout, query_scale=w.query_scale,
                                         softcap=w.softcap, window=win, workspace=ws,
                                         stream=stream)
    elif w.kind == "prefill":
        q, k, v = (t.to(dev) for t in prefill_inputs(w.B, w.T, w.S, w.H, w.Hkv, w.d, w.std,
                                                      w.seed))
        fn = lambda: g2.prefill(q, k, v, query_scale=w.query_scale, softcap=w.softcap,
                                window=win, stream=stream)
    elif w.kind == "decode":
        lengths, cu, q, k, v = decode_inputs(w.num_seqs, w.len_lo, w.len_hi, w.H, w.Hkv, w.d,
                                             w.std, w.seed)
        q, k, v, cu = q.to(dev), k.to(dev), v.to(dev), cu.to(dev)
        ws = g2.decode_workspace(q.shape[0], w.H, w.d, max(lengths), dev)
        fn = lambda: g2.decode(q, k, v, cu, max(lengths), query_scale=w.query_scale,
                               softcap=w.softcap, window=win, workspace=ws, stream=stream)
    else:
        Ts, Ss, cq, ck, q, k, v = varlen_inputs(w.num_seqs, w.len_lo, w.len_hi, w.H, w.Hkv,
                                                w.d, w.std, w.seed, tail_T=w.tail_T,
                                                tail_S=w.tail_S)
        q, k, v, cq, ck = q.to(dev), k.to(dev), v.to(dev), cq.to(dev), ck.to(dev)
        fn = lambda: g2.prefill_varlen(q, k, v, cq, ck, max(Ts), max(Ss),
                                       query_scale=w.query_scale, softcap=w.softcap,
                                       window=win, stream=stream)
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    print(json.dumps({"single": args.single, "steps": args.steps,
                      "ms_per_launch": a.elapsed_time(b) / max(args.steps, 1)}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true", help="skip the 9B/decode/varlen extras")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--single", default=None,
                    help="profile aid: run one case only, e.g. 9b:global or 27b_decode:local")
    args = ap.parse_args()
    if args.single:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        run_single(args, dev)
        return
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        # one rank per GPU: N GPUs need N ranks (torchrun --nproc-per-node N)
        sys.stderr.write(f"bench.py: --gpus {args.gpus} but WORLD_SIZE is {world}; launch "
                         f"{args.gpus} ranks with torchrun --nproc-per-node {args.gpus}\n")
        sys.exit(2)

    if args.impl == "reference":
        if world > 1 and rank != 0:
            return
        res = run_reference(args, rank, world)
        print(json.dumps(res), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    # the oracle's thread pool is created before any GPU work (never forked after it)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()
    res = run_ours(args, rank, world, dev)
    if rank == 0:
        if cpu is not None:
            res["cpu_baseline"] = cpu
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
