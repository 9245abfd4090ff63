#!/usr/bin/env python
"""Throughput of the exact-attention training step (causal fwd + bwd) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload c3|c4]
    python bench.py --sweep all|c5|splitkv|kv_outer|bwd  (supplementary per-case lines)
    python bench.py --traffic                   (cases for an ncu DRAM-bytes capture)
    python bench.py --traffic-report NCU_CSV    (that capture against the traffic model)

One step = the forward kernel (O, LSE) plus the backward (preprocess, main,
dQ convert) on one batch of seeded synthetic bf16 inputs that are already
resident in HBM.  The default workload is B=2, H=16, N=4096, d=128, causal
(the training-step configuration); the L2 cache is flushed before every timed
step by writing a 256 MiB buffer outside the step's events.

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch of
independent (batch, head) problems -- attention has no exchange step across
heads, so there is no collective on the data path ("scaling": "weak"); the
step time is the max over ranks.

Metric: algorithmic TFLOP/s, FLOPs = 4*B*H*N^2*d (forward; halved when causal)
and 2.5 times that for the backward.

``--impl reference`` times the CPU float64 oracle (the reference arm of this
library: there is no reference GPU code) on a bounded per-step sample of the
same workload on the host cores, and prints the same JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention fwd / fwd+bwd TFLOP/s (bf16, causal, d=128) and % of BF16 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0  # B200 datasheet dense bf16 (context; the measured peak is primary)


def rank_workload(w, rank):
    """The batch rank ``rank`` processes: same shapes, its own seeds.

    Attention over different (batch, head) slices shares nothing, so under
    torchrun every rank runs an independent batch (weak scaling) and no data
    crosses GPUs.
    """
    import dataclasses
    return dataclasses.replace(w, seed_base=w.seed_base + 1000 * rank)


# groups of (b, h) slices in the end-to-end leg (copies overlap compute).  The
# copies bound it (B200, PCIe: 55 GB/s one way, 50 GB/s each way at once, so
# 2.7 ms of copies per c3 step); B200, c3: 1 group 3.42 ms per step, 2 groups
# 2.95, 3 groups 3.26, 4 groups 3.13, 16 groups 3.67 -- more groups overlap
# more, but each call on fewer heads fills the GPU less (8 heads: 128 forward
# items for 148 SMs).
E2E_CHUNKS = 2


def max_over_ranks(values, world, device=None):
    """Element-wise max of a list of floats over all ranks (max-over-ranks timing)."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def job_tflops(flops_per_rank_step, world, ms_per_step):
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


def attention_flops(B, H, N, d, causal):
    fwd = 4.0 * B * H * N * N * d
    if causal:
        fwd /= 2.0
    return fwd, 2.5 * fwd


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def _strip_comments(text):
    """C++ source without comments and trailing blanks (what the compiler sees)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(ln.rstrip() for ln in text.splitlines() if ln.strip())


def source_digest():
    """Hash of the kernel code (comments excluded): ncu counters are only valid
    for this exact code."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_attention_117_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode())
            h.update(_strip_comments(f.read()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key, workload):
    """DRAM bytes per launch from the committed ncu summary, if it matches this code."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            data = json.load(f)
    except Exception:
        return None
    ent = data.get(workload, {}).get(kernel_key)
    if not ent or ent.get("source_digest") != source_digest():
        return None
    return ent.get("dram_bytes_per_launch")


def _clock_worker(index, conn, period_s):
    """Child process of ClockSampler: samples the SM clock and the clock-event
    reasons through NVML (read-only queries) until the parent asks for the
    samples; each sample carries its CLOCK_MONOTONIC time."""
    import time

    import pynvml
    pynvml.nvmlInit()
    h = pynvml.nvmlDeviceGetHandleByIndex(index)
    get = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
        pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
    mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
    # one query of each kind before the region: the first calls are slow (a
    # 12 ms region once got no sample of its own)
    pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
    get(h)
    out = []
    conn.send("ready")
    while not conn.poll():
        t = time.monotonic_ns()
        out.append((t, pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), mx, get(h)))
        time.sleep(period_s)
    conn.recv()
    conn.send(out)


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons while the
    timed region runs.  The NVML queries run in a child process (started,
    with spawn, before the region) so that they neither share the launching
    thread -- issued once per step from that thread they slowed the timed
    kernels by 4 % on B200 (measured A/B) -- nor wait for this process's
    interpreter lock, which a sampling thread here did (one sample in a 12 ms
    region).  The child samples about every 0.2 ms; the samples whose time
    falls inside the region are kept.  Where NVML is missing, nvidia-smi is
    queried from a thread every 200 ms."""

    NAMES = ("sw_power_cap", "hw_slowdown", "sw_thermal_slowdown", "hw_thermal_slowdown")
    BITS = (0x4, 0x8, 0x20, 0x40)  # nvmlClocksEventReason{SwPowerCap,HwSlowdown,Sw/HwThermal}
    SMI_FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                  "clocks_event_reasons.hw_thermal_slowdown,"
                  "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.samples = []  # (sm_mhz, max_mhz, set of active reasons)
        self.source = None
        self._proc = None
        self._conn = None
        self._stop = threading.Event()
        self._t = None
        try:
            import multiprocessing as mp

            import pynvml  # noqa: F401
            ctx = mp.get_context("spawn")
            self._conn, child = ctx.Pipe()
            self._proc = ctx.Process(target=_clock_worker, args=(index, child, 0.0002), daemon=True)
            self._proc.start()
            child.close()  # the child's end lives on in the child only
            deadline = time.monotonic() + 60
            while not self._conn.poll(0.1):
                if not self._proc.is_alive() or time.monotonic() > deadline:
                    raise RuntimeError("clock sampler did not start")
            if self._conn.recv() != "ready":
                raise RuntimeError("clock sampler did not start")
            self.source = "nvml"
        except Exception:
            self._stop_child()
            self.source = "nvidia-smi"

    def _stop_child(self):
        if self._proc is not None:
            try:
                self._proc.terminate()
                self._proc.join(timeout=5)
            except Exception:
                pass
        self._proc = None

    def _sample_smi(self):
        out = subprocess.run(
            ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.SMI_FIELDS}",
             "--format=csv,noheader,nounits"], capture_output=True, text=True, timeout=5)
        p = [x.strip() for x in out.stdout.strip().split(",")]
        if len(p) == 7 and p[0].replace(".", "").isdigit() and p[1].replace(".", "").isdigit():
            act = {"hw_slowdown": p[3], "hw_thermal_slowdown": p[4],
                   "sw_thermal_slowdown": p[5], "sw_power_cap": p[6]}
            self.samples.append((float(p[0]), float(p[1]),
                                 {k for k, v in act.items() if v.lower() == "active"}))

    def _run_smi(self):
        while not self._stop.is_set():
            try:
                self._sample_smi()
            except Exception:
                pass
            self._stop.wait(0.2)

    def __enter__(self):
        self._t0 = time.monotonic_ns()
        if self._proc is None:
            self._t = threading.Thread(target=self._run_smi, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        t1 = time.monotonic_ns()
        if self._proc is not None:
            try:
                self._conn.send("stop")
                raw = self._conn.recv() if self._conn.poll(30) else []
            except Exception:
                raw = []
            self._stop_child()
            self.add_nvml_samples(raw, self._t0, t1)
        else:
            self._stop.set()
            self._t.join(timeout=10)
        return False

    def add_nvml_samples(self, raw, t0, t1):
        """Keeps the NVML samples ``(monotonic ns, sm MHz, max MHz, reason bits)``
        taken inside [t0, t1]; a region shorter than one query keeps the nearest."""
        inside = [r for r in raw if t0 <= r[0] <= t1]
        if not inside and raw:
            inside = [min(raw, key=lambda r: abs(r[0] - (t0 + t1) // 2))]
        for _, sm, mx, bits in inside:
            self.samples.append((float(sm), float(mx),
                                 {n for n, b in zip(self.NAMES, self.BITS) if bits & b}))

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"],
                    "source": self.source}
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": max(s[1] for s in self.samples),
                "reasons": sorted(set().union(*(s[2] for s in self.samples))),
                "samples": len(self.samples), "source": self.source}


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = max((x.get("num_threads", 0) for x in info), default=0)
        return int(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_sample(w, budget_s, device_inputs=None, keep_first=False):
    """Times the float64 oracle (fwd + bwd) on whole (b, h) slices for ~budget_s.

    Returns (algorithmic TFLOP/s, description of the sample, first) where
    ``first`` is ``(b, h, O, LSE, (dQ, dK, dV))`` of the first slice timed if
    ``keep_first``, else None.
    """
    import numpy as np
    import torch

    import oracle
    from exact_attention_117_b200.workloads import make_inputs, sample_slices

    if device_inputs is None:
        device_inputs = make_inputs(w, "cpu")
    causal = True
    fwd1, bwd1 = attention_flops(1, 1, w.N, w.d, causal)
    order = sample_slices(w.B * w.H, w.B * w.H)
    done, t_total, first = 0, 0.0, None
    for idx in order:
        b, h = idx // w.H, idx % w.H
        sl = [device_inputs[k][b, h].float().cpu().numpy().astype(np.float64)
              for k in ("q", "k", "v", "do")]
        t0 = time.perf_counter()
        o_ref, lse_ref = oracle.attention_forward(sl[0], sl[1], sl[2], causal=causal,
                                                  scale=w.scale)
        g_ref = oracle.attention_backward(*sl, causal=causal, scale=w.scale)
        t_total += time.perf_counter() - t0
        if keep_first and first is None:
            first = (b, h, o_ref, lse_ref, g_ref)
        done += 1
        if t_total >= budget_s:
            break
    del torch
    tflops = done * (fwd1 + bwd1) / t_total / 1e12
    return tflops, (f"{done} of {w.B * w.H} (b,h) slices of the workload, fwd+bwd in float64 "
                    f"({t_total:.1f} s)"), first


def slice_errors(gpu, ref):
    """Errors of the timed run's outputs on one (b, h) slice against the oracle,
    with the stated tolerances (O rel-L2 5e-3, LSE abs 1e-3, gradients rel-L2
    1e-2; O max-abs 1e-2, where an element above that must be the bf16 output
    rounding itself -- half an ulp of 8-bit precision exceeds 1e-2 from |O| = 4)."""
    import numpy as np

    def rel(a, r):
        return float(np.linalg.norm(a - r) / max(np.linalg.norm(r), 1e-300))
    b, h, o_ref, lse_ref, g_ref = ref
    o, lse, dq, dk, dv = (np.asarray(t, dtype=np.float64) for t in gpu)
    out = {"slice": [b, h],
           "o_max_abs": float(np.max(np.abs(o - o_ref))), "o_rel_l2": rel(o, o_ref),
           "lse_max_abs": float(np.max(np.abs(lse - lse_ref))),
           "dq_rel_l2": rel(dq, g_ref[0]), "dk_rel_l2": rel(dk, g_ref[1]),
           "dv_rel_l2": rel(dv, g_ref[2])}
    # O max-abs above 1e-2 is allowed only where the excess is the bf16 output
    # rounding itself: there the output must be within one bf16 ulp of bf16(O_ref)
    import torch
    bad = np.abs(o - o_ref) > 1e-2
    o_bf = torch.from_numpy(o_ref[bad].astype(np.float32)).to(torch.bfloat16).double().numpy()
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(o_ref[bad]), 2.0 ** -126))) - 7)
    o_ok = bool(np.all(np.abs(o[bad] - o_bf) <= ulp))
    out["o_max_abs_excess_is_bf16_rounding"] = o_ok
    out["within_tolerance"] = bool(
        out["o_rel_l2"] <= 5e-3 and out["lse_max_abs"] <= 1e-3 and
        max(out["dq_rel_l2"], out["dk_rel_l2"], out["dv_rel_l2"]) <= 1e-2 and o_ok)
    return out


def line_config(w):
    """The ``config`` object of the JSON line; both arms print the same one."""
    return {"workload": f"{w.name}: causal fwd+bwd, B={w.B} H={w.H} N={w.N} d={w.d}",
            "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": True, "scale": w.scale,
            "per_rank": "independent copy of the batch on every rank",
            "l2": "flushed (256 MiB write) before every timed step, outside its events"}


def run_reference(args, w, rank):
    if rank != 0:
        return
    steps, warm = args.steps, args.warmup
    from exact_attention_117_b200.workloads import make_inputs
    x = make_inputs(w, "cpu")
    budget = max(0.5, min(10.0, 150.0 / max(1, steps + warm)))
    for _ in range(warm):
        oracle_sample(w, budget * 0.25, x)
    vals, descs = [], []
    t0 = time.perf_counter()
    for _ in range(steps):
        v, d, _ = oracle_sample(w, budget, x)
        vals.append(v)
        descs.append(d)
    wall = time.perf_counter() - t0
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": warm,
        "ms_per_step": 1000.0 * wall / steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": line_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_threads(),
                         "kind": "oracle", "sample": descs[-1]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from exact_attention_117_b200 import fa
    from exact_attention_117_b200.workloads import make_inputs

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    fa.load()
    causal = True
    B, H, N, d = w.B, w.H, w.N, w.d
    fwd_f, bwd_f = attention_flops(B, H, N, d, causal)
    x = make_inputs(rank_workload(w, rank), dev)
    q, k, v, do = x["q"], x["k"], x["v"], x["do"]
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(fa.workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        fa.forward(q, k, v, causal=causal, scale=w.scale, out=o, lse=lse, stream=stream)
        fa.backward(q, k, v, o, lse, do, causal=causal, scale=w.scale, dq=dq, dk=dk, dv=dv,
                    workspace=ws, stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(3, args.warmup)):
        flush.zero_()
        step()
    fa.check_device_error(stream)

    # ---------------------------------------------------------- device-timed region
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    evf = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk, fa.KernelTimer() as kt:
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            evf[i][0].record(stream)
            fa.forward(q, k, v, causal=causal, scale=w.scale, out=o, lse=lse, stream=stream)
            evf[i][1].record(stream)
            fa.backward(q, k, v, o, lse, do, causal=causal, scale=w.scale, dq=dq, dk=dk, dv=dv,
                        workspace=ws, stream=stream)
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    fa.check_device_error(stream)
    # outputs of the last timed step on slice (0, 0), for the oracle comparison
    timed_slice = [t[0, 0].double().cpu().numpy() for t in (o, lse, dq, dk, dv)]
    step_ms = sum(a.elapsed_time(b) for a, b in ev)
    fwd_ms = sum(a.elapsed_time(b) for a, b in evf)
    step_ms, fwd_ms = max_over_ranks([step_ms, fwd_ms], world, dev)
    ms_per_step = step_ms / args.steps
    fwd_ms_per = fwd_ms / args.steps
    bwd_ms_per = ms_per_step - fwd_ms_per
    value = job_tflops(fwd_f + bwd_f, world, ms_per_step)

    # ------------------------------------------------------------- end to end
    e2e = None
    if not args.no_e2e:
        host = {n: t.cpu().pin_memory() for n, t in (("q", q), ("k", k), ("v", v), ("do", do))}
        outs_host = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                     for n, t in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv))}
        dev_in = {n: torch.empty_like(t) for n, t in (("q", q), ("k", k), ("v", v), ("do", do))}
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = sum(t.numel() * t.element_size() for t in outs_host.values())

        # The (b, h) slices are independent problems, so the step runs as E2E_CHUNKS
        # groups of slices (each a [1, slices, N, d] call) on three streams:
        # inputs of group c+1 copy in while group c computes and group c-1's
        # results copy out (the two copy directions use separate engines).  A
        # group's buffers are reused only after the previous step is done with
        # them: its copy-in waits for that step's compute of the group, its
        # compute for that step's copy-out.
        bh = w.B * w.H
        n_chunks = max(1, min(args.e2e_chunks, bh))
        bounds = [(c * bh // n_chunks, (c + 1) * bh // n_chunks) for c in range(n_chunks)]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        s_comp = stream

        def flat(t):  # [1, B*H, ...] view of a [B, H, ...] tensor
            return t.view(1, bh, *t.shape[2:])

        ev_comp = [None] * n_chunks  # last compute of each group
        ev_out = [None] * n_chunks   # last copy-out of each group

        def e2e_step():
            for c, (a, b) in enumerate(bounds):
                with torch.cuda.stream(s_in):
                    if ev_comp[c] is not None:
                        s_in.wait_event(ev_comp[c])
                    for n in dev_in:
                        flat(dev_in[n])[:, a:b].copy_(flat(host[n])[:, a:b], non_blocking=True)
                    ev_i = torch.cuda.Event()
                    ev_i.record(s_in)
                s_comp.wait_event(ev_i)
                if ev_out[c] is not None:
                    s_comp.wait_event(ev_out[c])
                qc, kc, vc, doc = (flat(dev_in[n])[:, a:b] for n in ("q", "k", "v", "do"))
                oc, lc = flat(o)[:, a:b], flat(lse)[:, a:b]
                fa.forward(qc, kc, vc, causal=causal, scale=w.scale, out=oc, lse=lc,
                           stream=s_comp)
                fa.backward(qc, kc, vc, oc, lc, doc, causal=causal, scale=w.scale,
                            dq=flat(dq)[:, a:b], dk=flat(dk)[:, a:b], dv=flat(dv)[:, a:b],
                            workspace=ws, stream=s_comp)
                ev_c = torch.cuda.Event()
                ev_c.record(s_comp)
                ev_comp[c] = ev_c
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_c)
                    for n, src in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
                        flat(outs_host[n])[:, a:b].copy_(flat(src)[:, a:b], non_blocking=True)
                    ev_o = torch.cuda.Event()
                    ev_o.record(s_out)
                    ev_out[c] = ev_o

        def join():  # the timing stream waits for every copy-out issued so far
            for ev in ev_out:
                if ev is not None:
                    stream.wait_event(ev)

        for _ in range(2):
            e2e_step()
        join()
        barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        s_out.wait_event(e0)
        for _ in range(args.steps):
            e2e_step()
        join()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_ms = max_over_ranks([e0.elapsed_time(e1)], world, dev)[0] / args.steps
        e2e = {"value": job_tflops(fwd_f + bwd_f, world, e2e_ms), "unit": "TFLOP/s",
               "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "path": f"pinned host -> device copy, fa_fwd + fa_bwd through the C ABI, outputs "
                       f"copied back to pinned host; {n_chunks} groups of (b, h) slices "
                       f"pipelined over copy-in, compute and copy-out streams"}

    # ------------------------------------------------------- long-context leg
    long_ctx = None
    if not args.no_long_context:
        long_ctx = measure_long_context(rank, world, local_rank, dev, stream, flush, barrier)

    if rank != 0:
        return

    # ------------------------------------------------------------------ roofline
    peaks, peak_src = load_peaks()
    per_kernel = {kname: (kt.ms[kname] / kt.launches[kname] if kt.launches[kname] else 0.0)
                  for kname in fa.KERNELS}
    totals = {kname: kt.ms[kname] for kname in fa.KERNELS}
    peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    roof = roofline_entry(totals, per_kernel, {"fwd": fwd_f, "bwd_main": bwd_f}, peaks,
                          peak_src, lambda k: ncu_traffic(k, w.name))
    fwd_tf = fwd_f / (per_kernel["fwd"] * 1e-3) / 1e12 if per_kernel["fwd"] else None
    bwd_tf = bwd_f / (bwd_ms_per * 1e-3) / 1e12
    kernels = {kname: {"launches": kt.launches[kname], "total_ms": kt.ms[kname],
                       "share": kt.ms[kname] / max(1e-9, sum(totals.values()))}
               for kname in fa.KERNELS}

    cpu = None
    parity = None
    if world == 1 and not args.no_cpu_baseline:
        # the oracle runs on the very inputs of the timed steps; its first slice
        # (b, h) = (0, 0) is also compared with the timed run's outputs
        tf, desc, first = oracle_sample(w, args.cpu_seconds, x, keep_first=True)
        cpu = {"value": tf, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": desc}
        if first is not None and first[:2] == (0, 0):
            parity = slice_errors(timed_slice, first)

    launches = sum(kt.launches.values())
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": line_config(w),
        "fwd": {"ms": fwd_ms_per, "tflops": fwd_f / (fwd_ms_per * 1e-3) / 1e12,
                "kernel_tflops": fwd_tf, "pct_of_peak": 100.0 * (fwd_tf or 0) / peak_tf},
        "bwd": {"ms": bwd_ms_per, "tflops": bwd_tf, "pct_of_peak": 100.0 * bwd_tf / peak_tf},
        "pct_of_peak": 100.0 * value / world / peak_tf,
        "roofline": roof,
        "kernels": kernels,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk.summary(),
        "parity_vs_oracle": parity,
        "long_context": long_ctx,
        "env": run_env(dev),
    }
    print(json.dumps(line), flush=True)


def measure_long_context(rank, world, local_rank, dev, stream, flush, barrier, steps=5,
                         warmup=3):
    """The long-context training step (B=1 H=32 N=16384 d=128 causal, Q times 4),
    timed in the same process after the headline steps, with its own clock
    record: forward, backward and the roofline of its dominant kernel.  Every
    rank runs its own copy (the same collective steps on every rank)."""
    import torch

    from exact_attention_117_b200 import fa
    from exact_attention_117_b200.workloads import WORKLOADS, make_inputs
    w = WORKLOADS["c4"]
    B, H, N, d = w.B, w.H, w.N, w.d
    fwd_f, bwd_f = attention_flops(B, H, N, d, True)
    x = make_inputs(rank_workload(w, rank), dev)
    q, k, v, do = x["q"], x["k"], x["v"], x["do"]
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    ws = torch.empty(fa.workspace_size(B, H, N, d), dtype=torch.uint8, device=dev)

    def fwd():
        fa.forward(q, k, v, causal=True, scale=w.scale, out=o, lse=lse, stream=stream)

    def bwd():
        fa.backward(q, k, v, o, lse, do, causal=True, scale=w.scale, dq=dq, dk=dk, dv=dv,
                    workspace=ws, stream=stream)
    for _ in range(warmup):
        flush.zero_()
        fwd()
        bwd()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk, fa.KernelTimer() as kt:
        for i in range(steps):
            flush.zero_()
            ev[i][0].record(stream)
            fwd()
            ev[i][1].record(stream)
            bwd()
            ev[i][2].record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    fa.check_device_error(stream)
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    step_ms = sum(e[0].elapsed_time(e[2]) for e in ev)
    fwd_ms, step_ms = max_over_ranks([fwd_ms, step_ms], world, dev)
    fwd_ms, step_ms = fwd_ms / steps, step_ms / steps
    bwd_ms = step_ms - fwd_ms
    peaks, peak_src = load_peaks()
    peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    per_kernel = {kname: (kt.ms[kname] / kt.launches[kname] if kt.launches[kname] else 0.0)
                  for kname in fa.KERNELS}
    totals = {kname: kt.ms[kname] for kname in fa.KERNELS}
    fwd_ktf = fwd_f / (per_kernel["fwd"] * 1e-3) / 1e12 if per_kernel["fwd"] else None
    out = {
        "workload": f"{w.name}: causal fwd+bwd, B={B} H={H} N={N} d={d}, Q times {w.q_mult:g}",
        "steps": steps, "warmup": warmup, "ms_per_step": step_ms,
        "value": job_tflops(fwd_f + bwd_f, world, step_ms), "unit": "TFLOP/s",
        "pct_of_peak": 100.0 * (fwd_f + bwd_f) / (step_ms * 1e-3) / 1e12 / peak_tf,
        "fwd": {"ms": fwd_ms, "tflops": fwd_f / (fwd_ms * 1e-3) / 1e12, "kernel_tflops": fwd_ktf,
                "pct_of_peak": 100.0 * (fwd_ktf or 0.0) / peak_tf},
        "bwd": {"ms": bwd_ms, "tflops": bwd_f / (bwd_ms * 1e-3) / 1e12,
                "pct_of_peak": 100.0 * bwd_f / (bwd_ms * 1e-3) / 1e12 / peak_tf},
        "roofline": roofline_entry(totals, per_kernel, {"fwd": fwd_f, "bwd_main": bwd_f}, peaks,
                                   peak_src, lambda kname: ncu_traffic(kname, w.name)),
        "kernels": {kname: {"launches": kt.launches[kname], "total_ms": kt.ms[kname]}
                    for kname in fa.KERNELS if kt.launches[kname]},
        "clocks": clk.summary(),
        "l2": "flushed (256 MiB write) before every timed step, outside its events",
    }
    del x, q, k, v, do, o, lse, dq, dk, dv, ws
    torch.cuda.empty_cache()
    return out


def run_env(dev):
    """Versions of what produced the line: GPU, driver, CUDA runtime, torch, library."""
    import torch

    from exact_attention_117_b200 import fa
    env = {"gpu": torch.cuda.get_device_name(dev),
           "sm_count": torch.cuda.get_device_properties(dev).multi_processor_count,
           "torch": torch.__version__, "cuda_runtime": torch.version.cuda,
           "library_version": int(fa.load().fa_version()), "driver": None}
    try:
        import pynvml
        pynvml.nvmlInit()
        drv = pynvml.nvmlSystemGetDriverVersion()
        env["driver"] = drv.decode() if isinstance(drv, bytes) else drv
    except Exception:
        try:
            out = subprocess.run(["nvidia-smi", "--query-gpu=driver_version",
                                  "--format=csv,noheader"], capture_output=True, text=True,
                                 timeout=10)
            env["driver"] = out.stdout.strip().splitlines()[0] if out.stdout.strip() else None
        except Exception:
            pass
    return env


def roofline_entry(totals, per_kernel, kernel_flops, peaks, peak_src, traffic_of):
    """The `roofline` object for the kernel with the largest total time:
    achieved = its algorithmic FLOPs per launch / its average launch time,
    against the measured bf16 burst peak (primary) and, for context, the
    datasheet figure."""
    dom = max(totals, key=totals.get)
    peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    if dom in kernel_flops and per_kernel.get(dom):
        achieved = kernel_flops[dom] / (per_kernel[dom] * 1e-3) / 1e12
        return {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": peak_tf,
                "unit": "TFLOP/s", "frac": achieved / peak_tf,
                "peak_source": f"{peak_src} bf16 burst (MEASURED_PEAKS.json)"
                if peak_src == "measured" else "fallback 1590 TFLOP/s",
                "frac_of_nominal": achieved / NOMINAL_BF16_TFLOPS,
                "nominal_peak": NOMINAL_BF16_TFLOPS,
                "traffic": traffic_of(dom),
                "avg_launch_ms": per_kernel[dom],
                "algorithmic_flops_per_launch": kernel_flops[dom]}
    return {"kernel": dom, "bound": "hbm", "achieved": None, "peak": peaks.get("hbm_gbs"),
            "unit": "GB/s", "frac": None, "traffic": None}


def _time_device(fn, flush, stream, warmup=3, iters=10):
    """Median CUDA-event time (ms) of fn(), L2 flushed before each timed call."""
    import torch
    for _ in range(warmup):
        fn()
    times = []
    for _ in range(iters):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    times.sort()
    return times[len(times) // 2]


def run_sweep(args):
    """Supplementary measurements (one JSON line per case, not the headline line):
    the B*H*N = 2^20 sweep (d in {64, 128}, N in 512..8192, causal and full,
    forward and forward+backward) and the split-KV forward on few-head,
    long-sequence problems where one CTA per Q-tile pair leaves SMs idle."""
    import torch

    from exact_attention_117_b200 import fa
    from exact_attention_117_b200.workloads import Workload, make_inputs, sweep_workloads
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    peaks, _ = load_peaks()
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])

    def emit(case, tflops, ms):
        print(json.dumps({"sweep": case, "tflops": round(tflops, 1), "ms": round(ms, 4),
                          "pct_of_peak": round(100 * tflops / peak, 1)}), flush=True)

    class category:
        """Samples the SM clocks while one group of cases runs and prints them
        (a throttled group shows as a low median or an active reason)."""

        def __init__(self, name):
            self.name = name
            self.clk = ClockSampler(0)

        def __enter__(self):
            self.clk.__enter__()
            return self

        def __exit__(self, *exc):
            self.clk.__exit__(*exc)
            if not args.once:
                print(json.dumps({"sweep_clocks": self.name, **self.clk.summary()}), flush=True)
            return False

    if args.sweep in ("all", "c5"):
        with category("c5"):
            for w in sweep_workloads():
                if args.case and w.name != args.case:
                    continue
                x = make_inputs(w, dev)
                o = torch.empty_like(x["q"])
                lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
                g = [torch.empty_like(x["q"]) for _ in range(3)]
                ws = torch.empty(fa.workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8,
                                 device=dev)
                for causal in (True, False):
                    fwd_f, bwd_f = attention_flops(w.B, w.H, w.N, w.d, causal)

                    def fwd():
                        fa.forward(x["q"], x["k"], x["v"], causal=causal, out=o, lse=lse,
                                   stream=stream)

                    def step():
                        fwd()
                        fa.backward(x["q"], x["k"], x["v"], o, lse, x["do"], causal=causal,
                                    dq=g[0], dk=g[1], dv=g[2], workspace=ws, stream=stream)
                    tag = f"{w.name} {'causal' if causal else 'full'}"
                    if args.once:  # two forwards and one backward, untimed (for ncu)
                        fwd()
                        step()
                        continue
                    ms = _time_device(fwd, flush, stream)
                    emit(f"{tag} fwd", fwd_f / (ms * 1e-3) / 1e12, ms)
                    ms = _time_device(step, flush, stream)
                    emit(f"{tag} fwd+bwd", (fwd_f + bwd_f) / (ms * 1e-3) / 1e12, ms)
                del x, o, lse, g, ws
    if args.sweep in ("all", "bwd"):
        with category("bwd"):
            # the two backward variants on the headline workloads: fa_bwd (dQ by
            # fp32 atomics) and fa_bwd_deterministic (dQ by a query-tile pass)
            from exact_attention_117_b200.workloads import WORKLOADS
            for name in (("c3",) if args.once else ("c3", "c4")):
                w = WORKLOADS[name]
                x = make_inputs(w, dev)
                o = torch.empty_like(x["q"])
                lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
                g = [torch.empty_like(x["q"]) for _ in range(3)]
                ws = torch.empty(fa.workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8,
                                 device=dev)
                fwd_f, bwd_f = attention_flops(w.B, w.H, w.N, w.d, True)

                def fwd():
                    fa.forward(x["q"], x["k"], x["v"], causal=True, out=o, lse=lse, stream=stream)

                def bwd(det):
                    fa.backward(x["q"], x["k"], x["v"], o, lse, x["do"], causal=True, dq=g[0],
                                dk=g[1], dv=g[2], workspace=ws, stream=stream, deterministic=det)
                if args.once:  # two rounds of fwd, atomic bwd, deterministic bwd (for ncu)
                    for _ in range(2):
                        fwd()
                        bwd(False)
                        bwd(True)
                    continue
                ms = _time_device(fwd, flush, stream)
                emit(f"{name} causal fwd", fwd_f / (ms * 1e-3) / 1e12, ms)
                for det in (False, True):
                    fwd()
                    with fa.KernelTimer() as kt:
                        ms = _time_device(lambda: bwd(det), flush, stream)
                    per = {k: round(kt.ms[k] / kt.launches[k], 4) for k in kt.ms if kt.launches[k]}
                    emit(f"{name} causal bwd {'deterministic' if det else 'atomic dQ'} "
                         f"(per-kernel ms {per})", bwd_f / (ms * 1e-3) / 1e12, ms)
                del x, o, lse, g, ws
    if args.sweep in ("all", "kv_outer"):
        with category("kv_outer"):
            # loop-order ablation: the forward with the Q tiles outside (fa_fwd)
            # against the FlashAttention-1 order (KV tiles outside, one CTA per head)
            for B, H, N, causal in ((2, 16, 4096, True), (2, 16, 4096, False), (8, 32, 1024, True)):
                w = Workload(f"kv_outer_B{B}_H{H}_N{N}", B, H, N, 128, seed_base=600)
                x = make_inputs(w, dev, with_do=False)
                o = torch.empty_like(x["q"])
                lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
                wsk = torch.empty(fa.kv_outer_workspace_size(B, H, N, 128), dtype=torch.uint8,
                                  device=dev)
                fwd_f, _ = attention_flops(B, H, N, 128, causal)
                tag = f"{w.name} d=128 {'causal' if causal else 'full'}"

                def q_outer():
                    fa.forward(x["q"], x["k"], x["v"], causal=causal, out=o, lse=lse, stream=stream)

                def kv_outer():
                    fa.forward_kv_outer(x["q"], x["k"], x["v"], causal=causal, out=o, lse=lse,
                                        workspace=wsk, stream=stream)
                for name, fn in (("fwd Q-outer", q_outer), ("fwd KV-outer", kv_outer)):
                    if args.once:
                        fn()
                        continue
                    ms = _time_device(fn, flush, stream)
                    emit(f"{tag} {name}", fwd_f / (ms * 1e-3) / 1e12, ms)
                del x, o, lse, wsk
    if args.sweep in ("all", "splitkv"):
        with category("splitkv"):
            for B, H, N, causal in ((1, 1, 16384, False), (1, 1, 16384, True), (1, 2, 32768, False),
                                    (1, 4, 8192, False)):
                w = Workload(f"few_heads_B{B}_H{H}_N{N}", B, H, N, 128, seed_base=500)
                x = make_inputs(w, dev, with_do=False)
                o = torch.empty_like(x["q"])
                lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
                fwd_f, _ = attention_flops(B, H, N, 128, causal)
                tag = f"{w.name} d=128 {'causal' if causal else 'full'}"
                ms = _time_device(lambda: fa.forward(x["q"], x["k"], x["v"], causal=causal, out=o,
                                                     lse=lse, stream=stream), flush, stream)
                emit(f"{tag} fwd", fwd_f / (ms * 1e-3) / 1e12, ms)
                for splits in (2, 4, 8):
                    wsz = fa.splitkv_workspace_size(B, H, N, 128, splits)
                    wsp = torch.empty(wsz, dtype=torch.uint8, device=dev)
                    ms = _time_device(lambda: fa.forward_splitkv(
                        x["q"], x["k"], x["v"], causal=causal, num_splits=splits, out=o, lse=lse,
                        workspace=wsp, stream=stream), flush, stream)
                    emit(f"{tag} fwd split-KV x{splits}", fwd_f / (ms * 1e-3) / 1e12, ms)
    fa.check_device_error(stream)


TRAFFIC_N = (128, 256, 512, 1024, 2048, 4096)
TRAFFIC_BH = 16  # B=1, H=16, d=128, full (non-causal) attention


def run_traffic(args):
    """One launch per case, for an ncu DRAM-bytes capture: for each N, the
    forward kernel, then a naive attention that materialises S and P in HBM
    (torch: S = (scale Q) K^T, P = softmax(S), O = P V, all bf16, three
    kernels).  All inputs are created and synchronised before the first case,
    so the captured kernels after the first ``fwd_kernel`` are exactly the cases,
    in order."""
    import torch

    from exact_attention_117_b200 import fa
    from exact_attention_117_b200.workloads import Workload, make_inputs
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    d = 128
    cases = []
    for n in TRAFFIC_N:
        w = Workload(f"traffic_N{n}", 1, TRAFFIC_BH, n, d, seed_base=700 + n)
        x = make_inputs(w, dev, with_do=False)
        x["qs"] = (x["q"].float() * w.scale).to(torch.bfloat16)
        x["kt"] = x["k"].transpose(-1, -2)
        x["o"] = torch.empty_like(x["q"])
        x["lse"] = torch.empty((1, TRAFFIC_BH, n), dtype=torch.float32, device=dev)
        cases.append((w, x))
    torch.cuda.synchronize()
    for w, x in cases:
        fa.forward(x["q"], x["k"], x["v"], causal=False, scale=w.scale, out=x["o"], lse=x["lse"])
        s = torch.matmul(x["qs"], x["kt"])
        p = torch.softmax(s, dim=-1)
        torch.matmul(p, x["v"])
        del s, p
    torch.cuda.synchronize()
    fa.check_device_error()
    print(json.dumps({"traffic_cases": [w.N for w, _ in cases], "B": 1, "H": TRAFFIC_BH,
                      "d": d}))


def traffic_report(csv_path):
    """Markdown table: ncu dram__bytes of each case against the page-2 traffic
    model (oracle/traffic_model.py) times the B*H heads."""
    import csv

    from oracle.traffic_model import memory_work
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "Tbyte": 1e12}
    kernels = {}
    with open(csv_path, newline="") as f:
        lines = [ln for ln in f if ln.startswith('"')]
    for row in csv.DictReader(lines):
        k = kernels.setdefault(int(row["ID"]), {"name": row["Kernel Name"]})
        k[row["Metric Name"]] = float(row["Metric Value"].replace(",", "")) * \
            scale.get(row["Metric Unit"], 1)
    seq = [kernels[i] for i in sorted(kernels)]
    first = next(i for i, k in enumerate(seq) if "fwd_kernel" in k["name"])
    groups = []
    for k in seq[first:]:
        if "fwd_kernel" in k["name"]:
            groups.append({"fwd": k, "naive": []})
        else:
            groups[-1]["naive"].append(k)
    rd, wr = "dram__bytes_read.sum", "dram__bytes_write.sum"
    out = ["| N | fwd read MB (model / ncu) | fwd write MB (model / ncu) | "
           "naive read MB (model / ncu) | naive write MB (model / ncu) | naive kernels |",
           "|---|---|---|---|---|---|"]
    for n, g in zip(TRAFFIC_N, groups):
        m = memory_work(n, 128, elem_bytes=2, lse_bytes=4)
        bh = TRAFFIC_BH
        nr = sum(k.get(rd, 0) for k in g["naive"])
        nw = sum(k.get(wr, 0) for k in g["naive"])
        out.append(f"| {n} | {m['flash_read_bytes'] * bh / 1e6:.2f} / {g['fwd'].get(rd, 0) / 1e6:.2f}"
                   f" | {m['flash_write_bytes'] * bh / 1e6:.2f} / {g['fwd'].get(wr, 0) / 1e6:.2f}"
                   f" | {m['naive_read_bytes'] * bh / 1e6:.2f} / {nr / 1e6:.2f}"
                   f" | {m['naive_write_bytes'] * bh / 1e6:.2f} / {nw / 1e6:.2f}"
                   f" | {len(g['naive'])} |")
    text = "\n".join(out)
    print(text)
    return text


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="c3", choices=["c3", "c4"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-chunks", type=int, default=E2E_CHUNKS,
                    help="groups of (b, h) slices the end-to-end leg pipelines its copies over")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-long-context", action="store_true",
                    help="skip the long-context (B=1 H=32 N=16384) leg of the default line")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--sweep", choices=["all", "c5", "splitkv", "kv_outer", "bwd"], default=None,
                    help="supplementary per-case measurements instead of the headline line")
    ap.add_argument("--once", action="store_true",
                    help="with --sweep c5, kv_outer or bwd: run the cases once, untimed (for ncu)")
    ap.add_argument("--case", default=None,
                    help="with --sweep c5: only this workload (e.g. c5_d64_n4096)")
    ap.add_argument("--traffic", action="store_true",
                    help="one launch per traffic-model case (run under ncu for DRAM bytes)")
    ap.add_argument("--traffic-report", metavar="NCU_CSV", default=None,
                    help="compare an ncu --csv capture of --traffic with the traffic model")
    args = ap.parse_args()
    if args.sweep:
        run_sweep(args)
        return
    if args.traffic:
        run_traffic(args)
        return
    if args.traffic_report:
        traffic_report(args.traffic_report)
        return

    from exact_attention_117_b200.workloads import WORKLOADS
    w = WORKLOADS[args.workload]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        run_reference(args, w, rank)
        return

    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
