#!/usr/bin/env python
"""Benchmark of the grouped / latent-KV attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lka|reference] [--workload NAME]

Default workload: one GQA decode attention layer shaped like Llama-3.1-8B
(32 query heads, 8 KV heads, d_h = 128, bf16 KV cache, batch 64, s_q = 1,
per-sequence cache lengths uniform in [1024, 8192]; q/k/v N(0,1); scale
1/sqrt(128)).  A step is one gqa_attn call over the whole batch: split-KV
decode kernel plus log-sum-exp merge.  Inputs are seeded synthetic tensors
(synthetic.py) resident in HBM; their 2.1 GB exceed the 126 MB L2, and L2 is
flushed between timed steps anyway.

Prints ONE JSON line (rank 0).  `value` is the algorithmic HBM traffic of the
step (every cache byte once, q read once, out written once) divided by the
device time of a step, summed over ranks (weak scaling: every rank runs its own
replica of the workload; there is no collective on the data path).

--impl reference times the fp64 CPU oracle on the host cores instead (rank 0
only), on the same workload, metric and unit; each step is a bounded sample.

Under torchrun (N > 1) ranks synchronise with a barrier before and after the
timed region and the slowest rank's time is reported.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402
from latent_kv_attention_b200 import costs  # noqa: E402

METRIC = "decode-attention HBM GB/s (% of peak), TFLOPS (% of roofline), tokens/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ----------------------------------------------------------------------------- helpers
def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=FALLBACK_HBM_GBS, bf16_tflops=FALLBACK_BF16_TFLOPS, bf16_tflops_sustained=1400.0,
                source="fallback")


def source_hash(*rel_paths):
    h = hashlib.sha256()
    for r in rel_paths:
        with open(os.path.join(ROOT, r), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str, src_files):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel}@{workload}")
    if not e or e.get("source_hash") != source_hash(*src_files):
        return None
    return float(e["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def wait_first_sample(self, timeout_s=5.0):
        """Blocks until nvidia-smi has written a sample (so that samples cover what follows)."""
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < timeout_s:
            self.fh.flush()
            if os.path.getsize(self.path) > 0:
                return
            time.sleep(0.05)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = max(smax, float(parts[2]))
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- workloads
class GqaDecode:
    """One gqa_attn call over the Llama-3.1-8B-shaped decode batch."""

    kernel = "gqa_decode_kernel"
    src = ("latent_kv_attention_b200/csrc/gqa_decode.cu", "latent_kv_attention_b200/csrc/common.cuh")

    def __init__(self, name, device, reference=False):
        self.w = synthetic.WORKLOADS[name]
        w = self.w
        self.name = name
        self.inp = synthetic.make(w, device=device)
        self.lens = self.inp["cache_lens"].cpu().tolist()
        self.bytes = costs.gqa_bytes(self.lens, w["h_q"], w["h_kv"], w["d"], w["s_q"])
        self.flops = costs.gqa_flops(self.lens, w["h_q"], w["d"], w["s_q"], w["causal"])
        self.tokens = w["B"] * w["s_q"]
        if reference:
            return  # the reference arm only runs the oracle
        import latent_kv_attention_b200 as lka

        self.lka = lka
        self.out = torch.empty_like(self.inp["q"])
        ws = lka.library().gqa_attn_workspace_size(w["B"], w["h_q"], w["h_kv"], w["s_q"], w["d"], w["L_hi"])
        self.launches = 2 if ws > 256 else 1  # decode kernel (+ merge kernel when the cache is split)
        # end-to-end: the step's inputs (q, cache_lens) come from pinned host memory, out goes back to it
        self.q_host = self.inp["q"].cpu().pin_memory()
        self.lens_host = self.inp["cache_lens"].cpu().pin_memory()
        self.out_host = torch.empty_like(self.q_host).pin_memory()
        self.h2d = self.q_host.numel() * self.q_host.element_size() + self.lens_host.numel() * 4
        self.d2h = self.out_host.numel() * self.out_host.element_size()

    def step(self):
        i = self.inp
        self.lka.gqa_attn(i["q"], i["k"], i["v"], i["cache_lens"], causal=self.w["causal"], scale=i["scale"],
                          out=self.out)

    def step_e2e(self):
        i = self.inp
        i["q"].copy_(self.q_host, non_blocking=True)
        i["cache_lens"].copy_(self.lens_host, non_blocking=True)
        self.lka.gqa_attn(i["q"], i["k"], i["v"], i["cache_lens"], causal=self.w["causal"], scale=i["scale"],
                          out=self.out)
        self.out_host.copy_(self.out, non_blocking=True)

    def config(self):
        w = self.w
        return {"workload": self.name, "B": w["B"], "h_q": w["h_q"], "h_kv": w["h_kv"], "d_h": w["d"],
                "s_q": w["s_q"], "cache_lens": f"uniform [{w['L_lo']}, {w['L_hi']}]", "causal": w["causal"],
                "l2": "K/V cache larger than L2; L2 flushed between timed steps",
                "parallelism": "replicas"}

    # oracle on the host cores, on a bounded sample of the same workload
    def oracle_sample(self, target_s: float):
        import oracle

        i = self.inp
        n = 8
        rows = list(range(n))
        sub = {k: (v[:n].cpu() if isinstance(v, torch.Tensor) else v) for k, v in i.items()}
        q64, k64, v64 = sub["q"].double(), sub["k"].double(), sub["v"].double()
        t0 = time.perf_counter()
        oracle.gqa(q64, k64, v64, sub["cache_lens"], self.w["causal"], i["scale"])
        t1 = time.perf_counter() - t0
        reps = max(1, int(math.ceil(target_s / max(t1, 1e-3))) - 1)
        t0 = time.perf_counter()
        for _ in range(reps):
            oracle.gqa(q64, k64, v64, sub["cache_lens"], self.w["causal"], i["scale"])
        dt = time.perf_counter() - t0
        lens = [self.lens[r] for r in rows]
        w = self.w
        nbytes = costs.gqa_bytes(lens, w["h_q"], w["h_kv"], w["d"], w["s_q"]) * reps
        cores = oracle.threads_used(0, n * w["h_q"])
        return dict(value=nbytes / dt / 1e9, unit="GB/s", cores=cores, kind="oracle",
                    sample=f"first {n} of {w['B']} sequences ({sum(lens)} cache tokens), {reps} repetitions, "
                           f"{dt:.1f} s", seconds=dt, reps=reps, n=n)


WORKLOAD_CLASSES = {"gqa_decode_llama8b": GqaDecode, "gqa_decode_llama8b_b16": GqaDecode}


# ----------------------------------------------------------------------------- arms
def run_lka(args, rank, world, device):
    import latent_kv_attention_b200 as lka

    wl = WORKLOAD_CLASSES[args.workload](args.workload, device)
    pk = peaks()
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    for _ in range(max(3, args.warmup)):
        wl.step()
    torch.cuda.synchronize()
    lka.clear_status()

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(device.index if device.index is not None else 0)
    clocks.start()
    clocks.wait_first_sample()
    # keep the GPU under this load for ~1 s before the timed region so that the clock samples
    # (every 200 ms) describe the state the timed steps run in; the sampler runs through both
    t_soak = time.time()
    while time.time() - t_soak < 1.0:
        for _ in range(20):
            wl.step()
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    lka.kernel_timing(True)
    for s in range(args.steps):
        flush.zero_()  # L2 flush, outside the events
        starts[s].record()
        wl.step()
        ends[s].record()
    torch.cuda.synchronize()
    n_timed, kern_ms = lka.kernel_timing_read()
    lka.kernel_timing(False)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clk = clocks.stop()
    step_ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / args.steps
    status = lka.device_status()
    if status != 0:
        raise RuntimeError(f"device status after the timed region: {lka.status_string(status)}")

    # end to end through the public API with pinned host buffers
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(2):
        wl.step_e2e()
    torch.cuda.synchronize()
    e2e_total = 0.0
    for s in range(args.steps):
        flush.zero_()
        e_start.record()
        wl.step_e2e()
        e_end.record()
        e_end.synchronize()
        e2e_total += e_start.elapsed_time(e_end)
    e2e_ms = e2e_total / args.steps

    t = torch.tensor([step_ms, e2e_ms, kern_ms / max(1, n_timed)], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    step_ms, e2e_ms, kern_avg_ms = t.tolist()
    if rank != 0:
        return None

    gbs = wl.bytes * world / (step_ms * 1e-3) / 1e9
    tflops = wl.flops * world / (step_ms * 1e-3) / 1e12
    achieved = wl.bytes / (kern_avg_ms * 1e-3) / 1e9
    traffic = recorded_traffic(wl.kernel, wl.name, wl.src)
    line = {
        "metric": METRIC, "value": round(gbs, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) inputs, see synthetic.py)",
        "config": wl.config(),
        "tokens_per_s": round(wl.tokens * world / (step_ms * 1e-3), 1),
        "tflops": round(tflops, 3),
        "hbm_frac_of_peak": round(gbs / world / pk["hbm_gbs"], 4),
        "roofline": {"bound": "hbm", "kernel": wl.kernel, "achieved": round(achieved, 1), "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved / pk["hbm_gbs"], 4), "traffic": traffic,
                     "algorithmic_bytes_per_launch": wl.bytes, "launch_ms": round(kern_avg_ms, 4),
                     "peak_source": pk["source"] + " (MEASURED_PEAKS.json hbm_gbs)" if pk["source"] == "measured"
                     else "fallback"},
        "e2e": {"value": round(wl.bytes * world / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                "h2d_bytes_per_step": wl.h2d, "d2h_bytes_per_step": wl.d2h, "ms_per_step": round(e2e_ms, 4)},
        "gpu_launches": wl.launches * args.steps,
        "clocks": clk,
    }
    if world == 1 and not args.no_cpu_baseline:
        cb = wl.oracle_sample(args.cpu_seconds)
        line["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
        line["cpu_baseline"]["value"] = round(cb["value"], 4)
    return line


def run_reference(args, rank, world, device):
    """The oracle as it stands, on the host cores, same workload/metric/unit; rank 0 only."""
    if rank != 0:
        return None
    wl = WORKLOAD_CLASSES[args.workload](args.workload, device, reference=True)
    per_step = max(1.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        wl.oracle_sample(0.0)
    vals, secs, last = [], 0.0, None
    for _ in range(args.steps):
        last = wl.oracle_sample(min(per_step, 5.0))
        vals.append(last["value"])
        secs += last["seconds"]
    v = statistics.median(vals)
    return {
        "impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) inputs, see synthetic.py)", "config": wl.config(),
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": last["cores"], "kind": "oracle",
                         "sample": last["sample"]},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["lka", "reference"], default="lka")
    ap.add_argument("--workload", choices=sorted(WORKLOAD_CLASSES), default="gqa_decode_llama8b")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "lka" and not torch.cuda.is_available():
        raise SystemExit("bench.py --impl lka needs a CUDA device")
    device = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
    if device.type == "cuda":
        torch.cuda.set_device(device)
    if world > 1:
        backend = "nccl" if device.type == "cuda" else "gloo"
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    try:
        line = (run_lka if args.impl == "lka" else run_reference)(args, rank, world, device)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
