#!/usr/bin/env python
"""Benchmark of the grouped / latent-KV attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lka|reference] [--workload NAME] [--sweep]

Default workload: one GQA decode attention layer shaped like Llama-3.1-8B
(32 query heads, 8 KV heads, d_h = 128, bf16 KV cache, batch 64, s_q = 1,
per-sequence cache lengths uniform in [1024, 8192]; q/k/v N(0,1); scale
1/sqrt(128)).  A step is one gqa_attn call over the whole batch: split-KV
decode kernel plus log-sum-exp merge.  Inputs are seeded synthetic tensors
(synthetic.py) resident in HBM; their 2.1 GB exceed the 126 MB L2, and L2 is
flushed between timed steps anyway.

Unless --no-extras is given, the line also carries `other_paths`: the same
measurement (step time, GB/s, TFLOP/s, tokens/s, roofline of the main kernel,
end-to-end time) for the GQA layer over a paged cache (64-token pages) and
over an e4m3 cache, the
GQLA latent decode layer on the MQA-absorbed path (s_q = 1 and 2; s_q = 1 also
over a paged latent cache, and top-2048 sparse over a 16K cache), on the
per-group GQA path (s_q = 2), and for the GTA causal prefill.

Prints ONE JSON line (rank 0).  `value` is the algorithmic HBM traffic of the
step (every cache byte once, q read once, out written once) divided by the
device time of a step, summed over ranks (weak scaling: every rank runs its own
replica of the workload; there is no collective on the data path).

--sweep measures the long-context decode sweep instead (batch 64, s_q 1,
every cache 1K, 2K, ... 64K tokens, GQA layout and latent layout on the
MQA-absorbed path) and prints one JSON line with an entry per point.

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
import re
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic  # noqa: E402
from latent_kv_attention_b200 import costs, sharding  # noqa: E402

METRIC = "decode-attention HBM GB/s (% of peak), TFLOPS (% of roofline), tokens/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
# NVIDIA's B200 datasheet figures, reported beside the measured peaks: HBM3e 8 TB/s, dense bf16 2.25 PFLOP/s
DATASHEET_HBM_GBS = 8000.0
DATASHEET_BF16_TFLOPS = 2250.0


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


def _code_only(text: str) -> str:
    """C/C++/CUDA source without its comments and blank lines (a comment edit leaves the kernel as it was)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def source_hash(*rel_paths):
    h = hashlib.sha256()
    for r in rel_paths:
        with open(os.path.join(ROOT, r), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
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
def _pinned(t):
    return t.cpu().pin_memory()


def _nbytes(*ts):
    return sum(t.numel() * t.element_size() for t in ts)


class Workload:
    """One attention-layer call over a synthetic batch (a bench `step`), with its algorithmic costs."""

    kernel = ""
    src = ()
    bound = "hbm"
    oracle_n = 8  # sequences in the oracle's bounded sample

    def __init__(self, name, device, reference=False):
        self.name = name
        self.w = synthetic.WORKLOADS[name]
        self.device = device
        self.inp = synthetic.make(self.w, device=device)
        self.lens = self.inp["cache_lens"].cpu().tolist()
        self.setup_costs()
        if reference:
            return
        import latent_kv_attention_b200 as lka

        self.lka = lka
        self.setup_device()

    # e2e: per-step inputs come from pinned host buffers, the result goes back to one
    def step_e2e(self):
        for dst, src in self.h2d_pairs:
            dst.copy_(src, non_blocking=True)
        self.step()
        self.out_host.copy_(self.out, non_blocking=True)

    @property
    def h2d(self):
        return sum(_nbytes(src) for _, src in self.h2d_pairs)

    @property
    def d2h(self):
        return _nbytes(self.out_host)


class GqaDecode(Workload):
    """gqa_attn over the Llama-3.1-8B-shaped decode batch: split-KV decode kernel (the mma.sync instance for bf16
    caches) + log-sum-exp merge."""

    kernel = "gqa_decode_mma8_kernel"  # the 8-row tensor-core form (4 query rows per KV head)
    src = ("latent_kv_attention_b200/csrc/gqa_decode.cu", "latent_kv_attention_b200/csrc/common.cuh",
           "latent_kv_attention_b200/csrc/tc.cuh")

    def setup_costs(self):
        w = self.w
        self.bytes = costs.gqa_bytes(self.lens, w["h_q"], w["h_kv"], w["d"], w["s_q"])
        self.flops = costs.gqa_flops(self.lens, w["h_q"], w["d"], w["s_q"], w["causal"])
        self.tokens = w["B"] * w["s_q"]

    def setup_device(self):
        w, i = self.w, self.inp
        self.out = torch.empty_like(i["q"])
        ws = self.lka.library().gqa_attn_workspace_size(w["B"], w["h_q"], w["h_kv"], w["s_q"], w["d"], w["L_hi"])
        self.launches = 2 if ws > 256 else 1  # decode kernel (+ merge kernel when the cache is split)
        self.h2d_pairs = [(i["q"], _pinned(i["q"])), (i["cache_lens"], _pinned(i["cache_lens"]))]
        self.out_host = torch.empty_like(self.out, device="cpu").pin_memory()

    def step(self):
        i = self.inp
        self.lka.gqa_attn(i["q"], i["k"], i["v"], i["cache_lens"], causal=self.w["causal"], scale=i["scale"],
                          out=self.out)

    def config(self):
        w = self.w
        return {"workload": self.name, "B": w["B"], "h_q": w["h_q"], "h_kv": w["h_kv"], "d_h": w["d"],
                "s_q": w["s_q"],
                "cache_lens": w["L_hi"] if w["L_lo"] == w["L_hi"] else f"uniform [{w['L_lo']}, {w['L_hi']}]",
                "causal": w["causal"],
                "l2": "K/V cache larger than L2; L2 flushed between timed steps", "parallelism": "replicas"}

    def oracle_run(self, n):
        import oracle

        sub = {k: (v[:n].cpu().double() if isinstance(v, torch.Tensor) and k != "cache_lens" else v)
               for k, v in self.inp.items()}
        lens = self.inp["cache_lens"][:n].cpu()
        w = self.w
        fn = lambda: oracle.gqa(sub["q"], sub["k"], sub["v"], lens, w["causal"], self.inp["scale"])  # noqa: E731
        nbytes = costs.gqa_bytes(lens.tolist(), w["h_q"], w["h_kv"], w["d"], w["s_q"])
        return fn, nbytes, oracle.threads_used(0, n * w["h_q"]), f"first {n} of {w['B']} sequences"


class GqaDecodeSharded(GqaDecode):
    """gqa_attn on this rank's slice of the KV heads and their query heads (`--shard heads`): head-axis tensor
    parallelism with no exchange inside the attention (latent_kv_attention_b200.sharding).  Every rank draws the
    same seeded layer and keeps its slice; the job's time is the slowest rank's, its bytes the whole layer's."""

    def __init__(self, name, device, rank, world, reference=False):
        self.rank, self.world = rank, world
        super().__init__(name, device, reference)

    def setup_costs(self):
        self.full_w = self.w
        w = dict(self.w)
        (q0, q1), (k0, k1) = sharding.gqa_head_slice(w["h_q"], w["h_kv"], self.rank, self.world)
        i = self.inp
        i["q"] = i["q"][:, q0:q1].contiguous()
        i["k"] = i["k"][:, k0:k1].contiguous()
        i["v"] = i["v"][:, k0:k1].contiguous()
        w["h_q"], w["h_kv"] = q1 - q0, k1 - k0
        self.w = w
        super().setup_costs()

    def config(self):
        c = super().config()
        c["h_q"], c["h_kv"] = self.full_w["h_q"], self.full_w["h_kv"]
        c["parallelism"] = f"heads{self.world} (KV heads split over the ranks, no collective in the call)"
        return c


class GqaDecodePaged(GqaDecode):
    """gqa_attn_paged over the same decode batch with the K/V cache in 64-token pages of a shuffled pool."""

    def setup_device(self):
        super().setup_device()
        for k in ("k", "v"):  # the contiguous copies are not used by the paged step
            self.inp.pop(k, None)
        torch.cuda.empty_cache()

    def step(self):
        i = self.inp
        self.lka.gqa_attn_paged(i["q"], i["k_pages"], i["v_pages"], i["block_table"], i["cache_lens"],
                                causal=self.w["causal"], scale=i["scale"], out=self.out)

    def config(self):
        c = super().config()
        c["page_size"] = self.w["page_size"]
        c["cache_layout"] = "paged (shuffled page pool + block table)"
        return c


class GqaDecodeFp8(GqaDecode):
    """gqa_attn_fp8kv over the same decode batch with the K/V cache in e4m3 (one scale per KV head)."""

    kernel = "gqa_decode_mma8_kernel"  # its e4m3 instance (f16 MMAs)

    def setup_costs(self):
        w = self.w
        self.bytes = costs.gqa_bytes(self.lens, w["h_q"], w["h_kv"], w["d"], w["s_q"], kv_elem=1)
        self.flops = costs.gqa_flops(self.lens, w["h_q"], w["d"], w["s_q"], w["causal"])
        self.tokens = w["B"] * w["s_q"]

    def setup_device(self):
        w, i = self.w, self.inp
        self.out = torch.empty_like(i["q"])
        ws = self.lka.library().gqa_attn_fp8kv_workspace_size(w["B"], w["h_q"], w["h_kv"], w["s_q"], w["d"], w["L_hi"])
        self.launches = 2 if ws > 256 else 1
        self.h2d_pairs = [(i["q"], _pinned(i["q"])), (i["cache_lens"], _pinned(i["cache_lens"]))]
        self.out_host = torch.empty_like(self.out, device="cpu").pin_memory()

    def step(self):
        i = self.inp
        self.lka.gqa_attn_fp8kv(i["q"], i["k"], i["v"], i["k_scale"], i["v_scale"], i["cache_lens"],
                                causal=self.w["causal"], scale=i["scale"], out=self.out)

    def config(self):
        c = super().config()
        c["cache_dtype"] = "e4m3 (per-KV-head scales)"
        return c


class GqaPrefill(GqaDecode):
    """gqa_attn causal prefill of the Llama-3.1-8B layer (4096 queries over their own cache): the tensor-core
    prefill kernel (128-query x 128-key tiles, tcgen05 MMAs, one CTA per query tile and head)."""

    kernel = "gta_attn_kernel"
    src = ("latent_kv_attention_b200/csrc/gta_attn.cu", "latent_kv_attention_b200/csrc/tc.cuh",
           "latent_kv_attention_b200/csrc/common.cuh")
    bound = "tensor"
    oracle_n = 1

    def kernel_work(self, pk):
        return "tensor", self.flops

    def setup_device(self):
        super().setup_device()
        self.launches = 1  # 32 query tiles x 32 heads x 2 sequences fill the GPU: no key splits to merge

    def config(self):
        c = super().config()
        c["l2"] = "inputs 134 MB (q, k, v); L2 flushed between timed steps"
        return c

    def oracle_run(self, n):
        import oracle

        w, i = self.w, self.inp
        # a bounded sample: the last 256 query positions of the first sequence (each sees 3841 .. 4096 keys)
        t0 = w["s_q"] - 256
        q = i["q"][:1, :, t0:].cpu().double()
        k, v = i["k"][:1].cpu().double(), i["v"][:1].cpu().double()
        lens = torch.tensor([w["L_hi"]], dtype=torch.int32)
        fn = lambda: oracle.gqa(q, k, v, lens, True, i["scale"])  # noqa: E731
        nbytes = costs.gqa_bytes([w["L_hi"]], w["h_q"], w["h_kv"], w["d"], 256)
        return fn, nbytes, oracle.threads_used(0, w["h_q"]), "last 256 queries of the first sequence"


class LatentAbsorbed(Workload):
    """latent_absorbed_attn over the GQLA/MLA decode batch: absorb GEMM, latent attention, up-projection."""

    kernel = "latent_attn_kernel"
    src = ("latent_kv_attention_b200/csrc/latent_attn.cu", "latent_kv_attention_b200/csrc/tc.cuh",
           "latent_kv_attention_b200/csrc/common.cuh")

    def setup_costs(self):
        w = self.w
        self.bytes = costs.latent_bytes(self.lens, w["h_q"], w["g"], w["d_h"], w["r_kv"], w["d_r"], w["s_q"])
        self.core_flops = costs.latent_core_flops(self.lens, w["h_q"], w["r_kv"], w["d_r"], w["s_q"], w["causal"])
        self.flops = self.core_flops + costs.latent_proj_flops(w["B"], w["h_q"], w["d_h"], w["r_kv"], w["s_q"])
        self.tokens = w["B"] * w["s_q"]

    def kernel_work(self, pk):
        """(bound, achieved-unit work per launch, peak) of the attention kernel: roofline = slower of the two."""
        cache = sum(self.lens) * (self.w["r_kv"] + self.w["d_r"]) * 2
        t_mem = cache / (pk["hbm_gbs"] * 1e9)
        t_tc = self.core_flops / (pk["bf16_tflops"] * 1e12)
        return ("tensor", self.core_flops) if t_tc > t_mem else ("hbm", cache)

    def setup_device(self):
        w, i = self.w, self.inp
        self.out = torch.empty_like(i["q_c"])
        ws = self.lka.library().latent_absorbed_attn_workspace_size(w["B"], w["h_q"], w["g"], w["s_q"], w["d_h"],
                                                                    w["r_kv"], w["d_r"], w["L_hi"])
        rows = w["B"] * w["s_q"] * w["h_q"]
        split = ws > 256 + 2 * (rows * w["r_kv"] * 2 + 256)
        self.launches = 3 + (1 if split else 0)  # absorb GEMM, attention, (+ merge), up-projection GEMM
        self.h2d_pairs = [(i["q_c"], _pinned(i["q_c"])), (i["q_r"], _pinned(i["q_r"])),
                          (i["cache_lens"], _pinned(i["cache_lens"]))]
        self.out_host = torch.empty_like(self.out, device="cpu").pin_memory()

    def step(self):
        i = self.inp
        self.lka.latent_absorbed_attn(i["q_c"], i["q_r"], i["w_uk"], i["w_uv"], i["latent"], i["cache_lens"],
                                      causal=self.w["causal"], scale=i["scale"], out=self.out)

    def config(self):
        w = self.w
        return {"workload": self.name, "B": w["B"], "h_q": w["h_q"], "g": w["g"], "d_h": w["d_h"], "r_kv": w["r_kv"],
                "d_r": w["d_r"], "s_q": w["s_q"], "cache_lens": w["L_hi"], "causal": w["causal"],
                "path": "MQA-absorbed", "l2": "latent cache larger than L2; L2 flushed between timed steps",
                "parallelism": "replicas"}

    def oracle_run(self, n):
        import oracle

        i = self.inp
        sub = {k: (v[:n].cpu().double() if k in ("q_c", "q_r", "latent") else v) for k, v in i.items()}
        lens = i["cache_lens"][:n].cpu()
        w_uk, w_uv = i["w_uk"].cpu().double(), i["w_uv"].cpu().double()
        w = self.w
        fn = lambda: oracle.latent_absorbed(sub["q_c"], sub["q_r"], w_uk, w_uv, sub["latent"], lens,  # noqa: E731
                                            w["causal"], i["scale"])
        nbytes = costs.latent_bytes(lens.tolist(), w["h_q"], w["g"], w["d_h"], w["r_kv"], w["d_r"], w["s_q"])
        return fn, nbytes, oracle.threads_used(0, n * w["h_q"]), f"first {n} of {w['B']} sequences"


class LatentAbsorbedFp8(LatentAbsorbed):
    """latent_absorbed_attn_fp8kv over the same decode batch with the latent cache in e4m3 (one scale for the
    latent part, one for the RoPE key)."""

    def setup_costs(self):
        super().setup_costs()
        w = self.w
        self.bytes = costs.latent_bytes(self.lens, w["h_q"], w["g"], w["d_h"], w["r_kv"], w["d_r"], w["s_q"],
                                        cache_elem=1)

    def kernel_work(self, pk):
        cache = sum(self.lens) * (self.w["r_kv"] + self.w["d_r"])
        t_mem = cache / (pk["hbm_gbs"] * 1e9)
        t_tc = self.core_flops / (pk["bf16_tflops"] * 1e12)  # f16 tensor-core rate = bf16 rate
        return ("tensor", self.core_flops) if t_tc > t_mem else ("hbm", cache)

    def step(self):
        i = self.inp
        self.lka.latent_absorbed_attn_fp8kv(i["q_c"], i["q_r"], i["w_uk"], i["w_uv"], i["latent8"], i["kv_scale"],
                                            i["cache_lens"], causal=self.w["causal"], scale=i["scale"], out=self.out)

    def config(self):
        c = super().config()
        c["cache_dtype"] = "e4m3 (per-part scales)"
        return c

    def oracle_run(self, n):
        import oracle

        i = self.inp
        sub = {k: (v[:n].cpu() if k in ("q_c", "q_r", "latent8") else v) for k, v in i.items()}
        lens = i["cache_lens"][:n].cpu()
        w_uk, w_uv, sc = i["w_uk"].cpu(), i["w_uv"].cpu(), i["kv_scale"].cpu()
        w = self.w
        fn = lambda: oracle.latent_absorbed_fp8kv(sub["q_c"], sub["q_r"], w_uk, w_uv, sub["latent8"], sc,  # noqa: E731
                                                  lens, w["causal"], i["scale"])
        nbytes = costs.latent_bytes(lens.tolist(), w["h_q"], w["g"], w["d_h"], w["r_kv"], w["d_r"], w["s_q"],
                                    cache_elem=1)
        return fn, nbytes, oracle.threads_used(0, n * w["h_q"]), f"first {n} of {w['B']} sequences"


class LatentAbsorbedPaged(LatentAbsorbed):
    """latent_absorbed_attn_paged over the s_q = 1 batch with the latent cache in 64-token pages of a shuffled pool."""

    def setup_device(self):
        super().setup_device()
        self.inp.pop("latent", None)  # the contiguous copy is not used by the paged step
        torch.cuda.empty_cache()

    def step(self):
        i = self.inp
        self.lka.latent_absorbed_attn_paged(i["q_c"], i["q_r"], i["w_uk"], i["w_uv"], i["latent_pages"],
                                            i["block_table"], i["cache_lens"], causal=self.w["causal"],
                                            scale=i["scale"], out=self.out)

    def config(self):
        c = super().config()
        c["page_size"] = self.w["page_size"]
        c["cache_layout"] = "paged (shuffled page pool + block table)"
        return c


class LatentSparse(LatentAbsorbed):
    """latent_absorbed_attn_sparse: every query attends to 2048 selected tokens of its 16K-token latent cache
    (gather of the selected rows into the workspace, then the dense latent kernels over them)."""

    def setup_costs(self):
        w = self.w
        sel = [w["topk"]] * w["B"]  # every list holds topk visible positions
        self.bytes = costs.latent_bytes(sel, w["h_q"], w["g"], w["d_h"], w["r_kv"], w["d_r"], w["s_q"])
        self.core_flops = costs.latent_core_flops(sel, w["h_q"], w["r_kv"], w["d_r"], w["s_q"], False)
        self.flops = self.core_flops + costs.latent_proj_flops(w["B"], w["h_q"], w["d_h"], w["r_kv"], w["s_q"])
        self.tokens = w["B"] * w["s_q"]
        self.sel_lens = sel

    def kernel_work(self, pk):
        cache = sum(self.sel_lens) * (self.w["r_kv"] + self.w["d_r"]) * 2
        t_mem = cache / (pk["hbm_gbs"] * 1e9)
        t_tc = self.core_flops / (pk["bf16_tflops"] * 1e12)
        return ("tensor", self.core_flops) if t_tc > t_mem else ("hbm", cache)

    def setup_device(self):
        w, i = self.w, self.inp
        self.out = torch.empty_like(i["q_c"])
        self.launches = 8  # select, gather, lens, absorb GEMM, attention, merge, up-projection, finish (+ status fold)
        self.h2d_pairs = [(i["q_c"], _pinned(i["q_c"])), (i["q_r"], _pinned(i["q_r"])),
                          (i["indices"], _pinned(i["indices"])), (i["cache_lens"], _pinned(i["cache_lens"]))]
        self.out_host = torch.empty_like(self.out, device="cpu").pin_memory()

    def step(self):
        i = self.inp
        self.lka.latent_absorbed_attn_sparse(i["q_c"], i["q_r"], i["w_uk"], i["w_uv"], i["latent"], i["indices"],
                                             i["cache_lens"], scale=i["scale"], out=self.out)

    def config(self):
        c = super().config()
        c.update(path="MQA-absorbed, top-k sparse (indices given)", topk=self.w["topk"],
                 l2="selected rows 151 MB > L2; L2 flushed between timed steps")
        return c


class LatentExpanded(LatentAbsorbed):
    """latent_expand_gqa_attn over the per-group expanded cache (made once, outside the timed steps)."""

    kernel = "expanded_attn_kernel"
    src = ("latent_kv_attention_b200/csrc/expanded_attn.cu", "latent_kv_attention_b200/csrc/tc.cuh",
           "latent_kv_attention_b200/csrc/common.cuh")

    def setup_costs(self):
        w = self.w
        self.bytes = costs.expanded_bytes(self.lens, w["h_q"], w["g"], w["d_h"], w["d_r"], w["s_q"])
        self.core_flops = costs.expanded_flops(self.lens, w["h_q"], w["d_h"], w["d_r"], w["s_q"], w["causal"])
        self.flops = self.core_flops
        self.tokens = w["B"] * w["s_q"]

    def kernel_work(self, pk):
        cache = sum(self.lens) * (2 * self.w["g"] * self.w["d_h"] + self.w["d_r"]) * 2
        return "hbm", cache

    def setup_device(self):
        w, i = self.w, self.inp
        self.kc, self.vc, self.kr = self.lka.latent_expand_cache(i["latent"], i["w_uk"], i["w_uv"])
        del i["latent"]
        self.out = torch.empty_like(i["q_c"])
        ws = self.lka.library().latent_expand_gqa_attn_workspace_size(w["B"], w["h_q"], w["g"], w["s_q"], w["d_h"],
                                                                      w["d_r"], w["L_hi"])
        self.launches = 2 if ws > 256 else 1
        self.h2d_pairs = [(i["q_c"], _pinned(i["q_c"])), (i["q_r"], _pinned(i["q_r"])),
                          (i["cache_lens"], _pinned(i["cache_lens"]))]
        self.out_host = torch.empty_like(self.out, device="cpu").pin_memory()

    def step(self):
        i = self.inp
        self.lka.latent_expand_gqa_attn(i["q_c"], i["q_r"], self.kc, self.vc, self.kr, i["cache_lens"],
                                        causal=self.w["causal"], scale=i["scale"], out=self.out)

    def config(self):
        c = super().config()
        c["path"] = "per-group GQA over the expanded cache"
        return c


class GtaPrefill(Workload):
    """gta_shared_score_attn causal prefill: one score matrix per group of 4 heads."""

    kernel = "gta_attn_kernel"
    src = ("latent_kv_attention_b200/csrc/gta_attn.cu", "latent_kv_attention_b200/csrc/tc.cuh",
           "latent_kv_attention_b200/csrc/common.cuh")
    bound = "tensor"
    oracle_n = 1

    def setup_costs(self):
        w = self.w
        self.bytes = costs.gta_bytes(self.lens, w["G"], w["H"], w["d_qk"], w["d_v"], w["s_q"])
        self.flops = costs.gta_flops(self.lens, w["G"], w["H"], w["d_qk"], w["d_v"], w["s_q"], w["causal"])
        self.core_flops = self.flops
        self.tokens = w["B"] * w["s_q"]

    def kernel_work(self, pk):
        return "tensor", self.flops

    def setup_device(self):
        i = self.inp
        w = self.w
        self.out = torch.empty((w["B"], w["H"], w["s_q"], w["d_v"]), dtype=torch.bfloat16, device=self.device)
        ws = self.lka.library().gta_shared_score_attn_workspace_size(w["B"], w["G"], w["H"], w["s_q"], w["d_qk"],
                                                                     w["d_v"], w["L_hi"])
        self.launches = 2 if ws > 256 else 1  # attention (+ merge of key splits)
        self.h2d_pairs = [(i[k], _pinned(i[k])) for k in ("q_g", "k_g", "v", "cache_lens")]
        self.out_host = torch.empty_like(self.out, device="cpu").pin_memory()

    def step(self):
        i = self.inp
        self.lka.gta_shared_score_attn(i["q_g"], i["k_g"], i["v"], i["cache_lens"], causal=self.w["causal"],
                                       scale=i["scale"], out=self.out)

    def config(self):
        w = self.w
        return {"workload": self.name, "B": w["B"], "G": w["G"], "H": w["H"], "d_qk": w["d_qk"], "d_v": w["d_v"],
                "s_q": w["s_q"], "cache_lens": w["L_hi"], "causal": w["causal"],
                "l2": "inputs 126 MB; L2 flushed between timed steps", "parallelism": "replicas"}

    def oracle_run(self, n):
        import oracle

        i = self.inp
        sub = {k: (v[:n].cpu().double() if k in ("q_g", "k_g", "v") else v) for k, v in i.items()}
        lens = i["cache_lens"][:n].cpu()
        w = self.w
        fn = lambda: oracle.gta(sub["q_g"], sub["k_g"], sub["v"], lens, w["causal"], i["scale"])  # noqa: E731
        nbytes = costs.gta_bytes(lens.tolist(), w["G"], w["H"], w["d_qk"], w["d_v"], w["s_q"])
        self.oracle_flops = costs.gta_flops(lens.tolist(), w["G"], w["H"], w["d_qk"], w["d_v"], w["s_q"], w["causal"])
        return fn, nbytes, oracle.threads_used(0, n * w["H"]), f"first {n} of {w['B']} sequences"


class GtaChunkedPrefillPaged(GtaPrefill):
    """gta_shared_score_attn_paged: a 1024-token prefill chunk per sequence against 4096 cached tokens held in
    64-token pages of a shuffled pool (bottom-right causal)."""

    def setup_device(self):
        super().setup_device()
        for k in ("k_g", "v"):  # the contiguous copies are not used by the paged step
            self.inp.pop(k, None)
        torch.cuda.empty_cache()
        i = self.inp
        self.h2d_pairs = [(i[k], _pinned(i[k])) for k in ("q_g", "k_pages", "v_pages", "block_table", "cache_lens")]

    def step(self):
        i = self.inp
        self.lka.gta_shared_score_attn_paged(i["q_g"], i["k_pages"], i["v_pages"], i["block_table"], i["cache_lens"],
                                             causal=self.w["causal"], scale=i["scale"], out=self.out)

    def config(self):
        c = super().config()
        c["page_size"] = self.w["page_size"]
        c["cache_layout"] = "paged (shuffled page pool + block table)"
        c["l2"] = "inputs ~105 MB; L2 flushed between timed steps"
        return c

    def oracle_run(self, n):
        import oracle

        i = self.inp
        w = self.w
        sub = {k: i[k][:n].cpu() for k in ("q_g", "block_table", "cache_lens")}
        kp, vp = i["k_pages"].cpu(), i["v_pages"].cpu()
        fn = lambda: oracle.gta_paged(sub["q_g"], kp, vp, sub["block_table"], sub["cache_lens"], w["causal"],  # noqa: E731
                                      i["scale"])
        lens = sub["cache_lens"].tolist()
        nbytes = costs.gta_bytes(lens, w["G"], w["H"], w["d_qk"], w["d_v"], w["s_q"])
        self.oracle_flops = costs.gta_flops(lens, w["G"], w["H"], w["d_qk"], w["d_v"], w["s_q"], w["causal"])
        return fn, nbytes, oracle.threads_used(0, n * w["H"]), f"first {n} of {w['B']} sequences"


GqaDecode.kernel_work = lambda self, pk: ("hbm", self.bytes)

WORKLOAD_CLASSES = {
    "gqa_decode_llama8b": GqaDecode,
    "gqa_decode_llama8b_b16": GqaDecode,
    "gqa_decode_llama8b_paged": GqaDecodePaged,
    "gqa_decode_llama8b_fp8": GqaDecodeFp8,
    "latent_decode_4k_sq1": LatentAbsorbed,
    "latent_decode_4k_sq2": LatentAbsorbed,
    "latent_decode_4k_sq1_paged": LatentAbsorbedPaged,
    "latent_decode_4k_sq1_fp8": LatentAbsorbedFp8,
    "latent_sparse_16k_top2048": LatentSparse,
    "latent_expanded_4k_sq1": LatentExpanded,
    "latent_expanded_4k_sq2": LatentExpanded,
    "gta_prefill_4k": GtaPrefill,
    "gta_chunked_prefill_4k_paged": GtaChunkedPrefillPaged,
    "gqa_prefill_llama8b_4k": GqaPrefill,
    "gqa_prefill_llama8b_2k_b1": GqaPrefill,
    # smaller cases for full ncu captures
    "latent_decode_4k_sq1_b32": LatentAbsorbed,
    "latent_expanded_4k_sq2_b16": LatentExpanded,
    "gta_prefill_4k_b2": GtaPrefill,
}
# the long-context sweep (batch 64, s_q 1, cache length 1K ... 64K) over the GQA and the latent layout
WORKLOAD_CLASSES.update({name: (GqaDecode if name.startswith("gqa") else LatentAbsorbed) for name in synthetic.SWEEP})
EXTRAS = ["gqa_decode_llama8b_paged", "gqa_decode_llama8b_fp8", "latent_decode_4k_sq1", "latent_decode_4k_sq1_paged",
          "latent_decode_4k_sq1_fp8", "latent_decode_4k_sq2",
          "latent_sparse_16k_top2048", "latent_expanded_4k_sq2", "gta_prefill_4k",
          "gta_chunked_prefill_4k_paged", "gqa_prefill_llama8b_4k"]


def oracle_sample(wl, target_s: float):
    """Times the oracle, as it stands, on the first few sequences, repeated to about target_s seconds."""
    fn, nbytes, cores, what = wl.oracle_run(wl.oracle_n)
    t0 = time.perf_counter()
    fn()
    t1 = time.perf_counter() - t0
    reps = max(1, int(math.ceil(target_s / max(t1, 1e-3))) - 1) if target_s > 0 else 1
    t0 = time.perf_counter()
    for _ in range(reps):
        fn()
    dt = time.perf_counter() - t0
    return dict(value=nbytes * reps / dt / 1e9, unit="GB/s", cores=cores, kind="oracle",
                sample=f"{what}, {reps} repetition(s), {dt:.1f} s", seconds=dt)


# ----------------------------------------------------------------------------- arms
def measure(wl, steps, warmup, pk, device, world, soak_s=1.0, clocks=None):
    """Device time of `steps` steps (CUDA events per step, L2 flushed between steps), the main kernel's
    average launch time from the library's event hook, and the end-to-end time through host buffers."""
    lka = wl.lka
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    for _ in range(max(3, warmup)):
        wl.step()
    torch.cuda.synchronize()
    lka.clear_status()
    if clocks is not None:
        clocks.start()
        clocks.wait_first_sample()
    # keep the GPU under this load for ~soak_s before the timed steps, so the clock samples (every 200 ms)
    # describe the state the timed steps run in
    t_soak = time.time()
    while time.time() - t_soak < soak_s:
        for _ in range(10):
            wl.step()
        torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    lka.kernel_timing(True)
    for s in range(steps):
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
    clk = clocks.stop() if clocks is not None else None
    step_ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / steps
    status = lka.device_status()
    if status != 0:
        raise RuntimeError(f"{wl.name}: device status after the timed steps: {lka.status_string(status)}")
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(2):
        wl.step_e2e()
    torch.cuda.synchronize()
    e2e_total = 0.0
    for s in range(steps):
        flush.zero_()
        e_start.record()
        wl.step_e2e()
        e_end.record()
        e_end.synchronize()
        e2e_total += e_start.elapsed_time(e_end)
    step_ms, e2e_ms, kern_ms = max_over_ranks([step_ms, e2e_total / steps, kern_ms / max(1, n_timed)], world, device)
    bound, work = wl.kernel_work(pk)
    if bound == "hbm":
        peak, unit, achieved = pk["hbm_gbs"], "GB/s", work / (kern_ms * 1e-3) / 1e9
        peak_src = "hbm_gbs"
    else:
        peak, unit, achieved = pk["bf16_tflops"], "TFLOP/s", work / (kern_ms * 1e-3) / 1e12
        peak_src = "bf16_tflops (burst)"
    traffic = recorded_traffic(wl.kernel, wl.name, wl.src)
    datasheet = DATASHEET_HBM_GBS if unit == "GB/s" else DATASHEET_BF16_TFLOPS
    roof = {"bound": bound, "kernel": wl.kernel, "achieved": round(achieved, 1), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4), "traffic": traffic, "algorithmic_work_per_launch": work,
            "launch_ms": round(kern_ms, 4),
            "peak_source": f"{pk['source']} (MEASURED_PEAKS.json {peak_src})" if pk["source"] == "measured"
            else "fallback",
            "datasheet_peak": datasheet, "datasheet_frac": round(achieved / datasheet, 4)}
    return dict(step_ms=step_ms, e2e_ms=e2e_ms, roofline=roof, clocks=clk)


def max_over_ranks(values, world, device):
    """Element-wise maximum of per-rank timings over all ranks (the slowest rank sets the job's time)."""
    if world <= 1:
        return list(values)
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def summary(wl, m, world):
    t = m["step_ms"] * 1e-3
    return {"ms_per_step": round(m["step_ms"], 4), "gbs": round(wl.bytes * world / t / 1e9, 1),
            "tflops": round(wl.flops * world / t / 1e12, 2), "tokens_per_s": round(wl.tokens * world / t, 1),
            "roofline": m["roofline"],
            "e2e_ms_per_step": round(m["e2e_ms"], 4), "config": wl.config()}


def run_lka(args, rank, world, device):
    pk = peaks()
    sharded = args.shard == "heads"
    if sharded:
        if WORKLOAD_CLASSES[args.workload] is not GqaDecode:
            raise SystemExit("--shard heads applies to the contiguous GQA decode workloads")
        wl = GqaDecodeSharded(args.workload, device, rank, world)
    else:
        wl = WORKLOAD_CLASSES[args.workload](args.workload, device)
    clocks = ClockSampler(device.index if device.index is not None else 0)
    m = measure(wl, args.steps, args.warmup, pk, device, world, clocks=clocks)
    extras = {}
    if not args.no_extras and not sharded:
        for name in EXTRAS:
            if name == args.workload:
                continue
            x = WORKLOAD_CLASSES[name](name, device)
            extras[name] = summary(x, measure(x, min(args.steps, 20), args.warmup, pk, device, world, soak_s=0.3),
                                   world)
            del x
            torch.cuda.empty_cache()
    if rank != 0:
        return None
    t = m["step_ms"] * 1e-3
    gbs = wl.bytes * world / t / 1e9
    line = {
        "metric": METRIC, "value": round(gbs, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(m["step_ms"], 4), "higher_is_better": True,
        "scaling": "strong" if sharded else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) inputs, see synthetic.py)",
        "config": wl.config(),
        "tokens_per_s": round(wl.tokens * world / t, 1),
        "tflops": round(wl.flops * world / t / 1e12, 3),
        "hbm_frac_of_peak": round(gbs / world / pk["hbm_gbs"], 4),
        "roofline": m["roofline"],
        "e2e": {"value": round(wl.bytes * world / (m["e2e_ms"] * 1e-3) / 1e9, 1), "unit": "GB/s",
                "h2d_bytes_per_step": wl.h2d, "d2h_bytes_per_step": wl.d2h, "ms_per_step": round(m["e2e_ms"], 4)},
        "gpu_launches": wl.launches * args.steps,
        "clocks": m["clocks"],
    }
    if extras:
        line["other_paths"] = extras
    if world == 1 and not args.no_cpu_baseline:
        cb = oracle_sample(wl, args.cpu_seconds)
        line["cpu_baseline"] = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}
        line["cpu_baseline"]["value"] = round(cb["value"], 4)
    # The MQA-absorbed latent decode (s_q 1 and 2) summarised last, so that a reader keeping only the end of
    # the line still sees both roofline fractions.
    lat = {}
    for name, key in (("latent_decode_4k_sq1", "s_q1"), ("latent_decode_4k_sq2", "s_q2")):
        x = extras.get(name)
        if x is None and name == args.workload:
            x = {"ms_per_step": round(m["step_ms"], 4), "roofline": m["roofline"]}
        if x is not None:
            r = x["roofline"]
            lat[key] = {"frac": r["frac"], "bound": r["bound"], "achieved": r["achieved"], "unit": r["unit"],
                        "launch_ms": r["launch_ms"], "step_ms": x["ms_per_step"]}
    if lat:
        line["latent_absorbed"] = lat
    return line


def run_sweep(args, rank, world, device):
    """The long-context decode sweep: every point of synthetic.SWEEP measured like the main workload (device
    time per step with L2 flushed between steps, the main kernel's roofline, end to end through host buffers);
    one JSON line with one entry per point, clocks sampled over the whole sweep."""
    pk = peaks()
    clocks = ClockSampler(device.index if device.index is not None else 0)
    clocks.start()
    clocks.wait_first_sample()
    points = {}
    for name in synthetic.SWEEP:
        wl = WORKLOAD_CLASSES[name](name, device)
        m = measure(wl, min(args.steps, 10), args.warmup, pk, device, world, soak_s=0.2)
        points[name] = summary(wl, m, world)
        points[name]["gpu_launches"] = wl.launches * min(args.steps, 10)
        del wl
        torch.cuda.empty_cache()
    clk = clocks.stop()
    if rank != 0:
        return None
    return {"metric": METRIC, "mode": "long-context sweep (batch 64, s_q 1, cache length 1K-64K)",
            "unit": "GB/s", "n_gpus": world, "steps": min(args.steps, 10), "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) inputs, see synthetic.py)", "clocks": clk, "points": points}


def run_reference(args, rank, world, device):
    """The oracle as it stands, on the host cores, same workload/metric/unit; rank 0 only."""
    if rank != 0:
        return None
    wl = WORKLOAD_CLASSES[args.workload](args.workload, device, reference=True)
    per_step = max(0.5, min(5.0, 60.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(wl, 0.0)
    vals, secs, last = [], 0.0, None
    for _ in range(args.steps):
        last = oracle_sample(wl, per_step)
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
    ap.add_argument("--no-extras", action="store_true", help="measure only --workload, not the other paths")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="N > 1: independent replicas (default, weak scaling) or the layer's KV heads split over the "
                         "ranks (strong scaling)")
    ap.add_argument("--sweep", action="store_true",
                    help="measure the long-context sweep (GQA and latent layouts, cache length 1K-64K) instead")
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
        if args.impl == "reference":
            line = run_reference(args, rank, world, device)
        else:
            line = (run_sweep if args.sweep else run_lka)(args, rank, world, device)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
