#!/usr/bin/env python3
"""Benchmark: the projection GEMMs of one LLaDA-8B-shaped denoising step on B200.

A step is one pass of the whole hot path over one synthetic canvas: for each of the
32 layers, RMSNorm and quantize the attention input once (one fused kernel) and run
Q, K and V in one launch, quantize and run O, RMSNorm and quantize the FFN input once
and run gate and up in one launch, apply SwiGLU to the gate/up outputs and quantize
(one fused kernel) and run down (Q6_K); then RMSNorm and quantize the final hidden
state and run the 126464-wide output projection (Q6_K) on the 32 rows of the current
block only.  Weights are random
(the GGUF Q4_K / Q6_K distributions of the synthetic workloads), drawn on the device,
repacked once and kept resident (4.77 GB, far above the 126 MB L2, so every step
streams them from HBM).

One JSON line on rank 0.  `value` is algorithmic int8 TOPS (2*M*N*K summed over the
step's GEMMs) over the device-timed step; `ms_per_step` is the step time.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--model llada-8b|dream-7b] [--canvas L] [--layers n]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "int8 TOPS & weight GB/s of dllm_qgemm (% roofline); ms/LLaDA-8B-shaped step"
UNIT = "int8 TOPS"
PEAKS_FILE = ROOT / "MEASURED_PEAKS.json"
TRAFFIC_FILE = ROOT / "profiles" / "qgemm_dram_traffic.json"
FALLBACK_HBM_GBS = 6650.0
P_INT8_NOMINAL = 4.5e15  # dense int8 tensor ops/s of a B200 (datasheet)
FALLBACK_BF16_TFLOPS = 1590.0  # dense bf16 (= f16) tensor TFLOP/s measured earlier on this machine (burst)
# special-function unit: 16 ex2 per clock per SM x 148 SMs x 1.965 GHz (max SM clock)
SFU_EX2_PER_S = 16 * 148 * 1.965e9
Q4, Q6, Q8 = 12, 14, 8


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=500)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--model", default="llada-8b")
    p.add_argument("--canvas", type=int, default=128)
    p.add_argument("--layers", type=int, default=None, help="override the layer count (small profiling cases)")
    p.add_argument("--cpu-layers", type=int, default=6,
                   help="layers the oracle recomputes in full (the first n-1 and the last); the others are "
                        "sampled on 1/64 of their output columns")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--config", choices=["c1", "c2", "c3", "act", "attn", "q80"], default=None,
                   help="time one of the single-GEMM workloads instead of the step: c1 attention projections "
                        "(QKV in one launch + O, 160 rows), c2 FFN (gate/up + down) over canvases 160..1024, "
                        "c3 output projection on 1..32 requested rows, act the fused quantizers at the step's "
                        "canvas and at 2^24 elements, attn the bidirectional attention over canvases 128..4096, "
                        "q80 Q8_0 projections of the model's shapes; one JSON line per case")
    p.add_argument("--parallel", choices=["replicas", "nsplit"], default="replicas",
                   help="with several ranks: replicas (each GPU runs the whole step, weak scaling) or nsplit "
                        "(each GPU owns 1/N of every projection's weight rows, outputs all-gathered over NCCL, "
                        "strong scaling)")
    p.add_argument("--record-traffic", metavar="CSV", default=None,
                   help="write the stored GEMM DRAM traffic (profiles/qgemm_dram_traffic.json) from the ncu CSV "
                        "of a 1-layer step (its first five qgemm launches: QKV, O, gate/up, down, output) and exit")
    p.add_argument("--gather-last", action="store_true",
                   help="the last layer's O and FFN, and the final norm, on the requested rows only")
    return p.parse_args()


# ---------------------------------------------------------------------------- workload

class Gemm:
    def __init__(self, name, qtype, N, K, M_out, M_act, nseg=1):
        self.name, self.qtype, self.N, self.K, self.M_out, self.M_act = name, qtype, N, K, M_out, M_act

    @property
    def ops(self):
        return 2 * self.M_out * self.N * self.K

    @property
    def weight_bytes(self):
        return self.N * (self.K // 256) * {Q4: 144, Q6: 210, Q8: 272}[self.qtype]

    @property
    def bytes(self):
        per = 1 + 4 / 256 + (16 / 256 if self.qtype == Q4 else 0)  # codes, scales (and Q4_K's sums)
        return self.weight_bytes + self.M_act * self.K * per + self.M_out * self.N * 4


def step_gemms(model, L, n_layers, gather_last=False):
    """The GEMM launches of one step, in order (QKV and gate/up are single launches).
    gather_last: past attention, the last layer runs on the requested rows only."""
    h, f, R = model.hidden, model.ffn, min(L, model.out_rows)

    def layer(m):
        return [Gemm("qkv", Q4, model.q_out + 2 * model.kv_out, h, L, L),
                Gemm("o", Q4, h, h, m, m),
                Gemm("gate_up", Q4, 2 * f, h, m, m),
                Gemm("down", Q6, h, f, m, m)]
    last = layer(R if gather_last else L)
    return layer(L) * (n_layers - 1) + last + [Gemm("output", Q6, model.vocab, h, R, R)]


# bytes written per activation element by every quantizer: the int8 code, plus the f32
# scale per 256 and the two-float scaled sum per 32 (4/256 + 64/256)
ACT_OUT_BYTES = 1 + 4 / 256 + 64 / 256


def act_kernel_plan(model, L, n_layers, gather_last=False):
    """The quantizer launch in front of each GEMM of the step, in launch order:
    (kernel, rows, K).  Same order as step_gemms."""
    h, f, R = model.hidden, model.ffn, min(L, model.out_rows)
    plan = []
    for l in range(n_layers):
        m = R if gather_last and l == n_layers - 1 else L
        plan += [("rmsnorm_quantize", L, h), ("quantize_act", m, h), ("rmsnorm_quantize", m, h),
                 ("swiglu_quantize", m, f)]
    plan.append(("rmsnorm_quantize", R if gather_last else L, h))
    return plan


def act_bytes(kernel, M, K):
    """Algorithmic bytes of one quantizer launch: f32 inputs read (x; gate and up), the
    gains of RMSNorm, and the quantized activation written."""
    read = {"rmsnorm_quantize": 4, "quantize_act": 4, "swiglu_quantize": 8}[kernel]
    return M * K * (read + ACT_OUT_BYTES) + (K * 4 if kernel == "rmsnorm_quantize" else 0)


def act_rooflines(durations_ms, plan, hbm_gbs):
    """Per quantizer kernel: launches timed, mean duration, achieved GB/s of algorithmic
    bytes and its fraction of hbm_gbs.  durations_ms[a] is launch a's time (None if not
    timed)."""
    agg = {}
    for (kernel, M, K), d in zip(plan, durations_ms):
        if d is None or d <= 0:
            continue
        a = agg.setdefault(kernel, [0, 0.0, 0.0])
        a[0] += 1
        a[1] += d
        a[2] += act_bytes(kernel, M, K)
    out = {}
    for kernel, (n, ms, nbytes) in sorted(agg.items()):
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[kernel] = {"launches_timed": n, "mean_us": round(ms * 1e3 / n, 3), "achieved_gbs": round(gbs, 1),
                       "frac": round(gbs / hbm_gbs, 4)}
    return out


def split_durations(evs, n_marks):
    """Per-launch times from S steps of events: evs[i][j] is recorded after the j-th
    launch of step i, a quantizer at even j and its GEMM at odd j.  Returns the GEMM ms
    per step, the quantizer ms per step, and each quantizer's mean ms (None for the
    step's first quantizer, which has no mark before it)."""
    S = len(evs)
    gemm_ms = quant_ms = 0.0
    act = [0.0] * (n_marks // 2)
    for e in evs:
        for j in range(0, n_marks, 2):
            if j > 0:
                d = e[j - 1].elapsed_time(e[j])
                quant_ms += d
                act[j // 2] += d
            gemm_ms += e[j].elapsed_time(e[j + 1])
    return gemm_ms / S, quant_ms / S, [None] + [x / S for x in act[1:]]


def roofline_time(gemms, hbm_gbs, p_int8):
    return sum(max(g.bytes / (hbm_gbs * 1e9), g.ops / p_int8) for g in gemms)


def load_tensor_peak():
    """Dense bf16 tensor TFLOP/s (the f16 rate is the same): burst figure."""
    if PEAKS_FILE.exists():
        d = json.loads(PEAKS_FILE.read_text())
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


def load_peaks():
    if PEAKS_FILE.exists():
        d = json.loads(PEAKS_FILE.read_text())
        return float(d.get("hbm_gbs", FALLBACK_HBM_GBS)), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# The sources the GEMM kernel and its launch plan are built from (the attention and the
# fused quantizers live in files of their own and do not move the GEMM's DRAM traffic).
GEMM_SOURCES = ("dllm.cu", "layout.cuh", "ptx.cuh", "qgemm.cuh")


def kernel_source_hash(texts=None):
    """Hash of the GEMM's CUDA sources with `//` comments and blank lines removed, so
    that a comment edit does not mark stored ncu counters as stale."""
    import re
    if texts is None:
        texts = [(ROOT / "quantized_int8_gemm_q4_b200" / "csrc" / f).read_text() for f in GEMM_SOURCES]
    h = hashlib.sha256()
    for t in texts:
        code = [re.sub(r"\s*//.*$", "", line).rstrip() for line in t.splitlines()]
        h.update("\n".join(line for line in code if line).encode())
    return h.hexdigest()[:16]


TRAFFIC_SHAPES = ("qkv", "o", "gate_up", "down", "output")
TRAFFIC_COMMAND = ("ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum "
                   "--clock-control none -k regex:qgemm -s 0 -c 5 --csv --log-file {csv} "
                   "python bench.py --layers 1 --steps 1 --warmup 3 --no-cpu --no-e2e")


def record_traffic(args):
    """Per-launch DRAM bytes of the GEMM from one ncu capture of the 1-layer step, whose
    five GEMM launches have the full step's per-launch shapes, weighted by the full
    step's launch mix and keyed to the current kernel source."""
    import csv
    per = {}
    with open(args.record_traffic, newline="") as f:
        for row in csv.DictReader(line for line in f if not line.startswith("==")):
            if "qgemm" not in row.get("Kernel Name", ""):
                continue
            unit = row["Metric Unit"]
            val = float(row["Metric Value"].replace(",", ""))
            scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "ns": 1e-3, "us": 1.0, "usecond": 1.0,
                     "nsecond": 1e-3, "msecond": 1e3}[unit]
            per.setdefault(int(row["ID"]), {})[row["Metric Name"]] = val * scale
    ids = sorted(per)[:len(TRAFFIC_SHAPES)]
    if len(ids) != len(TRAFFIC_SHAPES):
        sys.exit(f"expected {len(TRAFFIC_SHAPES)} qgemm launches in {args.record_traffic}, found {len(ids)}")
    shapes = {name: {"dram_read": int(per[i]["dram__bytes_read.sum"]), "dram_write": int(per[i]["dram__bytes_write.sum"]),
                     "us_cold": round(per[i]["gpu__time_duration.sum"], 2)} for name, i in zip(TRAFFIC_SHAPES, ids)}
    from quantized_int8_gemm_q4_b200 import synth
    model = synth.MODELS[args.model]()
    n_layers = model.n_layers
    step = step_gemms(model, args.canvas, n_layers)
    counts = {"qkv": n_layers, "o": n_layers, "gate_up": n_layers, "down": n_layers, "output": 1}
    total = sum(counts[k] * (v["dram_read"] + v["dram_write"]) for k, v in shapes.items())
    key = f"{args.model}_L{args.canvas}"
    out = {
        "what": "DRAM bytes (read + write) per qgemm_kernel launch, mean over the step's launch mix "
                f"({n_layers} x QKV, O, gate/up, down + the output projection), from one ncu capture of the "
                "1-layer step whose five GEMM launches have the full step's per-launch shapes",
        "command": TRAFFIC_COMMAND.format(csv=args.record_traffic),
        "kernel_source_sha": kernel_source_hash(),
        "per_launch_bytes": {key: round(total / len(step))},
        "per_launch_shape": shapes,
        f"algorithmic_bytes_per_launch_{key}": round(sum(g.bytes for g in step) / len(step)),
        "note": "the f32 outputs and the quantized activations stay in L2 within a launch, so DRAM traffic is "
                "the weight stream plus little else: no weight byte is read twice",
    }
    TRAFFIC_FILE.write_text(json.dumps(out, indent=1) + "\n")
    return out


def stored_traffic(workload_key):
    """Per-launch DRAM bytes of the GEMM kernel from a stored ncu capture, if it was
    taken on the current kernel source; otherwise None."""
    if not TRAFFIC_FILE.exists():
        return None
    d = json.loads(TRAFFIC_FILE.read_text())
    if d.get("kernel_source_sha") != kernel_source_hash():
        return None
    return d.get("per_launch_bytes", {}).get(workload_key)


# ---------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        lines = Path(self.path).read_text().splitlines()
        os.unlink(self.path)
        return self.summarize(lines)

    @staticmethod
    def summarize(lines):
        """Median SM clock, max clock and the throttle reasons seen, from nvidia-smi
        csv lines (noheader, nounits) in FIELDS order."""
        rows = []
        for line in lines:
            parts = [s.strip() for s in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def workload_config(model, L, n_layers, n_rows, world, gather_last=False):
    """The `config` object both arms report: the workload, not the implementation."""
    gemms = step_gemms(model, L, n_layers, gather_last)
    tail = (f"; past attention, the last layer and the final norm run on the {n_rows} requested rows only"
            if gather_last else "")
    return {"workload": f"{model.name}-shaped denoising step: {n_layers} layers (RMSNorm+quantize -> QKV, "
                        f"quantize -> O, RMSNorm+quantize -> gate/up Q4_K, SwiGLU+quantize -> down Q6_K) + "
                        f"final RMSNorm+quantize -> output projection (Q6_K, {model.vocab} wide) on {n_rows} "
                        f"requested rows{tail}",
            "canvas_tokens": L, "layers": n_layers,
            "weight_bytes_per_step": int(sum(g.weight_bytes for g in gemms)),
            "l2": "inputs larger than L2: every step streams all weights from HBM",
            "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"}


# ---------------------------------------------------------------------------- ranks

def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest of every rank's value (each rank's device-timed region); every rank
    gets it.  Uses the default process group (NCCL on GPUs, gloo in CPU tests)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Units processed by all ranks together per second, over the slowest rank's time."""
    return units_per_rank * world / (ms * 1e-3)


# ---------------------------------------------------------------------------- our arm

def run_ours(args, rank, world):
    import torch
    from quantized_int8_gemm_q4_b200 import build, dllm, synth

    build.build()
    dllm.load()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    model = synth.MODELS[args.model]()
    n_layers = args.layers or model.n_layers
    L = args.canvas
    h, f = model.hidden, model.ffn
    seed = 4  # the full-step workload's seed

    # ---- weights: draw GGUF blocks on the device, repack once, keep resident.  The
    # oracle's sample (cpu_baseline) keeps host copies of the weight rows it recomputes.
    do_cpu = rank == 0 and not args.no_cpu
    sample = parity_sample(model, n_layers, args.cpu_layers, seed) if do_cpu else {}
    w_host = {}
    layers = []
    for l in range(n_layers):
        mats = {}
        for pi, p in enumerate(model.layer):
            g = synth.device_weights(p.qtype, p.N, p.K, seed, l, pi, device=dev)
            if (l, p.name) in sample:
                n0, n1 = sample[(l, p.name)]
                w_host[(l, p.name)] = g.view(p.N, -1)[n0:n1].cpu().numpy().reshape(n1 - n0, p.K // 256, -1)
            w = torch.empty(dllm.dllm_repacked_bytes(p.qtype, p.N, p.K), dtype=torch.uint8, device=dev)
            (dllm.dllm_repack_q4k if p.qtype == Q4 else dllm.dllm_repack_q6k)(g, p.N, p.K, w)
            del g
            mats[p.name] = w
        layers.append(mats)
    g = synth.device_weights(Q6, model.vocab, h, seed, 999, 0, device=dev)
    if do_cpu:
        w_host["output"] = g.cpu().numpy().reshape(model.vocab, h // 256, -1)
    w_out = torch.empty(dllm.dllm_repacked_bytes(Q6, model.vocab, h), dtype=torch.uint8, device=dev)
    dllm.dllm_repack_q6k(g, model.vocab, h, w_out)
    del g
    torch.cuda.synchronize()

    # ---- the step's f32 inputs, one contiguous buffer: the residual stream entering
    # each layer's attention and FFN norms, the attention output and the final hidden
    # state.  The down projection's input is the SwiGLU of the gate/up outputs.
    sizes = [L * h] * 4
    xin = torch.empty(sum(sizes), dtype=torch.float32, device=dev)
    views, off = [], 0
    for i, sz in enumerate(sizes):
        v = xin[off:off + sz].view(L, -1)
        v.copy_(synth.device_activations(L, sz // L, seed, 100 + (4 if i == 3 else i), device=dev))
        views.append(v)
        off += sz
    x_attn, x_o, x_ffn, x_fin = views
    gam_host = synth.norm_weights(2 * n_layers + 1, h, seed)   # attn, ffn per layer; final
    gam = torch.from_numpy(gam_host).to(dev)
    eps = model.norm_eps
    act_h = dllm.alloc_act(L, h, dev)
    act_f = dllm.alloc_act(L, f, dev)
    o_q = torch.empty((L, model.q_out), device=dev)
    o_k = torch.empty((L, model.kv_out), device=dev)
    o_v = torch.empty((L, model.kv_out), device=dev)
    o_o = torch.empty((L, h), device=dev)
    o_g = torch.empty((L, f), device=dev)
    o_u = torch.empty((L, f), device=dev)
    o_d = torch.empty((L, h), device=dev)
    rows_np = synth.block_rows(L, model.out_rows, seed) if L >= 64 else np.arange(min(L, model.out_rows),
                                                                                     dtype=np.int32)
    rows = torch.from_numpy(rows_np).to(dev)
    logits = torch.empty((len(rows_np), model.vocab), device=dev)
    R = len(rows_np)
    act_hr = dllm.alloc_act(R, h, dev)  # compact activations of the requested rows
    act_fr = dllm.alloc_act(R, f, dev)
    # one zero-filled workspace, large enough for every GEMM of the step (stream-ordered)
    wsb = max(dllm.dllm_qgemm_workspace_bytes(Q4, model.q_out + 2 * model.kv_out, h, L),
              dllm.dllm_qgemm_workspace_bytes(Q4, h, h, L),
              dllm.dllm_qgemm_workspace_bytes(Q4, 2 * f, h, L),
              dllm.dllm_qgemm_workspace_bytes(Q6, h, f, L),
              dllm.dllm_qgemm_workspace_bytes(Q6, model.vocab, h, L, len(rows_np)),
              # the requested-rows shapes of --gather-last
              dllm.dllm_qgemm_workspace_bytes(Q4, h, h, R),
              dllm.dllm_qgemm_workspace_bytes(Q4, 2 * f, h, R),
              dllm.dllm_qgemm_workspace_bytes(Q6, h, f, R),
              dllm.dllm_qgemm_workspace_bytes(Q6, model.vocab, h, R))
    ws = dllm.alloc_workspace(max(wsb, 256), dev)

    def step(ev=None, after_layer=None, gemm_only=False):
        k = 0

        def mark():
            nonlocal k
            if ev is not None:
                ev[k].record()
                k += 1

        for l in range(n_layers):
            W = layers[l]
            gemm_only or dllm.dllm_rmsnorm_quantize(x_attn, L, h, h, gam[2 * l], eps, None, 0, *act_h)
            mark()
            dllm.dllm_qkv_qgemm(W["q"], W["k"], W["v"], Q4, model.q_out, model.kv_out, h, *act_h, L,
                                o_q, model.q_out, o_k, o_v, model.kv_out, ws, wsb)
            mark()
            if args.gather_last and l == n_layers - 1:
                # past attention only the requested positions continue: the attention output
                # of those rows (compact), the FFN input gathered from the canvas by the norm
                gemm_only or dllm.dllm_quantize_act(x_o, R, h, h, *act_hr)
                mark()
                dllm.dllm_qgemm(W["o"], Q4, h, h, *act_hr, R, None, 0, o_o, h, ws, wsb)
                mark()
                gemm_only or dllm.dllm_rmsnorm_quantize(x_ffn, L, h, h, gam[2 * l + 1], eps, rows, R, *act_hr)
                mark()
                dllm.dllm_qkv_qgemm(W["gate"], W["up"], None, Q4, f, f, h, *act_hr, R, o_g, f, o_u, None, f,
                                    ws, wsb)
                mark()
                gemm_only or dllm.dllm_swiglu_quantize(o_g, o_u, R, f, f, *act_fr)
                mark()
                dllm.dllm_qgemm(W["down"], Q6, h, f, *act_fr, R, None, 0, o_d, h, ws, wsb)
                mark()
                continue
            gemm_only or dllm.dllm_quantize_act(x_o, L, h, h, *act_h)
            mark()
            dllm.dllm_qgemm(W["o"], Q4, h, h, *act_h, L, None, 0, o_o, h, ws, wsb)
            mark()
            gemm_only or dllm.dllm_rmsnorm_quantize(x_ffn, L, h, h, gam[2 * l + 1], eps, None, 0, *act_h)
            mark()
            dllm.dllm_qkv_qgemm(W["gate"], W["up"], None, Q4, f, f, h, *act_h, L, o_g, f, o_u, None, f, ws, wsb)
            mark()
            gemm_only or dllm.dllm_swiglu_quantize(o_g, o_u, L, f, f, *act_f)
            mark()
            dllm.dllm_qgemm(W["down"], Q6, h, f, *act_f, L, None, 0, o_d, h, ws, wsb)
            mark()
            if after_layer is not None:
                after_layer(l)
        if args.gather_last:
            # the last layer's output exists for the requested rows only (compact)
            gemm_only or dllm.dllm_rmsnorm_quantize(x_fin, R, h, h, gam[2 * n_layers], eps, None, 0, *act_hr)
            mark()
            dllm.dllm_qgemm(w_out, Q6, model.vocab, h, *act_hr, R, None, 0, logits, model.vocab, ws, wsb)
            mark()
        else:
            gemm_only or dllm.dllm_rmsnorm_quantize(x_fin, L, h, h, gam[2 * n_layers], eps, None, 0, *act_h)
            mark()
            dllm.dllm_qgemm(w_out, Q6, model.vocab, h, *act_h, L, rows, len(rows_np), logits, model.vocab,
                            ws, wsb)
            mark()

    # + the row gather of the output projection, unless the final norm gathers the rows
    launches_per_step = n_layers * 8 + (2 if args.gather_last else 3)
    gemms = step_gemms(model, L, n_layers, args.gather_last)

    # eager warm-up of every kernel (attribute setup happens outside capture)
    step()
    torch.cuda.synchronize()
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK

    # graphs: g1 = one step, gS = S steps (the timed region replays these; no events
    # inside), gE = S steps with an event after every quantize and every GEMM launch
    # (a second pass, right after the timed region, for per-launch durations)
    S = max(1, min(args.steps, 10))
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    g1 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g1, stream=s):
        step()
    gS = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gS, stream=s):
        for i in range(S):
            step()
    n_marks = 2 * len(gemms)
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(n_marks)] for _ in range(S)]
    gE = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gE, stream=s):
        for i in range(S):
            step(evs[i])
    torch.cuda.synchronize()

    # ---- warm-up: W steps (plus one untimed replay of each multi-step graph, which
    # uploads it)
    with torch.cuda.stream(s):
        for _ in range(args.warmup):
            g1.replay()
        gS.replay()
        gE.replay()
    torch.cuda.synchronize()

    sampler = None
    if rank == 0:
        sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
        sampler.start()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        t0.record(s)
        for _ in range(args.steps // S):
            gS.replay()
        for _ in range(args.steps % S):
            g1.replay()
        t1.record(s)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    elapsed_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK

    # ---- per-launch durations: S more steps with events on the launching stream (for
    # the quantizers' own rooflines; events add a fixed cost to every launch)
    with torch.cuda.stream(s):
        gE.replay()
    torch.cuda.synchronize()
    ev_gemm_ms, ev_quant_ms, act_launch_ms = split_durations(evs, n_marks)
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK
    del gE

    # ---- the GEMM time of a step, event-free: the same step with its quantizer launches
    # left out (their outputs stay in place), replayed and timed like the headline
    gG = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gG, stream=s):
        for i in range(S):
            step(gemm_only=True)
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        for _ in range(2):
            gG.replay()
    torch.cuda.synchronize()
    reps = max(1, args.steps // S)
    g0 = torch.cuda.Event(enable_timing=True)
    g1e = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        g0.record(s)
        for _ in range(reps):
            gG.replay()
        g1e.record(s)
    torch.cuda.synchronize()
    gemm_ms = max_over_ranks(g0.elapsed_time(g1e) / (reps * S), world, dev)
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK
    del gG

    # ---- the int8 tensor-core peak of this GPU: back-to-back 128 x 256 x 32 MMAs with A
    # in tensor memory, one CTA per SM
    p_int8_meas = measure_int8_peak(dllm, torch, dev)

    # ---- outputs for the parity check: one eager step, keeping each sampled projection's
    # output columns and the logits
    gpu_out = {}
    if do_cpu and not args.gather_last:
        outs = {"q": o_q, "k": o_k, "v": o_v, "o": o_o, "gate": o_g, "up": o_u, "down": o_d}

        def keep(l):
            for name, buf in outs.items():
                if (l, name) in sample:
                    n0, n1 = sample[(l, name)]
                    gpu_out[(l, name)] = buf[:, n0:n1].cpu().numpy().copy()
        step(after_layer=keep)
        torch.cuda.synchronize()
        gpu_out["output"] = logits.cpu().numpy().copy()
        assert dllm.dllm_get_device_status() == dllm.DLLM_OK

    ms_step = elapsed_ms / args.steps
    ops_step = sum(g.ops for g in gemms)
    wbytes_step = sum(g.weight_bytes for g in gemms)
    abytes_step = sum(g.bytes for g in gemms)
    hbm_gbs, peak_kind = load_peaks()
    p_int8 = P_INT8_NOMINAL
    tstar = roofline_time(gemms, hbm_gbs, p_int8)
    tstar_meas = roofline_time(gemms, hbm_gbs, p_int8_meas) if p_int8_meas else None
    value = whole_job_rate(ops_step, world, ms_step) / 1e12

    # ---- end to end through the public API with host buffers.  Every step copies its
    # input canvas in from pinned host memory and its logits back out; as in a serving
    # loop, those copies run on their own streams and overlap the neighbouring steps'
    # compute (two device staging buffers each way, handed over with events).
    e2e = None
    if not args.no_e2e and rank == 0:
        x_host = torch.empty(xin.numel(), dtype=torch.float32, pin_memory=True)
        x_host.copy_(xin.reshape(-1).cpu())
        out_host = [torch.empty(logits.shape, dtype=torch.float32, pin_memory=True) for _ in range(2)]
        x_stage = [torch.empty_like(xin) for _ in range(2)]
        o_stage = [torch.empty_like(logits) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev = lambda: torch.cuda.Event(enable_timing=False)
        in_ready, in_free = [ev(), ev()], [ev(), ev()]
        out_ready, out_free = [ev(), ev()], [ev(), ev()]
        for b in range(2):
            in_free[b].record(s)
            out_free[b].record(s_out)
        ke = max(2, min(args.steps, 100))
        torch.cuda.synchronize()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(s_in)
        for it in range(ke):
            b = it & 1
            with torch.cuda.stream(s_in):           # input of step it
                s_in.wait_event(in_free[b])
                x_stage[b].copy_(x_host.view_as(xin), non_blocking=True)
                in_ready[b].record(s_in)
            with torch.cuda.stream(s):              # step it
                s.wait_event(in_ready[b])
                xin.copy_(x_stage[b], non_blocking=True)
                in_free[b].record(s)
                g1.replay()
                s.wait_event(out_free[b])
                o_stage[b].copy_(logits, non_blocking=True)
                out_ready[b].record(s)
            with torch.cuda.stream(s_out):          # logits of step it
                s_out.wait_event(out_ready[b])
                out_host[b].copy_(o_stage[b], non_blocking=True)
                out_free[b].record(s_out)
        s_out.wait_stream(s)
        a1.record(s_out)
        torch.cuda.synchronize()
        ms_e2e = a0.elapsed_time(a1) / ke
        assert torch.equal(out_host[(ke - 1) & 1], logits.cpu())
        e2e = {"value": ops_step / (ms_e2e * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": ms_e2e,
               "h2d_bytes_per_step": int(xin.numel() * 4), "d2h_bytes_per_step": int(logits.numel() * 4),
               "copies": "each step's input in and logits out through pinned host buffers, on their own "
                         "streams, overlapping the neighbouring steps' compute"}

    traffic = None if args.gather_last else stored_traffic(f"{args.model}_L{L}")
    roof = None
    if gemm_ms > 0:
        achieved = abytes_step / (gemm_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_gbs, "unit": "GB/s",
                "frac": round(achieved / hbm_gbs, 4), "traffic": traffic,
                "kernel": "qgemm_kernel",
                "peak_source": ("measured hbm_gbs from MEASURED_PEAKS.json" if peak_kind == "measured"
                                else f"fallback {FALLBACK_HBM_GBS:.0f} GB/s (no MEASURED_PEAKS.json)"),
                "launches_per_step": len(gemms), "gemm_ms_per_step": round(gemm_ms, 4),
                "algorithmic_bytes_per_step": int(abytes_step),
                "algorithmic_bytes_per_launch": int(abytes_step / len(gemms)),
                "mean_launch_us": round(gemm_ms * 1e3 / len(gemms), 3),
                "traffic_per": "launch, mean over the step's launch mix (DRAM read + write, ncu)",
                "durations": f"the step's {len(gemms)} GEMM launches alone (quantizer launches left out), "
                             f"CUDA-graph replays of {S} steps timed with CUDA events like the headline"}

    # the quantizers' own rooflines (the step's first quantizer has no mark before it)
    try:
        hbm_for_act, _ = load_peaks()
        act = act_rooflines(act_launch_ms, act_kernel_plan(model, L, n_layers, args.gather_last), hbm_for_act)
        act["durations"] = ("CUDA events from the previous GEMM's end to the quantizer's end, in the same "
                            "second pass; they include each launch's event cost")
    except Exception as ex:  # a report, never a reason to lose the bench line
        act = {"error": repr(ex)}

    cpu, parity = None, None
    if do_cpu:
        x_host = {"attn": x_attn.cpu().numpy(), "o": x_o.cpu().numpy(), "ffn": x_ffn.cpu().numpy(),
                  "fin": x_fin.cpu().numpy()}
        cpu, parity = cpu_baseline(model, L, sample, w_host, gpu_out, rows_np, x_host, gam_host, n_layers)
        if args.gather_last:
            parity = {"checked": False, "reason": "the parity check runs on the full-canvas step only"}

    del gS, g1
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": dict(workload_config(model, L, n_layers, len(rows_np), world, args.gather_last),
                       graph=f"CUDA graphs of {S} steps, replayed; no events inside the timed region"),
        "weight_gbs": round(wbytes_step / (ms_step * 1e-3) / 1e9, 1),
        "step_roofline": {"t_star_ms": round(tstar * 1e3, 4), "frac": round(tstar * 1e3 / ms_step, 4),
                          "p_int8_tops": p_int8 / 1e12, "p_int8_source": "nominal dense B200 figure",
                          "t_star_ms_measured_peak": round(tstar_meas * 1e3, 4) if tstar_meas else None,
                          "frac_measured_peak": round(tstar_meas * 1e3 / ms_step, 4) if tstar_meas else None,
                          "p_int8_tops_measured": round(p_int8_meas / 1e12, 1) if p_int8_meas else None,
                          "p_int8_measured_by": "dllm_bench_mma_i8: 128x256x32 int8 MMAs, A in tensor memory, "
                                                "one CTA per SM, this run",
                          "hbm_gbs": hbm_gbs},
        "gemm_ms_per_step": round(gemm_ms, 4),
        "quantize_ms_per_step": round(max(0.0, ms_step - gemm_ms), 4),
        "quantize_ms_note": "step time minus the GEMM-only time of the same step",
        "roofline": roof, "act_kernels": act, "cpu_baseline": cpu, "parity": parity, "e2e": e2e,
        "clocks": clocks,
        "gpu_launches": launches_per_step * args.steps,
    }
    return result


def run_nsplit(args, rank, world):
    """The step with every projection column-parallel over the ranks (nsplit module):
    each rank repacks its rows of every weight matrix; per layer it quantizes its own
    copy of the inputs, runs its rows of QKV, O, gate/up and down, and all-gathers the
    f32 outputs (the down input: its SwiGLU K-slice, quantized, is gathered instead).
    Eager launches timed with CUDA events; max over ranks."""
    import torch
    from quantized_int8_gemm_q4_b200 import build, dllm, nsplit, synth

    build.build()
    dllm.load()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    model = synth.MODELS[args.model]()
    n_layers = args.layers or model.n_layers
    L, h, f = args.canvas, model.hidden, model.ffn
    seed = 4

    def shard(qt, N, K, *sub):
        n0, n1, _ = nsplit.shard_rows(N, world, rank)
        g = synth.device_weights(qt, N, K, seed, *sub, device=dev).view(N, -1)[n0:n1].contiguous().view(-1)
        return nsplit.ColumnParallelQGemm(g, qt, N, K, world, rank, dev)

    layers = []
    for l in range(n_layers):
        layers.append({p.name: shard(p.qtype, p.N, p.K, l, pi) for pi, p in enumerate(model.layer)})
    out_proj = shard(Q6, model.vocab, h, 999, 0)
    torch.cuda.synchronize()
    x = {n: synth.device_activations(L, h, seed, 100 + i, device=dev) for i, n in enumerate(("attn", "o", "ffn"))}
    x_fin = synth.device_activations(L, h, seed, 104, device=dev)
    gam = torch.from_numpy(synth.norm_weights(2 * n_layers + 1, h, seed)).to(dev)
    rows = torch.from_numpy(synth.block_rows(L, model.out_rows, seed)).to(dev)
    R = rows.numel()
    act_h, act_r = dllm.alloc_act(L, h, dev), dllm.alloc_act(R, h, dev)
    k0, k1 = nsplit.shard_k(f, world, rank)
    act_fl, act_f = dllm.alloc_act(L, k1 - k0, dev), dllm.alloc_act(L, f, dev)
    P = layers[0]
    bufs = {}
    for name, cp, M in [(n, P[n], L) for n in ("q", "k", "v", "o", "gate", "up", "down")] + [("out", out_proj, R)]:
        bufs[name] = (torch.zeros((M, cp.Wp), device=dev), torch.empty((M, cp.N), device=dev),
                      torch.empty((world * M, cp.Wp), device=dev))
    wsb = max(max(cp.workspace_bytes(L) for cp in P.values()), out_proj.workspace_bytes(R), 256)
    ws = dllm.alloc_workspace(wsb, dev)
    gl, ul = bufs["gate"][0], bufs["up"][0]
    fs = k1 - k0  # this rank's gate/up columns are the down input's K-slice

    def proj(cp, name, act, M):
        loc, full, scr = bufs[name]
        cp(act, M, full, loc, scr, ws, wsb)

    def step():
        for l in range(n_layers):
            W = layers[l]
            dllm.dllm_rmsnorm_quantize(x["attn"], L, h, h, gam[2 * l], model.norm_eps, None, 0, *act_h)
            for n in ("q", "k", "v"):
                proj(W[n], n, act_h, L)
            dllm.dllm_quantize_act(x["o"], L, h, h, *act_h)
            proj(W["o"], "o", act_h, L)
            dllm.dllm_rmsnorm_quantize(x["ffn"], L, h, h, gam[2 * l + 1], model.norm_eps, None, 0, *act_h)
            W["gate"].local(act_h, L, gl, ws, wsb)
            W["up"].local(act_h, L, ul, ws, wsb)
            dllm.dllm_swiglu_quantize(gl, ul, L, fs, W["gate"].Wp, *act_fl)
            nsplit.gather_act_k(act_fl, act_f, world)
            proj(W["down"], "down", act_f, L)
        dllm.dllm_rmsnorm_quantize(x_fin, L, h, h, gam[2 * n_layers], model.norm_eps, rows, R, *act_r)
        proj(out_proj, "out", act_r, R)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid)) if rank == 0 else None
    if sampler:
        sampler.start()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    ms_step = max_over_ranks(t0.elapsed_time(t1), world, dev) / args.steps
    assert dllm.dllm_get_device_status() == dllm.DLLM_OK
    gemms = step_gemms(model, L, n_layers)
    ops_step = sum(g.ops for g in gemms)
    cfg = workload_config(model, L, n_layers, R, world)
    cfg["parallelism"] = f"nsplit x{world}: weight rows column-parallel, f32 outputs all-gathered (NCCL)"
    cfg["graph"] = "eager launches (collectives in the step)"
    # our kernels per rank and step: per layer 4 quantizers + 7 GEMMs; the final norm and
    # the output projection (the gathers are NCCL / copy kernels, not counted)
    per_rank_launches = n_layers * 11 + 2
    return {
        "metric": METRIC, "value": round(ops_step / (ms_step * 1e-3) / 1e12, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "int8", "data": "synthetic", "config": cfg,
        "roofline": None, "cpu_baseline": None, "e2e": None,
        "parity": {"checked": False, "reason": "the split's gather logic is checked against the oracle by "
                                              "tests/test_nsplit.py; the GEMMs are the step's own kernels"},
        "clocks": clocks, "gpu_launches": per_rank_launches * args.steps,
    }


def parity_sample(model, n_layers, full_layers, seed):
    """The oracle's sample of the step, as (layer, projection) -> output column range
    [n0, n1): the first full_layers - 1 layers and the last in full, every other layer's
    Q, K, V, O, gate and up on one random contiguous 1/64 of their output columns."""
    rng = np.random.default_rng([seed, 17])
    full = set(range(max(0, min(full_layers - 1, n_layers - 1)))) | {n_layers - 1}
    out = {}
    for l in range(n_layers):
        for p in model.layer:
            if l in full:
                out[(l, p.name)] = (0, p.N)
            elif p.name != "down":
                w = max(8, p.N // 64)
                n0 = int(rng.integers(0, p.N - w + 1))
                out[(l, p.name)] = (n0, n0 + w)
    return out


def parity_ratio(got, ref64, T):
    """max over elements of |gpu - oracle| / max(1e-5 |oracle|, 1e-6 T): at most 1 passes."""
    bound = np.maximum(1e-5 * np.abs(ref64), 1e-6 * T)
    return float(np.max(np.abs(got.astype(np.float64) - ref64) / np.maximum(bound, 1e-300)))


def cpu_baseline(model, L, sample, w_host, gpu_out, rows_np, x_host, gam, n_layers, max_threads=None):
    """The oracle, as it stands, on a bounded sample of the same step (same weights, same
    inputs): the projections in `sample` with their RMSNorm and quantizers, the down
    projection of the fully sampled layers (from the oracle's own gate/up outputs), and the
    output projection on the requested rows.  Returns (cpu_baseline, parity): the timed
    baseline, and the element-wise check of the GPU outputs in gpu_out against it."""
    import oracle
    nt = max_threads or oracle.max_threads()
    h, eps = model.hidden, model.norm_eps
    projs = {p.name: p for p in model.layer}
    ops = 0
    worst, worst_at, compared, n_proj = 0.0, None, 0, 0

    def check(key, got, ref64, T):
        nonlocal worst, worst_at, compared, n_proj
        r = parity_ratio(got, ref64, T)
        compared += got.size
        n_proj += 1
        if r > worst:
            worst, worst_at = r, key

    t0 = time.perf_counter()
    n_full = 0
    for l in range(n_layers):
        acts = {}
        if any((l, n) in sample for n in ("q", "k", "v")):
            acts["attn"] = oracle.rmsnorm_quantize(x_host["attn"], gam[2 * l], eps)[:2]
        if (l, "o") in sample:
            acts["o"] = oracle.quantize_act(x_host["o"])[:2]
        if any((l, n) in sample for n in ("gate", "up")):
            acts["ffn"] = oracle.rmsnorm_quantize(x_host["ffn"], gam[2 * l + 1], eps)[:2]
        f32 = {}
        for name, src in (("q", "attn"), ("k", "attn"), ("v", "attn"), ("o", "o"), ("gate", "ffn"), ("up", "ffn")):
            if (l, name) not in sample:
                continue
            p = projs[name]
            n0, n1 = sample[(l, name)]
            out32, ref64, T = oracle.qgemm(p.qtype, w_host[(l, name)], n1 - n0, p.K, *acts[src], nthreads=nt)
            ops += 2 * L * (n1 - n0) * p.K
            f32[name] = out32
            if (l, name) in gpu_out:
                check((l, name), gpu_out[(l, name)], ref64, T)
        if (l, "down") in sample:
            n_full += 1
            p = projs["down"]
            q, sc, _ = oracle.swiglu_quantize(f32["gate"], f32["up"])
            oracle.qgemm(p.qtype, w_host[(l, "down")], p.N, p.K, q, sc, nthreads=nt)
            ops += 2 * L * p.N * p.K
    q, sc, _ = oracle.rmsnorm_quantize(x_host["fin"], gam[2 * n_layers], eps)
    _, ref64, T = oracle.qgemm(Q6, w_host["output"], model.vocab, h, q, sc, rows=rows_np, nthreads=nt)
    ops += 2 * len(rows_np) * model.vocab * h
    if "output" in gpu_out:
        check("output", gpu_out["output"], ref64, T)
    dt = time.perf_counter() - t0
    cpu = {"value": round(ops / dt / 1e12, 6), "unit": UNIT, "cores": nt, "kind": "oracle", "seconds": round(dt, 2),
           "sample": f"{n_full} of {model.n_layers} layers in full (RMSNorm, quantize, SwiGLU and all seven "
                     f"projections), the Q/K/V/O/gate/up projections of the other layers on a random 1/64 of "
                     f"their output columns, and the output projection on {len(rows_np)} rows; canvas {L}; the "
                     f"step's own weights and inputs"}
    parity = None
    if gpu_out:
        parity = {"checked": True, "projections": n_proj, "elements": int(compared),
                  "max_err_over_bound": round(worst, 4), "worst_at": str(worst_at),
                  "bound": "|gpu - oracle| <= max(1e-5 |oracle|, 1e-6 sum|terms|), element by element",
                  "sample": "the cpu_baseline sample: layer 0 .. and the last layer in full, 1/64 of the columns "
                            "of every other layer, and the logits",
                  "not_compared": "down: its input is the SwiGLU of the step's own f32 gate/up outputs, whose "
                                  "last-place rounding the oracle does not share (the GPU tests check that chain "
                                  "with the bracket rule); the oracle's down is timed, not compared"}
    return cpu, parity


def measure_int8_peak(dllm, torch, dev, iters=8192):
    """Dense int8 tensor ops/s of this GPU: every SM issues back-to-back 128 x 256 x 32
    kind::i8 MMAs with A in tensor memory (dllm_bench_mma_i8); total ops over the slowest
    SM's device time."""
    ctas = torch.cuda.get_device_properties(dev).multi_processor_count
    ns = torch.zeros(ctas, dtype=torch.int64, device=dev)
    dllm.dllm_bench_mma_i8(256, 1, 1, 1, 64, ctas, ns)
    dllm.dllm_bench_mma_i8(256, 1, 1, 1, iters, ctas, ns)
    torch.cuda.synchronize()
    t = float(ns.max().item()) * 1e-9
    if t <= 0:
        return None
    return 2 * 128 * 256 * 32 * iters * ctas / t


# ---------------------------------------------------------------------------- single-GEMM configs

def config_cases(name, model):
    """(label, [Gemm per launch], M canvas, rows) of a single-GEMM workload."""
    h, f = model.hidden, model.ffn
    if name == "c1":
        M = 160
        return [("qkv+o", [Gemm("qkv", Q4, model.q_out + 2 * model.kv_out, h, M, M), Gemm("o", Q4, h, h, M, M)],
                 M, None)]
    if name == "c2":
        return [(f"ffn M={M}", [Gemm("gate_up", Q4, 2 * f, h, M, M), Gemm("down", Q6, h, f, M, M)], M, None)
                for M in (160, 256, 512, 1024)]
    if name == "q80":
        return ([(f"q80 o M={M}", [Gemm("q80_o", Q8, h, h, M, M)], M, None) for M in (32, 128, 160, 512)] +
                [("q80 qkv-wide M=160", [Gemm("q80_qkv", Q8, model.q_out + 2 * model.kv_out, h, 160, 160)], 160, None)])
    return [(f"output rows={R}", [Gemm("output", Q6, model.vocab, h, R, R)], 160, R) for R in (1, 2, 4, 8, 16, 32)]


def run_act_config(args, dllm, torch, dev, model):
    """Device time of the three quantizer kernels at the step's canvas and at 2^24
    elements (inputs beyond L2 at the large size), against their algorithmic bytes."""
    hbm_gbs, peak_kind = load_peaks()
    lines = []
    h, f, eps = model.hidden, model.ffn, model.norm_eps
    for M in (args.canvas, 4096):
        for kernel, K in (("quantize_act", h), ("rmsnorm_quantize", h), ("swiglu_quantize", f)):
            Mk = M if kernel != "swiglu_quantize" else max(1, M * h // f)  # same element count at 2^24
            if M == args.canvas:
                Mk = M
            x = torch.randn((Mk, K), device=dev)
            u = torch.randn((Mk, K), device=dev)
            gam = torch.rand(K, device=dev) + 0.5
            q, sc, su = dllm.alloc_act(Mk, K, dev)

            def run():
                if kernel == "quantize_act":
                    dllm.dllm_quantize_act(x, Mk, K, K, q, sc, su)
                elif kernel == "rmsnorm_quantize":
                    dllm.dllm_rmsnorm_quantize(x, Mk, K, K, gam, eps, None, 0, q, sc, su)
                else:
                    dllm.dllm_swiglu_quantize(x, u, Mk, K, K, q, sc, su)
            for _ in range(3):
                run()
            torch.cuda.synchronize()
            reps = 50
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(reps):
                run()
            e1.record()
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / reps
            nbytes = act_bytes(kernel, Mk, K)
            gbs = nbytes / (us * 1e-6) / 1e9
            lines.append({"metric": "GB/s of algorithmic bytes (% of HBM)", "config": {
                "workload": "act", "kernel": kernel, "rows": Mk, "K": K, "elements": Mk * K},
                "us": round(us, 2), "bytes": int(nbytes), "achieved_gbs": round(gbs, 1),
                "frac": round(gbs / hbm_gbs, 4), "hbm_gbs": hbm_gbs, "hbm_source": peak_kind,
                "timing": f"CUDA events over {reps} back-to-back launches"})
            assert dllm.dllm_get_device_status() == dllm.DLLM_OK
            del x, u, q, sc, su
    return lines


def run_attn_config(args, dllm, torch, dev, model):
    """Device time of dllm_attention per launch at the model's head layout, canvases
    128..1024 (the step sweep) and 4096, inputs rotated over copies beyond L2, against
    t* = max(FLOPs / f16 tensor peak, exponentials / special-function-unit rate), with
    the SM clock sampled while the launches run."""
    from quantized_int8_gemm_q4_b200 import synth
    peak_tf, peak_kind = load_tensor_peak()
    H, Hkv, dh = model.heads, model.kv_heads, model.hidden // model.heads
    sampler = ClockSampler("GPU-" + str(torch.cuda.get_device_properties(dev).uuid))
    lines = []
    for L in (128, 256, 512, 1024, 4096):
        nbytes = 2 * (L * H * dh + 2 * L * Hkv * dh)
        copies = max(1, min(16, int(3 * 126e6 // nbytes) + 1))
        ins = [synth.device_attention_inputs(L, L, H, Hkv, dh, 6, L, c, device=dev) for c in range(copies)]
        o = torch.empty((L, H, dh), dtype=torch.float32, device=dev)

        def run(i):
            q, k, v = ins[i % copies]
            dllm.dllm_attention(q, k, v, L, L, H, Hkv, dh, o)
        for i in range(5):
            run(i)
        torch.cuda.synchronize()
        # the launches replayed from a CUDA graph: device time, not host launch time
        reps = max(20, min(args.steps, 200))
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for i in range(reps):
                run(i)
        g.replay()
        torch.cuda.synchronize()
        # replays for about half a second, long enough for the clock sampler to see it
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        n_rep = max(1, min(2000, int(0.5 / max(e0.elapsed_time(e1) * 1e-3, 1e-6))))
        sampler.start()
        e0.record()
        for _ in range(n_rep):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        clocks = sampler.stop()
        assert dllm.dllm_get_device_status() == dllm.DLLM_OK
        us = e0.elapsed_time(e1) * 1e3 / (reps * n_rep)
        del g
        nt = dllm.dllm_debug_attention_tiles(L, H, torch.cuda.get_device_properties(dev).multi_processor_count)
        flops = 4.0 * L * L * dh * H
        t_tc = flops / (peak_tf * 1e12) * 1e6
        t_sfu = L * L * H / SFU_EX2_PER_S * 1e6
        tstar = max(t_tc, t_sfu)
        lines.append({"metric": "f16 tensor TFLOP/s of dllm_attention (% of t*)", "config": {
            "workload": "attn", "model": model.name, "Lq": L, "Lk": L, "heads": H, "kv_heads": Hkv, "dh": dh},
            "us": round(us, 2), "tflops": round(flops / (us * 1e-6) / 1e12, 1), "t_star_us": round(tstar, 2),
            "bound": "tensor" if t_tc >= t_sfu else "sfu", "frac": round(tstar / us, 4),
            "peak_tflops": peak_tf, "peak_source": peak_kind, "query_tiles_per_cta": nt,
            "ctas": -(-L // (128 * nt)) * H,
            "timing": f"CUDA events around {n_rep} replays of a graph of {reps} launches, inputs rotated over "
                      f"{copies} copies beyond L2", "clocks": clocks})
        del ins, o
        torch.cuda.empty_cache()
    return lines


def run_config(args):
    """Device time of each launch of a single-GEMM workload, weights rotated over enough
    copies to exceed L2, against t* = max(bytes / HBM, ops / int8 peak) per launch."""
    import torch
    from quantized_int8_gemm_q4_b200 import build, dllm, synth
    build.build()
    dllm.load()
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    model = synth.MODELS[args.model]()
    if args.config == "act":
        return run_act_config(args, dllm, torch, dev, model)
    if args.config == "attn":
        return run_attn_config(args, dllm, torch, dev, model)
    hbm_gbs, peak_kind = load_peaks()
    p_meas = measure_int8_peak(dllm, torch, dev)
    lines = []
    for label, gemms, M, R in config_cases(args.config, model):
        mats = []  # per launch: list of weight-copy tuples
        for gi, g in enumerate(gemms):
            parts = ([(model.q_out, 0), (model.kv_out, 1), (model.kv_out, 2)] if g.name == "qkv" else
                     [(model.ffn, 0), (model.ffn, 1)] if g.name == "gate_up" else [(g.N, 0)])
            wbytes = sum(dllm.dllm_repacked_bytes(g.qtype, n, g.K) for n, _ in parts)
            copies = max(1, min(8, int(3 * 126e6 // wbytes) + 1))
            cps = []
            for c in range(copies):
                ws_ = []
                for n, pi in parts:
                    gg = synth.device_weights(g.qtype, n, g.K, 4, gi, pi, c, device=dev)
                    w = torch.empty(dllm.dllm_repacked_bytes(g.qtype, n, g.K), dtype=torch.uint8, device=dev)
                    {Q4: dllm.dllm_repack_q4k, Q6: dllm.dllm_repack_q6k, Q8: dllm.dllm_repack_q80}[g.qtype](gg, n, g.K, w)
                    del gg
                    ws_.append(w)
                cps.append(ws_)
            mats.append(cps)
        acts = {}
        for g in gemms:
            if g.K not in acts:
                x = synth.device_activations(M, g.K, 4, g.K, device=dev)
                acts[g.K] = dllm.alloc_act(M, g.K, dev)
                dllm.dllm_quantize_act(x, M, g.K, g.K, *acts[g.K])
        rows = torch.from_numpy(synth.block_rows(M, R, 4)).to(dev) if R else None
        outs = [torch.empty((R or M, g.N), device=dev) for g in gemms]
        wsb = max(dllm.dllm_qgemm_workspace_bytes(g.qtype, g.N, g.K, M, R or 0) for g in gemms)
        work = dllm.alloc_workspace(max(wsb, 256), dev)

        def launch(gi, i):
            g, w = gemms[gi], mats[gi][i % len(mats[gi])]
            o = outs[gi]
            if g.name == "qkv":
                dllm.dllm_qkv_qgemm(w[0], w[1], w[2], Q4, model.q_out, model.kv_out, g.K, *acts[g.K], M,
                                    o[:, :model.q_out], g.N, o[:, model.q_out:model.q_out + model.kv_out],
                                    o[:, model.q_out + model.kv_out:], g.N, work, wsb)
            elif g.name == "gate_up":
                dllm.dllm_qkv_qgemm(w[0], w[1], None, Q4, model.ffn, model.ffn, g.K, *acts[g.K], M,
                                    o[:, :model.ffn], g.N, o[:, model.ffn:], None, g.N, work, wsb)
            else:
                dllm.dllm_qgemm(w[0], g.qtype, g.N, g.K, *acts[g.K], M, rows, R or 0, o, g.N, work, wsb)
        reps = max(20, args.steps)
        res = []
        for gi, g in enumerate(gemms):
            for i in range(5):
                launch(gi, i)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for i in range(reps):
                launch(gi, i)
            e1.record()
            torch.cuda.synchronize()
            us = e0.elapsed_time(e1) * 1e3 / reps
            t_hbm = g.bytes / (hbm_gbs * 1e9) * 1e6
            t_tc = g.ops / p_meas * 1e6 if p_meas else g.ops / P_INT8_NOMINAL * 1e6
            tstar = max(t_hbm, t_tc)
            res.append({"launch": g.name, "N": g.N, "K": g.K, "rows_out": g.M_out, "us": round(us, 2),
                        "t_star_us": round(tstar, 2), "frac": round(tstar / us, 4),
                        "bound": "hbm" if t_hbm >= t_tc else "tensor",
                        "int8_tops": round(g.ops / (us * 1e-6) / 1e12, 1),
                        "weight_gbs": round(g.weight_bytes / (us * 1e-6) / 1e9, 1)})
        assert dllm.dllm_get_device_status() == dllm.DLLM_OK
        tot_us = sum(r["us"] for r in res)
        tot_star = sum(r["t_star_us"] for r in res)
        lines.append({"metric": METRIC, "config": {"workload": args.config, "case": label, "canvas_tokens": M,
                                                    "model": model.name},
                      "launches": res, "us": round(tot_us, 2), "t_star_us": round(tot_star, 2),
                      "frac": round(tot_star / tot_us, 4), "hbm_gbs": hbm_gbs, "hbm_source": peak_kind,
                      "p_int8_tops_measured": round(p_meas / 1e12, 1) if p_meas else None,
                      "timing": f"CUDA events over {reps} launches, weights rotated over copies beyond L2"})
        del mats, outs, work
        torch.cuda.empty_cache()
    return lines


# ---------------------------------------------------------------------------- reference arm

def run_reference(args):
    """The oracle on the host cores: same metric, each step a bounded sample of the step.

    One sample = one layer's fused quantizers on full rows (RMSNorm -> quantize for the
    attention and FFN inputs, quantize for O, SwiGLU -> quantize for down) and the same
    fraction phi of the output columns of every projection (Q, K, V, O, gate, up, down)
    and of the output projection on the requested rows, so the op mix is the step's.
    phi is calibrated so that warm-up + steps take about two minutes."""
    import oracle
    from quantized_int8_gemm_q4_b200 import synth
    model = synth.MODELS[args.model]()
    L, h, f, seed = args.canvas, model.hidden, model.ffn, 4
    nt = oracle.max_threads()
    projs = [(p.name, p.qtype, p.N, p.K, synth.weights(p.qtype, p.N, p.K, seed, 0, pi))
             for pi, p in enumerate(model.layer)]
    R = min(L, model.out_rows)
    w_out = synth.weights(Q6, model.vocab, h, seed, 999, 0)
    x_attn, x_o, x_ffn, x_fin = (synth.activations(L, h, seed, 100 + i) for i in (0, 1, 2, 4))
    g_ffn = synth.activations(L, f, seed, 200)
    u_ffn = synth.activations(L, f, seed, 201)
    gam = synth.norm_weights(3, h, seed)
    rows = synth.block_rows(L, R, seed) if L >= 64 else np.arange(R, dtype=np.int32)
    eps = model.norm_eps

    def sample(phi, i):
        """One step's sample; returns its int8 ops."""
        qa, sa, _ = oracle.rmsnorm_quantize(x_attn, gam[0], eps)
        qo, so, _ = oracle.quantize_act(x_o)
        qf, sf, _ = oracle.rmsnorm_quantize(x_ffn, gam[1], eps)
        qd, sd, _ = oracle.swiglu_quantize(g_ffn, u_ffn)
        qr, sr, _ = oracle.rmsnorm_quantize(x_fin[rows], gam[2], eps)
        acts = {"q": (qa, sa), "k": (qa, sa), "v": (qa, sa), "o": (qo, so), "gate": (qf, sf), "up": (qf, sf),
                "down": (qd, sd)}
        ops = 0
        for name, qt, N, K, w in projs:
            cols = max(1, int(round(phi * N)))
            n0 = (i * cols) % (N - cols + 1)
            oracle.qgemm(qt, w, N, K, *acts[name], n0=n0, n1=n0 + cols, nthreads=nt)
            ops += 2 * L * cols * K
        cols = max(1, int(round(phi * model.vocab)))
        n0 = (i * cols) % (model.vocab - cols + 1)
        oracle.qgemm(Q6, w_out, model.vocab, h, qr, sr, n0=n0, n1=n0 + cols, nthreads=nt)
        return ops + 2 * R * cols * h

    phi0 = 1.0 / 512
    t0 = time.perf_counter()
    sample(phi0, 0)
    t_cal = time.perf_counter() - t0
    budget = 120.0 / max(1, args.steps + args.warmup)
    phi = float(min(1.0, max(1.0 / 8192, phi0 * budget / max(t_cal, 1e-9))))
    for i in range(args.warmup):
        sample(phi, i)
    t0 = time.perf_counter()
    ops = 0
    for i in range(args.steps):
        ops += sample(phi, i)
    dt = time.perf_counter() - t0
    v = ops / dt / 1e12
    desc = (f"per step: one layer's fused quantizers on full rows (M={L}) and {phi:.5f} of the output columns of "
            f"every projection (Q, K, V, O, gate, up, down) and of the output projection on {R} rows")
    return {
        "impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "ms_per_step_note": "time of one bounded sample, not of a full step",
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": workload_config(model, L, model.n_layers, R, args.gpus),
        "cpu_baseline": {"value": round(v, 6), "unit": UNIT, "cores": nt, "kind": "oracle", "sample": desc},
        "e2e": {"value": round(v, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    if args.record_traffic:
        print(json.dumps(record_traffic(args)["per_launch_bytes"]), flush=True)
        return
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if args.config:
        for line in run_config(args):
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    res = run_nsplit(args, rank, world) if args.parallel == "nsplit" else run_ours(args, rank, world)
    if rank == 0:
        print(json.dumps(res), flush=True)
    par = res.get("parity") or {}
    parity_failed = bool(par.get("checked")) and par["max_err_over_bound"] > 1.0
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if parity_failed:
        sys.exit("parity check failed: the GPU step's outputs are outside the oracle's bound")


if __name__ == "__main__":
    main()
