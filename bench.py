#!/usr/bin/env python
"""Benchmark of the MXFP8 grouped expert MLP (forward + backward) on B200.

One step = one pass of the whole hot path over one batch: MXFP8 quantisation of W1
and W2, routing, permute + quantise of x, fc1 grouped GEMM with the fused
SwiGLU x prob -> MXFP8 epilogue, fc2 grouped GEMM, combine, then the backward
(permute + quantise of dy, fc2 data-gradient GEMM with the fused SwiGLU backward,
dprob reduction, fc2 and fc1 weight-gradient GEMMs, fc1 data-gradient GEMM, combine).

Default workload: the Mixtral-8x7B-shaped layer (8192 tokens, hidden 4096, FFN 14336,
8 experts, top-2). Prints one JSON line (rank 0). `--impl reference` times the fp64
CPU oracle on a bounded sample of the same workload instead.

Multi-GPU (`torchrun ... bench.py --gpus N`): independent replicas, one per GPU (the
path has no exchange step on one node without expert parallelism): weak scaling,
timing = max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "grouped-MLP fwd+bwd TFLOP/s & tokens/s on 1 B200; % of MXFP8 peak / HBM BW"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP8_OVER_BF16 = 4.5 / 2.25     # nominal dense ratio (MXFP8 / bf16) on B200
SPEC_FP8_TFLOPS = 4500.0
GEMM_FLOP_FACTOR = {"fc1_swiglu": 4, "fc2": 2, "fc2_dgrad_swiglu_bwd": 2, "fc2_wgrad": 2, "fc1_dgrad": 4,
                    "fc1_wgrad": 4}     # x M*H*F
GEMM_KERNEL_SOURCES = ["mxfp8_grouped_gemm_moe_b200/csrc/gemm.cu", "mxfp8_grouped_gemm_moe_b200/csrc/ptx_sm100.cuh",
                       "mxfp8_grouped_gemm_moe_b200/csrc/mxmoe_device.cuh",
                       "mxfp8_grouped_gemm_moe_b200/csrc/tensor_map.h"]
QUANT_KERNEL_SOURCES = ["mxfp8_grouped_gemm_moe_b200/csrc/quantize.cu",
                        "mxfp8_grouped_gemm_moe_b200/csrc/mxmoe_device.cuh",
                        "mxfp8_grouped_gemm_moe_b200/csrc/ptx_sm100.cuh"]


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["mxmoe", "reference"], default="mxmoe")
    p.add_argument("--config", default="mixtral", help="tiny | small | mixtral | mixtral_zipf | genomics")
    p.add_argument("--tokens", type=int, default=0, help="override the token count (profiling runs)")
    p.add_argument("--experts", type=int, default=0, help="override the expert count (profiling runs)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-rows", type=int, default=512, help="routed rows in the CPU oracle sample")
    p.add_argument("--cpu-fslice", type=int, default=2048, help="FFN columns in the CPU oracle sample")
    p.add_argument("--no-bf16-compare", action="store_true",
                   help="skip the comparison timings (the bf16 layer's step, the alternative recipes)")
    p.add_argument("--no-workloads", action="store_true",
                   help="skip the other workloads' steps (Mixtral with Zipf routing, genomics)")
    p.add_argument("--stage", choices=["all", "permute_quantize"], default="all",
                   help="permute_quantize: time only the routing and the gathered permute + quantise of x "
                        "(a profiling case that holds well under 1 GB); prints its own JSON line")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


_COMMENT = re.compile(r"//[^\n]*|/\*.*?\*/", re.S)


def source_hash(paths, root=ROOT):
    """Hash of the kernel sources' code: comments and whitespace are dropped, so that a
    change to the comments alone keeps a traffic measurement valid."""
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(root, p), encoding="utf-8") as f:
            code = _COMMENT.sub(" ", f.read())
        h.update(" ".join(code.split()).encode())
    return h.hexdigest()[:16]


def load_traffic(kernel_key, paths, units):
    """DRAM bytes (read + write) per launch from the committed ncu summary
    profiles/dram_traffic.txt, if it was taken on the current kernel source (else None).
    Line format: <kernel key> <source hash> <DRAM bytes per unit of work>."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        f = line.split()
        if len(f) == 3 and not line.startswith("#") and f[0] == kernel_key:
            return float(f[2]) * units if f[1] == source_hash(paths) else None
    return None


# ----------------------------------------------------------------------------- clocks
def smi_id(dev_index):
    """nvidia-smi's id of CUDA device `dev_index`: its UUID (nvidia-smi numbers every GPU of
    the machine and ignores CUDA_VISIBLE_DEVICES, so an index could name another GPU)."""
    try:
        import torch
        u = str(torch.cuda.get_device_properties(dev_index).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev_index)


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    _n = 0

    def __init__(self, gpu_index):
        self.gpu = smi_id(gpu_index)
        self.proc = None
        ClockSampler._n += 1   # one file per sampler: several run in one process
        self.path = os.path.join("/tmp", f"mxmoe_clocks_{os.getpid()}_{ClockSampler._n}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append(dict(sm=float(f[1]), smax=float(f[2]), power=float(f[3]), hw=f[5], hwt=f[6], swt=f[7],
                                 pcap=f[8]))
            except ValueError:
                continue
        os.remove(self.path)
        if not rows:
            return None
        pmax = max(r["power"] for r in rows)
        load = [r for r in rows if r["power"] >= 0.5 * pmax] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                              ("pcap", "sw_power_cap")):
                if r[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(load), "power_w_max": pmax}


# ----------------------------------------------------------------------------- distributed
def dist_setup(args):
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import torch
        import torch.distributed as dist
        lr = int(os.environ.get("LOCAL_RANK", "0"))
        if args.impl == "mxmoe":
            torch.cuda.set_device(lr)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", lr))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=600))
        return dist, dist.get_rank(), ws, lr
    return None, 0, 1, 0


def barrier(dist):
    if dist is not None:
        dist.barrier()


def max_over_ranks(dist, v):
    if dist is None:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- CPU oracle sample
def _keep_freed_memory():
    """glibc: serve large numpy temporaries from the heap and keep freed memory, so the
    CPU baseline is not dominated by page faults on fresh mmap'd buffers."""
    try:
        import ctypes
        libc = ctypes.CDLL("libc.so.6")
        libc.mallopt(-3, 1 << 30)        # M_MMAP_THRESHOLD
        libc.mallopt(-1, 2 ** 31 - 1)    # M_TRIM_THRESHOLD
    except OSError:
        pass


def oracle_sample(cfg, rows, f_slice):
    """The fp64 oracle (as it stands) on a bounded sample of the workload: the first
    `rows` tokens routed to expert 0 and the first `f_slice` FFN columns of that
    expert (gate rows [0, f), up rows [F, F+f), W2 columns [0, f)), forward + backward.
    Every step of the path scales linearly in rows and in f, so the sample's
    throughput stands for the workload's. Returns (seconds, flops, description, rows)."""
    import numpy as np

    import moe_workloads as wl
    from oracle import moe as omoe

    _keep_freed_memory()
    idx, probs = wl.make_routing(cfg)
    sel = (idx == 0).nonzero()[:rows]
    toks, slots = sel[:, 0], sel[:, 1]
    M = len(toks)
    fs = min(f_slice, cfg.F)
    x = wl.make_activations(cfg)[toks]
    dy = wl.make_grad_output(cfg)[toks]
    p = probs[toks, slots].reshape(M, 1)
    W1, W2 = wl.make_expert_weights(cfg, 0)
    W1s = np.concatenate([W1[:fs].float().numpy(), W1[cfg.F:cfg.F + fs].float().numpy()]).astype(np.float64)
    W2s = W2[:, :fs].float().numpy().astype(np.float64)
    f = lambda t: t.float().numpy().astype(np.float64)  # noqa: E731
    xs, dys, ps = f(x), f(dy), f(p)
    one = np.zeros((M, 1), dtype=np.int64)
    t0 = time.perf_counter()
    _, saved = omoe.mlp_fwd(xs, one, ps, W1s[None], W2s[None])
    omoe.mlp_bwd(dys, saved, ps, W1s[None], W2s[None])
    dt = time.perf_counter() - t0
    desc = (f"expert 0 of the {cfg.name} workload: its first {M} routed rows x H={cfg.H} x the first {fs} of "
            f"F={cfg.F} FFN columns (weights sliced accordingly); fp64 numpy oracle forward+backward incl. "
            f"MXFP8 quantisation of weights and activations")
    return dt, 18.0 * M * cfg.H * fs, desc, M


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def run_reference(args, cfg, dist, rank, world):
    if rank != 0:
        return
    times, flops, desc, M = [], 0.0, "", 0
    for i in range(args.warmup + args.steps):
        dt, flops, desc, M = oracle_sample(cfg, args.cpu_rows, args.cpu_fslice)
        if i >= args.warmup:
            times.append(dt)
    sec = sum(times) / len(times)
    tflops = flops / sec / 1e12
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": tflops, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_json(cfg, world),
            "tokens_per_s": tflops * 1e12 / (18.0 * cfg.k * cfg.H * cfg.F),
            "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
            "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_json(cfg, world):
    return {"workload": f"{cfg.name}: MoE expert MLP layer, {cfg.T} tokens, hidden {cfg.H}, FFN {cfg.F}, "
                        f"{cfg.E} experts, top-{cfg.k}, fwd+bwd",
            "tokens": cfg.T, "hidden": cfg.H, "ffn": cfg.F, "experts": cfg.E, "top_k": cfg.k,
            "routing": cfg.routing, "seed": cfg.seed, "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
            "l2": "inputs larger than L2 (weights alone are several GB); no flush needed",
            "flops_per_step": cfg.fwdbwd_flops}


# ----------------------------------------------------------------------------- GPU arm
def time_recipes(cfg, layer, W1, W2, x, idx, probs, dy, y, dx, dW1, dW2, dprobs, stream, steps):
    """The same full step (weights quantised, forward, backward) under the layer's
    alternative recipes, beside the headline: E5M2 gradients (the backward's dY and dGU in
    E5M2), G / U recomputed in the backward instead of saved, the round-up scale rule, and
    per-tensor FP8 in place of MXFP8. CUDA events over `steps` steps after two warm-up
    steps; the saved-activation bytes of each recipe."""
    import torch

    import mxfp8_grouped_gemm_moe_b200 as mx
    lib = mx.load()
    a = (cfg.T, cfg.k, cfg.E, cfg.H, cfg.F)
    out = {}
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for name, recipe in (("grad_e5m2", mx.RECIPE_GRAD_E5M2), ("recompute_gu", mx.RECIPE_RECOMPUTE_GU),
                         ("scale_ceil", mx.RECIPE_SCALE_CEIL)):
        rule = mx.SCALE_RULE_CEIL if recipe & mx.RECIPE_SCALE_CEIL else mx.SCALE_RULE_OCP
        if recipe & mx.RECIPE_RECOMPUTE_GU:
            saved = torch.empty(lib.grouped_mlp_saved_size_ex(*a, recipe), dtype=torch.uint8, device=x.device)
            ws = torch.empty(lib.grouped_mlp_workspace_size_ex(*a, recipe), dtype=torch.uint8, device=x.device)
        else:
            saved, ws = layer.saved, layer.ws

        def step():
            mx.mxmoe_weights_quantize(W1, W2, out=layer.wq, scale_rule=rule)
            mx.grouped_mlp_fwd(x, idx, probs, layer.wq, cfg.E, cfg.F, saved, ws, y, recipe=recipe)
            mx.grouped_mlp_bwd(dy, saved, layer.wq, *a, ws, dx, dW1, dW2, dprobs, recipe=recipe)
        for _ in range(2):
            step()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / steps
        out[name] = {"ms_per_step": ms, "tflops": cfg.fwdbwd_flops / (ms * 1e-3) / 1e12,
                     "saved_bytes": lib.grouped_mlp_saved_size_ex(*a, recipe),
                     "workspace_bytes": lib.grouped_mlp_workspace_size_ex(*a, recipe)}
        del saved, ws
    torch.cuda.empty_cache()
    # per-tensor FP8 (its own layer object: weights with per-expert amax, delayed scaling of
    # Z / dGU rolled after every step, as a training loop would)
    fl = mx.GroupedMLP(*a, device=x.device, precision="fp8")
    fl.quantize_weights(W1, W2)
    fl.forward(x, idx, probs, y)
    fl.backward(dy, dx, dW1, dW2, dprobs)
    fl.roll_amax()

    def fstep():
        fl.quantize_weights(W1, W2)
        fl.forward(x, idx, probs, y)
        fl.backward(dy, dx, dW1, dW2, dprobs)
        fl.roll_amax()
    for _ in range(2):
        fstep()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        fstep()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    out["fp8_tensor"] = {"ms_per_step": ms, "tflops": cfg.fwdbwd_flops / (ms * 1e-3) / 1e12,
                         "saved_bytes": lib.grouped_mlp_saved_size_ex(*a, mx.RECIPE_FP8_TENSOR),
                         "workspace_bytes": lib.grouped_mlp_workspace_size_ex(*a, mx.RECIPE_FP8_TENSOR),
                         "note": "per-tensor FP8 E4M3 (one fp32 multiplier per tensor, per expert for the weights; "
                                 "delayed scaling of Z and dGU); includes the amax passes over x, dY and the weights"}
    del fl
    torch.cuda.empty_cache()
    out["default_saved_bytes"] = lib.grouped_mlp_saved_size(*a)
    out["note"] = ("same step as the headline under each recipe; tflops counts the headline's algorithmic FLOPs "
                   "(the recompute's extra fc1 GEMM is not credited)")
    return out


def layer_memory(cfg):
    """Device bytes of the layer's buffers, MXFP8 vs bf16: prepared weights, activations
    saved by the forward for the backward, and scratch."""
    import mxfp8_grouped_gemm_moe_b200 as mx
    lib = mx.load()
    a = (cfg.T, cfg.k, cfg.E, cfg.H, cfg.F)
    return {"mxfp8": {"weights": lib.mxmoe_weights_size(cfg.E, cfg.H, cfg.F),
                      "saved": lib.grouped_mlp_saved_size(*a), "workspace": lib.grouped_mlp_workspace_size(*a)},
            "bf16": {"weights": lib.mxmoe_weights_bf16_size(cfg.E, cfg.H, cfg.F),
                     "saved": lib.grouped_mlp_bf16_saved_size(*a),
                     "workspace": lib.grouped_mlp_bf16_workspace_size(*a)}}


def time_bf16_layer(cfg, W1, W2, x, idx, probs, dy, stream, dev, steps):
    """The same fused forward + backward on the bf16 layer (grouped_mlp_bf16_*: bf16 copies
    instead of quantisers, kind::f16 GEMMs, bf16 Z / dGU from the fused epilogues), weights
    prepared every step as in the MXFP8 step: the 16-bit comparison point."""
    import torch

    import mxfp8_grouped_gemm_moe_b200 as mx
    layer = mx.GroupedMLP(cfg.T, cfg.k, cfg.E, cfg.H, cfg.F, device=dev, precision="bf16")
    y = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)
    dx = torch.empty_like(y)
    dW1 = torch.empty((cfg.E, 2 * cfg.F, cfg.H), dtype=torch.float32, device=dev)
    dW2 = torch.empty((cfg.E, cfg.H, cfg.F), dtype=torch.float32, device=dev)
    dprobs = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=dev)

    def step():
        layer.quantize_weights(W1, W2)
        layer.forward(x, idx, probs, y)
        layer.backward(dy, dx, dW1, dW2, dprobs)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    mx.mxmoe_profile_enable(64 * (steps + 1))
    mx.mxmoe_profile_read()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    stages = mx.mxmoe_profile_read()
    mx.mxmoe_profile_disable()
    ms = e0.elapsed_time(e1) / steps
    per = {}
    for name, t in stages:
        per.setdefault(name, []).append(t)
    MHF = float(cfg.M) * cfg.H * cfg.F
    st_ms = {n: sum(v) / len(v) for n, v in per.items()}
    out = {"ms_per_step": ms, "tflops": cfg.fwdbwd_flops / (ms * 1e-3) / 1e12, "stages_ms": st_ms,
           "gemm_tflops": {n: GEMM_FLOP_FACTOR[n] * MHF / (t * 1e-3) / 1e12
                           for n, t in st_ms.items() if n in GEMM_FLOP_FACTOR},
           "note": "bf16 layer (grouped_mlp_bf16_fwd/bwd), same step as the headline; quant_* stages are "
                   "bf16 row + transposed copies here"}
    del layer, y, dx, dW1, dW2, dprobs
    torch.cuda.empty_cache()
    return out


def hbm_stage_bytes(cfg):
    """Algorithmic HBM bytes of the bandwidth-bound stages (one read of the inputs, one
    write of the outputs, scales included)."""
    return {
        "quant_x": cfg.T * cfg.H * 2 + 2 * (cfg.M * cfg.H + cfg.M * cfg.H / 32),
        "quant_dy": cfg.T * cfg.H * 2 + 2 * (cfg.M * cfg.H + cfg.M * cfg.H / 32),
        "combine": cfg.M * cfg.H * 2 + cfg.T * cfg.H * 2,
        "combine_dx": cfg.M * cfg.H * 2 + cfg.T * cfg.H * 2,
        "quant_w1": cfg.E * 2 * cfg.F * cfg.H * (2 + 2 * (1 + 1 / 32)),
        "quant_w2": cfg.E * cfg.F * cfg.H * (2 + 2 * (1 + 1 / 32)),
    }


def stage_table(cfg, stages, peaks):
    """Per-stage mean time over the timed steps, with TFLOP/s (GEMMs) or GB/s (HBM-bound
    stages) and the fraction of the measured peak."""
    MHF = float(cfg.M) * cfg.H * cfg.F
    fp8_peak = peaks["bf16_tflops_sustained"] * FP8_OVER_BF16
    hbm_bytes = hbm_stage_bytes(cfg)
    per = {}
    for name, t in stages:
        per.setdefault(name, []).append(t)
    out = {}
    for name, ts in per.items():
        a = sum(ts) / len(ts)
        ent = {"ms": a, "launches": len(ts)}
        if name in GEMM_FLOP_FACTOR:
            tf = GEMM_FLOP_FACTOR[name] * MHF / (a * 1e-3) / 1e12
            ent.update(tflops=tf, frac_of_measured=tf / fp8_peak, frac_of_spec=tf / SPEC_FP8_TFLOPS)
        elif name in hbm_bytes:
            gbs = hbm_bytes[name] / (a * 1e-3) / 1e9
            ent.update(gbs=gbs, frac_of_measured=gbs / peaks["hbm_gbs"])
        out[name] = ent
    return out


def time_workload(name, dev, steps, warmup, peaks):
    """One more workload's full step (weights quantised, forward, backward), timed on its
    own with CUDA events: ms, TFLOP/s, tokens/s, per-stage fractions and the clocks seen.
    Inputs as for the headline (routing from the CPU recipe, dense tensors from a seeded
    CUDA generator), already resident in HBM."""
    import torch

    import moe_workloads as wl
    import mxfp8_grouped_gemm_moe_b200 as mx
    cfg = wl.CONFIGS[name]
    idx_h, probs_h = wl.make_routing(cfg)
    g = torch.Generator(device=dev)
    g.manual_seed(cfg.seed)
    W1 = (torch.randn((cfg.E, 2 * cfg.F, cfg.H), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    W2 = (torch.randn((cfg.E, cfg.H, cfg.F), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    x = torch.randn((cfg.T, cfg.H), generator=g, device=dev).to(torch.bfloat16)
    dy = torch.randn((cfg.T, cfg.H), generator=g, device=dev).to(torch.bfloat16)
    idx, probs = idx_h.to(dev), probs_h.to(dev)
    layer = mx.GroupedMLP(cfg.T, cfg.k, cfg.E, cfg.H, cfg.F, device=dev)
    y = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)
    dx = torch.empty_like(y)
    dW1 = torch.empty((cfg.E, 2 * cfg.F, cfg.H), dtype=torch.float32, device=dev)
    dW2 = torch.empty((cfg.E, cfg.H, cfg.F), dtype=torch.float32, device=dev)
    dprobs = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        layer.quantize_weights(W1, W2)
        layer.forward(x, idx, probs, y)
        layer.backward(dy, dx, dW1, dW2, dprobs)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index or 0)
    mx.mxmoe_profile_enable(64 * (steps + 1))
    mx.mxmoe_profile_read()
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    stages = mx.mxmoe_profile_read()
    mx.mxmoe_profile_disable()
    ms = e0.elapsed_time(e1) / steps
    st = stage_table(cfg, stages, peaks)
    gemm_ms = sum(v["ms"] for n, v in st.items() if n in GEMM_FLOP_FACTOR)
    MHF = float(cfg.M) * cfg.H * cfg.F
    m_splits = torch.bincount(idx_h.reshape(-1).long(), minlength=cfg.E)
    out = {"config": config_json(cfg, 1), "ms_per_step": ms, "tflops": cfg.fwdbwd_flops / (ms * 1e-3) / 1e12,
           "tokens_per_s": cfg.T / (ms * 1e-3), "gemm_tflops": 18.0 * MHF / (gemm_ms * 1e-3) / 1e12,
           "gemm_frac_of_measured_fp8": 18.0 * MHF / (gemm_ms * 1e-3) / 1e12
           / (peaks["bf16_tflops_sustained"] * FP8_OVER_BF16),
           "m_splits_min_max": [int(m_splits.min()), int(m_splits.max())], "stages": st, "clocks": clk,
           "steps": steps, "warmup": warmup}
    del layer, W1, W2, x, dy, y, dx, dW1, dW2, dprobs
    torch.cuda.empty_cache()
    return out


def run_permute_quantize(args, cfg):
    """Profiling mode: the routing, then --warmup untimed and --steps timed calls of the
    gathered permute + quantise of x (rowwise and colwise MXFP8, MMA scale layout) into
    preallocated outputs through the C ABI, each timed call after an L2 flush."""
    import ctypes
    import statistics

    import torch

    import moe_workloads as wl
    import mxfp8_grouped_gemm_moe_b200 as mx

    lib = mx.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    idx_h, probs_h = wl.make_routing(cfg)
    g = torch.Generator(device=dev)
    g.manual_seed(cfg.seed)
    x = torch.randn((cfg.T, cfg.H), generator=g, device=dev).to(torch.bfloat16)
    r = mx.moe_permute(idx_h.to(dev), probs_h.to(dev), cfg.E)
    cap = r["token_of_row"].numel()
    nrows = r["seg_off"][cfg.E:]
    row = mx.MXFP8.empty(cap, cfg.H, mx.SCALE_MMA, dev)
    col = mx.MXFP8.empty(cfg.H, cap, mx.SCALE_MMA, dev)
    rs, cs = row.as_struct(), col.as_struct()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def call():
        st = lib.mxfp8_quantize(mx._ptr(x), mx.DTYPE_BF16, 1, cfg.T, cfg.H, mx._ptr(r["token_of_row"]),
                                mx._ptr(nrows), cap, ctypes.byref(rs), ctypes.byref(cs), mx._stream())
        mx._check("mxfp8_quantize", st)

    for _ in range(args.warmup):
        call()
    ev = []
    for _ in range(args.steps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        call()
        e1.record()
        ev.append((e0, e1))
    torch.cuda.synchronize()
    ms = statistics.median(a.elapsed_time(b) for a, b in ev)
    rows = int(nrows.item())
    alg = cfg.T * cfg.H * 2 + 2 * rows * cfg.H * (1 + 1 / 32)
    print(json.dumps({"stage": "permute_quantize", "workload": cfg.name, "steps": args.steps, "ms": ms,
                      "gbs": alg / ms / 1e6, "algorithmic_bytes": alg, "rows": rows, "capacity": cap}), flush=True)


def run_gpu(args, cfg, dist, rank, world, local_rank):
    import torch

    import moe_workloads as wl
    import mxfp8_grouped_gemm_moe_b200 as mx

    mx.load()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    # inputs: routing from the workload recipe (CPU, seeded); dense tensors drawn with a
    # seeded CUDA generator (same distributions as the recipe; resident in HBM)
    idx_h, probs_h = wl.make_routing(cfg)
    g = torch.Generator(device=dev)
    g.manual_seed(cfg.seed)
    W1 = (torch.randn((cfg.E, 2 * cfg.F, cfg.H), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    W2 = (torch.randn((cfg.E, cfg.H, cfg.F), generator=g, device=dev) * 0.02).to(torch.bfloat16)
    x = torch.randn((cfg.T, cfg.H), generator=g, device=dev).to(torch.bfloat16)
    dy = torch.randn((cfg.T, cfg.H), generator=g, device=dev).to(torch.bfloat16)
    idx, probs = idx_h.to(dev), probs_h.to(dev)
    layer = mx.GroupedMLP(cfg.T, cfg.k, cfg.E, cfg.H, cfg.F, device=dev)
    y = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)
    dx = torch.empty_like(y)
    dW1 = torch.empty((cfg.E, 2 * cfg.F, cfg.H), dtype=torch.float32, device=dev)
    dW2 = torch.empty((cfg.E, cfg.H, cfg.F), dtype=torch.float32, device=dev)
    dprobs = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        layer.quantize_weights(W1, W2)
        layer.forward(x, idx, probs, y)
        layer.backward(dy, dx, dW1, dW2, dprobs)

    mx.mxmoe_clear_device_status()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- device-resident timed region (stage events on, clocks sampled)
    clocks = ClockSampler(local_rank)
    mx.mxmoe_profile_enable(64 * (args.steps + 1))
    mx.mxmoe_profile_read()
    clocks.start()
    barrier(dist)
    torch.cuda.synchronize()
    n0 = mx.mxmoe_launch_count()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(args.steps):
        step()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(dist)
    launches = mx.mxmoe_launch_count() - n0
    ms = ev0.elapsed_time(ev1) / args.steps
    stages = mx.mxmoe_profile_read()
    mx.mxmoe_profile_disable()
    ms = max_over_ranks(dist, ms)

    # ---- end to end through the public API with host buffers: every step copies its
    # inputs (x, top-k ids, probabilities, dY) from pinned host memory and reads its
    # results (y, dX, dprobs) back. The copies run on a side stream, double-buffered, so
    # step i+1's inputs travel while step i computes (a pipelined training loop); all of
    # them sit inside the timed region.
    e2e = None
    if not args.no_e2e:
        pin = lambda t: t.cpu().pin_memory()  # noqa: E731
        x_h, dy_h, idx_h2, probs_h2 = pin(x), pin(dy), pin(idx), pin(probs)
        y_h, dx_h, dp_h = pin(y), pin(dx), pin(dprobs)
        h2d = sum(t.numel() * t.element_size() for t in (x_h, dy_h, idx_h2, probs_h2))
        d2h = sum(t.numel() * t.element_size() for t in (y_h, dx_h, dp_h))
        bufs = [dict(x=torch.empty_like(x), dy=torch.empty_like(dy), idx=torch.empty_like(idx),
                     probs=torch.empty_like(probs)) for _ in range(2)]
        cs = torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()  # noqa: E731

        outs = [dict(y=torch.empty_like(y), dx=torch.empty_like(dx), dprobs=torch.empty_like(dprobs))
                for _ in range(2)]

        def run_e2e(nsteps):
            # the forward's inputs (x, routing) and the backward's (dY) complete separately,
            # so a step's forward starts while its dY is still on the way
            loaded_fwd, loaded, consumed, read_done = [None, None], [None, None], [None, None], [None, None]

            def load(i):
                b = bufs[i % 2]
                with torch.cuda.stream(cs):
                    if consumed[i % 2] is not None:
                        cs.wait_event(consumed[i % 2])
                    b["x"].copy_(x_h, non_blocking=True)
                    b["idx"].copy_(idx_h2, non_blocking=True)
                    b["probs"].copy_(probs_h2, non_blocking=True)
                    loaded_fwd[i % 2] = ev()
                    loaded_fwd[i % 2].record(cs)
                    b["dy"].copy_(dy_h, non_blocking=True)
                    loaded[i % 2] = ev()
                    loaded[i % 2].record(cs)

            load(0)
            for i in range(nsteps):
                b, o = bufs[i % 2], outs[i % 2]
                stream.wait_event(loaded_fwd[i % 2])
                if read_done[i % 2] is not None:
                    stream.wait_event(read_done[i % 2])
                if i + 1 < nsteps:
                    load(i + 1)
                layer.quantize_weights(W1, W2)
                layer.forward(b["x"], b["idx"], b["probs"], o["y"])
                fwd_done = ev()
                fwd_done.record(stream)
                stream.wait_event(loaded[i % 2])
                layer.backward(b["dy"], o["dx"], dW1, dW2, o["dprobs"])
                bwd_done = ev()
                bwd_done.record(stream)
                consumed[i % 2] = bwd_done
                with torch.cuda.stream(cs):
                    cs.wait_event(fwd_done)
                    y_h.copy_(o["y"], non_blocking=True)
                    cs.wait_event(bwd_done)
                    dx_h.copy_(o["dx"], non_blocking=True)
                    dp_h.copy_(o["dprobs"], non_blocking=True)
                    read_done[i % 2] = ev()
                    read_done[i % 2].record(cs)

        run_e2e(args.warmup)
        torch.cuda.synchronize()
        barrier(dist)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cs.wait_event(e0)
        run_e2e(args.steps)
        tail = ev()
        tail.record(cs)
        stream.wait_event(tail)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(dist)
        ems = max_over_ranks(dist, e0.elapsed_time(e1) / args.steps)
        e2e = {"value": world * cfg.fwdbwd_flops / (ems * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ems,
               "tokens_per_s": world * cfg.T / (ems * 1e-3),
               "note": "inputs copied host->device and results read back every step, on a side stream "
                       "overlapping the neighbouring steps' compute"}
    # clocks sampled over both timed runs of the step (device-resident, then end to end)
    clk = clocks.stop()
    # ---- the same step under the alternative recipes (E5M2 gradients; G / U recomputed)
    recipes = None
    if rank == 0 and world == 1 and not args.no_bf16_compare:
        recipes = time_recipes(cfg, layer, W1, W2, x, idx, probs, dy, y, dx, dW1, dW2, dprobs, stream,
                               min(args.steps, 5))

    # ---- the same step on the bf16 layer: the 16-bit comparison point, timed on its own
    bf16_layer = None
    if rank == 0 and world == 1 and not args.no_bf16_compare:
        bf16_layer = time_bf16_layer(cfg, W1, W2, x, idx, probs, dy, stream, dev, min(args.steps, 5))

    # ---- the other workloads of the target (skewed Mixtral routing; genomics), each
    # timed on its own after the headline
    workloads = None
    if rank == 0 and world == 1 and not args.no_workloads and cfg.name == "mixtral":
        peaks0, _ = load_peaks()
        workloads = {n: time_workload(n, dev, min(args.steps, 5), 2, peaks0) for n in ("mixtral_zipf", "genomics")}

    # ---- router (the step upstream of the layer; timed on its own, not part of `value`)
    router = None
    if rank == 0:
        lg = torch.randn((cfg.T, cfg.E), generator=g, device=dev)
        ridx, rp = mx.moe_router_topk(lg, cfg.k)
        rdp = torch.randn_like(rp)
        rdl = mx.moe_router_topk_bwd(lg, ridx, rdp)
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        times = []
        for fn in (lambda: mx.moe_router_topk(lg, cfg.k), lambda: mx.moe_router_topk_bwd(lg, ridx, rdp)):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            r0.record(stream)
            for _ in range(20):
                fn()
            r1.record(stream)
            torch.cuda.synchronize()
            times.append(r0.elapsed_time(r1) / 20)
        fb = cfg.T * cfg.E * 4 + cfg.T * cfg.k * 8
        bb = 2 * cfg.T * cfg.E * 4 + cfg.T * cfg.k * 8
        router = {"fwd_ms": times[0], "bwd_ms": times[1], "fwd_gbs": fb / (times[0] * 1e-3) / 1e9,
                  "bwd_gbs": bb / (times[1] * 1e-3) / 1e9,
                  "note": "softmax over all experts + top-k, and its backward, on [T, E] fp32 logits; "
                          "timed separately (the layer's input routing is given)"}
        del lg, ridx, rp, rdp, rdl


    st, where = mx.mxmoe_get_device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} (site {where}) after the benchmark")

    # ---- per-stage times and rooflines
    peaks, peak_kind = load_peaks()
    MHF = float(cfg.M) * cfg.H * cfg.F
    hbm_bytes = hbm_stage_bytes(cfg)
    fp8_peak = peaks["bf16_tflops_sustained"] * FP8_OVER_BF16
    stage_json = stage_table(cfg, stages, peaks)
    gemm_names = [n for n in stage_json if n in GEMM_FLOP_FACTOR]
    dom = max(gemm_names, key=lambda n: stage_json[n]["ms"])
    dom_units = GEMM_FLOP_FACTOR[dom] * MHF
    roofline = {"bound": "tensor", "kernel": f"mxgemm_kernel ({dom})", "achieved": stage_json[dom]["tflops"],
                "peak": fp8_peak, "unit": "TFLOP/s", "frac": stage_json[dom]["tflops"] / fp8_peak,
                "peak_source": f"{peak_kind} bf16 sustained x {FP8_OVER_BF16:g} (nominal MXFP8/bf16 ratio)",
                "frac_of_spec_4500": stage_json[dom]["tflops"] / SPEC_FP8_TFLOPS,
                "traffic": load_traffic(f"{dom}:{cfg.name}", GEMM_KERNEL_SOURCES, 1.0)}
    # the largest HBM-bound kernel of the step: the W1 quantiser (rowwise + colwise copies)
    q = stage_json.get("quant_w1", {})
    roofline_hbm = {"bound": "hbm", "kernel": "mxfp8_quantize_tma_kernel (W1 rowwise + colwise)",
                    "achieved": q.get("gbs"), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": (q.get("gbs") or 0) / peaks["hbm_gbs"], "peak_source": peak_kind,
                    "algorithmic_bytes": hbm_bytes["quant_w1"],
                    "traffic": load_traffic(f"quant_w1:{cfg.name}", QUANT_KERNEL_SOURCES, 1.0)}
    gemm_ms = sum(stage_json[n]["ms"] for n in gemm_names)
    value = world * cfg.fwdbwd_flops / (ms * 1e-3) / 1e12
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "mxfp8-e4m3 (fp32 accumulate)", "data": "synthetic",
            "config": config_json(cfg, world),
            "tokens_per_s": world * cfg.T / (ms * 1e-3),
            "gemm_tflops": (18.0 * MHF) / (gemm_ms * 1e-3) / 1e12,
            "gemm_frac_of_measured_fp8": (18.0 * MHF) / (gemm_ms * 1e-3) / 1e12 / fp8_peak,
            "roofline": roofline, "roofline_hbm": roofline_hbm, "stages": stage_json,
            "gpu_launches": launches, "e2e": e2e, "clocks": clk, "router": router}
    if workloads is not None:
        line["workloads"] = workloads
    if recipes is not None:
        line["recipes"] = recipes
    if bf16_layer is not None:
        bf16_layer["speedup_mxfp8_over_bf16"] = bf16_layer["ms_per_step"] / ms
        bf16_layer["memory_bytes"] = layer_memory(cfg)
        line["bf16_layer"] = bf16_layer
    return line


def main():
    args = parse_args()
    dist, rank, world, local_rank = dist_setup(args)
    import dataclasses

    import moe_workloads as wl
    cfg = wl.CONFIGS[args.config]
    if args.tokens:
        cfg = dataclasses.replace(cfg, T=args.tokens, name=f"{cfg.name}_T{args.tokens}")
    if args.experts:
        cfg = dataclasses.replace(cfg, E=args.experts, k=min(cfg.k, args.experts), name=f"{cfg.name}_E{args.experts}")
    try:
        if args.impl == "reference":
            run_reference(args, cfg, dist, rank, world)
            return
        if args.stage == "permute_quantize":
            if rank == 0:
                run_permute_quantize(args, cfg)
            return
        line = run_gpu(args, cfg, dist, rank, world, local_rank)
        if rank == 0:
            if not args.no_cpu_baseline and world == 1:
                dt, flops, desc, M = oracle_sample(cfg, args.cpu_rows, args.cpu_fslice)
                line["cpu_baseline"] = {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
                                        "kind": "oracle", "sample": desc, "seconds": dt,
                                        "tokens_per_s": flops / dt / (18.0 * cfg.k * cfg.H * cfg.F)}
            print(json.dumps(line), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
