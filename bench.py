"""Benchmark of the SMoE MLP forward + backward (one B200 per process).

A step is one pass of the whole path over one batch of synthetic tokens:
router (logits, top-k, gates), reorder (sort), the six expert GEMMs (H = x W1 with
the activation, y = A W2 gated and combined, dA' = dy W2^T with the gate-gradient
and activation-backward epilogue, dW2, dW1, dx = dH W1^T combined), the router
backward and every weight gradient written in full.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own replica on its GPU (the path has
no exchange step of its own): the timed region is bracketed by a barrier and a
device synchronisation, and the elapsed time is the maximum over ranks.
Rank 0 prints one JSON line.

--impl reference times the CPU oracle (the plain fp64 restatement of the method)
on the host cores, on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from sparse_mixture_experts_smoe_b200.inputs import (  # noqa: E402
    WORKLOADS, make_mlp_inputs, make_moa_inputs, mlp_flops, moa_attn_flops)

METRIC = "SMoE MLP fwd+bwd tokens/s on 1 B200; % of dense BF16 tensor peak"
METRIC_MOA = "Mixture-of-Attention layer (router, per-expert Wq/Wo, shared Wk/Wv, causal attention core) fwd+bwd tokens/s on 1 B200"
# NVIDIA's nominal dense (no 2:4 sparsity) bf16 tensor throughput of one B200.
NOMINAL_DENSE_BF16_TFLOPS = 2250.0
DEFAULT_WORKLOAD = "mixtral_bf16_swiglu"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ---------------------------------------------------------------------------
# distributed plumbing (replicas only)
# ---------------------------------------------------------------------------
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch.distributed as dist
    dev = torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self):
        self.lines, self.proc, self.thread = [], None, None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        try:
            uuid = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
            cmd += ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            pass
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# per-kernel algorithmic work (FLOPs for the GEMMs, bytes for the rest)
# ---------------------------------------------------------------------------
def kernel_work(cfg):
    T, d, f, E, k = cfg["T"], cfg["d"], cfg["f"], cfg["E"], cfg["k"]
    S = T * k
    mf = 2 * f if cfg["act"] == "swiglu" else f
    b = 4 if cfg.get("dtype") == "f32" else 2  # bytes per element of the layer's dtype
    flops = {
        "gemm.fwd_up": 2.0 * S * d * mf, "gemm.fwd_down": 2.0 * S * f * d,
        "gemm.bwd_dA": 2.0 * S * d * f, "gemm.bwd_dW2": 2.0 * S * f * d,
        "gemm.bwd_dW1": 2.0 * S * d * mf, "gemm.bwd_dx": 2.0 * S * mf * d,
    }
    bytes_ = {
        "route": T * d * b + d * E * b + S * 8,
        "sort": 2 * S * 4 + S * 4 + (E + 1) * 4,
        # slot rows in the layer dtype (+ one int32 grouped row per slot), output rows
        "combine.y": S * d * b + S * 4 + T * d * b,
        "combine.dx": S * d * b + S * 4 + T * d * b + S * 8,
        "dg_reduce": S * 4 * max(1, math.ceil(f / 256)) + S * 8,
        "route_dl": S * 12,
        "route_dw": T * d * b + S * 8 + d * E * 4,
        "transpose_wr": 2 * d * E * b,
    }
    return flops, bytes_


# ---------------------------------------------------------------------------
# the oracle as a CPU baseline (bounded samples)
# ---------------------------------------------------------------------------
def oracle_step(c, cfg, n_tok):
    import oracle
    x = c["x"][:n_tok]
    dy = c["dy"][:n_tok]
    idx, gates = oracle.route(x, c["w_r"], c["b_r"], cfg["k"])
    oracle.mlp_fwd(x, c["w1"], c["w2"], cfg["act"], idx, gates)
    oracle.mlp_bwd_full(x, c["w_r"], c["w1"], c["w2"], cfg["act"], idx, gates, dy)


# DRAM bytes per launch measured by ncu (dram__bytes_read.sum + dram__bytes_write.sum)
# for the workload's GEMM kernels, with the SHA-256 of the kernel source they were
# taken on; a value whose source has changed since is not reported.
TRAFFIC_TABLE = os.path.join(ROOT, "profiles", "dram_traffic_mixtral_bf16_swiglu.md")
KERNEL_SOURCE = os.path.join(ROOT, "sparse_mixture_experts_smoe_b200", "csrc", "gemm_tc.cu")


def measured_traffic(kernel: str, workload: str):
    import hashlib
    try:
        with open(KERNEL_SOURCE, "rb") as fh:
            digest = hashlib.sha256(fh.read()).hexdigest()
        with open(TRAFFIC_TABLE) as fh:
            rows = [ln for ln in fh if ln.startswith("|")]
    except OSError:
        return None
    for ln in rows:
        cells = [c.strip() for c in ln.strip().strip("|").split("|")]
        # | workload | kernel | read bytes | write bytes | source sha256 | ...
        if len(cells) >= 5 and cells[0] == workload and cells[1] == kernel and cells[4] == digest:
            try:
                return int(float(cells[2])) + int(float(cells[3]))
            except ValueError:
                return None
    return None


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as fh:
            for ln in fh:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_threads() -> int:
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    return int(os.environ.get("OMP_NUM_THREADS", cores))


def oracle_baseline(cfg, budget_s=12.0, seed=0):
    """tokens/s of the oracle's full fwd+bwd on a token sample sized to ~budget_s."""
    inp = make_mlp_inputs(cfg, seed=seed, device="cpu")
    c = {k: v for k, v in inp.items()}
    n = 1
    while True:  # grow the sample until it takes about budget_s
        t0 = time.perf_counter()
        oracle_step(c, cfg, n)
        dt = time.perf_counter() - t0
        if dt >= budget_s / 2 or n >= cfg["T"]:
            break
        n = min(cfg["T"], 2 * n)
    return {"value": n / dt, "unit": "tokens/s", "cores": oracle_threads(), "cpu": cpu_model(),
            "kind": "oracle",
            "sample": f"{n} of the {cfg['T']} tokens: routing, forward and full backward "
                      f"(dx, gate and router gradients, every expert weight gradient) in fp64 "
                      f"plain loops, {dt:.1f} s"}


def run_reference(args, world, rank):
    cfg = WORKLOADS[args.workload]
    if rank != 0:
        return
    inp = make_mlp_inputs(cfg, seed=0, device="cpu")
    # size each step to ~3 s of oracle work (fixed costs make per-token time non-linear)
    n = 1
    while True:
        t0 = time.perf_counter()
        oracle_step(inp, cfg, n)
        if time.perf_counter() - t0 >= 1.5 or n >= cfg["T"]:
            break
        n = min(cfg["T"], 2 * n)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(inp, cfg, n)
    el = time.perf_counter() - t0
    value = n * args.steps / el
    cores = oracle_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * el / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": args.workload, "T": cfg["T"], "d": cfg["d"],
                                        "f": cfg["f"], "E": cfg["E"], "k": cfg["k"],
                                        "act": cfg["act"], "tokens_per_step": n},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "cpu": cpu_model(),
                         "kind": "oracle",
                         "sample": f"{n} tokens per step of the {cfg['T']}-token workload"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our path
# ---------------------------------------------------------------------------
def moa_oracle_baseline(cfg, budget_s=12.0, seed=0):
    """tokens/s of the oracle's Mixture-of-Attention layer fwd+bwd on a bounded sample:
    the first n tokens of the first sequence (so their causal windows are complete)."""
    import oracle
    inp = make_moa_inputs(cfg, seed=seed, device="cpu")
    k, E, L, heads = cfg["k"], cfg["E"], cfg["L"], cfg["heads"]
    n = 8
    while True:
        t0 = time.perf_counter()
        x, dz = inp["x"][:n], inp["dz"][:n]
        idx, g = oracle.route(x, inp["w_r"], None, k)
        ss, off = oracle.sort(idx, E)
        tok, one = np.arange(n, dtype=np.int32), np.array([0, n], np.int32)
        q = oracle.pl_fwd(x, inp["wq"], ss, off, k, 0, 1)
        kk = oracle.pl_fwd(x, inp["wk"], tok, one, 1, 1, 1)
        v = oracle.pl_fwd(x, inp["wv"], tok, one, 1, 1, 1)
        o = oracle.moa_attn(q, kk, v, ss, k, L, heads)["o"]
        oracle.pl_fwd(o, inp["wo"], ss, off, 1, 1, 0, g.ravel(), k)
        bo = oracle.pl_bwd(dz, o, inp["wo"], ss, off, 1, 1, 0, g.ravel(), k, want_dg=True)
        ba = oracle.moa_attn(q, kk, v, ss, k, L, heads, dout=bo["dx"])
        oracle.pl_bwd(ba["dq"], x, inp["wq"], ss, off, k, 0, 1)
        oracle.pl_bwd(ba["dk"], x, inp["wk"], tok, one, 1, 1, 1)
        oracle.pl_bwd(ba["dv"], x, inp["wv"], tok, one, 1, 1, 1)
        oracle.route_bwd(x, inp["w_r"], idx, g, bo["dg"].reshape(n, k))
        dt = time.perf_counter() - t0
        if dt >= budget_s / 2 or n >= min(cfg["T"], L):
            break
        n = min(cfg["T"], L, 2 * n)
    return {"value": n / dt, "unit": "tokens/s", "cores": oracle_threads(), "cpu": cpu_model(),
            "kind": "oracle",
            "sample": f"the first {n} of the {cfg['T']} tokens (one sequence prefix): routing, sort, "
                      f"query/key/value/output projections, causal attention core and every "
                      f"backward in fp64 plain loops, {dt:.1f} s"}


def moa_kernel_work(cfg):
    """Algorithmic work per launch of the Mixture-of-Attention layer's kernels."""
    T, d, E, k, h = cfg["T"], cfg["d"], cfg["E"], cfg["k"], cfg["h"]
    af = moa_attn_flops(cfg)["fwd"]  # two width-128 products per (query, key) pair
    flops = {
        "moa.attn_fwd": af,           # S = Q K^T, O += P V
        "moa.attn_dq": 1.5 * af,      # S, dP = dO V^T, dQ += dS K
        "moa.attn_dkv": 2.0 * af,     # S^T, dP^T, dV += P^T dO, dK += dS^T Q
    }
    bytes_ = {"moa.attn_dsum": 2 * T * k * h * 2 + T * k * cfg["heads"] * 4}
    return flops, bytes_


def run_moa(args, world, rank, cfg):
    """The whole Mixture-of-Attention layer, forward and backward: route, sort, per-expert
    query projection (scatter->group, fan-out k), shared key and value projections
    (one-expert ParallelLinear), the causal attention core, per-expert output projection
    (group->scatter, gated k-way combine); backward through all of them, the router
    included.  The layer's dx is the router's term plus three projection parts (query,
    key, value); the step leaves the key and value parts as separate outputs (summing
    them would be two [T, d] additions)."""
    import sparse_mixture_experts_smoe_b200 as smoe
    dev = torch.device("cuda", torch.cuda.current_device())
    inp = make_moa_inputs(cfg, seed=rank, device=dev)
    T, d, E, k, h, L, heads = cfg["T"], cfg["d"], cfg["E"], cfg["k"], cfg["h"], cfg["L"], cfg["heads"]
    one = torch.tensor([0, T], dtype=torch.int32, device=dev)
    ident = torch.arange(T, dtype=torch.int32, device=dev)
    x, w_r = inp["x"], inp["w_r"]

    def step():
        idx, gates = smoe.smoe_route(x, w_r, None, k)
        ss, off = smoe.smoe_sort(idx, E)
        q = smoe.parallel_linear_fwd(x, inp["wq"], ss, off, k, 0, 1)
        kk = smoe.parallel_linear_fwd(x, inp["wk"], ident, one, 1, 1, 1)
        v = smoe.parallel_linear_fwd(x, inp["wv"], ident, one, 1, 1, 1)
        o, lse = smoe.smoe_moa_attn_fwd(q, kk, v, ss, k, L, heads)
        smoe.parallel_linear_fwd(o, inp["wo"], ss, off, 1, 1, 0, gates, k)
        do, _, dg = smoe.parallel_linear_bwd(inp["dz"], o, inp["wo"], ss, off, 1, 1, 0, gates, k,
                                             want_dgates=True)
        dq, dk, dv = smoe.smoe_moa_attn_bwd(q, kk, v, o, lse, do, ss, k, L, heads)
        dx, _, _ = smoe.parallel_linear_bwd(dq, x, inp["wq"], ss, off, k, 0, 1)
        smoe.parallel_linear_bwd(dk, x, inp["wk"], ident, one, 1, 1, 1)
        smoe.parallel_linear_bwd(dv, x, inp["wv"], ident, one, 1, 1, 1)
        smoe.smoe_route_bwd(x, w_r, idx, gates, dg.view(T, k), dx=dx)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0, smoe.lib().smoe_last_error()
    stream = torch.cuda.current_stream()
    barrier(world)
    clk = ClockSampler()
    clk.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clocks = clk.stop()
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world) / args.steps
    if smoe.smoe_check() != 0:
        raise SystemExit("device error word set during the MoA benchmark")
    # per-kernel times: a second pass with every launch bracketed by CUDA events
    smoe.smoe_profile_begin(64 * (args.steps + 1))
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    prof = smoe.smoe_profile_end()
    proj = 3 * (2.0 * T * k * d * h + 2 * 2.0 * T * d * h + 2.0 * T * k * h * d)  # fwd + 2x bwd
    attn = moa_attn_flops(cfg)["fwd_bwd"]
    flops = proj + attn
    tokens = T * world
    tflops = flops * world / (ms / 1e3) / 1e12
    peaks = load_peaks()
    fk, bk = moa_kernel_work(cfg)
    kernels = {}
    for name, (cnt, tot) in prof.items():
        per = tot / max(1, cnt) if tot > 0 else None
        ent = {"launches": cnt, "ms_total": round(tot, 4), "ms_per_launch": None if per is None else round(per, 4)}
        if name in fk and per:
            ent["tflops"] = round(fk[name] / (per / 1e3) / 1e12, 1)
        elif name in bk and per:
            ent["gbs"] = round(bk[name] / (per / 1e3) / 1e9, 1)
        kernels[name] = ent
    # the attention core's dominant kernel against the tensor roofline
    att = {n: kernels[n] for n in fk if n in kernels}
    dom = max(att.items(), key=lambda kv: kv[1]["ms_total"])[0] if att else None
    roofline = None
    if dom is not None and kernels[dom].get("tflops"):
        ach = kernels[dom]["tflops"]
        roofline = {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops_sustained"],
                    "unit": "TFLOP/s", "frac": round(ach / peaks["bf16_tflops_sustained"], 4),
                    "peak_kind": f"bf16 sustained, {peaks['source']}", "traffic": None}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = moa_oracle_baseline(cfg)
    line = {
        "metric": METRIC_MOA, "value": round(tokens / (ms / 1e3), 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "T": T, "d": d, "E": E, "k": k, "h": h, "L": L,
                   "heads": heads, "parallelism": f"replicas x{world}"},
        "tflops": round(tflops, 1),
        "tflops_split": {"projections": round(proj / (ms / 1e3) / 1e12, 1),
                         "attention_core_share_of_flops": round(attn / flops, 4)},
        "frac_of_bf16_peak": {"burst": round(tflops / peaks["bf16_tflops"], 4),
                              "sustained": round(tflops / peaks["bf16_tflops_sustained"], 4),
                              "peaks": peaks["source"]},
        "peak_mem_gb": round(torch.cuda.max_memory_allocated(dev) / 1e9, 2),
        "gpu_launches": sum(c for c, _ in prof.values()),
        "roofline": roofline,
        "kernels": kernels,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# granularity / sparsity sweeps of the SMoE MLP (one JSON line per configuration;
# not the benchmark's contract line)
# ---------------------------------------------------------------------------
SWEEP_T, SWEEP_D = 16384, 2048
SWEEPS = {
    # E*f and k*f constant: the same parameters and FLOPs per token, finer experts
    "granularity": [(8, 1, 4096), (16, 2, 2048), (32, 4, 1024), (64, 8, 512), (128, 16, 256)],
    # E and f fixed, more experts per token
    "sparsity": [(64, 1, 512), (64, 2, 512), (64, 4, 512), (64, 8, 512)],
    # the same kernels as one dense SwiGLU MLP (E = 1, k = 1: every gate is exactly 1)
    "dense": [(1, 1, 4096)],
}


# small-T forward (inference) on the Mixtral-shaped layer: with a handful of rows per
# expert the forward reads each used expert's weights once, so the bound is HBM
DECODE_T = [1, 8, 64, 512]


def run_decode(args, world, rank):
    import sparse_mixture_experts_smoe_b200 as smoe
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    base = WORKLOADS[DEFAULT_WORKLOAD]
    for T in DECODE_T:
        cfg = dict(base, T=T)
        d, f, E, k = cfg["d"], cfg["f"], cfg["E"], cfg["k"]
        torch.cuda.empty_cache()
        inp = make_mlp_inputs(cfg, seed=rank, device=dev, with_dy=False)
        st = smoe.SMoEMLPState(T, d, f, E, k, cfg["act"], torch.bfloat16, dev, with_grad=False)
        p = (inp["x"], inp["w_r"], inp["b_r"], inp["w1"], inp["w2"])
        for _ in range(args.warmup):
            smoe.smoe_mlp_fwd(st, *p)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            smoe.smoe_mlp_fwd(st, *p)
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
        ms = max_over_ranks(e0.elapsed_time(e1), world) / args.steps
        if smoe.smoe_check() != 0:
            raise SystemExit(f"device error word set in decode T={T}")
        rows = (st.expert_offsets[1:] - st.expert_offsets[:-1]).cpu()
        used = int((rows > 0).sum())
        mf = 2 * f if cfg["act"] == "swiglu" else f
        wbytes = used * (d * mf + f * d) * 2  # weights of the experts that received rows
        gbs = wbytes / (ms / 1e3) / 1e9
        line = {"sweep": "decode", "T": T, "d": d, "f": f, "E": E, "k": k, "act": cfg["act"],
                "dtype": "bf16", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_fwd": round(ms, 4), "tokens_per_s": round(T * world / (ms / 1e3), 1),
                "experts_used": used, "weight_bytes": wbytes,
                "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                             "traffic": None},
                "l2": "weights larger than L2, no flush"}
        if rank == 0:
            print(json.dumps(line), flush=True)
        # the same forward with e4m3 expert weights (codes + per-column fp32 scales):
        # half the weight bytes per token
        w1q, s1 = smoe.smoe_quantize_weights_fp8(inp["w1"])
        w2q, s2 = smoe.smoe_quantize_weights_fp8(inp["w2"])
        q = (inp["x"], inp["w_r"], inp["b_r"], w1q, s1, w2q, s2)
        for _ in range(args.warmup):
            smoe.smoe_mlp_fwd_fp8(st, *q)
        torch.cuda.synchronize()
        barrier(world)
        e0.record()
        for _ in range(args.steps):
            smoe.smoe_mlp_fwd_fp8(st, *q)
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
        ms8 = max_over_ranks(e0.elapsed_time(e1), world) / args.steps
        if smoe.smoe_check() != 0:
            raise SystemExit(f"device error word set in FP8 decode T={T}")
        wbytes8 = used * (d * mf + f * d) + used * (mf + d) * 4
        gbs8 = wbytes8 / (ms8 / 1e3) / 1e9
        line8 = dict(line, dtype="e4m3 weights, bf16 activations", ms_fwd=round(ms8, 4),
                     tokens_per_s=round(T * world / (ms8 / 1e3), 1), weight_bytes=wbytes8,
                     roofline={"bound": "hbm", "achieved": round(gbs8, 1), "peak": peaks["hbm_gbs"],
                               "unit": "GB/s", "frac": round(gbs8 / peaks["hbm_gbs"], 4), "traffic": None},
                     speedup_vs_bf16=round(ms / ms8, 3))
        if rank == 0:
            print(json.dumps(line8), flush=True)
        del st, inp, p, q, w1q, w2q


def run_library_bar(args, world, rank):
    """The six expert products of the Mixtral-shaped layer as dense batched products
    with equal slices (8 experts x 4096 rows, i.e. perfectly balanced routing and
    no gather), timed through torch.bmm (cuBLAS): a reference bar for the per-kernel
    times of the benchmark, not part of the path.  Outputs are bf16 (the library's
    weight gradients are fp32)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    cfg = WORKLOADS[DEFAULT_WORKLOAD]
    E, d, f = cfg["E"], cfg["d"], cfg["f"]
    M = cfg["T"] * cfg["k"] // E
    g = torch.Generator(device=dev)
    g.manual_seed(rank)

    def r(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.bfloat16)

    prods = {
        "fwd_up": lambda: (r(E, M, d), r(E, d, 2 * f)),
        "fwd_down": lambda: (r(E, M, f), r(E, f, d)),
        "bwd_dA": lambda: (r(E, M, d), r(E, f, d).transpose(1, 2)),
        "bwd_dx": lambda: (r(E, M, 2 * f), r(E, d, 2 * f).transpose(1, 2)),
        "bwd_dW2": lambda: (r(E, M, f).transpose(1, 2), r(E, M, d)),
        "bwd_dW1": lambda: (r(E, M, d).transpose(1, 2), r(E, M, 2 * f)),
    }
    for name, make in prods.items():
        torch.cuda.empty_cache()
        a, b = make()
        for _ in range(args.warmup):
            torch.bmm(a, b)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            torch.bmm(a, b)
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
        ms = max_over_ranks(e0.elapsed_time(e1), world) / args.steps
        fl = 2.0 * E * a.shape[1] * a.shape[2] * b.shape[2]
        if rank == 0:
            print(json.dumps({"sweep": "library", "product": name, "impl": "torch.bmm (cuBLAS), bf16 out",
                              "shape": [E, a.shape[1], a.shape[2], b.shape[2]], "steps": args.steps,
                              "ms": round(ms, 4), "tflops": round(fl / (ms / 1e3) / 1e12, 1)}), flush=True)
        del a, b


def run_sweep(args, world, rank):
    import sparse_mixture_experts_smoe_b200 as smoe
    if args.sweep == "decode":
        return run_decode(args, world, rank)
    if args.sweep == "library":
        return run_library_bar(args, world, rank)
    dev = torch.device("cuda", torch.cuda.current_device())
    peaks = load_peaks()
    names = list(SWEEPS) if args.sweep == "all" else [args.sweep]
    for name in names:
        for (E, k, f) in SWEEPS[name]:
            cfg = dict(kind="mlp", T=SWEEP_T, d=SWEEP_D, f=f, E=E, k=k, act="swiglu", dtype="bf16")
            torch.cuda.empty_cache()
            torch.cuda.reset_peak_memory_stats(dev)
            inp = make_mlp_inputs(cfg, seed=rank, device=dev)
            st = smoe.SMoEMLPState(SWEEP_T, SWEEP_D, f, E, k, "swiglu", torch.bfloat16, dev)
            p = (inp["x"], inp["w_r"], inp["b_r"], inp["w1"], inp["w2"])

            def fwd():
                smoe.smoe_mlp_fwd(st, *p)

            def fwd_bwd():
                smoe.smoe_mlp_fwd(st, *p)
                smoe.smoe_mlp_bwd(st, *p, inp["dy"])

            def timed(fn):
                for _ in range(args.warmup):
                    fn()
                torch.cuda.synchronize()
                barrier(world)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(args.steps):
                    fn()
                e1.record()
                torch.cuda.synchronize()
                barrier(world)
                return max_over_ranks(e0.elapsed_time(e1), world) / args.steps

            ms = timed(fwd_bwd)
            ms_f = timed(fwd)
            if smoe.smoe_check() != 0:
                raise SystemExit(f"device error word set in sweep {name} E={E} k={k}")
            fl = mlp_flops(cfg)
            tf = fl["fwd_bwd"] / (ms / 1e3) / 1e12
            line = {"sweep": name, "E": E, "k": k, "f": f, "T": SWEEP_T, "d": SWEEP_D, "act": "swiglu",
                    "dtype": "bf16", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                    "ms_fwd_bwd": round(ms, 4), "tokens_per_s": round(SWEEP_T * world / (ms / 1e3), 1),
                    "tflops": round(tf, 1), "frac_of_burst": round(tf / peaks["bf16_tflops"], 4),
                    "ms_fwd": round(ms_f, 4),
                    "tflops_fwd": round(fl["fwd"] / (ms_f / 1e3) / 1e12, 1),
                    "peak_mem_gb": round(torch.cuda.max_memory_allocated(dev) / 1e9, 2)}
            if rank == 0:
                print(json.dumps(line), flush=True)
            del st, inp, p


def run_ours(args, world, rank):
    import sparse_mixture_experts_smoe_b200 as smoe
    cfg = dict(WORKLOADS[args.workload])
    if args.tokens:
        cfg["T"] = args.tokens
    if cfg["kind"] == "moa":
        return run_moa(args, world, rank, cfg)
    if cfg["kind"] != "mlp":
        raise SystemExit("unknown workload kind")
    dev = torch.device("cuda", torch.cuda.current_device())
    dt = torch.bfloat16 if cfg["dtype"] == "bf16" else torch.float32
    inp = make_mlp_inputs(cfg, seed=rank, device=dev)
    st = smoe.SMoEMLPState(cfg["T"], cfg["d"], cfg["f"], cfg["E"], cfg["k"], cfg["act"], dt, dev)
    params = (inp["x"], inp["w_r"], inp["b_r"], inp["w1"], inp["w2"])
    stream = torch.cuda.current_stream()

    def step(x=None, dy=None):
        p = params if x is None else (x,) + params[1:]
        smoe.smoe_mlp_fwd(st, *p)
        smoe.smoe_mlp_bwd(st, *p, inp["dy"] if dy is None else dy)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0, smoe.lib().smoe_last_error()

    # ---- timed region: device events, max over ranks; clocks sampled meanwhile.
    # Nothing else is recorded on the stream in here (no per-launch events). ----
    clocks = ClockSampler()
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world) / args.steps
    assert smoe.smoe_check() == 0, smoe.lib().smoe_last_error()

    # ---- per-kernel times: the same K steps again, each launch of the library
    # bracketed by CUDA events on its stream (a separate, instrumented pass) ----
    smoe.smoe_profile_begin(64 * (args.steps + 1))
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    prof = smoe.smoe_profile_end()
    ms_instr = max_over_ranks(e0.elapsed_time(e1), world) / args.steps

    # ---- forward alone (reported beside the metric) ----
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        smoe.smoe_mlp_fwd(st, *params)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_fwd = max_over_ranks(e0.elapsed_time(e1), world) / args.steps

    # ---- end to end through the public API with host buffers ----
    # Every step copies its own inputs in from pinned host memory and reads its
    # result back, all inside the timed region.  The copies run on a second stream:
    # step i+1's inputs load into the spare buffer pair while step i computes, and
    # step i's y is read back while its backward runs (step i+1's forward waits
    # until that read is done before it overwrites y).
    x_h = inp["x"].cpu().pin_memory()
    dy_h = inp["dy"].cpu().pin_memory()
    y_hs = [torch.empty(st.y.shape, dtype=st.y.dtype).pin_memory() for _ in range(2)]
    bufs = [(torch.empty_like(inp["x"]), torch.empty_like(inp["dy"])) for _ in range(2)]
    copy = torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_free = [torch.cuda.Event() for _ in range(2)]
    ev_y, ev_yread = torch.cuda.Event(), torch.cuda.Event()

    def load(slot):
        with torch.cuda.stream(copy):
            bufs[slot][0].copy_(x_h, non_blocking=True)
            bufs[slot][1].copy_(dy_h, non_blocking=True)
            ev_in[slot].record(copy)

    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    copy.wait_event(e0)
    load(0)
    for i in range(args.steps):
        slot = i % 2
        if i + 1 < args.steps:
            if i >= 1:
                copy.wait_event(ev_free[1 - slot])  # step i-1 is done with that pair
            load(1 - slot)
        stream.wait_event(ev_in[slot])
        if i >= 1:
            stream.wait_event(ev_yread)  # step i-1's y has been read back
        xb, dyb = bufs[slot]
        pp = (xb,) + params[1:]
        smoe.smoe_mlp_fwd(st, *pp)
        ev_y.record(stream)
        with torch.cuda.stream(copy):
            copy.wait_event(ev_y)
            y_hs[slot].copy_(st.y, non_blocking=True)
            ev_yread.record(copy)
        smoe.smoe_mlp_bwd(st, *pp, dyb)
        ev_free[slot].record(stream)
    stream.wait_event(ev_yread)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1), world) / args.steps
    y_h = y_hs[0]
    h2d = x_h.numel() * x_h.element_size() + dy_h.numel() * dy_h.element_size()
    d2h = y_h.numel() * y_h.element_size()

    peaks = load_peaks()
    fl = mlp_flops(cfg)
    tokens = cfg["T"] * world
    value = tokens / (ms / 1e3)
    tflops = fl["fwd_bwd"] / (ms / 1e3) / 1e12
    flops_k, bytes_k = kernel_work(cfg)
    kernels = {}
    for name, (cnt, tot) in prof.items():
        per_launch_ms = tot / max(1, cnt) if tot > 0 else None
        ent = {"launches": cnt, "ms_total": round(tot, 4),
               "ms_per_launch": None if per_launch_ms is None else round(per_launch_ms, 4)}
        if name in flops_k and per_launch_ms:
            ent["tflops"] = round(flops_k[name] / (per_launch_ms / 1e3) / 1e12, 1)
        elif name in bytes_k and per_launch_ms:
            ent["gbs"] = round(bytes_k[name] / (per_launch_ms / 1e3) / 1e9, 1)
        kernels[name] = ent
    launches = sum(c for c, _ in prof.values())
    # dominant kernel: largest share of the timed region
    dom = max(prof.items(), key=lambda kv: kv[1][1])[0] if prof else None
    roofline = None
    if dom is not None:
        cnt, tot = prof[dom]
        per = tot / cnt / 1e3
        if dom in flops_k:
            ach = flops_k[dom] / per / 1e12
            roofline = {"kernel": dom, "bound": "tensor", "achieved": round(ach, 1),
                         "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                         "frac": round(ach / peaks["bf16_tflops_sustained"], 4),
                         "peak_kind": f"bf16 sustained, {peaks['source']}",
                         "frac_of_burst_peak": round(ach / peaks["bf16_tflops"], 4),
                         "traffic": None if args.tokens else measured_traffic(dom, args.workload)}
        else:
            ach = bytes_k.get(dom, 0) / per / 1e9
            roofline = {"kernel": dom, "bound": "hbm", "achieved": round(ach, 1),
                        "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": round(ach / peaks["hbm_gbs"], 4), "traffic": None}
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_baseline(cfg)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if dt == torch.bfloat16 else "f32",
        "data": "synthetic",
        "config": {"workload": args.workload + ("" if not args.tokens else f"-T{cfg['T']}"), "T": cfg["T"], "d": cfg["d"], "f": cfg["f"],
                   "E": cfg["E"], "k": cfg["k"], "act": cfg["act"], "parallelism": f"replicas x{world}",
                   "l2": "inputs larger than L2 (x 134 MB, weights 2.8 GB), no flush"},
        "tflops_fwd_bwd": round(tflops, 1),
        "frac_of_bf16_peak": {"burst": round(tflops / peaks["bf16_tflops"], 4),
                              "sustained": round(tflops / peaks["bf16_tflops_sustained"], 4),
                              "peaks": peaks["source"],
                              "nominal_dense": round(tflops / NOMINAL_DENSE_BF16_TFLOPS, 4)},
        "peak_mem_gb": round(torch.cuda.max_memory_allocated(dev) / 1e9, 2),
        "expert_rows": (st.expert_offsets[1:] - st.expert_offsets[:-1]).cpu().tolist(),
        "fwd": {"tokens_per_s": round(tokens / (ms_fwd / 1e3), 1), "ms_per_step": round(ms_fwd, 4),
                "tflops": round(fl["fwd"] / (ms_fwd / 1e3) / 1e12, 1)},
        "e2e": {"value": round(tokens / (ms_e2e / 1e3), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(ms_e2e, 4)},
        "gpu_launches": launches,
        "roofline": roofline,
        "kernels": kernels,
        "kernels_pass": {"what": "per-launch CUDA events over a second pass of the same K steps, "
                                 "after the clean timed region",
                         "ms_per_step": round(ms_instr, 4)},
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", choices=["granularity", "sparsity", "dense", "decode", "library", "all"],
                    default=None,
                    help="time the SMoE MLP over a set of (E, k, f) shapes instead of the benchmark line")
    ap.add_argument("--tokens", type=int, default=0,
                    help="override T (smaller cases for profiler captures; never a bench line)")
    args = ap.parse_args()
    world, rank, _ = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        elif args.sweep:
            run_sweep(args, world, rank)
        else:
            run_ours(args, world, rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
