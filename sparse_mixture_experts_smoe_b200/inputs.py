"""Seeded synthetic inputs for the SMoE MLP and ParallelLinear workloads.

This module holds no arithmetic of the method: it only draws random tensors with
the shapes and distributions of the five workloads (listed in ``WORKLOADS``) and
builds the router bias of the skewed workload.  The tests hand the same tensors
to the CUDA library and to the CPU oracle.

Recipe (every tensor has its own stream, so changing one shape never shifts
another):  ``torch.randn`` on the requested device from a ``torch.Generator``
seeded with ``seed * 1000 + stream_id``, in fp32, scaled by its standard
deviation, then rounded to the storage dtype (bf16 round-to-nearest-even).

  x  ~ N(0, 1)            [T, d]
  W_r ~ N(0, 1/d)         [d, E]           (router weight, stored in x's dtype)
  W1 ~ N(0, 1/d)          [E, d, m*f]      (m = 2 for SwiGLU: gate | up columns)
  W2 ~ N(0, 1/f)          [E, f, d]
  dY ~ N(0, 1)            [T, d]           (upstream gradient)
  dgates ~ N(0, 1)        [T, k] fp32      (router backward on its own)
  b_r                     [E] fp32, zero except the skewed workload (below)

Skewed workload: experts get ranks r = 1..E from a seeded permutation;
b_r[e] = -s * ln(r_e) for r_e <= E - n_empty and -1e4 otherwise, so exactly
``n_empty`` experts can never be selected (k < E - n_empty).

Mixture-of-Attention projections: x [T, d]; Wq [E, d, h] ~ N(0, 1/d);
Wo [E, h, d] ~ N(0, 1/h); shared Wk, Wv [1, d, h] ~ N(0, 1/d); per-slot attention output o [T*k, h] ~ N(0, 1) in
grouped order; upstream gradients dz [T, d] and dq [T*k, h] ~ N(0, 1).
Mixture-of-Attention core: the T tokens are sequences of L = 2048 tokens; queries
q [T*k, h] (grouped), shared keys and values k, v [T, h] and the upstream
gradient do [T*k, h] ~ N(0, 1); h = heads * 128 with heads = 4.
"""
from __future__ import annotations

import math

import torch

# The five workloads, with the sizes they are specified at.
WORKLOADS = {
    "tiny_fp32_gelu": dict(kind="mlp", T=256, d=128, f=256, E=8, k=2, dtype="f32", act="gelu"),
    "small_bf16_gelu": dict(kind="mlp", T=4096, d=1024, f=4096, E=8, k=2, dtype="bf16",
                            act="gelu"),
    "mixtral_bf16_swiglu": dict(kind="mlp", T=16384, d=4096, f=14336, E=8, k=2, dtype="bf16",
                                act="swiglu"),
    "finegrained_zipf_bf16_swiglu": dict(kind="mlp", T=16384, d=2048, f=512, E=64, k=8,
                                         dtype="bf16", act="swiglu", zipf_s=1.2, n_empty=4),
    "moa_bf16": dict(kind="moa", T=8192, d=2048, E=16, k=4, h=512, dtype="bf16", L=2048, heads=4),
}

_STREAM = {"x": 1, "w_r": 2, "w1": 3, "w2": 4, "dy": 5, "perm": 6, "wq": 7, "wo": 8, "o": 9,
           "dz": 10, "dq": 11, "dg": 12, "aq": 13, "ak": 14, "av": 15, "ado": 16, "wk": 17,
           "wv": 18}


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def _randn(shape, std, stream, seed, device, dtype):
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + _STREAM[stream])
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def zipf_bias(E: int, s: float, n_empty: int, seed: int) -> torch.Tensor:
    """Router bias giving Zipf-like expert popularity and ``n_empty`` dead experts."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed * 1000 + _STREAM["perm"])
    perm = torch.randperm(E, generator=g)
    rank = torch.empty(E, dtype=torch.int64)
    rank[perm] = torch.arange(1, E + 1)
    b = torch.empty(E, dtype=torch.float32)
    for e in range(E):
        r = int(rank[e])
        b[e] = -s * math.log(r) if r <= E - n_empty else -1.0e4
    return b


def make_mlp_inputs(cfg: dict, seed: int = 0, device="cpu", with_dy: bool = True) -> dict:
    T, d, f, E = cfg["T"], cfg["d"], cfg["f"], cfg["E"]
    dt = torch_dtype(cfg["dtype"])
    m = 2 if cfg["act"] == "swiglu" else 1
    out = {
        "x": _randn((T, d), 1.0, "x", seed, device, dt),
        "w_r": _randn((d, E), 1.0 / math.sqrt(d), "w_r", seed, device, dt),
        "w1": _randn((E, d, m * f), 1.0 / math.sqrt(d), "w1", seed, device, dt),
        "w2": _randn((E, f, d), 1.0 / math.sqrt(f), "w2", seed, device, dt),
    }
    if "zipf_s" in cfg:
        out["b_r"] = zipf_bias(E, cfg["zipf_s"], cfg["n_empty"], seed).to(device)
    else:
        out["b_r"] = None
    if with_dy:
        out["dy"] = _randn((T, d), 1.0, "dy", seed, device, dt)
    return out


def make_router_inputs(cfg: dict, seed: int = 0, device="cpu") -> dict:
    """Router-only inputs of a workload: x, W_r and b_r as in ``make_mlp_inputs``
    (same streams, so the same values), plus upstream gate gradients
    dgates ~ N(0, 1) [T, k] in fp32 for the router backward on its own."""
    T, d, E, k = cfg["T"], cfg["d"], cfg["E"], cfg["k"]
    dt = torch_dtype(cfg["dtype"])
    out = {
        "x": _randn((T, d), 1.0, "x", seed, device, dt),
        "w_r": _randn((d, E), 1.0 / math.sqrt(d), "w_r", seed, device, dt),
        "b_r": (zipf_bias(E, cfg["zipf_s"], cfg["n_empty"], seed).to(device)
                if "zipf_s" in cfg else None),
        "dgates": _randn((T, k), 1.0, "dg", seed, device, torch.float32),
    }
    return out


def make_moa_inputs(cfg: dict, seed: int = 0, device="cpu") -> dict:
    T, d, E, k, h = cfg["T"], cfg["d"], cfg["E"], cfg["k"], cfg["h"]
    dt = torch_dtype(cfg["dtype"])
    return {
        "x": _randn((T, d), 1.0, "x", seed, device, dt),
        "w_r": _randn((d, E), 1.0 / math.sqrt(d), "w_r", seed, device, dt),
        "b_r": None,
        "wq": _randn((E, d, h), 1.0 / math.sqrt(d), "wq", seed, device, dt),
        "wo": _randn((E, h, d), 1.0 / math.sqrt(h), "wo", seed, device, dt),
        # shared key and value projections of the attention core (one "expert" each)
        "wk": _randn((1, d, h), 1.0 / math.sqrt(d), "wk", seed, device, dt),
        "wv": _randn((1, d, h), 1.0 / math.sqrt(d), "wv", seed, device, dt),
        "o": _randn((T * k, h), 1.0, "o", seed, device, dt),
        "dz": _randn((T, d), 1.0, "dz", seed, device, dt),
        "dq": _randn((T * k, h), 1.0, "dq", seed, device, dt),
    }


def make_moa_attn_inputs(cfg: dict, seed: int = 0, device="cpu") -> dict:
    """Inputs of the Mixture-of-Attention core at a workload's sizes: x and W_r (the
    router, as in ``make_moa_inputs``), per-slot queries q [T*k, h] in grouped order,
    shared keys and values k, v [T, h] and the upstream gradient do [T*k, h], all
    N(0, 1) in bf16 (h = heads * 128)."""
    T, d, E, k, h = cfg["T"], cfg["d"], cfg["E"], cfg["k"], cfg["h"]
    dt = torch_dtype(cfg["dtype"])
    return {
        "x": _randn((T, d), 1.0, "x", seed, device, dt),
        "w_r": _randn((d, E), 1.0 / math.sqrt(d), "w_r", seed, device, dt),
        "q": _randn((T * k, h), 1.0, "aq", seed, device, dt),
        "k": _randn((T, h), 1.0, "ak", seed, device, dt),
        "v": _randn((T, h), 1.0, "av", seed, device, dt),
        "do": _randn((T * k, h), 1.0, "ado", seed, device, dt),
    }


def moa_attn_flops(cfg: dict) -> dict:
    """Algorithmic FLOPs of the causal attention core: per head and query row, two
    products of width 128 over its window (scores and P V), the window of query
    token t being t - (sequence start) + 1 keys; backward = 2.5 x forward (dS K,
    dP = dO V^T, dV, dK plus the score recomputation)."""
    T, k, heads, L = cfg["T"], cfg["k"], cfg["heads"], cfg["L"]
    keys = 0
    for s0 in range(0, T, L):
        n = min(L, T - s0)
        keys += n * (n + 1) // 2  # sum of window lengths over the sequence's tokens
    fwd = 2.0 * 2 * 128 * keys * k * heads
    return {"fwd": fwd, "bwd": 2.5 * fwd, "fwd_bwd": 3.5 * fwd}


def mlp_flops(cfg: dict) -> dict:
    """Algorithmic FLOPs of the expert GEMMs (router excluded): fwd = 2*T*k*d*f*m'
    with m' = 2 (GELU: W1 and W2) or 3 (SwiGLU: gate, up, down); bwd = 2 * fwd."""
    m = 3 if cfg["act"] == "swiglu" else 2
    fwd = 2.0 * cfg["T"] * cfg["k"] * cfg["d"] * cfg["f"] * m
    return {"fwd": fwd, "bwd": 2 * fwd, "fwd_bwd": 3 * fwd}
