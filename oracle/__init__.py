"""ctypes wrapper of the fp64 CPU oracle in ``smoe_oracle.cpp``.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` import this package.
The CUDA library never links, loads or calls it, and it imports nothing from the
CUDA package.

Every function takes CPU tensors or numpy arrays holding the stored values
(float32, or bfloat16 as a torch tensor) and returns fp64 numpy arrays, except the
integer routing outputs.  The definitions follow the ScatterMoE pages as listed
in the header of ``smoe_oracle.cpp`` (readings R1-R8 there).

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
against independent mathematics (brute force, closed forms, library routines,
finite differences, invariants).
"""
from __future__ import annotations

import ctypes
import fcntl
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "smoe_oracle.cpp")
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None

ACT = {"gelu": 0, "swiglu": 1, "none": 2}


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc (plain -O3, OpenMP, no FP contraction)."""
    lock_path = os.path.join(_HERE, ".build.lock")
    with open(lock_path, "w") as lock:
        fcntl.flock(lock, fcntl.LOCK_EX)
        stale = (not os.path.exists(_SO)) or os.path.getmtime(_SO) < os.path.getmtime(_SRC)
        if force or stale:
            tmp = _SO + ".tmp"
            cmd = ["g++", "-O3", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC",
                   "-o", tmp, _SRC]
            subprocess.run(cmd, check=True)
            os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = ctypes.CDLL(_SO)
    return _lib


def _stored(a):
    """(contiguous numpy array of the stored bits, dtype code 0=f32 / 1=bf16 / 2=f64)."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().cpu().contiguous()
            if a.dtype == torch.bfloat16:
                return a.view(torch.int16).numpy(), 1
            if a.dtype == torch.float32:
                return a.numpy(), 0
            if a.dtype == torch.float64:
                return a.numpy(), 2
            if a.dtype == torch.int32:
                return a.numpy(), -1
            raise TypeError(f"unsupported tensor dtype {a.dtype}")
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    if a.dtype == np.float32:
        return a, 0
    if a.dtype == np.float64:
        return a, 2
    if a.dtype == np.int32:
        return a, -1
    raise TypeError(f"unsupported array dtype {a.dtype}")


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _i32(a):
    if a is None:
        return None
    arr, code = _stored(a) if not isinstance(a, np.ndarray) else (np.ascontiguousarray(a), -1)
    arr = np.ascontiguousarray(arr, dtype=np.int32)
    return arr


def _f64(a):
    """fp64 values (bf16 tensors are converted by value, not by bits)."""
    if a is None:
        return None
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return np.ascontiguousarray(a.detach().cpu().double().numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(a, dtype=np.float64)


def _f32(a):
    if a is None:
        return None
    arr, code = _stored(a)
    if code == 1:
        raise TypeError("expected fp32 values")
    return np.ascontiguousarray(arr, dtype=np.float32)


# --------------------------------------------------------------------------
# routing and sort (R1-R3)
# --------------------------------------------------------------------------
def router_logits_f32(x, w_r, b_r=None):
    """fp32 logits in the CUDA route kernel's documented accumulation order."""
    lib = _load()
    xs, dt = _stored(x)
    ws, dtw = _stored(w_r)
    assert dt == dtw and dt in (0, 1)
    T, d = xs.shape
    E = ws.shape[1]
    b = _f32(b_r)
    out = np.empty((T, E), np.float32)
    lib.oracle_router_logits_f32(_p(xs), _p(ws), ctypes.c_int(dt), _p(b), T, d, E, _p(out))
    return out


def router_logits_f64(x, w_r, b_r=None):
    lib = _load()
    xs, dt = _stored(x)
    ws, _ = _stored(w_r)
    T, d = xs.shape
    E = ws.shape[1]
    b = _f32(b_r)
    out = np.empty((T, E), np.float64)
    lib.oracle_router_logits_f64(_p(xs), _p(ws), ctypes.c_int(dt), _p(b), T, d, E, _p(out))
    return out


def topk_gates(logits_f32, k):
    lib = _load()
    lg = np.ascontiguousarray(logits_f32, dtype=np.float32)
    T, E = lg.shape
    idx = np.empty((T, k), np.int32)
    gates = np.empty((T, k), np.float64)
    lib.oracle_topk_gates(_p(lg), T, E, k, _p(idx), _p(gates))
    return idx, gates


def route(x, w_r, b_r, k):
    """(topk_idx int32 [T,k], gates fp64 [T,k]) -- R1 with the R2 decision precision."""
    return topk_gates(router_logits_f32(x, w_r, b_r), k)


def sort(topk_idx, E):
    """(sorted_slot int32 [T*k], expert_offsets int32 [E+1]) -- R3."""
    lib = _load()
    idx = _i32(topk_idx)
    T, k = idx.shape
    ss = np.empty(T * k, np.int32)
    off = np.empty(E + 1, np.int32)
    lib.oracle_sort(_p(idx), T, k, E, _p(ss), _p(off))
    return ss, off


def route_bwd(x, w_r, topk_idx, gates, dgates):
    """Router backward alone (R5): {"dl": [T,k], "dx": [T,d] (the router's share of
    dx), "dw_r": [d,E], "db_r": [E]}, all fp64, for gate gradients ``dgates``."""
    lib = _load()
    xs, dt = _stored(x)
    ws, dtw = _stored(w_r)
    assert dt == dtw and dt in (0, 1, 2)
    T, d = xs.shape
    E = ws.shape[1]
    idx = _i32(topk_idx)
    k = idx.shape[1]
    g = _f64(gates)
    dg = _f64(dgates)
    assert g.shape == (T, k) and dg.shape == (T, k)
    out = {"dl": np.empty((T, k)), "dx": np.empty((T, d)), "dw_r": np.empty((d, E)),
           "db_r": np.empty(E)}
    lib.oracle_route_bwd(_p(xs), _p(ws), dt, T, d, E, k, _p(idx), _p(g), _p(dg), _p(out["dl"]),
                         _p(out["dx"]), _p(out["dw_r"]), _p(out["db_r"]))
    return out


def moa_attn(q, k, v, sorted_slot, kslots, L, heads, dout=None, q_rows=None, kv_tokens=None,
             want_dkv=True):
    """Mixture-of-Attention core (R7): {"o", "lse"} for grouped rows ``q_rows`` (all if
    None); with ``dout`` also "dq" for those rows and, when ``want_dkv``, "dk", "dv"
    for tokens ``kv_tokens`` (all if None).  All fp64."""
    lib = _load()
    qs, dt = _stored(q)
    ks, dtk = _stored(k)
    vs, dtv = _stored(v)
    assert dt == dtk == dtv
    ds = None
    if dout is not None:
        ds, dtd = _stored(dout)
        assert dtd == dt
    S, W = qs.shape
    T = ks.shape[0]
    dh = W // heads
    ss = _i32(sorted_slot)
    assert ss.size == S == T * kslots
    rows = None if q_rows is None else _i32(np.asarray(q_rows, np.int32))
    nq = S if rows is None else rows.size
    toks = None if kv_tokens is None else _i32(np.asarray(kv_tokens, np.int32))
    nkv = 0 if (dout is None or not want_dkv) else (T if toks is None else toks.size)
    out = {"o": np.empty((nq, W)), "lse": np.empty((nq, heads))}
    if dout is not None:
        out["dq"] = np.empty((nq, W))
        if want_dkv:
            out["dk"] = np.empty((nkv, W))
            out["dv"] = np.empty((nkv, W))
    lib.oracle_moa_attn(_p(qs), _p(ks), _p(vs), _p(ds), dt, _p(ss), T, kslots, L, heads, dh,
                        _p(rows), nq, _p(toks), nkv, _p(out["o"]), _p(out["lse"]),
                        _p(out.get("dq")), _p(out.get("dk")), _p(out.get("dv")))
    return out


def e4m3_round(v):
    """Values rounded to the nearest e4m3 value (ties to even, saturating at 448)."""
    lib = _load()
    a = np.ascontiguousarray(v, dtype=np.float64).ravel()
    out = np.empty_like(a)
    lib.oracle_e4m3_round(_p(a), a.size, _p(out))
    return out.reshape(np.shape(v))


def e4m3_decode(codes):
    lib = _load()
    b = np.ascontiguousarray(codes, dtype=np.uint8).ravel()
    out = np.empty(b.size)
    lib.oracle_e4m3_decode(_p(b), b.size, _p(out))
    return out.reshape(np.shape(codes))


def quantize_weights_fp8(w):
    """W [E, K, N] -> (codes uint8 [E, N, K] (K-major), scales fp32 [E, N])."""
    lib = _load()
    ws, dt = _stored(w)
    E, K, N = ws.shape
    codes = np.empty((E, N, K), np.uint8)
    scales = np.empty((E, N), np.float32)
    lib.oracle_quantize_weights_fp8(_p(ws), dt, E, K, N, _p(codes), _p(scales))
    return codes, scales


def quantize_rows_fp8(x):
    """x [rows, cols] -> (codes uint8 [rows, cols], scales fp32 [rows])."""
    lib = _load()
    xs, dt = _stored(x)
    rows, cols = xs.shape
    codes = np.empty((rows, cols), np.uint8)
    scales = np.empty(rows, np.float32)
    lib.oracle_quantize_rows_fp8(_p(xs), dt, rows, cols, _p(codes), _p(scales))
    return codes, scales


def mlp_fwd_fp8(x, w1q, s1, w2q, s2, act_name, topk_idx, gates, tokens=None, want_a=False):
    """FP8 forward (R8) with weights quantised by ``quantize_weights_fp8``:
    {"y": [n_tok, d], "a": [n_tok*k, f] (bf16-rounded A, slot order) if want_a}."""
    lib = _load()
    xs, dtx = _stored(x)
    T, d = xs.shape
    E, mf, d2 = w1q.shape
    assert d2 == d
    f = w2q.shape[2]
    idx = _i32(topk_idx)
    k = idx.shape[1]
    g = _f64(gates)
    tok = np.arange(T, dtype=np.int32) if tokens is None else _i32(tokens)
    n = tok.size
    y = np.empty((n, d))
    a = np.empty((n * k, f)) if want_a else None
    lib.oracle_mlp_fwd_fp8(_p(xs), dtx, _p(np.ascontiguousarray(w1q)), _p(np.ascontiguousarray(s1)),
                           _p(np.ascontiguousarray(w2q)), _p(np.ascontiguousarray(s2)), d, f, E, k,
                           ACT[act_name], _p(idx), _p(g), _p(tok), n, _p(y), _p(a))
    out = {"y": y}
    if want_a:
        out["a"] = a
    return out


def act(kind, z):
    """(value, derivative) of gelu(tanh) (kind 'gelu') or silu (kind 'silu')."""
    lib = _load()
    zz = np.ascontiguousarray(z, dtype=np.float64).ravel()
    v = np.empty_like(zz)
    g = np.empty_like(zz)
    lib.oracle_act(0 if kind == "gelu" else 1, _p(zz), zz.size, _p(v), _p(g))
    return v, g


# --------------------------------------------------------------------------
# SMoE MLP (R4, R5)
# --------------------------------------------------------------------------
def _mlp_dims(x, w1, w2, act_name):
    xs, dtx = _stored(x)
    w1s, dtw = _stored(w1)
    w2s, dtw2 = _stored(w2)
    assert dtx == dtw == dtw2, "x, W1 and W2 must share one dtype"
    T, d = xs.shape
    E, f, d2 = w2s.shape
    assert d2 == d and w1s.shape[0] == E and w1s.shape[1] == d
    mf = 2 * f if act_name == "swiglu" else f
    assert w1s.shape[2] == mf, (w1s.shape, mf)
    return xs, dtx, w1s, w2s, dtw, T, d, f, E, mf


def mlp_fwd(x, w1, w2, act_name, topk_idx, gates, tokens=None, want_ha=False):
    lib = _load()
    xs, dtx, w1s, w2s, dtw, T, d, f, E, mf = _mlp_dims(x, w1, w2, act_name)
    idx = _i32(topk_idx)
    k = idx.shape[1]
    g = _f64(gates)
    tok = np.arange(T, dtype=np.int32) if tokens is None else _i32(tokens)
    n = tok.size
    y = np.empty((n, d), np.float64)
    h = np.empty((n * k, mf), np.float64) if want_ha else None
    a = np.empty((n * k, f), np.float64) if want_ha else None
    lib.oracle_mlp_fwd(_p(xs), dtx, _p(w1s), _p(w2s), dtw, d, f, E, k, ACT[act_name], _p(idx),
                       _p(g), _p(tok), n, _p(y), _p(h), _p(a))
    return {"y": y, "h": h, "a": a}


def mlp_bwd_tokens(x, w_r, w1, w2, act_name, topk_idx, gates, dy, tokens=None):
    lib = _load()
    xs, dtx, w1s, w2s, dtw, T, d, f, E, mf = _mlp_dims(x, w1, w2, act_name)
    wrs, dtr = _stored(w_r)
    assert dtr == dtx
    idx = _i32(topk_idx)
    k = idx.shape[1]
    g = _f64(gates)
    dyv = _f64(dy)
    tok = np.arange(T, dtype=np.int32) if tokens is None else _i32(tokens)
    n = tok.size
    dx = np.empty((n, d), np.float64)
    dg = np.empty((n, k), np.float64)
    dl = np.empty((n, k), np.float64)
    lib.oracle_mlp_bwd_tokens(_p(xs), dtx, _p(wrs), _p(w1s), _p(w2s), dtw, d, f, E, k,
                              ACT[act_name], _p(idx), _p(g), _p(dyv), _p(tok), n, _p(dx), _p(dg),
                              _p(dl))
    return {"dx": dx, "dg": dg, "dl": dl}


def mlp_bwd_full(x, w_r, w1, w2, act_name, topk_idx, gates, dy):
    lib = _load()
    xs, dtx, w1s, w2s, dtw, T, d, f, E, mf = _mlp_dims(x, w1, w2, act_name)
    wrs, dtr = _stored(w_r)
    assert dtr == dtx
    idx = _i32(topk_idx)
    k = idx.shape[1]
    g = _f64(gates)
    dyv = _f64(dy)
    out = {
        "dx": np.empty((T, d)), "dg": np.empty((T, k)), "dw1": np.empty((E, d, mf)),
        "dw2": np.empty((E, f, d)), "dw_r": np.empty((d, E)), "db_r": np.empty(E),
    }
    lib.oracle_mlp_bwd_full(_p(xs), dtx, _p(wrs), _p(w1s), _p(w2s), dtw, T, d, f, E, k,
                            ACT[act_name], _p(idx), _p(g), _p(dyv), _p(out["dx"]), _p(out["dg"]),
                            _p(out["dw1"]), _p(out["dw2"]), _p(out["dw_r"]), _p(out["db_r"]))
    return out


def mlp_dw_sampled(x, w1, w2, act_name, topk_idx, gates, dy, cols1, rows2):
    """Columns ``cols1`` of every dW1[e] -> [E, d, len(cols1)]; rows ``rows2`` of
    every dW2[e] -> [E, len(rows2), d]."""
    lib = _load()
    xs, dtx, w1s, w2s, dtw, T, d, f, E, mf = _mlp_dims(x, w1, w2, act_name)
    idx = _i32(topk_idx)
    k = idx.shape[1]
    g = _f64(gates)
    dyv = _f64(dy)
    c1 = _i32(np.asarray(cols1, np.int32))
    r2 = _i32(np.asarray(rows2, np.int32))
    dw1 = np.empty((E, d, c1.size))
    dw2 = np.empty((E, r2.size, d))
    lib.oracle_mlp_dw_sampled(_p(xs), dtx, _p(w1s), _p(w2s), dtw, T, d, f, E, k, ACT[act_name],
                              _p(idx), _p(g), _p(dyv), _p(c1), c1.size, _p(r2), r2.size, _p(dw1),
                              _p(dw2))
    return dw1, dw2


# --------------------------------------------------------------------------
# ParallelLinear (R6)
# --------------------------------------------------------------------------
def pl_fwd(x, w, sorted_slot, offsets, fan_out, grouped_in, grouped_out, gates=None,
           combine_k=0, out_rows=None):
    lib = _load()
    xs, dtx = _stored(x)
    ws, dtw = _stored(w)
    E, K, N = ws.shape
    ss = _i32(sorted_slot)
    off = _i32(offsets)
    S = ss.size
    g = _f64(gates).ravel() if gates is not None else None
    if out_rows is None:
        n_out = (S // combine_k) if combine_k > 0 else S
        rows = None
    else:
        rows = _i32(np.asarray(out_rows, np.int32))
        n_out = rows.size
    y = np.empty((n_out, N))
    lib.oracle_pl_fwd(_p(xs), dtx, _p(ws), dtw, K, N, E, _p(ss), _p(off), S, fan_out,
                      int(grouped_in), int(grouped_out), _p(g), combine_k, _p(rows), n_out, _p(y))
    return y


def pl_bwd(dy, x, w, sorted_slot, offsets, fan_out, grouped_in, grouped_out, gates=None,
           combine_k=0, want_dx=True, want_dw=True, want_dg=False, dx_rows=None, dw_cols=None,
           dg_slots=None):
    lib = _load()
    dys, dtd = _stored(dy)
    xs, dtx = _stored(x)
    ws, dtw = _stored(w)
    E, K, N = ws.shape
    x_rows = xs.shape[0]
    ss = _i32(sorted_slot)
    off = _i32(offsets)
    S = ss.size
    g = _f64(gates).ravel() if gates is not None else None
    rows = None if dx_rows is None else _i32(np.asarray(dx_rows, np.int32))
    n_dx = x_rows if rows is None else rows.size
    cols = None if dw_cols is None else _i32(np.asarray(dw_cols, np.int32))
    n_dw = N if cols is None else cols.size
    slots = None if dg_slots is None else _i32(np.asarray(dg_slots, np.int32))
    n_dg = S if slots is None else slots.size
    dx = np.empty((n_dx, K)) if want_dx else None
    dw = np.empty((E, K, n_dw)) if want_dw else None
    dgv = np.empty(n_dg) if want_dg else None
    lib.oracle_pl_bwd(_p(dys), dtd, _p(xs), dtx, _p(ws), dtw, x_rows, K, N, E, _p(ss), _p(off), S,
                      fan_out, int(grouped_in), int(grouped_out), _p(g), combine_k, _p(rows), n_dx,
                      _p(dx), _p(cols), n_dw, _p(dw), _p(slots), n_dg, _p(dgv))
    return {"dx": dx, "dw": dw, "dg": dgv}
