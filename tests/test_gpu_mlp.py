"""GPU parity of the SMoE MLP (smoe_mlp_fwd / smoe_mlp_bwd) and of the
Mixture-of-Attention projections against the CPU oracle.

* reduced shapes (several tiles, ragged tails, an empty expert) and the tiny
  fp32 workload: every output and gradient, element by element;
* the full-size workloads, in the launch configuration the benchmark times:
  sampled token rows of y, dx and the gate gradients, sampled columns/rows of the
  expert weight gradients, and, for the router weight gradient, properties that
  hold at any size.
Routing indices, sorted slots and offsets are always compared bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_smoe_b200 as smoe
from sparse_mixture_experts_smoe_b200.inputs import WORKLOADS, make_mlp_inputs, make_moa_inputs

from ._util import assert_close, np64

pytestmark = pytest.mark.gpu


def _run_mlp(cfg, inp):
    dt = inp["x"].dtype
    st = smoe.SMoEMLPState(cfg["T"], cfg["d"], cfg["f"], cfg["E"], cfg["k"], cfg["act"], dt, "cuda")
    args = (inp["x"], inp["w_r"], inp["b_r"], inp["w1"], inp["w2"])
    smoe.smoe_mlp_fwd(st, *args)
    smoe.smoe_mlp_bwd(st, *args, inp["dy"])
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    return st


def _cpu(inp):
    return {k: (None if v is None else v.cpu()) for k, v in inp.items()}


def _check_routing(cfg, st, c):
    ref_idx, ref_g = oracle.route(c["x"], c["w_r"], c["b_r"], cfg["k"])
    np.testing.assert_array_equal(st.topk_idx.cpu().numpy(), ref_idx)
    ref_ss, ref_off = oracle.sort(ref_idx, cfg["E"])
    np.testing.assert_array_equal(st.sorted_slot.cpu().numpy(), ref_ss)
    np.testing.assert_array_equal(st.expert_offsets.cpu().numpy(), ref_off)
    assert_close("gates", st.gates, ref_g, torch.float32)
    return ref_idx, ref_g, ref_ss


def _check_full(cfg, inp):
    """Every output element against the oracle (small shapes)."""
    dt = inp["x"].dtype
    st = _run_mlp(cfg, inp)
    c = _cpu(inp)
    idx, gates, ss = _check_routing(cfg, st, c)
    fwd = oracle.mlp_fwd(c["x"], c["w1"], c["w2"], cfg["act"], idx, gates, want_ha=True)
    assert_close("y", st.y, fwd["y"], dt)
    # saved H and A are grouped: grouped row i holds slot ss[i]
    assert_close("h", st.h, fwd["h"][ss], dt)
    assert_close("a", st.a, fwd["a"][ss], dt)
    bwd = oracle.mlp_bwd_full(c["x"], c["w_r"], c["w1"], c["w2"], cfg["act"], idx, gates, c["dy"])
    assert_close("dx", st.dx, bwd["dx"], dt)
    assert_close("dgates", st.dgates, bwd["dg"], dt)
    assert_close("dw1", st.dw1, bwd["dw1"], dt)
    assert_close("dw2", st.dw2, bwd["dw2"], dt)
    assert_close("dw_r", st.dw_r, bwd["dw_r"], dt)
    assert_close("db_r", st.db_r, bwd["db_r"], dt)
    counts = np.diff(st.expert_offsets.cpu().numpy())
    for e in np.nonzero(counts == 0)[0]:
        assert np.all(st.dw1[e].cpu().numpy() == 0) and np.all(st.dw2[e].cpu().numpy() == 0)
    return st


def test_tiny_fp32_gelu_full():
    cfg = WORKLOADS["tiny_fp32_gelu"]
    _check_full(cfg, make_mlp_inputs(cfg, device="cuda"))


REDUCED = {
    "gelu_bf16": dict(kind="mlp", T=300, d=264, f=392, E=6, k=2, dtype="bf16", act="gelu"),
    "swiglu_bf16": dict(kind="mlp", T=300, d=264, f=200, E=6, k=2, dtype="bf16", act="swiglu"),
    # whole 64-column slabs and K = 4096 for the up projection: its MN-major weights
    # load through the slab view (SwiGLU's last gate run crosses into the up half)
    "swiglu_bf16_slabs": dict(kind="mlp", T=300, d=4096, f=192, E=6, k=2, dtype="bf16", act="swiglu"),
    "gelu_bf16_slabs": dict(kind="mlp", T=300, d=4096, f=448, E=5, k=2, dtype="bf16", act="gelu"),
    "swiglu_bf16_zipf": dict(kind="mlp", T=257, d=136, f=128, E=16, k=4, dtype="bf16",
                             act="swiglu", zipf_s=1.2, n_empty=3),
    "swiglu_f32": dict(kind="mlp", T=200, d=72, f=136, E=4, k=2, dtype="f32", act="swiglu"),
    "single_expert_bf16": dict(kind="mlp", T=130, d=128, f=136, E=1, k=1, dtype="bf16",
                               act="gelu"),
    # shapes the granularity and sparsity sweeps reach: 128 experts with k = 16, top-1
    "e128_k16_bf16": dict(kind="mlp", T=96, d=136, f=72, E=128, k=16, dtype="bf16",
                          act="swiglu"),
    "top1_bf16": dict(kind="mlp", T=200, d=136, f=136, E=32, k=1, dtype="bf16", act="swiglu"),
    # decode-sized batches: a few rows per tile, most experts empty
    "decode_t1_bf16": dict(kind="mlp", T=1, d=264, f=392, E=8, k=2, dtype="bf16", act="swiglu"),
    "decode_t5_bf16": dict(kind="mlp", T=5, d=264, f=392, E=8, k=2, dtype="bf16", act="swiglu"),
    # few enough tiles that the down projection splits its K (4 splits, ragged last K-block)
    "decode_t2_splitk_bf16": dict(kind="mlp", T=2, d=264, f=1000, E=8, k=2, dtype="bf16",
                                  act="swiglu"),
}

# K = 4096 over expert slices of 2200 rows (every token routed to both experts): under
# GEMM policy 1 the up projection and dA' gather with 4 warps and dW1 and dW2 run on
# the pair dW kernel (ragged pair tiles, a ragged N tile); policy 0 as a baseline
LONG_K = dict(kind="mlp", T=2200, d=4096, f=200, E=2, k=2, dtype="bf16", act="swiglu")


@pytest.mark.parametrize("policy", [0, 1])
def test_mlp_long_k_policies(policy):
    smoe.smoe_set_gemm_policy(policy)
    try:
        _check_full(LONG_K, make_mlp_inputs(LONG_K, seed=1, device="cuda"))
    finally:
        smoe.smoe_set_gemm_policy(0)


@pytest.mark.parametrize("name", list(REDUCED))
def test_mlp_reduced_full(name):
    cfg = REDUCED[name]
    st = _check_full(cfg, make_mlp_inputs(cfg, seed=1, device="cuda"))
    if cfg["E"] == 1:      # closed form: gates are exactly 1 and the router gradient vanishes
        assert torch.all(st.gates == 1.0)
        assert torch.all(st.dw_r == 0.0)


@pytest.mark.parametrize("T", [1, 8])
def test_decode_forward_mixtral_shape(T):
    """The small-T forward the decode sweep times (Mixtral-shaped layer, T tokens):
    routing bit for bit, every element of y, H and A."""
    cfg = dict(WORKLOADS["mixtral_bf16_swiglu"], T=T)
    inp = make_mlp_inputs(cfg, seed=3, device="cuda", with_dy=False)
    st = smoe.SMoEMLPState(T, cfg["d"], cfg["f"], cfg["E"], cfg["k"], cfg["act"], torch.bfloat16,
                           "cuda", with_grad=False)
    smoe.smoe_mlp_fwd(st, inp["x"], inp["w_r"], inp["b_r"], inp["w1"], inp["w2"])
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    c = _cpu(inp)
    idx, gates, ss = _check_routing(cfg, st, c)
    fwd = oracle.mlp_fwd(c["x"], c["w1"], c["w2"], cfg["act"], idx, gates, want_ha=True)
    assert_close("y", st.y, fwd["y"], torch.bfloat16)
    assert_close("h", st.h, fwd["h"][ss], torch.bfloat16)
    assert_close("a", st.a, fwd["a"][ss], torch.bfloat16)


def test_mlp_is_deterministic():
    cfg = REDUCED["swiglu_bf16_zipf"]
    inp = make_mlp_inputs(cfg, seed=2, device="cuda")
    a = _run_mlp(cfg, inp)
    b = _run_mlp(cfg, inp)
    for n in ("y", "h", "a", "dx", "dw1", "dw2", "dw_r", "db_r", "dgates"):
        assert torch.equal(getattr(a, n), getattr(b, n)), n


def _sampled(cfg, n_tok=6, n_col=3, seed=0):
    """Full-size run; oracle on sampled tokens / weight-gradient columns."""
    inp = make_mlp_inputs(cfg, device="cuda")
    dt = inp["x"].dtype
    st = _run_mlp(cfg, inp)
    c = _cpu(inp)
    idx, gates, ss = _check_routing(cfg, st, c)
    T, f, d = cfg["T"], cfg["f"], cfg["d"]
    mf = 2 * f if cfg["act"] == "swiglu" else f
    rng = np.random.default_rng(seed)
    toks = np.unique(np.concatenate([[0, T - 1], rng.choice(T, n_tok, replace=False)])).astype(np.int32)
    fwd = oracle.mlp_fwd(c["x"], c["w1"], c["w2"], cfg["act"], idx, gates, tokens=toks, want_ha=True)
    assert_close("y[tokens]", st.y[torch.from_numpy(toks).long().cuda()], fwd["y"], dt)
    inv = np.empty_like(ss)
    inv[ss] = np.arange(ss.size)
    slots = (toks[:, None] * cfg["k"] + np.arange(cfg["k"])[None, :]).ravel()
    rows = torch.from_numpy(inv[slots]).long().cuda()
    assert_close("h[slots]", st.h[rows], fwd["h"], dt)
    assert_close("a[slots]", st.a[rows], fwd["a"], dt)
    bwd = oracle.mlp_bwd_tokens(c["x"], c["w_r"], c["w1"], c["w2"], cfg["act"], idx, gates, c["dy"],
                                tokens=toks)
    tl = torch.from_numpy(toks).long().cuda()
    assert_close("dx[tokens]", st.dx[tl], bwd["dx"], dt)
    assert_close("dgates[tokens]", st.dgates[tl], bwd["dg"], dt)
    cols1 = np.unique(np.concatenate([[0, mf - 1], rng.choice(mf, n_col, replace=False)]))
    rows2 = np.unique(np.concatenate([[0, f - 1], rng.choice(f, n_col, replace=False)]))
    dw1c, dw2r = oracle.mlp_dw_sampled(c["x"], c["w1"], c["w2"], cfg["act"], idx, gates, c["dy"],
                                       cols1, rows2)
    assert_close("dw1[:, :, cols]", st.dw1[:, :, torch.from_numpy(cols1).long().cuda()], dw1c, dt)
    assert_close("dw2[:, rows, :]", st.dw2[:, torch.from_numpy(rows2).long().cuda(), :], dw2r, dt)
    # router gradient: dl sums to zero over each token's experts (the gates sum to one),
    # so the columns of dW_r and db_r sum to zero over experts
    dw_r, db_r = np64(st.dw_r), np64(st.db_r)
    assert abs(db_r.sum()) <= 1e-3 * np.abs(db_r).sum() + 1e-6
    assert np.max(np.abs(dw_r.sum(1))) <= 1e-3 * np.max(np.abs(dw_r).sum(1)) + 1e-6
    counts = np.diff(st.expert_offsets.cpu().numpy())
    for e in np.nonzero(counts == 0)[0]:
        assert torch.all(st.dw1[e] == 0) and torch.all(st.dw2[e] == 0)
    return st


@pytest.mark.parametrize("name", ["small_bf16_gelu", "mixtral_bf16_swiglu",
                                  "finegrained_zipf_bf16_swiglu"])
def test_mlp_full_size_sampled(name):
    st = _sampled(WORKLOADS[name])
    del st
    torch.cuda.empty_cache()


def test_moa_projections_full_size_sampled():
    """Mixture-of-Attention projections: Wq scatter->group (fan-out k), Wo
    group->scatter with the gated k-way combine, forward and backward."""
    cfg = WORKLOADS["moa_bf16"]
    inp = make_moa_inputs(cfg, device="cuda")
    T, k, E, d, h = cfg["T"], cfg["k"], cfg["E"], cfg["d"], cfg["h"]
    idx, gates = smoe.smoe_route(inp["x"], inp["w_r"], None, k)
    ss, off = smoe.smoe_sort(idx, E)
    q = smoe.parallel_linear_fwd(inp["x"], inp["wq"], ss, off, k, 0, 1)
    z = smoe.parallel_linear_fwd(inp["o"], inp["wo"], ss, off, 1, 1, 0, gates, k)
    dx, dwq, _ = smoe.parallel_linear_bwd(inp["dq"], inp["x"], inp["wq"], ss, off, k, 0, 1)
    do, dwo, dgt = smoe.parallel_linear_bwd(inp["dz"], inp["o"], inp["wo"], ss, off, 1, 1, 0, gates,
                                            k, want_dgates=True)
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    c = _cpu(inp)
    ref_idx, ref_g = oracle.route(c["x"], c["w_r"], None, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    ref_ss, ref_off = oracle.sort(ref_idx, E)
    np.testing.assert_array_equal(ss.cpu().numpy(), ref_ss)
    g64 = ref_g.ravel()
    rng = np.random.default_rng(1)
    S = T * k
    rows_i = np.unique(np.concatenate([[0, S - 1], rng.choice(S, 8, replace=False)])).astype(np.int32)
    toks = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 8, replace=False)])).astype(np.int32)
    slots = np.unique(np.concatenate([[0, S - 1], rng.choice(S, 16, replace=False)])).astype(np.int32)
    cols_q = np.array([0, 5, h - 1], np.int32)
    cols_o = np.array([0, 77, d - 1], np.int32)
    L = lambda a: torch.from_numpy(a).long().cuda()  # noqa: E731
    bf = torch.bfloat16
    assert_close("q", q[L(rows_i)], oracle.pl_fwd(c["x"], c["wq"], ref_ss, ref_off, k, 0, 1,
                                                  out_rows=rows_i), bf)
    assert_close("z", z[L(toks)], oracle.pl_fwd(c["o"], c["wo"], ref_ss, ref_off, 1, 1, 0, g64, k,
                                                out_rows=toks), bf)
    rq = oracle.pl_bwd(c["dq"], c["x"], c["wq"], ref_ss, ref_off, k, 0, 1, dx_rows=toks,
                       dw_cols=cols_q)
    assert_close("dx", dx[L(toks)], rq["dx"], bf)
    assert_close("dWq", dwq[:, :, L(cols_q)], rq["dw"], bf)
    ro = oracle.pl_bwd(c["dz"], c["o"], c["wo"], ref_ss, ref_off, 1, 1, 0, g64, k, want_dg=True,
                       dx_rows=rows_i, dw_cols=cols_o, dg_slots=slots)
    assert_close("do", do[L(rows_i)], ro["dx"], bf)
    assert_close("dWo", dwo[:, :, L(cols_o)], ro["dw"], bf)
    assert_close("dgates", dgt[L(slots)], ro["dg"], bf)


def test_library_allocates_nothing():
    """With the caller's buffers in place, a forward and backward step allocates no
    device memory at all (the library only uses the caller's workspace)."""
    cfg = REDUCED["swiglu_bf16"]
    inp = make_mlp_inputs(cfg, seed=2, device="cuda")
    st = smoe.SMoEMLPState(cfg["T"], cfg["d"], cfg["f"], cfg["E"], cfg["k"], cfg["act"],
                           torch.bfloat16, "cuda")
    p = (inp["x"], inp["w_r"], inp["b_r"], inp["w1"], inp["w2"])
    smoe.smoe_mlp_fwd(st, *p)
    smoe.smoe_mlp_bwd(st, *p, inp["dy"])
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats()
    before = torch.cuda.memory_allocated()
    for _ in range(2):
        smoe.smoe_mlp_fwd(st, *p)
        smoe.smoe_mlp_bwd(st, *p, inp["dy"])
    torch.cuda.synchronize()
    assert torch.cuda.max_memory_allocated() == before
    assert smoe.smoe_check() == 0
