"""Pins of the CPU oracle against mathematics that does not come from the oracle.

Each test checks one oracle function against something independent of its code:
values derived by hand from the documented router order (tests/golden), brute
force over all k-subsets, exact integer arithmetic, library routines (numpy's
stable argsort, torch's gelu/silu and matmul), a dense evaluate-every-expert
reference, the E=1/k=1 closed form, permutation equivariance, linearity and fp64
central finite differences.  A plausible mistake in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a wrong reduction order) fails at least
one of them.  All tests are CPU-only and small.
"""
import itertools
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------
# router logits
# --------------------------------------------------------------------------
def test_router_logits_documented_order_golden():
    spec = json.load(open(os.path.join(GOLDEN, "router_order_cases.json")))
    d, E = spec["d"], spec["E"]
    for case in spec["cases"]:
        x = np.zeros((1, d), np.float32)
        w = np.ones((d, E), np.float32)
        for i, v in case["x"].items():
            x[0, int(i)] = v
        for i, v in case["w"].items():
            w[int(i), 0] = v
        b = None if case["b"] is None else np.array([case["b"]], np.float32)
        got = oracle.router_logits_f32(x, w, b)[0, 0]
        assert got == np.float32(case["expected"]), (case["name"], float(got), case["expected"])


def test_router_logits_exact_integer_indexing():
    # small integers: every fp32 operation is exact, so the logits equal the
    # integer dot products whatever the order -- pins the x / W_r / b indexing
    r = _rng(1)
    T, d, E = 7, 40, 5
    x = r.integers(-3, 4, (T, d)).astype(np.float32)
    w = r.integers(-3, 4, (d, E)).astype(np.float32)
    b = r.integers(-5, 6, E).astype(np.float32)
    want = x.astype(np.int64) @ w.astype(np.int64) + b.astype(np.int64)
    got = oracle.router_logits_f32(x, w, b)
    np.testing.assert_array_equal(got, want.astype(np.float32))
    np.testing.assert_array_equal(oracle.router_logits_f64(x, w, b), want.astype(np.float64))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_router_logits_within_fp32_error_bound(dtype):
    # forward error bound of an fp32 dot product of length d: gamma_d * sum|x w|
    g = torch.Generator().manual_seed(3)
    T, d, E = 33, 256, 8
    x = torch.randn(T, d, generator=g).to(dtype)
    w = (torch.randn(d, E, generator=g) / 16).to(dtype)
    l32 = oracle.router_logits_f32(x, w).astype(np.float64)
    l64 = oracle.router_logits_f64(x, w)
    xd, wd = x.double().numpy(), w.double().numpy()
    np.testing.assert_allclose(l64, xd @ wd, rtol=0, atol=1e-12)
    u = 2.0 ** -24
    gamma = d * u / (1 - d * u)
    bound = gamma * (np.abs(xd) @ np.abs(wd))
    assert np.all(np.abs(l32 - l64) <= bound + 1e-30)


# --------------------------------------------------------------------------
# top-k and gates
# --------------------------------------------------------------------------
def test_topk_matches_brute_force_subsets():
    r = _rng(2)
    T, E, k = 60, 7, 3
    logits = r.standard_normal((T, E)).astype(np.float32)
    idx, gates = oracle.topk_gates(logits, k)
    for t in range(T):
        best = max(itertools.combinations(range(E), k),
                   key=lambda s: sum(float(logits[t, e]) for e in s))
        assert set(idx[t]) == set(best)
        vals = [logits[t, e] for e in idx[t]]
        assert all(vals[j] >= vals[j + 1] for j in range(k - 1))
        sel = logits[t, idx[t]].astype(np.float64)
        ex = np.exp(sel - sel.max())
        np.testing.assert_allclose(gates[t], ex / ex.sum(), rtol=1e-15, atol=0)


def test_topk_gates_equal_softmax_topk_renormalised():
    r = _rng(4)
    T, E, k = 100, 16, 4
    logits = (3 * r.standard_normal((T, E))).astype(np.float32)
    idx, gates = oracle.topk_gates(logits, k)
    p = torch.softmax(torch.from_numpy(logits).double(), dim=-1)
    top = torch.topk(p, k, dim=-1)
    ren = top.values / top.values.sum(-1, keepdim=True)
    assert np.array_equal(np.sort(idx, 1), np.sort(top.indices.numpy(), 1))
    np.testing.assert_allclose(gates, ren.numpy(), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(gates.sum(1), 1.0, rtol=0, atol=1e-15)


def test_topk_ties_go_to_lower_expert():
    logits = np.array([[1.0, 2.0, 2.0, 0.5, 2.0],
                       [0.0, 0.0, 0.0, 0.0, 0.0]], np.float32)
    idx, gates = oracle.topk_gates(logits, 3)
    assert idx.tolist() == [[1, 2, 4], [0, 1, 2]]
    np.testing.assert_allclose(gates, 1.0 / 3.0, rtol=1e-15)


# --------------------------------------------------------------------------
# sort
# --------------------------------------------------------------------------
@pytest.mark.parametrize("T,k,E", [(1, 1, 1), (50, 2, 8), (300, 8, 64), (17, 4, 5)])
def test_sort_matches_numpy_stable_argsort(T, k, E):
    r = _rng(T * 31 + E)
    idx = r.integers(0, E, (T, k)).astype(np.int32)
    if E > 3:
        idx[idx == 3] = 2  # an empty expert
    ss, off = oracle.sort(idx, E)
    np.testing.assert_array_equal(ss, np.argsort(idx.ravel(), kind="stable"))
    counts = np.bincount(idx.ravel(), minlength=E)
    np.testing.assert_array_equal(off, np.concatenate([[0], np.cumsum(counts)]))
    # invariants: each slot once, experts non-decreasing, slots ascending per expert
    assert sorted(ss.tolist()) == list(range(T * k))
    e_sorted = idx.ravel()[ss]
    assert np.all(np.diff(e_sorted) >= 0)
    for e in range(E):
        seg = ss[off[e]:off[e + 1]]
        assert np.all(np.diff(seg) > 0)


# --------------------------------------------------------------------------
# activations
# --------------------------------------------------------------------------
def test_activations_against_torch_and_closed_forms():
    z = np.concatenate([np.linspace(-8, 8, 161), [0.0, 30.0, -30.0, 1e-3, -1e-3]])
    zt = torch.from_numpy(z).requires_grad_(True)
    for kind, fn in [("gelu", lambda t: F.gelu(t, approximate="tanh")), ("silu", F.silu)]:
        v, g = oracle.act(kind, z)
        ref = fn(zt)
        (gr,) = torch.autograd.grad(ref.sum(), zt)
        np.testing.assert_allclose(v, ref.detach().numpy(), rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(g, gr.numpy(), rtol=1e-12, atol=1e-14)
        assert v[161] == 0.0                      # act(0) = 0
        assert abs(v[162] - 30.0) < 1e-10         # ~ identity for large z
        assert abs(v[163]) < 1e-10                # ~ 0 for very negative z
    # derivative by central difference
    h = 1e-6
    for kind in ("gelu", "silu"):
        vp, _ = oracle.act(kind, z + h)
        vm, _ = oracle.act(kind, z - h)
        _, g = oracle.act(kind, z)
        np.testing.assert_allclose((vp - vm) / (2 * h), g, rtol=1e-7, atol=1e-8)


# --------------------------------------------------------------------------
# SMoE MLP forward
# --------------------------------------------------------------------------
def _tiny_mlp(seed, T, d, f, E, k, act, dtype=torch.float64):
    g = torch.Generator().manual_seed(seed)
    m = 2 if act == "swiglu" else 1
    x = torch.randn(T, d, generator=g, dtype=torch.float64).to(dtype)
    w_r = (torch.randn(d, E, generator=g, dtype=torch.float64) / d ** 0.5).to(dtype)
    w1 = (torch.randn(E, d, m * f, generator=g, dtype=torch.float64) / d ** 0.5).to(dtype)
    w2 = (torch.randn(E, f, d, generator=g, dtype=torch.float64) / f ** 0.5).to(dtype)
    dy = torch.randn(T, d, generator=g, dtype=torch.float64)
    return x, w_r, w1, w2, dy


def _dense_masked_reference(x, w1, w2, act, idx, gates):
    """Evaluate every expert on every token, then keep the top-k with their gates."""
    X, W1, W2 = x.double(), w1.double(), w2.double()
    T, E, f = X.shape[0], W1.shape[0], W2.shape[1]
    outs = []
    for e in range(E):
        H = X @ W1[e]
        A = F.gelu(H, approximate="tanh") if act == "gelu" else F.silu(H[:, :f]) * H[:, f:]
        outs.append(A @ W2[e])
    Y = torch.stack(outs, 1)                          # [T, E, d]
    mask = torch.zeros(T, E, dtype=torch.float64)
    mask.scatter_(1, torch.from_numpy(idx).long(), torch.from_numpy(gates))
    return (mask[:, :, None] * Y).sum(1).numpy()


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_mlp_fwd_equals_dense_masked_reference(act, dtype):
    x, w_r, w1, w2, _ = _tiny_mlp(5, 24, 16, 12, 6, 2, act, dtype)
    idx, gates = oracle.route(x, w_r, None, 2)
    out = oracle.mlp_fwd(x, w1, w2, act, idx, gates, want_ha=True)
    ref = _dense_masked_reference(x, w1, w2, act, idx, gates)
    np.testing.assert_allclose(out["y"], ref, rtol=1e-12, atol=1e-12)
    # the saved pre-activation of slot (t, j) is x_t W1[e]
    X, W1 = x.double(), w1.double()
    for p in [0, 7, 47]:
        t, j = divmod(p, 2)
        np.testing.assert_allclose(out["h"][p], (X[t] @ W1[idx[t, j]]).numpy(), rtol=1e-12,
                                   atol=1e-12)


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_mlp_single_expert_is_dense_mlp(act):
    x, w_r, w1, w2, dy = _tiny_mlp(6, 10, 8, 6, 1, 1, act, torch.float32)
    idx, gates = oracle.route(x, w_r, None, 1)
    assert np.all(idx == 0) and np.all(gates == 1.0)
    X, W1, W2 = x.double(), w1.double()[0], w2.double()[0]
    f = W2.shape[0]
    H = X @ W1
    A = F.gelu(H, approximate="tanh") if act == "gelu" else F.silu(H[:, :f]) * H[:, f:]
    np.testing.assert_allclose(oracle.mlp_fwd(x, w1, w2, act, idx, gates)["y"], (A @ W2).numpy(),
                               rtol=1e-12, atol=1e-12)
    full = oracle.mlp_bwd_full(x, w_r, w1, w2, act, idx, gates, dy)
    assert np.all(full["dw_r"] == 0.0) and np.all(full["db_r"] == 0.0)


def test_mlp_linear_in_w2():
    x, w_r, w1, w2, _ = _tiny_mlp(7, 12, 8, 6, 4, 2, "swiglu", torch.float32)
    idx, gates = oracle.route(x, w_r, None, 2)
    y1 = oracle.mlp_fwd(x, w1, w2, "swiglu", idx, gates)["y"]
    y3 = oracle.mlp_fwd(x, w1, w2 * 4, "swiglu", idx, gates)["y"]
    np.testing.assert_allclose(y3, 4 * y1, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_mlp_token_permutation_equivariance(act):
    x, w_r, w1, w2, dy = _tiny_mlp(8, 20, 8, 6, 4, 2, act, torch.float32)
    idx, gates = oracle.route(x, w_r, None, 2)
    perm = np.random.default_rng(0).permutation(20)
    a = oracle.mlp_bwd_full(x, w_r, w1, w2, act, idx, gates, dy)
    b = oracle.mlp_bwd_full(x[perm], w_r, w1, w2, act, idx[perm], gates[perm], dy[perm])
    ya = oracle.mlp_fwd(x, w1, w2, act, idx, gates)["y"]
    yb = oracle.mlp_fwd(x[perm], w1, w2, act, idx[perm], gates[perm])["y"]
    np.testing.assert_allclose(yb, ya[perm], rtol=1e-14, atol=1e-14)
    for key in ("dx", "dg"):
        np.testing.assert_allclose(b[key], a[key][perm], rtol=1e-12, atol=1e-13)
    for key in ("dw1", "dw2", "dw_r", "db_r"):
        np.testing.assert_allclose(b[key], a[key], rtol=1e-11, atol=1e-12)


# --------------------------------------------------------------------------
# SMoE MLP backward: fp64 central finite differences through the whole layer
# --------------------------------------------------------------------------
def _route_with_margin(x, w_r, b, k, min_margin):
    l = (x @ w_r + b).numpy()
    order = np.argsort(-l, axis=1, kind="stable")
    srt = np.take_along_axis(l, order, 1)
    assert np.all(srt[:, k - 1] - srt[:, k] > min_margin), "pick another seed"
    return order[:, :k].astype(np.int32)


def _loss(x, w_r, b, w1, w2, act, idx, dy):
    """L = <y, dY> with y from the oracle and gates = softmax of the selected logits."""
    l = x @ w_r + b
    sel = torch.gather(l, 1, torch.from_numpy(idx).long())
    gates = torch.softmax(sel, dim=1)
    y = oracle.mlp_fwd(x, w1, w2, act, idx, gates.numpy())["y"]
    return float((y * dy.numpy()).sum())


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_mlp_backward_finite_differences(act):
    T, d, f, E, k = 5, 8, 6, 4, 2
    for seed in range(20, 60):
        x, w_r, w1, w2, dy = _tiny_mlp(seed, T, d, f, E, k, act)
        b = torch.randn(E, generator=torch.Generator().manual_seed(seed), dtype=torch.float64)
        l = (x @ w_r + b).numpy()
        s = np.sort(l, 1)[:, ::-1]
        if np.all(s[:, k - 1] - s[:, k] > 1e-2):
            break
    idx = _route_with_margin(x, w_r, b, k, 1e-2)
    sel = torch.gather(x @ w_r + b, 1, torch.from_numpy(idx).long())
    gates = torch.softmax(sel, 1).numpy()
    an = oracle.mlp_bwd_full(x, w_r, w1, w2, act, idx, gates, dy)
    # db is not an oracle input in fp32 form here: the loss closes over b directly
    h = 1e-6
    params = {"x": x, "w_r": w_r, "b": b, "w1": w1, "w2": w2}
    key_of = {"x": "dx", "w_r": "dw_r", "b": "db_r", "w1": "dw1", "w2": "dw2"}
    for name, tensor in params.items():
        fd = np.zeros(tensor.numel())
        flat = tensor.view(-1)
        for q in range(tensor.numel()):
            old = float(flat[q])
            flat[q] = old + h
            lp = _loss(params["x"], params["w_r"], params["b"], params["w1"], params["w2"], act, idx, dy)
            flat[q] = old - h
            lm = _loss(params["x"], params["w_r"], params["b"], params["w1"], params["w2"], act, idx, dy)
            flat[q] = old
            fd[q] = (lp - lm) / (2 * h)
        ref = an[key_of[name]].ravel()
        err = np.max(np.abs(fd - ref)) / np.max(np.abs(ref))
        assert err < 1e-6, (name, err)
    # gate gradient: dL/dg[t,j] = <dY_t, o_{t,j}>
    fd = np.zeros_like(gates)
    for t in range(T):
        for j in range(k):
            gp, gm = gates.copy(), gates.copy()
            gp[t, j] += h
            gm[t, j] -= h
            yp = oracle.mlp_fwd(x, w1, w2, act, idx, gp)["y"]
            ym = oracle.mlp_fwd(x, w1, w2, act, idx, gm)["y"]
            fd[t, j] = ((yp - ym) * dy.numpy()).sum() / (2 * h)
    assert np.max(np.abs(fd - an["dg"])) / np.max(np.abs(an["dg"])) < 1e-6


def test_route_bwd_finite_differences():
    """The router backward alone: L = sum_{t,j} dg[t,j] * g[t,j](x W_r + b), the gates
    the softmax over each token's (fixed) selected logits.  Central differences of L
    in x, W_r and b against the oracle's dx, dW_r and db; a repeated expert index
    across tokens and an expert nobody picks are both present."""
    T, d, E, k = 7, 9, 5, 3
    g = torch.Generator().manual_seed(41)
    x = torch.randn(T, d, generator=g, dtype=torch.float64)
    w_r = torch.randn(d, E, generator=g, dtype=torch.float64)
    b = torch.randn(E, generator=g, dtype=torch.float64)
    b[E - 1] = -50.0  # never selected: its dW_r column and db entry are exactly zero
    dg = torch.randn(T, k, generator=g, dtype=torch.float64).numpy()
    idx = _route_with_margin(x, w_r, b, k, 1e-3)
    gates = torch.softmax(torch.gather(x @ w_r + b, 1, torch.from_numpy(idx).long()), 1).numpy()
    an = oracle.route_bwd(x, w_r, idx, gates, dg)

    def loss(xv, wv, bv):
        sel = torch.gather(xv @ wv + bv, 1, torch.from_numpy(idx).long())
        return float((torch.softmax(sel, 1).numpy() * dg).sum())

    h = 1e-6
    params = {"x": x, "w_r": w_r, "b": b}
    key_of = {"x": "dx", "w_r": "dw_r", "b": "db_r"}
    for name, tensor in params.items():
        flat = tensor.view(-1)
        fd = np.zeros(tensor.numel())
        for q in range(tensor.numel()):
            old = float(flat[q])
            flat[q] = old + h
            lp = loss(x, w_r, b)
            flat[q] = old - h
            lm = loss(x, w_r, b)
            flat[q] = old
            fd[q] = (lp - lm) / (2 * h)
        ref = an[key_of[name]].ravel()
        assert np.max(np.abs(fd - ref)) / np.max(np.abs(ref)) < 1e-6, name
    assert np.all(an["dw_r"][:, E - 1] == 0.0) and an["db_r"][E - 1] == 0.0
    # the logit gradients of a token sum to zero (its gates sum to one)
    assert np.max(np.abs(an["dl"].sum(1))) < 1e-12


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_route_bwd_agrees_with_the_mlp_backward(dtype):
    """Fed the MLP backward's own gate gradients, the standalone router backward
    gives the MLP's dW_r and db, and its dx is the MLP's dx minus the expert path."""
    x, w_r, w1, w2, dy = _tiny_mlp(12, 40, 24, 16, 6, 2, "swiglu", dtype)
    idx, gates = oracle.route(x, w_r, None, 2)
    full = oracle.mlp_bwd_full(x, w_r, w1, w2, "swiglu", idx, gates, dy)
    r = oracle.route_bwd(x, w_r, idx, gates, full["dg"])
    np.testing.assert_allclose(r["dw_r"], full["dw_r"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(r["db_r"], full["db_r"], rtol=1e-12, atol=1e-13)
    # the expert path alone: the MLP backward of a router whose weights are zero
    # (dx_expert does not depend on W_r once idx and gates are fixed)
    no_router = oracle.mlp_bwd_full(x, torch.zeros_like(w_r), w1, w2, "swiglu", idx, gates, dy)
    np.testing.assert_allclose(r["dx"] + no_router["dx"], full["dx"], rtol=1e-11, atol=1e-12)


def test_mlp_backward_token_subset_and_sampled_dw_agree_with_full():
    x, w_r, w1, w2, dy = _tiny_mlp(9, 30, 16, 12, 5, 2, "swiglu", torch.float32)
    idx, gates = oracle.route(x, w_r, None, 2)
    full = oracle.mlp_bwd_full(x, w_r, w1, w2, "swiglu", idx, gates, dy)
    toks = np.array([3, 0, 29, 11], np.int32)
    sub = oracle.mlp_bwd_tokens(x, w_r, w1, w2, "swiglu", idx, gates, dy, tokens=toks)
    np.testing.assert_allclose(sub["dx"], full["dx"][toks], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(sub["dg"], full["dg"][toks], rtol=1e-13, atol=1e-14)
    cols1 = [0, 5, 11, 12, 23]
    rows2 = [0, 7, 11]
    dw1c, dw2r = oracle.mlp_dw_sampled(x, w1, w2, "swiglu", idx, gates, dy, cols1, rows2)
    np.testing.assert_allclose(dw1c, full["dw1"][:, :, cols1], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dw2r, full["dw2"][:, rows2, :], rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# ParallelLinear
# --------------------------------------------------------------------------
def _pl_problem(seed, T, K, N, E, k, dtype=torch.float64):
    g = torch.Generator().manual_seed(seed)
    idx = torch.randint(0, E, (T, k), generator=g).int().numpy()
    ss, off = oracle.sort(idx, E)
    w = (torch.randn(E, K, N, generator=g, dtype=torch.float64) / K ** 0.5).to(dtype)
    gates = torch.rand(T * k, generator=g, dtype=torch.float64).numpy()
    return idx, ss, off, w, gates, g


MODES = [  # (grouped_in, grouped_out, fan_out, combine)
    (0, 1, "k", False),   # scatter -> group, token-shaped input read k times
    (1, 0, 1, True),      # group -> scatter with k-way combine
    (1, 0, 1, False),     # group -> scatter, slot-shaped output
    (1, 1, 1, False),     # group -> group
    (0, 0, 1, False),     # scatter -> scatter, slot-shaped input
    (0, 0, "k", True),    # scatter -> scatter with combine, token-shaped input
]


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("gated", [False, True])
def test_pl_fwd_equals_dense_every_expert(mode, gated):
    gi, go, fo, comb = mode
    T, K, N, E, k = 9, 6, 5, 4, 2
    idx, ss, off, w, gates, g = _pl_problem(11, T, K, N, E, k)
    fan_out = k if fo == "k" else 1
    x_rows = T * k if (gi or fan_out == 1) else T
    x = torch.randn(x_rows, K, generator=g, dtype=torch.float64)
    gv = gates if gated else None
    y = oracle.pl_fwd(x, w, ss, off, fan_out, gi, go, gv, k if comb else 0)
    # dense: every grouped row times every expert, then keep its own expert
    e_of_row = np.repeat(np.arange(E), np.diff(off))
    xin = x[np.arange(T * k)] if gi else x[torch.from_numpy(ss // fan_out).long()]
    Yall = torch.einsum("sk,ekn->sen", xin, w.double())
    v = Yall[torch.arange(T * k), torch.from_numpy(e_of_row).long()].numpy()
    if gated:
        v = v * gates[ss][:, None]
    if comb:
        ref = np.zeros((T, N))
        for i in range(T * k):
            ref[ss[i] // k] += v[i]
    else:
        ref = np.zeros((T * k, N))
        for i in range(T * k):
            ref[i if go else ss[i]] = v[i]
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-14)
    # subsets of output rows agree with the full result
    rows = [0, y.shape[0] - 1, 3]
    np.testing.assert_allclose(oracle.pl_fwd(x, w, ss, off, fan_out, gi, go, gv, k if comb else 0,
                                             out_rows=rows), y[rows], rtol=0, atol=0)


@pytest.mark.parametrize("mode", MODES)
def test_pl_backward_finite_differences(mode):
    gi, go, fo, comb = mode
    T, K, N, E, k = 5, 4, 3, 3, 2
    idx, ss, off, w, gates, g = _pl_problem(12, T, K, N, E, k)
    fan_out = k if fo == "k" else 1
    x_rows = T * k if (gi or fan_out == 1) else T
    x = torch.randn(x_rows, K, generator=g, dtype=torch.float64)
    ck = k if comb else 0
    y_rows = T if comb else T * k
    dy = torch.randn(y_rows, N, generator=g, dtype=torch.float64)
    an = oracle.pl_bwd(dy, x, w, ss, off, fan_out, gi, go, gates, ck, want_dg=True)
    h = 1e-6

    def loss(xx, ww, gg):
        return float((oracle.pl_fwd(xx, ww, ss, off, fan_out, gi, go, gg, ck) * dy.numpy()).sum())

    for name, tensor, key in [("x", x, "dx"), ("w", w, "dw")]:
        fd = np.zeros(tensor.numel())
        flat = tensor.view(-1)
        for q in range(tensor.numel()):
            old = float(flat[q])
            flat[q] = old + h
            lp = loss(x, w, gates)
            flat[q] = old - h
            lm = loss(x, w, gates)
            flat[q] = old
            fd[q] = (lp - lm) / (2 * h)
        ref = an[key].ravel()
        assert np.max(np.abs(fd - ref)) / np.max(np.abs(ref)) < 1e-6, name
    fd = np.zeros(T * k)
    for p in range(T * k):
        gp, gm = gates.copy(), gates.copy()
        gp[p] += h
        gm[p] -= h
        fd[p] = (loss(x, w, gp) - loss(x, w, gm)) / (2 * h)
    assert np.max(np.abs(fd - an["dg"])) / np.max(np.abs(an["dg"])) < 1e-6


def test_mlp_equals_parallel_linear_composition():
    """The SMoE MLP is ParallelLinear(scatter->group, fan-out k), the activation,
    then ParallelLinear(group->scatter, gated k-way combine)."""
    x, w_r, w1, w2, dy = _tiny_mlp(13, 16, 8, 6, 4, 2, "gelu", torch.float32)
    idx, gates = oracle.route(x, w_r, None, 2)
    ss, off = oracle.sort(idx, 4)
    H = oracle.pl_fwd(x, w1, ss, off, 2, 0, 1)
    A = F.gelu(torch.from_numpy(H), approximate="tanh").numpy()
    Y = oracle.pl_fwd(A, w2.double(), ss, off, 1, 1, 0, gates.ravel(), 2)
    np.testing.assert_allclose(Y, oracle.mlp_fwd(x, w1, w2, "gelu", idx, gates)["y"], rtol=1e-12,
                               atol=1e-12)


# --------------------------------------------------------------------------
# Mixture-of-Attention core (grouped per-expert queries, shared keys/values)
# --------------------------------------------------------------------------
def _moa_problem(seed, T, L, kslots, E, heads, dh, dtype=torch.float64):
    g = torch.Generator().manual_seed(seed)
    idx = torch.stack([torch.randperm(E, generator=g)[:kslots] for _ in range(T)]).int().numpy()
    ss, _ = oracle.sort(idx, E)
    W = heads * dh
    q = torch.randn(T * kslots, W, generator=g, dtype=torch.float64).to(dtype)
    k = torch.randn(T, W, generator=g, dtype=torch.float64).to(dtype)
    v = torch.randn(T, W, generator=g, dtype=torch.float64).to(dtype)
    dout = torch.randn(T * kslots, W, generator=g, dtype=torch.float64).to(dtype)
    return ss, q, k, v, dout


def test_moa_attn_equals_torch_sdpa():
    """Every query row against torch's scaled-dot-product attention (fp64, CPU) with
    an explicit mask: query (t, j) sees the keys of its own sequence up to t."""
    T, L, kslots, E, heads, dh = 12, 6, 3, 5, 2, 8
    ss, q, k, v, _ = _moa_problem(3, T, L, kslots, E, heads, dh)
    out = oracle.moa_attn(q, k, v, ss, kslots, L, heads)
    S = T * kslots
    tok = torch.from_numpy(ss.astype(np.int64)) // kslots          # token of grouped row i
    mask = (torch.arange(T)[None, :] <= tok[:, None]) & (torch.arange(T)[None, :] // L == tok[:, None] // L)
    qh = q.view(S, heads, dh).transpose(0, 1)                      # [heads, S, dh]
    kh = k.view(T, heads, dh).transpose(0, 1)
    vh = v.view(T, heads, dh).transpose(0, 1)
    ref = F.scaled_dot_product_attention(qh, kh, vh, attn_mask=mask[None])  # [heads, S, dh]
    ref = ref.transpose(0, 1).reshape(S, heads * dh).numpy()
    np.testing.assert_allclose(out["o"], ref, rtol=1e-12, atol=1e-12)
    s = torch.einsum("hid,hjd->hij", qh, kh) / dh ** 0.5
    lse = torch.logsumexp(s.masked_fill(~mask[None], -torch.inf), dim=-1).T.numpy()
    np.testing.assert_allclose(out["lse"], lse, rtol=1e-12, atol=1e-12)


def test_moa_attn_backward_finite_differences():
    T, L, kslots, E, heads, dh = 6, 3, 2, 3, 2, 4
    ss, q, k, v, dout = _moa_problem(5, T, L, kslots, E, heads, dh)
    an = oracle.moa_attn(q, k, v, ss, kslots, L, heads, dout=dout)

    def loss():
        return float((oracle.moa_attn(q, k, v, ss, kslots, L, heads)["o"] * dout.numpy()).sum())

    h = 1e-6
    for name, tensor, key in (("q", q, "dq"), ("k", k, "dk"), ("v", v, "dv")):
        flat = tensor.view(-1)
        fd = np.zeros(tensor.numel())
        for i in range(tensor.numel()):
            old = float(flat[i])
            flat[i] = old + h
            lp = loss()
            flat[i] = old - h
            lm = loss()
            flat[i] = old
            fd[i] = (lp - lm) / (2 * h)
        ref = an[key].ravel()
        assert np.max(np.abs(fd - ref)) / np.max(np.abs(ref)) < 1e-6, name


def test_moa_attn_single_token_sequences_and_subsets():
    """L = 1: every query sees only its own token, so o = v[t] exactly, lse = <q, k_t>/sqrt(dh),
    dq = dk = 0 and dv[t] = the sum of dout over the token's k slots.  Row and token
    subsets of a longer problem equal the full computation."""
    T, kslots, E, heads, dh = 7, 2, 4, 2, 4
    ss, q, k, v, dout = _moa_problem(8, T, 1, kslots, E, heads, dh)
    out = oracle.moa_attn(q, k, v, ss, kslots, 1, heads, dout=dout)
    tok = ss // kslots
    np.testing.assert_array_equal(out["o"], v.numpy()[tok])
    qh = q.numpy().reshape(-1, heads, dh)
    kh = k.numpy().reshape(-1, heads, dh)[tok]
    np.testing.assert_allclose(out["lse"], (qh * kh).sum(-1) / dh ** 0.5, rtol=1e-13, atol=1e-13)
    assert np.all(out["dq"] == 0) and np.all(out["dk"] == 0)
    dv = np.zeros((T, heads * dh))
    np.add.at(dv, tok, dout.numpy())
    np.testing.assert_allclose(out["dv"], dv, rtol=1e-13, atol=1e-13)
    T, L = 16, 8
    ss, q, k, v, dout = _moa_problem(9, T, L, kslots, E, heads, dh)
    full = oracle.moa_attn(q, k, v, ss, kslots, L, heads, dout=dout)
    rows, toks = np.array([0, 5, 31, 17], np.int32), np.array([15, 0, 8, 3], np.int32)
    sub = oracle.moa_attn(q, k, v, ss, kslots, L, heads, dout=dout, q_rows=rows, kv_tokens=toks)
    for key in ("o", "lse", "dq"):
        np.testing.assert_allclose(sub[key], full[key][rows], rtol=1e-12, atol=1e-13)
    for key in ("dk", "dv"):
        np.testing.assert_allclose(sub[key], full[key][toks], rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# FP8 (e4m3) inference forward
# --------------------------------------------------------------------------
def test_e4m3_rounding_matches_torch_float8():
    """Round-to-nearest-even into e4m3 against torch's float8_e4m3fn conversion, on
    every representable magnitude, the midpoints between neighbours (ties), random
    values over the whole range including subnormals, and saturation at 448."""
    reps = np.unique(np.abs(torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn)
                            .float().numpy().astype(np.float64)))
    reps = reps[np.isfinite(reps)]
    mids = (reps[1:] + reps[:-1]) / 2
    r = _rng(5)
    rnd = np.concatenate([r.uniform(-448, 448, 4000), r.uniform(-0.05, 0.05, 2000),
                          np.ldexp(r.uniform(1, 2, 500), r.integers(-12, 9, 500))])
    v = np.concatenate([reps, -reps, mids, -mids, rnd])
    v = v[np.abs(v) <= 448]  # beyond 448 torch gives NaN; saturation is checked below
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(oracle.e4m3_round(v), want)
    assert oracle.e4m3_round(np.array([449.0, 460.0, -1000.0])).tolist() == [448.0, 448.0, -448.0]
    # codes decode back to the values (every finite code)
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)
    np.testing.assert_array_equal(oracle.e4m3_decode(codes),
                                  torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy())


def test_fp8_quantisation_of_rows_and_weights():
    """Each row (or weight column) maps its largest magnitude to 448 exactly, every
    code decodes to e4m3(fl32(v / scale)), and the weight codes are the columns'
    codes laid out K-major."""
    g = torch.Generator().manual_seed(6)
    x = (torch.randn(7, 40, generator=g) * 3).to(torch.bfloat16)
    x[3] = 0
    codes, sc = oracle.quantize_rows_fp8(x)
    xv = x.float().numpy()
    amax = np.abs(xv).max(1)
    np.testing.assert_array_equal(sc, np.where(amax > 0, (amax / np.float32(448)).astype(np.float32), 1))
    dec = oracle.e4m3_decode(codes)
    want = torch.from_numpy((xv / sc[:, None]).astype(np.float32)).to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(dec, want)
    assert np.all(np.abs(dec).max(1)[amax > 0] == 448)
    w = (torch.randn(3, 24, 10, generator=g) / 5).to(torch.bfloat16)
    wc, ws = oracle.quantize_weights_fp8(w)
    for e in range(3):
        c2, s2 = oracle.quantize_rows_fp8(w[e].T.contiguous())
        np.testing.assert_array_equal(wc[e], c2)
        np.testing.assert_array_equal(ws[e], s2)


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_fp8_forward_equals_dequantised_dense_reference(act):
    """The FP8 forward equals the dense evaluate-every-expert-and-mask reference run on
    the dequantised codes (torch, fp64): x8 * sx and w8 * s per column, A rounded to
    bf16 and requantised per row; and it stays close to the exact bf16 forward."""
    T, d, f, E, k = 12, 32, 24, 4, 2
    x, w_r, w1, w2, _ = _tiny_mlp(14, T, d, f, E, k, act, torch.bfloat16)
    idx, gates = oracle.route(x, w_r, None, k)
    w1q, s1 = oracle.quantize_weights_fp8(w1)
    w2q, s2 = oracle.quantize_weights_fp8(w2)
    out = oracle.mlp_fwd_fp8(x, w1q, s1, w2q, s2, act, idx, gates, want_a=True)
    x8, sx = oracle.quantize_rows_fp8(x)
    xd = torch.from_numpy(oracle.e4m3_decode(x8) * sx[:, None].astype(np.float64))
    W1 = torch.from_numpy(oracle.e4m3_decode(w1q) * s1[:, :, None].astype(np.float64)).transpose(1, 2)
    W2 = torch.from_numpy(oracle.e4m3_decode(w2q) * s2[:, :, None].astype(np.float64)).transpose(1, 2)
    y = torch.zeros(T, d, dtype=torch.float64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            h = xd[t] @ W1[e]
            a = F.gelu(h, approximate="tanh") if act == "gelu" else F.silu(h[:f]) * h[f:]
            a = a.float().to(torch.bfloat16).double()
            np.testing.assert_allclose(out["a"][t * k + j], a.numpy(), rtol=0, atol=0)
            a8, sa = oracle.quantize_rows_fp8(a[None])
            ad = torch.from_numpy(oracle.e4m3_decode(a8)[0] * np.float64(sa[0]))
            y[t] += gates[t, j] * (ad @ W2[e])
    np.testing.assert_allclose(out["y"], y.numpy(), rtol=1e-12, atol=1e-12)
    # e4m3 keeps 3 mantissa bits (relative steps up to 2^-3); with 24-32 terms per
    # product little of that averages out, so only a loose agreement is expected here
    exact = oracle.mlp_fwd(x, w1, w2, act, idx, gates)["y"]
    assert np.max(np.abs(out["y"] - exact)) / np.max(np.abs(exact)) < 0.25
