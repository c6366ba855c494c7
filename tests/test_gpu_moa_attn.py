"""GPU parity of the Mixture-of-Attention core (smoe_moa_attn_fwd / _bwd) against the
CPU oracle: every element of o, lse, dq, dk and dv at reduced shapes (several query
tiles and key blocks per sequence, ragged sequence ends, padding rows when 128 is
not a multiple of kslots), sampled rows at the full Mixture-of-Attention workload,
run-to-run determinism, and the whole layer (router, per-expert query projection,
attention, per-expert output projection with the gated combine) composed at a
reduced size."""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_smoe_b200 as smoe
from sparse_mixture_experts_smoe_b200.inputs import WORKLOADS, make_moa_attn_inputs

from ._util import assert_close

pytestmark = pytest.mark.gpu
BF = torch.bfloat16

SHAPES = {
    # T, L, kslots, E, heads
    "two_sequences_k4": dict(T=384, L=192, kslots=4, E=6, heads=2),
    "ragged_last_sequence_k3": dict(T=300, L=160, kslots=3, E=5, heads=1),
    "single_sequence_k1": dict(T=260, L=260, kslots=1, E=3, heads=2),
    "many_slots_k8": dict(T=200, L=100, kslots=8, E=10, heads=1),
}


def _routing(T, kslots, E, seed):
    g = torch.Generator().manual_seed(seed)
    idx = torch.stack([torch.randperm(E, generator=g)[:kslots] for _ in range(T)]).int()
    ss, off = oracle.sort(idx.numpy(), E)
    return idx, ss, off


def _problem(cfg, seed):
    T, kslots, E, heads = cfg["T"], cfg["kslots"], cfg["E"], cfg["heads"]
    _, ss, _ = _routing(T, kslots, E, seed)
    g = torch.Generator(device="cuda").manual_seed(seed)
    W = heads * 128
    mk = lambda rows: torch.randn(rows, W, generator=g, device="cuda").to(BF)  # noqa: E731
    return ss, mk(T * kslots), mk(T), mk(T), mk(T * kslots)


@pytest.mark.parametrize("name", list(SHAPES))
def test_moa_attn_every_element(name):
    cfg = SHAPES[name]
    T, L, kslots, heads = cfg["T"], cfg["L"], cfg["kslots"], cfg["heads"]
    ss, q, k, v, dout = _problem(cfg, seed=11)
    ss_d = torch.from_numpy(ss).cuda()
    o, lse = smoe.smoe_moa_attn_fwd(q, k, v, ss_d, kslots, L, heads)
    dq, dk, dv = smoe.smoe_moa_attn_bwd(q, k, v, o, lse, dout, ss_d, kslots, L, heads)
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    ref = oracle.moa_attn(q.cpu(), k.cpu(), v.cpu(), ss, kslots, L, heads, dout=dout.cpu())
    assert_close("o", o, ref["o"], BF)
    assert_close("lse", lse, ref["lse"], BF)
    assert_close("dq", dq, ref["dq"], BF)
    assert_close("dk", dk, ref["dk"], BF)
    assert_close("dv", dv, ref["dv"], BF)


def test_moa_attn_is_deterministic():
    cfg = SHAPES["two_sequences_k4"]
    ss, q, k, v, dout = _problem(cfg, seed=12)
    ss_d = torch.from_numpy(ss).cuda()
    outs = []
    for _ in range(2):
        o, lse = smoe.smoe_moa_attn_fwd(q, k, v, ss_d, cfg["kslots"], cfg["L"], cfg["heads"])
        outs.append((o, lse) + smoe.smoe_moa_attn_bwd(q, k, v, o, lse, dout, ss_d, cfg["kslots"],
                                                      cfg["L"], cfg["heads"]))
    for x, y in zip(*outs):
        assert torch.equal(x, y)


def test_moa_attn_full_size_sampled():
    """The Mixture-of-Attention workload (T = 8192 tokens in sequences of 2048,
    16 experts, top-4, 4 heads of 128): routing through smoe_route / smoe_sort, the
    attention core at full size, sampled grouped rows (o, lse, dq) and sampled
    tokens of one sequence (dk, dv) against the oracle."""
    cfg = WORKLOADS["moa_bf16"]
    inp = make_moa_attn_inputs(cfg, device="cuda")
    T, k, E, L, heads = cfg["T"], cfg["k"], cfg["E"], cfg["L"], cfg["heads"]
    c = {n: t.cpu() for n, t in inp.items() if t is not None}
    idx, _ = oracle.route(c["x"], c["w_r"], None, k)
    ss, _ = oracle.sort(idx, E)
    ss_d = torch.from_numpy(ss).cuda()
    q, kk, v, dout = inp["q"], inp["k"], inp["v"], inp["do"]
    o, lse = smoe.smoe_moa_attn_fwd(q, kk, v, ss_d, k, L, heads)
    dq, dk, dv = smoe.smoe_moa_attn_bwd(q, kk, v, o, lse, dout, ss_d, k, L, heads)
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    rng = np.random.default_rng(0)
    S = T * k
    rows = np.unique(np.concatenate([[0, S - 1], rng.choice(S, 24, replace=False)])).astype(np.int32)
    seq = 2  # dk/dv: tokens of one sequence (its first, last and a sample)
    toks = np.unique(np.concatenate([[seq * L, seq * L + L - 1],
                                     seq * L + rng.choice(L, 10, replace=False)])).astype(np.int32)
    ref = oracle.moa_attn(c["q"], c["k"], c["v"], ss, k, L, heads, dout=c["do"], q_rows=rows,
                          kv_tokens=toks)
    R = torch.from_numpy(rows).long().cuda()
    Tk = torch.from_numpy(toks).long().cuda()
    assert_close("o[rows]", o[R], ref["o"], BF)
    assert_close("lse[rows]", lse[R], ref["lse"], BF)
    assert_close("dq[rows]", dq[R], ref["dq"], BF)
    assert_close("dk[tokens]", dk[Tk], ref["dk"], BF)
    assert_close("dv[tokens]", dv[Tk], ref["dv"], BF)


def test_moa_layer_forward_composed():
    """The whole Mixture-of-Attention layer forward at a reduced size: route, sort,
    q = ParallelLinear(x, Wq; scatter->group), shared k = x Wk and v = x Wv (one-expert
    ParallelLinear), the attention core, z = ParallelLinear(o, Wo; group->scatter,
    gated combine).  The oracle composes its own routing, ParallelLinear and
    attention in fp64 (each stage's input rounded to bf16 as the GPU stores it)."""
    T, L, d, E, k, heads = 256, 128, 256, 6, 2, 2
    h = heads * 128
    g = torch.Generator(device="cuda").manual_seed(21)
    x = torch.randn(T, d, generator=g, device="cuda").to(BF)
    w_r = (torch.randn(d, E, generator=g, device="cuda") / d ** 0.5).to(BF)
    wq = (torch.randn(E, d, h, generator=g, device="cuda") / d ** 0.5).to(BF)
    wk = (torch.randn(1, d, h, generator=g, device="cuda") / d ** 0.5).to(BF)
    wv = (torch.randn(1, d, h, generator=g, device="cuda") / d ** 0.5).to(BF)
    wo = (torch.randn(E, h, d, generator=g, device="cuda") / h ** 0.5).to(BF)
    idx, gates = smoe.smoe_route(x, w_r, None, k)
    ss, off = smoe.smoe_sort(idx, E)
    one = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    ident = torch.arange(T, dtype=torch.int32, device="cuda")
    q = smoe.parallel_linear_fwd(x, wq, ss, off, k, 0, 1)
    kk = smoe.parallel_linear_fwd(x, wk, ident, one, 1, 1, 1)
    v = smoe.parallel_linear_fwd(x, wv, ident, one, 1, 1, 1)
    o, _ = smoe.smoe_moa_attn_fwd(q, kk, v, ss, k, L, heads)
    z = smoe.parallel_linear_fwd(o, wo, ss, off, 1, 1, 0, gates, k)
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    xc = x.cpu()
    ridx, rg = oracle.route(xc, w_r.cpu(), None, k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ridx)
    rss, roff = oracle.sort(ridx, E)
    tok = np.arange(T, dtype=np.int32)
    toff = np.array([0, T], np.int32)
    rq = oracle.pl_fwd(xc, wq.cpu(), rss, roff, k, 0, 1)
    rk = oracle.pl_fwd(xc, wk.cpu(), tok, toff, 1, 1, 1)
    rv = oracle.pl_fwd(xc, wv.cpu(), tok, toff, 1, 1, 1)
    bf = lambda a: torch.from_numpy(a).to(BF)  # noqa: E731  (the GPU stores each stage in bf16)
    ro = oracle.moa_attn(bf(rq), bf(rk), bf(rv), rss, k, L, heads)["o"]
    rz = oracle.pl_fwd(bf(ro), wo.cpu(), rss, roff, 1, 1, 0, rg.ravel(), k)
    assert_close("q", q, rq, BF)
    assert_close("o", o, ro, BF)
    assert_close("z", z, rz, BF)
