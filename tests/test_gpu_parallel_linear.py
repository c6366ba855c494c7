"""GPU parity of parallel_linear_fwd / parallel_linear_bwd against the CPU oracle
in every grouped/scattered combination, gated and ungated, fp32 and bf16, on
shapes that span several tiles with ragged tails and an empty expert."""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_smoe_b200 as smoe

from ._util import TOL, assert_close

pytestmark = pytest.mark.gpu

MODES = {  # name: (grouped_in, grouped_out, fan_out is k?, combine?)
    "scatter2group_fanout": (0, 1, True, False),
    "group2scatter_combine": (1, 0, False, True),
    "group2scatter": (1, 0, False, False),
    "group2group": (1, 1, False, False),
    "scatter2scatter": (0, 0, False, False),
    "scatter2scatter_fanout_combine": (0, 0, True, True),
}

SHAPES = {torch.float32: dict(T=150, k=2, K=136, N=72, E=5),
          torch.bfloat16: dict(T=300, k=2, K=264, N=392, E=5)}


def _problem(dtype, mode, gated, seed=0, shape=None):
    sh = shape or SHAPES[dtype]
    T, k, K, N, E = sh["T"], sh["k"], sh["K"], sh["N"], sh["E"]
    gi, go, fo_k, comb = MODES[mode]
    g = torch.Generator(device="cuda").manual_seed(seed)
    idx = torch.randint(0, E, (T, k), generator=g, device="cuda", dtype=torch.int32)
    if E > 4:
        idx[idx == 3] = 1                      # expert 3 is empty
        idx[: T // 3] = torch.where(idx[: T // 3] == 0, 4, idx[: T // 3])  # skew the sizes
    ss, off = smoe.smoe_sort(idx, E)
    fan_out = k if fo_k else 1
    x_rows = T * k if (gi or fan_out == 1) else T
    x = torch.randn(x_rows, K, generator=g, device="cuda").to(dtype)
    w = (torch.randn(E, K, N, generator=g, device="cuda") / K ** 0.5).to(dtype)
    gates = torch.rand(T * k, generator=g, device="cuda") if gated else None
    ck = k if comb else 0
    y_rows = T if comb else T * k
    dy = torch.randn(y_rows, N, generator=g, device="cuda").to(dtype)
    return dict(idx=idx, ss=ss, off=off, x=x, w=w, gates=gates, fan_out=fan_out, gi=gi, go=go,
                ck=ck, dy=dy)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("gated", [False, True])
def test_parallel_linear_fwd_bwd(dtype, mode, gated):
    P = _problem(dtype, mode, gated)
    y = smoe.parallel_linear_fwd(P["x"], P["w"], P["ss"], P["off"], P["fan_out"], P["gi"], P["go"],
                                 P["gates"], P["ck"])
    dx, dw, dg = smoe.parallel_linear_bwd(P["dy"], P["x"], P["w"], P["ss"], P["off"], P["fan_out"],
                                          P["gi"], P["go"], P["gates"], P["ck"], want_dgates=gated)
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    ss, off = P["ss"].cpu().numpy(), P["off"].cpu().numpy()
    gts = None if P["gates"] is None else P["gates"].cpu().double().numpy()
    ref_y = oracle.pl_fwd(P["x"].cpu(), P["w"].cpu(), ss, off, P["fan_out"], P["gi"], P["go"], gts,
                          P["ck"])
    assert_close("y", y, ref_y, dtype)
    ref = oracle.pl_bwd(P["dy"].cpu(), P["x"].cpu(), P["w"].cpu(), ss, off, P["fan_out"], P["gi"],
                        P["go"], gts, P["ck"], want_dg=gated)
    assert_close("dx", dx, ref["dx"], dtype)
    assert_close("dw", dw, ref["dw"], dtype)
    assert np.all(dw[3].cpu().numpy() == 0.0)      # the empty expert's gradient is written as 0
    if gated:
        assert_close("dgates", dg, ref["dg"], dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_parallel_linear_bwd_dw_only_gated(dtype):
    """dw alone with gates: no dx GEMM runs, and the dW kernel applies the gates
    to the rows it gathers (no gated copy of x)."""
    P = _problem(dtype, "group2scatter_combine", True, seed=3)
    _, dw, _ = smoe.parallel_linear_bwd(P["dy"], P["x"], P["w"], P["ss"], P["off"], P["fan_out"],
                                        P["gi"], P["go"], P["gates"], P["ck"], want_dx=False)
    ref = oracle.pl_bwd(P["dy"].cpu(), P["x"].cpu(), P["w"].cpu(), P["ss"].cpu().numpy(),
                        P["off"].cpu().numpy(), P["fan_out"], P["gi"], P["go"],
                        P["gates"].cpu().double().numpy(), P["ck"], want_dx=False)
    assert_close("dw", dw, ref["dw"], dtype)


def test_parallel_linear_is_deterministic():
    P = _problem(torch.bfloat16, "scatter2scatter_fanout_combine", True, seed=5)
    outs = []
    for _ in range(2):
        y = smoe.parallel_linear_fwd(P["x"], P["w"], P["ss"], P["off"], P["fan_out"], P["gi"],
                                     P["go"], P["gates"], P["ck"])
        r = smoe.parallel_linear_bwd(P["dy"], P["x"], P["w"], P["ss"], P["off"], P["fan_out"],
                                     P["gi"], P["go"], P["gates"], P["ck"], want_dgates=True)
        outs.append([y] + list(r))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


SLICES = [0, 1, 127, 128, 129, 255, 256, 257]  # rows per expert: empty, one row, tile edges


def _sized_problem(dtype, mode, gated, sizes, seed=0):
    """k = 1 routing with exactly sizes[e] rows for expert e (shuffled over tokens)."""
    K, N = (264, 392) if dtype == torch.bfloat16 else (136, 72)
    E, T, k = len(sizes), sum(sizes), 1
    gi, go, fo_k, comb = MODES[mode]
    g = torch.Generator(device="cuda").manual_seed(seed)
    ids = torch.cat([torch.full((n,), e, dtype=torch.int32) for e, n in enumerate(sizes)])
    perm = torch.randperm(T, generator=torch.Generator().manual_seed(seed))
    idx = ids[perm].reshape(T, k).cuda()
    ss, off = smoe.smoe_sort(idx, E)
    assert off.cpu().tolist() == np.concatenate([[0], np.cumsum(sizes)]).tolist()
    x = torch.randn(T, K, generator=g, device="cuda").to(dtype)
    w = (torch.randn(E, K, N, generator=g, device="cuda") / K ** 0.5).to(dtype)
    gates = torch.rand(T, generator=g, device="cuda") if gated else None
    dy = torch.randn(T, N, generator=g, device="cuda").to(dtype)
    return dict(ss=ss, off=off, x=x, w=w, gates=gates, fan_out=1, gi=gi, go=go,
                ck=k if comb else 0, dy=dy)


def _check_problem(P, dtype, gated):
    y = smoe.parallel_linear_fwd(P["x"], P["w"], P["ss"], P["off"], P["fan_out"], P["gi"], P["go"],
                                 P["gates"], P["ck"])
    dx, dw, dg = smoe.parallel_linear_bwd(P["dy"], P["x"], P["w"], P["ss"], P["off"], P["fan_out"],
                                          P["gi"], P["go"], P["gates"], P["ck"], want_dgates=gated)
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    ss, off = P["ss"].cpu().numpy(), P["off"].cpu().numpy()
    gts = None if P["gates"] is None else P["gates"].cpu().double().numpy()
    assert_close("y", y, oracle.pl_fwd(P["x"].cpu(), P["w"].cpu(), ss, off, P["fan_out"], P["gi"],
                                       P["go"], gts, P["ck"]), dtype)
    ref = oracle.pl_bwd(P["dy"].cpu(), P["x"].cpu(), P["w"].cpu(), ss, off, P["fan_out"], P["gi"],
                        P["go"], gts, P["ck"], want_dg=gated)
    assert_close("dx", dx, ref["dx"], dtype)
    assert_close("dw", dw, ref["dw"], dtype)
    if gated:
        assert_close("dgates", dg, ref["dg"], dtype)
    return dw


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("gated", [False, True])
def test_parallel_linear_tile_boundaries(dtype, mode, gated):
    """Expert slices of 0, 1, 127, 128, 129, 255, 256 and 257 rows: empty experts,
    one-row tiles, exact tiles, one row past a tile (ragged warps and the per-row
    store path next to the boxed one)."""
    dw = _check_problem(_sized_problem(dtype, mode, gated, SLICES), dtype, gated)
    assert np.all(dw[0].cpu().numpy() == 0.0)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_parallel_linear_all_tokens_to_one_expert(dtype):
    dw = _check_problem(_sized_problem(dtype, "scatter2group_fanout", True, [0, 0, 300, 0]), dtype, True)
    assert np.all(dw[[0, 1, 3]].cpu().numpy() == 0.0)


@pytest.mark.parametrize("mode", ["scatter2group_fanout", "group2scatter_combine", "group2group"])
def test_parallel_linear_gated_dw_narrow(mode):
    """Gated dW with a narrow output (K, N <= 128): the gate is applied by the
    single-CTA dW kernel (wider products use the CTA-pair kernel), with the
    gathered operand on either side and a grouped operand gathered row by row."""
    P = _problem(torch.bfloat16, mode, True, seed=7, shape=dict(T=260, k=2, K=120, N=96, E=5))
    dx, dw, dg = smoe.parallel_linear_bwd(P["dy"], P["x"], P["w"], P["ss"], P["off"], P["fan_out"],
                                          P["gi"], P["go"], P["gates"], P["ck"], want_dgates=True)
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    ref = oracle.pl_bwd(P["dy"].cpu(), P["x"].cpu(), P["w"].cpu(), P["ss"].cpu().numpy(),
                        P["off"].cpu().numpy(), P["fan_out"], P["gi"], P["go"],
                        P["gates"].cpu().double().numpy(), P["ck"], want_dg=True)
    assert_close("dx", dx, ref["dx"], torch.bfloat16)
    assert_close("dw", dw, ref["dw"], torch.bfloat16)
    assert_close("dgates", dg, ref["dg"], torch.bfloat16)
    assert np.all(dw[3].cpu().numpy() == 0.0)


@pytest.mark.parametrize("mode", ["group2group", "scatter2group_fanout", "group2scatter_combine"])
def test_parallel_linear_long_k_pairs(mode):
    """K = 4096 over slices of at least 2048 rows per expert under GEMM policy 1:
    the TMA-fed products run on CTA pairs (tiles in panels), the gathered ones
    gather with 4 warps, and the dW of a gathered operand runs on the pair dW
    kernel; every element against the oracle (ragged pair tiles and a ragged N
    tile)."""
    gated = mode == "group2scatter_combine"
    P = _problem(torch.bfloat16, mode, gated, seed=5, shape=dict(T=2200, k=2, K=4096, N=264, E=2))
    smoe.smoe_set_gemm_policy(1)
    try:
        y = smoe.parallel_linear_fwd(P["x"], P["w"], P["ss"], P["off"], P["fan_out"], P["gi"], P["go"],
                                     P["gates"], P["ck"])
        dx, dw, dg = smoe.parallel_linear_bwd(P["dy"], P["x"], P["w"], P["ss"], P["off"], P["fan_out"],
                                              P["gi"], P["go"], P["gates"], P["ck"], want_dgates=gated)
        torch.cuda.synchronize()
    finally:
        smoe.smoe_set_gemm_policy(0)
    assert smoe.smoe_check() == 0
    ss, off = P["ss"].cpu().numpy(), P["off"].cpu().numpy()
    assert np.diff(off).min() >= 2048
    gts = None if P["gates"] is None else P["gates"].cpu().double().numpy()
    ref_y = oracle.pl_fwd(P["x"].cpu(), P["w"].cpu(), ss, off, P["fan_out"], P["gi"], P["go"], gts,
                          P["ck"])
    assert_close("y", y, ref_y, torch.bfloat16)
    ref = oracle.pl_bwd(P["dy"].cpu(), P["x"].cpu(), P["w"].cpu(), ss, off, P["fan_out"], P["gi"],
                        P["go"], gts, P["ck"], want_dg=gated)
    assert_close("dx", dx, ref["dx"], torch.bfloat16)
    assert_close("dw", dw, ref["dw"], torch.bfloat16)
    if gated:
        assert_close("dgates", dg, ref["dg"], torch.bfloat16)


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("gated", [False, True])
def test_parallel_linear_slab_shapes(mode, gated):
    """K = 4096 and N a multiple of 64: the MN-major weights (forward) and both
    operands of a TMA-fed dW load through the slab view (one TMA load per run of
    64-column slabs); every element against the oracle, with a ragged last N tile
    (N = 320) and an empty expert."""
    P = _problem(torch.bfloat16, mode, gated, seed=7, shape=dict(T=300, k=2, K=4096, N=320, E=5))
    y = smoe.parallel_linear_fwd(P["x"], P["w"], P["ss"], P["off"], P["fan_out"], P["gi"], P["go"],
                                 P["gates"], P["ck"])
    dx, dw, dg = smoe.parallel_linear_bwd(P["dy"], P["x"], P["w"], P["ss"], P["off"], P["fan_out"],
                                          P["gi"], P["go"], P["gates"], P["ck"], want_dgates=gated)
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    ss, off = P["ss"].cpu().numpy(), P["off"].cpu().numpy()
    gts = None if P["gates"] is None else P["gates"].cpu().double().numpy()
    ref_y = oracle.pl_fwd(P["x"].cpu(), P["w"].cpu(), ss, off, P["fan_out"], P["gi"], P["go"], gts,
                          P["ck"])
    assert_close("y", y, ref_y, torch.bfloat16)
    ref = oracle.pl_bwd(P["dy"].cpu(), P["x"].cpu(), P["w"].cpu(), ss, off, P["fan_out"], P["gi"],
                        P["go"], gts, P["ck"], want_dg=gated)
    assert_close("dx", dx, ref["dx"], torch.bfloat16)
    assert_close("dw", dw, ref["dw"], torch.bfloat16)
    assert np.all(dw[3].cpu().numpy() == 0.0)
    if gated:
        assert_close("dgates", dg, ref["dg"], torch.bfloat16)
