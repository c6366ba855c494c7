"""GPU parity of smoe_route and smoe_sort against the CPU oracle: bit-exact
indices, sorted slots and offsets; gates within fp32 rounding of the fp64 oracle.
Runs every workload at its full size (routing is cheap for the oracle) plus edge
cases."""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_smoe_b200 as smoe
from sparse_mixture_experts_smoe_b200.inputs import WORKLOADS, make_mlp_inputs, make_moa_inputs

from ._util import rel_err

pytestmark = pytest.mark.gpu


def _router_inputs(name):
    cfg = WORKLOADS[name]
    inp = make_moa_inputs(cfg, device="cuda") if cfg["kind"] == "moa" else \
        make_mlp_inputs(cfg, device="cuda", with_dy=False)
    return cfg, inp["x"], inp["w_r"], inp["b_r"]


def _check_route(x, w_r, b_r, k):
    idx, gates = smoe.smoe_route(x, w_r, b_r, k)
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    ref_idx, ref_g = oracle.route(x.cpu(), w_r.cpu(), None if b_r is None else b_r.cpu(), k)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
    assert rel_err(gates, ref_g) < 2e-6
    return idx, ref_idx


def _check_sort(idx, E):
    ss, off = smoe.smoe_sort(idx, E)
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    ref_ss, ref_off = oracle.sort(idx.cpu().numpy(), E)
    np.testing.assert_array_equal(off.cpu().numpy(), ref_off)
    np.testing.assert_array_equal(ss.cpu().numpy(), ref_ss)
    return ss, off


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_route_and_sort_full_size(name):
    cfg, x, w_r, b_r = _router_inputs(name)
    idx, ref_idx = _check_route(x, w_r, b_r, cfg["k"])
    ss, off = _check_sort(idx, cfg["E"])
    counts = np.diff(off.cpu().numpy())
    if "n_empty" in cfg:
        assert np.sum(counts == 0) >= cfg["n_empty"]
    # report how many tokens an fp64 router would route differently (near ties)
    l64 = oracle.router_logits_f64(x.cpu(), w_r.cpu(), None if b_r is None else b_r.cpu())
    top64 = np.sort(np.argsort(-l64, axis=1, kind="stable")[:, :cfg["k"]], 1)
    flips = int(np.sum(np.any(top64 != np.sort(ref_idx, 1), axis=1)))
    print(f"{name}: tokens whose fp64 top-k differs: {flips}")


@pytest.mark.parametrize("T,d,E,k,dtype", [
    (1, 8, 1, 1, torch.float32),       # one token, one expert
    (37, 40, 3, 3, torch.bfloat16),    # k == E, d not a multiple of 32, ragged warps
    (129, 264, 16, 4, torch.float32),
    (500, 128, 64, 8, torch.bfloat16),  # the two-token-per-warp path
    (300, 96, 128, 16, torch.bfloat16),  # the largest E and k
    (64, 1024, 8, 2, torch.bfloat16),   # several staged W_r chunks
])
def test_route_edge_shapes(T, d, E, k, dtype):
    g = torch.Generator(device="cuda").manual_seed(T + d + E)
    x = torch.randn(T, d, generator=g, device="cuda").to(dtype)
    w_r = (torch.randn(d, E, generator=g, device="cuda") / d ** 0.5).to(dtype)
    b_r = torch.randn(E, generator=g, device="cuda") * 0.1
    _check_route(x, w_r, b_r, k)
    _check_route(x, w_r, None, k)


def test_route_ties_go_to_lower_expert():
    # all-zero tokens: every logit equals its bias; equal biases tie
    T, d, E, k = 8, 64, 8, 3
    x = torch.zeros(T, d, device="cuda", dtype=torch.bfloat16)
    w_r = torch.randn(d, E, device="cuda").to(torch.bfloat16)
    b_r = torch.tensor([0.5, 1.0, 1.0, 0.0, 1.0, -1.0, 0.5, 1.0], device="cuda")
    idx, gates = smoe.smoe_route(x, w_r, b_r, k)
    assert idx.cpu().tolist() == [[1, 2, 4]] * T
    np.testing.assert_allclose(gates.cpu().numpy(), 1.0 / 3.0, rtol=1e-6)


@pytest.mark.parametrize("E,k", [(64, 6), (128, 9)])
def test_route_ties_and_nan_follow_the_scan(E, k):
    """Logits equal to the bias (x = 0): a five-way tie spread over lanes and slots
    goes to the lower ids; a NaN logit is taken only when it is the first free
    expert (the scan starts there and a comparison with NaN never replaces it),
    and is skipped anywhere else -- as in the oracle's scan."""
    T, d = 6, 64
    x = torch.zeros(T, d, device="cuda", dtype=torch.bfloat16)
    w_r = torch.randn(d, E, device="cuda").to(torch.bfloat16)
    b = torch.zeros(E)
    b[[3, 40, 35, 8, E - 1]] = 1.0
    b[[17, 50]] = 2.0
    nan_first, nan_later = b.clone(), b.clone()
    nan_first[0] = float("nan")
    nan_later[40] = float("nan")
    for bias in (b, nan_first, nan_later):
        idx, gates = smoe.smoe_route(x, w_r, bias.cuda(), k)
        torch.cuda.synchronize()
        ref_idx, ref_g = oracle.route(x.cpu(), w_r.cpu(), bias, k)
        np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx)
        np.testing.assert_allclose(gates.cpu().numpy(), ref_g, rtol=2e-6, equal_nan=True)
    assert idx.cpu().tolist()[0][:4] == [17, 50, 3, 8]


@pytest.mark.parametrize("T,k,E,pattern", [
    (1, 1, 1, "uniform"),
    (5000, 2, 8, "uniform"),        # several 4096-slot chunks plus a ragged tail
    (3000, 8, 64, "skew"),          # empty and tiny experts
    (4096, 4, 16, "one"),           # everything to one expert
    (2000, 3, 1000, "uniform"),     # many experts, most empty
])
def test_sort_edge_cases(T, k, E, pattern):
    g = torch.Generator(device="cuda").manual_seed(T * 7 + E)
    if pattern == "uniform":
        idx = torch.randint(0, E, (T, k), generator=g, device="cuda", dtype=torch.int32)
    elif pattern == "one":
        idx = torch.full((T, k), E // 2, device="cuda", dtype=torch.int32)
    else:
        p = torch.arange(1, E + 1, device="cuda", dtype=torch.float64) ** -1.5
        p[E // 2:E // 2 + 4] = 0
        idx = torch.multinomial(p, T * k, replacement=True, generator=g).view(T, k).int()
    _check_sort(idx, E)


def test_sort_reports_out_of_range_ids():
    idx = torch.randint(0, 8, (100, 2), device="cuda", dtype=torch.int32)
    idx[17, 1] = 8      # one past the end
    idx[50, 0] = -3
    smoe.smoe_sort(idx, 8)
    assert smoe.smoe_check() == -4       # SMOE_ERR_DATA
    assert smoe.smoe_check() == 0        # the word is cleared once read


def test_device_wait_timeout_becomes_host_error():
    """A bounded device wait on a barrier nothing completes gives up, and the host
    sees SMOE_ERR_TIMEOUT from smoe_check; the word is then clear and the library
    keeps working (the failure path without a fault or a hang)."""
    smoe.smoe_selftest_wait_timeout(20000)  # 20 ms
    assert smoe.smoe_check() == -5  # SMOE_ERR_TIMEOUT
    assert b"bounded device wait" in smoe.lib().smoe_last_error()
    assert smoe.smoe_check() == 0
    x = torch.randn(64, 128, device="cuda").to(torch.bfloat16)
    w_r = (torch.randn(128, 8, device="cuda") / 128 ** 0.5).to(torch.bfloat16)
    _check_route(x, w_r, None, 2)
