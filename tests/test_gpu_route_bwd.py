"""GPU parity of the router backward (smoe_route_bwd) against the CPU oracle,
every element of dW_r, db and the router's share of dx, at the specified
workloads' full sizes and at shapes chosen to reach each instance of the router
weight-gradient kernel.

The weight gradient sums each expert's slots in runs of R expert-sorted slots over
column slabs of 256 or 512 bf16 (128 or 256 fp32) columns; the run length and slab
width follow from T*k and d:
  * tiny fp32 workload (T*k = 512, d = 128) and the small bf16 workload
    (T*k = 8192, d = 1024): R = 32, one 16-byte load per lane;
  * T*k = 98304, d = 256 (bf16) and T*k = 32768, d = 2048 (fp32): R = 32, two loads;
  * the Mixtral-shaped workload (T*k = 32768, d = 4096): R = 64, two loads;
  * the fine-grained workload (T*k = 131072, d = 2048): R = 128, two loads.
Routing (indices and gates) comes from the oracle and is handed to both sides;
the upstream gate gradients are seeded N(0, 1).
"""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_smoe_b200 as smoe
from sparse_mixture_experts_smoe_b200.inputs import WORKLOADS, make_router_inputs

from ._util import assert_close

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_fp32_gelu": WORKLOADS["tiny_fp32_gelu"],
    "small_bf16_gelu": WORKLOADS["small_bf16_gelu"],
    "mixtral_bf16_swiglu": WORKLOADS["mixtral_bf16_swiglu"],
    "finegrained_zipf_bf16_swiglu": WORKLOADS["finegrained_zipf_bf16_swiglu"],
    "run32_two_loads_bf16": dict(T=12288, d=256, E=32, k=8, dtype="bf16"),
    "run32_two_loads_f32": dict(T=16384, d=2048, E=8, k=2, dtype="f32"),
    "ragged_bf16": dict(T=1001, d=200, E=12, k=3, dtype="bf16"),
}


@pytest.mark.parametrize("name", list(CASES))
def test_route_bwd_every_element(name):
    cfg = CASES[name]
    inp = make_router_inputs(cfg, seed=4, device="cuda")
    x, w_r, b_r, dgates = inp["x"], inp["w_r"], inp["b_r"], inp["dgates"]
    dt = x.dtype
    xc, wc = x.cpu(), w_r.cpu()
    idx, gates = oracle.route(xc, wc, None if b_r is None else b_r.cpu(), cfg["k"])
    gates32 = torch.from_numpy(gates.astype(np.float32))
    ref = oracle.route_bwd(xc, wc, idx, gates32, dgates.cpu())
    dx = torch.zeros_like(x)
    dw_r, db_r = smoe.smoe_route_bwd(x, w_r, torch.from_numpy(idx).cuda(), gates32.cuda(), dgates,
                                     dx=dx)
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    assert_close("dw_r", dw_r, ref["dw_r"], dt)
    assert_close("db_r", db_r, ref["db_r"], dt)
    assert_close("dx (router share)", dx, ref["dx"], dt)
    # an expert that no slot selected has an exactly zero column
    unused = np.setdiff1d(np.arange(cfg["E"]), np.unique(idx))
    for e in unused:
        assert torch.all(dw_r[:, int(e)] == 0) and float(db_r[int(e)]) == 0.0


def test_route_bwd_accumulates_into_dx():
    """dx is accumulated (+=), as the MLP backward relies on."""
    cfg = CASES["ragged_bf16"]
    inp = make_router_inputs(cfg, seed=5, device="cuda")
    x, w_r, dgates = inp["x"], inp["w_r"], inp["dgates"]
    xc, wc = x.cpu(), w_r.cpu()
    idx, gates = oracle.route(xc, wc, None, cfg["k"])
    gates32 = torch.from_numpy(gates.astype(np.float32))
    ref = oracle.route_bwd(xc, wc, idx, gates32, dgates.cpu())
    base = torch.full_like(x, 0.5)
    dx = base.clone()
    smoe.smoe_route_bwd(x, w_r, torch.from_numpy(idx).cuda(), gates32.cuda(), dgates, dx=dx)
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    assert_close("dx - 0.5", dx.float() - 0.5, ref["dx"], torch.bfloat16)
