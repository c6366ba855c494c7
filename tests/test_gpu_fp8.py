"""GPU parity of the FP8 inference forward (smoe_quantize_weights_fp8 and
smoe_mlp_fwd_fp8) against the CPU oracle.  The weight codes and scales are
compared value for value with the oracle's own quantisation (both take the
decision in fp32); the forward's outputs (y, the saved bf16 activations h and a)
against the oracle's FP8 forward, which quantises x and A itself, at reduced
shapes and at decode sizes of the Mixtral-shaped layer (including the split-K
down projection)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_smoe_b200 as smoe
from sparse_mixture_experts_smoe_b200.inputs import WORKLOADS, make_mlp_inputs

from ._util import assert_close

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


def test_weight_quantisation_matches_the_oracle():
    g = torch.Generator(device="cuda").manual_seed(3)
    w = (torch.randn(3, 272, 200, generator=g, device="cuda") * 0.05).to(BF)
    w[1, :, 7] = 0  # an all-zero column: scale 1, codes 0
    codes, scales = smoe.smoe_quantize_weights_fp8(w)
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    rc, rs = oracle.quantize_weights_fp8(w.cpu())
    np.testing.assert_array_equal(scales.cpu().numpy(), rs)
    np.testing.assert_array_equal(oracle.e4m3_decode(codes.cpu().numpy()), oracle.e4m3_decode(rc))


FWD = {
    "swiglu_reduced": dict(T=300, d=272, f=400, E=6, k=2, act="swiglu", dtype="bf16"),
    "gelu_reduced": dict(T=257, d=144, f=528, E=5, k=2, act="gelu", dtype="bf16"),
    "zipf_reduced": dict(T=200, d=128, f=128, E=16, k=4, act="swiglu", dtype="bf16", zipf_s=1.2,
                         n_empty=3),
    "decode_t2_splitk": dict(T=2, d=272, f=1008, E=8, k=2, act="swiglu", dtype="bf16"),
}


def _run_fp8(cfg, inp):
    st = smoe.SMoEMLPState(cfg["T"], cfg["d"], cfg["f"], cfg["E"], cfg["k"], cfg["act"], BF, "cuda",
                           with_grad=False)
    w1q, s1 = smoe.smoe_quantize_weights_fp8(inp["w1"])
    w2q, s2 = smoe.smoe_quantize_weights_fp8(inp["w2"])
    smoe.smoe_mlp_fwd_fp8(st, inp["x"], inp["w_r"], inp["b_r"], w1q, s1, w2q, s2)
    torch.cuda.synchronize()
    assert smoe.smoe_check() == 0
    return st


def _check(cfg, inp, st, tokens=None):
    c = {n: (None if v is None else v.cpu()) for n, v in inp.items()}
    idx, gates = oracle.route(c["x"], c["w_r"], c["b_r"], cfg["k"])
    np.testing.assert_array_equal(st.topk_idx.cpu().numpy(), idx)
    ss, off = oracle.sort(idx, cfg["E"])
    np.testing.assert_array_equal(st.sorted_slot.cpu().numpy(), ss)
    w1q, s1 = oracle.quantize_weights_fp8(c["w1"])
    w2q, s2 = oracle.quantize_weights_fp8(c["w2"])
    ref = oracle.mlp_fwd_fp8(c["x"], w1q, s1, w2q, s2, cfg["act"], idx, gates, tokens=tokens,
                             want_a=True)
    toks = np.arange(cfg["T"]) if tokens is None else np.asarray(tokens)
    assert_close("y", st.y[torch.from_numpy(toks).long().cuda()], ref["y"], BF)
    inv = np.empty_like(ss)
    inv[ss] = np.arange(ss.size)
    slots = (toks[:, None] * cfg["k"] + np.arange(cfg["k"])[None, :]).ravel()
    assert_close("a", st.a[torch.from_numpy(inv[slots]).long().cuda()], ref["a"], BF)


@pytest.mark.parametrize("name", list(FWD))
def test_fp8_forward_every_element(name):
    cfg = FWD[name]
    inp = make_mlp_inputs(cfg, seed=5, device="cuda", with_dy=False)
    st = _run_fp8(cfg, inp)
    _check(cfg, inp, st)


@pytest.mark.parametrize("T", [1, 8])
def test_fp8_forward_mixtral_shape_decode(T):
    """The decode-sized FP8 forward of the Mixtral-shaped layer (d=4096, f=14336,
    E=8, k=2): routing bit for bit, every element of y and of A."""
    cfg = dict(WORKLOADS["mixtral_bf16_swiglu"], T=T)
    inp = make_mlp_inputs(cfg, seed=6, device="cuda", with_dy=False)
    st = _run_fp8(cfg, inp)
    _check(cfg, inp, st)


def test_fp8_forward_close_to_bf16_forward():
    """At the small workload's width the FP8 forward stays within a few percent of the
    bf16 forward on the same inputs (e4m3 keeps 3 mantissa bits)."""
    cfg = dict(WORKLOADS["small_bf16_gelu"], T=512)
    inp = make_mlp_inputs(cfg, seed=7, device="cuda", with_dy=False)
    st8 = _run_fp8(cfg, inp)
    st = smoe.SMoEMLPState(cfg["T"], cfg["d"], cfg["f"], cfg["E"], cfg["k"], cfg["act"], BF, "cuda",
                           with_grad=False)
    smoe.smoe_mlp_fwd(st, inp["x"], inp["w_r"], inp["b_r"], inp["w1"], inp["w2"])
    torch.cuda.synchronize()
    y8, y = st8.y.float(), st.y.float()
    assert float((y8 - y).abs().max() / y.abs().max()) < 0.08
