"""CPU-only checks of the C-ABI library: it loads, exports every entry point that
include/smoe.h declares, and rejects bad arguments on the host before touching
the GPU."""
import ctypes
import os
import re

import pytest

import sparse_mixture_experts_smoe_b200 as smoe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[a-zA-Z_][a-zA-Z0-9_]*\s*\*?\s*([a-z_][a-z0-9_]*)\s*\(",
                             src, flags=re.M):
            names.add(m.group(1))
    return names


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ("smoe_route", "smoe_route_bwd", "smoe_sort", "parallel_linear_fwd",
              "parallel_linear_bwd", "smoe_mlp_fwd", "smoe_mlp_bwd", "smoe_check",
              "smoe_last_error", "smoe_workspace_size"):
        assert n in names, n


def test_library_exports_every_declared_symbol():
    L = smoe.lib()
    missing = [n for n in sorted(_declared_functions()) if not hasattr(L, n)]
    assert not missing, missing


def test_version_and_empty_error():
    assert "sm_100a" in smoe.smoe_version()


V = ctypes.c_void_p
FAKE = V(0x10000)  # never dereferenced: validation fails or T == 0 returns first


def test_route_rejects_bad_arguments_on_host():
    L = smoe.lib()
    # k > E
    assert L.smoe_route(FAKE, FAKE, None, 4, 8, 2, 3, 1, FAKE, FAKE, None) == -1
    assert b"k" in L.smoe_last_error()
    # d not a multiple of 8
    assert L.smoe_route(FAKE, FAKE, None, 4, 12, 8, 2, 1, FAKE, FAKE, None) == -1
    # NULL x
    assert L.smoe_route(None, FAKE, None, 4, 8, 8, 2, 1, FAKE, FAKE, None) == -1
    # misaligned x
    assert L.smoe_route(V(0x10004), FAKE, None, 4, 8, 8, 2, 1, FAKE, FAKE, None) == -1
    # bad dtype
    assert L.smoe_route(FAKE, FAKE, None, 4, 8, 8, 2, 7, FAKE, FAKE, None) == -1
    # T == 0 is a no-op that touches nothing
    assert L.smoe_route(None, None, None, 0, 8, 8, 2, 1, None, None, None) == 0


def test_parallel_linear_rejects_bad_flags_on_host():
    L = smoe.lib()
    args = dict(x=FAKE, x_rows=8, K=16, w=FAKE, N=16, E=2, ss=FAKE, off=FAKE, S=8, fan=1,
                gi=1, go=0, gates=None, ck=2, y=FAKE, dt=1, ws=FAKE, wsb=1 << 20, st=None)

    def call(**kw):
        a = dict(args, **kw)
        return L.parallel_linear_fwd(a["x"], a["x_rows"], a["K"], a["w"], a["N"], a["E"], a["ss"],
                                     a["off"], a["S"], a["fan"], a["gi"], a["go"], a["gates"],
                                     a["ck"], a["y"], a["dt"], a["ws"], a["wsb"], a["st"])

    assert call(go=1) == -1                 # combine with a grouped output
    assert call(S=9) == -1                  # num_slots not divisible by combine_k
    assert call(K=12) == -1                 # K not a multiple of 8
    assert call(gi=1, x_rows=4) == -1       # grouped input needs x_rows == num_slots
    assert call(gi=0, fan=1, x_rows=4) == -1  # x_rows * fan_out < num_slots
    assert call(fan=0) == -1
    assert call(wsb=16) == -1               # workspace too small for the combine buffer
    assert call(S=0, x_rows=0, gi=0) == 0   # empty problem
    # dgates without gates
    assert L.parallel_linear_bwd(FAKE, FAKE, FAKE, 8, 16, 16, 2, FAKE, FAKE, 8, 1, 1, 0, None, 0,
                                 FAKE, FAKE, FAKE, 1, FAKE, 1 << 20, None) == -1


def test_sort_and_mlp_reject_bad_arguments_on_host():
    L = smoe.lib()
    assert L.smoe_sort(FAKE, 4, 2, 0, FAKE, FAKE, FAKE, 1024, None) == -1       # E == 0
    assert L.smoe_sort(FAKE, 4, 2, 8, FAKE, FAKE, None, 0, None) == -1          # no workspace
    d = smoe.MlpDesc(16, 64, 64, 4, 5, 1, 1)                                    # k > E
    t = smoe.MlpTensors()
    assert L.smoe_mlp_fwd(ctypes.byref(d), ctypes.byref(t), None) == -1
    d = smoe.MlpDesc(16, 64, 64, 4, 2, 7, 1)                                    # bad act
    assert L.smoe_mlp_fwd(ctypes.byref(d), ctypes.byref(t), None) == -1
    d = smoe.MlpDesc(16, 64, 64, 4, 2, 1, 1)                                    # NULL tensors
    assert L.smoe_mlp_fwd(ctypes.byref(d), ctypes.byref(t), None) == -1
    assert b"NULL" in L.smoe_last_error()


def test_workspace_queries_are_consistent():
    L = smoe.lib()
    for T, k, E, d, f in [(256, 2, 8, 128, 256), (16384, 2, 8, 4096, 14336), (16384, 8, 64, 2048, 512)]:
        for dt in (0, 1):
            desc = smoe.MlpDesc(T, d, f, E, k, 1, dt)
            fwd = L.smoe_mlp_workspace_size(ctypes.byref(desc), 0)
            bwd = L.smoe_mlp_workspace_size(ctypes.byref(desc), 1)
            # forward: sort counts + one [T*k, d] combine buffer of the layer's dtype,
            # nothing the size of a grouped copy of x is needed beyond that
            es = 4 if dt == 0 else 2
            assert fwd >= T * k * d * es and fwd < T * k * d * es + (1 << 20)
            assert bwd > fwd
            assert L.smoe_workspace_size(3, T, k, E, d, f, dt) == fwd
            assert L.smoe_workspace_size(4, T, k, E, d, f, dt) == bwd


@pytest.mark.parametrize("T,k,E,d", [(1, 1, 1, 8), (1, 1, 128, 8), (3, 2, 128, 8), (37, 3, 3, 40),
                                     (256, 2, 8, 128), (16384, 8, 64, 2048), (16384, 2, 8, 4096)])
def test_router_backward_fits_the_mlp_backward_workspace(T, k, E, d):
    """smoe_route_bwd's header promises that the MLP backward's workspace size covers
    it (its sort, slot order, dl and the weight gradient's run partials)."""
    L = smoe.lib()
    for dt in (0, 1):
        rb = L.smoe_workspace_size(5, T, k, E, d, 8, dt)
        assert 0 < rb <= L.smoe_workspace_size(4, T, k, E, d, 8, dt)
        # run partials: (T*k / R + E) rows of d + 1 floats with R >= 32, nothing per
        # (token, expert)
        assert rb < T * k * 16 + ((T * k + 31) // 32 + E) * (d + 1) * 4 + 4096 + 256 * 8


def test_workspaces_hold_no_copy_of_token_rows():
    """The library never allocates, so a grouped or padded copy of x or dY would have
    to live in its workspace.  Mixtral-shaped sizes: the forward workspace is exactly
    the sort counts, one int32 per slot (its grouped row) and one bf16 [T*k, d]
    buffer (the k-way combine's gated slot rows); what the backward needs beyond its
    documented large buffers (dH, gA and the dx slot rows) is far smaller than
    another bf16 [T*k, d] copy."""
    import ctypes
    import sparse_mixture_experts_smoe_b200 as smoe
    T, d, f, E, k = 16384, 4096, 14336, 8, 2
    S = T * k
    L = smoe.lib()
    a256 = lambda n: (n + 255) // 256 * 256  # noqa: E731
    sort = L.smoe_workspace_size(0, T, k, E, d, f, 1)
    desc = smoe.MlpDesc(T, d, f, E, k, smoe.ACT["swiglu"], smoe.BF16)
    fwd = L.smoe_mlp_workspace_size(ctypes.byref(desc), 0)
    bwd = L.smoe_mlp_workspace_size(ctypes.byref(desc), 1)
    assert fwd == a256(sort) + a256(S * 4) + a256(S * d * 2)
    # backward: dH [T*k, 2f], g*A [T*k, f] (dW2's gated operand) and the dx slot
    # rows [T*k, d]; the rest is small
    big = a256(S * 2 * f * 2) + a256(S * f * 2) + a256(S * d * 2)
    assert 0 < bwd - big < S * d * 2 // 4


def test_decode_workspace_holds_the_split_k_partials():
    """A one-token Mixtral-shaped forward splits the down projection's K four ways (2
    experts x 16 N tiles cannot fill 148 SMs): its workspace is the sort counts, the
    grouped row of each slot, the bf16 slot rows and 4 fp32 partial copies of them.
    From 8 tokens on, the tiles can fill the GPU and no partials are reserved."""
    import ctypes
    import sparse_mixture_experts_smoe_b200 as smoe
    L = smoe.lib()
    a256 = lambda n: (n + 255) // 256 * 256  # noqa: E731
    d, f, E, k = 4096, 14336, 8, 2
    for T, splits in ((1, 4), (8, 1)):
        S = T * k
        desc = smoe.MlpDesc(T, d, f, E, k, smoe.ACT["swiglu"], smoe.BF16)
        fwd = L.smoe_mlp_workspace_size(ctypes.byref(desc), 0)
        sort = L.smoe_workspace_size(0, T, k, E, d, f, 1)
        part = a256(splits * S * d * 4) if splits > 1 else 0
        assert fwd == a256(sort) + a256(S * 4) + a256(S * d * 2) + part


def test_limits_are_stated_and_enforced_per_entry_point():
    """Each entry point's size limit (smoe.h): the largest allowed value passes host
    validation (T == 0, so nothing runs), the next one is refused before any launch."""
    L = smoe.lib()
    hdr = open(os.path.join(ROOT, "include", "smoe.h")).read()
    lim = {n: int(re.search(r"#define %s (\d+)" % n, hdr).group(1))
           for n in ("SMOE_MAX_ROUTED_EXPERTS", "SMOE_MAX_TOPK", "SMOE_MAX_EXPERTS")}
    Er, Kmax, Emax = lim["SMOE_MAX_ROUTED_EXPERTS"], lim["SMOE_MAX_TOPK"], lim["SMOE_MAX_EXPERTS"]
    # router: E and k
    assert L.smoe_route(None, None, None, 0, 8, Er, Kmax, 1, None, None, None) == 0
    assert L.smoe_route(None, None, None, 0, 8, Er + 1, 2, 1, None, None, None) == -1
    assert L.smoe_route(None, None, None, 0, 8, Er, Kmax + 1, 1, None, None, None) == -1
    # router backward: same limits (T == 0 with valid sizes only zeroes the outputs,
    # which needs a device, so the boundary is checked on the refusals)
    args = (FAKE, FAKE, FAKE, FAKE, FAKE, 4, 8)
    assert L.smoe_route_bwd(*args, Er + 1, 2, 1, None, FAKE, None, FAKE, 1 << 20, None) == -1
    assert L.smoe_route_bwd(*args, Er, Kmax + 1, 1, None, FAKE, None, FAKE, 1 << 20, None) == -1
    # the MLP: E and k, through its workspace query (0 = refused)
    ok = smoe.MlpDesc(16, 64, 64, Er, Kmax, 1, 1)
    assert L.smoe_mlp_workspace_size(ctypes.byref(ok), 1) > 0
    for bad in (smoe.MlpDesc(16, 64, 64, Er + 1, 2, 1, 1), smoe.MlpDesc(16, 64, 64, Er, Kmax + 1, 1, 1)):
        assert L.smoe_mlp_workspace_size(ctypes.byref(bad), 1) == 0
        assert L.smoe_mlp_fwd(ctypes.byref(bad), ctypes.byref(smoe.MlpTensors()), None) == -1
    # sort and the allocation-free sort: E
    assert L.smoe_sort(FAKE, 4, 2, Emax + 1, FAKE, FAKE, FAKE, 1 << 20, None) == -1
    assert L.smoe_sort_static(FAKE, 4, 2, Emax + 1, FAKE, FAKE, None) == -1
    assert L.smoe_sort(FAKE, 4, 2, Emax, FAKE, FAKE, None, 0, None) == -1  # passes E, fails on ws
    assert b"workspace" in L.smoe_last_error()
    # ParallelLinear: E (the empty problem with E at the limit is a no-op)
    pl = lambda E, S: L.parallel_linear_fwd(FAKE, S, 16, FAKE, 16, E, FAKE, FAKE, S, 1, 1, 1,  # noqa: E731
                                            None, 0, FAKE, 1, None, 0, None)
    assert pl(Emax, 0) == 0
    assert pl(Emax + 1, 0) == -1


def test_slot_count_overflow_is_refused():
    """T*k beyond int32 is refused on the host by every entry point that takes T and k."""
    L = smoe.lib()
    T, k = (1 << 30), 4
    assert L.smoe_route(FAKE, FAKE, None, T, 8, 8, k, 1, FAKE, FAKE, None) == -1
    assert L.smoe_sort(FAKE, T, k, 8, FAKE, FAKE, FAKE, 1 << 20, None) == -1
    assert L.smoe_sort_static(FAKE, T, k, 8, FAKE, FAKE, None) == -1
    assert L.smoe_route_bwd(FAKE, FAKE, FAKE, FAKE, FAKE, T, 8, 8, k, 1, None, FAKE, None, FAKE,
                            1 << 20, None) == -1
    assert L.smoe_workspace_size(0, T, k, 8, 8, 8, 1) == 0
    d = smoe.MlpDesc(T, 64, 64, 8, k, 1, 1)
    assert L.smoe_mlp_workspace_size(ctypes.byref(d), 0) == 0


@pytest.mark.parametrize("grouped_in,fan_out", [(1, 1), (0, 4), (0, 1)])
def test_gated_parallel_linear_backward_adds_no_copy_of_x(grouped_in, fan_out):
    """With gates, the ParallelLinear backward's workspace grows only by the gate
    gradient's per-column-tile partials ([num_slots, ceil(K / tile)] fp32): dW's
    gate multiplies x's rows inside the dW kernel, so no [num_slots, K] gated or
    grouped copy of x exists (the MoA shapes: 32768 slots, K = 2048, N = 512)."""
    L = smoe.lib()
    S, K, N, E = 32768, 2048, 512, 16
    x_rows = S if (grouped_in or fan_out == 1) else S // fan_out
    a256 = lambda n: (n + 255) // 256 * 256  # noqa: E731
    for dt, tile in ((1, 256), (0, 64)):
        gated = L.parallel_linear_bwd_workspace_size(x_rows, S, K, N, E, fan_out, grouped_in, 0, 1, 0, dt)
        plain = L.parallel_linear_bwd_workspace_size(x_rows, S, K, N, E, fan_out, grouped_in, 0, 0, 0, dt)
        assert gated - plain == a256(S * ((K + tile - 1) // tile) * 4)
        es = 2 if dt == 1 else 4
        # the only [num_slots, K] buffer is the dx slot rows of a fan-out combine
        combine = a256(S * K * es) + a256(S * 4) if (not grouped_in and fan_out > 1) else 0
        assert plain == combine


def test_gemm_policy_accepts_only_its_values():
    L = smoe.lib()
    assert L.smoe_set_gemm_policy(2) == -1 and b"policy" in L.smoe_last_error()
    assert L.smoe_set_gemm_policy(-1) == -1
    assert L.smoe_set_gemm_policy(1) == 0
    assert L.smoe_set_gemm_policy(0) == 0
