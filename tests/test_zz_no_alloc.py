"""smoe_sort_static: the sort for callers that cannot allocate device memory.

Such callers (a runtime that plans all memory up front, code running during
CUDA-graph capture) cannot hand the library a workspace, so this entry point
keeps its scratch in a fixed device array of the library.  The test calls it
through the C ABI and checks it bit for bit against the oracle's stable sort and
against smoe_sort (which uses a caller workspace), on calls in a row with
different routings, so that state left in the shared array by one call cannot
leak into the next; one case fits the single-block path (at most 4096 slots and
128 experts), the others take the three-kernel path.  This file
is collected last on purpose; it must pass alone in a fresh process as well.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import sparse_mixture_experts_smoe_b200 as smoe

pytestmark = pytest.mark.gpu


def _routing(T, k, E, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    idx = torch.randint(0, E, (T, k), generator=g, device="cuda", dtype=torch.int32)
    idx[: T // 5] = E - 1  # one heavy expert and a ragged tail of blocks
    return idx


def test_sort_static_matches_workspace_sort_on_consecutive_calls():
    cases = [(5000, 2, 8, 1), (3001, 8, 64, 2), (1000, 2, 8, 4), (5000, 2, 8, 3)]
    for T, k, E, seed in cases:
        idx = _routing(T, k, E, seed)
        ref_ss, ref_off = oracle.sort(idx.cpu(), E)
        ws_ss, ws_off = smoe.smoe_sort(idx, E)
        ss, off = smoe.smoe_sort_static(idx, E)
        torch.cuda.synchronize()
        assert smoe.smoe_check() == 0
        np.testing.assert_array_equal(off.cpu().numpy(), ref_off)
        np.testing.assert_array_equal(ss.cpu().numpy(), ref_ss)
        np.testing.assert_array_equal(ws_off.cpu().numpy(), ref_off)
        np.testing.assert_array_equal(ws_ss.cpu().numpy(), ref_ss)


def test_sort_static_rejects_sizes_beyond_its_scratch():
    L = smoe.lib()
    idx = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    out = torch.zeros(8, dtype=torch.int32, device="cuda")
    # ceil(T*k/4096) * E = 256 * 1024 > 65536 entries: refused before any launch
    rc = L.smoe_sort_static(ctypes.c_void_p(idx.data_ptr()), 1 << 19, 2, 1024,
                            ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(out.data_ptr()), None)
    assert rc == -1
    assert b"static scratch" in L.smoe_last_error()
