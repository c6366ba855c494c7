"""Thin Python binding of libsmoe.so (C ABI in ``include/smoe.h``).

Every function here has the name of the C entry point it calls and only
marshals arguments: it checks tensor shapes/dtypes/devices, allocates outputs and
the workspace with torch (device memory is torch's job here), and passes raw
pointers and the current CUDA stream.  All arithmetic runs in the CUDA kernels of
libsmoe.so.  There is no fallback: if the library cannot be loaded, every call
raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .inputs import WORKLOADS  # noqa: F401  (re-exported for bench/tests)

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libsmoe.so")
_lib = None

SMOE_OK = 0
F32, BF16 = 0, 1
ACT = {"gelu": 0, "swiglu": 1, "none": 2}
OP = {"sort": 0, "pl_fwd": 1, "pl_bwd": 2, "mlp_fwd": 3, "mlp_bwd": 4, "route_bwd": 5}

_c_int, _c_size, _vp = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p


class SmoeError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"smoe error {code}: {msg}")
        self.code = code


class MlpDesc(ctypes.Structure):
    _fields_ = [("T", _c_int), ("d", _c_int), ("f", _c_int), ("E", _c_int), ("k", _c_int),
                ("act", _c_int), ("dtype", _c_int)]


class MlpTensors(ctypes.Structure):
    _fields_ = [(n, _vp) for n in ("x", "w_r", "b_r", "w1", "w2", "y", "topk_idx", "gates",
                                   "sorted_slot", "expert_offsets", "h", "a", "dy", "dx", "dw1",
                                   "dw2", "dw_r", "db_r", "dgates", "workspace")] + \
               [("workspace_bytes", _c_size)]


class Fp8Weights(ctypes.Structure):
    _fields_ = [("w1q", _vp), ("s1", _vp), ("w2q", _vp), ("s2", _vp)]


def library_path() -> str:
    return _LIB_PATH


def lib():
    """Load libsmoe.so (building it in-tree first if it is missing and nvcc exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        from . import build as _build
        _build.build()
    L = ctypes.CDLL(_LIB_PATH)
    L.smoe_last_error.restype = ctypes.c_char_p
    L.smoe_version.restype = ctypes.c_char_p
    L.smoe_check.argtypes = [_vp]
    L.smoe_workspace_size.restype = _c_size
    L.smoe_workspace_size.argtypes = [_c_int] * 7
    L.smoe_route.argtypes = [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp]
    L.smoe_route_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _c_int,
                                 _vp, _vp, _vp, _vp, _c_size, _vp]
    L.smoe_sort.argtypes = [_vp, _c_int, _c_int, _c_int, _vp, _vp, _vp, _c_size, _vp]
    L.smoe_sort_static.argtypes = [_vp, _c_int, _c_int, _c_int, _vp, _vp, _vp]
    L.smoe_selftest_wait_timeout.argtypes = [_c_int, _vp]
    L.smoe_set_gemm_policy.argtypes = [_c_int]
    L.parallel_linear_fwd_workspace_size.restype = _c_size
    L.parallel_linear_fwd_workspace_size.argtypes = [_c_int] * 6
    L.parallel_linear_fwd.argtypes = [_vp, _c_int, _c_int, _vp, _c_int, _c_int, _vp, _vp, _c_int,
                                      _c_int, _c_int, _c_int, _vp, _c_int, _vp, _c_int, _vp,
                                      _c_size, _vp]
    L.parallel_linear_bwd_workspace_size.restype = _c_size
    L.parallel_linear_bwd_workspace_size.argtypes = [_c_int] * 11
    L.parallel_linear_bwd.argtypes = [_vp, _vp, _vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp,
                                      _c_int, _c_int, _c_int, _c_int, _vp, _c_int, _vp, _vp, _vp,
                                      _c_int, _vp, _c_size, _vp]
    L.smoe_quantize_weights_fp8.argtypes = [_vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp]
    L.smoe_mlp_fp8_workspace_size.restype = _c_size
    L.smoe_mlp_fp8_workspace_size.argtypes = [ctypes.POINTER(MlpDesc)]
    L.smoe_mlp_fwd_fp8.argtypes = [ctypes.POINTER(MlpDesc), ctypes.POINTER(MlpTensors),
                                   ctypes.POINTER(Fp8Weights), _vp]
    L.smoe_moa_attn_workspace_size.restype = _c_size
    L.smoe_moa_attn_workspace_size.argtypes = [_c_int] * 4
    L.smoe_moa_attn_fwd.argtypes = [_vp, _vp, _vp, _vp] + [_c_int] * 6 + [_vp, _vp, _vp, _c_size, _vp]
    L.smoe_moa_attn_bwd.argtypes = [_vp] * 7 + [_c_int] * 6 + [_vp] * 4 + [_c_size, _vp]
    L.smoe_mlp_workspace_size.restype = _c_size
    L.smoe_mlp_workspace_size.argtypes = [ctypes.POINTER(MlpDesc), _c_int]
    L.smoe_mlp_fwd.argtypes = [ctypes.POINTER(MlpDesc), ctypes.POINTER(MlpTensors), _vp]
    L.smoe_mlp_bwd.argtypes = [ctypes.POINTER(MlpDesc), ctypes.POINTER(MlpTensors), _vp]
    L.smoe_profile_begin.argtypes = [_c_int]
    L.smoe_profile_end.argtypes = []
    L.smoe_profile_entry.argtypes = [_c_int, ctypes.POINTER(ctypes.c_char_p),
                                     ctypes.POINTER(_c_int), ctypes.POINTER(ctypes.c_double)]
    _lib = L
    return L


def _check(rc: int):
    if rc != SMOE_OK:
        raise SmoeError(rc, lib().smoe_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _workspace(nbytes: int, device) -> torch.Tensor:
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


def smoe_check(stream=None) -> int:
    """Synchronise and return the device error status (0 = OK)."""
    return lib().smoe_check(_stream(stream))


def smoe_profile_begin(max_launches: int = 4096):
    """Start bracketing every library kernel launch with CUDA events."""
    _check(lib().smoe_profile_begin(max_launches))


def smoe_profile_end() -> dict:
    """Stop recording; {kernel name: (launches, total ms)} since smoe_profile_begin."""
    L = lib()
    n = L.smoe_profile_end()
    if n < 0:
        _check(n)
    out = {}
    for i in range(n):
        name, cnt, ms = ctypes.c_char_p(), _c_int(), ctypes.c_double()
        _check(L.smoe_profile_entry(i, ctypes.byref(name), ctypes.byref(cnt), ctypes.byref(ms)))
        out[name.value.decode()] = (cnt.value, ms.value)
    return out


def smoe_version() -> str:
    return lib().smoe_version().decode()


def smoe_workspace_size(op: str, T, k, E, d, f, dtype) -> int:
    dt = BF16 if dtype == torch.bfloat16 else F32
    return lib().smoe_workspace_size(OP[op], T, k, E, d, f, dt)


def smoe_route(x, w_r, b_r, k, topk_idx=None, gates=None, stream=None):
    T, d = x.shape
    E = w_r.shape[1]
    _need(x, "x")
    _need(w_r, "w_r", x.dtype, (d, E))
    if b_r is not None:
        _need(b_r, "b_r", torch.float32, (E,))
    if topk_idx is None:
        topk_idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
    if gates is None:
        gates = torch.empty((T, k), dtype=torch.float32, device=x.device)
    _check(lib().smoe_route(_ptr(x), _ptr(w_r), _ptr(b_r), T, d, E, k, _dt(x), _ptr(topk_idx),
                            _ptr(gates), _stream(stream)))
    return topk_idx, gates


def smoe_route_bwd(x, w_r, topk_idx, gates, dgates, dx=None, want_db=True, stream=None):
    """Router backward; accumulates into ``dx`` if given.  Returns (dw_r, db_r)."""
    T, d = x.shape
    E = w_r.shape[1]
    k = topk_idx.shape[1]
    for t, n in ((x, "x"), (w_r, "w_r"), (topk_idx, "topk_idx"), (gates, "gates"), (dgates, "dgates")):
        _need(t, n)
    dw_r = torch.empty((d, E), dtype=torch.float32, device=x.device)
    db_r = torch.empty((E,), dtype=torch.float32, device=x.device) if want_db else None
    ws = _workspace(smoe_workspace_size("route_bwd", T, k, E, d, 8, x.dtype), x.device)
    _check(lib().smoe_route_bwd(_ptr(x), _ptr(w_r), _ptr(topk_idx), _ptr(gates), _ptr(dgates), T,
                                d, E, k, _dt(x), _ptr(dx), _ptr(dw_r), _ptr(db_r), _ptr(ws),
                                ws.numel(), _stream(stream)))
    return dw_r, db_r


def smoe_sort(topk_idx, E, stream=None):
    _need(topk_idx, "topk_idx", torch.int32)
    T, k = topk_idx.shape
    ss = torch.empty((T * k,), dtype=torch.int32, device=topk_idx.device)
    off = torch.empty((E + 1,), dtype=torch.int32, device=topk_idx.device)
    ws = _workspace(lib().smoe_workspace_size(OP["sort"], T, k, E, 8, 8, 0), topk_idx.device)
    _check(lib().smoe_sort(_ptr(topk_idx), T, k, E, _ptr(ss), _ptr(off), _ptr(ws), ws.numel(),
                           _stream(stream)))
    return ss, off


def smoe_set_gemm_policy(policy: int):
    """Kernel-selection policy of the tensor-core GEMMs for later calls (0: one
    CTA per tile, the default; 1: CTA pairs and 4-warp gathers on long-K products
    over large expert slices; see smoe.h)."""
    _check(lib().smoe_set_gemm_policy(int(policy)))


def smoe_selftest_wait_timeout(limit_us: int, stream=None):
    """Run the library's bounded device wait on a barrier nothing completes; the
    next smoe_check returns SMOE_ERR_TIMEOUT (see smoe.h)."""
    _check(lib().smoe_selftest_wait_timeout(int(limit_us), _stream(stream)))


def smoe_sort_static(topk_idx, E, sorted_slot=None, expert_offsets=None, stream=None):
    """smoe_sort without a workspace: the library keeps the per-block counts in
    a fixed device array of its own (for callers that cannot allocate; see
    smoe_sort_static in smoe.h for the size limit and the no-overlap rule)."""
    _need(topk_idx, "topk_idx", torch.int32)
    T, k = topk_idx.shape
    if sorted_slot is None:
        sorted_slot = torch.empty((T * k,), dtype=torch.int32, device=topk_idx.device)
    if expert_offsets is None:
        expert_offsets = torch.empty((E + 1,), dtype=torch.int32, device=topk_idx.device)
    _check(lib().smoe_sort_static(_ptr(topk_idx), T, k, E, _ptr(sorted_slot),
                                  _ptr(expert_offsets), _stream(stream)))
    return sorted_slot, expert_offsets


def parallel_linear_fwd(x, w, sorted_slot, expert_offsets, fan_out, grouped_in, grouped_out,
                        gates=None, combine_k=0, y=None, stream=None):
    x_rows, K = x.shape
    E, K2, N = w.shape
    assert K2 == K
    S = sorted_slot.numel()
    _need(x, "x")
    _need(w, "w", x.dtype)
    _need(sorted_slot, "sorted_slot", torch.int32)
    _need(expert_offsets, "expert_offsets", torch.int32, (E + 1,))
    if gates is not None:
        _need(gates, "gates", torch.float32)
    rows = S // combine_k if combine_k > 0 else S
    if y is None:
        y = torch.empty((rows, N), dtype=x.dtype, device=x.device)
    ws = _workspace(lib().parallel_linear_fwd_workspace_size(S, K, N, E, combine_k, _dt(x)), x.device)
    _check(lib().parallel_linear_fwd(_ptr(x), x_rows, K, _ptr(w), N, E, _ptr(sorted_slot),
                                     _ptr(expert_offsets), S, fan_out, int(grouped_in),
                                     int(grouped_out), _ptr(gates), combine_k, _ptr(y), _dt(x),
                                     _ptr(ws), ws.numel(), _stream(stream)))
    return y


def parallel_linear_bwd(dy, x, w, sorted_slot, expert_offsets, fan_out, grouped_in, grouped_out,
                        gates=None, combine_k=0, want_dx=True, want_dw=True, want_dgates=False,
                        stream=None):
    x_rows, K = x.shape
    E, _, N = w.shape
    S = sorted_slot.numel()
    for t, n in ((dy, "dy"), (x, "x"), (w, "w")):
        _need(t, n)
    dx = torch.empty_like(x) if want_dx else None
    dw = torch.empty((E, K, N), dtype=torch.float32, device=x.device) if want_dw else None
    dg = torch.empty((S,), dtype=torch.float32, device=x.device) if want_dgates else None
    ws = _workspace(lib().parallel_linear_bwd_workspace_size(
        x_rows, S, K, N, E, fan_out, int(grouped_in), int(grouped_out), int(gates is not None),
        combine_k, _dt(x)), x.device)
    _check(lib().parallel_linear_bwd(_ptr(dy), _ptr(x), _ptr(w), x_rows, K, N, E, _ptr(sorted_slot),
                                     _ptr(expert_offsets), S, fan_out, int(grouped_in),
                                     int(grouped_out), _ptr(gates), combine_k, _ptr(dx), _ptr(dw),
                                     _ptr(dg), _dt(x), _ptr(ws), ws.numel(), _stream(stream)))
    return dx, dw, dg


def smoe_moa_attn_fwd(q, k, v, sorted_slot, kslots, L, heads, stream=None):
    """Mixture-of-Attention core forward: (o [T*kslots, heads*dh] grouped like q,
    lse [T*kslots, heads] fp32)."""
    S, W = q.shape
    T = k.shape[0]
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, q.dtype)
    _need(sorted_slot, "sorted_slot", torch.int32, (S,))
    o = torch.empty_like(q)
    lse = torch.empty((S, heads), dtype=torch.float32, device=q.device)
    ws = _workspace(lib().smoe_moa_attn_workspace_size(T, kslots, heads, 0), q.device)
    _check(lib().smoe_moa_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(sorted_slot), T, L, kslots, heads,
                                   W // heads, _dt(q), _ptr(o), _ptr(lse), _ptr(ws), ws.numel(),
                                   _stream(stream)))
    return o, lse


def smoe_moa_attn_bwd(q, k, v, o, lse, dout, sorted_slot, kslots, L, heads, stream=None):
    """Mixture-of-Attention core backward: (dq grouped like q, dk, dv like k, v)."""
    S, W = q.shape
    T = k.shape[0]
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _need(t, n, q.dtype)
    _need(lse, "lse", torch.float32, (S, heads))
    _need(sorted_slot, "sorted_slot", torch.int32, (S,))
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = _workspace(lib().smoe_moa_attn_workspace_size(T, kslots, heads, 1), q.device)
    _check(lib().smoe_moa_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout),
                                   _ptr(sorted_slot), T, L, kslots, heads, W // heads, _dt(q),
                                   _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(),
                                   _stream(stream)))
    return dq, dk, dv


def smoe_quantize_weights_fp8(w, stream=None):
    """W [E, K, N] bf16 -> (codes uint8 [E, N, K] e4m3, K-major; scales fp32 [E, N])."""
    _need(w, "w", torch.bfloat16)
    E, K, N = w.shape
    codes = torch.empty((E, N, K), dtype=torch.uint8, device=w.device)
    scales = torch.empty((E, N), dtype=torch.float32, device=w.device)
    _check(lib().smoe_quantize_weights_fp8(_ptr(w), E, K, N, BF16, _ptr(codes), _ptr(scales),
                                           _stream(stream)))
    return codes, scales


def smoe_mlp_fwd_fp8(st, x, w_r, b_r, w1q, s1, w2q, s2, stream=None):
    """FP8 forward into the state's y, h, a and routing buffers (see smoe.h)."""
    for t_, n in ((x, "x"), (w_r, "w_r")):
        _need(t_, n, torch.bfloat16)
    for t_, n in ((w1q, "w1q"), (w2q, "w2q")):
        _need(t_, n, torch.uint8)
    for t_, n in ((s1, "s1"), (s2, "s2")):
        _need(t_, n, torch.float32)
    d = st.desc
    ws_bytes = lib().smoe_mlp_fp8_workspace_size(ctypes.byref(d))
    if ws_bytes == 0:
        _check(-1)
    ws = _workspace(ws_bytes, x.device)
    t = st.tensors(x, w_r, b_r, None, None)
    t.workspace = ws.data_ptr()
    t.workspace_bytes = ws.numel()
    w8 = Fp8Weights(w1q.data_ptr(), s1.data_ptr(), w2q.data_ptr(), s2.data_ptr())
    _check(lib().smoe_mlp_fwd_fp8(ctypes.byref(d), ctypes.byref(t), ctypes.byref(w8), _stream(stream)))


class SMoEMLPState:
    """Buffers of one SMoE MLP layer call: parameters, saved forward outputs and
    gradients, all allocated by torch once and reused across steps."""

    def __init__(self, T, d, f, E, k, act, dtype, device, with_grad=True):
        self.desc = MlpDesc(T, d, f, E, k, ACT[act], BF16 if dtype == torch.bfloat16 else F32)
        m = 2 if act == "swiglu" else 1
        dev = torch.device(device)
        S = T * k
        e = lambda *s, dt=dtype: torch.empty(s, dtype=dt, device=dev)  # noqa: E731
        self.y = e(T, d)
        self.topk_idx = e(T, k, dt=torch.int32)
        self.gates = e(T, k, dt=torch.float32)
        self.sorted_slot = e(S, dt=torch.int32)
        self.expert_offsets = e(E + 1, dt=torch.int32)
        self.h = e(S, m * f)
        self.a = e(S, f)
        if with_grad:
            self.dx = e(T, d)
            self.dw1 = e(E, d, m * f, dt=torch.float32)
            self.dw2 = e(E, f, d, dt=torch.float32)
            self.dw_r = e(d, E, dt=torch.float32)
            self.db_r = e(E, dt=torch.float32)
            self.dgates = e(T, k, dt=torch.float32)
        L = lib()
        nbytes = max(L.smoe_mlp_workspace_size(ctypes.byref(self.desc), 0),
                     L.smoe_mlp_workspace_size(ctypes.byref(self.desc), 1) if with_grad else 0)
        self.workspace = _workspace(nbytes, dev)

    def tensors(self, x, w_r, b_r, w1, w2, dy=None) -> MlpTensors:
        t = MlpTensors()
        ptr = lambda v: None if v is None else v.data_ptr()  # noqa: E731
        t.x, t.w_r, t.b_r, t.w1, t.w2 = ptr(x), ptr(w_r), ptr(b_r), ptr(w1), ptr(w2)
        for n in ("y", "topk_idx", "gates", "sorted_slot", "expert_offsets", "h", "a"):
            setattr(t, n, getattr(self, n).data_ptr())
        if dy is not None:
            t.dy = dy.data_ptr()
            for n in ("dx", "dw1", "dw2", "dw_r", "db_r", "dgates"):
                setattr(t, n, getattr(self, n).data_ptr())
        t.workspace = self.workspace.data_ptr()
        t.workspace_bytes = self.workspace.numel()
        return t


def _check_mlp_params(st, x, w_r, b_r, w1, w2):
    D = st.desc
    m = 2 if D.act == ACT["swiglu"] else 1
    dt = torch.bfloat16 if D.dtype == BF16 else torch.float32
    _need(x, "x", dt, (D.T, D.d))
    _need(w_r, "w_r", dt, (D.d, D.E))
    if b_r is not None:
        _need(b_r, "b_r", torch.float32, (D.E,))
    _need(w1, "w1", dt, (D.E, D.d, m * D.f))
    _need(w2, "w2", dt, (D.E, D.f, D.d))


def smoe_mlp_fwd(st: SMoEMLPState, x, w_r, b_r, w1, w2, stream=None):
    _check_mlp_params(st, x, w_r, b_r, w1, w2)
    t = st.tensors(x, w_r, b_r, w1, w2)
    _check(lib().smoe_mlp_fwd(ctypes.byref(st.desc), ctypes.byref(t), _stream(stream)))
    return st.y


def smoe_mlp_bwd(st: SMoEMLPState, x, w_r, b_r, w1, w2, dy, stream=None):
    _check_mlp_params(st, x, w_r, b_r, w1, w2)
    _need(dy, "dy", x.dtype, x.shape)
    t = st.tensors(x, w_r, b_r, w1, w2, dy)
    _check(lib().smoe_mlp_bwd(ctypes.byref(st.desc), ctypes.byref(t), _stream(stream)))
    return st.dx
