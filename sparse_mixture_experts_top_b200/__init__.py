"""Python binding of libmoe_b200.so, the sm_100a hard-routed sparse MoE
layer forward.

Argument marshalling only: every function here checks shapes and dtypes,
allocates outputs with PyTorch on the inputs' device, passes raw device
pointers and the current CUDA stream to the C ABI (``include/moe.h``), and
raises on a non-OK status. All arithmetic runs in the library's CUDA
kernels; there is no CPU path. Importing this module fails loudly if the
library is missing or cannot be loaded.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_RANGE = range(7)
F32, BF16, F16 = 0, 1, 2
W_F32, W_BF16, W_Q4G64 = 0, 1, 2
REGIME_AUTO, REGIME_GEMV, REGIME_TC = 0, 1, 2

EXPORTS = ("moe_route", "moe_topk", "moe_sort_rows_workspace", "moe_sort_rows",
           "moe_sort_rows_noalloc", "moe_sort_block_m",
           "moe_grouped_swiglu_workspace", "moe_grouped_swiglu", "moe_grouped_down",
           "moe_combine", "moe_forward_workspace", "moe_pack_gate_up",
           "moe_forward", "moe_forward_layout", "moe_device_status", "moe_status_str",
           "moe_version", "moe_set_wait_cycles", "moe_selftest_wait_timeout")


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_str(status)} (status {status})")
        self.status = status


class Experts(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("E", ctypes.c_int32), ("d", ctypes.c_int32),
                ("F", ctypes.c_int32), ("w_gu", ctypes.c_void_p), ("s_gu", ctypes.c_void_p),
                ("b_gu", ctypes.c_void_p), ("w_dn", ctypes.c_void_p), ("s_dn", ctypes.c_void_p),
                ("b_dn", ctypes.c_void_p), ("act", ctypes.c_int32)]


class WsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("logits", "topk_idx", "topk_w", "order", "inv_order", "row_map", "counts",
                 "row_off", "tile_off", "sort_ws", "h", "ys", "x16", "total")] + \
               [("regime", ctypes.c_int32), ("BM", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python sparse_mixture_experts_top_b200/build.py` (needs nvcc)")
    L = ctypes.CDLL(LIB_PATH)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.moe_route.argtypes = [P, I, P, P, I, I, I, I, P, P, P, P]
    L.moe_topk.argtypes = [P, I, I, I, P, P, P]
    L.moe_sort_rows_workspace.argtypes = [I, I, I]
    L.moe_sort_rows_workspace.restype = S
    L.moe_sort_rows.argtypes = [P, I, I, I, I, P, P, P, P, P, P, P, S, P]
    L.moe_grouped_swiglu_workspace.argtypes = [I, I, I, I]
    L.moe_grouped_swiglu_workspace.restype = S
    L.moe_grouped_swiglu.argtypes = [P, I, P, P, P, I, I, I, ctypes.POINTER(Experts), P, P, S, I,
                                     P]
    L.moe_grouped_down.argtypes = [P, I, P, P, I, I, I, ctypes.POINTER(Experts), P, I, P]
    L.moe_combine.argtypes = [P, P, P, I, I, I, I, P, P]
    L.moe_forward_workspace.argtypes = [I, I, I, I, I, I, I, I]
    L.moe_forward_workspace.restype = S
    L.moe_forward.argtypes = [P, I, P, P, ctypes.POINTER(Experts), I, I, P, P, S, I, P]
    L.moe_forward_layout.argtypes = [I, I, I, I, I, I, I, I, ctypes.POINTER(WsLayout)]
    L.moe_sort_block_m.argtypes = []
    L.moe_sort_block_m.restype = ctypes.c_int
    L.moe_sort_rows_noalloc.argtypes = [P, I, I, I, I, P, P, P, P, P, P, P]
    L.moe_pack_gate_up.argtypes = [I, I, I, I, P, P, P, P, P, P, P, P, P, P]
    L.moe_pack_gate_up.restype = ctypes.c_int
    L.moe_device_status.argtypes = []
    L.moe_set_wait_cycles.argtypes = [ctypes.c_longlong]
    L.moe_set_wait_cycles.restype = ctypes.c_int
    L.moe_selftest_wait_timeout.argtypes = [I, ctypes.c_longlong, P, P]
    L.moe_selftest_wait_timeout.restype = ctypes.c_int
    L.moe_status_str.argtypes = [I]
    L.moe_status_str.restype = ctypes.c_char_p
    L.moe_version.restype = ctypes.c_char_p
    for name in ("moe_route", "moe_topk", "moe_sort_rows", "moe_sort_rows_noalloc",
                 "moe_grouped_swiglu",
                 "moe_grouped_down", "moe_combine", "moe_forward", "moe_forward_layout",
                 "moe_device_status"):
        getattr(L, name).restype = ctypes.c_int
    return L


lib = _load()


def status_str(s: int) -> str:
    return lib.moe_status_str(s).decode()


def version() -> str:
    return lib.moe_version().decode()


def _check(st: int, what: str):
    if st != OK:
        raise MoeError(st, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


_DT = {torch.float32: F32, torch.bfloat16: BF16, torch.float16: F16}


def _dt_of(dtype) -> int:
    if dtype not in _DT:
        raise TypeError(f"activations must be bfloat16, float16 or float32, got {dtype}")
    return _DT[dtype]


def _dt(t: torch.Tensor) -> int:
    return _dt_of(t.dtype)


def _dev(*ts):
    for t in ts:
        if t is not None and (t.device.type != "cuda" or not t.is_contiguous()):
            raise ValueError("inputs must be contiguous CUDA tensors")


W_Q4G32, W_Q4G128, W_Q8G64 = 3, 4, 5
_FMT = {"f32": W_F32, "bf16": W_BF16, "q4": W_Q4G64, "q4g32": W_Q4G32, "q4g128": W_Q4G128,
        "q8": W_Q8G64}
ACT_SWIGLU, ACT_GEGLU_TANH = 0, 1
_ACT = {"swiglu": ACT_SWIGLU, "geglu": ACT_GEGLU_TANH}


def experts_struct(ex) -> Experts:
    """C view of an expert-weight set (any object with fmt, E, d, F, w_gu,
    s_gu, b_gu, w_dn, s_dn, b_dn, tensors on the device; act, "swiglu" or
    "geglu", defaults to "swiglu")."""
    _dev(ex.w_gu, ex.w_dn, ex.s_gu, ex.b_gu, ex.s_dn, ex.b_dn)
    fmt = _FMT[ex.fmt] if isinstance(ex.fmt, str) else int(ex.fmt)
    act = getattr(ex, "act", "swiglu")
    act = _ACT[act] if isinstance(act, str) else int(act)
    return Experts(fmt, ex.E, ex.d, ex.F, _ptr(ex.w_gu), _ptr(ex.s_gu), _ptr(ex.b_gu),
                   _ptr(ex.w_dn), _ptr(ex.s_dn), _ptr(ex.b_dn), act)


# ------------------------------------------------------------------ stages

def route(x, w_router, router_bias, k, stream=None):
    """-> (logits fp32 [T,E], topk_idx int32 [T,k], topk_w fp32 [T,k])"""
    _dev(x, w_router, router_bias)
    T, d = x.shape
    E = w_router.shape[0]
    dev = x.device
    logits = torch.empty(T, E, dtype=torch.float32, device=dev)
    idx = torch.empty(T, k, dtype=torch.int32, device=dev)
    w = torch.empty(T, k, dtype=torch.float32, device=dev)
    _check(lib.moe_route(_ptr(x), _dt(x), _ptr(w_router), _ptr(router_bias), T, d, E, k,
                         _ptr(logits), _ptr(idx), _ptr(w), _stream(stream)), "moe_route")
    return logits, idx, w


def topk(logits, k, stream=None):
    """-> (topk_idx int32 [T,k], topk_w fp32 [T,k]) from fp32 logits [T,E]"""
    _dev(logits)
    T, E = logits.shape
    idx = torch.empty(T, k, dtype=torch.int32, device=logits.device)
    w = torch.empty(T, k, dtype=torch.float32, device=logits.device)
    _check(lib.moe_topk(_ptr(logits), T, E, k, _ptr(idx), _ptr(w), _stream(stream)), "moe_topk")
    return idx, w


@dataclass
class SortTables:
    order: torch.Tensor
    inv_order: torch.Tensor
    row_map: torch.Tensor
    counts: torch.Tensor
    row_off: torch.Tensor
    tile_off: torch.Tensor
    BM: int


def sort_rows(topk_idx, E, BM, stream=None) -> SortTables:
    _dev(topk_idx)
    T, k = topk_idx.shape
    R = T * k
    dev = topk_idx.device
    u32 = lambda n: torch.empty(n, dtype=torch.uint32, device=dev)
    i32 = lambda n: torch.empty(n, dtype=torch.int32, device=dev)
    order, inv, rmap = u32(R), u32(R), u32(R)
    counts, roff, toff = i32(E), i32(E + 1), i32(E + 1)
    nws = lib.moe_sort_rows_workspace(T, k, E)
    ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=dev)
    _check(lib.moe_sort_rows(_ptr(topk_idx), T, k, E, BM, _ptr(order), _ptr(inv), _ptr(rmap),
                             _ptr(counts), _ptr(roff), _ptr(toff), _ptr(ws), nws,
                             _stream(stream)), "moe_sort_rows")
    return SortTables(order, inv, rmap, counts, roff, toff, BM)


def grouped_swiglu(x, tables: SortTables, k, experts, regime=REGIME_AUTO, ws=None, stream=None):
    """-> h [T*k, F]: fp16 for bf16 or fp16 x, fp32 for fp32 x"""
    _dev(x)
    T = x.shape[0]
    ex = experts_struct(experts)
    hdt = torch.float32 if x.dtype == torch.float32 else torch.float16
    h = torch.empty(T * k, experts.F, dtype=hdt, device=x.device)
    nws = lib.moe_grouped_swiglu_workspace(T, k, experts.d, _dt(x))
    if ws is None:
        ws = torch.empty(max(nws, 16), dtype=torch.uint8, device=x.device)
    _check(lib.moe_grouped_swiglu(_ptr(x), _dt(x), _ptr(tables.row_map), _ptr(tables.row_off),
                                  _ptr(tables.tile_off), tables.BM, T, k, ctypes.byref(ex),
                                  _ptr(h), _ptr(ws), ws.numel(), regime, _stream(stream)),
           "moe_grouped_swiglu")
    return h


def grouped_down(h, tables: SortTables, T, k, experts, regime=REGIME_AUTO, stream=None,
                 dtype=None):
    """-> ys [T*k, d]: fp16 for 16-bit activations (fp16 h), fp32 for fp32.
    `dtype` is the layer's activation type (torch.bfloat16, torch.float16 or
    torch.float32); it may be left out for fp32 h, which only fp32
    activations produce."""
    _dev(h)
    ex = experts_struct(experts)
    if dtype is None:
        if h.dtype != torch.float32:
            raise TypeError("grouped_down: pass dtype, the activation type (bf16 or fp16) "
                            "the fp16 h was computed from")
        dtype = torch.float32
    adt = _dt_of(dtype)
    want = torch.float32 if adt == F32 else torch.float16
    if h.dtype != want:
        raise TypeError(f"h must be {want} for {dtype} activations")
    ys = torch.empty(T * k, experts.d, dtype=h.dtype, device=h.device)
    _check(lib.moe_grouped_down(_ptr(h), adt, _ptr(tables.row_off), _ptr(tables.tile_off),
                                tables.BM, T, k, ctypes.byref(ex), _ptr(ys), regime,
                                _stream(stream)), "moe_grouped_down")
    return ys


def combine(ys, inv_order, topk_w, T, k, dtype=torch.bfloat16, stream=None):
    """-> y [T, d] in `dtype` from ys [T*k, d] (fp16 for 16-bit `dtype`, fp32 for fp32)"""
    _dev(ys, inv_order, topk_w)
    want = torch.float32 if dtype == torch.float32 else torch.float16
    if ys.dtype != want:
        raise TypeError(f"ys must be {want} for {dtype} outputs")
    d = ys.shape[1]
    y = torch.empty(T, d, dtype=dtype, device=ys.device)
    _check(lib.moe_combine(_ptr(ys), _ptr(inv_order), _ptr(topk_w), T, k, d,
                           _dt_of(dtype), _ptr(y),
                           _stream(stream)), "moe_combine")
    return y


# ------------------------------------------------------------------ forward

def _fmt_code(fmt) -> int:
    return _FMT[fmt] if isinstance(fmt, str) else int(fmt)


def forward_layout(T, d, E, k, F, dtype, wfmt, regime=REGIME_AUTO) -> WsLayout:
    """moe_forward's workspace layout for experts of weight format `wfmt`
    (a name such as "q4", or a moe_wfmt code)."""
    L = WsLayout()
    dt = _dt_of(dtype)
    _check(lib.moe_forward_layout(T, d, E, k, F, dt, _fmt_code(wfmt), regime, ctypes.byref(L)),
           "moe_forward_layout")
    return L


def sort_block_m() -> int:
    """BM of the tensor-core regime (moe_sort_block_m)."""
    return lib.moe_sort_block_m()


def forward_workspace(x, experts, k, regime=REGIME_AUTO):
    """A workspace tensor large enough for moe_forward on these shapes."""
    L = forward_layout(x.shape[0], experts.d, experts.E, k, experts.F, x.dtype, experts.fmt,
                       regime)
    return torch.empty(max(L.total, 256), dtype=torch.uint8, device=x.device)


def forward(x, w_router, router_bias, experts, k, regime=REGIME_AUTO, ws=None, out=None,
            stream=None):
    """The whole layer: y [T, d] in x's dtype."""
    _dev(x, w_router, router_bias)
    T = x.shape[0]
    ex = experts_struct(experts)
    if ws is None:
        ws = forward_workspace(x, experts, k, regime)
    y = out if out is not None else torch.empty(T, experts.d, dtype=x.dtype, device=x.device)
    _check(lib.moe_forward(_ptr(x), _dt(x), _ptr(w_router), _ptr(router_bias), ctypes.byref(ex),
                           T, k, _ptr(y), _ptr(ws), ws.numel(), regime, _stream(stream)),
           "moe_forward")
    return y


def pack_gate_up(fmt, w_g, w_u, s_g=None, b_g=None, s_u=None, b_u=None, stream=None):
    """Fused [gate|up] tensors (w_gu, s_gu, b_gu) from separate gate and up
    projections [E][F][...] on the device; s_gu, b_gu are None unless q4."""
    _dev(w_g, w_u, s_g, b_g, s_u, b_u)
    E, F = w_g.shape[0], w_g.shape[1]
    fmt_c = _FMT[fmt] if isinstance(fmt, str) else int(fmt)
    per_word = {W_Q4G64: 8, W_Q4G32: 8, W_Q4G128: 8, W_Q8G64: 4}.get(fmt_c, 1)
    d = w_g.shape[2] * per_word
    group = {W_Q4G64: 64, W_Q4G32: 32, W_Q4G128: 128, W_Q8G64: 64}.get(fmt_c, 0)
    w_gu = torch.empty((E, 2 * F) + tuple(w_g.shape[2:]), dtype=w_g.dtype, device=w_g.device)
    s_gu = b_gu = None
    if group:
        s_gu = torch.empty((E, 2 * F, d // group), dtype=s_g.dtype, device=s_g.device)
        b_gu = torch.empty_like(s_gu)
    _check(lib.moe_pack_gate_up(fmt_c, E, d, F, _ptr(w_g), _ptr(s_g), _ptr(b_g), _ptr(w_u),
                                _ptr(s_u), _ptr(b_u), _ptr(w_gu), _ptr(s_gu), _ptr(b_gu),
                                _stream(stream)), "moe_pack_gate_up")
    return w_gu, s_gu, b_gu


def device_status() -> int:
    """Status word of device-side errors since the last read (resets it)."""
    return lib.moe_device_status()


def set_wait_cycles(cycles: int):
    """Bound of every device-side wait, in SM cycles (0: the default, ~1 s)."""
    _check(lib.moe_set_wait_cycles(int(cycles)), "moe_set_wait_cycles")
