"""CPU fp64 oracle of the hard-routed sparse MoE layer forward.

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg import this package. It shares no code with the
CUDA library and never calls it; the product path never imports it.

The arithmetic lives in ``moe_oracle.c`` (plain C, double precision). This
module compiles it with gcc into ``liborc_moe.so`` next to the source and
marshals numpy/torch host arrays into it. Every function mirrors one step of
the layer (see the header of ``moe_oracle.c`` for the passage each follows):

* ``router_logits``  -- L = x . W_r + b                     (fp64)
* ``topk``           -- ranked selection and renormalised weights
* ``topk_weights_full_softmax`` -- the same weights via softmax over all E
* ``sort_rows``      -- stable sort of routed slots, row and tile tables
* ``expert_swiglu``  -- h = silu(x W_g^T) * (x W_u^T) over sorted rows
* ``expert_down``    -- ys = h W_d^T over sorted rows
* ``expert_gate_up`` / ``expert_down_abs`` -- pre-activations and sums of
  absolute products, used by the tests to bound rounding errors
* ``combine``        -- y[t] = sum_j w[t,j] ys[inv_order[t k + j]]
* ``forward``        -- the whole layer
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liborc_moe.so")

ACT = {"f32": 0, "bf16": 1, "f16": 2}
WFMT = {"f32": 0, "bf16": 1, "q4": 2, "q4g32": 3, "q4g128": 4, "q8": 5}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wno-unused-function",
                               "-D_GNU_SOURCE", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P, I, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        L.orc_router_logits.argtypes = [P, I, P, P, I, I, I, P, I]
        L.orc_topk.argtypes = [P, I, I, I, P, P]
        L.orc_topk_weights_full_softmax.argtypes = [P, P, I, I, I, P]
        L.orc_sort_rows.argtypes = [P, I, I, I, I, P, P, P, P, P, P]
        L.orc_expert_swiglu.argtypes = [P, I, P, P, I, I, I, I, P, P, P, P, I, I]
        L.orc_expert_down.argtypes = [P, P, I, I, I, I, P, P, P, P, I]
        L.orc_combine.argtypes = [P, P, P, I, I, I, P]
        L.orc_forward.argtypes = [P, I, P, P, I, I, I, I, I, I, I, P, P, P, P, P, P,
                                  P, P, P, P, P, P, I, I]
        L.orc_expert_gate_up.argtypes = [P, I, P, P, I, I, I, I, P, P, P, P, P, P, P, I]
        L.orc_expert_down_abs.argtypes = [P, P, I, I, I, I, P, P, P, P, I]
        L.orc_weight_value.argtypes = [I, P, P, P, I, I, I, I, I]
        L.orc_weight_value.restype = D
        _lib = L
    return _lib


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


# ------------------------------------------------------------- marshalling

def _np(a, dtype=None):
    """Host, C-contiguous numpy view of a numpy array or CPU torch tensor.
    bf16 and uint32 torch tensors are passed as raw 16/32-bit words."""
    if a is None:
        return None
    try:
        import torch
        if isinstance(a, torch.Tensor):
            t = a.detach()
            if t.device.type != "cpu":
                raise ValueError("oracle inputs must be host tensors")
            t = t.contiguous()
            if t.dtype == torch.bfloat16:
                return t.view(torch.int16).numpy().view(np.uint16)
            if t.dtype == torch.uint32:
                return t.view(torch.int32).numpy().view(np.uint32)
            a = t.numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(a)
    if dtype is not None and a.dtype != dtype:
        a = a.astype(dtype)
    return a


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _act_code(a) -> int:
    """0 for fp32 storage, 1 for bf16 (passed as uint16 words), 2 for IEEE
    binary16 (numpy float16, passed as its own 16-bit words)."""
    if a.dtype == np.float32:
        return ACT["f32"]
    if a.dtype == np.uint16:
        return ACT["bf16"]
    if a.dtype == np.float16:
        return ACT["f16"]
    raise TypeError(f"activation dtype {a.dtype} not supported")


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what}: invalid arguments (rc={rc})")


# --------------------------------------------------------------- the steps

def router_logits(x, w_router, bias, nthreads=None):
    """fp64 logits [T, E] = x . W_r + bias (w_router stored [E, d])."""
    xa, wa = _np(x), _np(w_router)
    ba = _np(bias, np.float32)
    T, d = xa.shape
    E = wa.shape[0]
    L = np.empty((T, E), np.float64)
    _check(lib().orc_router_logits(_p(xa), _act_code(xa), _p(wa), _p(ba), T, d, E, _p(L),
                                   nthreads or default_threads()), "router_logits")
    return L


def topk(logits, k):
    """(idx int32 [T,k], w fp64 [T,k]) from logits [T, E] (any float dtype,
    taken exactly as doubles)."""
    La = _np(logits).astype(np.float64)
    T, E = La.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    _check(lib().orc_topk(_p(La), T, E, k, _p(idx), _p(w)), "topk")
    return idx, w


def topk_weights_full_softmax(logits, idx):
    La = _np(logits).astype(np.float64)
    ia = _np(idx, np.int32)
    T, E = La.shape
    k = ia.shape[1]
    w = np.empty((T, k), np.float64)
    _check(lib().orc_topk_weights_full_softmax(_p(La), _p(ia), T, E, k, _p(w)), "full softmax")
    return w


@dataclass
class SortTables:
    order: np.ndarray
    inv_order: np.ndarray
    row_map: np.ndarray
    counts: np.ndarray
    row_off: np.ndarray
    tile_off: np.ndarray


def sort_rows(idx, E, BM) -> SortTables:
    ia = _np(idx, np.int32)
    T, k = ia.shape
    R = T * k
    order = np.empty(R, np.uint32)
    inv = np.empty(R, np.uint32)
    rmap = np.empty(R, np.uint32)
    counts = np.empty(E, np.int32)
    roff = np.empty(E + 1, np.int32)
    toff = np.empty(E + 1, np.int32)
    _check(lib().orc_sort_rows(_p(ia), T, k, E, BM, _p(order), _p(inv), _p(rmap), _p(counts),
                               _p(roff), _p(toff)), "sort_rows")
    return SortTables(order, inv, rmap, counts, roff, toff)


def _wargs(experts, which):
    if which == "gu":
        w, s, b = experts.w_gu, experts.s_gu, experts.b_gu
    else:
        w, s, b = experts.w_dn, experts.s_dn, experts.b_dn
    wa = _np(w)
    if experts.fmt == "f32":
        wa = wa.astype(np.float32, copy=False)
    return wa, _np(s), _np(b)


# the gate's activation of the GLU: SwiGLU (silu) or GeGLU (tanh-form GELU)
ACTS = {"swiglu": 0, "geglu": 1}


def act_code(experts) -> int:
    return ACTS[getattr(experts, "act", "swiglu")]


def expert_swiglu(x, row_map, row_off, experts, nthreads=None):
    xa = _np(x)
    rm = _np(row_map, np.uint32)
    ro = _np(row_off, np.int32)
    w, s, b = _wargs(experts, "gu")
    R = rm.shape[0]
    h = np.empty((R, experts.F), np.float64)
    _check(lib().orc_expert_swiglu(_p(xa), _act_code(xa), _p(rm), _p(ro), experts.E, experts.d,
                                   experts.F, WFMT[experts.fmt], _p(w), _p(s), _p(b), _p(h),
                                   act_code(experts), nthreads or default_threads()),
           "expert_swiglu")
    return h


def expert_gate_up(x, row_map, row_off, experts, nthreads=None):
    """(g, u, |x|.|w_gate|, |x|.|w_up|), each fp64 [R, F], for sorted rows."""
    xa = _np(x)
    rm = _np(row_map, np.uint32)
    ro = _np(row_off, np.int32)
    w, s, b = _wargs(experts, "gu")
    R = rm.shape[0]
    out = [np.empty((R, experts.F), np.float64) for _ in range(4)]
    _check(lib().orc_expert_gate_up(_p(xa), _act_code(xa), _p(rm), _p(ro), experts.E, experts.d,
                                    experts.F, WFMT[experts.fmt], _p(w), _p(s), _p(b),
                                    *[_p(o) for o in out], nthreads or default_threads()),
           "expert_gate_up")
    return tuple(out)


def expert_down_abs(h, row_off, experts, nthreads=None):
    """|h[i]| . |w_dn[e][o]| for sorted rows, fp64 [R, d]."""
    ha = _np(h).astype(np.float64)
    ro = _np(row_off, np.int32)
    w, s, b = _wargs(experts, "dn")
    out = np.empty((ha.shape[0], experts.d), np.float64)
    _check(lib().orc_expert_down_abs(_p(ha), _p(ro), experts.E, experts.d, experts.F,
                                     WFMT[experts.fmt], _p(w), _p(s), _p(b), _p(out),
                                     nthreads or default_threads()), "expert_down_abs")
    return out


def expert_down(h, row_off, experts, nthreads=None):
    ha = _np(h).astype(np.float64)
    ro = _np(row_off, np.int32)
    w, s, b = _wargs(experts, "dn")
    R = ha.shape[0]
    ys = np.empty((R, experts.d), np.float64)
    _check(lib().orc_expert_down(_p(ha), _p(ro), experts.E, experts.d, experts.F,
                                 WFMT[experts.fmt], _p(w), _p(s), _p(b), _p(ys),
                                 nthreads or default_threads()), "expert_down")
    return ys


def combine(ys, inv_order, w, T, k):
    ya = _np(ys).astype(np.float64)
    ia = _np(inv_order, np.uint32)
    wa = _np(w).astype(np.float64)
    d = ya.shape[1]
    y = np.empty((T, d), np.float64)
    _check(lib().orc_combine(_p(ya), _p(ia), _p(wa), T, k, d, _p(y)), "combine")
    return y


@dataclass
class ForwardResult:
    y: np.ndarray
    logits64: np.ndarray
    idx: np.ndarray
    w: np.ndarray
    h: np.ndarray | None = None
    ys: np.ndarray | None = None


def forward(x, w_router, bias, experts, k, BM=1, keep_intermediates=False, nthreads=None):
    xa, wra = _np(x), _np(w_router)
    ba = _np(bias, np.float32)
    T, d = xa.shape
    E, F = experts.E, experts.F
    R = T * k
    wg, sg, bg = _wargs(experts, "gu")
    wd, sd, bd = _wargs(experts, "dn")
    y = np.empty((T, d), np.float64)
    L = np.empty((T, E), np.float64)
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    h = np.empty((R, F), np.float64) if keep_intermediates else None
    ys = np.empty((R, d), np.float64) if keep_intermediates else None
    _check(lib().orc_forward(_p(xa), _act_code(xa), _p(wra), _p(ba), T, d, E, k, F, BM,
                             WFMT[experts.fmt], _p(wg), _p(sg), _p(bg), _p(wd), _p(sd), _p(bd),
                             _p(y), _p(L), _p(idx), _p(w), _p(h), _p(ys),
                             act_code(experts), nthreads or default_threads()), "forward")
    return ForwardResult(y, L, idx, w, h, ys)


def weight_value(experts, which, e, r, c):
    """Dequantised value of one element of one expert weight matrix."""
    w, s, b = _wargs(experts, which)
    rows, cols = (2 * experts.F, experts.d) if which == "gu" else (experts.d, experts.F)
    return lib().orc_weight_value(WFMT[experts.fmt], _p(w), _p(s), _p(b), rows, cols, e, r, c)
