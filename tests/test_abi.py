"""The C ABI library: it loads, exports every symbol include/moe.h declares,
and rejects bad arguments on the host before any launch (runs without a GPU:
none of these calls reaches the CUDA runtime)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def moe():
    import __graft_entry__
    __graft_entry__.build()
    import sparse_mixture_experts_top_b200 as m
    return m


def test_header_declares_the_entry_points():
    names = _declared()
    for n in ("moe_route", "moe_topk", "moe_sort_rows", "moe_grouped_swiglu", "moe_grouped_down",
              "moe_combine", "moe_forward", "moe_forward_workspace"):
        assert n in names


def test_library_exports_every_declared_symbol(moe):
    lib = ctypes.CDLL(moe.LIB_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_binding_names_match_exports(moe):
    assert sorted(moe.EXPORTS) == _declared()


def test_status_strings(moe):
    for s in range(7):
        assert moe.status_str(s)
    assert "sm_100a" in moe.version()


P = None   # null pointer


def _ex(moe, fmt=2, E=8, d=128, F=256, w=0x1000):
    return moe.Experts(fmt, E, d, F, w, w, w, w, w, w)


def test_forward_rejects_bad_arguments_without_launching(moe):
    L = moe.lib
    ex = _ex(moe)
    fake = ctypes.c_void_p(0x10000)
    # null x
    assert L.moe_forward(P, moe.BF16, fake, P, ctypes.byref(ex), 4, 2, fake, fake, 1 << 30, 0, P) == moe.ERR_INVALID_ARG
    # k > E
    assert L.moe_forward(fake, moe.BF16, fake, P, ctypes.byref(ex), 4, 9, fake, fake, 1 << 30, 0, P) == moe.ERR_INVALID_ARG
    # k = 0
    assert L.moe_forward(fake, moe.BF16, fake, P, ctypes.byref(ex), 4, 0, fake, fake, 1 << 30, 0, P) == moe.ERR_INVALID_ARG
    # negative T
    assert L.moe_forward(fake, moe.BF16, fake, P, ctypes.byref(ex), -1, 2, fake, fake, 1 << 30, 0, P) == moe.ERR_INVALID_ARG
    # d not a multiple of 64
    bad = _ex(moe, d=100)
    assert L.moe_forward(fake, moe.BF16, fake, P, ctypes.byref(bad), 4, 2, fake, fake, 1 << 30, 0, P) == moe.ERR_UNSUPPORTED
    # q4 weights with fp32 activations
    assert L.moe_forward(fake, moe.F32, fake, P, ctypes.byref(ex), 4, 2, fake, fake, 1 << 30, 0, P) == moe.ERR_UNSUPPORTED
    # bf16 or fp32 weights with fp16 activations
    for fmt in (moe.W_BF16, moe.W_F32):
        assert L.moe_forward(fake, moe.F16, fake, P, ctypes.byref(_ex(moe, fmt=fmt)), 4, 2, fake, fake, 1 << 30, 0, P) == moe.ERR_UNSUPPORTED
    # unknown activation dtype
    assert L.moe_forward(fake, 3, fake, P, ctypes.byref(ex), 4, 2, fake, fake, 1 << 30, 0, P) == moe.ERR_INVALID_ARG
    # unknown weight format
    bad = _ex(moe, fmt=7)
    assert L.moe_forward(fake, moe.BF16, fake, P, ctypes.byref(bad), 4, 2, fake, fake, 1 << 30, 0, P) == moe.ERR_INVALID_ARG
    # unknown gate activation
    bad = _ex(moe)
    bad.act = 7
    assert L.moe_forward(fake, moe.BF16, fake, P, ctypes.byref(bad), 4, 2, fake, fake, 1 << 30, 0, P) == moe.ERR_INVALID_ARG
    # workspace too small / missing
    assert L.moe_forward(fake, moe.BF16, fake, P, ctypes.byref(ex), 4, 2, fake, fake, 16, 0, P) == moe.ERR_WORKSPACE
    assert L.moe_forward(fake, moe.BF16, fake, P, ctypes.byref(ex), 4, 2, fake, P, 1 << 30, 0, P) == moe.ERR_WORKSPACE
    # misaligned x
    assert L.moe_forward(ctypes.c_void_p(0x10008), moe.BF16, fake, P, ctypes.byref(ex), 4, 2, fake, fake, 1 << 30, 0, P) == moe.ERR_INVALID_ARG
    # E too large, k too large
    assert L.moe_forward(fake, moe.BF16, fake, P, ctypes.byref(_ex(moe, E=2048)), 4, 2, fake, fake, 1 << 30, 0, P) == moe.ERR_UNSUPPORTED
    assert L.moe_forward(fake, moe.BF16, fake, P, ctypes.byref(_ex(moe, E=64)), 4, 33, fake, fake, 1 << 30, 0, P) == moe.ERR_UNSUPPORTED
    # T = 0 is a no-op
    assert L.moe_forward(fake, moe.BF16, fake, P, ctypes.byref(ex), 0, 2, fake, fake, 0, 0, P) == moe.OK


def test_stage_calls_reject_bad_arguments(moe):
    L = moe.lib
    fake = ctypes.c_void_p(0x10000)
    ex = _ex(moe)
    assert L.moe_topk(P, 4, 8, 2, fake, fake, P) == moe.ERR_INVALID_ARG
    assert L.moe_topk(fake, 4, 8, 9, fake, fake, P) == moe.ERR_INVALID_ARG
    assert L.moe_topk(fake, 0, 8, 2, fake, fake, P) == moe.OK
    assert L.moe_route(fake, 5, fake, P, 4, 128, 8, 2, fake, fake, fake, P) == moe.ERR_INVALID_ARG
    assert L.moe_route(fake, moe.BF16, fake, P, 4, 100, 8, 2, fake, fake, fake, P) == moe.ERR_UNSUPPORTED
    assert L.moe_sort_rows(fake, 4, 2, 8, 0, fake, fake, fake, fake, fake, fake, fake, 1 << 20, P) == moe.ERR_INVALID_ARG
    assert L.moe_sort_rows(fake, 4000, 2, 8, 8, fake, fake, fake, fake, fake, fake, P, 0, P) == moe.ERR_WORKSPACE
    assert L.moe_sort_rows(fake, 4000, 2, 8, 8, fake, fake, fake, fake, fake, fake, fake, 8, P) == moe.ERR_WORKSPACE
    assert L.moe_grouped_swiglu(fake, moe.BF16, P, fake, fake, 8, 4, 2, ctypes.byref(ex), fake, fake, 1 << 20, 0, P) == moe.ERR_INVALID_ARG
    assert L.moe_grouped_swiglu(fake, moe.BF16, fake, fake, fake, 0, 4, 2, ctypes.byref(ex), fake, fake, 1 << 20, 0, P) == moe.ERR_INVALID_ARG
    # the tensor-core regime needs its fp16 staging workspace
    ex256 = _ex(moe, d=256)
    assert L.moe_grouped_swiglu(fake, moe.BF16, fake, fake, fake, 128, 4, 2, ctypes.byref(ex256), fake, P, 0, 2, P) == moe.ERR_WORKSPACE
    # ... and tiles d by 256: d = 128 is not a shape it takes
    assert L.moe_grouped_swiglu(fake, moe.BF16, fake, fake, fake, 128, 4, 2, ctypes.byref(ex), fake, fake, 1 << 20, 2, P) == moe.ERR_UNSUPPORTED
    assert L.moe_grouped_down(fake, moe.BF16, fake, fake, 128, 4, 2, ctypes.byref(ex), fake, 2, P) == moe.ERR_UNSUPPORTED
    assert L.moe_grouped_swiglu_workspace(4, 2, 128, moe.BF16) >= 4 * 2 * 128 * 2
    assert L.moe_grouped_down(fake, moe.BF16, fake, fake, 8, 4, 2, P, fake, 0, P) == moe.ERR_INVALID_ARG
    # the tensor-core regime takes bf16 activations only
    exf = _ex(moe, fmt=0)
    assert L.moe_grouped_down(fake, moe.F32, fake, fake, 128, 4, 2, ctypes.byref(exf), fake, 2, P) == moe.ERR_UNSUPPORTED
    assert L.moe_combine(fake, fake, fake, 4, 2, 100, moe.BF16, fake, P) == moe.ERR_UNSUPPORTED
    assert L.moe_combine(P, fake, fake, 4, 2, 128, moe.BF16, fake, P) == moe.ERR_INVALID_ARG
    assert L.moe_combine(fake, fake, fake, 0, 2, 128, moe.BF16, fake, P) == moe.OK


def test_pack_gate_up_rejects_bad_arguments(moe):
    L = moe.lib
    fake = ctypes.c_void_p(0x10000)
    # unknown format, zero sizes, d not a multiple of 64, missing q4 scales
    assert L.moe_pack_gate_up(7, 2, 64, 64, fake, fake, fake, fake, fake, fake, fake, fake, fake, P) == moe.ERR_INVALID_ARG
    assert L.moe_pack_gate_up(moe.W_BF16, 0, 64, 64, fake, P, P, fake, P, P, fake, P, P, P) == moe.ERR_INVALID_ARG
    assert L.moe_pack_gate_up(moe.W_BF16, 2, 96, 64, fake, P, P, fake, P, P, fake, P, P, P) == moe.ERR_UNSUPPORTED
    assert L.moe_pack_gate_up(moe.W_Q4G64, 2, 64, 64, fake, P, fake, fake, fake, fake, fake, fake, fake, P) == moe.ERR_INVALID_ARG


def test_regime_choice(moe):
    """AUTO takes the tensor-core kernels wherever they tile the shape with
    16-bit activations, except that the whole-layer call keeps the fused
    decode kernel while it applies and fewer than E rows are routed; the
    weight-streaming kernels for fp32 and for shapes or formats the
    tensor-core kernels do not take."""
    torch = __import__("torch")
    prefill = (2048, 2048, 512, 10, 512)       # 40 rows per expert
    decode = lambda T: (T, 2048, 128, 8, 768)  # the decode layer at T tokens
    small_e512 = (4, 2048, 512, 10, 512)       # 40 rows, E > 256: no fused kernel
    for dt in (torch.bfloat16, torch.float16):
        assert moe.forward_layout(*prefill, dt, "q4").regime == moe.REGIME_TC
        for T in (1, 8, 15):                   # T k < E: the fused decode kernel
            assert moe.forward_layout(*decode(T), dt, "q4").regime == moe.REGIME_GEMV
        for T in (16, 32):
            assert moe.forward_layout(*decode(T), dt, "q4").regime == moe.REGIME_TC
        assert moe.forward_layout(*small_e512, dt, "q4").regime == moe.REGIME_TC
    # the fused decode kernel takes q4 only: q8 at the same shape goes to TC
    assert moe.forward_layout(*decode(8), torch.bfloat16, "q8").regime == moe.REGIME_TC
    assert moe.forward_layout(*prefill, torch.float32, "f32").regime == moe.REGIME_GEMV
    # bf16 weights: F % 256 == 128 is a shape the tensor-core kernels tile
    # (q4 needs F % 256 == 0)
    acc = (512, 2048, 8, 2, 640)
    assert moe.forward_layout(*acc, torch.bfloat16, "bf16").regime == moe.REGIME_TC
    assert moe.forward_layout(*acc, torch.bfloat16, "q4").regime == moe.REGIME_GEMV
    decode = decode(8)
    # an explicit regime is kept
    assert moe.forward_layout(*decode, torch.bfloat16, "q4", moe.REGIME_TC).regime == moe.REGIME_TC
    with pytest.raises(TypeError):
        moe.forward_layout(*decode, torch.int8, "q4")
    # an unknown weight format is refused
    L = moe.WsLayout()
    assert moe.lib.moe_forward_layout(*decode, moe.BF16, 9, 0, ctypes.byref(L)) == moe.ERR_INVALID_ARG


def test_sort_block_m_is_the_tensor_core_tile(moe):
    """moe_sort_block_m is the BM the tensor-core regime needs: the layout of a
    forward that resolves to that regime sorts with it, and a stage call in
    that regime with another BM is refused."""
    torch = __import__("torch")
    bm = moe.sort_block_m()
    assert bm == 128
    L = moe.forward_layout(2048, 2048, 512, 10, 512, torch.bfloat16, "q4")
    assert L.regime == moe.REGIME_TC and L.BM == bm
    fake = ctypes.c_void_p(0x10000)
    ex = _ex(moe, d=256)
    assert moe.lib.moe_grouped_down(fake, moe.BF16, fake, fake, bm // 2, 4, 2, ctypes.byref(ex),
                                    fake, 2, P) == moe.ERR_INVALID_ARG


def test_forward_layout_is_consistent(moe):
    for (T, d, E, k, F) in [(1, 2048, 128, 8, 768), (2048, 2048, 512, 10, 512), (16, 128, 8, 2, 256)]:
        L = moe.forward_layout(T, d, E, k, F, __import__("torch").bfloat16, "q4")
        offs = [L.logits, L.topk_idx, L.topk_w, L.order, L.inv_order, L.row_map, L.counts,
                L.row_off, L.tile_off, L.sort_ws, L.h, L.ys, L.x16]
        assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
        assert L.ys + T * k * d * 2 <= L.x16          # fp16 ys for bf16 activations
        # fp16 token rows: T of them, or all T*k rows in sorted order (tensor cores)
        assert L.x16 + (T * k if L.regime == moe.REGIME_TC else T) * d * 2 <= L.total
        assert L.h + T * k * F * 2 <= L.ys
        assert L.BM >= 1 and L.regime in (moe.REGIME_GEMV, moe.REGIME_TC)
        assert moe.lib.moe_forward_workspace(T, d, E, k, F, moe.BF16, moe.W_Q4G64, 0) == L.total
        # fp16 activations take the same layout as bf16 ones
        L16 = moe.forward_layout(T, d, E, k, F, __import__("torch").float16, "q4")
        assert (L16.total, L16.x16, L16.regime, L16.BM) == (L.total, L.x16, L.regime, L.BM)
