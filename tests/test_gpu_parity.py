"""GPU parity: every stage of the CUDA path and the whole layer against the
fp64 CPU oracle, on the same seeded inputs, through the C ABI.

Integer outputs (top-k indices from identical logits, order, inv_order,
row_map, counts, row_off, tile_off) must match bit for bit. Floating outputs
must satisfy max |gpu - oracle| <= 2e-2 * RMS(oracle) for bf16 activations
and 1e-4 * RMS for the all-fp32 workload. End-to-end runs where the GPU
computes its own fp32 logits may flip a selection only where the oracle's
k-th and (k+1)-th logits are within the logit error bound; such tokens are
counted and left out of the output comparison.
"""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from parity_util import (TOL_BF16, TOL_F32, U_F16, assert_close_rms, assert_h_close,
                         assert_ys_close, kth_gap, to_np, topk_ref)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_mixture_experts_top_b200 as m
    return m


def _tol(act):
    return TOL_F32 if act == "f32" else TOL_BF16


def _host(ex):
    return ex.to("cpu")


# ------------------------------------------------------------------ top-k

@pytest.mark.parametrize("ties", [False, True])
@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (37, 8, 2), (64, 128, 8), (300, 256, 8),
                                   (513, 512, 10), (33, 1000, 32), (50, 7, 7), (20, 33, 5)])
def test_topk_bit_exact_from_identical_logits(moe, orc, ties, T, E, k):
    lg = mi.random_logits(T, E, seed=T * 7 + E, ties=ties)
    idx, w = moe.topk(lg.to(DEV), k)
    oidx, ow = orc.topk(lg.double().numpy(), k)
    np.testing.assert_array_equal(to_np(idx), oidx)
    np.testing.assert_allclose(to_np(w), ow, rtol=0, atol=2e-6)


def test_topk_signed_zero_and_nan(moe, orc):
    lg = torch.tensor([[-0.0, 0.0, -1.0, float("nan")],
                       [float("nan"), -5.0, -0.0, 0.0],
                       [1.0, 1.0, 1.0, 1.0]], dtype=torch.float32)
    idx, _ = moe.topk(lg.to(DEV), 3)
    np.testing.assert_array_equal(to_np(idx), topk_ref(lg.numpy(), 3))
    oidx, _ = orc.topk(lg.double().numpy(), 3)
    np.testing.assert_array_equal(to_np(idx), oidx)


# ------------------------------------------------------------------ route

@pytest.mark.parametrize("name,T", [("tiny", 16), ("decode_t1", 1), ("decode_t32", 32),
                                    ("prefill", 256), ("skewed", 64), ("acceptance", 100),
                                    ("prefill", 2048), ("skewed", 520), ("acceptance", 512)])
def test_route_logits_and_selection(moe, orc, name, T):
    _check_route(moe, orc, mi.workload(name, T=T), T)


def _check_route(moe, orc, wl, T):
    g = torch.Generator().manual_seed(11)
    x = torch.randn(T, wl.d, generator=g).to(mi._act_dtype(wl.act))
    wr = (torch.randn(wl.E, wl.d, generator=g) / wl.d ** 0.5).to(x.dtype)
    bias = mi.make_router_bias(wl, 0)
    logits, idx, w = moe.route(x.to(DEV), wr.to(DEV), None if bias is None else bias.to(DEV), wl.k)
    L64 = orc.router_logits(x, wr, bias)
    # error bound of an fp32 sum of d products in any order: d * eps32 * sum |x_i w_i|
    absdot = np.abs(x.double().numpy()) @ np.abs(wr.double().numpy()).T
    bound = wl.d * 2.0 ** -24 * absdot + 1e-6
    gl = to_np(logits).astype(np.float64)
    assert (np.abs(gl - L64) <= bound).all()
    # selection: the GPU picks the exact top-k of its own logits ...
    gidx = to_np(idx)
    np.testing.assert_array_equal(gidx, topk_ref(to_np(logits), wl.k))
    # ... and agrees with the oracle except where the oracle's k-th gap is
    # within twice the logit error bound
    oidx, ow = orc.topk(L64.astype(np.float32), wl.k)
    flips = np.where((gidx != oidx).any(axis=1))[0]
    gap = kth_gap(L64, wl.k)
    for t in flips:
        assert gap[t] <= 2 * bound[t].max(), (t, gap[t], gidx[t], oidx[t])
    keep = np.setdiff1d(np.arange(T), flips)
    # softmax weights move by at most 2 * max|dL| when the logits move by dL
    dl = np.abs(gl - L64.astype(np.float32)).max(axis=1, keepdims=True)
    assert (np.abs(to_np(w)[keep] - ow[keep]) <= 2e-6 + 2 * dl[keep]).all()
    assert len(flips) <= max(1, T // 50)


# ------------------------------------------------------------------ sort

@pytest.mark.parametrize("T,E,k,BM,skew", [
    (1, 128, 8, 8, 0.0), (32, 128, 8, 8, 0.0), (16, 8, 2, 8, 0.0), (100, 8, 2, 128, 0.0),
    (512, 8, 2, 128, 0.5),                 # R = 1024: single-block path, the boundary
    (513, 8, 2, 128, 0.0),                 # R = 1026: multi-block path
    (2048, 512, 10, 128, 0.02),            # prefill-sized, skewed, empty experts
    (4096, 256, 8, 128, 0.05),             # 32,768 rows
    (3000, 1000, 3, 64, 0.0), (7, 1024, 32, 1, 0.0)])
def test_sort_bit_exact(moe, orc, T, E, k, BM, skew):
    idx = mi.random_topk_idx(T, E, k, seed=T + E + k, skew=skew)
    st = moe.sort_rows(idx.to(DEV), E, BM)
    ref = orc.sort_rows(idx.numpy(), E, BM)
    for name in ("order", "inv_order", "row_map", "counts", "row_off", "tile_off"):
        np.testing.assert_array_equal(to_np(getattr(st, name)), getattr(ref, name), err_msg=name)


def test_sort_all_rows_to_one_expert(moe, orc):
    T, E, k = 700, 64, 3
    idx = torch.tensor([[5, 9, 63]] * T, dtype=torch.int32)
    st = moe.sort_rows(idx.to(DEV), E, 128)
    ref = orc.sort_rows(idx.numpy(), E, 128)
    for name in ("order", "inv_order", "row_map", "counts", "row_off", "tile_off"):
        np.testing.assert_array_equal(to_np(getattr(st, name)), getattr(ref, name), err_msg=name)


# ------------------------------------------------------------------ experts

STAGE_CASES = [
    # workload, T override, regime (1 = weight-streaming, 2 = tensor core), BM, skew
    ("tiny", 16, 1, 8, 0.0),
    ("decode_t1", 1, 1, 8, 0.0),
    ("decode_t32", 32, 1, 8, 0.0),
    ("acceptance", 64, 1, 32, 0.0),
    ("prefill", 96, 1, 8, 0.02),
    # tensor-core kernels: bf16 weights; q4 weights; one row per tile (N = 16);
    # skewed routing with experts above 128 rows (several token tiles) and
    # empty experts; the large-d workload
    ("acceptance", 300, 2, 128, 0.0),
    ("decode_t32", 32, 2, 128, 0.0),
    ("decode_t1", 1, 2, 128, 0.0),
    ("prefill", 200, 2, 128, 0.0),
    ("prefill", 600, 2, 128, 0.5),
    ("skewed", 24, 2, 128, 0.3),
]


def _stage_setup(wl, T, seed, skew):
    # the workload as given (activation type, weight format), with T tokens
    layer = mi.make_layer(mi.Workload(**{**wl.__dict__, "T": T}), seed=seed, device=DEV)
    idx = mi.random_topk_idx(T, wl.E, wl.k, seed=seed + 1, skew=skew)
    return layer, idx


@pytest.mark.parametrize("name,T,regime,BM,skew", STAGE_CASES)
def test_grouped_swiglu_parity(moe, orc, name, T, regime, BM, skew):
    wl = mi.workload(name, T=T)
    layer, idx = _stage_setup(wl, T, 21, skew)
    st = moe.sort_rows(idx.to(DEV), wl.E, BM)
    h = moe.grouped_swiglu(layer.x, st, wl.k, layer.experts, regime=regime)
    ref_st = orc.sort_rows(idx.numpy(), wl.E, BM)
    hx = _host(layer.experts)
    href = orc.expert_swiglu(layer.x.cpu(), ref_st.row_map, ref_st.row_off, hx)
    if wl.act == "f32":
        assert_close_rms(h, href, TOL_F32, f"h[{name}]")
    else:
        assert h.dtype == torch.float16
        g, u, ga, ua = orc.expert_gate_up(layer.x.cpu(), ref_st.row_map, ref_st.row_off, hx)
        # q4 weights are dequantised to fp16 (bf16 weights are exact in fp16)
        u_w = U_F16 if mi.q4_group(wl.wfmt) else 0.0
        assert_h_close(h, href, g, u, ga, ua, wl.d, u_w, U_F16, TOL_BF16, f"h[{name}]")


@pytest.mark.parametrize("name,T,regime,BM,skew", STAGE_CASES)
def test_grouped_down_parity(moe, orc, name, T, regime, BM, skew):
    wl = mi.workload(name, T=T)
    layer, idx = _stage_setup(wl, T, 22, skew)
    st = moe.sort_rows(idx.to(DEV), wl.E, BM)
    hin = mi.random_rows(T * wl.k, wl.F, seed=23,
                         dtype=torch.float16 if wl.act == "bf16" else torch.float32)
    ys = moe.grouped_down(hin.to(DEV), st, T, wl.k, layer.experts, regime=regime,
                          dtype=layer.x.dtype)
    ref_st = orc.sort_rows(idx.numpy(), wl.E, BM)
    hx = _host(layer.experts)
    yref = orc.expert_down(hin.double().numpy(), ref_st.row_off, hx)
    # ys is stored in fp16 for bf16 activations, fp32 for fp32
    assert ys.dtype == (torch.float16 if wl.act == "bf16" else torch.float32)
    habs = orc.expert_down_abs(hin.double().numpy(), ref_st.row_off, hx)
    u_w = U_F16 if mi.q4_group(wl.wfmt) else 0.0
    u_ys = U_F16 if wl.act == "bf16" else 0.0
    assert_ys_close(ys, yref, habs, u_w, _tol(wl.act), f"ys[{name}]", u_ys=u_ys, F=wl.F)


@pytest.mark.parametrize("T,k,d,dt", [(1, 8, 2048, torch.bfloat16), (16, 2, 128, torch.float32),
                                      (2048, 10, 2048, torch.bfloat16), (5, 3, 64, torch.bfloat16),
                                      (1, 8, 2048, torch.float16), (300, 10, 2048, torch.float16)])
def test_combine_parity(moe, orc, T, k, d, dt):
    E = max(k, 16)
    idx = mi.random_topk_idx(T, E, k, seed=31)
    st = orc.sort_rows(idx.numpy(), E, 8)
    # ys arrive in fp16 for 16-bit outputs, fp32 for fp32
    ys = mi.random_ys(T * k, d, seed=32,
                      dtype=torch.float32 if dt == torch.float32 else torch.float16)
    w = mi.random_weights(T, k, seed=33)
    inv = torch.from_numpy(st.inv_order.view(np.int32)).view(torch.uint32)
    y = moe.combine(ys.to(DEV), inv.to(DEV), w.to(DEV), T, k, dtype=dt)
    yref = orc.combine(ys.double().numpy(), st.inv_order, w.double().numpy(), T, k)
    g = to_np(y).astype(np.float64)
    # an fp32 sum of k products (each rounding <= 2^-24 relative of the
    # partial sum), then one rounding to the output dtype
    # unit roundoff of the output type (8-, 11- or 24-bit precision)
    u = {torch.bfloat16: 2.0 ** -8, torch.float16: 2.0 ** -11, torch.float32: 2.0 ** -24}[dt]
    mag = np.abs(w.double().numpy())[:, :, None] * np.abs(ys.double().numpy()[st.inv_order.reshape(T, k)])
    bound = u * np.abs(yref) + (k + 1) * 2.0 ** -24 * mag.sum(axis=1) * (1 + u)
    assert (np.abs(g - yref) <= bound).all()


# ------------------------------------------------------------------ forward

def _forward_and_compare(moe, orc, layer, sample=None, regime=0):
    wl = layer.wl
    y = moe.forward(layer.x, layer.w_router, layer.router_bias, layer.experts, wl.k, regime=regime)
    torch.cuda.synchronize()
    rows = np.arange(wl.T) if sample is None else np.asarray(sample)
    xs = layer.x.cpu()[rows]
    r = orc.forward(xs, layer.w_router.cpu(), None if layer.router_bias is None else layer.router_bias.cpu(),
                    _host(layer.experts), wl.k)
    # the GPU's own routing (read back through the oracle-independent route call)
    logits, gidx, _ = moe.route(layer.x, layer.w_router, layer.router_bias, wl.k)
    gidx = to_np(gidx)[rows]
    flips = np.where((gidx != r.idx).any(axis=1))[0]
    if len(flips):
        absdot = np.abs(xs.double().numpy()) @ np.abs(layer.w_router.cpu().double().numpy()).T
        bound = wl.d * 2.0 ** -24 * absdot.max(axis=1) + 1e-6
        gap = kth_gap(r.logits64, wl.k)
        assert (gap[flips] <= 2 * bound[flips]).all()
    keep = np.setdiff1d(np.arange(len(rows)), flips)
    assert len(flips) <= max(1, len(rows) // 50)
    return assert_close_rms(to_np(y)[rows][keep], r.y[keep], _tol(wl.act), f"y[{wl.name}]")


@pytest.mark.parametrize("name,seed,regime", [("tiny", 0, 0), ("tiny", 1, 0), ("tiny", 2, 0),
                                              ("decode_t1", 0, 0), ("decode_t1", 1, 0),
                                              # the fused decode kernel; AUTO (tensor cores)
                                              ("decode_t32", 0, 1), ("decode_t32", 2, 0)])
def test_forward_parity_full(moe, orc, name, seed, regime):
    layer = mi.make_layer(name, seed=seed, device=DEV)
    _forward_and_compare(moe, orc, layer, regime=regime)


def test_forward_parity_acceptance(moe, orc):
    layer = mi.make_layer("acceptance", seed=0, device=DEV)
    _forward_and_compare(moe, orc, layer, sample=np.arange(0, 512, 4))


@pytest.mark.parametrize("regime", [0, 1])
def test_forward_parity_prefill_sampled(moe, orc, regime):
    layer = mi.make_layer("prefill", seed=0, device=DEV)
    rng = np.random.default_rng(0)
    _forward_and_compare(moe, orc, layer, sample=np.sort(rng.choice(2048, 96, replace=False)),
                         regime=regime)
    assert moe.device_status() == moe.OK


def test_forward_parity_dense_soft_routing(moe, orc):
    """k = E selects every expert and the renormalised weights are the full
    softmax: the layer is then dense soft routing, the baseline of the PRD's
    acceptance test ("5.5 real sparse MoE kernels (Metal)", Acceptance)."""
    layer = mi.make_layer("acceptance", seed=0, device=DEV)
    E = layer.wl.E
    y = moe.forward(layer.x, layer.w_router, None, layer.experts, E)
    torch.cuda.synchronize()
    rows = np.arange(0, layer.wl.T, 32)
    r = orc.forward(layer.x.cpu()[rows], layer.w_router.cpu(), None, _host(layer.experts), E)
    assert_close_rms(to_np(y)[rows], r.y, TOL_BF16, "y[acceptance, k = E]")
    assert moe.device_status() == moe.OK


def test_forward_parity_decode_t32_tensor_core(moe, orc):
    layer = mi.make_layer("decode_t32", seed=1, device=DEV)
    _forward_and_compare(moe, orc, layer, regime=2)


@pytest.mark.slow
def test_forward_parity_skewed_sampled(moe, orc):
    layer = mi.make_layer("skewed", seed=0, device=DEV)
    rng = np.random.default_rng(1)
    _forward_and_compare(moe, orc, layer, sample=np.sort(rng.choice(4096, 24, replace=False)))


# ------------------------------------------------------------------ GeGLU

@pytest.mark.parametrize("name,T,regime,BM", [("decode_t32", 32, 1, 8), ("prefill", 200, 2, 128),
                                              ("acceptance", 300, 2, 128)])
def test_grouped_geglu_parity(moe, orc, name, T, regime, BM):
    """The tanh-GELU GLU (mlx-lm PR #2044, "When it applies") through the
    weight-streaming and tensor-core gate|up kernels."""
    wl = mi.workload(name, T=T)
    layer, idx = _stage_setup(wl, T, 23, 0.0)
    ex = layer.experts.with_act("geglu")
    st = moe.sort_rows(idx.to(DEV), wl.E, BM)
    h = moe.grouped_swiglu(layer.x, st, wl.k, ex, regime=regime)
    ref_st = orc.sort_rows(idx.numpy(), wl.E, BM)
    hx = _host(ex)
    href = orc.expert_swiglu(layer.x.cpu(), ref_st.row_map, ref_st.row_off, hx)
    g, u, ga, ua = orc.expert_gate_up(layer.x.cpu(), ref_st.row_map, ref_st.row_off, hx)
    u_w = U_F16 if mi.q4_group(wl.wfmt) else 0.0
    assert_h_close(h, href, g, u, ga, ua, wl.d, u_w, U_F16, TOL_BF16, f"h[{name}, GeGLU]",
                   act="geglu")


@pytest.mark.parametrize("name", ["decode_t1", "decode_t32"])
def test_forward_geglu_fused_decode(moe, orc, name):
    layer = mi.make_layer(name, seed=5, device=DEV)
    layer.experts = layer.experts.with_act("geglu")
    _forward_and_compare(moe, orc, layer, regime=1)


def test_forward_geglu_prefill_sampled(moe, orc):
    layer = mi.make_layer("prefill", seed=1, device=DEV)
    layer.experts = layer.experts.with_act("geglu")
    rng = np.random.default_rng(2)
    _forward_and_compare(moe, orc, layer, sample=np.sort(rng.choice(2048, 48, replace=False)))


# ------------------------------------------------------------------ packing

@pytest.mark.parametrize("name", ["tiny", "acceptance", "decode_t32"])
def test_pack_separate_gate_up(moe, name):
    """Separate gate and up projections packed into the fused [gate|up]
    layout (DS4Server issue #112, "Kernel contract": fused or separate
    gate/up weights) give the fused tensors byte for byte, and so the same
    forward."""
    layer = mi.make_layer(mi.workload(name, T=8), seed=7, device=DEV)
    ex = layer.experts
    F = ex.F
    split = lambda t: (None, None) if t is None else (t[:, :F].contiguous(), t[:, F:].contiguous())
    wg, wu = split(ex.w_gu)
    sg, su = split(ex.s_gu)
    bg, bu = split(ex.b_gu)
    w_gu, s_gu, b_gu = moe.pack_gate_up(ex.fmt, wg, wu, sg, bg, su, bu)
    torch.cuda.synchronize()
    assert torch.equal(w_gu, ex.w_gu)
    if mi.q4_group(ex.fmt):
        assert torch.equal(s_gu, ex.s_gu) and torch.equal(b_gu, ex.b_gu)
    packed = mi.Experts(ex.fmt, ex.E, ex.d, F, w_gu, ex.w_dn, s_gu, b_gu, ex.s_dn, ex.b_dn)
    a = moe.forward(layer.x, layer.w_router, layer.router_bias, ex, layer.wl.k)
    b = moe.forward(layer.x, layer.w_router, layer.router_bias, packed, layer.wl.k)
    assert torch.equal(a.view(torch.int16) if a.dtype != torch.float32 else a,
                       b.view(torch.int16) if b.dtype != torch.float32 else b)


# ------------------------------------------------------------------ q4 groups 32 / 128

@pytest.mark.parametrize("wfmt", ["q4g32", "q4g128"])
@pytest.mark.parametrize("name,T", [("decode_t1", 1), ("decode_t32", 32)])
def test_forward_q4_group_sizes_fused_decode(moe, orc, wfmt, name, T):
    """4-bit weights with groups of 32 and 128 (DS4Server issue #112, "Kernel
    contract") through the fused decode kernel."""
    layer = mi.make_layer(mi.workload(name, T=T, wfmt=wfmt), seed=6, device=DEV)
    _forward_and_compare(moe, orc, layer, regime=1)


@pytest.mark.parametrize("wfmt", ["q4g32", "q4g128"])
def test_grouped_stages_q4_group_sizes(moe, orc, wfmt):
    """The weight-streaming gate|up and down kernels with groups of 32 / 128."""
    wl = mi.workload("decode_t32", T=32, wfmt=wfmt)
    layer, idx = _stage_setup(wl, 32, 29, 0.0)
    st = moe.sort_rows(idx.to(DEV), wl.E, 8)
    h = moe.grouped_swiglu(layer.x, st, wl.k, layer.experts, regime=1)
    ref_st = orc.sort_rows(idx.numpy(), wl.E, 8)
    hx = _host(layer.experts)
    href = orc.expert_swiglu(layer.x.cpu(), ref_st.row_map, ref_st.row_off, hx)
    g, u, ga, ua = orc.expert_gate_up(layer.x.cpu(), ref_st.row_map, ref_st.row_off, hx)
    assert_h_close(h, href, g, u, ga, ua, wl.d, U_F16, U_F16, TOL_BF16, f"h[{wfmt}]")
    ys = moe.grouped_down(h, st, 32, wl.k, layer.experts, regime=1, dtype=layer.x.dtype)
    yref = orc.expert_down(to_np(h).astype(np.float64), ref_st.row_off, hx)
    habs = orc.expert_down_abs(to_np(h).astype(np.float64), ref_st.row_off, hx)
    assert_ys_close(ys, yref, habs, U_F16, TOL_BF16, f"ys[{wfmt}]", u_ys=U_F16, F=wl.F)


@pytest.mark.parametrize("wfmt,T,regime", [("q4g128", 300, 1), ("q4g32", 1024, 0)])
def test_forward_q4_group_sizes_prefill_shape(moe, orc, wfmt, T, regime):
    """Prefill shapes: 300 tokens on the weight-streaming kernels (asked
    for); 1,024 tokens resolve to the tcgen05 kernels."""
    L = moe.forward_layout(T, 2048, 512, 10, 512, torch.bfloat16, wfmt, regime)
    assert L.regime == (moe.REGIME_TC if regime == 0 else moe.REGIME_GEMV)
    layer = mi.make_layer(mi.workload("prefill", T=T, wfmt=wfmt), seed=8, device=DEV)
    rng = np.random.default_rng(3)
    _forward_and_compare(moe, orc, layer, sample=np.sort(rng.choice(T, 32, replace=False)),
                         regime=regime)
    assert moe.device_status() == moe.OK


# ------------------------------------------------------------------ 8-bit affine

def test_grouped_stages_q8(moe, orc):
    """8-bit affine weights (mlxcel PR #275, "Multi-bit handling") through the
    weight-streaming gate|up and down kernels."""
    wl = mi.workload("decode_t32", T=32, wfmt="q8")
    layer, idx = _stage_setup(wl, 32, 31, 0.0)
    st = moe.sort_rows(idx.to(DEV), wl.E, 8)
    h = moe.grouped_swiglu(layer.x, st, wl.k, layer.experts, regime=1)
    ref_st = orc.sort_rows(idx.numpy(), wl.E, 8)
    hx = _host(layer.experts)
    href = orc.expert_swiglu(layer.x.cpu(), ref_st.row_map, ref_st.row_off, hx)
    g, u, ga, ua = orc.expert_gate_up(layer.x.cpu(), ref_st.row_map, ref_st.row_off, hx)
    # the SIMT kernel dequantises in fp32: 2^-24 per weight
    assert_h_close(h, href, g, u, ga, ua, wl.d, 2.0 ** -24, U_F16, TOL_BF16, "h[q8]")
    ys = moe.grouped_down(h, st, 32, wl.k, layer.experts, regime=1, dtype=layer.x.dtype)
    yref = orc.expert_down(to_np(h).astype(np.float64), ref_st.row_off, hx)
    habs = orc.expert_down_abs(to_np(h).astype(np.float64), ref_st.row_off, hx)
    assert_ys_close(ys, yref, habs, 2.0 ** -24, TOL_BF16, "ys[q8]", u_ys=U_F16, F=wl.F)


@pytest.mark.parametrize("name,T", [("decode_t1", 1), ("prefill", 64)])
def test_forward_q8(moe, orc, name, T):
    layer = mi.make_layer(mi.workload(name, T=T, wfmt="q8"), seed=9, device=DEV)
    _forward_and_compare(moe, orc, layer)


# ------------------------------------------------------------------ fp16 activations

@pytest.mark.parametrize("name,T", [("decode_t32", 32), ("prefill", 512), ("skewed", 300)])
def test_route_f16(moe, orc, name, T):
    """IEEE half activations and router weight: the weight-streaming router
    (32 tokens) and the tensor-core one (fp16 operands, 300 and 512 tokens)."""
    _check_route(moe, orc, mi.workload(name, T=T, act="f16"), T)


@pytest.mark.parametrize("name,T,regime,BM,wfmt", [
    ("decode_t32", 32, 1, 8, "q4"),          # mma.sync GEMV, x read in place
    ("decode_t32", 32, 1, 32, "q4"),         # SIMT GEMV (tiles above 16 rows)
    ("decode_t32", 32, 1, 8, "q8"),          # SIMT GEMV, 8-bit weights
    ("prefill", 600, 2, 128, "q4"),          # tcgen05 kernels, fp16 gather
])
def test_grouped_stages_f16(moe, orc, name, T, regime, BM, wfmt):
    wl = mi.workload(name, T=T, act="f16", wfmt=wfmt)
    layer, idx = _stage_setup(wl, T, 41, 0.2)
    assert layer.x.dtype == torch.float16
    st = moe.sort_rows(idx.to(DEV), wl.E, BM)
    h = moe.grouped_swiglu(layer.x, st, wl.k, layer.experts, regime=regime)
    assert h.dtype == torch.float16
    ref_st = orc.sort_rows(idx.numpy(), wl.E, BM)
    hx = _host(layer.experts)
    href = orc.expert_swiglu(layer.x.cpu(), ref_st.row_map, ref_st.row_off, hx)
    g, u, ga, ua = orc.expert_gate_up(layer.x.cpu(), ref_st.row_map, ref_st.row_off, hx)
    # the SIMT kernels dequantise in fp32, the tensor-core ones to fp16
    simt = BM > 16 or wfmt == "q8"
    u_w = 2.0 ** -24 if simt else U_F16
    assert_h_close(h, href, g, u, ga, ua, wl.d, u_w, U_F16, TOL_BF16, f"h[f16 {name} {wfmt}]")
    ys = moe.grouped_down(h, st, T, wl.k, layer.experts, regime=regime, dtype=layer.x.dtype)
    yref = orc.expert_down(to_np(h).astype(np.float64), ref_st.row_off, hx)
    habs = orc.expert_down_abs(to_np(h).astype(np.float64), ref_st.row_off, hx)
    assert_ys_close(ys, yref, habs, u_w, TOL_BF16, f"ys[f16 {name} {wfmt}]", u_ys=U_F16, F=wl.F)
    assert moe.device_status() == moe.OK


@pytest.mark.parametrize("name,T,wfmt", [("decode_t1", 1, "q4"), ("decode_t32", 32, "q4"),
                                         ("decode_t32", 32, "q4g128"), ("decode_t1", 1, "q8"),
                                         ("prefill", 300, "q4")])
def test_forward_f16(moe, orc, name, T, wfmt):
    """The whole layer on fp16 activations in the weight-streaming regime: the
    one-launch decode kernel (q4, up to 32 tokens), the separate
    weight-streaming stages (q8; 300 tokens)."""
    layer = mi.make_layer(mi.workload(name, T=T, act="f16", wfmt=wfmt), seed=12, device=DEV)
    y = moe.forward(layer.x, layer.w_router, layer.router_bias, layer.experts, layer.wl.k,
                    regime=1)
    assert y.dtype == torch.float16
    _forward_and_compare(moe, orc, layer, regime=1)
    assert moe.device_status() == moe.OK


def test_forward_f16_prefill_tensor_cores(moe, orc):
    layer = mi.make_layer(mi.workload("prefill", act="f16"), seed=13, device=DEV)
    rng = np.random.default_rng(5)
    _forward_and_compare(moe, orc, layer, sample=np.sort(rng.choice(2048, 64, replace=False)),
                         regime=2)
    assert moe.device_status() == moe.OK


def test_forward_deterministic(moe):
    layer = mi.make_layer("decode_t32", seed=3, device=DEV)
    a = moe.forward(layer.x, layer.w_router, None, layer.experts, layer.wl.k)
    b = moe.forward(layer.x, layer.w_router, None, layer.experts, layer.wl.k)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("name,regime", [("acceptance", 0), ("prefill", 0), ("decode_t1", 0),
                                         ("decode_t32", 1), ("decode_t32", 0)])
def test_forward_repeats_bit_exact(moe, name, regime):
    """Every path gives the same bits on every repeat (tensor-core kernels for
    acceptance, prefill and 32-token decode, the fused decode kernel for one
    token and for 32 when asked for). A raw weight
    stage released before the dequantising warps' shared-memory loads had
    read it let the next TMA overwrite its first rows under them: a few
    features of one tile came out wrong in about one run in five (bf16
    weights); 24 repeats catch a race of that rate with near certainty."""
    layer = mi.make_layer(name, seed=0, device=DEV)
    wl = layer.wl
    ws = moe.forward_workspace(layer.x, layer.experts, wl.k, regime)
    ref = moe.forward(layer.x, layer.w_router, layer.router_bias, layer.experts, wl.k,
                      regime=regime, ws=ws).clone()
    for _ in range(24):
        y = moe.forward(layer.x, layer.w_router, layer.router_bias, layer.experts, wl.k,
                        regime=regime, ws=ws)
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    assert moe.device_status() == moe.OK


def test_forward_zero_tokens(moe):
    layer = mi.make_layer(mi.workload("decode_t1", T=0), seed=0, device=DEV)
    y = moe.forward(layer.x, layer.w_router, None, layer.experts, 8)
    assert y.shape == (0, 2048)


def test_forward_intermediates_match_stage_calls(moe):
    """moe_forward's workspace holds the same routing and tables as the stage
    calls produce (bit-exact)."""
    layer = mi.make_layer("decode_t32", seed=4, device=DEV)
    wl = layer.wl
    ws = moe.forward_workspace(layer.x, layer.experts, wl.k)
    moe.forward(layer.x, layer.w_router, None, layer.experts, wl.k, ws=ws)
    L = moe.forward_layout(wl.T, wl.d, wl.E, wl.k, wl.F, layer.x.dtype, wl.wfmt)
    R = wl.T * wl.k
    seg = lambda off, n, dt: ws[off:off + n * 4].view(dt)
    _, idx, _ = moe.route(layer.x, layer.w_router, None, wl.k)
    assert torch.equal(seg(L.topk_idx, R, torch.int32), idx.view(-1))
    st = moe.sort_rows(idx, wl.E, L.BM)
    assert torch.equal(seg(L.order, R, torch.int32), st.order.view(torch.int32))
    assert torch.equal(seg(L.tile_off, wl.E + 1, torch.int32), st.tile_off)
    assert moe.device_status() == moe.OK


# ------------------------------------------------------------------ other formats on the tensor cores

TC_FORMAT_CASES = [
    # workload, T, weight format, activations, skew
    ("prefill", 600, "q4g32", "bf16", 0.3),
    ("prefill", 600, "q4g128", "bf16", 0.0),
    ("prefill", 600, "q8", "bf16", 0.3),
    ("prefill", 600, "q8", "f16", 0.0),
    ("skewed", 24, "q4g32", "bf16", 0.3),      # d = 7168: 28 raw stages per unit
]


@pytest.mark.parametrize("name,T,wfmt,act,skew", TC_FORMAT_CASES)
def test_tc_stages_other_formats(moe, orc, name, T, wfmt, act, skew):
    """q4 with groups of 32 and 128, and 8-bit affine weights, through the
    tcgen05 gate|up and down kernels (DS4Server issue #112, "Kernel
    contract": 4 or 8 bits, groups 32/64/128; mlxcel PR #275, "Multi-bit
    handling"). Weights are dequantised to fp16 operands (u_w = 2^-11)."""
    wl = mi.workload(name, T=T, wfmt=wfmt, act=act)
    layer, idx = _stage_setup(wl, T, 51, skew)
    st = moe.sort_rows(idx.to(DEV), wl.E, moe.sort_block_m())
    h = moe.grouped_swiglu(layer.x, st, wl.k, layer.experts, regime=moe.REGIME_TC)
    ref_st = orc.sort_rows(idx.numpy(), wl.E, moe.sort_block_m())
    hx = _host(layer.experts)
    href = orc.expert_swiglu(layer.x.cpu(), ref_st.row_map, ref_st.row_off, hx)
    g, u, ga, ua = orc.expert_gate_up(layer.x.cpu(), ref_st.row_map, ref_st.row_off, hx)
    assert_h_close(h, href, g, u, ga, ua, wl.d, U_F16, U_F16, TOL_BF16, f"h[{name} {wfmt} {act}]")
    ys = moe.grouped_down(h, st, T, wl.k, layer.experts, regime=moe.REGIME_TC, dtype=layer.x.dtype)
    yref = orc.expert_down(to_np(h).astype(np.float64), ref_st.row_off, hx)
    habs = orc.expert_down_abs(to_np(h).astype(np.float64), ref_st.row_off, hx)
    assert_ys_close(ys, yref, habs, U_F16, TOL_BF16, f"ys[{name} {wfmt} {act}]", u_ys=U_F16,
                    F=wl.F)
    assert moe.device_status() == moe.OK


@pytest.mark.parametrize("wfmt,act", [("q4g32", "bf16"), ("q4g128", "f16"), ("q8", "bf16")])
def test_forward_other_formats_tensor_cores(moe, orc, wfmt, act):
    """The whole layer at the prefill shape resolves to the tcgen05 kernels
    for these formats and matches the oracle on sampled tokens."""
    wl = mi.workload("prefill", wfmt=wfmt, act=act)
    L = moe.forward_layout(wl.T, wl.d, wl.E, wl.k, wl.F, mi._act_dtype(act), wfmt)
    assert L.regime == moe.REGIME_TC
    layer = mi.make_layer(wl, seed=17, device=DEV)
    rng = np.random.default_rng(7)
    _forward_and_compare(moe, orc, layer, sample=np.sort(rng.choice(wl.T, 48, replace=False)))
    assert moe.device_status() == moe.OK


@pytest.mark.parametrize("wfmt", ["q4g32", "q8"])
def test_forward_other_formats_repeat_bit_exact(moe, wfmt):
    layer = mi.make_layer(mi.workload("prefill", T=1024, wfmt=wfmt), seed=3, device=DEV)
    wl = layer.wl
    ws = moe.forward_workspace(layer.x, layer.experts, wl.k)
    ref = moe.forward(layer.x, layer.w_router, layer.router_bias, layer.experts, wl.k, ws=ws).clone()
    for _ in range(8):
        y = moe.forward(layer.x, layer.w_router, layer.router_bias, layer.experts, wl.k, ws=ws)
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    assert moe.device_status() == moe.OK
