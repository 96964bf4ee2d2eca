"""CPU checks of the comparison rules the GPU parity tests apply to the
intermediate stages (tests/parity_util.py): an emulation of the roundings the
tensor-core kernels document must pass them, and small corruptions confined
to a few elements must not."""
import numpy as np
import pytest
import torch

import moe_inputs as mi
from parity_util import TOL_BF16, U_F16, assert_h_close, assert_ys_close


def _decode_q4(words, scales, biases, group):
    # element j of a word is bits [4j, 4j+3]; value = scale * q + bias per group
    w = words.view(torch.int32).numpy().astype(np.int64) & 0xFFFFFFFF
    q = np.stack([(w >> (4 * j)) & 0xF for j in range(8)], axis=-1)
    q = q.reshape(*w.shape[:-1], w.shape[-1] * 8).astype(np.float64)
    return np.repeat(scales.double().numpy(), group, -1) * q + np.repeat(biases.double().numpy(), group, -1)


@pytest.fixture(scope="module")
def case(orc):
    wl = mi.workload("prefill", T=48, d=256, E=4, k=2, F=128)
    L = mi.make_layer(wl, seed=31)
    idx = mi.random_topk_idx(wl.T, wl.E, wl.k, seed=32, skew=0.3).numpy()
    st = orc.sort_rows(idx, wl.E, 4)
    ex = L.experts
    href = orc.expert_swiglu(L.x, st.row_map, st.row_off, ex)
    g, u, ga, ua = orc.expert_gate_up(L.x, st.row_map, st.row_off, ex)
    # the kernels' arithmetic: fp16 operands (x exact, weights rounded to
    # fp16), fp32 accumulation, silu in fp32, h rounded to fp16
    Wgu = torch.from_numpy(_decode_q4(ex.w_gu, ex.s_gu, ex.b_gu, 64)).half().float()
    x16 = L.x.float().half().float()
    h16 = np.empty_like(href)
    for e in range(wl.E):
        r0, r1 = int(st.row_off[e]), int(st.row_off[e + 1])
        X = x16[torch.from_numpy(st.row_map[r0:r1].astype(np.int64))]
        gg, uu = X @ Wgu[e, :wl.F].T, X @ Wgu[e, wl.F:].T
        h16[r0:r1] = (torch.nn.functional.silu(gg) * uu).half().double().numpy()
    return wl, st, ex, href, (g, u, ga, ua), h16


def test_emulated_kernel_roundings_pass(case):
    wl, _, _, href, (g, u, ga, ua), h16 = case
    assert_h_close(torch.from_numpy(h16), href, g, u, ga, ua, wl.d, U_F16, U_F16, TOL_BF16, "h")


def test_small_local_corruption_fails(case):
    """An error of 1 % of RMS(h) on one small element stays under the
    contract's 2e-2 * RMS rule but fails the per-element rule."""
    wl, _, _, href, (g, u, ga, ua), h16 = case
    bad = h16.copy()
    i = int(np.argmin(np.abs(href)))
    bad.flat[i] += 1e-2 * float(np.sqrt(np.mean(href ** 2)))
    with pytest.raises(AssertionError, match="per-element"):
        assert_h_close(torch.from_numpy(bad), href, g, u, ga, ua, wl.d, U_F16, U_F16, TOL_BF16, "h")


def test_swapped_rows_fail(case):
    wl, st, _, href, (g, u, ga, ua), h16 = case
    bad = h16.copy()
    bad[[0, 1]] = bad[[1, 0]]
    with pytest.raises(AssertionError):
        assert_h_close(torch.from_numpy(bad), href, g, u, ga, ua, wl.d, U_F16, U_F16, TOL_BF16, "h")


def test_down_emulation_passes_and_corruption_fails(orc, case):
    wl, st, ex, _, _, h16 = case
    yref = orc.expert_down(h16, st.row_off, ex)
    habs = orc.expert_down_abs(h16, st.row_off, ex)
    Wd = torch.from_numpy(_decode_q4(ex.w_dn, ex.s_dn, ex.b_dn, 64)).half().float()
    H = torch.from_numpy(h16).float()
    ys = np.empty_like(yref)
    for e in range(wl.E):
        r0, r1 = int(st.row_off[e]), int(st.row_off[e + 1])
        ys[r0:r1] = (H[r0:r1] @ Wd[e].T).half().double().numpy()
    assert_ys_close(torch.from_numpy(ys), yref, habs, U_F16, TOL_BF16, "ys", u_ys=U_F16, F=wl.F)
    bad = ys.copy()
    i = int(np.argmin(np.abs(yref)))
    bad.flat[i] += 1e-2 * float(np.sqrt(np.mean(yref ** 2)))
    with pytest.raises(AssertionError, match="per-element"):
        assert_ys_close(torch.from_numpy(bad), yref, habs, U_F16, TOL_BF16, "ys", u_ys=U_F16, F=wl.F)
