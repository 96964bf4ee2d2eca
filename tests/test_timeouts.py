"""Failure detection on the device: every wait in the library's kernels is
bounded, and a wait that runs out records MOE_ERR_TIMEOUT in the device status
word and lets the kernel return, leaving the context usable.

No GPU is faulted, trapped or hung here. The waits are made to run out in two
ways: (1) a one-block self-test kernel whose single wait can never be met (an
mbarrier given one of its two arrivals; a grid barrier of a one-CTA grid
waiting for a second arrival), with a bound of a million cycles; (2) real
forwards run with a bound of one cycle (moe_set_wait_cycles), so that the
first wait that is not already satisfied gives up and the kernel takes its
abort path: every role leaves its loop, the copies and MMAs in flight are
waited for with the full bound, tensor memory is released. The next forward
with the default bound must give the same bits as before."""
import ctypes

import pytest
import torch

import moe_inputs as mi

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def moe():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import sparse_mixture_experts_top_b200 as m
    return m


@pytest.mark.parametrize("which", [0, 1, 2],
                         ids=["tc_mbarrier", "decode_mbarrier", "decode_grid_barrier"])
def test_selftest_wait_runs_out(moe, which):
    assert moe.device_status() == moe.OK
    scratch = torch.zeros(4, dtype=torch.int32, device="cuda")
    st = moe.lib.moe_selftest_wait_timeout(which, 1_000_000, ctypes.c_void_p(scratch.data_ptr()),
                                           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == moe.OK, moe.status_str(st)
    torch.cuda.synchronize()
    assert moe.device_status() == moe.ERR_TIMEOUT
    assert moe.device_status() == moe.OK          # reading cleared it


def test_selftest_rejects_bad_arguments(moe):
    P = ctypes.c_void_p
    assert moe.lib.moe_selftest_wait_timeout(3, 1000, None, None) == moe.ERR_INVALID_ARG
    assert moe.lib.moe_selftest_wait_timeout(0, 0, None, None) == moe.ERR_INVALID_ARG
    assert moe.lib.moe_selftest_wait_timeout(2, 1000, None, None) == moe.ERR_INVALID_ARG
    assert moe.lib.moe_set_wait_cycles(-1) == moe.ERR_INVALID_ARG


def _bits(y):
    return y.view(torch.int16) if y.dtype != torch.float32 else y.view(torch.int32)


@pytest.mark.parametrize("name,T,regime", [
    ("prefill", 600, 2),        # router, gate|up and down on the tcgen05 kernels
    ("decode_t32", 32, 1),      # the one-launch fused decode kernel (grid barriers)
])
def test_forward_aborts_on_short_bound_and_recovers(moe, name, T, regime):
    layer = mi.make_layer(mi.workload(name, T=T), seed=41, device="cuda")
    wl = layer.wl
    ws = moe.forward_workspace(layer.x, layer.experts, wl.k, regime)
    fwd = lambda: moe.forward(layer.x, layer.w_router, layer.router_bias, layer.experts, wl.k,
                              regime=regime, ws=ws)
    ref = fwd().clone()
    torch.cuda.synchronize()
    assert moe.device_status() == moe.OK
    seen = []
    try:
        moe.set_wait_cycles(1)
        for _ in range(3):
            fwd()
            torch.cuda.synchronize()
            seen.append(moe.device_status())
            if seen[-1] == moe.ERR_TIMEOUT:
                break
    finally:
        moe.set_wait_cycles(0)
    assert seen[-1] == moe.ERR_TIMEOUT, seen
    # the context is usable and the next forward is exact again
    y = fwd()
    torch.cuda.synchronize()
    assert moe.device_status() == moe.OK
    assert torch.equal(_bits(y), _bits(ref))
