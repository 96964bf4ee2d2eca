"""moe_sort_rows_noalloc: the dispatch sort for callers that cannot allocate
device memory (a host framework that owns all device memory and gives an
operator no allocator or workspace). It keeps its scratch in a static device
array inside the library instead of a caller workspace; its results must be
the same, bit for bit, as moe_sort_rows with a workspace, and a second call
must not see anything left over from the first (the array is shared by every
call). Collected last so a run that stops at the first failure has already
run every other test."""
import ctypes

import numpy as np
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


def _noalloc(moe, idx, E, BM):
    T, k = idx.shape
    R = T * k
    dev = idx.device
    out = {n: torch.empty(R, dtype=torch.uint32, device=dev) for n in ("order", "inv_order", "row_map")}
    out["counts"] = torch.full((E,), -1, dtype=torch.int32, device=dev)
    out["row_off"] = torch.full((E + 1,), -1, dtype=torch.int32, device=dev)
    out["tile_off"] = torch.full((E + 1,), -1, dtype=torch.int32, device=dev)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = moe.lib.moe_sort_rows_noalloc(p(idx), T, k, E, BM, p(out["order"]), p(out["inv_order"]),
                                       p(out["row_map"]), p(out["counts"]), p(out["row_off"]),
                                       p(out["tile_off"]), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == moe.OK, moe.status_str(st)
    return out


def test_noalloc_sort_matches_workspace_sort_on_two_calls_in_a_row(moe):
    # first call: a multi-chunk sort with skew and empty experts (the path
    # that uses the scratch); second call: different sizes and ids, so any
    # stale per-chunk count from the first call would change the result
    cases = [(2048, 512, 10, 128, 0.02, 1), (1500, 64, 6, 64, 0.3, 2)]
    # then the documented limit, which fills the whole scratch: 32,768 rows
    # (32 chunks) over 1,024 experts
    cases.append((4096, 1024, 8, 128, 0.0, 3))
    for T, E, k, BM, skew, seed in cases:
        idx = mi.random_topk_idx(T, E, k, seed=seed, skew=skew).cuda()
        got = _noalloc(moe, idx, E, BM)
        ref = moe.sort_rows(idx, E, BM)
        torch.cuda.synchronize()
        for name in ("order", "inv_order", "row_map", "counts", "row_off", "tile_off"):
            a = got[name].cpu().view(torch.int32).numpy()
            b = getattr(ref, name).cpu().view(torch.int32).numpy()
            np.testing.assert_array_equal(a, b, err_msg=name)


def test_noalloc_sort_rejects_sizes_beyond_its_scratch(moe):
    fake = ctypes.c_void_p(0x10000)
    # 32768 rows is the limit; 32769 is refused on the host, before any launch
    assert moe.lib.moe_sort_rows_noalloc(fake, 32769, 1, 8, 128, fake, fake, fake, fake, fake,
                                         fake, None) == moe.ERR_UNSUPPORTED
    # 1,024 experts is the limit; 1,025 is refused the same way
    assert moe.lib.moe_sort_rows_noalloc(fake, 16, 2, 1025, 128, fake, fake, fake, fake, fake,
                                         fake, None) == moe.ERR_UNSUPPORTED
