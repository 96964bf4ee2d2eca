"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks one oracle step against something the oracle does not
compute itself: hand-worked fixtures from the format and routing definitions
(tests/golden/), library routines (numpy / torch fp64 matmuls, scipy softmax,
Python's sorted), closed forms, invariants, and a brute-force per-token loop.
Each is chosen so that a plausible slip in the oracle (a wrong nibble or
group index, a dropped bias, a transposed operand, a wrong tie-break, an
unstable sort, a swapped gate/up) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import moe_inputs as mi

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------ weight format

def _load_q4_fixture():
    words = {}
    groups = {}
    expect = []
    with open(os.path.join(GOLDEN, "q4_format.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            tok = line.split()
            if tok[0] == "words":
                words[int(tok[1])] = [int(w, 16) for w in tok[2:]]
            elif tok[0] == "group":
                groups[(int(tok[1]), int(tok[2]))] = (int(tok[3], 16), int(tok[4], 16))
            elif tok[0] == "expect":
                expect.append((int(tok[1]), int(tok[2]), float(tok[3])))
    return words, groups, expect


def test_q4_format_golden(orc):
    """Dequantisation of hand-made words matches the values worked by hand."""
    words, groups, expect = _load_q4_fixture()
    rows, cols = 2, 128
    w = np.array([words[r] for r in range(rows)], dtype=np.uint32).reshape(1, rows, cols // 8)
    s = np.zeros((1, rows, cols // 64), np.uint16)
    b = np.zeros((1, rows, cols // 64), np.uint16)
    for (r, g), (sv, bv) in groups.items():
        s[0, r, g] = sv
        b[0, r, g] = bv
    # as the "gu" matrix of an expert stack with 2F = 2 rows and d = 128
    ex = mi.Experts("q4", 1, cols, 1, torch.from_numpy(w.view(np.int32)).view(torch.uint32),
                    torch.zeros(1, cols, 1, dtype=torch.uint32),
                    torch.from_numpy(s.view(np.int16)).view(torch.bfloat16),
                    torch.from_numpy(b.view(np.int16)).view(torch.bfloat16), None, None)
    assert len(expect) >= 20
    for r, c, v in expect:
        assert orc.weight_value(ex, "gu", 0, r, c) == v, (r, c, v)


def test_q4_forward_equals_dense_forward_on_same_values(orc):
    """The oracle's q4 branch and its f32 branch agree on the whole layer when
    the f32 weights hold the dequantised values element by element (checks
    row/column/group indexing of the packed branch inside the matmuls)."""
    wl = mi.workload("tiny", T=6, d=128, E=3, k=2, F=64, wfmt="q4")
    L = mi.make_layer(wl, seed=3)
    ex = L.experts
    gu = np.empty((ex.E, 2 * ex.F, ex.d), np.float32)
    dn = np.empty((ex.E, ex.d, ex.F), np.float32)
    for e in range(ex.E):
        for r in range(2 * ex.F):
            for c in range(ex.d):
                gu[e, r, c] = orc.weight_value(ex, "gu", e, r, c)
        for r in range(ex.d):
            for c in range(ex.F):
                dn[e, r, c] = orc.weight_value(ex, "dn", e, r, c)
    dense = mi.Experts("f32", ex.E, ex.d, ex.F, torch.from_numpy(gu), torch.from_numpy(dn))
    a = orc.forward(L.x, L.w_router, L.router_bias, ex, wl.k)
    b = orc.forward(L.x, L.w_router, L.router_bias, dense, wl.k)
    np.testing.assert_array_equal(a.idx, b.idx)
    np.testing.assert_allclose(a.y, b.y, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("fmt", ["q4g32", "q4g128"])
def test_q4_other_group_sizes_dequantise_to_the_encoded_weights(orc, fmt):
    """Groups of 32 and 128 (DS4Server issue #112, "Kernel contract"): the
    oracle's value of every element is within half a quantisation step of the
    fp32 weight the generator encoded. A wrong group index takes another
    group's scale and bias and misses by far more than that (the groups are
    given very different ranges)."""
    G = mi.q4_group(fmt)
    K = 256
    torch.manual_seed(1)
    # group j spans [-(j + 1), j + 1] / 4: every group's scale and bias differ
    spread = (torch.arange(K // G, dtype=torch.float32) + 1.0).repeat_interleave(G) / 4
    w = (torch.rand(1, 3, K) * 2 - 1) * spread
    p, s, b = mi.quantize_q4g64(w, G)
    ex = mi.Experts(fmt, 1, K, 2, p, torch.zeros(1, K, 1, dtype=torch.uint32), s, b)
    for r in range(3):
        for c in range(K):
            step = float(s[0, r, c // G].float())
            got = orc.weight_value(ex, "gu", 0, r, c)
            assert abs(got - float(w[0, r, c])) <= 0.5 * step * (1 + 1e-2) + 1e-6, (r, c)


def test_q8_dequantises_to_the_encoded_weights(orc):
    """8-bit affine (mlxcel PR #275, "Multi-bit handling"): every element of
    the oracle's dequantisation is within half a quantisation step (plus the
    bf16 rounding of scale and bias) of the fp32 weight the generator encoded.
    A wrong byte index or group index takes another element's code or another
    group's scale and misses by far more."""
    K = 256
    torch.manual_seed(2)
    spread = (torch.arange(K // 64, dtype=torch.float32) + 1.0).repeat_interleave(64) / 4
    w = (torch.rand(1, 3, K) * 2 - 1) * spread
    p, s, b = mi.quantize_q8g64(w)
    ex = mi.Experts("q8", 1, K, 2, p, torch.zeros(1, K, 1, dtype=torch.uint32), s, b)
    for r in range(3):
        for c in range(K):
            step = float(s[0, r, c // 64].float())
            bias = float(b[0, r, c // 64].float())
            got = orc.weight_value(ex, "gu", 0, r, c)
            # half a step, plus what the bf16 rounding of scale (2^-9 relative,
            # over 255 steps) and bias can leave at the clamped ends of a group
            bound = 0.5 * step + 255 * step * 2.0 ** -9 + abs(bias) * 2.0 ** -8 + 1e-6
            assert abs(got - float(w[0, r, c])) <= bound, (r, c)


def test_q4_encoder_roundtrip_is_close(orc):
    """Generator sanity (not a pin of the oracle): dequantised weights stay
    within half a quantisation step of the fp32 weights they encode."""
    torch.manual_seed(0)
    w = torch.randn(1, 4, 128) / 8
    p, s, b = mi.quantize_q4g64(w)
    ex = mi.Experts("q4", 1, 128, 2, p, torch.zeros(1, 128, 1, dtype=torch.uint32), s, b)
    for r in range(4):
        for c in range(0, 128, 7):
            step = float(s[0, r, c // 64].float())
            assert abs(orc.weight_value(ex, "gu", 0, r, c) - float(w[0, r, c])) <= 0.5 * step + 1e-2 * step + 1e-6


# ------------------------------------------------------------ router logits

def test_logits_match_library_matmul(orc):
    for name, bias in (("tiny", False), ("tiny", True)):
        wl = mi.workload(name, bias="normal0.5" if bias else "none")
        L = mi.make_layer(wl, seed=1)
        got = orc.router_logits(L.x, L.w_router, L.router_bias)
        ref = L.x.double().numpy() @ L.w_router.double().numpy().T
        if L.router_bias is not None:
            ref = ref + L.router_bias.double().numpy()[None, :]
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_logits_bf16_match_library_matmul(orc):
    wl = mi.workload("decode_t32", d=256, E=16)
    L = mi.make_layer(wl, seed=2)
    got = orc.router_logits(L.x, L.w_router, None)
    ref = L.x.double().numpy() @ L.w_router.double().numpy().T
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_f16_activations_decode_every_finite_half(orc):
    """Every finite IEEE binary16 pattern, read as an activation against a
    unit router weight, comes back as its exact value: checked against
    Python's own half-precision unpacking and a few closed forms (1, the
    smallest subnormal 2^-24, the largest finite 65504, -2, a negative subnormal, the smallest normal)."""
    import struct
    bits = np.arange(65536, dtype=np.uint32)
    finite = ((bits >> 10) & 0x1F) != 0x1F
    bits = bits[finite].astype(np.uint16)
    x = bits.view(np.float16).reshape(-1, 1)
    got = orc.router_logits(x, np.ones((1, 1), np.float16), None)[:, 0]
    ref = np.array([struct.unpack("<e", struct.pack("<H", int(b)))[0] for b in bits])
    np.testing.assert_array_equal(got, ref)
    by_bits = dict(zip(bits.tolist(), got.tolist()))
    assert by_bits[0x3C00] == 1.0
    assert by_bits[0x0001] == 2.0 ** -24
    assert by_bits[0x7BFF] == 65504.0
    assert by_bits[0xC000] == -2.0
    assert by_bits[0x8001] == -(2.0 ** -24)
    assert by_bits[0x0400] == 2.0 ** -14       # smallest normal


@pytest.mark.parametrize("act", ["f16", "bf16"])
def test_16bit_forward_equals_f32_forward_on_same_values(orc, act):
    """The whole layer on 16-bit activations equals the layer on fp32
    activations holding the same values (both exact in fp32): the oracle reads
    x and the router weight through the 16-bit decoding at every use."""
    wl = mi.workload("tiny", T=7, d=128, E=4, k=2, F=64, wfmt="q4", act=act)
    L = mi.make_layer(wl, seed=4)
    a = orc.forward(L.x, L.w_router, L.router_bias, L.experts, wl.k)
    b = orc.forward(L.x.float(), L.w_router.float(), L.router_bias, L.experts, wl.k)
    np.testing.assert_array_equal(a.idx, b.idx)
    np.testing.assert_array_equal(a.y, b.y)
    np.testing.assert_array_equal(a.logits64, b.logits64)


def test_logits_f16_match_library_matmul(orc):
    wl = mi.workload("decode_t32", d=256, E=16, act="f16")
    L = mi.make_layer(wl, seed=2)
    assert L.x.dtype == torch.float16
    got = orc.router_logits(L.x, L.w_router, None)
    ref = L.x.double().numpy() @ L.w_router.double().numpy().T
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------ top-k

def _golden_topk_cases():
    cases = []
    with open(os.path.join(GOLDEN, "topk_cases.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            k, logits, idx, w = [p.strip() for p in line.split("|")]
            cases.append((int(k), [float(v) for v in logits.split()],
                          [int(v) for v in idx.split()], [float(v) for v in w.split()]))
    return cases


@pytest.mark.parametrize("case", _golden_topk_cases())
def test_topk_golden(orc, case):
    k, logits, idx, w = case
    got_idx, got_w = orc.topk(np.array([logits]), k)
    assert got_idx[0].tolist() == idx
    np.testing.assert_allclose(got_w[0], w, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("ties", [False, True])
@pytest.mark.parametrize("E,k", [(8, 2), (16, 5), (7, 7), (33, 8)])
def test_topk_bruteforce(orc, ties, E, k):
    """Selection equals a full sort by (value descending, index ascending)."""
    Lg = mi.random_logits(40, E, seed=E * 100 + k, ties=ties).double().numpy()
    idx, _ = orc.topk(Lg, k)
    for t in range(Lg.shape[0]):
        ranked = sorted(range(E), key=lambda e: (-Lg[t, e], e))
        assert idx[t].tolist() == ranked[:k]


def test_topk_weights_two_forms_agree(orc):
    """Softmax over the selection equals softmax over all experts
    renormalised over the selection (the full denominator cancels)."""
    for seed, (E, k) in enumerate([(8, 2), (128, 8), (512, 10), (256, 8)]):
        Lg = mi.random_logits(50, E, seed=seed).double().numpy() * 3
        idx, w = orc.topk(Lg, k)
        w2 = orc.topk_weights_full_softmax(Lg, idx)
        np.testing.assert_allclose(w, w2, rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-12)
        assert (np.diff(w, axis=1) <= 1e-15).all()      # best first


def test_topk_k_equals_E_is_plain_softmax(orc):
    Lg = mi.random_logits(30, 6, seed=9).double().numpy()
    idx, w = orc.topk(Lg, 6)
    p = scipy.special.softmax(Lg, axis=1)
    for t in range(30):
        np.testing.assert_allclose(w[t], p[t, idx[t]], rtol=1e-12, atol=1e-15)


def test_topk_rejects_bad_k(orc):
    with pytest.raises(ValueError):
        orc.topk(np.zeros((2, 4)), 5)
    with pytest.raises(ValueError):
        orc.topk(np.zeros((2, 4)), 0)


# ------------------------------------------------------------ sort

@pytest.mark.parametrize("T,E,k,BM,skew", [(16, 8, 2, 4, 0.0), (37, 16, 3, 8, 0.3),
                                            (200, 64, 8, 16, 0.15), (5, 128, 8, 64, 0.0),
                                            (1, 4, 4, 1, 0.0), (0, 8, 2, 4, 0.0)])
def test_sort_invariants_and_bruteforce(orc, T, E, k, BM, skew):
    idx = mi.random_topk_idx(T, E, k, seed=T + E, skew=skew).numpy()
    st = orc.sort_rows(idx, E, BM)
    R = T * k
    flat = idx.reshape(-1)
    brute = sorted(range(R), key=lambda r: (flat[r], r))
    assert st.order.tolist() == brute
    assert sorted(st.order.tolist()) == list(range(R))                  # permutation
    assert (st.inv_order[st.order] == np.arange(R)).all()               # inv o order = id
    assert (st.order[st.inv_order] == np.arange(R)).all()
    assert (st.row_map == st.order // k).all()
    assert (np.diff(flat[st.order]) >= 0).all()                         # grouped by expert
    np.testing.assert_array_equal(st.counts, np.bincount(flat, minlength=E))
    assert st.row_off[0] == 0 and st.row_off[E] == R
    np.testing.assert_array_equal(np.diff(st.row_off), st.counts)
    np.testing.assert_array_equal(np.diff(st.tile_off), -(-st.counts // BM))
    for e in range(E):                      # rows of one expert: tokens strictly increase
        rows = st.row_map[st.row_off[e]:st.row_off[e + 1]]
        assert (np.diff(rows.astype(np.int64)) > 0).all()


def test_sort_rejects_out_of_range_ids(orc):
    with pytest.raises(ValueError):
        orc.sort_rows(np.array([[0, 9]], np.int32), 8, 4)


# ------------------------------------------------------------ expert FFN

def _torch_dense_ffn(x, wgu, wdn):
    """One expert's SwiGLU FFN with torch fp64 matmuls and torch's silu."""
    F = wdn.shape[1]
    g = x @ wgu[:F].T
    u = x @ wgu[F:].T
    return torch.nn.functional.silu(g) * u, (torch.nn.functional.silu(g) * u) @ wdn.T


def test_single_expert_is_dense_swiglu_ffn(orc):
    """E = 1, k = 1: the layer is a plain SwiGLU FFN (w = 1)."""
    wl = mi.workload("tiny", T=9, d=64, E=1, k=1, F=128)
    L = mi.make_layer(wl, seed=4)
    r = orc.forward(L.x, L.w_router, None, L.experts, 1, keep_intermediates=True)
    x = L.x.double()
    h, y = _torch_dense_ffn(x, L.experts.w_gu[0].double(), L.experts.w_dn[0].double())
    np.testing.assert_allclose(r.w, 1.0)
    np.testing.assert_allclose(r.h, h.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(r.y, y.numpy(), rtol=1e-11, atol=1e-12)


def test_single_expert_is_dense_geglu_ffn(orc):
    """E = 1, k = 1 with the tanh-GELU GLU (mlx-lm PR #2044, "When it
    applies"): a plain GeGLU FFN, checked against torch's own tanh-form GELU
    on fp64 matmuls. A wrong constant or a dropped cubic term in the oracle's
    GELU fails this."""
    wl = mi.workload("tiny", T=9, d=64, E=1, k=1, F=128)
    L = mi.make_layer(wl, seed=4)
    ex = L.experts.with_act("geglu")
    r = orc.forward(L.x, L.w_router, None, ex, 1, keep_intermediates=True)
    x = L.x.double()
    wgu, wdn = ex.w_gu[0].double(), ex.w_dn[0].double()
    F = wl.F
    g, u = x @ wgu[:F].T, x @ wgu[F:].T
    h = torch.nn.functional.gelu(g, approximate="tanh") * u
    y = h @ wdn.T
    np.testing.assert_allclose(r.h, h.numpy(), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(r.y, y.numpy(), rtol=1e-11, atol=1e-12)
    # and it is not the SwiGLU result
    rs = orc.forward(L.x, L.w_router, None, L.experts, 1)
    assert np.abs(rs.y - r.y).max() > 1e-3 * np.abs(r.y).max()


@pytest.mark.parametrize("wfmt,act", [("f32", "f32"), ("bf16", "bf16")])
def test_dense_soft_routing_restricted_to_topk(orc, wfmt, act):
    """The sorted, grouped oracle equals a dense reference that runs every
    expert on every token (torch fp64 matmuls) and keeps only the selected
    experts' outputs times their weights -- no sort, no row map, no unsort."""
    wl = mi.workload("tiny", T=24, d=64, E=6, k=3, F=96, wfmt=wfmt, act=act, bias="normal0.5")
    L = mi.make_layer(wl, seed=5)
    r = orc.forward(L.x, L.w_router, L.router_bias, L.experts, wl.k, BM=4)
    x = L.x.double()
    y = torch.zeros(wl.T, wl.d, dtype=torch.float64)
    for e in range(wl.E):
        _, ye = _torch_dense_ffn(x, L.experts.w_gu[e].double(), L.experts.w_dn[e].double())
        mask = torch.from_numpy((r.idx == e).astype(np.float64))          # [T, k]
        gate = (mask * torch.from_numpy(r.w)).sum(dim=1, keepdim=True)   # w[t] if e selected
        y += gate * ye
    np.testing.assert_allclose(r.y, y.numpy(), rtol=1e-10, atol=1e-12)


def test_stage_functions_compose_to_forward(orc):
    """Calling the steps one by one gives the forward's result."""
    wl = mi.workload("tiny", T=10, d=64, E=5, k=2, F=64, wfmt="q4", act="bf16")
    L = mi.make_layer(wl, seed=6)
    r = orc.forward(L.x, L.w_router, None, L.experts, wl.k, BM=4, keep_intermediates=True)
    lg = orc.router_logits(L.x, L.w_router, None)
    np.testing.assert_array_equal(lg, r.logits64)
    idx, w = orc.topk(lg.astype(np.float32), wl.k)
    np.testing.assert_array_equal(idx, r.idx)
    st = orc.sort_rows(idx, wl.E, 4)
    h = orc.expert_swiglu(L.x, st.row_map, st.row_off, L.experts)
    np.testing.assert_array_equal(h, r.h)
    ys = orc.expert_down(h, st.row_off, L.experts)
    np.testing.assert_array_equal(ys, r.ys)
    y = orc.combine(ys, st.inv_order, w, wl.T, wl.k)
    np.testing.assert_array_equal(y, r.y)


def test_bruteforce_per_token_loop(orc):
    """Pure-Python per-token loops: rank experts, take k, run each expert's
    FFN with three nested loops, add with the weights."""
    wl = mi.workload("tiny", T=5, d=16, E=4, k=2, F=8)
    L = mi.make_layer(wl, seed=7)
    r = orc.forward(L.x, L.w_router, None, L.experts, wl.k)
    x = L.x.tolist()
    wr = L.w_router.tolist()
    gu = L.experts.w_gu.tolist()
    dn = L.experts.w_dn.tolist()
    for t in range(wl.T):
        logit = [float(np.float32(sum(x[t][i] * wr[e][i] for i in range(wl.d)))) for e in range(wl.E)]
        ranked = sorted(range(wl.E), key=lambda e: (-logit[e], e))[: wl.k]
        z = sum(math.exp(logit[e] - max(logit)) for e in ranked)
        out = [0.0] * wl.d
        for e in ranked:
            we = math.exp(logit[e] - max(logit)) / z
            h = []
            for f in range(wl.F):
                g = sum(x[t][i] * gu[e][f][i] for i in range(wl.d))
                u = sum(x[t][i] * gu[e][wl.F + f][i] for i in range(wl.d))
                h.append(g / (1 + math.exp(-g)) * u)
            for o in range(wl.d):
                out[o] += we * sum(h[f] * dn[e][o][f] for f in range(wl.F))
        assert r.idx[t].tolist() == ranked
        np.testing.assert_allclose(r.y[t], out, rtol=1e-9, atol=1e-12)


def test_combine_by_hand(orc):
    """y[t] = sum_j w[t,j] * ys[inv_order[t*k + j]] on a 2-token example."""
    ys = np.array([[1.0, 2.0], [10.0, 20.0], [100.0, 200.0], [1000.0, 2000.0]])
    inv = np.array([3, 0, 1, 2], np.uint32)     # token 0 -> rows 3, 0 ; token 1 -> rows 1, 2
    w = np.array([[0.5, 0.25], [2.0, -1.0]])
    y = orc.combine(ys, inv, w, 2, 2)
    np.testing.assert_array_equal(y, [[500.25, 1000.5], [-80.0, -160.0]])


def test_outputs_finite_on_workload_shapes(orc):
    for name in ("tiny",):
        L = mi.make_layer(name, seed=0)
        r = orc.forward(L.x, L.w_router, L.router_bias, L.experts, L.wl.k, keep_intermediates=True)
        assert np.isfinite(r.y).all() and np.isfinite(r.h).all() and np.isfinite(r.w).all()


def test_zero_tokens(orc):
    wl = mi.workload("tiny", T=0)
    L = mi.make_layer(wl, seed=0)
    r = orc.forward(L.x, L.w_router, None, L.experts, wl.k)
    assert r.y.shape == (0, wl.d)


@pytest.mark.slow
def test_zipf_bias_gives_stated_skew(orc):
    """The skewed workload's router bias yields experts with more than 10x the
    mean rows and experts with none (routing by the oracle's top-k on fp64
    logits from a library matmul)."""
    wl = mi.WORKLOADS["skewed"]
    gx = torch.Generator().manual_seed(0)
    x = torch.randn(wl.T, wl.d, generator=gx).to(torch.bfloat16).double().numpy()
    wr = (torch.randn(wl.E, wl.d, generator=gx) / math.sqrt(wl.d)).to(torch.bfloat16).double().numpy()
    b = mi.make_router_bias(wl, 0).double().numpy()
    idx, _ = orc.topk((x @ wr.T + b).astype(np.float32), wl.k)
    counts = np.bincount(idx.reshape(-1), minlength=wl.E)
    assert counts.max() > 10 * counts.mean()
    assert (counts == 0).any()


# ------------------------------------------------------------ error-bound helpers

def _decode_q4_by_definition(words, scales, biases, group):
    """A test-side decoding of 4-bit affine weights written from the format's
    definition alone: element j of a 32-bit word is bits [4j, 4j+3], groups of
    `group` consecutive input elements share one bf16 scale and bias, value =
    scale * q + bias. Shares nothing with the oracle's decoder."""
    w = words.view(torch.int32).numpy().astype(np.int64) & 0xFFFFFFFF      # [..., K/8]
    q = np.stack([(w >> (4 * j)) & 0xF for j in range(8)], axis=-1)        # [..., K/8, 8]
    q = q.reshape(*w.shape[:-1], w.shape[-1] * 8).astype(np.float64)       # [..., K]
    s = np.repeat(scales.double().numpy(), group, axis=-1)
    b = np.repeat(biases.double().numpy(), group, axis=-1)
    return s * q + b


def _expert_weights_fp64(ex, which):
    """[E, rows, cols] fp64 values of an expert stack ("gu" or "dn")."""
    w = ex.w_gu if which == "gu" else ex.w_dn
    if mi.q4_group(ex.fmt):
        s, b = (ex.s_gu, ex.b_gu) if which == "gu" else (ex.s_dn, ex.b_dn)
        return _decode_q4_by_definition(w, s, b, mi.q4_group(ex.fmt))
    return w.double().numpy()


def _routed_tables(orc, T, E, k, seed):
    """Sort tables of a skewed random routing with at least one empty expert,
    so that row_map is not the identity and expert blocks differ in size."""
    idx = mi.random_topk_idx(T, E - 1, k, seed=seed, skew=0.6).numpy()
    idx = np.where(idx >= 2, idx + 1, idx).astype(np.int32)        # expert 2 gets no rows
    st = orc.sort_rows(idx, E, 4)
    assert (st.counts == 0).any() and len(set(st.counts.tolist())) > 2
    assert (st.row_map != np.arange(T * k) // k).any()
    return st


@pytest.mark.parametrize("wfmt,act", [("f32", "f32"), ("bf16", "bf16"), ("q4", "bf16"),
                                      ("q4g32", "f16")])
def test_expert_gate_up_against_library_matmul(orc, wfmt, act):
    """orc.expert_gate_up (the pre-activations and the absolute-product sums
    the GPU parity tests build their per-element bounds from) against torch
    fp64 matmuls on a test-side decoding of the weights: for every expert e
    and its sorted rows i, with X = x[row_map[i]],
        g = X Wg_e^T, u = X Wu_e^T, ga = |X| |Wg_e|^T, ua = |X| |Wu_e|^T,
    Wg_e = rows 0..F-1 and Wu_e = rows F..2F-1 of expert e's fused block.
    A swapped gate/up, a dropped fabs, a row read without row_map or another
    expert's weights each fail it. And h from orc.expert_swiglu is silu(g) u
    from torch's silu on the same g and u."""
    T, E, k, d, F = 40, 6, 3, 128, 64
    wl = mi.workload("tiny", T=T, d=d, E=E, k=k, F=F, wfmt=wfmt, act=act)
    L = mi.make_layer(wl, seed=17)
    st = _routed_tables(orc, T, E, k, seed=18)
    g, u, ga, ua = orc.expert_gate_up(L.x, st.row_map, st.row_off, L.experts)
    W = _expert_weights_fp64(L.experts, "gu")                       # [E, 2F, d]
    x = L.x.double().numpy()
    for e in range(E):
        r0, r1 = int(st.row_off[e]), int(st.row_off[e + 1])
        X = torch.from_numpy(x[st.row_map[r0:r1].astype(np.int64)])
        Wg, Wu = torch.from_numpy(W[e, :F]), torch.from_numpy(W[e, F:])
        for got, want in ((g, X @ Wg.T), (u, X @ Wu.T), (ga, X.abs() @ Wg.abs().T),
                          (ua, X.abs() @ Wu.abs().T)):
            np.testing.assert_allclose(got[r0:r1], want.numpy(), rtol=1e-12, atol=1e-13)
    assert (ga >= np.abs(g)).all() and (ua >= np.abs(u)).all()
    h = orc.expert_swiglu(L.x, st.row_map, st.row_off, L.experts)
    gt, ut = torch.from_numpy(g), torch.from_numpy(u)
    np.testing.assert_allclose(h, (torch.nn.functional.silu(gt) * ut).numpy(), rtol=1e-12,
                               atol=1e-14)


@pytest.mark.parametrize("wfmt", ["f32", "q4", "q4g128"])
def test_expert_down_and_abs_against_library_matmul(orc, wfmt):
    """orc.expert_down and orc.expert_down_abs against torch fp64 matmuls on a
    test-side decoding of the weights: for the sorted rows i of expert e,
    ys = h Wd_e^T and |h| |Wd_e|^T. Rows of h carry random signs, so a
    dropped fabs changes the sums; the expert blocks differ in size, so a
    wrong row_off or expert fails."""
    T, E, k, d, F = 30, 5, 2, 128, 128
    wl = mi.workload("tiny", T=T, d=d, E=E, k=k, F=F, wfmt=wfmt,
                     act="f32" if wfmt == "f32" else "bf16")
    L = mi.make_layer(wl, seed=19)
    st = _routed_tables(orc, T, E, k, seed=20)
    h = mi.random_rows(T * k, F, seed=21, dtype=torch.float32).double().numpy()
    assert (h < 0).any() and (h > 0).any()
    ys = orc.expert_down(h, st.row_off, L.experts)
    habs = orc.expert_down_abs(h, st.row_off, L.experts)
    W = _expert_weights_fp64(L.experts, "dn")                       # [E, d, F]
    for e in range(E):
        r0, r1 = int(st.row_off[e]), int(st.row_off[e + 1])
        H, Wd = torch.from_numpy(h[r0:r1]), torch.from_numpy(W[e])
        np.testing.assert_allclose(ys[r0:r1], (H @ Wd.T).numpy(), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(habs[r0:r1], (H.abs() @ Wd.abs().T).numpy(), rtol=1e-12,
                                   atol=1e-13)
    assert (habs >= np.abs(ys)).all()
