"""Comparison rules shared by the GPU parity tests (test-side only)."""
import numpy as np
import torch

# bf16 activations: max |gpu - oracle| <= 2e-2 * RMS(oracle)
TOL_BF16 = 2e-2
# unit roundoff of fp16 (11-bit precision): the expert GEMMs' operand format
# for bf16 activations, and the storage of h
U_F16 = 2.0 ** -11
# fp32 activations and weights throughout: fp32 accumulation and one fp32
# rounding per stored value, against fp64 -> 1e-4 * RMS leaves > 100x margin
TOL_F32 = 1e-4


def to_np(t):
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu()
        if t.dtype == torch.bfloat16:
            t = t.float()
        if t.dtype == torch.uint32:
            return t.view(torch.int32).numpy().view(np.uint32)
        return t.numpy()
    return np.asarray(t)


def rms(a) -> float:
    a = np.asarray(a, dtype=np.float64)
    return float(np.sqrt(np.mean(a * a))) if a.size else 0.0


def assert_close_rms(gpu, ref, tol, what="", rounded_to=None):
    """max |gpu - ref| <= tol * RMS(ref). With rounded_to="bf16" (an
    intermediate the kernel stores in bf16) each element may in addition
    differ by one bf16 rounding of its own value, 2^-8 * |ref| (twice the
    half-ulp bound, for the fp32 error it is added to)."""
    g = to_np(gpu).astype(np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite GPU output"
    if r.size == 0:
        return 0.0
    err = np.abs(g - r)
    bound = tol * rms(r)
    if rounded_to == "bf16":
        excess = err - (bound + 2.0 ** -8 * np.abs(r))
        i = int(np.argmax(excess))
        assert excess.flat[i] <= 0, (f"{what}: |err| {err.flat[i]:.3e} at {i} (ref {r.flat[i]:.4e}) > "
                                     f"{tol} * RMS {rms(r):.3e} + 2^-8 |ref|")
    else:
        e = float(err.max())
        assert e <= bound, f"{what}: max|err| {e:.3e} > {tol} * RMS {rms(r):.3e} = {bound:.3e}"
    return float(err.max()) / max(rms(r), 1e-300)


def topk_ref(logits_np, k):
    """Top-k by (value descending, index ascending), -0 == +0, NaN last;
    Python's sorted, for property checks of GPU output."""
    T, E = logits_np.shape
    out = np.empty((T, k), np.int32)
    for t in range(T):
        row = logits_np[t]
        key = lambda e: (1, 0.0, e) if np.isnan(row[e]) else (0, -float(row[e]), e)
        out[t] = sorted(range(E), key=key)[:k]
    return out


def kth_gap(logits_np, k):
    """Smallest gap between neighbouring ranks among the k+1 largest logits of
    each token: a selection (or its best-first order) can change only where
    such a gap is within the logit error."""
    s = -np.sort(-logits_np.astype(np.float64), axis=1)
    m = min(k + 1, logits_np.shape[1])
    if m < 2:
        return np.full(logits_np.shape[0], np.inf)
    return (s[:, : m - 1] - s[:, 1:m]).min(axis=1)


def _act_and_slope(g, act):
    """The gate activation and its derivative: silu, or the tanh form of GELU
    (0.5 g (1 + tanh(z)), z = sqrt(2/pi) (g + 0.044715 g^3))."""
    if act == "geglu":
        c = np.sqrt(2.0 / np.pi)
        th = np.tanh(c * (g + 0.044715 * g ** 3))
        a = 0.5 * g * (1.0 + th)
        da = 0.5 * (1.0 + th) + 0.5 * g * (1.0 - th * th) * c * (1.0 + 3 * 0.044715 * g * g)
        return a, da
    sig = 1.0 / (1.0 + np.exp(-g))
    return g * sig, sig * (1.0 + g * (1.0 - sig))


def assert_h_close(h_gpu, href, g, u, ga, ua, d, u_w, u_h, tol, what="", act="swiglu"):
    """h = act(g) * u as the kernels compute it: weights rounded to the
    operand format before the products (unit roundoff u_w, so |dg| <= u_w *
    sum |x w|; 0 when the weights are exact in it), products accumulated in
    fp32 (2 d 2^-24 * sum |x w| with margin), h rounded once to its storage
    format (u_h |h|). The first-order bound per element is
        tol * RMS(h) + u_h |h| + |u act'(g)| dg + |act(g)| du."""
    gh = to_np(h_gpu).astype(np.float64)
    assert gh.shape == href.shape, (what, gh.shape, href.shape)
    assert np.isfinite(gh).all(), f"{what}: non-finite GPU output"
    if href.size == 0:
        return 0.0
    acc = 2.0 * d * 2.0 ** -24
    dg = (u_w + acc) * ga
    du = (u_w + acc) * ua
    a, da = _act_and_slope(g, act)
    bound = tol * rms(href) + u_h * np.abs(href) + np.abs(u * da) * dg + np.abs(a) * du
    err = np.abs(gh - href)
    i = int(np.argmax(err - bound))
    assert err.flat[i] <= bound.flat[i], (f"{what}: |err| {err.flat[i]:.3e} at {i} "
                                          f"(ref {href.flat[i]:.4e}) > bound {bound.flat[i]:.3e}")
    return float(err.max()) / max(rms(href), 1e-300)


def assert_ys_close(ys_gpu, yref, habs, u_w, tol, what="", u_ys=0.0):
    """ys = h . W_d^T accumulated in fp32: weights rounded to the operand
    format (unit roundoff u_w) add at most u_w * sum |h w|; storing ys in a
    format of unit roundoff u_ys adds u_ys * |ys| (+ half its smallest
    subnormal step, 2^-25 for fp16)."""
    g = to_np(ys_gpu).astype(np.float64)
    assert g.shape == yref.shape and np.isfinite(g).all(), what
    if yref.size == 0:
        return 0.0
    bound = tol * rms(yref) + u_w * habs
    if u_ys:
        bound = bound + u_ys * np.abs(yref) + 2.0 ** -25
    err = np.abs(g - yref)
    i = int(np.argmax(err - bound))
    assert err.flat[i] <= bound.flat[i], (f"{what}: |err| {err.flat[i]:.3e} at {i} "
                                          f"(ref {yref.flat[i]:.4e}) > bound {bound.flat[i]:.3e}")
    return float(err.max()) / max(rms(yref), 1e-300)
