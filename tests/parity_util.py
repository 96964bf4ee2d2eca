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


def assert_close_rms(gpu, ref, tol, what=""):
    """max |gpu - ref| <= tol * RMS(ref)."""
    g = to_np(gpu).astype(np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite GPU output"
    if r.size == 0:
        return 0.0
    e = float(np.abs(g - r).max())
    bound = tol * rms(r)
    assert e <= bound, f"{what}: max|err| {e:.3e} > {tol} * RMS {rms(r):.3e} = {bound:.3e}"
    return e / max(rms(r), 1e-300)


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


def _check_stage(gpu, ref, elem_bound, tol, what):
    """The two rules every intermediate stage (h, ys) must meet:
    (a) the contract's rule for floating outputs, max |gpu - ref| <= tol *
        RMS(ref), over the whole tensor; and
    (b) per element, |gpu - ref| <= 2 * (the first-order effect of the
        roundings the kernel documents) + 1e-3 * RMS(ref). The factor 2 and
        the small floor cover second-order terms and fp16 subnormals; (b) is
        far tighter than (a) for most elements, so an error confined to a few
        small elements (a wrong token row, a swapped feature) fails it even
        where it stays under (a)."""
    g = to_np(gpu).astype(np.float64)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite GPU output"
    if ref.size == 0:
        return 0.0
    err = np.abs(g - ref)
    r = rms(ref)
    e = float(err.max())
    assert e <= tol * r, f"{what}: max|err| {e:.3e} > {tol} * RMS {r:.3e} = {tol * r:.3e}"
    bound = 2.0 * elem_bound + 1e-3 * r
    i = int(np.argmax(err - bound))
    assert err.flat[i] <= bound.flat[i], (f"{what}: |err| {err.flat[i]:.3e} at {i} "
                                          f"(ref {ref.flat[i]:.4e}) > per-element bound "
                                          f"{bound.flat[i]:.3e}")
    return e / max(r, 1e-300)


def assert_h_close(h_gpu, href, g, u, ga, ua, d, u_w, u_h, tol, what="", act="swiglu"):
    """h = act(g) * u as the kernels compute it: weights rounded to the
    operand format before the products (unit roundoff u_w, so |dg| <= u_w *
    sum |x w|; 0 when the weights are exact in it), d products accumulated in
    fp32 (at most d 2^-24 * sum |x w|), h rounded once to its storage format
    (u_h |h|). The first-order effect per element is
        u_h |h| + |u act'(g)| dg + |act(g)| du,
    checked as _check_stage's rule (b), next to the contract's rule (a)."""
    href = np.asarray(href, dtype=np.float64)
    acc = d * 2.0 ** -24
    dg = (u_w + acc) * ga
    du = (u_w + acc) * ua
    a, da = _act_and_slope(g, act)
    elem = u_h * np.abs(href) + np.abs(u * da) * dg + np.abs(a) * du
    return _check_stage(h_gpu, href, elem, tol, what)


def assert_ys_close(ys_gpu, yref, habs, u_w, tol, what="", u_ys=0.0, F=0):
    """ys = h . W_d^T accumulated in fp32 over F products: weights rounded to
    the operand format (unit roundoff u_w) add at most u_w * sum |h w|, the
    fp32 sum at most F 2^-24 * sum |h w|, and storing ys in a format of unit
    roundoff u_ys adds u_ys |ys| (+ half the smallest fp16 subnormal step,
    2^-25). Checked as _check_stage's rules (a) and (b)."""
    yref = np.asarray(yref, dtype=np.float64)
    assert F > 0, "F: the length of the down projection's sums"
    elem = (u_w + F * 2.0 ** -24) * habs
    if u_ys:
        elem = elem + u_ys * np.abs(yref) + 2.0 ** -25
    return _check_stage(ys_gpu, yref, elem, tol, what)
