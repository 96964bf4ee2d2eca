"""Seeded synthetic inputs for the hard-routed sparse MoE layer forward.

This module is shared by the oracle-side tests and by the CUDA-side tests and
benchmark. It only *creates* data: random activations, router weights and
expert weights of the workloads' shapes and distributions, and the 4-bit
affine encoder that turns fp32 expert weights into the packed input format.
It holds none of the layer's arithmetic (no logits, no softmax, no top-k, no
sort, no dequantisation, no expert matmul, no combine).

Workloads (shapes and value distributions):

* ``tiny``       T=16   d=128  E=8   k=2  F=256  fp32 activations and weights
* ``acceptance`` T=512  d=2048 E=8   k=2  F=5632 bf16 activations and weights
                 (the acceptance shape of "5.5 real sparse MoE kernels
                 (Metal)", section "Scope -- in": 8 experts, top-2, d_model 2048)
* ``decode_t1`` / ``decode_t32``  T=1 / T=32, d=2048 E=128 k=8 F=768, q4 experts
* ``prefill``    T=2048 d=2048 E=512 k=10 F=512, q4 experts, router bias
                 N(0, 0.5) per expert (the 2,048-token chunk, 20,480 routed rows,
                 of DS4Server issue #112, "Kernel contract")
* ``skewed``     T=4096 d=7168 E=256 k=8 F=2048, q4 experts, Zipf(s=1.1)
                 expert-popularity bias on the router logits

Expert weights are drawn N(0, 1/d_in), activations N(0, 1), the router weight
N(0, 1/d). Values are rounded to bf16 wherever the workload says bf16.

Storage layouts (all row-major, the library's canonical format):

* ``x``         [T, d]
* ``w_router``  [E, d]   (row e holds column e of the router matrix W_r [d, E])
* ``router_bias`` [E] fp32 or None
* unquantised experts: ``w_gu`` [E, 2F, d] (rows 0..F-1 gate, F..2F-1 up),
  ``w_dn`` [E, d, F]
* q4 experts: ``w_gu`` uint32 [E, 2F, d/8], ``s_gu``/``b_gu`` bf16 [E, 2F, d/64],
  ``w_dn`` uint32 [E, d, F/8], ``s_dn``/``b_dn`` bf16 [E, d, F/64];
  element j of a 32-bit word sits in bits [4j, 4j+3] (low nibble first),
  group g covers input elements [64g, 64g+63].
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

GROUP = 64

# tensor ids used to derive independent sub-seeds
_TID_X, _TID_WR, _TID_BIAS, _TID_GU, _TID_DN, _TID_PERM = 1, 2, 3, 4, 5, 6
_TID_IDX, _TID_LOGITS, _TID_H, _TID_YS, _TID_W = 7, 8, 9, 10, 11


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    F: int
    act: str          # "f32" | "bf16" | "f16"
    wfmt: str         # "f32" | "bf16" | "q4" (group 64) | "q4g32" | "q4g128" | "q8"
    bias: str = "none"  # "none" | "normal0.5" | "zipf1.1"
    note: str = ""

    @property
    def R(self) -> int:
        return self.T * self.k


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 16, 128, 8, 2, 256, "f32", "f32"),
        Workload("acceptance", 512, 2048, 8, 2, 5632, "bf16", "bf16"),
        Workload("decode_t1", 1, 2048, 128, 8, 768, "bf16", "q4"),
        Workload("decode_t32", 32, 2048, 128, 8, 768, "bf16", "q4"),
        Workload("prefill", 2048, 2048, 512, 10, 512, "bf16", "q4", "normal0.5"),
        Workload("skewed", 4096, 7168, 256, 8, 2048, "bf16", "q4", "zipf1.1"),
    ]
}


def workload(name: str, **overrides) -> Workload:
    base = WORKLOADS[name]
    if not overrides:
        return base
    d = dict(base.__dict__)
    d.update(overrides)
    return Workload(**d)


def _gen(seed: int, tid: int, sub: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + tid * 1_009 + sub * 7_919) % (2**62))
    return g


def _act_dtype(act: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[act]


def q4_group(wfmt: str) -> int:
    """Group size of a 4-bit format name ("q4" is group 64), 0 otherwise."""
    return {"q4": 64, "q4g32": 32, "q4g128": 128}.get(wfmt, 0)


def quantize_q4g64(w: torch.Tensor, group: int = GROUP):
    """Encode fp32 weights [..., n, K] into the packed 4-bit affine format.

    Data generation only: per group of `group` consecutive input elements
    take min and max, scale = bf16((max - min) / 15), bias = bf16(min), and
    q = clamp(round_half_even((w - bias) / scale), 0, 15). Returns
    (packed uint32 [..., n, K/8], scales bf16 [..., n, K/group], biases bf16).
    """
    *lead, K = w.shape
    assert K % group == 0
    wg = w.float().reshape(*lead, K // group, group)
    mn = wg.amin(dim=-1)
    mx = wg.amax(dim=-1)
    scale = ((mx - mn) / 15.0).clamp_min(1e-8).to(torch.bfloat16)
    bias = mn.to(torch.bfloat16)
    q = torch.round((wg - bias.float().unsqueeze(-1)) / scale.float().unsqueeze(-1))
    q = q.clamp_(0, 15).to(torch.int64).reshape(*lead, K // 8, 8)
    shifts = torch.arange(8, device=w.device, dtype=torch.int64) * 4
    words = (q << shifts).sum(dim=-1)               # < 2**32, exact in int64
    packed = words.to(torch.int64)
    # reinterpret the low 32 bits as uint32 storage
    packed = torch.where(packed >= 2**31, packed - 2**32, packed).to(torch.int32)
    return packed.view(torch.uint32), scale, bias


def quantize_q8g64(w: torch.Tensor):
    """Encode fp32 weights [..., n, K] into the packed 8-bit affine format:
    per group of 64 inputs scale = bf16((max - min) / 255), bias = bf16(min),
    q = clamp(round_half_even((w - bias) / scale), 0, 255), byte j of each
    uint32 word = element j (data generation only)."""
    *lead, K = w.shape
    assert K % GROUP == 0
    wg = w.float().reshape(*lead, K // GROUP, GROUP)
    mn = wg.amin(dim=-1)
    mx = wg.amax(dim=-1)
    scale = ((mx - mn) / 255.0).clamp_min(1e-8).to(torch.bfloat16)
    bias = mn.to(torch.bfloat16)
    q = torch.round((wg - bias.float().unsqueeze(-1)) / scale.float().unsqueeze(-1))
    q = q.clamp_(0, 255).to(torch.int64).reshape(*lead, K // 4, 4)
    shifts = torch.arange(4, device=w.device, dtype=torch.int64) * 8
    words = (q << shifts).sum(dim=-1)
    words = torch.where(words >= 2**31, words - 2**32, words).to(torch.int32)
    return words.view(torch.uint32), scale, bias


def pack_nibbles(q: torch.Tensor) -> torch.Tensor:
    """Pack integer codes q[..., K] (values 0..15) into uint32 [..., K/8],
    low nibble first. Used to build hand-made fixtures."""
    *lead, K = q.shape
    q = q.to(torch.int64).reshape(*lead, K // 8, 8)
    shifts = torch.arange(8, dtype=torch.int64, device=q.device) * 4
    words = (q << shifts).sum(dim=-1)
    words = torch.where(words >= 2**31, words - 2**32, words).to(torch.int32)
    return words.view(torch.uint32)


@dataclass
class Experts:
    fmt: str
    E: int
    d: int
    F: int
    w_gu: torch.Tensor
    w_dn: torch.Tensor
    s_gu: torch.Tensor | None = None
    b_gu: torch.Tensor | None = None
    s_dn: torch.Tensor | None = None
    b_dn: torch.Tensor | None = None
    act: str = "swiglu"       # the GLU's gate activation: "swiglu" or "geglu"

    def to(self, device) -> "Experts":
        mv = lambda t: None if t is None else t.to(device)
        return Experts(self.fmt, self.E, self.d, self.F, mv(self.w_gu), mv(self.w_dn),
                       mv(self.s_gu), mv(self.b_gu), mv(self.s_dn), mv(self.b_dn), self.act)

    def with_act(self, act: str) -> "Experts":
        """The same weights with another GLU activation."""
        return Experts(self.fmt, self.E, self.d, self.F, self.w_gu, self.w_dn, self.s_gu,
                       self.b_gu, self.s_dn, self.b_dn, act)

    def select(self, experts) -> "Experts":
        """Copy of the listed experts only (for sampled checks on the host)."""
        ix = torch.as_tensor(experts, dtype=torch.long, device=self.w_gu.device)
        sl = lambda t: None if t is None else t.index_select(0, ix)
        return Experts(self.fmt, len(ix), self.d, self.F, sl(self.w_gu), sl(self.w_dn),
                       sl(self.s_gu), sl(self.b_gu), sl(self.s_dn), sl(self.b_dn), self.act)

    def nbytes_per_expert(self) -> int:
        tot = 0
        for t in (self.w_gu, self.w_dn, self.s_gu, self.b_gu, self.s_dn, self.b_dn):
            if t is not None:
                tot += t[0].numel() * t.element_size()
        return tot


@dataclass
class Layer:
    wl: Workload
    x: torch.Tensor
    w_router: torch.Tensor
    router_bias: torch.Tensor | None
    experts: Experts
    meta: dict = field(default_factory=dict)


def make_experts(wl: Workload, seed: int, device="cpu") -> Experts:
    E, d, F = wl.E, wl.d, wl.F
    gu, dn = [], []
    sgu, bgu, sdn, bdn = [], [], [], []
    for e in range(E):
        g1 = _gen(seed, _TID_GU, e, device)
        g2 = _gen(seed, _TID_DN, e, device)
        wgu = torch.randn(2 * F, d, generator=g1, device=device) / math.sqrt(d)
        wdn = torch.randn(d, F, generator=g2, device=device) / math.sqrt(F)
        if wl.wfmt == "f32":
            gu.append(wgu)
            dn.append(wdn)
        elif wl.wfmt == "bf16":
            gu.append(wgu.to(torch.bfloat16))
            dn.append(wdn.to(torch.bfloat16))
        elif wl.wfmt == "q8":
            p, s, b = quantize_q8g64(wgu)
            gu.append(p); sgu.append(s); bgu.append(b)
            p, s, b = quantize_q8g64(wdn)
            dn.append(p); sdn.append(s); bdn.append(b)
        elif q4_group(wl.wfmt):
            p, s, b = quantize_q4g64(wgu, q4_group(wl.wfmt))
            gu.append(p); sgu.append(s); bgu.append(b)
            p, s, b = quantize_q4g64(wdn, q4_group(wl.wfmt))
            dn.append(p); sdn.append(s); bdn.append(b)
        else:
            raise ValueError(wl.wfmt)
    st = lambda xs: torch.stack(xs) if xs else None
    return Experts(wl.wfmt, E, d, F, st(gu), st(dn), st(sgu), st(bgu), st(sdn), st(bdn))


def make_router_bias(wl: Workload, seed: int, device="cpu"):
    if wl.bias == "none":
        return None
    if wl.bias == "normal0.5":
        g = _gen(seed, _TID_BIAS, 0, device)
        return (torch.randn(wl.E, generator=g, device=device) * 0.5).float()
    if wl.bias == "zipf1.1":
        # A seeded permutation gives each expert a popularity rank r in 1..E;
        # Zipf(s) popularity p_r ~ r^-s enters the logits as s * ln(1/r)
        # (the additive constant of log-popularity cancels in the softmax).
        g = _gen(seed, _TID_PERM, 0, "cpu")
        rank = torch.randperm(wl.E, generator=g) + 1
        return (-1.1 * torch.log(rank.double())).float().to(device)
    raise ValueError(wl.bias)


def make_layer(wl: Workload | str, seed: int = 0, device="cpu") -> Layer:
    if isinstance(wl, str):
        wl = WORKLOADS[wl]
    dt = _act_dtype(wl.act)
    gx = _gen(seed, _TID_X, 0, device)
    x = torch.randn(wl.T, wl.d, generator=gx, device=device).to(dt)
    gr = _gen(seed, _TID_WR, 0, device)
    w_router = (torch.randn(wl.E, wl.d, generator=gr, device=device) / math.sqrt(wl.d)).to(dt)
    bias = make_router_bias(wl, seed, device)
    experts = make_experts(wl, seed, device)
    return Layer(wl, x, w_router, bias, experts)


# --------------------------------------------------------------------------
# inputs for single-stage checks


def random_topk_idx(T: int, E: int, k: int, seed: int, skew: float = 0.0, device="cpu"):
    """k distinct expert ids per token, int32 [T, k]. With skew > 0 the draw
    favours low expert ids (weights exp(-skew * e)), giving empty and
    overfull experts."""
    g = _gen(seed, _TID_IDX, 0, "cpu")
    if T == 0:
        return torch.zeros(0, k, dtype=torch.int32, device=device)
    if skew <= 0:
        keys = torch.rand(T, E, generator=g)
    else:
        # Gumbel-top-k draw without replacement from weights exp(-skew*e)
        u = torch.rand(T, E, generator=g).clamp_min(1e-12)
        keys = -skew * torch.arange(E, dtype=torch.float32) - torch.log(-torch.log(u))
    idx = torch.argsort(keys, dim=1, descending=True)[:, :k]
    return idx.to(torch.int32).to(device)


def random_logits(T: int, E: int, seed: int, ties: bool = False, device="cpu"):
    """fp32 logits [T, E]. With ties=True values are drawn from a small set
    (multiples of 0.25 in [-2, 2], signed zeros included) so that equal
    values, including equal values at the k-th boundary, are frequent."""
    g = _gen(seed, _TID_LOGITS, 0, "cpu")
    if ties:
        v = torch.randint(-8, 9, (T, E), generator=g).float() * 0.25
        neg0 = torch.rand(T, E, generator=g) < 0.5
        v = torch.where((v == 0) & neg0, torch.tensor(-0.0), v)
    else:
        v = torch.randn(T, E, generator=g) * 2.0
    return v.to(device)


def random_rows(n: int, width: int, seed: int, tid: int = _TID_H, dtype=torch.bfloat16, device="cpu"):
    g = _gen(seed, tid, 0, "cpu")
    return torch.randn(n, width, generator=g).to(dtype).to(device)


def random_ys(n: int, width: int, seed: int, dtype=torch.bfloat16, device="cpu"):
    return random_rows(n, width, seed, _TID_YS, dtype, device)


def random_weights(T: int, k: int, seed: int, device="cpu"):
    g = _gen(seed, _TID_W, 0, "cpu")
    w = torch.rand(T, k, generator=g) + 0.05
    return w.float().to(device)
