"""Seeded synthetic inputs for the BEAM MoE layer.

This module only draws random tensors with the shapes and statistics of the
workloads; it holds none of the layer's arithmetic (no logits, no top-K, no
mask test, no expert math).  The tests feed the same tensors to the CUDA
library and to the CPU oracle, and the benchmark uses them as its workload.

Workload recipe (all synthetic; the trained models of the paper are not used):

* Shapes are those of Qwen3-30B-A3B's MoE layer (d=2048, E=128 experts, top-8,
  I=768, no shared experts), the tiny fp32 layer (d=128, E=8, K=2, I=256), and
  the large fine-grained layer (d=7168, E=256, K=8, I=2048).
* Tokens x: i.i.d. N(0,1) rows rescaled to RMS 1 (an RMSNorm output with unit
  scale).  For the bf16 layers the last feature is then set to 1: it is a
  bias feature, so a bias on a router logit is a weight in column d-1.
* Main router W_gate ~ N(0, 1/d).  Load skew: column d-1 of W_gate holds
  -1.1*ln(rank_e) for a seeded ranking of the experts, so the router's softmax
  prior is Zipf(1.1) over experts.  The large layer uses no skew.
* Mask router W_mask (bf16 layers): N(0, 1/d) with column d-1 = -gamma.  The
  mask pre-activation of a candidate is then approximately N(-gamma, (d-1)/d),
  so gamma = sqrt((d-1)/d) * Phi^-1(1 - f) targets a kept fraction f; the
  fraction actually kept is measured by the library's own counters and
  reported.  f = 1 uses W_mask = 0 exactly (every sigmoid equals 0.5).
* Tiny fp32 layer: x = N(0, I) + mu with a random mean vector |mu| = 0.5 and
  W_mask[e] = N(0, 1/d) - gamma*mu, gamma calibrated offline by the oracle
  (tests/golden/tiny_gamma.json) to keep about half of the candidates.
* Experts: W1 (gate), W3 (up) ~ N(0, 1/d) as [E, I, d]; W2 (down) ~ N(0, 1/I)
  as [E, d, I].  Shared experts (DeepSeekV2-Lite shape: 2 of them, Qwen1.5-MoE
  shape: 4) are drawn the same way from their own seeds.
* f = 0 (every candidate masked): W_mask = 0 except -1 in the bias column.

Each tensor has its own seed (base seed + a fixed offset, plus 1000 per layer
of a stack), drawn with a torch.Generator on the target device.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from statistics import NormalDist

import torch

# Per-tensor seed offsets.
_OFF_X, _OFF_WG, _OFF_WM, _OFF_W1, _OFF_W3, _OFF_W2, _OFF_RANK, _OFF_MU = range(1, 9)
_OFF_SHARED = 20
_OFF_DY = 30
_LAYER_STRIDE = 1000


@dataclass(frozen=True)
class Shape:
    d: int
    E: int
    K: int
    I: int
    renorm: int
    dtype: str  # "bf16" or "f32"


TINY = Shape(d=128, E=8, K=2, I=256, renorm=0, dtype="f32")
QWEN3 = Shape(d=2048, E=128, K=8, I=768, renorm=1, dtype="bf16")
LARGE = Shape(d=7168, E=256, K=8, I=2048, renorm=1, dtype="bf16")
# Layers with always-on shared experts (the two such models of the BEAM
# evaluation): routed experts and shared experts both of width I = 1408,
# softmax over all experts restricted to the top-K (no renormalisation).
DSV2_LITE = Shape(d=2048, E=64, K=6, I=1408, renorm=0, dtype="bf16")
DSV2_LITE_SHARED = 2
QWEN15_MOE = Shape(d=2048, E=60, K=4, I=1408, renorm=0, dtype="bf16")
QWEN15_MOE_SHARED = 4


def torch_dtype(shape: Shape):
    return torch.bfloat16 if shape.dtype == "bf16" else torch.float32


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, std, seed, device, dtype):
    out = torch.empty(shape, dtype=torch.float32, device=device)
    out.normal_(0.0, std, generator=_gen(device, seed))
    return out.to(dtype)


def gamma_for_fraction(f: float, d: int) -> float:
    """Mask bias that keeps about a fraction f of candidates (bias-feature recipe)."""
    if not 0.0 < f < 1.0:
        raise ValueError("f must lie in (0, 1); f = 1 is W_mask = 0")
    return math.sqrt((d - 1) / d) * NormalDist().inv_cdf(1.0 - f)


def make_tokens(shape: Shape, T: int, seed: int = 0, device="cpu", bias_feature=True,
                layer: int = 0):
    """x [T, d]: RMS-1 rows; last feature = 1 for the bias-feature recipe."""
    s = seed + layer * _LAYER_STRIDE + _OFF_X
    x = _normal((T, shape.d), 1.0, s, device, torch.float32)
    if T:
        x = x / x.pow(2).mean(dim=1, keepdim=True).sqrt().clamp_min(1e-6)
    if bias_feature:
        x[:, shape.d - 1] = 1.0
    return x.to(torch_dtype(shape))


def make_experts(shape: Shape, seed: int = 0, device="cpu", layer: int = 0):
    """(W1, W3, W2): gate and up [E, I, d], down [E, d, I]."""
    base = seed + layer * _LAYER_STRIDE
    dt = torch_dtype(shape)
    W1 = _normal((shape.E, shape.I, shape.d), 1.0 / math.sqrt(shape.d), base + _OFF_W1,
                 device, dt)
    W3 = _normal((shape.E, shape.I, shape.d), 1.0 / math.sqrt(shape.d), base + _OFF_W3,
                 device, dt)
    W2 = _normal((shape.E, shape.d, shape.I), 1.0 / math.sqrt(shape.I), base + _OFF_W2,
                 device, dt)
    return W1, W3, W2


def make_shared_experts(shape: Shape, n_shared: int, seed: int = 0, device="cpu",
                        layer: int = 0):
    """(W1s, W3s, W2s) of n_shared always-on experts of width shape.I, drawn
    like the routed experts: [S, I, d], [S, I, d], [S, d, I]."""
    sh = Shape(d=shape.d, E=n_shared, K=1, I=shape.I, renorm=shape.renorm, dtype=shape.dtype)
    return make_experts(sh, seed=seed + _OFF_SHARED, device=device, layer=layer)


def make_gate(shape: Shape, seed: int = 0, device="cpu", zipf: float | None = 1.1,
              layer: int = 0):
    """W_gate [E, d] ~ N(0, 1/d); with zipf, column d-1 = -zipf*ln(rank)."""
    base = seed + layer * _LAYER_STRIDE
    Wg = _normal((shape.E, shape.d), 1.0 / math.sqrt(shape.d), base + _OFF_WG, device,
                 torch.float32)
    if zipf is not None:
        perm = torch.randperm(shape.E, generator=_gen("cpu", base + _OFF_RANK))
        rank = torch.empty(shape.E, dtype=torch.float32)
        rank[perm] = torch.arange(1, shape.E + 1, dtype=torch.float32)
        Wg[:, shape.d - 1] = (-zipf * torch.log(rank)).to(Wg.device)
    return Wg.to(torch_dtype(shape))


def make_mask(shape: Shape, f: float, seed: int = 0, device="cpu", layer: int = 0):
    """W_mask [E, d] for a target kept fraction f (bias-feature recipe); f=1 -> zeros;
    f=0 -> zeros with -1 in the bias column (every mask pre-activation is -1)."""
    if f >= 1.0:
        return torch.zeros((shape.E, shape.d), dtype=torch_dtype(shape), device=device)
    if f <= 0.0:
        Wm = torch.zeros((shape.E, shape.d), dtype=torch.float32, device=device)
        Wm[:, shape.d - 1] = -1.0
        return Wm.to(torch_dtype(shape))
    base = seed + layer * _LAYER_STRIDE
    Wm = _normal((shape.E, shape.d), 1.0 / math.sqrt(shape.d), base + _OFF_WM, device,
                 torch.float32)
    Wm[:, shape.d - 1] = -gamma_for_fraction(f, shape.d)
    return Wm.to(torch_dtype(shape))


def make_tiny(T: int = 64, seed: int = 0, gamma: float | None = None, device="cpu"):
    """The tiny fp32 layer: x = N(0,I) + mu, W_mask = N(0,1/d) - gamma*mu.

    Returns a dict of float32 tensors: x, W_gate, W_mask, W1, W3, W2, mu.  With
    gamma None, W_mask is built with gamma = 0.
    """
    sh = TINY
    mu = _normal((sh.d,), 1.0, seed + _OFF_MU, device, torch.float32)
    mu = mu * (0.5 / mu.norm())
    x = _normal((T, sh.d), 1.0, seed + _OFF_X, device, torch.float32) + mu
    Wg = _normal((sh.E, sh.d), 1.0 / math.sqrt(sh.d), seed + _OFF_WG, device, torch.float32)
    Wm = _normal((sh.E, sh.d), 1.0 / math.sqrt(sh.d), seed + _OFF_WM, device, torch.float32)
    Wm = Wm - (0.0 if gamma is None else float(gamma)) * mu[None, :]
    W1, W3, W2 = make_experts(sh, seed, device)
    return dict(x=x, W_gate=Wg, W_mask=Wm, W1=W1, W3=W3, W2=W2, mu=mu)


def make_upstream_grad(shape: Shape, T: int, seed: int = 0, device="cpu"):
    """dy [T, d] for the backward pass: i.i.d. N(0, 1), in the layer's dtype."""
    return _normal((T, shape.d), 1.0, seed + _OFF_DY, device, torch_dtype(shape))


def bf16_bits(t: torch.Tensor):
    """Raw 16-bit patterns of a bf16 tensor as a numpy int16 array (CPU)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy()


def host_array(t: torch.Tensor):
    """A tensor in the oracle's storage format: bf16 -> raw bits, f32 -> float32."""
    if t.dtype == torch.bfloat16:
        return bf16_bits(t)
    return t.detach().contiguous().cpu().to(torch.float32).numpy()


# ------------------------------------------------------- 48-layer stack --
# Decode through a stack of independent Qwen3-shaped layers: each layer has its
# own seeded weights (seed + 1000 * layer) and its own mask router, drawn for a
# kept fraction in [0.10, 0.60].  The next layer's input is the previous
# layer's output plus N(0, 0.1^2) noise, rescaled to RMS 1 (the RMSNorm in
# front of every MoE layer of these models) with the bias feature restored.
STACK_LAYERS = 48
_OFF_STACK_F, _OFF_STACK_NOISE = 9, 10


def stack_kept_fraction(layer: int, seed: int = 0) -> float:
    g = _gen("cpu", seed + layer * _LAYER_STRIDE + _OFF_STACK_F)
    return float(0.10 + 0.50 * torch.rand((), generator=g).item())


def stack_next_input(out: torch.Tensor, layer: int, seed: int = 0):
    """Input of layer `layer` + 1 from the output of layer `layer`."""
    noise = _normal(tuple(out.shape), 0.1, seed + layer * _LAYER_STRIDE + _OFF_STACK_NOISE,
                    out.device, torch.float32)
    x = out.float() + noise
    if x.shape[0]:
        x = x / x.pow(2).mean(dim=1, keepdim=True).sqrt().clamp_min(1e-6)
    x[:, x.shape[1] - 1] = 1.0
    return x.to(out.dtype)
