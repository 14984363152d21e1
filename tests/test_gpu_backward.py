"""Training-mode backward through the C ABI on B200, against the fp64 oracle.

The oracle routes with the library's own fp32 logits (beam_moe_route gives
the same logits the backward computes), so every candidate, mask decision and
softmax weight is the same on both sides; the gradients are then compared
tensor by tensor, normwise: max|gpu - ref| <= tol * max|ref|.

Bars (derived from the arithmetic):
* fp32 layer: 1e-4 (fp32 accumulation over d = 128 / I = 256 terms).
* bf16 layer, expert-weight gradients: 1e-3 (fp32 sums of exact bf16
  products; dh, da, db are fp32).
* bf16 layer, dx and the router gradients: 1e-2.  They go through
  u = <dy, E_k(x)>, whose expert output is computed from H rounded to bf16 (the
  down GEMM's operand): a relative error of at most 2^-9 per element of H.

Also checked: experts with no kept pair keep exactly zero weight gradients; a
second call adds exactly the same gradients (accumulation); two calls are
bitwise equal.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from dynamic_expert_routing_router_b200 import abi, inputs

from _parity import gpu_route, host

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
DEV = "cuda"


def _zeros(E, d, I, masked):
    z = lambda *s: torch.zeros(s, dtype=torch.float32, device=DEV)  # noqa: E731
    return dict(dx=z(1, 1), dW_gate=z(E, d), dW_mask=z(E, d) if masked else None,
                dW1=z(E, I, d), dW3=z(E, I, d), dW2=z(E, d, I))


def gpu_backward(dsc, x, Wg, Wm, W1, W3, W2, dy, beta, grads=None, ws=None):
    T, d, E, I = dsc.T, dsc.d, dsc.E, dsc.I
    g = grads or _zeros(E, d, I, Wm is not None)
    g["dx"] = torch.full((T, d), float("nan"), dtype=torch.float32, device=DEV)
    ws = ws if ws is not None else abi.alloc_backward_workspace(dsc, DEV)
    abi.backward(dsc, x, Wg, Wm, W1, W3, W2, dy, beta, g["dx"], g["dW_gate"], g["dW_mask"],
                 g["dW1"], g["dW3"], g["dW2"], ws)
    abi.check(dsc, ws)
    torch.cuda.synchronize()
    return g, ws


def _normwise(gpu, ref, tol, what):
    gpu = np.asarray(gpu, np.float64)
    m = np.abs(ref).max() if ref.size else 0.0
    diff = np.abs(gpu - ref).max() if ref.size else 0.0
    assert diff <= tol * m + 1e-30, (what, diff, m)


def _compare(g, ref, sel, tol_router, tol_expert):
    _normwise(g["dx"].cpu().numpy(), ref["dx"], tol_router, "dx")
    _normwise(g["dW_gate"].cpu().numpy(), ref["dW_gate"], tol_router, "dW_gate")
    if ref["dW_mask"] is not None:
        _normwise(g["dW_mask"].cpu().numpy(), ref["dW_mask"], tol_router, "dW_mask")
    for key in ("dW1", "dW3", "dW2"):
        _normwise(g[key][sel].cpu().numpy(), ref[key], tol_expert, key)


def test_tiny_f32_backward_matches_oracle():
    gamma = json.load(open(os.path.join(HERE, "golden", "tiny_gamma.json")))["gamma"]
    L = {k: v.to(DEV) for k, v in inputs.make_tiny(T=64, seed=0, gamma=gamma).items()}
    sh = inputs.TINY
    dsc = abi.desc(64, sh.d, sh.E, sh.I, sh.K, "f32", sh.renorm)
    dy = inputs.make_upstream_grad(sh, 64, seed=1, device=DEV)
    beta = 0.05
    g, _ = gpu_backward(dsc, L["x"], L["W_gate"], L["W_mask"], L["W1"], L["W3"], L["W2"], dy,
                        beta)
    rt = gpu_route(dsc, L["x"], L["W_gate"], L["W_mask"])
    ref = oracle.backward(host(L["x"]), host(L["W_gate"]), host(L["W_mask"]), host(L["W1"]),
                          host(L["W3"]), host(L["W2"]), host(dy), sh.K, sh.renorm, "f32",
                          beta=beta, logits=rt["logits"])
    _compare(g, ref, slice(None), 1e-4, 1e-4)


DECODE = [(8, 0.15, 1), (64, 0.35, 1), (64, 1.0, 1), (32, 0.35, 0)]


@pytest.mark.parametrize("T,f,renorm", DECODE, ids=[f"T{t}_f{f}_r{r}" for t, f, r in DECODE])
def test_bf16_decode_backward_matches_oracle(T, f, renorm):
    sh = inputs.Shape(2048, 128, 8, 768, renorm, "bf16")
    x = inputs.make_tokens(sh, T, seed=T + 11, device=DEV)
    Wg = inputs.make_gate(sh, seed=2, device=DEV)
    Wm = inputs.make_mask(sh, f, seed=2, device=DEV)
    W1, W3, W2 = inputs.make_experts(sh, seed=2, device=DEV)
    dy = inputs.make_upstream_grad(sh, T, seed=T, device=DEV)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", renorm)
    beta = 0.01
    g, ws = gpu_backward(dsc, x, Wg, Wm, W1, W3, W2, dy, beta)
    rt = gpu_route(dsc, x, Wg, Wm)
    kept = np.bincount(rt["idx"][rt["idx"] >= 0], minlength=sh.E)
    touched = np.flatnonzero(kept)
    # experts with no kept pair: weight gradients exactly zero (never written)
    untouched = np.flatnonzero(kept == 0)
    for key in ("dW1", "dW3", "dW2"):
        assert (g[key][torch.as_tensor(untouched, device=DEV)] == 0).all(), key
    sel = sorted(set(touched[:2].tolist()) | set(touched[-1:].tolist()))
    Wmh = host(Wm)
    ref = oracle.backward(host(x), host(Wg), Wmh, host(W1), host(W3), host(W2), host(dy), sh.K,
                          renorm, "bf16", beta=beta, experts=sel, logits=rt["logits"])
    _compare(g, ref, torch.as_tensor(sel, device=DEV), 1e-2, 1e-3)
    # accumulation: a second call adds the same gradients (x + x = 2x exactly)
    first = {k: v.clone() for k, v in g.items() if v is not None and k != "dx"}
    g2, _ = gpu_backward(dsc, x, Wg, Wm, W1, W3, W2, dy, beta, grads=g, ws=ws)
    for k, v in first.items():
        assert torch.equal(g2[k], 2 * v), k


def test_bf16_backward_hot_expert_spans_several_row_tiles():
    """An expert that is the top candidate of all T = 300 tokens and kept for
    nearly all of them: its candidate (and kept) rows span three 128-row tiles
    of the tensor-core GEMMs and two 256-row chunks of the weight-gradient
    kernels, paths a decode batch of 128 tokens never reaches."""
    T, hot = 300, 3
    sh = inputs.Shape(256, 16, 4, 256, 1, "bf16")
    x = inputs.make_tokens(sh, T, seed=31, device=DEV)  # last feature = 1
    Wg = inputs.make_gate(sh, seed=4, device=DEV)
    Wm = inputs.make_mask(sh, 0.35, seed=4, device=DEV)
    Wg[hot, sh.d - 1] = 6.0  # a candidate of every token
    Wm[hot, sh.d - 1] = 3.0  # and kept unless x . W_mask[hot] < -3
    W1, W3, W2 = inputs.make_experts(sh, seed=4, device=DEV)
    dy = inputs.make_upstream_grad(sh, T, seed=9, device=DEV)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    beta = 0.01
    g, _ = gpu_backward(dsc, x, Wg, Wm, W1, W3, W2, dy, beta)
    rt = gpu_route(dsc, x, Wg, Wm)
    kept = np.bincount(rt["idx"][rt["idx"] >= 0], minlength=sh.E)
    assert kept[hot] > 2 * 128, kept[hot]
    touched = np.flatnonzero(kept)
    sel = sorted({hot, int(touched[0]), int(touched[-1])})
    ref = oracle.backward(host(x), host(Wg), host(Wm), host(W1), host(W3), host(W2), host(dy),
                          sh.K, sh.renorm, "bf16", beta=beta, experts=sel, logits=rt["logits"])
    _compare(g, ref, torch.as_tensor(sel, device=DEV), 1e-2, 1e-3)
    assert torch.count_nonzero(g["dW2"][hot]) > 0


def test_bf16_backward_without_mask_and_repeatable():
    T = 16
    sh = inputs.QWEN3
    x = inputs.make_tokens(sh, T, seed=5, device=DEV)
    Wg = inputs.make_gate(sh, seed=3, device=DEV)
    W1, W3, W2 = inputs.make_experts(sh, seed=3, device=DEV)
    dy = inputs.make_upstream_grad(sh, T, seed=7, device=DEV)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    g1, _ = gpu_backward(dsc, x, Wg, None, W1, W3, W2, dy, 0.0)
    g2, _ = gpu_backward(dsc, x, Wg, None, W1, W3, W2, dy, 0.0)
    for k in ("dx", "dW_gate", "dW1", "dW3", "dW2"):
        assert torch.equal(g1[k], g2[k]), k
    rt = gpu_route(dsc, x, Wg, None)
    sel = sorted(set(rt["idx"][rt["idx"] >= 0].tolist()))[:2]
    ref = oracle.backward(host(x), host(Wg), None, host(W1), host(W3), host(W2), host(dy), sh.K,
                          sh.renorm, "bf16", experts=sel, logits=rt["logits"])
    _compare(g1, ref, torch.as_tensor(sel, device=DEV), 1e-2, 1e-3)


def test_backward_empty_batch_touches_nothing():
    """T = 0: OK, and no gradient is written (pointers stay non-null, as for
    the forward: a placeholder stands in for the empty token arrays)."""
    sh = inputs.QWEN3
    dsc = abi.desc(0, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    ph = torch.zeros((16,), dtype=torch.float32, device=DEV)
    Wg = inputs.make_gate(sh, device=DEV)
    Wm = inputs.make_mask(sh, 0.5, device=DEV)
    W = [torch.zeros((sh.E, sh.I, sh.d), dtype=torch.bfloat16, device=DEV) for _ in range(2)]
    W2 = torch.zeros((sh.E, sh.d, sh.I), dtype=torch.bfloat16, device=DEV)
    g = _zeros(sh.E, sh.d, sh.I, True)
    ws = abi.alloc_backward_workspace(dsc, DEV)
    abi.backward(dsc, ph, Wg, Wm, W[0], W[1], W2, ph, 0.1, ph, g["dW_gate"], g["dW_mask"],
                 g["dW1"], g["dW3"], g["dW2"], ws)
    abi.check(dsc, ws)
    for k in ("dW_gate", "dW_mask", "dW1", "dW3", "dW2"):
        assert (g[k] == 0).all()
    assert (ph == 0).all()
