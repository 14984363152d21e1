"""The one-launch decode layer (bf16, T <= 16) against the fp64 oracle.

At these sizes beam_moe_forward runs router, top-K + mask, grouping, both
expert projections and the combine in one kernel, and beam_moe_route (and the
backward) take their logits from the same router units.  Checked here, on
shapes that reach every unit size and every top-K width of that kernel:

* its own logits (the workspace's single router split) against the oracle's
  fp64 logits, element by element;
* its routing and grouping bit for bit against the oracle's decisions on
  those logits, and bit for bit equal to beam_moe_route's;
* its output rows (every token) and expert rows against the oracle, and the
  combine against its own rows of Y;
* the cases the method has at this size: every candidate masked, tokens
  with no kept candidate beside others, no mask (vanilla top-K), the
  threshold tau, K = 1 and K = 16;
* repeated calls (its counters reset every call), CUDA-graph replay, and
  calls on a workspace left dirty by another shape.
"""
import numpy as np
import pytest
import torch

import oracle
from dynamic_expert_routing_router_b200 import abi, inputs

from _parity import (assert_combine, assert_expert_rows, assert_grouping_bitexact,
                     assert_logits, assert_routing_bitexact, assert_values, compact_experts,
                     gpu_route, host, oracle_from_logits, pick_experts, report)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def one_launch_up_to_16_tokens():
    """Every batch of at most 16 tokens takes the one-launch path here (the
    library's default stops at 4)."""
    prev = abi.set_one_launch_tokens(16)
    yield
    abi.set_one_launch_tokens(prev)

DEV = "cuda"

SHAPES = [
    # (name, T, d, E, I, K, renorm, f, mask)
    ("qwen3_T1", 1, 2048, 128, 768, 8, 1, 0.15, True),
    ("qwen3_T2_renorm0", 2, 2048, 128, 768, 8, 0, 0.35, True),
    ("qwen3_T5", 5, 2048, 128, 768, 8, 1, 0.6, True),
    ("qwen3_T16", 16, 2048, 128, 768, 8, 1, 0.35, True),
    ("qwen3_T16_all_kept", 16, 2048, 128, 768, 8, 1, 1.0, True),
    ("qwen3_T7_no_mask", 7, 2048, 128, 768, 8, 1, 1.0, False),
    ("qwen15_like_T16_E60_K4", 16, 2048, 60, 1408, 4, 0, 0.35, True),
    ("top1_T11", 11, 1024, 32, 256, 1, 1, 0.5, True),
    ("top16_E256_T9", 9, 512, 256, 384, 16, 1, 0.6, True),
    ("tiny_T16_d128", 16, 128, 8, 128, 2, 0, 0.5, True),
    ("large_T1_d7168_E256", 1, 7168, 256, 2048, 8, 1, 0.5, True),
    ("some_tokens_masked_T12", 12, 2048, 128, 768, 8, 1, 0.08, True),
]


def _layer(name, T, d, E, I, K, renorm, f, mask, seed=3):
    sh = inputs.Shape(d=d, E=E, K=K, I=I, renorm=renorm, dtype="bf16")
    x = inputs.make_tokens(sh, T, seed=seed + T, device=DEV)
    Wg = inputs.make_gate(sh, seed=seed, device=DEV)
    Wm = inputs.make_mask(sh, f, seed=seed, device=DEV) if mask else None
    W1, W3, W2 = inputs.make_experts(sh, seed=seed, device=DEV)
    return sh, x, Wg, Wm, W1, W3, W2


@pytest.mark.parametrize("name,T,d,E,I,K,renorm,f,mask", SHAPES, ids=[s[0] for s in SHAPES])
def test_one_launch_layer_matches_oracle(name, T, d, E, I, K, renorm, f, mask):
    sh, x, Wg, Wm, W1, W3, W2 = _layer(name, T, d, E, I, K, renorm, f, mask)
    dsc = abi.desc(T, d, E, I, K, "bf16", renorm)
    P = abi.plan(dsc)
    assert P["one_launch"] == 1 and abi.kernel_count(dsc) == 1
    ws = abi.alloc_workspace(dsc, DEV)
    ws.fill_(0xA5)  # no reliance on a clean workspace
    out = torch.full((T, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    abi.forward(dsc, x, Wg, Wm, W1, W3, W2, out, ws)
    abi.check(dsc, ws)
    v = abi.workspace_views(dsc, ws)
    lg = v["partial"][0].cpu().numpy()
    g = dict(idx=v["idx"].cpu().numpy(), w=v["w"].cpu().numpy(),
             counts=v["counts"].cpu().numpy(), hist=v["hist"].cpu().numpy(),
             logits=lg if mask else np.concatenate([lg[:, :E], np.zeros((T, E), np.float32)], 1))
    # logits: the kernel's own, against the oracle's fp64 logits
    assert_logits(g, x, Wg, Wm, "bf16", K, renorm, name=f"one_launch_{name}")
    o = oracle_from_logits(g["logits"], E, K, renorm, mask)
    assert_routing_bitexact(g, o)
    assert_grouping_bitexact(dsc, v, g["idx"])
    # the same decisions and weights, bit for bit, as the routing call
    r = gpu_route(dsc, x, Wg, Wm)
    for k in ("idx", "w", "counts", "hist"):
        assert np.array_equal(r[k], g[k]), k
    assert np.array_equal(r["logits"][:, :E], lg[:, :E])
    # values: every token (the oracle is handed only the experts in use)
    c1, c3, c2, cidx = compact_experts(W1, W3, W2, g["idx"])
    ref = oracle.experts(host(x), c1, c3, c2, cidx, o["w"], "bf16")
    worst = assert_values(out, ref, g["idx"], "bf16")
    assert_combine(out, v, "bf16")
    nrow, wrow = assert_expert_rows(v, x, W1, W3, W2, "bf16", pick_experts(g["counts"]))
    report(name=f"one_launch_{name}", kind="values", tokens=T, worst_token_excess=worst,
           expert_rows=nrow, worst_expert_row=wrow)


def test_one_launch_every_candidate_masked():
    sh, x, Wg, _, W1, W3, W2 = _layer("", 16, 2048, 128, 768, 8, 1, 0.0, True)
    Wm = inputs.make_mask(sh, 0.0, device=DEV)
    dsc = abi.desc(16, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    ws = abi.alloc_workspace(dsc, DEV)
    out = torch.full((16, sh.d), 1.0, dtype=torch.bfloat16, device=DEV)
    abi.forward(dsc, x, Wg, Wm, W1, W3, W2, out, ws)
    abi.check(dsc, ws)
    v = abi.workspace_views(dsc, ws)
    assert (out == 0).all()
    assert (v["idx"] == -1).all() and (v["counts"] == 0).all()
    assert v["hist"].cpu().tolist() == [16] + [0] * sh.K
    assert v["meta"].cpu().tolist()[:3] == [0, 0, 0]


@pytest.mark.parametrize("tau", [0.3, 0.7])
def test_one_launch_threshold_tau(tau):
    sh, x, Wg, Wm, W1, W3, W2 = _layer("", 8, 2048, 128, 768, 8, 1, 0.35, True, seed=11)
    dsc = abi.desc(8, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    dsc.mask_logit_threshold = abi.tau_logit(tau)
    ws = abi.alloc_workspace(dsc, DEV)
    out = torch.empty((8, sh.d), dtype=torch.bfloat16, device=DEV)
    abi.forward(dsc, x, Wg, Wm, W1, W3, W2, out, ws)
    abi.check(dsc, ws)
    v = abi.workspace_views(dsc, ws)
    lg = v["partial"][0].cpu().numpy()
    o = oracle_from_logits(lg, sh.E, sh.K, sh.renorm, True, dsc.mask_logit_threshold)
    g = dict(idx=v["idx"].cpu().numpy(), w=v["w"].cpu().numpy(),
             counts=v["counts"].cpu().numpy(), hist=v["hist"].cpu().numpy())
    assert_routing_bitexact(g, o)
    c1, c3, c2, cidx = compact_experts(W1, W3, W2, g["idx"])
    ref = oracle.experts(host(x), c1, c3, c2, cidx, o["w"], "bf16")
    assert_values(out, ref, g["idx"], "bf16")


def test_one_launch_repeated_calls_graph_replay_and_dirty_workspace():
    """Counters reset every call: back-to-back calls, a CUDA-graph replay and a
    workspace used before by a larger batch all give the first call's bits."""
    sh, x, Wg, Wm, W1, W3, W2 = _layer("", 6, 2048, 128, 768, 8, 1, 0.35, True, seed=5)
    dsc = abi.desc(6, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    ws = abi.alloc_workspace(dsc, DEV)
    ref = torch.empty((6, sh.d), dtype=torch.bfloat16, device=DEV)
    abi.forward(dsc, x, Wg, Wm, W1, W3, W2, ref, ws)
    abi.check(dsc, ws)
    out = torch.empty_like(ref)
    for _ in range(5):
        out.zero_()
        abi.forward(dsc, x, Wg, Wm, W1, W3, W2, out, ws)
        abi.check(dsc, ws)
        assert torch.equal(out, ref)
    # a workspace last used by a 16-token call (more rows, other counters)
    big = abi.desc(16, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    wsb = abi.alloc_workspace(big, DEV)
    xb = inputs.make_tokens(sh, 16, seed=77, device=DEV)
    ob = torch.empty((16, sh.d), dtype=torch.bfloat16, device=DEV)
    abi.forward(big, xb, Wg, Wm, W1, W3, W2, ob, wsb)
    abi.check(big, wsb)
    out.zero_()
    abi.forward(dsc, x, Wg, Wm, W1, W3, W2, out, wsb)
    abi.check(dsc, wsb)
    assert torch.equal(out, ref)
    # graph replay (the header clear and the kernel are both captured)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    gout = torch.zeros_like(ref)
    with torch.cuda.stream(s):
        abi.forward(dsc, x, Wg, Wm, W1, W3, W2, gout, ws, stream=s)  # warm-up outside capture
        s.synchronize()
        with torch.cuda.graph(g, stream=s):
            abi.forward(dsc, x, Wg, Wm, W1, W3, W2, gout, ws, stream=s)
    for _ in range(3):
        gout.zero_()
        g.replay()
        torch.cuda.synchronize()
        abi.check(dsc, ws)
        assert torch.equal(gout, ref)
