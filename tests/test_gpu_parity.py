"""CUDA library vs. the fp64 oracle, through the C ABI, on B200.

Workloads: the tiny fp32 layer (d=128, E=8, K=2, I=256, no renorm), the
Qwen3-30B-A3B-shaped bf16 layer at decode (T = 1..128) and prefill (T = 8192)
for several kept fractions, the large fine-grained layer (d=7168, E=256,
I=2048), and edge shapes (E not a multiple of 128, K = 1, K = 16, ragged T,
T = 0, renorm off).  See tests/_parity.py for the bars.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from dynamic_expert_routing_router_b200 import abi, inputs

from _parity import (BF16_TOL_RMS, assert_combine, assert_expert_rows,
                     assert_grouping_bitexact, assert_logits, assert_routing_bitexact,
                     assert_token_sample, assert_values, bf16_excess, compact_experts,
                     gpu_forward, gpu_route, host, oracle_from_logits, oracle_values,
                     pick_experts, report, strided_rows)

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
DEV = "cuda"


@pytest.fixture(scope="module")
def qwen3_experts():
    torch.cuda.init()
    return inputs.make_experts(inputs.QWEN3, seed=0, device=DEV)


@pytest.fixture(scope="module")
def qwen3_experts_host(qwen3_experts):
    return tuple(host(W) for W in qwen3_experts)


def _tiny(gamma):
    L = inputs.make_tiny(T=64, seed=0, gamma=gamma, device="cpu")
    return {k: v.to(DEV) for k, v in L.items()}


# ------------------------------------------------------------------ tiny --

def test_tiny_f32_layer_matches_oracle():
    gamma = json.load(open(os.path.join(HERE, "golden", "tiny_gamma.json")))["gamma"]
    L = _tiny(gamma)
    sh = inputs.TINY
    dsc = abi.desc(64, sh.d, sh.E, sh.I, sh.K, "f32", sh.renorm)
    g = gpu_route(dsc, L["x"], L["W_gate"], L["W_mask"])
    o = oracle_from_logits(g["logits"], sh.E, sh.K, sh.renorm, True)
    assert_routing_bitexact(g, o)
    # GPU fp32 logits against the oracle's fp64 logits
    r, z = oracle.logits(host(L["x"]), host(L["W_gate"]), host(L["W_mask"]), "f32")
    np.testing.assert_allclose(g["logits"], np.concatenate([r, z], 1), rtol=0, atol=1e-5)
    assert_logits(g, L["x"], L["W_gate"], L["W_mask"], "f32", sh.K, sh.renorm, name="tiny_f32")
    kept = (g["idx"] >= 0).mean()
    assert 0.35 <= kept <= 0.65, kept
    out, ws = gpu_forward(dsc, L["x"], L["W_gate"], L["W_mask"], L["W1"], L["W3"], L["W2"])
    views = abi.workspace_views(dsc, ws)
    assert np.array_equal(views["idx"].cpu().numpy(), g["idx"])
    assert_grouping_bitexact(dsc, views, g["idx"])
    ref = oracle_values(L["x"], L["W1"], L["W3"], L["W2"], g["idx"], o["w"], "f32")
    assert_values(out, ref, g["idx"], "f32")
    assert_combine(out, views, "f32")
    assert_expert_rows(views, L["x"], L["W1"], L["W3"], L["W2"], "f32", range(sh.E))


def test_tiny_f32_zero_mask_is_vanilla_topk_bitwise():
    L = _tiny(0.0)
    sh = inputs.TINY
    dsc = abi.desc(64, sh.d, sh.E, sh.I, sh.K, "f32", sh.renorm)
    Wz = torch.zeros_like(L["W_mask"])
    out0, _ = gpu_forward(dsc, L["x"], L["W_gate"], Wz, L["W1"], L["W3"], L["W2"])
    outn, _ = gpu_forward(dsc, L["x"], L["W_gate"], None, L["W1"], L["W3"], L["W2"])
    assert torch.equal(out0, outn)
    g = gpu_route(dsc, L["x"], L["W_gate"], Wz)
    assert (g["idx"] >= 0).all() and g["hist"][sh.K] == 64
    o = oracle_from_logits(g["logits"], sh.E, sh.K, sh.renorm, False)
    ref = oracle_values(L["x"], L["W1"], L["W3"], L["W2"], o["idx"], o["w"], "f32")
    assert_values(outn, ref, o["idx"], "f32")


def test_tiny_f32_minus_inf_gate_row_gets_zero_weights():
    """One token's gate logits overflow to -inf in fp32 (x[t,0] = 1e30 against
    W_gate[:, 0] = -1e10): its softmax is 0/0, so its weights are 0 and its
    output row is 0 -- no NaN anywhere.  Decisions bit-exact with the oracle
    fed the same (partly -inf) logits; every other token as usual.  Feature 0
    meets zero columns of W_mask, W1 and W3, so the rest of the layer stays
    finite."""
    gamma = json.load(open(os.path.join(HERE, "golden", "tiny_gamma.json")))["gamma"]
    L = inputs.make_tiny(T=64, seed=0, gamma=gamma, device="cpu")
    t0 = 17
    L["x"][:, 0] = 0.0
    L["x"][t0, 0] = 1e30
    L["W_gate"][:, 0] = -1e10
    L["W_mask"][:, 0] = 0.0
    L["W1"][:, :, 0] = 0.0
    L["W3"][:, :, 0] = 0.0
    L = {k: v.to(DEV) for k, v in L.items()}
    sh = inputs.TINY
    dsc = abi.desc(64, sh.d, sh.E, sh.I, sh.K, "f32", sh.renorm)
    g = gpu_route(dsc, L["x"], L["W_gate"], L["W_mask"])
    assert np.isneginf(g["logits"][t0, :sh.E]).all()
    assert np.isfinite(g["w"]).all() and (g["w"][t0] == 0).all()
    o = oracle_from_logits(g["logits"], sh.E, sh.K, sh.renorm, True)
    assert_routing_bitexact(g, o)
    out, ws = gpu_forward(dsc, L["x"], L["W_gate"], L["W_mask"], L["W1"], L["W3"], L["W2"])
    assert torch.isfinite(out).all() and (out[t0] == 0).all()
    ref = oracle_values(L["x"], L["W1"], L["W3"], L["W2"], g["idx"], o["w"], "f32")
    assert_values(out, ref, g["idx"], "f32")


# ---------------------------------------------------------------- decode --

DECODE = [(T, f) for T in (1, 8, 32, 128) for f in (0.15, 0.35, 0.6, 1.0)]


@pytest.mark.parametrize("T,f", DECODE)
def test_qwen3_decode_matches_oracle(T, f, qwen3_experts, qwen3_experts_host):
    sh = inputs.QWEN3
    W1, W3, W2 = qwen3_experts
    x = inputs.make_tokens(sh, T, seed=100 + T, device=DEV)
    Wg = inputs.make_gate(sh, seed=0, device=DEV)
    Wm = inputs.make_mask(sh, f, seed=0, device=DEV)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    g = gpu_route(dsc, x, Wg, Wm)
    o = oracle_from_logits(g["logits"], sh.E, sh.K, sh.renorm, True)
    assert_routing_bitexact(g, o)
    assert_logits(g, x, Wg, Wm, "bf16", sh.K, sh.renorm, name=f"decode_T{T}_f{f}")
    out, ws = gpu_forward(dsc, x, Wg, Wm, W1, W3, W2)
    views = abi.workspace_views(dsc, ws)
    assert np.array_equal(views["idx"].cpu().numpy(), g["idx"])
    assert np.array_equal(views["w"].cpu().numpy(), g["w"])
    assert_grouping_bitexact(dsc, views, g["idx"])
    h1, h3, h2 = qwen3_experts_host
    ref = oracle.experts(host(x), h1, h3, h2, g["idx"], o["w"], "bf16")  # every token
    worst = assert_values(out, ref, g["idx"], "bf16")
    assert_combine(out, views, "bf16")
    nrow, wrow = assert_expert_rows(views, x, W1, W3, W2, "bf16", pick_experts(g["counts"]))
    report(name=f"decode_T{T}_f{f}", kind="values", tokens=T, worst_token_excess=worst,
           expert_rows=nrow, worst_expert_row=wrow)
    if f >= 1.0:
        assert (g["idx"] >= 0).all()


# --------------------------------------------------------------- prefill --

@pytest.mark.parametrize("f", [0.15, 0.35, 1.0])
def test_qwen3_prefill_matches_oracle(f, qwen3_experts, qwen3_experts_host):
    sh = inputs.QWEN3
    T = 8192
    W1, W3, W2 = qwen3_experts
    x = inputs.make_tokens(sh, T, seed=7, device=DEV)
    Wg = inputs.make_gate(sh, seed=0, device=DEV)
    Wm = inputs.make_mask(sh, f, seed=0, device=DEV)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    g = gpu_route(dsc, x, Wg, Wm)
    o = oracle_from_logits(g["logits"], sh.E, sh.K, sh.renorm, True)
    assert_routing_bitexact(g, o)
    # histogram over 0..K kept experts covers the whole batch
    assert g["hist"].sum() == T and len(g["hist"]) == sh.K + 1
    kept = (g["idx"] >= 0).mean()
    if f < 1.0:
        assert abs(kept - f) < 0.05, kept
        assert g["hist"][0] >= 0.01 * T, g["hist"]  # >= 1% of tokens fully masked
    else:
        assert g["hist"][sh.K] == T
    out, ws = gpu_forward(dsc, x, Wg, Wm, W1, W3, W2)
    views = abi.workspace_views(dsc, ws)
    assert np.array_equal(views["idx"].cpu().numpy(), g["idx"])
    assert_grouping_bitexact(dsc, views, g["idx"])
    assert_logits(g, x, Wg, Wm, "bf16", sh.K, sh.renorm, name=f"prefill_T{T}_f{f}")
    h1, h3, h2 = qwen3_experts_host
    # every 32nd token plus both ends: each expert's rows are in token order,
    # so the sample reaches the middle tiles of every expert's row range
    rows = strided_rows(T, 32)
    worst = assert_token_sample(out, x, h1, h3, h2, g["idx"], o["w"], "bf16", rows)
    assert_combine(out, views, "bf16")
    # whole experts: the hottest spans many 128-row tiles
    nrow, wrow = assert_expert_rows(views, x, W1, W3, W2, "bf16", pick_experts(g["counts"]))
    report(name=f"prefill_T{T}_f{f}", kind="values", tokens=len(rows),
           worst_token_excess=worst, expert_rows=nrow, worst_expert_row=wrow,
           hottest_expert_rows=int(g["counts"].max()))


# ------------------------------------------------------------ invariants --

def test_zero_mask_equals_no_mask_bitwise_bf16(qwen3_experts):
    sh = inputs.QWEN3
    W1, W3, W2 = qwen3_experts
    for T in (32, 1024):
        x = inputs.make_tokens(sh, T, seed=3, device=DEV)
        Wg = inputs.make_gate(sh, seed=0, device=DEV)
        dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
        out0, ws0 = gpu_forward(dsc, x, Wg, torch.zeros_like(Wg), W1, W3, W2)
        outn, wsn = gpu_forward(dsc, x, Wg, None, W1, W3, W2)
        assert torch.equal(out0, outn)
        assert (abi.workspace_views(dsc, ws0)["idx"] >= 0).all()


def test_unused_experts_are_never_read(qwen3_experts):
    """NaN in every expert without a kept pair changes nothing (bitwise)."""
    sh = inputs.QWEN3
    T = 32
    x = inputs.make_tokens(sh, T, seed=11, device=DEV)
    Wg = inputs.make_gate(sh, seed=0, device=DEV)
    Wm = inputs.make_mask(sh, 0.15, seed=0, device=DEV)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    W1, W3, W2 = (W.clone() for W in qwen3_experts)
    out, ws = gpu_forward(dsc, x, Wg, Wm, W1, W3, W2)
    counts = abi.workspace_views(dsc, ws)["counts"].cpu()
    unused = torch.nonzero(counts == 0).flatten().to(DEV)
    assert len(unused) > sh.E // 2
    for W in (W1, W3, W2):
        W.index_fill_(0, unused, float("nan"))
    out2, _ = gpu_forward(dsc, x, Wg, Wm, W1, W3, W2)
    assert torch.isfinite(out2.float()).all()
    assert torch.equal(out, out2)


def test_all_masked_batch_outputs_zero(qwen3_experts):
    sh = inputs.QWEN3
    T = 64
    W1, W3, W2 = qwen3_experts
    x = inputs.make_tokens(sh, T, seed=5, device=DEV)
    Wg = inputs.make_gate(sh, seed=0, device=DEV)
    Wm = torch.zeros_like(Wg)
    Wm[:, sh.d - 1] = -1.0  # z = -1 for every expert (bias feature x[d-1] = 1)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    out, ws = gpu_forward(dsc, x, Wg, Wm, W1, W3, W2)
    v = abi.workspace_views(dsc, ws)
    assert (v["idx"] == -1).all() and v["hist"][0].item() == T and v["meta"][0].item() == 0
    assert (out.float() == 0).all()


def test_route_and_forward_agree_and_are_deterministic(qwen3_experts):
    sh = inputs.QWEN3
    W1, W3, W2 = qwen3_experts
    T = 200  # ragged against every tile size
    x = inputs.make_tokens(sh, T, seed=21, device=DEV)
    Wg = inputs.make_gate(sh, seed=0, device=DEV)
    Wm = inputs.make_mask(sh, 0.35, seed=0, device=DEV)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    g = gpu_route(dsc, x, Wg, Wm)
    out1, ws = gpu_forward(dsc, x, Wg, Wm, W1, W3, W2)
    out2, _ = gpu_forward(dsc, x, Wg, Wm, W1, W3, W2, ws=ws)
    assert torch.equal(out1, out2)
    v = abi.workspace_views(dsc, ws)
    assert np.array_equal(v["idx"].cpu().numpy(), g["idx"])
    assert np.array_equal(v["counts"].cpu().numpy(), g["counts"])


def test_cuda_graph_replay_matches_eager(qwen3_experts):
    sh = inputs.QWEN3
    W1, W3, W2 = qwen3_experts
    T = 128
    x = inputs.make_tokens(sh, T, seed=31, device=DEV)
    Wg = inputs.make_gate(sh, seed=0, device=DEV)
    Wm = inputs.make_mask(sh, 0.35, seed=0, device=DEV)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    ref, ws = gpu_forward(dsc, x, Wg, Wm, W1, W3, W2)
    out = torch.empty_like(ref)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        abi.forward(dsc, x, Wg, Wm, W1, W3, W2, out, ws, stream=s)  # warm-up
        s.synchronize()
        with torch.cuda.graph(graph, stream=s):
            abi.forward(dsc, x, Wg, Wm, W1, W3, W2, out, ws, stream=s)
    out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    # new inputs written into the captured buffers are picked up
    x2 = inputs.make_tokens(sh, T, seed=32, device=DEV)
    x.copy_(x2)
    graph.replay()
    torch.cuda.synchronize()
    ref2, _ = gpu_forward(dsc, x2, Wg, Wm, W1, W3, W2)
    assert torch.equal(out, ref2)


# ---------------------------------------------------- threshold ablation --

@pytest.mark.parametrize("tau", [0.3, 0.7])
def test_mask_threshold_tau_matches_oracle(tau, qwen3_experts, qwen3_experts_host):
    """Eq. (6) with tau != 0.5 (the paper's threshold ablation): decisions
    bit-exact with the oracle fed the same logits and the same fp32 threshold,
    values within the bar, kept fraction ordered by tau."""
    sh = inputs.QWEN3
    W1, W3, W2 = qwen3_experts
    T = 64
    x = inputs.make_tokens(sh, T, seed=77, device=DEV)
    Wg = inputs.make_gate(sh, seed=0, device=DEV)
    Wm = inputs.make_mask(sh, 0.5, seed=0, device=DEV)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm, tau=tau)
    thr = dsc.mask_logit_threshold
    assert thr != 0.0
    g = gpu_route(dsc, x, Wg, Wm)
    o = oracle_from_logits(g["logits"], sh.E, sh.K, sh.renorm, True, tau_logit=thr)
    assert_routing_bitexact(g, o)
    assert_logits(g, x, Wg, Wm, "bf16", sh.K, sh.renorm, tau_logit=thr, name=f"tau_{tau}")
    base = gpu_route(abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm), x, Wg, Wm)
    kept, kept05 = (g["idx"] >= 0).sum(), (base["idx"] >= 0).sum()
    assert (kept < kept05) if tau > 0.5 else (kept > kept05)
    out, ws = gpu_forward(dsc, x, Wg, Wm, W1, W3, W2)
    views = abi.workspace_views(dsc, ws)
    assert_grouping_bitexact(dsc, views, g["idx"])
    h1, h3, h2 = qwen3_experts_host
    ref = oracle.experts(host(x), h1, h3, h2, g["idx"], o["w"], "bf16")  # every token
    assert_values(out, ref, g["idx"], "bf16")
    assert_combine(out, views, "bf16")


# ----------------------------------------------------------- edge shapes --

EDGE = [
    # (name, T, d, E, I, K, renorm, f)
    ("qwen15_like_E60", 40, 2048, 60, 1408, 4, 0, 0.35),
    ("dsv2lite_like_E64", 33, 2048, 64, 1408, 6, 1, 0.5),
    ("top1", 17, 1024, 32, 256, 1, 1, 0.5),
    ("top16_E256", 9, 512, 256, 384, 16, 1, 0.6),
    ("ragged_T3_renorm0", 3, 2048, 128, 768, 8, 0, 0.35),
    ("T1_all_kept", 1, 2048, 128, 768, 8, 1, 1.0),
    ("bn64_T600", 600, 1024, 128, 256, 8, 1, 0.35),
    ("bn32_T400", 400, 2048, 128, 768, 8, 1, 0.6),
    # the chunked grouping's larger chunks: 128 tokens (T > 16384) and 256
    # tokens (T > 32768), with a ragged last chunk
    ("chunked_T20000_ct128", 20000, 128, 8, 128, 2, 0, 0.5),
    ("chunked_T40003_ct256", 40003, 128, 16, 128, 2, 1, 0.35),
]


@pytest.mark.parametrize("name,T,d,E,I,K,renorm,f", EDGE, ids=[e[0] for e in EDGE])
def test_edge_shapes_match_oracle(name, T, d, E, I, K, renorm, f):
    sh = inputs.Shape(d=d, E=E, K=K, I=I, renorm=renorm, dtype="bf16")
    x = inputs.make_tokens(sh, T, seed=T, device=DEV)
    Wg = inputs.make_gate(sh, seed=1, device=DEV)
    Wm = inputs.make_mask(sh, f, seed=1, device=DEV)
    W1, W3, W2 = inputs.make_experts(sh, seed=1, device=DEV)
    dsc = abi.desc(T, d, E, I, K, "bf16", renorm)
    g = gpu_route(dsc, x, Wg, Wm)
    o = oracle_from_logits(g["logits"], E, K, renorm, True)
    assert_routing_bitexact(g, o)
    assert_logits(g, x, Wg, Wm, "bf16", K, renorm, name=f"edge_{name}")
    out, ws = gpu_forward(dsc, x, Wg, Wm, W1, W3, W2)
    views = abi.workspace_views(dsc, ws)
    assert_grouping_bitexact(dsc, views, g["idx"])
    ref = oracle_values(x, W1, W3, W2, g["idx"], o["w"], "bf16")
    assert_values(out, ref, g["idx"], "bf16")
    assert_combine(out, views, "bf16")
    assert_expert_rows(views, x, W1, W3, W2, "bf16", pick_experts(g["counts"]))


def test_empty_batch_is_a_no_op():
    sh = inputs.QWEN3
    dsc = abi.desc(0, sh.d, sh.E, sh.I, sh.K, "bf16", 1)
    ws = abi.alloc_workspace(dsc, DEV)
    x = torch.empty((0, sh.d), dtype=torch.bfloat16, device=DEV)
    W = torch.empty((16,), dtype=torch.bfloat16, device=DEV)
    out = torch.empty((0, sh.d), dtype=torch.bfloat16, device=DEV)
    abi.forward(dsc, x if x.numel() else W, W, None, W, W, W, out if out.numel() else W, ws)
    abi.check(dsc, ws)


# ----------------------------------------------------------------- large --

@pytest.mark.parametrize("T,f", [(16, 0.15), (16, 0.5), (4096, 0.15), (4096, 0.5)])
def test_large_layer_matches_oracle(T, f, large_layer):
    sh = inputs.LARGE
    W1, W3, W2, Wg = large_layer
    x = inputs.make_tokens(sh, T, seed=40 + T, device=DEV)
    Wm = inputs.make_mask(sh, f, seed=0, device=DEV)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    g = gpu_route(dsc, x, Wg, Wm)
    o = oracle_from_logits(g["logits"], sh.E, sh.K, sh.renorm, True)
    assert_routing_bitexact(g, o)
    assert_logits(g, x, Wg, Wm, "bf16", sh.K, sh.renorm, name=f"large_T{T}_f{f}")
    out, ws = gpu_forward(dsc, x, Wg, Wm, W1, W3, W2)
    views = abi.workspace_views(dsc, ws)
    assert_grouping_bitexact(dsc, views, g["idx"])
    # tokens spread over the batch (oracle on the experts they use only)
    rows = strided_rows(T, max(1, T // 4), ends=2)
    worst = assert_token_sample(out, x, W1, W3, W2, g["idx"], o["w"], "bf16", rows,
                                compact=True)
    assert_combine(out, views, "bf16")
    nrow, wrow = assert_expert_rows(views, x, W1, W3, W2, "bf16",
                                    pick_experts(g["counts"], n_random=1), max_rows=96)
    report(name=f"large_T{T}_f{f}", kind="values", tokens=len(rows), worst_token_excess=worst,
           expert_rows=nrow, worst_expert_row=wrow)


@pytest.fixture(scope="module")
def large_layer():
    sh = inputs.LARGE
    W1, W3, W2 = inputs.make_experts(sh, seed=0, device=DEV)
    Wg = inputs.make_gate(sh, seed=0, device=DEV, zipf=None)
    yield W1, W3, W2, Wg
    del W1, W3, W2
    torch.cuda.empty_cache()


# ------------------------------------------------------ 48-layer stack --

def test_48_layer_decode_stack_matches_oracle():
    """The 48-layer stack (48 x 1.2 GB of expert weights on the GPU): every
    layer's routing is bit-exact with the oracle fed that layer's logits, and
    every eighth layer's outputs match the oracle on sampled tokens, each layer
    fed the GPU's own input (teacher forcing)."""
    sh = inputs.QWEN3
    T = 64
    x = inputs.make_tokens(sh, T, seed=501, device=DEV)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    ws = abi.alloc_workspace(dsc, DEV)
    kept = []
    for layer in range(inputs.STACK_LAYERS):
        W1, W3, W2 = inputs.make_experts(sh, seed=0, device=DEV, layer=layer)
        Wg = inputs.make_gate(sh, seed=0, device=DEV, layer=layer)
        Wm = inputs.make_mask(sh, inputs.stack_kept_fraction(layer), seed=0, device=DEV,
                              layer=layer)
        g = gpu_route(dsc, x, Wg, Wm)
        o = oracle_from_logits(g["logits"], sh.E, sh.K, sh.renorm, True)
        assert_routing_bitexact(g, o)
        assert_logits(g, x, Wg, Wm, "bf16", sh.K, sh.renorm, name=f"stack_layer{layer}")
        out, _ = gpu_forward(dsc, x, Wg, Wm, W1, W3, W2, ws=ws)
        assert_combine(out, abi.workspace_views(dsc, ws), "bf16")
        if layer % 8 == 7:
            assert_token_sample(out, x, W1, W3, W2, g["idx"], o["w"], "bf16",
                                strided_rows(T, 16, ends=1), compact=True)
        kept.append((g["idx"] >= 0).mean())
        x = inputs.stack_next_input(out, layer)
        del W1, W3, W2
    assert 0.05 < min(kept) and max(kept) < 0.7, kept


# -------------------------------------------------------- shared experts --

SHARED = [
    # (name, shape, n_shared, T, kept fraction)
    ("dsv2lite_decode_T33", inputs.DSV2_LITE, inputs.DSV2_LITE_SHARED, 33, 0.35),
    ("dsv2lite_prefill_T2048", inputs.DSV2_LITE, inputs.DSV2_LITE_SHARED, 2048, 0.35),
    ("dsv2lite_decode_T300_renorm", inputs.Shape(2048, 64, 6, 1408, 1, "bf16"), 2, 300, 0.6),
    ("qwen15_decode_T40", inputs.QWEN15_MOE, inputs.QWEN15_MOE_SHARED, 40, 0.15),
    ("qwen15_decode_T1_unmasked", inputs.QWEN15_MOE, inputs.QWEN15_MOE_SHARED, 1, 1.0),
]


@pytest.mark.parametrize("name,sh,S,T,f", SHARED, ids=[c[0] for c in SHARED])
def test_shared_experts_match_oracle(name, sh, S, T, f):
    """Always-on shared experts (news article §5) on top of the masked routed
    experts: routing bit-exact, outputs = routed sum + shared experts."""
    d, E, K, I, renorm = sh.d, sh.E, sh.K, sh.I, sh.renorm
    x = inputs.make_tokens(sh, T, seed=T + 5, device=DEV)
    Wg = inputs.make_gate(sh, seed=3, device=DEV)
    Wm = inputs.make_mask(sh, f, seed=3, device=DEV)
    W1, W3, W2 = inputs.make_experts(sh, seed=3, device=DEV)
    W1s, W3s, W2s = inputs.make_shared_experts(sh, S, seed=3, device=DEV)
    dsc = abi.desc(T, d, E, I, K, "bf16", renorm, n_shared=S, I_shared=I)
    g = gpu_route(dsc, x, Wg, Wm)
    o = oracle_from_logits(g["logits"], E, K, renorm, True)
    assert_routing_bitexact(g, o)
    assert_logits(g, x, Wg, Wm, "bf16", K, renorm, name=f"shared_{name}")
    ws = abi.alloc_workspace(dsc, DEV)
    out = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    abi.forward_shared(dsc, x, Wg, Wm, W1, W3, W2, W1s, W3s, W2s, out, ws)
    abi.check(dsc, ws)
    # every 16th token and both ends, end to end (routed sum + shared experts)
    rows = strided_rows(T, 16)
    xr = host(x[torch.as_tensor(rows, device=DEV)])
    ref = oracle.experts(xr, host(W1), host(W3), host(W2), g["idx"][rows], o["w"][rows], "bf16")
    oracle.add_shared(ref, xr, host(W1s), host(W3s), host(W2s), "bf16")
    o_rows = out.float().cpu().numpy().astype(np.float64)[rows]
    assert (bf16_excess(o_rows, ref) <= BF16_TOL_RMS).all()
    views = abi.workspace_views(dsc, ws)
    # one slab of the shared experts' rows per split of their down reduction
    assert_combine(out, views, "bf16", n_shared=S * views["plan"]["sh_split2"], ys=views["ys"])


def test_shared_experts_serve_all_masked_tokens():
    """Every candidate masked: the output is the shared experts alone."""
    sh, S, T = inputs.DSV2_LITE, inputs.DSV2_LITE_SHARED, 48
    d, E, K, I = sh.d, sh.E, sh.K, sh.I
    x = inputs.make_tokens(sh, T, seed=9, device=DEV)
    Wg = inputs.make_gate(sh, seed=3, device=DEV)
    Wm = inputs.make_mask(sh, 0.0, device=DEV)
    W1, W3, W2 = inputs.make_experts(sh, seed=3, device=DEV)
    W1s, W3s, W2s = inputs.make_shared_experts(sh, S, seed=3, device=DEV)
    dsc = abi.desc(T, d, E, I, K, "bf16", sh.renorm, n_shared=S, I_shared=I)
    ws = abi.alloc_workspace(dsc, DEV)
    out = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    abi.forward_shared(dsc, x, Wg, Wm, W1, W3, W2, W1s, W3s, W2s, out, ws)
    abi.check(dsc, ws)
    assert (abi.workspace_views(dsc, ws)["idx"] == -1).all()
    ref = np.zeros((T, d))
    oracle.add_shared(ref, host(x), host(W1s), host(W3s), host(W2s), "bf16")
    assert (bf16_excess(out.float().cpu().numpy().astype(np.float64), ref) <= BF16_TOL_RMS).all()


def test_shared_experts_second_stream_graph_replay_and_dirty_workspace():
    """The shared experts run on a second stream forked from the caller's and
    joined before the combine.  Repeated calls, a CUDA-graph capture of the
    call (fork and join become graph edges) and a workspace left dirty give
    bitwise the same output; no call is left unjoined (the capture ends)."""
    sh, S, T = inputs.DSV2_LITE, inputs.DSV2_LITE_SHARED, 64
    d, E, K, I = sh.d, sh.E, sh.K, sh.I
    x = inputs.make_tokens(sh, T, seed=21, device=DEV)
    Wg = inputs.make_gate(sh, seed=3, device=DEV)
    Wm = inputs.make_mask(sh, 0.15, seed=3, device=DEV)
    W1, W3, W2 = inputs.make_experts(sh, seed=3, device=DEV)
    W1s, W3s, W2s = inputs.make_shared_experts(sh, S, seed=3, device=DEV)
    dsc = abi.desc(T, d, E, I, K, "bf16", sh.renorm, n_shared=S, I_shared=I)
    ws = abi.alloc_workspace(dsc, DEV)
    ws.fill_(0xA5)
    ref = torch.empty((T, d), dtype=torch.bfloat16, device=DEV)
    abi.forward_shared(dsc, x, Wg, Wm, W1, W3, W2, W1s, W3s, W2s, ref, ws)
    abi.check(dsc, ws)
    out = torch.empty_like(ref)
    for _ in range(3):
        out.zero_()
        abi.forward_shared(dsc, x, Wg, Wm, W1, W3, W2, W1s, W3s, W2s, out, ws)
        abi.check(dsc, ws)
        assert torch.equal(out, ref)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    gout = torch.zeros_like(ref)
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            abi.forward_shared(dsc, x, Wg, Wm, W1, W3, W2, W1s, W3s, W2s, gout, ws, stream=s)
    for _ in range(3):
        gout.zero_()
        g.replay()
        torch.cuda.synchronize()
        abi.check(dsc, ws)
        assert torch.equal(gout, ref)


_FIRST_CALL_CAPTURED = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
from dynamic_expert_routing_router_b200 import abi, inputs
sh, S, T = inputs.DSV2_LITE, inputs.DSV2_LITE_SHARED, 24
x = inputs.make_tokens(sh, T, seed=41, device="cuda")
Wg = inputs.make_gate(sh, seed=3, device="cuda")
Wm = inputs.make_mask(sh, 0.35, seed=3, device="cuda")
W1, W3, W2 = inputs.make_experts(sh, seed=3, device="cuda")
W1s, W3s, W2s = inputs.make_shared_experts(sh, S, seed=3, device="cuda")
dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm, n_shared=S, I_shared=sh.I)
ws = abi.alloc_workspace(dsc, "cuda")
gout = torch.zeros((T, sh.d), dtype=torch.bfloat16, device="cuda")
torch.cuda.synchronize()
s = torch.cuda.Stream()
s.wait_stream(torch.cuda.current_stream())
g = torch.cuda.CUDAGraph()
with torch.cuda.stream(s):
    with torch.cuda.graph(g, stream=s):  # the process's first shared-expert call
        abi.forward_shared(dsc, x, Wg, Wm, W1, W3, W2, W1s, W3s, W2s, gout, ws, stream=s)
g.replay()
torch.cuda.synchronize()
abi.check(dsc, ws)
ref = torch.empty_like(gout)
abi.forward_shared(dsc, x, Wg, Wm, W1, W3, W2, W1s, W3s, W2s, ref, ws)  # eager: second stream
abi.check(dsc, ws)
assert torch.equal(gout, ref)
print("ok")
"""


def test_shared_experts_first_call_inside_a_capture():
    """A process whose first shared-expert call is captured: the library
    creates no stream inside the capture and runs the shared experts on the
    caller's stream; the replay equals a later eager call (second stream)
    bit for bit."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _FIRST_CALL_CAPTURED, root], capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr
