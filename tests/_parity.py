"""Helpers shared by the GPU parity tests: run the CUDA library through its C
ABI, run the oracle on the same inputs, and compare.

Routing decisions (candidate ids, mask, counts, histogram, grouping) must be
bit-exact when the oracle is fed the library's own fp32 logits; values are
compared with the oracle's fp64 expert math applied to those decisions.

  fp32 layer: max|out - ref| <= 1e-4 * max|ref|  (normwise relative error)
  bf16 layer: for every token t that keeps an expert,
      max_j ( |out_tj - ref_tj| - ulp_bf16(ref_tj)/2 ) <= 2e-2 * RMS_j(ref_t)

and tokens with no kept candidate must be exactly 0 in both.  Two readings of
the bf16 bar "max-abs-error <= 2e-2 x RMS(ref output)": the RMS is per token
(each token's output is its own vector, and the softmax weights of its kept
experts scale tokens by an order of magnitude against each other), and the
output's own rounding to bf16 is not counted as error: rounding the exact fp64
result to bf16 alone already exceeds 2e-2 x RMS at the largest elements
(test_tolerance_reading.py shows it on CPU).
"""
import numpy as np
import torch

import oracle
from dynamic_expert_routing_router_b200 import abi, inputs

BF16_TOL_RMS = 2e-2
F32_TOL_MAX = 1e-4


def host(t):
    return inputs.host_array(t)


def gpu_route(dsc, x, Wg, Wm):
    """beam_moe_route -> numpy dict (idx, w, counts, hist, logits)."""
    T, K, E = dsc.T, dsc.K, dsc.E
    dev = x.device
    idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    w = torch.empty((T, K), dtype=torch.float32, device=dev)
    counts = torch.empty((E,), dtype=torch.int32, device=dev)
    hist = torch.empty((K + 1,), dtype=torch.int32, device=dev)
    logits = torch.full((T, 2 * E), float("nan"), dtype=torch.float32, device=dev)
    ws = abi.alloc_workspace(dsc, dev)
    abi.route(dsc, x, Wg, Wm, idx, w, counts, hist, logits, ws)
    abi.check(dsc, ws)
    return {k: v.cpu().numpy() for k, v in
            dict(idx=idx, w=w, counts=counts, hist=hist, logits=logits).items()}


def gpu_forward(dsc, x, Wg, Wm, W1, W3, W2, ws=None):
    if ws is None:
        ws = abi.alloc_workspace(dsc, x.device)
    out = torch.empty((dsc.T, dsc.d), dtype=x.dtype, device=x.device)
    abi.forward(dsc, x, Wg, Wm, W1, W3, W2, out, ws)
    abi.check(dsc, ws)
    return out, ws


def oracle_from_logits(logits, E, K, renorm, has_mask, tau_logit=0.0):
    r = np.ascontiguousarray(logits[:, :E])
    z = np.ascontiguousarray(logits[:, E:]) if has_mask else None
    return oracle.route(r, z, K, renorm, tau_logit)


def assert_routing_bitexact(g, o):
    assert np.array_equal(g["idx"], o["idx"]), "candidate/mask decisions differ"
    assert np.array_equal(g["counts"], o["counts"])
    assert np.array_equal(g["hist"], o["hist"])
    # weights: fp32 softmax vs the oracle's fp64 softmax of the same logits
    np.testing.assert_allclose(g["w"], o["w"], rtol=2e-6, atol=1e-7)
    assert (g["w"][g["idx"] < 0] == 0).all()


def assert_grouping_bitexact(dsc, views, idx):
    """The library's padded expert grouping equals the oracle's permutation."""
    E, K = dsc.E, dsc.K
    BN = views["plan"]["BN"]
    offsets, pairs = oracle.permutation(idx, E)
    expect, tiles = [], []
    for e in range(E):
        seg = list(pairs[offsets[e]:offsets[e + 1]])
        row0 = len(expect)
        for j in range(0, len(seg), BN):
            tiles.append((e, row0 + j, min(BN, len(seg) - j)))
        expect += seg + [-1] * ((-len(seg)) % BN)
    meta = views["meta"].cpu().numpy()
    assert meta[0] == len(tiles) and meta[1] == len(expect) and meta[2] == len(pairs)
    pair = views["pair"].cpu().numpy()[: len(expect)]
    assert np.array_equal(pair, np.array(expect, np.int32))
    got_tiles = views["tiles"].cpu().numpy()[: len(tiles), :3]
    assert np.array_equal(got_tiles, np.array(tiles, np.int32).reshape(-1, 3))
    pos = views["pair_pos"].cpu().numpy()
    t, k = np.nonzero(idx >= 0)
    assert np.array_equal(pair[pos[t, k]], (t * K + k).astype(np.int32))


def bf16_half_ulp(a):
    """Half a unit in the last place of bfloat16 (8 significant bits) at |a|."""
    a = np.abs(np.asarray(a, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(e - 8), 0.0)


def bf16_excess(o, ref):
    """Per token: max_j(|o - ref| - ulp/2) / RMS_j(ref), for rows of ref != 0."""
    half = bf16_half_ulp(np.maximum(np.abs(o), np.abs(ref)))
    ex = (np.abs(o - ref) - half).max(axis=1)
    rms = np.sqrt((ref ** 2).mean(axis=1))
    return ex / np.where(rms > 0, rms, 1.0)


def assert_values(out, ref, idx, dtype, rows=None):
    """out: torch [T,d] (or the sampled rows), ref: fp64 [n,d] for `rows`."""
    o = out.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        o = o[rows]
        idx = idx[rows]
    empty = (idx < 0).all(axis=1)
    assert (o[empty] == 0).all() and (ref[empty] == 0).all(), "all-masked tokens must be 0"
    diff = np.abs(o - ref).max() if o.size else 0.0
    if dtype == "bf16":
        worst = bf16_excess(o[~empty], ref[~empty]).max() if (~empty).any() else 0.0
        assert worst <= BF16_TOL_RMS, worst
        return worst
    else:
        mx = np.abs(ref).max() if ref.size else 0.0
        assert diff <= F32_TOL_MAX * mx + 1e-30, (diff, mx)
    return diff


def oracle_values(x, W1, W3, W2, idx, w, dtype, t_begin=0, t_end=None):
    return oracle.experts(host(x), host(W1), host(W3), host(W2), idx, w, dtype,
                          t_begin=t_begin, t_end=t_end)


def compact_experts(W1, W3, W2, idx):
    """Host copies of only the experts in `idx` (>= 0) and idx remapped to them."""
    used = np.unique(idx[idx >= 0])
    remap = -np.ones(W1.shape[0], np.int64)
    remap[used] = np.arange(len(used))
    sel = torch.as_tensor(used, device=W1.device, dtype=torch.long)
    if len(used) == 0:
        sel = torch.zeros(1, device=W1.device, dtype=torch.long)
    c1, c3, c2 = (host(W.index_select(0, sel)) for W in (W1, W3, W2))
    new_idx = np.where(idx >= 0, remap[np.maximum(idx, 0)], -1).astype(np.int32)
    return c1, c3, c2, new_idx
