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
    """Half a unit in the last place of bfloat16 (8 significant bits) at |a|;
    below the smallest normal, 2^-126, the spacing stays that of the
    subnormals, 2^-133."""
    a = np.abs(np.asarray(a, np.float64))
    e = np.maximum(np.floor(np.log2(np.where(a > 0, a, 1.0))), -126.0)
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


# ------------------------------------------------ router logits vs oracle --
# The library's fp32 router logits (tensor cores for bf16, CUDA cores for fp32)
# against the oracle's fp64 logits of the same stored inputs.  Bar, element by
# element: |gpu - ref| <= LOGIT_TOL * sum_j |x_tj * W_ej|, the size of the
# terms the fp32 sum adds (a sum of d terms in fp32 errs by at most about
# d * 2^-24 of that in the worst case, ~sqrt(d) * 2^-24 typically).
LOGIT_TOL = 1e-5

REPORT = []  # per-workload observations (written out by conftest when asked)


def report(**kv):
    REPORT.append(kv)


def assert_logits(g, x, Wg, Wm, dtype, K, renorm, tau_logit=0.0, name=""):
    """Returns the worst |gpu - ref| / sum|x w| over r and z; also reports the
    routing-decision flip rate between the library's decisions and the
    oracle's decisions taken on its own fp64 logits (reported, not gated)."""
    r, z = oracle.logits(host(x), host(Wg), None if Wm is None else host(Wm), dtype)
    E = r.shape[1]
    xa = x.double().abs()
    worst = 0.0
    for ref, W, lo in ((r, Wg, 0), (z, Wm, E)):
        if ref is None:
            continue
        bound = (xa @ W.double().abs().T).cpu().numpy()
        got = g["logits"][:, lo:lo + E].astype(np.float64)
        err = np.abs(got - ref)
        ratio = err / np.where(bound > 0, bound, 1.0)
        assert (err <= LOGIT_TOL * bound + 1e-30).all(), \
            f"router logits off the fp64 oracle: worst {ratio.max():.3g} of sum|x w|"
        worst = max(worst, float(ratio.max()) if ratio.size else 0.0)
    o64 = oracle.route(r, z, K, renorm, tau_logit)
    flips = g["idx"] != o64["idx"]
    report(name=name, kind="router", T=int(r.shape[0]), worst_logit_err_rel=worst,
           slot_flip_rate=float(flips.mean()) if flips.size else 0.0,
           token_flip_rate=float(flips.any(axis=1).mean()) if flips.size else 0.0)
    return worst


# --------------------------------------------- combine, teacher-forced ----

def assert_combine(out, views, dtype, n_shared=0, ys=None):
    """Every token: out_t = sum over kept k (slot order) of w_tk * Y[pos(t,k)]
    (+ the shared experts' rows), from the library's own Y, in fp64.  Bar: the
    output's rounding (half an ulp, bf16) plus 1e-6 of sum |w y| for the fp32
    sums (at most 16 + n_shared terms, each rounded at 2^-24)."""
    idx = views["idx"].cpu().numpy()
    w = views["w"].cpu().numpy().astype(np.float64)
    pos = views["pair_pos"].cpu().numpy()
    Y = views["y"]
    T, K = idx.shape
    d = Y.shape[1]
    ref = np.zeros((T, d))
    mag = np.zeros((T, d))
    t, k = np.nonzero(idx >= 0)
    if len(t):
        rows = torch.as_tensor(pos[t, k].astype(np.int64), device=Y.device)
        Yk = Y.index_select(0, rows).double().cpu().numpy()
        contrib = w[t, k][:, None] * Yk
        # slot order per token: np.add.at accumulates in the order of (t, k)
        np.add.at(ref, t, contrib)
        np.add.at(mag, t, np.abs(contrib))
    if n_shared:
        Ys = ys.double().cpu().numpy().reshape(n_shared, T, d)
        for s in range(n_shared):
            ref += Ys[s]
            mag += np.abs(Ys[s])
    o = out.float().cpu().numpy().astype(np.float64)
    tol = 1e-6 * mag
    if dtype == "bf16":
        tol = tol + bf16_half_ulp(np.maximum(np.abs(o), np.abs(ref)))
    bad = np.abs(o - ref) > tol
    if bad.any():
        at = np.argwhere(bad)[:5]
        detail = [(int(i), int(j), float(o[i, j]), float(ref[i, j]), float(tol[i, j]))
                  for i, j in at]
        raise AssertionError(f"combine differs at {int(bad.sum())} elements, first "
                             f"(t, j, out, ref, tol): {detail}")
    empty = (idx < 0).all(axis=1)
    if not n_shared:
        assert (o[empty] == 0).all()


# ----------------------------------------- per-expert rows vs the oracle --

def pick_experts(counts, n_random=2, seed=0):
    """The hottest expert (most rows: spans the most tiles), the highest-id
    expert with a kept pair, and n_random others with kept pairs (seeded)."""
    used = np.nonzero(counts > 0)[0]
    if len(used) == 0:
        return []
    pick = {int(np.argmax(counts)), int(used[-1])}
    rng = np.random.default_rng(seed)
    rest = [e for e in used if e not in pick]
    for e in rng.permutation(rest)[:n_random]:
        pick.add(int(e))
    return sorted(pick)


def assert_expert_rows(views, x, W1, W3, W2, dtype, experts, max_rows=512):
    """Y rows (the library's fp32 per-pair expert outputs) of `experts` against
    the oracle's E_e(x_t) for their kept pairs: every row up to max_rows,
    else an even stride that still reaches every tile.  Bar per row: bf16
    max_j |Y - ref| <= 2e-2 * RMS_j(ref) (Y is fp32: no output rounding to
    discount); fp32 max|Y - ref| <= 1e-4 * max|ref| over the rows.  Returns
    (rows checked, worst ratio)."""
    idx = views["idx"].cpu().numpy()
    pos = views["pair_pos"].cpu().numpy()
    Y = views["y"]
    checked, worst = 0, 0.0
    for e in experts:
        t, k = np.nonzero(idx == e)  # token order: the expert's row order
        if len(t) == 0:
            continue
        stride = max(1, -(-len(t) // max_rows))
        sel = np.unique(np.concatenate([np.arange(0, len(t), stride), [len(t) - 1]]))
        t, k = t[sel], k[sel]
        sel_e = torch.as_tensor([e], device=W1.device, dtype=torch.long)
        c1, c3, c2 = (host(W.index_select(0, sel_e)) for W in (W1, W3, W2))
        xs = host(x[torch.as_tensor(t.astype(np.int64), device=x.device)])
        one = np.zeros((len(t), 1), np.int32)
        ref = oracle.experts(xs, c1, c3, c2, one, np.ones((len(t), 1)), dtype)
        rows = torch.as_tensor(pos[t, k].astype(np.int64), device=Y.device)
        got = Y.index_select(0, rows).double().cpu().numpy()
        err = np.abs(got - ref).max(axis=1)
        if dtype == "bf16":
            rms = np.sqrt((ref ** 2).mean(axis=1))
            ratio = err / np.where(rms > 0, rms, 1.0)
            assert (ratio <= BF16_TOL_RMS).all(), (e, float(ratio.max()))
        else:
            ratio = err / max(np.abs(ref).max(), 1e-30)
            assert (ratio <= F32_TOL_MAX).all(), (e, float(ratio.max()))
        checked += len(t)
        worst = max(worst, float(ratio.max()))
    return checked, worst


def strided_rows(T, stride, ends=8):
    """Tokens 0..ends-1, every stride-th token, and the last `ends` tokens."""
    r = set(range(min(ends, T))) | set(range(0, T, stride)) | set(range(max(0, T - ends), T))
    return np.array(sorted(r), np.int64)


def assert_token_sample(out, x, W1, W3, W2, idx, w, dtype, rows, compact=False):
    """End-to-end output rows `rows` against the oracle (decisions shared);
    compact=True hands the oracle only the experts those rows use."""
    rows = np.asarray(rows, np.int64)
    sub_idx, sub_w = idx[rows], w[rows]
    xs = host(x[torch.as_tensor(rows, device=x.device)])
    if compact:
        c1, c3, c2, cidx = compact_experts(W1, W3, W2, sub_idx)
    else:
        c1, c3, c2 = W1, W3, W2
        cidx = sub_idx
    ref = oracle.experts(xs, c1, c3, c2, cidx, sub_w, dtype)
    o = out[torch.as_tensor(rows, device=out.device)]
    return assert_values(o, ref, sub_idx, dtype)
