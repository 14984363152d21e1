"""Pins of the fp64 oracle against facts the method and mathematics fix.

The oracle is the definition the CUDA path is compared with, so it is checked
here against things other than itself: library routines (sorts, softmax),
closed forms, the invariants the BEAM paper states, brute force over all 2^K
masks, and textbook special cases.  Each test names the mistake it would catch.

Paper: "BEAM: Binary Expert Activation Masking for Dynamic Routing in MoE"
(arXiv 2605.14438), §3.1 Eq. (1)-(3), §3.2 Eq. (4)-(8).
"""
import itertools
import math

import numpy as np
import pytest
from scipy.special import expit, softmax

import oracle

RNG = np.random.default_rng(1234)


def _rand_layer(T, d, E, I, rng, scale_gate=1.0):
    x = rng.standard_normal((T, d)).astype(np.float32)
    Wg = (rng.standard_normal((E, d)) * scale_gate / math.sqrt(d)).astype(np.float32)
    Wm = (rng.standard_normal((E, d)) / math.sqrt(d)).astype(np.float32)
    W1 = (rng.standard_normal((E, I, d)) / math.sqrt(d)).astype(np.float32)
    W3 = (rng.standard_normal((E, I, d)) / math.sqrt(d)).astype(np.float32)
    W2 = (rng.standard_normal((E, d, I)) / math.sqrt(I)).astype(np.float32)
    return x, Wg, Wm, W1, W3, W2


def _silu(a):
    return a * expit(a)


def _dense_expert(x, W1, W3, W2, e):
    """Expert e on every row of x, fp64 numpy matmuls (Eq. 3, delta = SiLU)."""
    x = x.astype(np.float64)
    a = x @ W1[e].astype(np.float64).T
    b = x @ W3[e].astype(np.float64).T
    return (_silu(a) * b) @ W2[e].astype(np.float64).T


# ---------------------------------------------------------------- routing --

def test_topk_matches_stable_library_sort():
    """Top-K with ties -> lower index equals a stable lexsort on (-r, id).

    Catches: ascending instead of descending order, ties to the higher index,
    off-by-one in K."""
    T, E, K = 200, 16, 5
    # Logits on a coarse grid so that exact ties are frequent.
    r = RNG.integers(-3, 4, size=(T, E)).astype(np.float64) * 0.5
    out = oracle.route(r, None, K, renorm=1)
    for t in range(T):
        order = np.lexsort((np.arange(E), -r[t]))  # primary key -r, then id
        assert list(out["cand"][t]) == list(order[:K])
    assert (out["idx"] == out["cand"]).all()  # no mask: every candidate kept


def test_softmax_weights_match_scipy_both_conventions():
    """renorm=1: softmax over the Top-K (Eq. 4), sums to 1.  renorm=0: the
    full softmax restricted to the Top-K, sums to < 1.

    Catches: a missing or wrong normaliser, a missing max shift (overflow),
    the two conventions swapped."""
    T, E, K = 64, 12, 3
    r = RNG.standard_normal((T, E)) * 30.0  # large spread: exp would overflow unshifted
    a = oracle.route(r, None, K, renorm=1)
    b = oracle.route(r, None, K, renorm=0)
    for t in range(T):
        c = a["cand"][t]
        np.testing.assert_allclose(a["g"][t], softmax(r[t][c]), rtol=1e-13, atol=1e-300)
        np.testing.assert_allclose(b["g"][t], softmax(r[t])[c], rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(a["g"].sum(1), 1.0, rtol=1e-14)
    assert (b["g"].sum(1) <= 1.0 + 1e-15).all()
    # With K = E both conventions are the same distribution.
    full = oracle.route(r, None, E, renorm=1)
    full0 = oracle.route(r, None, E, renorm=0)
    np.testing.assert_allclose(full["g"], full0["g"], rtol=1e-13)


def test_mask_threshold_is_sigmoid_half():
    """Eq. (6): m = 1 iff sigmoid(z) >= 0.5, i.e. iff z >= 0 (z = 0 kept).

    Catches: a strict '>' (z = 0 would drop every candidate at zero init),
    a flipped sign, comparing g instead of z."""
    E, K = 4, 4
    r = np.array([[4.0, 3.0, 2.0, 1.0]] * 6)
    z = np.array([
        [0.0, -0.0, 1e-300, -1e-300],
        [5.0, -5.0, 0.5, -0.5],
        [np.nan, 0.0, 0.0, 0.0],
        [-1.0, -1.0, -1.0, -1.0],
        [1.0, 1.0, 1.0, 1.0],
        [-1e-12, 1e-12, 0.0, 2.0],
    ])
    out = oracle.route(r, z, K, renorm=1)
    m = out["idx"] >= 0
    with np.errstate(invalid="ignore"):
        expect = np.where(np.isnan(z), False, expit(z) >= 0.5)
    # expit(+-1e-300) rounds to exactly 0.5, so use the exact rule there.
    expect[0] = [True, True, True, False]
    expect[5] = [False, True, True, True]
    assert (m == expect).all()
    # Eq. (7): masked weights are exactly 0, kept ones unchanged (no renorm).
    assert (out["w"][~m] == 0.0).all()
    assert (out["w"][m] == out["g"][m]).all()
    # kept per row: 3, 2, 3, 0, 4, 3
    assert list(out["hist"]) == [1, 0, 1, 3, 1]
    assert out["counts"].sum() == m.sum()


def test_counts_and_hist_are_consistent():
    """counts[e] = #kept pairs on e; hist[n] = #tokens with n kept."""
    T, E, K = 300, 10, 4
    r = RNG.standard_normal((T, E))
    z = RNG.standard_normal((T, E))
    out = oracle.route(r, z, K, renorm=0)
    kept = out["idx"][out["idx"] >= 0]
    assert (out["counts"] == np.bincount(kept, minlength=E)).all()
    assert (out["hist"] == np.bincount((out["idx"] >= 0).sum(1), minlength=K + 1)).all()


def test_permutation_matches_library_sort():
    """Kept pairs grouped by (expert, token) ascending; masked pairs absent."""
    T, E, K = 97, 9, 3
    r = RNG.standard_normal((T, E))
    z = RNG.standard_normal((T, E))
    out = oracle.route(r, z, K, renorm=1)
    offsets, pairs = oracle.permutation(out["idx"], E)
    triples = sorted((int(out["idx"][t, k]), t, k) for t in range(T) for k in range(K)
                     if out["idx"][t, k] >= 0)
    assert list(pairs) == [t * K + k for (_, t, k) in triples]
    assert list(np.diff(offsets)) == list(np.bincount([e for e, _, _ in triples],
                                                      minlength=E))


# ---------------------------------------------------------------- experts --

def test_swiglu_expert_closed_form():
    """Eq. (3) on diagonal weights: y_j = SiLU(a_j x_j) * (b_j x_j) * c_j.

    d = I = 2, one expert, K = 1 (weight 1).  Catches: SiLU applied to the up
    projection instead of the gate, a transposed or missing down projection,
    sigmoid instead of SiLU."""
    x = np.array([[1.0, -2.0]], np.float32)
    W1 = np.array([[[1.0, 0.0], [0.0, 0.5]]], np.float32)  # gate: a = (1, 0.5)
    W3 = np.array([[[2.0, 0.0], [0.0, 3.0]]], np.float32)  # up:   b = (2, 3)
    W2 = np.array([[[1.0, 0.0], [0.0, -4.0]]], np.float32)  # down: c = (1, -4)
    idx = np.zeros((1, 1), np.int32)
    w = np.ones((1, 1))
    y = oracle.experts(x, W1, W3, W2, idx, w, "f32")
    silu = lambda v: v / (1.0 + math.exp(-v))  # noqa: E731
    expect = [silu(1.0) * 2.0 * 1.0, silu(-1.0) * (-6.0) * (-4.0)]
    np.testing.assert_allclose(y[0], expect, rtol=1e-15)


def test_expert_matches_numpy_nonsquare():
    """One expert (K = E = 1, weight 1) equals numpy fp64 matmuls with d != I.

    Catches: W1/W3 [E,I,d] or W2 [E,d,I] read transposed, wrong expert stride."""
    x, Wg, _, W1, W3, W2 = _rand_layer(7, 24, 3, 40, RNG)
    for e in range(3):
        idx = np.full((7, 1), e, np.int32)
        y = oracle.experts(x, W1, W3, W2, idx, np.ones((7, 1)), "f32")
        np.testing.assert_allclose(y, _dense_expert(x, W1, W3, W2, e), rtol=1e-12,
                                   atol=1e-12)


def test_dense_special_case_is_softmax_gated_moe():
    """K = E, renorm = 1, W_mask = 0: a dense softmax-gated MoE (einsum).

    Catches: dropped experts, weights applied to the wrong expert, the mask
    dropping candidates at z = 0."""
    T, d, E, I = 11, 16, 5, 20
    x, Wg, _, W1, W3, W2 = _rand_layer(T, d, E, I, RNG)
    Wm = np.zeros((E, d), np.float32)
    y, rt, r, z = oracle.forward(x, Wg, Wm, W1, W3, W2, K=E, renorm=1, dtype="f32")
    xd = x.astype(np.float64)
    gates = softmax(xd @ Wg.astype(np.float64).T, axis=1)  # [T,E]
    a = np.einsum("td,eid->tei", xd, W1.astype(np.float64))
    b = np.einsum("td,eid->tei", xd, W3.astype(np.float64))
    h = _silu(a) * b
    ye = np.einsum("tei,edi->ted", h, W2.astype(np.float64))
    ref = np.einsum("te,ted->td", gates, ye)
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-12)
    assert (rt["idx"] >= 0).all()


def test_zero_mask_router_equals_vanilla_topk():
    """W_mask = 0 gives sigmoid = 0.5 for every expert, so every candidate is
    kept and the layer equals vanilla Top-K MoE exactly (paper, zero init)."""
    T, d, E, I, K = 40, 32, 8, 24, 3
    x, Wg, _, W1, W3, W2 = _rand_layer(T, d, E, I, RNG)
    y0, rt0, _, z0 = oracle.forward(x, Wg, np.zeros((E, d), np.float32), W1, W3, W2, K,
                                    1, "f32")
    yv, rtv, _, _ = oracle.forward(x, Wg, None, W1, W3, W2, K, 1, "f32")
    assert (z0 == 0.0).all()
    assert (rt0["idx"] == rtv["idx"]).all() and (rt0["idx"] == rt0["cand"]).all()
    assert np.array_equal(y0, yv)  # bitwise
    assert rt0["hist"][K] == T


def test_all_masked_token_outputs_zero():
    """Every candidate masked -> the layer outputs exactly 0 (residual bypass)."""
    T, d, E, I, K = 9, 16, 6, 12, 2
    x, Wg, _, W1, W3, W2 = _rand_layer(T, d, E, I, RNG)
    Wm = np.zeros((E, d), np.float32)
    Wm[:, :] = -1.0  # z = -sum(x); make it negative for every token
    x = np.abs(x) + 0.1
    y, rt, _, z = oracle.forward(x, Wg, Wm, W1, W3, W2, K, 1, "f32")
    assert (z < 0).all() and (rt["idx"] == -1).all()
    assert (y == 0.0).all() and rt["hist"][0] == T and rt["counts"].sum() == 0


def test_masked_and_unselected_experts_are_never_read():
    """NaN weights on every expert that has no kept pair leave y finite and
    bitwise unchanged; perturbing a masked candidate's weights changes nothing."""
    T, d, E, I, K = 12, 16, 10, 8, 3
    x, Wg, Wm, W1, W3, W2 = _rand_layer(T, d, E, I, RNG)
    y, rt, _, _ = oracle.forward(x, Wg, Wm, W1, W3, W2, K, 1, "f32")
    unused = rt["counts"] == 0
    assert unused.any() and (rt["idx"] == -1).any()
    A1, A3, A2 = W1.copy(), W3.copy(), W2.copy()
    A1[unused] = np.nan
    A3[unused] = np.nan
    A2[unused] = np.nan
    y2 = oracle.experts(x, A1, A3, A2, rt["idx"], rt["w"], "f32")
    assert np.array_equal(y, y2)
    # A masked candidate of token 0..T-1 whose expert is otherwise unused.
    masked = set(int(rt["cand"][t, k]) for t in range(T) for k in range(K)
                 if rt["idx"][t, k] < 0) - set(np.flatnonzero(rt["counts"]))
    for e in masked:
        B1 = W1.copy()
        B1[e] *= 7.0
        assert np.array_equal(oracle.experts(x, B1, W3, W2, rt["idx"], rt["w"], "f32"), y)


@pytest.mark.parametrize("K,d", [(2, 16), (8, 64)])
def test_brute_force_all_masks(K, d):
    """For one token and every subset S of its K candidates, a mask router
    built to give z = +1 on S and z = -1 elsewhere yields
    y_S = sum_{k in S} g_k E_{c_k}(x) (dense numpy experts), and
    y_S + y_{C-S} = y_C (linearity of Eq. 8 in the mask)."""
    E, I = max(K + 2, 10), 12
    rng = np.random.default_rng(K)
    x, Wg, _, W1, W3, W2 = _rand_layer(1, d, E, I, rng)
    x64 = x.astype(np.float64)
    r, _ = oracle.logits(x, Wg, None, "f32")
    base = oracle.route(r, None, K, renorm=1)
    cand, g = base["cand"][0], base["g"][0]
    ye = {int(e): _dense_expert(x, W1, W3, W2, int(e))[0] for e in cand}
    nx2 = float((x64 ** 2).sum())
    ys = {}
    for bits in itertools.product([0, 1], repeat=K):
        Wm = np.zeros((E, d), np.float64)
        for k, s in enumerate(bits):
            Wm[cand[k]] = (2 * s - 1) * x64[0] / nx2
        Wm32 = Wm.astype(np.float32)
        y, rt, _, z = oracle.forward(x, Wg, Wm32, W1, W3, W2, K, 1, "f32")
        zc = z[0][cand]
        assert ((zc > 0.5) == np.array(bits, bool)).all() and (np.abs(zc) > 0.5).all()
        assert list(rt["idx"][0] >= 0) == [bool(b) for b in bits]
        expect = sum((g[k] * ye[int(cand[k])] for k in range(K) if bits[k]),
                     np.zeros(d))
        np.testing.assert_allclose(y[0], expect, rtol=1e-12, atol=1e-13)
        ys[bits] = y[0]
    full = ys[tuple([1] * K)]
    for bits, y in ys.items():
        comp = tuple(1 - b for b in bits)
        np.testing.assert_allclose(y + ys[comp], full, rtol=1e-12, atol=1e-13)
    assert (ys[tuple([0] * K)] == 0.0).all()


def test_expert_and_token_permutation_equivariance():
    """Relabelling experts (consistently in every weight) leaves y unchanged;
    permuting tokens permutes the rows of y.  Catches an expert id used to
    index one weight but not another, or cross-token leakage."""
    T, d, E, I, K = 23, 16, 7, 12, 3
    x, Wg, Wm, W1, W3, W2 = _rand_layer(T, d, E, I, RNG)
    y, rt, _, _ = oracle.forward(x, Wg, Wm, W1, W3, W2, K, 1, "f32")
    p = RNG.permutation(E)
    yp, rtp, _, _ = oracle.forward(x, Wg[p], Wm[p], W1[p], W3[p], W2[p], K, 1, "f32")
    assert np.array_equal(y, yp)
    inv = np.argsort(p)
    assert (np.where(rtp["idx"] >= 0, p[np.maximum(rtp["idx"], 0)], -1) == rt["idx"]).all()
    assert (inv[rt["cand"]] == rtp["cand"]).all()
    q = RNG.permutation(T)
    yq, _, _, _ = oracle.forward(x[q], Wg, Wm, W1, W3, W2, K, 1, "f32")
    assert np.array_equal(yq, y[q])


def test_figure3_shaped_example_closed_form():
    """The paper's Figure 3 setting (4 experts, K = 3) worked by hand.

    Logits r = (2, 0, 1, 0.5)*ln 2 -> candidates (0, 2, 3); softmax over the
    Top-K is (4, 2, 1.414...)/(7.414...).  Mask pre-activations (+1, *, -1, +2)
    keep experts 0 and 3.  Experts are diagonal (d = I = 2) with
    E_e(x)_j = SiLU(x_j) * x_j * s_e, s = (1, 10, 100, 1000)."""
    ln2 = math.log(2.0)
    # Use d = 3 with a bias-like third feature to place the logits exactly.
    d, E = 3, 4
    xv = np.array([[0.5, -1.5, 1.0]], np.float32)
    Wg = np.zeros((E, d), np.float32)
    Wg[:, 2] = np.array([2.0, 0.0, 1.0, 0.5], np.float32) * np.float32(ln2)
    Wm = np.zeros((E, d), np.float32)
    Wm[:, 2] = [1.0, 5.0, -1.0, 2.0]
    I = 3
    W1 = np.zeros((E, I, d), np.float32)
    W3 = np.zeros((E, I, d), np.float32)
    W2 = np.zeros((E, d, I), np.float32)
    s = [1.0, 10.0, 100.0, 1000.0]
    for e in range(E):
        for j in range(2):
            W1[e, j, j] = 1.0
            W3[e, j, j] = 1.0
            W2[e, j, j] = s[e]
    y, rt, r, z = oracle.forward(xv, Wg, Wm, W1, W3, W2, K=3, renorm=1, dtype="f32")
    assert list(rt["cand"][0]) == [0, 2, 3]
    assert list(rt["idx"][0]) == [0, -1, 3]
    r32 = np.float32(ln2)
    ex = [math.exp(float(np.float32(2.0) * r32) - float(np.float32(2.0) * r32)),
          math.exp(float(np.float32(1.0) * r32) - float(np.float32(2.0) * r32)),
          math.exp(float(np.float32(0.5) * r32) - float(np.float32(2.0) * r32))]
    g = [v / sum(ex) for v in ex]
    silu = lambda v: v / (1.0 + math.exp(-v))  # noqa: E731
    feat = [silu(0.5) * 0.5, silu(-1.5) * (-1.5), 0.0]
    expect = [(g[0] * s[0] + g[2] * s[3]) * f for f in feat]
    np.testing.assert_allclose(y[0], expect, rtol=1e-12)


@pytest.mark.parametrize("tau", [0.1, 0.3, 0.5, 0.7, 0.9])
def test_threshold_ablation_matches_sigmoid(tau):
    """The threshold ablation (news article §8: tau in 0.1 .. 0.9): a candidate
    is kept iff sigmoid(z) >= tau.  The oracle takes tau as its logit; checked
    against scipy's expit away from the boundary, and kept fractions fall as tau
    rises.  Catches a threshold applied to g instead of z, or the wrong side."""
    T, E, K = 400, 16, 4
    r = RNG.standard_normal((T, E))
    z = RNG.standard_normal((T, E)) * 3.0
    tl = math.log(tau / (1.0 - tau))
    out = oracle.route(r, z, K, renorm=1, tau_logit=tl)
    zc = np.take_along_axis(z, out["cand"], axis=1)
    sig = expit(zc)
    clear = np.abs(sig - tau) > 1e-9
    assert ((out["idx"] >= 0) == (sig >= tau))[clear].all()
    lo = oracle.route(r, z, K, renorm=1, tau_logit=math.log(0.05 / 0.95))
    hi = oracle.route(r, z, K, renorm=1, tau_logit=math.log(0.95 / 0.05))
    assert (lo["idx"] >= 0).sum() >= (out["idx"] >= 0).sum() >= (hi["idx"] >= 0).sum()
    if tau == 0.5:
        assert np.array_equal(out["idx"], oracle.route(r, z, K, renorm=1)["idx"])


def test_shared_experts_run_for_every_token_with_weight_one():
    """Shared experts (news article §5): always on, all-masked tokens
    included.  With every candidate masked the layer output is exactly the sum
    of the shared experts (numpy fp64); with a mask the shared part is the same
    whatever the routed part is.  Catches shared experts skipped for
    all-masked tokens, or scaled by a router weight."""
    T, d, E, I, K, S, Is = 9, 16, 6, 12, 2, 3, 20
    x, Wg, _, W1, W3, W2 = _rand_layer(T, d, E, I, RNG)
    W1s = (RNG.standard_normal((S, Is, d)) / math.sqrt(d)).astype(np.float32)
    W3s = (RNG.standard_normal((S, Is, d)) / math.sqrt(d)).astype(np.float32)
    W2s = (RNG.standard_normal((S, d, Is)) / math.sqrt(Is)).astype(np.float32)
    x = np.abs(x) + 0.1
    Wm_all = -np.ones((E, d), np.float32)  # z = -sum(x) < 0: every candidate masked
    y, rt, _, _ = oracle.forward(x, Wg, Wm_all, W1, W3, W2, K, 1, "f32",
                                 shared=(W1s, W3s, W2s))
    assert (rt["idx"] == -1).all()
    ref = sum(_dense_expert(x, W1s, W3s, W2s, s) for s in range(S))
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-13)
    # routed + shared = routed alone + shared alone, for a partly kept mask
    Wm = (RNG.standard_normal((E, d)) / math.sqrt(d)).astype(np.float32)
    yr, rt2, _, _ = oracle.forward(x, Wg, Wm, W1, W3, W2, K, 1, "f32")
    ys, _, _, _ = oracle.forward(x, Wg, Wm, W1, W3, W2, K, 1, "f32", shared=(W1s, W3s, W2s))
    assert 0 < (rt2["idx"] >= 0).sum() < T * K
    np.testing.assert_allclose(ys - yr, ref, rtol=1e-11, atol=1e-12)


# ------------------------------------------------------ bf16 storage decode --

def _bf16_patterns_finite():
    """Every finite bfloat16 bit pattern (exponent field not all ones), as int16."""
    u = np.arange(1 << 16, dtype=np.uint32)
    finite = ((u >> 7) & 0xFF) != 0xFF
    return u[finite].astype(np.uint16).view(np.int16)


def _torch_bf16_to_f64(bits):
    """Independent decode: torch's own bfloat16 -> float64 conversion."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def test_oracle_bf16_decode_of_every_finite_pattern():
    """The oracle widens bf16 storage (raw bits) to fp64 exactly as torch does,
    for every finite pattern, through both operands of its logits: a one-hot
    weight row picks one input element (x_tj * 1 + zeros is exact), and a
    one-hot input row picks one weight element.

    Catches: a wrong shift, byte order or sign handling in the decode, a
    flushed subnormal, or the two operands decoded differently."""
    pats = _bf16_patterns_finite()
    d = 256
    n = -(-len(pats) // d) * d
    flat = np.zeros(n, np.int16)
    flat[:len(pats)] = pats
    X = flat.reshape(-1, d)
    one = np.int16(0x3F80)  # bf16 1.0
    eye = np.zeros((d, d), np.int16)
    eye[np.arange(d), np.arange(d)] = one
    want = _torch_bf16_to_f64(X)
    r, _ = oracle.logits(X, eye, None, "bf16")   # r[t, e] = X[t, e]
    assert np.array_equal(r, want + 0.0)         # -0.0 sums to +0.0: compare values
    r2, _ = oracle.logits(eye, X, None, "bf16")  # r2[t, e] = X[e, t]
    assert np.array_equal(r2, (want + 0.0).T)


def test_oracle_bf16_layer_matches_numpy_on_torch_decode():
    """Logits and the expert sum on bf16 storage equal numpy fp64 arithmetic on
    torch's decode of the same bits: the logits bit for bit (sequential sums
    of exact products, written as a cumulative sum in the same order), the
    SwiGLU experts to 1e-12.

    Catches: the bf16 path reading a wrong stride or operand, or mixing the
    decode of x and of the weights."""
    import torch
    rng = np.random.default_rng(7)
    T, d, E, I, K = 9, 64, 6, 48, 3
    def b16(a):
        return torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).view(
            torch.int16).numpy()
    x = b16(rng.standard_normal((T, d)))
    Wg = b16(rng.standard_normal((E, d)) / 8)
    Wm = b16(rng.standard_normal((E, d)) / 8)
    W1 = b16(rng.standard_normal((E, I, d)) / 8)
    W3 = b16(rng.standard_normal((E, I, d)) / 8)
    W2 = b16(rng.standard_normal((E, d, I)) / 7)
    xf, Wgf, Wmf = (_torch_bf16_to_f64(a) for a in (x, Wg, Wm))
    r, z = oracle.logits(x, Wg, Wm, "bf16")
    r_np = np.cumsum(xf[:, None, :] * Wgf[None, :, :], axis=2)[..., -1]
    z_np = np.cumsum(xf[:, None, :] * Wmf[None, :, :], axis=2)[..., -1]
    assert np.array_equal(r, r_np) and np.array_equal(z, z_np)
    rt = oracle.route(r, z, K, renorm=1)
    y = oracle.experts(x, W1, W3, W2, rt["idx"], rt["w"], "bf16")
    W1f, W3f, W2f = (_torch_bf16_to_f64(a) for a in (W1, W3, W2))
    want = np.zeros((T, d))
    for t in range(T):
        for k in range(K):
            e = rt["idx"][t, k]
            if e < 0:
                continue
            a = W1f[e] @ xf[t]
            b = W3f[e] @ xf[t]
            want[t] += rt["w"][t, k] * (W2f[e] @ (_silu(a) * b))
    np.testing.assert_allclose(y, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_minus_inf_gate_logits_weigh_zero():
    """Eq. (1) writes -inf for the experts outside the Top-K, i.e. a -inf logit
    has weight 0.  A row with some -inf logits: the finite ones follow
    scipy's softmax as if the -inf entries were absent.  A row whose every
    logit is -inf has no defined softmax (0/0): its weights are 0 (reading).
    NaN and +inf are still rejected.

    Catches: inf - inf reaching the weights, a NaN weight spreading into y."""
    E, K = 6, 3
    r = np.array([[1.0, -np.inf, 0.5, -np.inf, 2.0, -1.0],
                  [-np.inf] * E,
                  [0.3, 0.1, -0.2, 0.4, -np.inf, 0.0]])
    for renorm in (0, 1):
        out = oracle.route(r, None, K, renorm)
        assert np.isfinite(out["w"]).all()
        assert (out["w"][1] == 0).all() and list(out["cand"][1]) == [0, 1, 2]
        for t in (0, 2):
            fin = np.isfinite(r[t])
            cand = out["cand"][t]
            if renorm:
                ref = softmax(r[t][cand])
            else:
                full = np.zeros(E)
                full[fin] = softmax(r[t][fin])
                ref = full[cand]
            np.testing.assert_allclose(out["w"][t], ref, rtol=1e-15, atol=0)
    for bad in (np.nan, np.inf):
        rb = r.copy()
        rb[0, 0] = bad
        with pytest.raises(FloatingPointError):
            oracle.route(rb, None, K, 1)
