"""Pins of the fp64 backward oracle (training mode of the BEAM layer).

The news article on BEAM (§4) trains the mask router through a
straight-through estimator and adds a penalty on the candidates' mask scores;
neither is printed as a formula.  The oracle's readings are stated in
oracle/beam_oracle.h.  They are pinned here against things other than
themselves:

* central finite differences of the (separately pinned) forward oracle, for
  every gradient the objective has with the candidates and the mask held
  fixed (ste=False);
* the straight-through term of the mask gradient, against finite differences
  of a soft-mask forward (candidate weights g * sigmoid(z)) built from the
  forward oracle's routing and expert routines: the derivative of that forward
  in W_mask is exactly the term the estimator passes through the threshold;
* closed forms: dy = 0 (only the penalty acts), W_mask = 0 (every sigmoid is
  1/2, so its derivative is 1/4), and an expert that is only ever a masked
  candidate (no weight gradient, but a mask gradient).

Inputs are float32 so that the oracle evaluates every perturbed point
exactly in fp64; each finite-difference step is the exact difference of the
two float32 points.
"""
import numpy as np
import pytest
from scipy.special import expit

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _layer(seed, T=4, d=8, E=5, I=6):
    rng = np.random.default_rng(seed)

    def f(*s, sc=1.0):
        return (rng.standard_normal(s) * sc).astype(np.float32)

    return dict(x=f(T, d), Wg=f(E, d, sc=0.6), Wm=f(E, d, sc=0.6), W1=f(E, I, d, sc=0.4),
                W3=f(E, I, d, sc=0.4), W2=f(E, d, I, sc=0.4), dy=f(T, d))


def _routing(L, K, renorm):
    r, z = oracle.logits(L["x"], L["Wg"], L["Wm"], "f32")
    rt = oracle.route(r, z, K, renorm)
    return r, z, rt


def _objective(L, K, renorm, beta):
    """sum <dy, y> + beta * sum of the candidates' sigmoid(z), and the routing."""
    y, rt, r, z = oracle.forward(L["x"], L["Wg"], L["Wm"], L["W1"], L["W3"], L["W2"], K,
                                 renorm, "f32")
    T = z.shape[0]
    pen = sum(expit(z[t, c]) for t in range(T) for c in rt["cand"][t])
    return float(np.sum(L["dy"].astype(np.float64) * y) + beta * pen), rt


def _fd(L, name, fn, max_entries=None, seed=0):
    """Central differences of fn(L) in every (or a sample of) entry of L[name].
    Entries whose perturbation changes the routing are skipped and counted."""
    A = L[name]
    flat = A.reshape(-1)
    ids = np.arange(flat.size)
    if max_entries is not None and flat.size > max_entries:
        ids = np.random.default_rng(seed).choice(flat.size, max_entries, replace=False)
    grads, skipped = {}, 0
    base_rt = fn(L)[1]
    for i in ids:
        v = flat[i]
        step = np.float32(1e-3) * max(np.float32(1.0), abs(v))
        hi, lo = np.float32(v + step), np.float32(v - step)
        flat[i] = hi
        fh, rh = fn(L)
        flat[i] = lo
        fl, rl = fn(L)
        flat[i] = v
        same = all(np.array_equal(rh[k], base_rt[k]) and np.array_equal(rl[k], base_rt[k])
                   for k in ("cand", "idx"))
        if not same:
            skipped += 1
            continue
        grads[int(i)] = (fh - fl) / (float(hi) - float(lo))
    return grads, skipped


def _check(fd, analytic, rtol=2e-5, atol=2e-6):
    a = analytic.reshape(-1)
    scale = max(1.0, float(np.max(np.abs(a))))
    for i, g in fd.items():
        assert abs(a[i] - g) <= atol * scale + rtol * abs(g), (i, a[i], g)


@pytest.mark.parametrize("renorm", [1, 0])
def test_backward_matches_finite_differences_with_mask_fixed(renorm):
    K, beta = 2, 0.3
    L = _layer(1)
    b = oracle.backward(L["x"], L["Wg"], L["Wm"], L["W1"], L["W3"], L["W2"], L["dy"], K,
                        renorm, "f32", beta=beta, ste=False)
    fn = lambda LL: _objective(LL, K, renorm, beta)  # noqa: E731
    total_skipped = 0
    for name, key in (("x", "dx"), ("Wg", "dW_gate"), ("Wm", "dW_mask"), ("W1", "dW1"),
                      ("W3", "dW3"), ("W2", "dW2")):
        fd, skipped = _fd(L, name, fn, max_entries=120)
        total_skipped += skipped
        assert len(fd) > 0
        _check(fd, b[key])
    assert total_skipped <= 3


def test_straight_through_term_is_the_soft_mask_gradient():
    """d/dW_mask of sum <dy, sum_k g_k sigmoid(z_k) E_k(x)> (candidates and g
    from the main router only) equals the estimator's mask gradient at beta=0."""
    K, renorm = 2, 1
    L = _layer(2)

    def soft(LL):
        r, z, rt = _routing(LL, K, renorm)
        T = z.shape[0]
        cand = rt["cand"]
        w = rt["g"] * expit(np.take_along_axis(z, cand.astype(np.int64), axis=1))
        y = oracle.experts(LL["x"], LL["W1"], LL["W3"], LL["W2"], cand, w, "f32")
        return float(np.sum(LL["dy"].astype(np.float64) * y)), rt

    b = oracle.backward(L["x"], L["Wg"], L["Wm"], L["W1"], L["W3"], L["W2"], L["dy"], K,
                        renorm, "f32", beta=0.0, ste=True)
    fd, skipped = _fd(L, "Wm", soft)
    assert skipped == 0
    _check(fd, b["dW_mask"])
    # and without the estimator the mask gets no gradient at beta = 0
    b0 = oracle.backward(L["x"], L["Wg"], L["Wm"], L["W1"], L["W3"], L["W2"], L["dy"], K,
                         renorm, "f32", beta=0.0, ste=False)
    assert np.all(b0["dW_mask"] == 0.0) and np.all(b0["dz"] == 0.0)


def test_u_is_the_dot_of_dy_with_each_candidates_expert_output():
    K, renorm = 3, 1
    L = _layer(3)
    r, z, rt = _routing(L, K, renorm)
    b = oracle.backward(L["x"], L["Wg"], L["Wm"], L["W1"], L["W3"], L["W2"], L["dy"], K,
                        renorm, "f32", beta=0.0)
    for k in range(K):
        w = np.zeros(rt["g"].shape)
        w[:, k] = 1.0
        y = oracle.experts(L["x"], L["W1"], L["W3"], L["W2"], rt["cand"], w, "f32")
        u = np.sum(L["dy"].astype(np.float64) * y, axis=1)
        np.testing.assert_allclose(b["u"][:, k], u, rtol=1e-12, atol=1e-12)


def test_zero_upstream_gradient_leaves_only_the_penalty():
    K, renorm, beta = 2, 1, 0.7
    L = _layer(4)
    L["dy"][:] = 0
    r, z, rt = _routing(L, K, renorm)
    b = oracle.backward(L["x"], L["Wg"], L["Wm"], L["W1"], L["W3"], L["W2"], L["dy"], K,
                        renorm, "f32", beta=beta)
    zc = np.take_along_axis(z, rt["cand"].astype(np.int64), axis=1)
    s = expit(zc)
    np.testing.assert_allclose(b["dz"], beta * s * (1 - s), rtol=1e-12)
    assert np.all(b["dW1"] == 0) and np.all(b["dW3"] == 0) and np.all(b["dW2"] == 0)
    assert np.all(b["dW_gate"] == 0)
    x = L["x"].astype(np.float64)
    Wm = L["Wm"].astype(np.float64)
    dx = np.einsum("tk,tkj->tj", b["dz"], Wm[rt["cand"]])
    np.testing.assert_allclose(b["dx"], dx, rtol=1e-12, atol=1e-14)
    dWm = np.zeros_like(Wm)
    for t in range(x.shape[0]):
        for k in range(K):
            dWm[rt["cand"][t, k]] += b["dz"][t, k] * x[t]
    np.testing.assert_allclose(b["dW_mask"], dWm, rtol=1e-12, atol=1e-14)


def test_zero_mask_router_has_sigmoid_slope_one_quarter():
    K, renorm, beta = 2, 0, 0.2
    L = _layer(5)
    L["Wm"][:] = 0
    r, z, rt = _routing(L, K, renorm)
    assert (rt["idx"] >= 0).all()  # W_mask = 0 keeps every candidate
    b = oracle.backward(L["x"], L["Wg"], L["Wm"], L["W1"], L["W3"], L["W2"], L["dy"], K,
                        renorm, "f32", beta=beta)
    np.testing.assert_allclose(b["dz"], (rt["g"] * b["u"] + beta) * 0.25, rtol=1e-12,
                               atol=1e-15)


def test_expert_that_is_only_masked_gets_no_weight_gradient():
    K, renorm = 2, 1
    L = _layer(6)
    L["x"][:, -1] = 1.0  # bias feature
    e = 2
    L["Wg"][e, -1] = 20.0  # a candidate of every token
    L["Wm"][e, -1] = -50.0  # masked for every token
    r, z, rt = _routing(L, K, renorm)
    assert (rt["cand"] == e).any(axis=1).all() and not (rt["idx"] == e).any()
    b = oracle.backward(L["x"], L["Wg"], L["Wm"], L["W1"], L["W3"], L["W2"], L["dy"], K,
                        renorm, "f32", beta=0.0, experts=[e, (e + 1) % 5])
    assert np.all(b["dW1"][0] == 0) and np.all(b["dW3"][0] == 0) and np.all(b["dW2"][0] == 0)
    # the straight-through estimator still reaches its mask row (tiny but exact)
    k = np.argmax(rt["cand"] == e, axis=1)
    s = expit(z[:, e])
    expect = (rt["g"][np.arange(len(k)), k] * b["u"][np.arange(len(k)), k] * s * (1 - s))
    np.testing.assert_allclose(b["dz"][np.arange(len(k)), k], expect, rtol=1e-12, atol=0)


def test_mask_disabled_has_no_mask_gradient_and_no_estimator_term():
    K, renorm = 2, 1
    L = _layer(7)
    args = (L["x"], L["Wg"], None, L["W1"], L["W3"], L["W2"], L["dy"], K, renorm, "f32")
    b1 = oracle.backward(*args, beta=0.5, ste=True)
    b0 = oracle.backward(*args, beta=0.5, ste=False)
    assert b1["dW_mask"] is None and np.all(b1["dz"] == 0)
    for k in ("dx", "dW_gate", "dW1", "dW3", "dW2"):
        assert np.array_equal(b1[k], b0[k])
