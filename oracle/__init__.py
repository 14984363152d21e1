"""fp64 CPU oracle of the BEAM-masked MoE layer forward pass.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow definition that the
CUDA library is checked against.  Only ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import it.  It shares no code with
the CUDA library and never calls into it; the product path never calls it.

The arithmetic lives in ``beam_oracle.c`` (plain C, fp64, OpenMP over tokens),
following "BEAM: Binary Expert Activation Masking for Dynamic Routing in MoE"
(arXiv 2605.14438), §3.1 Eq. (1)-(3) and §3.2 Eq. (4)-(8).  This module only
builds that file and marshals numpy arrays into it.

Storage dtypes: ``"bf16"`` arrays are passed as their raw 16-bit patterns
(numpy ``uint16``/``int16``), ``"f32"`` arrays as ``float32``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "beam_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

BF16 = 0
F32 = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile beam_oracle.c into liboracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall",
               "-o", _LIB_PATH, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        p = ctypes.c_void_p
        i = ctypes.c_int
        lib.oracle_logits.argtypes = [i, i, i, i, p, p, p, p, p]
        d = ctypes.c_double
        lib.oracle_route.argtypes = [i, i, i, i, d, p, p, p, p, p, p, p, p]
        lib.oracle_route_f32.argtypes = [i, i, i, i, d, p, p, p, p, p, p, p, p]
        lib.oracle_permutation.argtypes = [i, i, i, p, p, p]
        lib.oracle_experts.argtypes = [i, i, i, i, i, i, p, p, p, p, p, p, i, i, p, i]
        lib.oracle_max_threads.argtypes = []
        lib.oracle_shared_experts.argtypes = [i, i, i, i, i, p, p, p, p, i, i, p, i]
        lib.oracle_backward.argtypes = [i, i, i, i, i, i, i, d, d, i, p, p, p, p, p, p, p, i, p,
                                        p, p, p, p, p, p, p, p, p, p, i]
        for f in (lib.oracle_logits, lib.oracle_route, lib.oracle_route_f32,
                  lib.oracle_permutation, lib.oracle_experts, lib.oracle_max_threads,
                  lib.oracle_shared_experts, lib.oracle_backward):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _storage(a, dtype):
    """Contiguous array in the oracle's storage format for ``dtype``."""
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if dtype == "bf16":
        if a.dtype not in (np.uint16, np.int16):
            raise TypeError("bf16 arrays must be passed as raw 16-bit patterns")
        return a
    if dtype == "f32":
        return np.ascontiguousarray(a, dtype=np.float32)
    raise ValueError(dtype)


def _code(dtype):
    return BF16 if dtype == "bf16" else F32


def _check(rc, what):
    if rc == -2:
        raise FloatingPointError(f"oracle {what}: non-finite value in the data it used")
    if rc != 0:
        raise ValueError(f"oracle {what}: bad argument (rc={rc})")


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def logits(x, W_gate, W_mask, dtype):
    """r = x W_gate^T and z = x W_mask^T in fp64 (z is None without a mask)."""
    lib = _load()
    x, Wg, Wm = _storage(x, dtype), _storage(W_gate, dtype), _storage(W_mask, dtype)
    T, d = x.shape
    E = Wg.shape[0]
    r = np.empty((T, E), np.float64)
    z = np.empty((T, E), np.float64) if Wm is not None else None
    _check(lib.oracle_logits(T, d, E, _code(dtype), _ptr(x), _ptr(Wg), _ptr(Wm),
                             _ptr(r), _ptr(z)), "logits")
    return r, z


def route(r, z, K, renorm, tau_logit=0.0):
    """Top-K, softmax, binary mask and aggregation from given logits.

    ``r``/``z`` may be float64 (oracle logits) or float32 (another
    implementation's exported logits, widened exactly).  ``tau_logit`` is the
    mask threshold tau of Eq. (6) as its logit (0 = tau 0.5): a candidate is
    kept iff sigmoid(z) >= tau, i.e. z >= tau_logit.  Returns a dict with
    cand, g, idx, w, counts, hist.
    """
    lib = _load()
    T, E = r.shape
    out = dict(
        cand=np.empty((T, K), np.int32), g=np.empty((T, K), np.float64),
        idx=np.empty((T, K), np.int32), w=np.empty((T, K), np.float64),
        counts=np.empty((E,), np.int32), hist=np.empty((K + 1,), np.int32),
    )
    if r.dtype == np.float32:
        r = np.ascontiguousarray(r)
        z = None if z is None else np.ascontiguousarray(z, dtype=np.float32)
        fn = lib.oracle_route_f32
    else:
        r = np.ascontiguousarray(r, dtype=np.float64)
        z = None if z is None else np.ascontiguousarray(z, dtype=np.float64)
        fn = lib.oracle_route
    _check(fn(T, E, K, int(renorm), float(tau_logit), _ptr(r), _ptr(z), _ptr(out["cand"]),
              _ptr(out["g"]),
              _ptr(out["idx"]), _ptr(out["w"]), _ptr(out["counts"]), _ptr(out["hist"])),
           "route")
    return out


def permutation(idx, E):
    """Kept pairs grouped by expert (ascending), then token; entries t*K + k."""
    lib = _load()
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, K = idx.shape
    offsets = np.empty((E + 1,), np.int32)
    pairs = np.empty((max(T * K, 1),), np.int32)
    _check(lib.oracle_permutation(T, K, E, _ptr(idx), _ptr(offsets), _ptr(pairs)),
           "permutation")
    return offsets, pairs[: offsets[E]].copy()


def experts(x, W1, W3, W2, idx, w, dtype, t_begin=0, t_end=None, nthreads=0):
    """y[t] = sum_k w[t,k] * SwiGLU expert idx[t,k] applied to x[t], fp64."""
    lib = _load()
    x = _storage(x, dtype)
    W1, W3, W2 = _storage(W1, dtype), _storage(W3, dtype), _storage(W2, dtype)
    T, d = x.shape
    E, I, d1 = W1.shape
    if d1 != d or W3.shape != W1.shape or W2.shape != (E, d, I):
        raise ValueError("weight shapes must be W1,W3 [E,I,d] and W2 [E,d,I]")
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float64)
    K = idx.shape[1]
    if t_end is None:
        t_end = T
    y = np.empty((t_end - t_begin, d), np.float64)
    _check(lib.oracle_experts(T, d, E, I, K, _code(dtype), _ptr(x), _ptr(W1), _ptr(W3),
                              _ptr(W2), _ptr(idx), _ptr(w), t_begin, t_end, _ptr(y),
                              int(nthreads)), "experts")
    return y


def add_shared(y, x, W1s, W3s, W2s, dtype, t_begin=0, t_end=None, nthreads=0):
    """y[t - t_begin] += sum_s SwiGLU shared expert s applied to x[t] (weight 1)."""
    lib = _load()
    x = _storage(x, dtype)
    W1s, W3s, W2s = _storage(W1s, dtype), _storage(W3s, dtype), _storage(W2s, dtype)
    T, d = x.shape
    S, Is, d1 = W1s.shape
    if d1 != d or W3s.shape != W1s.shape or W2s.shape != (S, d, Is):
        raise ValueError("shared weights must be W1s,W3s [S,Is,d] and W2s [S,d,Is]")
    if t_end is None:
        t_end = T
    if y.shape != (t_end - t_begin, d) or y.dtype != np.float64 or not y.flags.c_contiguous:
        raise ValueError("y must be a contiguous float64 [t_end - t_begin, d] array")
    _check(lib.oracle_shared_experts(T, d, S, Is, _code(dtype), _ptr(x), _ptr(W1s), _ptr(W3s),
                                     _ptr(W2s), t_begin, t_end, _ptr(y), int(nthreads)),
           "shared experts")
    return y


def backward(x, W_gate, W_mask, W1, W3, W2, dy, K, renorm, dtype, beta=0.0, tau_logit=0.0,
             ste=True, experts=None, logits=None, nthreads=0):
    """Training-mode gradients of L = sum <dy, y> + beta * sum of the candidates'
    sigmoid(z), with the straight-through estimator (ste=False drops its term).
    `experts`: ids whose weight gradients are returned (None: all, in order).
    `logits`: [T, 2E] (r then z) to route with, e.g. another implementation's
    fp32 logits (widened exactly); None computes them.
    Returns a dict of fp64 arrays: dx, dW_gate, dW_mask (None without a mask),
    dW1, dW3 [n_sel, I, d], dW2 [n_sel, d, I], u and dz [T, K]."""
    lib = _load()
    x, dy = _storage(x, dtype), _storage(dy, dtype)
    Wg, Wm = _storage(W_gate, dtype), _storage(W_mask, dtype)
    W1, W3, W2 = _storage(W1, dtype), _storage(W3, dtype), _storage(W2, dtype)
    T, d = x.shape
    E, I, _ = W1.shape
    sel = None if experts is None else np.ascontiguousarray(experts, dtype=np.int32)
    r_in = z_in = None
    if logits is not None:
        lg = np.asarray(logits, dtype=np.float64)
        r_in = np.ascontiguousarray(lg[:, :E])
        z_in = np.ascontiguousarray(lg[:, E:2 * E]) if Wm is not None else None
    n_sel = E if sel is None else len(sel)
    out = dict(dx=np.empty((T, d)), dW_gate=np.empty((E, d)),
               dW_mask=np.zeros((E, d)) if Wm is not None else None,
               dW1=np.empty((n_sel, I, d)), dW3=np.empty((n_sel, I, d)),
               dW2=np.empty((n_sel, d, I)), u=np.empty((T, K)), dz=np.empty((T, K)))
    _check(lib.oracle_backward(T, d, E, I, K, int(renorm), _code(dtype), float(tau_logit),
                               float(beta), int(bool(ste)), _ptr(x), _ptr(Wg), _ptr(Wm),
                               _ptr(W1), _ptr(W3), _ptr(W2), _ptr(dy), n_sel, _ptr(sel),
                               _ptr(r_in), _ptr(z_in), _ptr(out["dx"]), _ptr(out["dW_gate"]), _ptr(out["dW_mask"]),
                               _ptr(out["dW1"]), _ptr(out["dW3"]), _ptr(out["dW2"]),
                               _ptr(out["u"]), _ptr(out["dz"]), int(nthreads)), "backward")
    return out


def forward(x, W_gate, W_mask, W1, W3, W2, K, renorm, dtype, nthreads=0, tau_logit=0.0,
            shared=None):
    """The whole layer: logits, routing, mask, experts (+ shared experts given as
    (W1s, W3s, W2s)).  Returns (y, route dict, r, z)."""
    r, z = logits(x, W_gate, W_mask, dtype)
    rt = route(r, z, K, renorm, tau_logit)
    y = experts(x, W1, W3, W2, rt["idx"], rt["w"], dtype, nthreads=nthreads)
    if shared is not None:
        add_shared(y, x, *shared, dtype, nthreads=nthreads)
    return y, rt, r, z
