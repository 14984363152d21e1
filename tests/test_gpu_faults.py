"""Failure detection and out-of-bounds writes, on the GPU, without faulting it.

* Bounded waits: the library's test switch (beam_moe_set_fault_injection)
  makes CTA 0 of one launch skip a shared-memory stage, so that its MMA
  issuer's bounded wait on that stage can only expire.  The call must come back
  with BEAM_ERR_TIMEOUT from beam_moe_check, with a short wait limit, and the
  next normal call on the same workspace must be clean and bitwise equal to a
  call on a fresh workspace.  Nothing traps, asserts on the device or spins
  without a bound: every wait in the kernels gives up after the limit.
* Guard bands (the stand-in for a memory checker): every output buffer and the
  workspace sit between canary words; route, forward, forward with shared
  experts and backward on ragged shapes must leave every canary unchanged.
"""
import numpy as np
import pytest
import torch

from dynamic_expert_routing_router_b200 import abi, inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def one_launch_up_to_16_tokens():
    """Every batch of at most 16 tokens takes the one-launch path here (the
    library's default stops at 4)."""
    prev = abi.set_one_launch_tokens(16)
    yield
    abi.set_one_launch_tokens(prev)

DEV = "cuda"
WAIT_LIMIT_NS = 50_000_000  # 50 ms instead of 1 s per bounded wait


class fault:
    """Context manager: fault injection on, always switched off again."""

    def __init__(self, mode):
        self.mode = mode

    def __enter__(self):
        abi.set_fault_injection(self.mode, WAIT_LIMIT_NS)

    def __exit__(self, *exc):
        torch.cuda.synchronize()
        abi.set_fault_injection(abi.FAULT_NONE, 0)


def _layer(sh, T, f, seed=0):
    x = inputs.make_tokens(sh, T, seed=seed + 1, device=DEV)
    Wg = inputs.make_gate(sh, seed=seed, device=DEV)
    Wm = inputs.make_mask(sh, f, seed=seed, device=DEV)
    W1, W3, W2 = inputs.make_experts(sh, seed=seed, device=DEV)
    return x, Wg, Wm, W1, W3, W2


@pytest.mark.parametrize("T", [4, 32, 2048],
                         ids=["decode_one_launch", "decode_fused_experts", "prefill_gate_up_gemm"])
def test_expert_wait_timeout_is_reported_then_recovers(T):
    sh = inputs.QWEN3
    x, Wg, Wm, W1, W3, W2 = _layer(sh, T, 0.35)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    ws = abi.alloc_workspace(dsc, DEV)
    out = torch.empty((T, sh.d), dtype=torch.bfloat16, device=DEV)
    with fault(abi.FAULT_EXPERT_STAGE):
        abi.forward(dsc, x, Wg, Wm, W1, W3, W2, out, ws)
        with pytest.raises(abi.BeamError) as ei:
            abi.check(dsc, ws)
    assert ei.value.status == 5  # BEAM_ERR_TIMEOUT
    # the same workspace, no fault: clean, and equal to a fresh workspace's result
    abi.forward(dsc, x, Wg, Wm, W1, W3, W2, out, ws)
    abi.check(dsc, ws)
    ref = torch.empty_like(out)
    ws2 = abi.alloc_workspace(dsc, DEV)
    abi.forward(dsc, x, Wg, Wm, W1, W3, W2, ref, ws2)
    abi.check(dsc, ws2)
    assert torch.equal(out, ref)


def test_router_wait_timeout_reaches_the_error_word_then_recovers():
    """A router CTA's expiry is carried to the error word by the top-K kernel."""
    sh = inputs.QWEN3
    T = 16
    x, Wg, Wm, W1, W3, W2 = _layer(sh, T, 0.35, seed=2)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    ws = abi.alloc_workspace(dsc, DEV)
    out = torch.empty((T, sh.d), dtype=torch.bfloat16, device=DEV)
    for call in ("forward", "route"):
        with fault(abi.FAULT_ROUTER_STAGE):
            if call == "forward":
                abi.forward(dsc, x, Wg, Wm, W1, W3, W2, out, ws)
            else:
                idx = torch.empty((T, sh.K), dtype=torch.int32, device=DEV)
                w = torch.empty((T, sh.K), dtype=torch.float32, device=DEV)
                cnt = torch.empty((sh.E,), dtype=torch.int32, device=DEV)
                abi.route(dsc, x, Wg, Wm, idx, w, cnt, workspace=ws)
            with pytest.raises(abi.BeamError) as ei:
                abi.check(dsc, ws)
        assert ei.value.status == 5, call
        abi.forward(dsc, x, Wg, Wm, W1, W3, W2, out, ws)
        abi.check(dsc, ws)  # the next call starts clean


def test_shared_expert_wait_timeout_reaches_the_error_word_then_recovers():
    """The shared experts' GEMMs run on a second stream beside the router and
    top-K; their expiry goes through a tagged header word that the combine
    folds into the error word."""
    sh, S, T = inputs.DSV2_LITE, inputs.DSV2_LITE_SHARED, 40
    x, Wg, Wm, W1, W3, W2 = _layer(sh, T, 0.35, seed=4)
    W1s, W3s, W2s = inputs.make_shared_experts(sh, S, seed=4, device=DEV)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm, n_shared=S, I_shared=sh.I)
    ws = abi.alloc_workspace(dsc, DEV)
    out = torch.empty((T, sh.d), dtype=torch.bfloat16, device=DEV)
    with fault(abi.FAULT_SHARED_STAGE):
        abi.forward_shared(dsc, x, Wg, Wm, W1, W3, W2, W1s, W3s, W2s, out, ws)
        with pytest.raises(abi.BeamError) as ei:
            abi.check(dsc, ws)
    assert ei.value.status == 5  # BEAM_ERR_TIMEOUT
    abi.forward_shared(dsc, x, Wg, Wm, W1, W3, W2, W1s, W3s, W2s, out, ws)
    abi.check(dsc, ws)
    ref = torch.empty_like(out)
    ws2 = abi.alloc_workspace(dsc, DEV)
    abi.forward_shared(dsc, x, Wg, Wm, W1, W3, W2, W1s, W3s, W2s, ref, ws2)
    abi.check(dsc, ws2)
    assert torch.equal(out, ref)


# ------------------------------------------------------------ guard bands --

GUARD = 1024  # bytes of canary on each side (a multiple of 256: keeps alignment)
CANARY = {torch.int32: 0x7BADBEEF, torch.float32: 0x7FC0DEAD, torch.bfloat16: 0x7FA5,
          torch.uint8: 0xA5}
_BITS = {torch.int32: torch.int32, torch.float32: torch.int32, torch.bfloat16: torch.int16,
         torch.uint8: torch.uint8}


class Guarded:
    """A device buffer of `shape` between two GUARD-byte canary bands."""

    def __init__(self, shape, dtype, fill=None):
        es = torch.empty((), dtype=dtype).element_size()
        n = int(np.prod(shape)) if len(shape) else 1
        g = GUARD // es
        self.g, self.n, self.dtype = g, n, dtype
        self.full = torch.empty(n + 2 * g, dtype=dtype, device=DEV)
        pat = CANARY[dtype]
        bits = self.full.view(_BITS[dtype])
        if _BITS[dtype] == torch.int16 and pat >= 1 << 15:
            pat -= 1 << 16
        bits.fill_(pat)
        self.pat = pat
        self.t = self.full[g:g + n].view(shape)
        if fill is not None:
            self.t.copy_(fill)

    def intact(self):
        bits = self.full.view(_BITS[self.dtype])
        return bool((bits[:self.g] == self.pat).all()) and \
            bool((bits[self.g + self.n:] == self.pat).all())


def _guard_ws(nbytes):
    return Guarded((nbytes,), torch.uint8)


GUARD_SHAPES = [
    # (name, T, d, E, I, K, renorm, f, dtype)
    ("T3_E60", 3, 1024, 60, 256, 4, 0, 0.5, "bf16"),
    ("T37_E60", 37, 1024, 60, 256, 4, 1, 0.35, "bf16"),
    ("T600_E60", 600, 1024, 60, 256, 4, 0, 0.6, "bf16"),
    ("T37_qwen3", 37, 2048, 128, 768, 8, 1, 0.35, "bf16"),
    ("T16_qwen3_one_launch", 16, 2048, 128, 768, 8, 1, 0.35, "bf16"),
    ("T5_E60_one_launch", 5, 2048, 60, 1408, 4, 0, 0.35, "bf16"),
    ("T2100_qwen3_prefill_tiles", 2100, 2048, 128, 768, 8, 1, 0.35, "bf16"),
    ("T4100_qwen3_256row_tiles", 4100, 2048, 128, 768, 8, 1, 0.6, "bf16"),
    ("T37_tiny_f32", 37, 128, 8, 256, 2, 0, 0.5, "f32"),
]


@pytest.mark.parametrize("name,T,d,E,I,K,renorm,f,dt", GUARD_SHAPES,
                         ids=[s[0] for s in GUARD_SHAPES])
def test_guard_bands_route_forward_backward(name, T, d, E, I, K, renorm, f, dt):
    sh = inputs.Shape(d=d, E=E, K=K, I=I, renorm=renorm, dtype=dt)
    tdt = inputs.torch_dtype(sh)
    x, Wg, Wm, W1, W3, W2 = _layer(sh, T, f, seed=T)
    dsc = abi.desc(T, d, E, I, K, dt, renorm)
    bufs = []

    def G(shape, dtype, fill=None):
        b = Guarded(shape, dtype, fill)
        bufs.append(b)
        return b.t

    # inputs inside guards too: a stray write into an input would show
    xg, Wgg, Wmg = G(x.shape, tdt, x), G(Wg.shape, tdt, Wg), G(Wm.shape, tdt, Wm)
    W1g, W3g, W2g = G(W1.shape, tdt, W1), G(W3.shape, tdt, W3), G(W2.shape, tdt, W2)
    # route
    wsb = _guard_ws(abi.workspace_size(dsc))
    bufs.append(wsb)
    idx, w = G((T, K), torch.int32), G((T, K), torch.float32)
    cnt, hist = G((E,), torch.int32), G((K + 1,), torch.int32)
    lg = G((T, 2 * E), torch.float32)
    abi.route(dsc, xg, Wgg, Wmg, idx, w, cnt, hist, lg, wsb.t)
    abi.check(dsc, wsb.t)
    # forward
    out = G((T, d), tdt)
    abi.forward(dsc, xg, Wgg, Wmg, W1g, W3g, W2g, out, wsb.t)
    abi.check(dsc, wsb.t)
    assert torch.isfinite(out.float()).all()
    # forward with shared experts (bf16 only)
    if dt == "bf16":
        S = 2
        dss = abi.desc(T, d, E, I, K, dt, renorm, n_shared=S, I_shared=I)
        W1s, W3s, W2s = inputs.make_shared_experts(sh, S, seed=T, device=DEV)
        W1sg, W3sg, W2sg = G(W1s.shape, tdt, W1s), G(W3s.shape, tdt, W3s), G(W2s.shape, tdt, W2s)
        wss = _guard_ws(abi.workspace_size(dss))
        bufs.append(wss)
        out_s = G((T, d), tdt)
        abi.forward_shared(dss, xg, Wgg, Wmg, W1g, W3g, W2g, W1sg, W3sg, W2sg, out_s, wss.t)
        abi.check(dss, wss.t)
        assert torch.isfinite(out_s.float()).all()
    # backward
    dy = G((T, d), tdt, inputs.make_upstream_grad(sh, T, seed=T, device=DEV))
    wsbw = _guard_ws(abi.backward_workspace_size(dsc))
    bufs.append(wsbw)
    f32 = torch.float32
    dx = G((T, d), f32)
    dWg_, dWm_ = G((E, d), f32, torch.zeros(E, d)), G((E, d), f32, torch.zeros(E, d))
    dW1 = G((E, I, d), f32, torch.zeros(E, I, d))
    dW3 = G((E, I, d), f32, torch.zeros(E, I, d))
    dW2 = G((E, d, I), f32, torch.zeros(E, d, I))
    abi.backward(dsc, xg, Wgg, Wmg, W1g, W3g, W2g, dy, 0.01, dx, dWg_, dWm_, dW1, dW3, dW2,
                 wsbw.t)
    abi.check(dsc, wsbw.t)
    torch.cuda.synchronize()
    assert torch.isfinite(dx).all()
    bad = [i for i, b in enumerate(bufs) if not b.intact()]
    assert not bad, f"canaries overwritten around buffers {bad}"
    # the inputs themselves are unchanged
    for a, b in ((xg, x), (Wgg, Wg), (Wmg, Wm), (W1g, W1), (W3g, W3), (W2g, W2)):
        assert torch.equal(a, b)
