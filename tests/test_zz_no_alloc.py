"""beam_moe_route_noalloc: routing for callers that cannot allocate device
memory -- for example a plugin whose host runtime owns all of the device
memory and gives its extensions none.  Its scratch is a fixed array inside the
library instead of a caller workspace.  Checked against beam_moe_route (which
takes a workspace) on two calls in a row with different batches, so the second
call runs over the first call's leftover scratch contents.  Both run the same
kernels with the same split count and summation order, so every output must
agree bit for bit.  This file is collected last.
"""
import numpy as np
import pytest
import torch

from dynamic_expert_routing_router_b200 import abi, inputs

pytestmark = pytest.mark.gpu


def _outputs(T, E, K, dev):
    return (torch.empty((T, K), dtype=torch.int32, device=dev),
            torch.empty((T, K), dtype=torch.float32, device=dev),
            torch.empty((E,), dtype=torch.int32, device=dev),
            torch.empty((K + 1,), dtype=torch.int32, device=dev),
            torch.full((T, 2 * E), float("nan"), dtype=torch.float32, device=dev))


def test_route_noalloc_matches_route_on_two_calls():
    dev = "cuda"
    sh = inputs.QWEN3
    Wg = inputs.make_gate(sh, seed=0, device=dev)
    for T, f, seed in ((128, 0.15, 1), (37, 0.6, 2)):  # second call smaller, other data
        x = inputs.make_tokens(sh, T, seed=seed, device=dev)
        Wm = inputs.make_mask(sh, f, seed=0, device=dev)
        dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
        ref = _outputs(T, sh.E, sh.K, dev)
        ws = abi.alloc_workspace(dsc, dev)
        abi.route(dsc, x, Wg, Wm, *ref, workspace=ws)
        got = _outputs(T, sh.E, sh.K, dev)
        abi.route_noalloc(dsc, x, Wg, Wm, *got)
        abi.route_noalloc_check()  # synchronises; the array's error word is clean
        r = [t.cpu().numpy() for t in ref]
        g = [t.cpu().numpy() for t in got]
        for a, b in zip(g, r):  # idx, w, counts, hist, logits: bit for bit
            assert a.dtype == b.dtype and np.array_equal(a.view(np.int32), b.view(np.int32))
        assert g[3].sum() == T and (g[0] >= 0).sum() == g[2].sum()
        assert not np.isnan(g[4]).any()


def test_route_noalloc_reports_a_router_timeout_then_recovers():
    """A bounded router wait made to expire (the library's test switch) is
    reported by beam_moe_route_noalloc_check; the next call is clean."""
    dev = "cuda"
    sh = inputs.QWEN3
    T = 16
    Wg = inputs.make_gate(sh, seed=0, device=dev)
    Wm = inputs.make_mask(sh, 0.35, seed=0, device=dev)
    x = inputs.make_tokens(sh, T, seed=5, device=dev)
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    got = _outputs(T, sh.E, sh.K, dev)
    try:
        abi.set_fault_injection(abi.FAULT_ROUTER_STAGE, 50_000_000)
        abi.route_noalloc(dsc, x, Wg, Wm, *got)
        with pytest.raises(abi.BeamError) as ei:
            abi.route_noalloc_check()
        assert ei.value.status == 5  # BEAM_ERR_TIMEOUT
    finally:
        torch.cuda.synchronize()
        abi.set_fault_injection(abi.FAULT_NONE, 0)
    abi.route_noalloc(dsc, x, Wg, Wm, *got)
    abi.route_noalloc_check()
    ref = _outputs(T, sh.E, sh.K, dev)
    abi.route(dsc, x, Wg, Wm, *ref, workspace=abi.alloc_workspace(dsc, dev))
    torch.cuda.synchronize()
    for a, b in zip(got, ref):
        assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_route_noalloc_rejects_batches_beyond_its_array():
    dev = "cuda"
    sh = inputs.QWEN3
    T = 20000  # the router partials alone need ~20 MB > 16 MiB
    dsc = abi.desc(T, sh.d, sh.E, sh.I, sh.K, "bf16", sh.renorm)
    assert abi.plan(dsc)["off_idx"] > abi.NOALLOC_SCRATCH_BYTES
    small = torch.zeros(64, dtype=torch.float32, device=dev)  # never read: rejected first
    with pytest.raises(abi.BeamError) as ei:
        abi.route_noalloc(dsc, small, small, small, small, small, small, small, small)
    assert ei.value.status == 3  # BEAM_ERR_WORKSPACE
